// sf_attn_decode_refine: decode attention over 2-bit resident K/V with the
// most-attended tokens refined to their full 4-bit codes.
//
// StrataFlux picks KV refinements by the attention weight computed from the
// low-bit keys (rag-lover.com explainer, 解説).  The pass structure:
//
//   A  score   per (KV head, token): resident scores of the Hq/Hkv query
//              heads of the group from the 2-bit keys, fp32, into scratch, on
//              the integer tensor cores; also a per-head histogram of the
//              scores (top 10 bits of the order-preserving key) and max |s|.
//   S  select  per query head: the k largest scores, exactly.  The fast fp32
//              scores carry a proven error bound eps; every token within
//              2*eps of the k-th largest fast score is a candidate, and the
//              candidates are re-scored exactly in fp64 (the key s*E with
//              E = sum_d q_d (c_d 2^b_f + m_f - z) is exact in fp64 under a
//              precondition on q checked here) and ranked by (key desc, token
//              asc).  So the chosen set equals the exact definition.  Runs as
//              a compaction over token chunks (from the histogram's bin of
//              the k-th score) and a finish per KV group (one cluster, one CTA
//              per query head), which also forms the group's union (ascending
//              list and token bitmask) and the refined scores of its tokens.
//   B  output  split over tokens: softmax over all tokens with the refined
//              (full-code) K and V for tokens in the union and the resident
//              ones elsewhere -- refined tokens are computed directly, never
//              by subtracting their resident contribution.
//   M  merge   per KV group, by the last CTA of pass B to finish: combine the
//              splits' (max, sum, output).
//
// Every scratch array lives in the caller's workspace; nothing is allocated.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include <cooperative_groups.h>

#include "attn_common.cuh"

namespace {

// Loads the group's query heads as fp32 into qs[GRP][D] and their sums
// (sequential fp32 order, d ascending) into qsum[GRP].
template <int GRP>
__device__ void load_q(const uint16_t* __restrict__ q, int g, float (*qs)[D], float* qsum) {
  for (int e = threadIdx.x; e < GRP * D; e += blockDim.x)
    qs[e / D][e % D] = sfd::bf16_bits_to_float(q[static_cast<size_t>(g) * GRP * D + e]);
  __syncthreads();
  if (threadIdx.x < GRP) {
    float s = 0.0f;
    for (int d = 0; d < D; ++d) s += qs[threadIdx.x][d];
    qsum[threadIdx.x] = s;
  }
  __syncthreads();
}

// ---- pass A on the tensor cores: integer MMA over code bytes ----------------
//
// Per KV group, the query heads become exact-as-possible fixed point: per
// head X_d = rint(q_d 2^(23 - e)), e the binary exponent of max |q| (every
// bf16 within 15 binades of the maximum is exact), split into three byte
// planes.  mma.m16n8k32 (u8 codes x u8/s8 planes, s32 accumulate) gives
// sum_d c_d X_d per plane exactly; the reduction order inside an MMA does not
// matter, so a code word becomes a fragment register with one shift and one
// mask ((w >> 2 tig) & 0x03030303 holds dims tig, tig+4, tig+8, tig+12), and
// the q planes are laid out in the same permuted order.  A warp scores 16
// tokens per MMA row tile for all heads of the group at once (n = heads).

template <int GRP>
__global__ void __launch_bounds__(128)
attn_score_mma_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                      const uint16_t* __restrict__ k_scale, const uint16_t* __restrict__ k_zero, int T,
                      float* __restrict__ score, float* __restrict__ smax, int32_t* __restrict__ hist,
                      uint32_t* __restrict__ amaxu) {
  __shared__ int qx[GRP][D];
  __shared__ float qsc[GRP], qsm[GRP];
  // per-head histogram of this CTA's scores over the top 10 bits of the
  // order-preserving key (pass S starts from the cluster of all CTAs' counts)
  __shared__ int hs[GRP][kHistBins];
  for (int i = threadIdx.x; i < GRP * kHistBins; i += blockDim.x) (&hs[0][0])[i] = 0;
  const int g = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // fixed-point query heads (warp h builds head h, 4 dims per lane)
  for (int h = warp; h < GRP; h += 4) {
    float v[4];
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[i] = sfd::bf16_bits_to_float(q[(static_cast<size_t>(g) * GRP + h) * D + 4 * lane + i]);
      am = fmaxf(am, fabsf(v[i]));
    }
    am = warp_max(am);
    int e = 0;
    if (am > 0.0f) frexpf(am, &e);
#pragma unroll
    for (int i = 0; i < 4; ++i) qx[h][4 * lane + i] = __float2int_rn(ldexpf(v[i], 23 - e));
    if (lane == 0) qsc[h] = ldexpf(1.0f, e - 23);
  }
  if (tid < GRP) {
    float sum = 0.0f;
    for (int d = 0; d < D; ++d) sum += sfd::bf16_bits_to_float(q[(static_cast<size_t>(g) * GRP + tid) * D + d]);
    qsm[tid] = sum;
  }
  __syncthreads();
  const int g8 = lane >> 2, tig = lane & 3;
  // B fragments: column n = g8 is query head g8 (zero beyond the group)
  uint32_t bq[4][3][2];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
#pragma unroll
    for (int half = 0; half < 2; ++half)
#pragma unroll
      for (int p = 0; p < 3; ++p) {
        uint32_t v = 0;
        if (g8 < GRP) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            v |= ((static_cast<uint32_t>(qx[g8][16 * (2 * ks + half) + tig + 4 * i]) >> (8 * p)) & 0xFFu) << (8 * i);
        }
        bq[ks][p][half] = v;
      }
  const int ntiles = (T + 15) / 16;
  float smx = 0.0f;
  float am0 = 0.0f, am1 = 0.0f;  // max |score| of this lane's heads 2 tig, 2 tig + 1
  // one tile = rows ta, tb of this thread: 2 x 32 bytes of codes plus the
  // rows' scale and zero; the next tile is fetched while this one is scored
  struct TileRegs {
    uint32_t wa[8], wb[8];
    uint16_t sa, za, sb, zb;
  };
  auto load_tile = [&](int tile, TileRegs& r) {
    const int ta = tile * 16 + g8, tb = ta + 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) { r.wa[i] = 0u; r.wb[i] = 0u; }
    r.sa = r.za = r.sb = r.zb = 0;
    if (ta < T) {
      const size_t row = static_cast<size_t>(g) * T + ta;
      const uint4* p4 = reinterpret_cast<const uint4*>(k_res + row * kWordsPerRow);
      const uint4 x0 = p4[0], x1 = p4[1];
      r.wa[0] = x0.x; r.wa[1] = x0.y; r.wa[2] = x0.z; r.wa[3] = x0.w;
      r.wa[4] = x1.x; r.wa[5] = x1.y; r.wa[6] = x1.z; r.wa[7] = x1.w;
      r.sa = k_scale[row];
      r.za = k_zero[row];
    }
    if (tb < T) {
      const size_t row = static_cast<size_t>(g) * T + tb;
      const uint4* p4 = reinterpret_cast<const uint4*>(k_res + row * kWordsPerRow);
      const uint4 x0 = p4[0], x1 = p4[1];
      r.wb[0] = x0.x; r.wb[1] = x0.y; r.wb[2] = x0.z; r.wb[3] = x0.w;
      r.wb[4] = x1.x; r.wb[5] = x1.y; r.wb[6] = x1.z; r.wb[7] = x1.w;
      r.sb = k_scale[row];
      r.zb = k_zero[row];
    }
  };
  const int tstride = gridDim.x * 4;
  int tile = blockIdx.x * 4 + warp;
  TileRegs cur;
  if (tile < ntiles) load_tile(tile, cur);
  for (; tile < ntiles; tile += tstride) {
    TileRegs nxt;
    if (tile + tstride < ntiles) load_tile(tile + tstride, nxt);
    const int ta = tile * 16 + g8, tb = ta + 8;
    int d0[4] = {0, 0, 0, 0}, d1[4] = {0, 0, 0, 0}, d2[4] = {0, 0, 0, 0};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const uint32_t a0 = (cur.wa[2 * ks] >> (2 * tig)) & 0x03030303u;
      const uint32_t a1 = (cur.wb[2 * ks] >> (2 * tig)) & 0x03030303u;
      const uint32_t a2 = (cur.wa[2 * ks + 1] >> (2 * tig)) & 0x03030303u;
      const uint32_t a3 = (cur.wb[2 * ks + 1] >> (2 * tig)) & 0x03030303u;
      mma_u8u8(d0, a0, a1, a2, a3, bq[ks][0][0], bq[ks][0][1]);
      mma_u8u8(d1, a0, a1, a2, a3, bq[ks][1][0], bq[ks][1][1]);
      mma_u8s8(d2, a0, a1, a2, a3, bq[ks][2][0], bq[ks][2][1]);
    }
    // d[i]: i = 0,1 -> token ta, heads 2 tig, 2 tig + 1; i = 2,3 -> token tb
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int h = 2 * tig + (i & 1);
      const int t = (i < 2) ? ta : tb;
      if (h < GRP && t < T) {
        const float sv = sfd::half_bits_to_float(i < 2 ? cur.sa : cur.sb);
        const float zv = sfd::half_bits_to_float(i < 2 ? cur.za : cur.zb);
        smx = fmaxf(smx, sv);
        const float P = (static_cast<float>(d2[i]) * 65536.0f + static_cast<float>(d1[i]) * 256.0f +
                         static_cast<float>(d0[i])) * qsc[h];
        const float E = fmaf(4.0f, P, (1.5f - zv) * qsm[h]);
        const float val = (sv * E) * kInvSqrtD;
        score[(static_cast<size_t>(g) * GRP + h) * T + t] = val;
        atomicAdd(&hs[h][okey32(val) >> 22], 1);
        if (i & 1) am1 = fmaxf(am1, fabsf(val));
        else am0 = fmaxf(am0, fabsf(val));
      }
    }
    cur = nxt;
  }
  smx = warp_max(smx);
  if (lane == 0) atomicMax(reinterpret_cast<unsigned int*>(smax + g), __float_as_uint(smx));
  // max |score| per head: lanes with the same tig hold the same two heads
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    am0 = fmaxf(am0, __shfl_xor_sync(0xffffffffu, am0, o));
    am1 = fmaxf(am1, __shfl_xor_sync(0xffffffffu, am1, o));
  }
  if (g8 == 0) {
    if (2 * tig < GRP) atomicMax(amaxu + g * GRP + 2 * tig, __float_as_uint(am0));
    if (2 * tig + 1 < GRP) atomicMax(amaxu + g * GRP + 2 * tig + 1, __float_as_uint(am1));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < GRP * kHistBins; i += blockDim.x) {
    const int c = (&hs[0][0])[i];
    if (c) atomicAdd(hist + static_cast<size_t>(g) * GRP * kHistBins + i, c);
  }
}

// ---- pass S, selection from the score histogram -----------------------------
//
// Pass A left, per query head, a histogram of its fast scores over the top 10
// bits of the order-preserving key, and max |score|.  The bin b1 holding the
// k-th largest score follows from the histogram alone.  Every token whose
// exact key can reach the top k has a fast score >= tau - 2 eps >= (lower
// edge of b1) - 2 eps, so:
//  A  compact: per (4096-token chunk, head), the tokens with fast score >=
//     lower(b1) - 2 eps, in token order, into the chunk's slot of a list;
//  B  finish (one cluster per KV group, one CTA per query head): concatenate
//     the chunks, find tau exactly by two more radix passes over the listed
//     scores of bin b1, keep the candidates >= tau - 2 eps, re-key them
//     exactly in fp64 and rank them (key desc, token asc); then the group's
//     CTAs build the union of their selections (bitmask and ascending list)
//     through distributed shared memory and each computes its head's refined
//     scores for the union tokens.

// Per-head threshold of the compaction and the histogram bin: all threads call.
__device__ void select_band(const int32_t* __restrict__ hist_h, int k, double eps_s, int* hsh, int* scan_scratch,
                            int* binfo, uint32_t* b1, int* kk, float* f_low) {
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hsh[i] = hist_h[i];
  __syncthreads();
  find_bin_from_top_block(hsh, kHistBins, k, binfo, scan_scratch);
  *b1 = static_cast<uint32_t>(binfo[0]);
  *kk = binfo[1];
  const float lower = from_okey32(*b1 << 22);
  *f_low = __double2float_rd(static_cast<double>(lower) - 2.0 * eps_s);
}

constexpr int kCompThreads = 256;

template <int GRP>
__global__ void __launch_bounds__(kCompThreads)
attn_select_compact_kernel(const uint16_t* __restrict__ q, int T, int k, const float* __restrict__ score,
                           const float* __restrict__ smax, const int32_t* __restrict__ hist,
                           const uint32_t* __restrict__ amaxu, int32_t* __restrict__ cand, int nchunks,
                           int32_t* __restrict__ status) {
  const int chunk = blockIdx.x, h = blockIdx.y, g = h / GRP;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ int hsh[kHistBins];
  __shared__ int scan_scratch[64];
  __shared__ int binfo[2];
  __shared__ double qd[D];
  __shared__ double l1_sh;
  __shared__ int qe_sh;
  select_q_prologue(q, h, g, qd, &l1_sh, &qe_sh, status);
  const double eps_s = select_eps(static_cast<double>(smax[g]), l1_sh, qe_sh, __uint_as_float(amaxu[h]));
  uint32_t b1;
  int kk;
  float f_low;
  select_band(hist + static_cast<size_t>(h) * kHistBins, k, eps_s, hsh, scan_scratch, binfo, &b1, &kk, &f_low);
  // warp w: tokens [chunk*4096 + 512 w, +512) as 16 rows of 32
  constexpr int kRowsPerWarp = kChunk / (kCompThreads / 32) / 32;
  const int t0 = chunk * kChunk + warp * 32 * kRowsPerWarp + lane;
  const int tend = min(T, chunk * kChunk + (warp + 1) * 32 * kRowsPerWarp);
  const float* sc = score + static_cast<size_t>(h) * T;
  bool p[kRowsPerWarp];
  int cnt = 0;
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int t = t0 + 32 * i;
    p[i] = t < tend && sc[t] >= f_low;
    cnt += __popc(__ballot_sync(0xffffffffu, p[i]));
  }
  if (lane == 0) scan_scratch[warp] = cnt;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < kCompThreads / 32 ? scan_scratch[lane] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane < kCompThreads / 32) scan_scratch[32 + lane] = incl - v;
    // the chunks' counts follow the Hq x T lists
    if (lane == 31) cand[static_cast<size_t>(gridDim.y) * T + static_cast<size_t>(h) * nchunks + chunk] = incl;
  }
  __syncthreads();
  int32_t* out = cand + static_cast<size_t>(h) * T + static_cast<size_t>(chunk) * kChunk;
  int o = scan_scratch[32 + warp];
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const unsigned bal = __ballot_sync(0xffffffffu, p[i]);
    if (p[i]) out[o + __popc(bal & lt)] = t0 + 32 * i;
    o += __popc(bal);
  }
}

constexpr int kFinThreads = 512;
constexpr int kFinKeys = 2048;     // candidates ranked pairwise from shared memory
constexpr int kFinChunks = 4096;   // chunk prefix sums in shared memory (T <= 2^24)
constexpr int kFinList = 4096;     // listed (token, score) pairs cached in shared memory
constexpr size_t kFinDynSmem = static_cast<size_t>(kFinList) * 8 + static_cast<size_t>(kFinKeys) * 4;

template <int GRP>
__global__ void __launch_bounds__(kFinThreads)
attn_select_finish_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                          const uint32_t* __restrict__ k_ref, const uint16_t* __restrict__ k_scale,
                          const uint16_t* __restrict__ k_zero, int T, int k, float* __restrict__ score,
                          const float* __restrict__ smax, const int32_t* __restrict__ hist,
                          const uint32_t* __restrict__ amaxu, int32_t* __restrict__ cand, int nchunks,
                          int32_t* __restrict__ list, double* __restrict__ kap, int32_t* __restrict__ sel_head,
                          uint32_t* __restrict__ umask, int words_t, int32_t* __restrict__ sel_out,
                          int32_t* __restrict__ sel_n, int32_t* __restrict__ status) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = static_cast<int>(cl.block_rank());
  const int h = blockIdx.x, g = h / GRP;
  const int tid = threadIdx.x;
  __shared__ int hr[2048];
  __shared__ int cpre[kFinChunks];
  __shared__ unsigned long long keys[kFinKeys];  // order-preserving exact keys, sorted with the tokens
  __shared__ double qd[D];
  __shared__ int scan_scratch[64];
  __shared__ int binfo[2];
  __shared__ double l1_sh;
  __shared__ int qe_sh, span_sh;
  __shared__ int cnt_sh;  // read remotely
  __shared__ uint32_t qpl[3][8][4];  // byte planes of the fixed-point q, in code-extraction order
  __shared__ long long qxsum_sh;
  extern __shared__ int fin_dyn[];
  int* ltok = fin_dyn;                                      // [kFinList]
  float* lsc = reinterpret_cast<float*>(fin_dyn + kFinList);  // [kFinList]
  int* ktok = fin_dyn + 2 * kFinList;                       // [kFinKeys] tokens of the sorted keys
  const float* sc = score + static_cast<size_t>(h) * T;
  int32_t* L = list + static_cast<size_t>(h) * T;  // concatenated list, token order
  int32_t* F = cand + static_cast<size_t>(h) * T;  // candidates (reuses the chunk lists once L is built)
  double* kp = kap + static_cast<size_t>(h) * T;
  const int cap = GRP * k;

  select_q_prologue(q, h, g, qd, &l1_sh, &qe_sh, status, &span_sh);
  // q as 24-bit fixed point X = q 2^(23 - qe): exact for every nonzero q
  // within 15 binades of the largest (bf16 has 8 significant bits)
  const bool int_keys = span_sh <= 15;
  if (int_keys) {
    if (tid < 96) {
      const int p = tid / 32, wi = (tid / 4) & 7, kq = tid & 3;
      uint32_t v = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int X = static_cast<int>(ldexp(qd[16 * wi + kq + 4 * b], 23 - qe_sh));
        v |= ((static_cast<uint32_t>(X) >> (8 * p)) & 0xFFu) << (8 * b);
      }
      qpl[p][wi][kq] = v;
    }
    if (tid < 32) {
      long long sx = 0;
      for (int d = tid; d < D; d += 32) sx += static_cast<long long>(ldexp(qd[d], 23 - qe_sh));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sx += __shfl_xor_sync(0xffffffffu, sx, o);
      if (tid == 0) qxsum_sh = sx;
    }
  }
  const double eps_s = select_eps(static_cast<double>(smax[g]), l1_sh, qe_sh, __uint_as_float(amaxu[h]));
  uint32_t b1;
  int kk;
  float f_low;
  select_band(hist + static_cast<size_t>(h) * kHistBins, k, eps_s, hr, scan_scratch, binfo, &b1, &kk, &f_low);

  // 1. concatenate the chunk lists (token order); with their fast scores in
  //    shared memory when they fit
  const int32_t* counts = cand + static_cast<size_t>(gridDim.x) * T + static_cast<size_t>(h) * nchunks;
  int m = 0;
  for (int base = 0; base < nchunks; base += kFinThreads) {
    const int c = base + tid;
    const int v = c < nchunks ? counts[c] : 0;
    int tot;
    const int pre = sfd::block_exclusive_scan(v, scan_scratch, &tot);
    if (c < nchunks) cpre[c] = m + pre;
    m += tot;
  }
  __syncthreads();
  for (int e = tid; e < m; e += kFinThreads) {
    int lo = 0, hi = nchunks - 1;  // last chunk with cpre <= e
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cpre[mid] <= e) lo = mid;
      else hi = mid - 1;
    }
    const int t = cand[static_cast<size_t>(h) * T + static_cast<size_t>(lo) * kChunk + (e - cpre[lo])];
    if (m <= kFinList) {
      ltok[e] = t;
      lsc[e] = sc[t];
    } else {
      L[e] = t;
    }
  }
  __syncthreads();
  const bool cached = m <= kFinList;
  auto tok_of = [&](int e) { return cached ? ltok[e] : L[e]; };
  auto score_of = [&](int e) { return cached ? lsc[e] : sc[L[e]]; };

  // 2. tau: two radix passes (11 + 11 bits) over the listed scores of bin b1
  uint32_t pre = b1 << 22;
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? 11 : 0;
    for (int i = tid; i < 2048; i += kFinThreads) hr[i] = 0;
    __syncthreads();
    const uint32_t pmask = pass == 0 ? 0xFFC00000u : 0xFFFFF800u;
    for (int e = tid; e < m; e += kFinThreads) {
      const uint32_t key = okey32(score_of(e));
      if ((key & pmask) == pre) atomicAdd(&hr[(key >> shift) & 2047u], 1);
    }
    __syncthreads();
    find_bin_from_top_block(hr, 2048, kk, binfo, scan_scratch);
    pre |= static_cast<uint32_t>(binfo[0]) << shift;
    kk = binfo[1];
  }
  const float tau = from_okey32(pre);
  const float fthr = __double2float_ru(static_cast<double>(tau) - 2.0 * eps_s);

  // 3. a token whose fast score exceeds tau + 2 eps outranks, by exact key,
  //    every token with fast score <= tau, so fewer than k tokens can rank
  //    above it: it is selected outright.  Only the band [tau - 2 eps,
  //    tau + 2 eps] is re-keyed and ranked (its candidates in token order).
  int32_t* sel = sel_head + static_cast<size_t>(h) * k;
  uint32_t* um = umask + static_cast<size_t>(g) * words_t;
  const double hi_band = static_cast<double>(tau) + 2.0 * eps_s;
  int nA = 0, ncand = 0;
  for (int base = 0; base < m; base += kFinThreads) {
    const int e = base + tid;
    const float sv_e = e < m ? score_of(e) : 0.0f;
    const bool inA = e < m && static_cast<double>(sv_e) > hi_band;
    const bool inB = e < m && !inA && sv_e >= fthr;
    const int t = e < m ? tok_of(e) : 0;
    int totA, totB;
    const int posA = sfd::block_exclusive_scan(inA ? 1 : 0, scan_scratch, &totA);
    const int posB = sfd::block_exclusive_scan(inB ? 1 : 0, scan_scratch, &totB);
    if (inA && nA + posA < k) {  // fewer than k by the bound; guarded against corrupt scores
      sel[nA + posA] = t;
      atomicOr(um + (t >> 5), 1u << (t & 31));
    }
    if (inB) F[ncand + posB] = t;
    nA += totA;
    ncand += totB;
  }
  __syncthreads();
  const int kB = max(0, k - nA);  // winners still to pick from the band (>= 1 by the bound)


  // 4. exact keys (four partial sums: exact under the precondition, so the
  //    order does not change the key)
  for (int i = tid; i < ncand; i += kFinThreads) {
    const int t = F[i];
    const size_t row = static_cast<size_t>(g) * T + t;
    const uint4* w4 = reinterpret_cast<const uint4*>(k_res + row * kWordsPerRow);
    const uint4 x0 = w4[0], x1 = w4[1];
    const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    const double sv = static_cast<double>(sfd::half_bits_to_float(k_scale[row]));
    const double z = static_cast<double>(sfd::half_bits_to_float(k_zero[row]));
    double key;
    if (int_keys) {
      // sum_d c_d X_d exactly with byte-plane dot products; E = 4 sum c q +
      // (1.5 - z) sum q is exact in fp64, so one fma returns it exactly
      unsigned d0 = 0, d1 = 0;
      int d2 = 0;
#pragma unroll
      for (int wi = 0; wi < 8; ++wi)
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          const unsigned c = (w[wi] >> (2 * kq)) & 0x03030303u;
          d0 = __dp4a(c, qpl[0][wi][kq], d0);
          d1 = __dp4a(c, qpl[1][wi][kq], d1);
          d2 = __dp4a(static_cast<int>(c), static_cast<int>(qpl[2][wi][kq]), d2);
        }
      const long long P = static_cast<long long>(d0) + 256ll * d1 + 65536ll * d2;
      const double cq = ldexp(static_cast<double>(P), qe_sh - 23);
      const double qsum = ldexp(static_cast<double>(qxsum_sh), qe_sh - 23);
      key = sv * fma(1.5 - z, qsum, 4.0 * cq);
    } else {
      double E[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
      for (int wi = 0; wi < 8; ++wi) {
        const uint32_t word = w[wi];
#pragma unroll 1
        for (int jj = 0; jj < 4; ++jj)
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = 4 * jj + u;
            const double c = static_cast<double>((word >> (2 * j)) & 3u);
            E[u] = fma(qd[16 * wi + j], c * 4.0 + 1.5 - z, E[u]);
          }
      }
      key = sv * ((E[0] + E[1]) + (E[2] + E[3]));
    }
    kp[i] = key;
    if (ncand <= kFinKeys) {
      keys[i] = okey64(key);
      ktok[i] = t;
    }
  }
  __syncthreads();

  // 5. rank the band by (key desc, token asc); its kB winners go to
  //    sel_head after the outright ones, and into the group's token bitmask
  if (ncand <= kFinKeys) {
    // bitonic sort of (key desc, token asc) over a power-of-two size,
    // padding with entries that order last; the first k are the selection
    int n2 = 1;
    while (n2 < ncand) n2 <<= 1;
    for (int i = ncand + tid; i < n2; i += kFinThreads) {
      keys[i] = 0ull;
      ktok[i] = 0x7FFFFFFF;
    }
    __syncthreads();
    for (int size = 2; size <= n2; size <<= 1)
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < (n2 >> 1); i += kFinThreads) {
          const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
          const unsigned long long ka = keys[lo], kb = keys[hi];
          const int ta = ktok[lo], tb = ktok[hi];
          const bool a_first = ka > kb || (ka == kb && ta < tb);
          if (a_first == ((lo & size) != 0)) {
            keys[lo] = kb;
            keys[hi] = ka;
            ktok[lo] = tb;
            ktok[hi] = ta;
          }
        }
        __syncthreads();
      }
    for (int r = tid; r < kB; r += kFinThreads) {
      const int t = ktok[r];
      sel[nA + r] = t;
      atomicOr(um + (t >> 5), 1u << (t & 31));
    }
  } else {
    select_rank_radix(F, ncand, kp, kB, hr, scan_scratch, binfo, sel + nA);
    __syncthreads();
    for (int i = tid; i < kB; i += kFinThreads) {
      const int t = sel[nA + i];
      atomicOr(um + (t >> 5), 1u << (t & 31));
    }
  }
  __threadfence();
  cl.sync();  // 1: the group's bitmask is complete

  // 6. union, ascending: CTA r of the cluster compacts words [r wper, (r+1) wper)
  const int wper = (words_t + GRP - 1) / GRP;
  const int w0 = min(words_t, rank * wper), w1 = min(words_t, w0 + wper);
  {
    const int chunk = (w1 - w0 + kFinThreads - 1) / kFinThreads;
    const int a0 = min(w1, w0 + tid * chunk), a1 = min(w1, a0 + chunk);
    int c = 0;
    for (int w = a0; w < a1; ++w) c += __popc(um[w]);
    int tot;
    int pos = sfd::block_exclusive_scan(c, scan_scratch, &tot);
    if (tid == 0) cnt_sh = tot;
    cl.sync();  // 2: every CTA's count is published
    int off = 0, U = 0;
    for (int r = 0; r < GRP; ++r) {
      const int cr = *cl.map_shared_rank(&cnt_sh, r);
      if (r < rank) off += cr;
      U += cr;
    }
    int32_t* out = sel_out + static_cast<size_t>(g) * cap;
    pos += off;
    for (int w = a0; w < a1; ++w) {
      uint32_t bits = um[w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1u;
        out[pos++] = 32 * w + b;
      }
    }
    if (rank == 0 && tid == 0) sel_n[g] = status[g] ? -1 - U : U;
  }
  cl.sync();  // 3: no shared-memory access across CTAs after this
}

// ---- pass B on the tensor cores ------------------------------------------------
//
// o_h = sum_t p_{h,t} v_t / sum_t p_{h,t} with v_t = s_t (4 c_t + 1.5 - z_t):
// the code part 4 sum_t alpha_{h,t} c_t, alpha_{h,t} = p_{h,t} s_t, is a
// product of the code matrix (dims x tokens, MMA rows = dims) with the weights
// (tokens x columns) on mma.m16n8k16 (f16 in, f32 accumulate).  Each weight
// is split into an f16 high part and an f16 remainder (columns h and GRP + h),
// so the products keep ~22 bits.  Codes enter as the f16 values 1024 + c,
// exact, built for one dim and a pair of tokens with one shift, one byte
// permute and one mask; the 1024 sum(alpha) they add is removed at the end.
// The offset part sum_t alpha_{h,t} (1.5 - z_t) is a scalar per head.
// Refined tokens (in the union) add alpha (c_f - 1.5), their refinement codes,
// on the CUDA cores; their scores were already refined in the score buffer.
//
// A CTA owns a token range of one KV group and walks it in sub-chunks of
// kSub tokens: the sub-chunk's score maximum per head is found first, so every
// weight is computed once, by one thread, relative to a fixed maximum and
// stored in shared memory (no per-tile online rescaling); the warps then run
// the MMAs over their tiles of 16 tokens, the codes staged by cp.async.

constexpr int kSub = 2048;         // tokens per sub-chunk
constexpr int kOutThreads = 256;
constexpr int kOW = kOutThreads / 32;
constexpr int kRing = 4;           // cp.async stages per warp
constexpr int kUCap = 512;         // refined rows per sub-chunk staged in shared memory
constexpr int kPerThr = kSub / kOutThreads;  // tokens of a sub-chunk per thread in the weight pass

template <int GRP>
struct OutCfg {
  static constexpr int NC = 2 * GRP;           // weight columns: high parts of the heads, then remainders
  static constexpr int NT = NC <= 8 ? 1 : 2;   // MMA n-tiles of 8 columns
  static constexpr int kStr = kSub + 8;        // halves per weight row: conflict-free fragment loads
  static constexpr size_t alpha_bytes = static_cast<size_t>(NT) * 8 * kStr * 2;
  static constexpr size_t ring_bytes = static_cast<size_t>(kOW) * kRing * 16 * kWordsPerRow * 4;
  static constexpr size_t ulist_bytes = static_cast<size_t>(kSub) * 4;
  static constexpr size_t vref_bytes = static_cast<size_t>(kUCap) * kWordsPerRow * 4;
  static constexpr size_t smem = alpha_bytes + ring_bytes + ulist_bytes + vref_bytes;
  static_assert(alpha_bytes >= static_cast<size_t>(GRP) * kMaxSplits * 4, "merge factors must fit the weight tile");
  static_assert(alpha_bytes >= static_cast<size_t>(kOW) * GRP * D * 4, "per-warp output tiles must fit the weight tile");
};

template <int GRP>
__global__ void __launch_bounds__(kOutThreads)
attn_out_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                const uint32_t* __restrict__ k_ref, const uint16_t* __restrict__ k_scale,
                const uint16_t* __restrict__ k_zero, const uint32_t* __restrict__ v_res,
                const uint32_t* __restrict__ v_ref, const uint16_t* __restrict__ v_scale,
                const uint16_t* __restrict__ v_zero, int T, int tps, int words_t, int splits, float* __restrict__ score,
                const uint32_t* __restrict__ umask, float* __restrict__ part, int32_t* __restrict__ done,
                float* __restrict__ out) {
  using C = OutCfg<GRP>;
  constexpr int NT = C::NT, kStr = C::kStr;
  extern __shared__ __align__(16) unsigned char smem[];
  __half* as = reinterpret_cast<__half*>(smem);                                      // [NT*8][kStr]
  uint32_t* ring = reinterpret_cast<uint32_t*>(smem + C::alpha_bytes);               // [kOW][kRing][16][8]
  int* ulist = reinterpret_cast<int*>(smem + C::alpha_bytes + C::ring_bytes);  // [kSub]
  uint32_t* vrs = reinterpret_cast<uint32_t*>(smem + C::alpha_bytes + C::ring_bytes +
                                              C::ulist_bytes);  // [kUCap][8] refinement rows of listed tokens
  __shared__ float red[kOW][GRP];
  __shared__ float red2[kOW][3 * GRP];
  __shared__ float Msh[GRP], Fsh[GRP];
  __shared__ int ucount;
  __shared__ float qs[GRP][D];
  __shared__ float qsum[GRP];
  __shared__ int uscan[33];

  const int g = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g8 = lane >> 2, tig = lane & 3;
  const int t0s = split * tps, t1s = min(T, t0s + tps);
  const size_t rowg = static_cast<size_t>(g) * T;

  for (int e = tid; e < (NT * 8 - C::NC) * kStr; e += kOutThreads) as[C::NC * kStr + e] = __float2half_rn(0.0f);
  if (tid < GRP) Msh[tid] = -INFINITY;
  load_q<GRP>(q, g, qs, qsum);  // contains __syncthreads

  float lsum[GRP], csum[GRP], asum[GRP], uo[GRP][4];
  float acc[NT][8][4];
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    lsum[h] = csum[h] = asum[h] = 0.0f;
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) uo[h][dd] = 0.0f;
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int w = 0; w < 8; ++w)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[nt][w][c] = 0.0f;
  // head of each of this lane's accumulator columns (-1: padding column)
  int colh[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int n = nt * 8 + 2 * tig + c;
      colh[nt][c] = n < GRP ? n : (n < 2 * GRP ? n - GRP : -1);
    }

  for (int c0 = t0s; c0 < t1s; c0 += kSub) {
    const int n = min(t1s, c0 + kSub) - c0;
    const int ntile = (n + 15) >> 4;
    const int tpw = (ntile + kOW - 1) / kOW;
    const int tile0 = min(ntile, warp * tpw), tile1 = min(ntile, tile0 + tpw);
    auto issue = [&](int ti) {
      const int st = (ti - tile0) % kRing;
      const int tok = 16 * ti + (lane >> 1);
      if (tok < n)
        cp_async16_attn(ring + ((warp * kRing + st) * 16 + (lane >> 1)) * kWordsPerRow + (lane & 1) * 4,
                        v_res + (rowg + c0 + tok) * kWordsPerRow + (lane & 1) * 4);
    };
    // start the code stream while the weights are being computed
    for (int i = 0; i < kRing - 1; ++i) {
      if (tile0 + i < tile1) issue(tile0 + i);
      cp_async_commit_attn();
    }

    // 0. the sub-chunk's refined tokens (ascending) from the group's bitmask;
    //    their refinement rows are staged for step 4, and their scores are
    //    recomputed from the full 4-bit key codes into the score buffer (this
    //    CTA owns the token range)
    {
      const int nw = (n + 31) >> 5;  // c0 is a multiple of 32
      uint32_t wbits = 0;
      if (tid < nw) {
        wbits = umask[static_cast<size_t>(g) * words_t + (c0 >> 5) + tid];
        const int rem = n - 32 * tid;
        if (rem < 32) wbits &= (1u << rem) - 1u;
      }
      int tot;
      int pos = sfd::block_exclusive_scan(__popc(wbits), uscan, &tot);  // nw <= kSub / 32 <= blockDim
      while (wbits) {
        const int b = __ffs(wbits) - 1;
        wbits &= wbits - 1u;
        ulist[pos++] = 32 * tid + b;
      }
      if (tid == 0) ucount = tot;
      __syncthreads();
    }
    const int nu = ucount;
    for (int u = tid; u < min(nu, kUCap); u += kOutThreads) {
      const uint32_t* src = v_ref + (rowg + c0 + ulist[u]) * kWordsPerRow;
      cp_async16_attn(vrs + u * kWordsPerRow, src);
      cp_async16_attn(vrs + u * kWordsPerRow + 4, src + 4);
    }
    cp_async_commit_attn();
    // warp per token, lane = dims 4 lane .. 4 lane + 3; four tokens' loads in
    // flight at a time
    for (int u0 = warp; u0 < nu; u0 += 4 * kOW) {
      uint32_t wr[4], wf[4], sz[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int u = u0 + j * kOW;
        wr[j] = wf[j] = sz[j] = 0;
        if (u < nu) {
          const size_t row = rowg + c0 + ulist[u];
          wr[j] = k_res[row * kWordsPerRow + (lane >> 2)];
          wf[j] = k_ref[row * kWordsPerRow + (lane >> 2)];
          sz[j] = static_cast<uint32_t>(k_scale[row]) | (static_cast<uint32_t>(k_zero[row]) << 16);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int u = u0 + j * kOW;
        if (u >= nu) break;  // uniform over the warp
        const uint32_t r = wr[j] >> ((lane & 3) * 8), f = wf[j] >> ((lane & 3) * 8);
        float P[GRP];
#pragma unroll
        for (int h = 0; h < GRP; ++h) P[h] = 0.0f;
#pragma unroll
        for (int dd = 0; dd < 4; ++dd) {
          const float c = static_cast<float>(((r >> (2 * dd)) & 3u) * 4u + ((f >> (2 * dd)) & 3u));
#pragma unroll
          for (int h = 0; h < GRP; ++h) P[h] = fmaf(qs[h][4 * lane + dd], c, P[h]);
        }
        const float sv = sfd::half_bits_to_float(sz[j] & 0xFFFFu);
        const float z = sfd::half_bits_to_float(sz[j] >> 16);
        const int t = c0 + ulist[u];
#pragma unroll
        for (int h = 0; h < GRP; ++h) {
          const float Ph = warp_sum(P[h]);
          if (lane == 0) score[(static_cast<size_t>(g) * GRP + h) * T + t] = (sv * fmaf(-z, qsum[h], Ph)) * kInvSqrtD;
        }
      }
    }
    __syncthreads();

    // 1. the sub-chunk's maximum score per head; this thread's tokens'
    //    scale, zero and union bit are fetched meanwhile
    uint32_t svz[kPerThr];
    {
      float mx[GRP];
#pragma unroll
      for (int h = 0; h < GRP; ++h) mx[h] = -INFINITY;
#pragma unroll
      for (int j = 0; j < kPerThr; ++j) {
        const int i = tid + j * kOutThreads;
        svz[j] = 0;
        if (i < n) {
          const size_t row = rowg + c0 + i;
          svz[j] = static_cast<uint32_t>(v_scale[row]) | (static_cast<uint32_t>(v_zero[row]) << 16);
#pragma unroll
          for (int h = 0; h < GRP; ++h)
            mx[h] = fmaxf(mx[h], score[(static_cast<size_t>(g) * GRP + h) * T + c0 + i]);
        }
      }
#pragma unroll
      for (int h = 0; h < GRP; ++h) {
        const float m = warp_max(mx[h]);
        if (lane == 0) red[warp][h] = m;
      }
      __syncthreads();
      if (tid < GRP) {
        float m = -INFINITY;
        for (int w = 0; w < kOW; ++w) m = fmaxf(m, red[w][tid]);
        const float mo = Msh[tid], mn = fmaxf(mo, m);
        Fsh[tid] = mo == -INFINITY ? 0.0f : __expf(mo - mn);
        Msh[tid] = mn;
      }
      __syncthreads();
    }
    float M[GRP], F[GRP];
    bool rescale = false;
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      M[h] = Msh[h];
      F[h] = Fsh[h];
      rescale |= F[h] != 1.0f;
    }
    if (rescale && c0 != t0s) {  // uniform over the block
#pragma unroll
      for (int h = 0; h < GRP; ++h) {
        lsum[h] *= F[h];
        csum[h] *= F[h];
        asum[h] *= F[h];
#pragma unroll
        for (int dd = 0; dd < 4; ++dd) uo[h][dd] *= F[h];
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float f0 = 1.0f, f1 = 1.0f;
#pragma unroll
        for (int h = 0; h < GRP; ++h) {
          if (colh[nt][0] == h) f0 = F[h];
          if (colh[nt][1] == h) f1 = F[h];
        }
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          acc[nt][w][0] *= f0; acc[nt][w][1] *= f1;
          acc[nt][w][2] *= f0; acc[nt][w][3] *= f1;
        }
      }
    }

    // 2. weights into shared memory (zero past the end of the last tile) and sums
#pragma unroll
    for (int j = 0; j < kPerThr; ++j) {
      const int i = tid + j * kOutThreads;
      if (j * kOutThreads >= 16 * ntile) break;  // uniform over the block
      const bool valid = i < n;
      if (i < 16 * ntile) {
        if (valid) {
          const float sv = sfd::half_bits_to_float(svz[j] & 0xFFFFu);
          const float zv = sfd::half_bits_to_float(svz[j] >> 16);
#pragma unroll
          for (int h = 0; h < GRP; ++h) {
            const float p = __expf(score[(static_cast<size_t>(g) * GRP + h) * T + c0 + i] - M[h]);
            const float al = p * sv;
            const __half ahi = __float2half_rn(al);
            const __half alo = __float2half_rn(al - __half2float(ahi));
            as[h * kStr + i] = ahi;
            as[(GRP + h) * kStr + i] = alo;
            lsum[h] += p;
            csum[h] = fmaf(al, 1.5f - zv, csum[h]);
            asum[h] += __half2float(ahi) + __half2float(alo);
          }
        } else {
#pragma unroll
          for (int h = 0; h < 2 * GRP; ++h) as[h * kStr + i] = __float2half_rn(0.0f);
        }
      }
    }
    __syncthreads();

    // 3. MMAs over this warp's tiles
    for (int ti = tile0; ti < tile1; ++ti) {
      if (ti + kRing - 1 < tile1) issue(ti + kRing - 1);
      cp_async_commit_attn();
      cp_async_wait_attn<kRing - 1>();
      __syncwarp();
      const uint32_t* vr = ring + (warp * kRing + (ti - tile0) % kRing) * 16 * kWordsPerRow;
      uint32_t b0[NT], b1[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const __half* ar = as + (nt * 8 + g8) * kStr + 16 * ti + 2 * tig;
        b0[nt] = *reinterpret_cast<const uint32_t*>(ar);
        b1[nt] = *reinterpret_cast<const uint32_t*>(ar + 8);
      }
      const uint4* ra = reinterpret_cast<const uint4*>(vr + (2 * tig) * kWordsPerRow);
      const uint4* rb = reinterpret_cast<const uint4*>(vr + (2 * tig + 1) * kWordsPerRow);
      const uint4* rc = reinterpret_cast<const uint4*>(vr + (2 * tig + 8) * kWordsPerRow);
      const uint4* rd = reinterpret_cast<const uint4*>(vr + (2 * tig + 9) * kWordsPerRow);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const uint4 A4 = ra[half], B4 = rb[half], C4 = rc[half], D4 = rd[half];
        const uint32_t wa[4] = {A4.x, A4.y, A4.z, A4.w}, wb[4] = {B4.x, B4.y, B4.z, B4.w};
        const uint32_t wc[4] = {C4.x, C4.y, C4.z, C4.w}, wd[4] = {D4.x, D4.y, D4.z, D4.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int w = half * 4 + j;  // dims 16 w .. 16 w + 15
          const uint32_t xa = wa[j] >> (2 * g8), xb = wb[j] >> (2 * g8);
          const uint32_t xc = wc[j] >> (2 * g8), xd = wd[j] >> (2 * g8);
          const uint32_t a0 = (__byte_perm(xa, xb, 0x5410) & 0x00030003u) | 0x64006400u;  // dim g8
          const uint32_t a1 = (__byte_perm(xa, xb, 0x7632) & 0x00030003u) | 0x64006400u;  // dim g8 + 8
          const uint32_t a2 = (__byte_perm(xc, xd, 0x5410) & 0x00030003u) | 0x64006400u;
          const uint32_t a3 = (__byte_perm(xc, xd, 0x7632) & 0x00030003u) | 0x64006400u;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_f16f32(acc[nt][w], a0, a1, a2, a3, b0[nt], b1[nt]);
        }
      }
      __syncwarp();
    }
    cp_async_wait_attn<0>();
    __syncthreads();  // the staged refinement rows come from every thread

    // 4. refined tokens: alpha (c_f - 1.5), lane = dims 4 lane .. 4 lane + 3
    for (int u = warp; u < nu; u += kOW) {
      const int i = ulist[u];
      const uint32_t wrow = u < kUCap ? vrs[u * kWordsPerRow + (lane >> 2)]
                                      : v_ref[(rowg + c0 + i) * kWordsPerRow + (lane >> 2)];
      const uint32_t wf = wrow >> ((lane & 3) * 8);
#pragma unroll
      for (int h = 0; h < GRP; ++h) {
        const float al = __half2float(as[h * kStr + i]) + __half2float(as[(GRP + h) * kStr + i]);
#pragma unroll
        for (int dd = 0; dd < 4; ++dd)
          uo[h][dd] = fmaf(al, static_cast<float>((wf >> (2 * dd)) & 3u) - 1.5f, uo[h][dd]);
      }
    }
    __syncthreads();  // weights and the list are rewritten by the next sub-chunk
  }

  // this warp's output tile ww[head][dim] (in units of the code part: uo
  // enters divided by 2^b_f = 4) in the dead weight tile, written in three
  // phases whose stores within a warp never collide (high columns, then
  // remainder columns, then the refined corrections); summed over warps below
  __syncthreads();  // every warp is done with the weight tile
  float* ww = reinterpret_cast<float*>(smem) + warp * GRP * D;
#pragma unroll
  for (int ph = 0; ph < 2; ++ph) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int w = 0; w < 8; ++w)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int n = nt * 8 + 2 * tig + (c & 1);
          const int hh = colh[nt][c & 1];
          if (hh < 0 || (n < GRP) != (ph == 0)) continue;
          float* dst = &ww[hh * D + 16 * w + g8 + 8 * (c >> 1)];
          *dst = ph == 0 ? acc[nt][w][c] : *dst + acc[nt][w][c];
        }
    __syncwarp();
  }
#pragma unroll
  for (int h = 0; h < GRP; ++h)
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) ww[h * D + 4 * lane + dd] += 0.25f * uo[h][dd];
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    const float l = warp_sum(lsum[h]), cs = warp_sum(csum[h]), a = warp_sum(asum[h]);
    if (lane == 0) {
      red2[warp][h] = l;
      red2[warp][GRP + h] = cs;
      red2[warp][2 * GRP + h] = a;
    }
  }
  __syncthreads();
  float* pg = part + static_cast<size_t>(g) * GRP * splits * (D + 2);
  for (int e = tid; e < GRP * (D + 2); e += kOutThreads) {
    const int h = e / (D + 2), j = e % (D + 2);
    float v;
    if (j == 0) {
      v = Msh[h];
    } else {
      float L = 0.0f, Cs = 0.0f, A = 0.0f;
      for (int w = 0; w < kOW; ++w) {
        L += red2[w][h];
        Cs += red2[w][GRP + h];
        A += red2[w][2 * GRP + h];
      }
      // resident value s (2^b_f c + m_f - z): code part 4 (acc - 1024 A), offset part Cs
      float o = 0.0f;
      if (j >= 2)
        for (int w = 0; w < kOW; ++w) o += reinterpret_cast<const float*>(smem)[(w * GRP + h) * D + j - 2];
      v = j == 1 ? L : fmaf(4.0f, o, fmaf(-4096.0f, A, Cs));
    }
    pg[(static_cast<size_t>(h) * splits + split) * (D + 2) + j] = v;
  }

  // the last CTA of the group to finish merges the splits
  __shared__ int last;
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(done + g, 1) == splits - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  float (*fct)[kMaxSplits] = reinterpret_cast<float (*)[kMaxSplits]>(smem);  // the weight tile is dead
  __shared__ float Lh[GRP];
  for (int e = tid; e < GRP * splits; e += kOutThreads) fct[e / splits][e % splits] = __ldcg(pg + e * (D + 2));
  __syncthreads();
  for (int h = warp; h < GRP; h += kOW) {
    float Mx = -INFINITY;
    for (int sp = lane; sp < splits; sp += 32) Mx = fmaxf(Mx, fct[h][sp]);
    Mx = warp_max(Mx);
    float Ls = 0.0f;
    for (int sp = lane; sp < splits; sp += 32) {
      const float ms = fct[h][sp];
      const float f = ms == -INFINITY ? 0.0f : __expf(ms - Mx);
      Ls = fmaf(f, __ldcg(pg + (h * splits + sp) * (D + 2) + 1), Ls);
      fct[h][sp] = f;
    }
    Ls = warp_sum(Ls);
    if (lane == 0) Lh[h] = Ls;
  }
  __syncthreads();
  // two outputs per thread, eight splits' partials of each in flight at once
  for (int e0 = tid; e0 < GRP * D; e0 += 2 * kOutThreads) {
    const int e1 = e0 + kOutThreads;
    const bool has1 = e1 < GRP * D;
    const int h0 = e0 / D, h1 = has1 ? e1 / D : h0;
    const float* p0 = pg + static_cast<size_t>(h0) * splits * (D + 2) + 2 + e0 % D;
    const float* p1 = pg + static_cast<size_t>(h1) * splits * (D + 2) + 2 + (has1 ? e1 % D : e0 % D);
    float A0 = 0.0f, A1 = 0.0f;
    for (int sp = 0; sp < splits; sp += 16) {
      float v0[16], v1[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int q = sp + u;
        v0[u] = q < splits ? __ldcg(p0 + static_cast<size_t>(q) * (D + 2)) : 0.0f;
        v1[u] = (has1 && q < splits) ? __ldcg(p1 + static_cast<size_t>(q) * (D + 2)) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int q = sp + u;
        if (q < splits) {
          A0 = fmaf(fct[h0][q], v0[u], A0);
          A1 = fmaf(fct[h1][q], v1[u], A1);
        }
      }
    }
    out[(static_cast<size_t>(g) * GRP + h0) * D + e0 % D] = A0 / Lh[h0];
    if (has1) out[(static_cast<size_t>(g) * GRP + h1) * D + e1 % D] = A1 / Lh[h1];
  }
}

__global__ void fill_all_kernel(int T, int grp, int k, int words_t, uint32_t* umask, int32_t* sel_out,
                                int32_t* sel_n) {
  const int g = blockIdx.y;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x)
    sel_out[static_cast<size_t>(g) * grp * k + t] = t;
  for (int w = blockIdx.x * blockDim.x + threadIdx.x; w < words_t; w += gridDim.x * blockDim.x) {
    const int lo = w * 32;
    const int nb = min(32, T - lo);
    umask[static_cast<size_t>(g) * words_t + w] = nb == 32 ? 0xFFFFFFFFu : ((1u << nb) - 1u);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) sel_n[g] = T;
}

template <int GRP>
sf_status run(const uint16_t* q, int Hq, int Hkv, int T, const sf_qkv* kv, int k, int32_t* sel_out, int32_t* sel_n,
              float* out, char* ws, const Layout& L, cudaStream_t s) {
  float* score = reinterpret_cast<float*>(ws + L.score);
  int32_t* cand = reinterpret_cast<int32_t*>(ws + L.cand);
  int32_t* cand2 = reinterpret_cast<int32_t*>(ws + L.cand2);
  double* kap = reinterpret_cast<double*>(ws + L.kap);
  int32_t* sel_head = reinterpret_cast<int32_t*>(ws + L.sel);
  uint32_t* umask = reinterpret_cast<uint32_t*>(ws + L.umask);
  float* part = reinterpret_cast<float*>(ws + L.part);
  float* smax = reinterpret_cast<float*>(ws + L.smax);
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  int32_t* done = reinterpret_cast<int32_t*>(ws + L.count);
  const int grp = GRP;
  const int sms = sf::sm_count();

  SF_CHECK_CUDA(cudaMemsetAsync(ws + L.smax, 0, L.total - L.smax, s));
  const int ntiles = (T + 15) / 16;
  dim3 ga(std::max(1, std::min((ntiles + 3) / 4, (4 * sms + Hkv - 1) / Hkv)), Hkv);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + L.hist);
  uint32_t* amaxu = reinterpret_cast<uint32_t*>(ws + L.amax);
  attn_score_mma_kernel<GRP><<<ga, 128, 0, s>>>(q, kv->k_res, kv->k_scale, kv->k_zero, T, score, smax, hist, amaxu);
  sf_status st = sf::check_launch("attn_score_mma_kernel");
  if (st != SF_OK) return st;
  if (k > 0 && k < T) {
    attn_select_compact_kernel<GRP><<<dim3(L.nchunks, Hq), kCompThreads, 0, s>>>(q, T, k, score, smax, hist, amaxu,
                                                                                cand, L.nchunks, status);
    st = sf::check_launch("attn_select_compact_kernel");
    if (st != SF_OK) return st;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(Hq));
    cfg.blockDim = dim3(kFinThreads);
    cfg.dynamicSmemBytes = kFinDynSmem;
    SF_CHECK_CUDA(cudaFuncSetAttribute(attn_select_finish_kernel<GRP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kFinDynSmem)));
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = GRP;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    SF_CHECK_CUDA(cudaLaunchKernelEx(&cfg, attn_select_finish_kernel<GRP>, q, kv->k_res, kv->k_ref, kv->k_scale,
                                     kv->k_zero, T, k, score, static_cast<const float*>(smax),
                                     static_cast<const int32_t*>(hist), static_cast<const uint32_t*>(amaxu), cand,
                                     L.nchunks, cand2, kap, sel_head, umask, L.words_t, sel_out, sel_n, status));
    st = sf::check_launch("attn_select_finish_kernel");
    if (st != SF_OK) return st;
  } else if (k == 0) {  // the token bitmask was cleared with the workspace
    SF_CHECK_CUDA(cudaMemsetAsync(sel_n, 0, sizeof(int32_t) * Hkv, s));
  } else {
    fill_all_kernel<<<dim3(32, Hkv), 256, 0, s>>>(T, grp, k, L.words_t, umask, sel_out, sel_n);
    st = sf::check_launch("fill_all_kernel");
    if (st != SF_OK) return st;
  }
  dim3 gb(L.splits, Hkv);
  SF_CHECK_CUDA(cudaFuncSetAttribute(attn_out_kernel<GRP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(OutCfg<GRP>::smem)));
  attn_out_kernel<GRP><<<gb, kOutThreads, OutCfg<GRP>::smem, s>>>(q, kv->k_res, kv->k_ref, kv->k_scale, kv->k_zero,
                                                                 kv->v_res, kv->v_ref, kv->v_scale, kv->v_zero, T,
                                                                 L.tps, L.words_t, L.splits, score, umask, part,
                                                                 done, out);
  return sf::check_launch("attn_out_kernel");
}

std::atomic<int> g_attn_path{SF_ATTN_AUTO};

// The cluster kernel where it applies (and is allowed), else the pipeline.
sf_status dispatch(const uint16_t* q, int Hq, int Hkv, int T, const sf_qkv* kv, int k, int32_t* sel_out,
                   int32_t* sel_n, float* out, char* ws, const Layout& L, cudaStream_t s) {
  const int path = g_attn_path.load(std::memory_order_relaxed);
  if (path != SF_ATTN_PIPELINE) {
    if (sf::attn_fused_eligible(Hq, Hkv, T))
      return sf::attn_fused_run(q, Hq, Hkv, T, kv, k, sel_out, sel_n, out, reinterpret_cast<double*>(ws + L.kap),
                                reinterpret_cast<int32_t*>(ws + L.cand), reinterpret_cast<int32_t*>(ws + L.sel),
                                reinterpret_cast<float*>(ws + L.part), reinterpret_cast<int32_t*>(ws + L.fcnt), s);
    if (path == SF_ATTN_CLUSTER)
      return sf::fail(SF_ENOTIMPL, "sf_attn_decode_refine: the cluster kernel does not apply to these sizes");
  }
  switch (Hq / Hkv) {
    case 1: return run<1>(q, Hq, Hkv, T, kv, k, sel_out, sel_n, out, ws, L, s);
    case 2: return run<2>(q, Hq, Hkv, T, kv, k, sel_out, sel_n, out, ws, L, s);
    case 4: return run<4>(q, Hq, Hkv, T, kv, k, sel_out, sel_n, out, ws, L, s);
    case 8: return run<8>(q, Hq, Hkv, T, kv, k, sel_out, sel_n, out, ws, L, s);
    default: return sf::fail(SF_ENOTIMPL, "sf_attn_decode_refine: Hq/Hkv must be 1, 2, 4 or 8");
  }
}

}  // namespace

extern "C" sf_status sf_attn_set_path(int path) {
  SF_REQUIRE(path == SF_ATTN_AUTO || path == SF_ATTN_CLUSTER || path == SF_ATTN_PIPELINE,
             "sf_attn_set_path: unknown path %d", path);
  g_attn_path.store(path, std::memory_order_relaxed);
  return SF_OK;
}

extern "C" sf_status sf_attn_workspace_size(int Hq, int Hkv, int d, int T, int k_tokens, size_t* bytes) {
  SF_REQUIRE(bytes, "sf_attn_workspace_size: null pointer");
  SF_REQUIRE(d == D, "sf_attn_workspace_size: head dim must be %d", D);
  SF_REQUIRE(Hkv >= 1 && Hq >= Hkv && Hq % Hkv == 0 && Hq / Hkv <= kMaxGrp, "sf_attn_workspace_size: bad head counts");
  SF_REQUIRE(T >= 1 && k_tokens >= 0 && k_tokens <= T, "sf_attn_workspace_size: bad T / k_tokens");
  *bytes = make_layout(Hq, Hkv, T, k_tokens, sf::sm_count()).total;
  return SF_OK;
}

extern "C" sf_status sf_attn_decode_refine(const uint16_t* q, int Hq, int Hkv, int d, int T, const sf_qkv* kv,
                                           int k_tokens, int32_t* sel_out, int32_t* sel_n, float* out,
                                           void* workspace, size_t ws_bytes, sf_stream_t stream) {
  SF_REQUIRE(q && kv && sel_out && sel_n && out && workspace, "sf_attn_decode_refine: null pointer");
  SF_REQUIRE(kv->k_res && kv->k_ref && kv->v_res && kv->v_ref && kv->k_scale && kv->k_zero && kv->v_scale &&
                 kv->v_zero,
             "sf_attn_decode_refine: null K/V view");
  SF_REQUIRE(kv->b_r == 2 && kv->b_f == 2, "sf_attn_decode_refine: only 2-bit resident + 2-bit refinement K/V");
  SF_REQUIRE(d == D, "sf_attn_decode_refine: head dim must be %d", D);
  SF_REQUIRE(Hkv >= 1 && Hq >= Hkv && Hq % Hkv == 0, "sf_attn_decode_refine: Hq must be a multiple of Hkv");
  SF_REQUIRE(T >= 1 && T <= (1 << 24), "sf_attn_decode_refine: T out of range");
  SF_REQUIRE(k_tokens >= 0 && k_tokens <= T, "sf_attn_decode_refine: k_tokens must be in [0, T]");
  SF_REQUIRE(sf::aligned(kv->k_res, 16) && sf::aligned(kv->v_res, 16) && sf::aligned(kv->k_ref, 16) &&
                 sf::aligned(kv->v_ref, 16),
             "sf_attn_decode_refine: code arrays must be 16-byte aligned");
  SF_REQUIRE(sf::aligned(workspace, 256), "sf_attn_decode_refine: workspace must be 256-byte aligned");
  const Layout L = make_layout(Hq, Hkv, T, k_tokens, sf::sm_count());
  SF_REQUIRE(ws_bytes >= L.total, "sf_attn_decode_refine: workspace too small (%zu < %zu)", ws_bytes, L.total);
  SF_REQUIRE(Hq / Hkv <= kMaxGrp && (Hq / Hkv & (Hq / Hkv - 1)) == 0,
             "sf_attn_decode_refine: Hq/Hkv must be 1, 2, 4 or 8");
  return dispatch(q, Hq, Hkv, T, kv, k_tokens, sel_out, sel_n, out, static_cast<char*>(workspace), L,
                  sf::as_cuda(stream));
}

// ---- refined attention without any device allocation ------------------------
//
// Some callers cannot allocate device memory at the point where they run
// attention: a serving runtime that owns a fixed memory pool and forbids
// allocations after start-up, a plugin inside a host framework that hands out
// no scratch, or code running where cudaMalloc would synchronize the device
// or is not permitted.  For them this variant takes its scratch from one
// array compiled into the library instead of from a caller workspace.
//
// The array is a file-scope __device__ symbol: every GPU that loads the
// library reserves it (kStaticScratchBytes) for the life of the process.  In
// host code its name is only a host-side stand-in, so the device address is
// looked up with cudaGetSymbolAddress, once per device, with that device
// current, on the first call made on that device.  All calls share the array;
// the per-call counters it holds are cleared at the start of every call, and
// calls whose work overlaps on the GPU (different streams, no ordering) race
// on it.
namespace {

constexpr size_t kStaticScratchBytes = size_t{24} << 20;  // 24 MiB
__device__ __align__(256) unsigned char g_attn_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

sf_status static_scratch_address(void** out) {
  int dev = 0;
  SF_CHECK_CUDA(cudaGetDevice(&dev));
  SF_REQUIRE(dev >= 0 && dev < kMaxDevices, "sf_attn_decode_refine_noalloc: device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess) return sf::cuda_fail(e, "cudaGetSymbolAddress(attention scratch)");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SF_OK;
}

}  // namespace

extern "C" sf_status sf_attn_decode_refine_noalloc(const uint16_t* q, int Hq, int Hkv, int d, int T,
                                                   const sf_qkv* kv, int k_tokens, int32_t* sel_out, int32_t* sel_n,
                                                   float* out, sf_stream_t stream) {
  SF_REQUIRE(q && kv && sel_out && sel_n && out, "sf_attn_decode_refine_noalloc: null pointer");
  SF_REQUIRE(kv->k_res && kv->k_ref && kv->v_res && kv->v_ref && kv->k_scale && kv->k_zero && kv->v_scale &&
                 kv->v_zero,
             "sf_attn_decode_refine_noalloc: null K/V view");
  SF_REQUIRE(kv->b_r == 2 && kv->b_f == 2, "sf_attn_decode_refine_noalloc: only 2-bit resident + 2-bit refinement K/V");
  SF_REQUIRE(d == D, "sf_attn_decode_refine_noalloc: head dim must be %d", D);
  SF_REQUIRE(Hkv >= 1 && Hq >= Hkv && Hq % Hkv == 0, "sf_attn_decode_refine_noalloc: Hq must be a multiple of Hkv");
  SF_REQUIRE(T >= 1 && T <= (1 << 24), "sf_attn_decode_refine_noalloc: T out of range");
  SF_REQUIRE(k_tokens >= 0 && k_tokens <= T, "sf_attn_decode_refine_noalloc: k_tokens must be in [0, T]");
  SF_REQUIRE(sf::aligned(kv->k_res, 16) && sf::aligned(kv->v_res, 16) && sf::aligned(kv->k_ref, 16) &&
                 sf::aligned(kv->v_ref, 16),
             "sf_attn_decode_refine_noalloc: code arrays must be 16-byte aligned");
  const Layout L = make_layout(Hq, Hkv, T, k_tokens, sf::sm_count());
  SF_REQUIRE(L.total <= kStaticScratchBytes,
             "sf_attn_decode_refine_noalloc: these sizes need %zu bytes of scratch but the built-in array holds %zu; "
             "use sf_attn_decode_refine with a caller workspace",
             L.total, kStaticScratchBytes);
  void* ws = nullptr;
  const sf_status st = static_scratch_address(&ws);
  if (st != SF_OK) return st;
  SF_REQUIRE(Hq / Hkv <= kMaxGrp && (Hq / Hkv & (Hq / Hkv - 1)) == 0,
             "sf_attn_decode_refine_noalloc: Hq/Hkv must be 1, 2, 4 or 8");
  return dispatch(q, Hq, Hkv, T, kv, k_tokens, sel_out, sel_n, out, static_cast<char*>(ws), L, sf::as_cuda(stream));
}
