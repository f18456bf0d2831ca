// sf_attn_decode_refine: decode attention over 2-bit resident K/V with the
// most-attended tokens refined to their full 4-bit codes.
//
// StrataFlux picks KV refinements by the attention weight computed from the
// low-bit keys (rag-lover.com explainer, 解説).  The pass structure:
//
//   A  score   per (KV head, token): resident scores of the Hq/Hkv query
//              heads of the group from the 2-bit keys, fp32, into scratch, on
//              the integer tensor cores; also a per-head histogram of the
//              scores (top 11 bits of the order-preserving key), max |s| and
//              max s.
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
//              list and token bitmask).
//   R  refine  per union token: its scores from the full 4-bit key codes,
//              in place in the score buffer, and the largest per head.
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
// Per KV group, the query heads become fixed point: per head
// X_d = rint(q_d 2^(14 - e)), e the binary exponent of max |q| (|X| <= 2^14;
// the rounding, |dq| <= 2^(e - 15), is inside the band's error bound eps),
// split into two signed byte planes X = d0 + 256 d1.  mma.m16n8k32 (u8 codes
// x s8 planes, s32 accumulate) gives sum_d c_d X_d per plane exactly; the
// reduction order inside an MMA does not matter, so a code word becomes a
// fragment register with one shift and one mask ((w >> 2 tig) & 0x03030303
// holds dims tig, tig+4, tig+8, tig+12), and the q planes are laid out in the
// same permuted order.  MMA column 2 h + p is (head h, plane p), so one MMA
// per 32 dims covers four heads and lane tig ends with both planes of head
// tig for its two tokens: a warp scores 16 tokens of four heads per four
// MMAs (two n-tiles for eight heads per group).

// A CTA owns a contiguous token range of one group; each warp streams its run
// of 16-token tiles through its own ring of kScRing cp.async stages (seven
// tiles in flight while one is scored), and the range's key scales and zeros
// are staged in shared memory at the start.

constexpr int kScThreads = 256;
constexpr int kScQFrac = 14;      // fraction bits of the fixed-point q (relative to 2^e)
constexpr int kScW = kScThreads / 32;
constexpr int kScRing = 8;        // cp.async stages per warp, one 16-token tile each
constexpr int kScMaxTok = 4096;   // tokens per CTA at most
static_assert(kScMaxTok % kScThreads == 0, "the key scales are staged in whole rounds");

__host__ __device__ constexpr size_t score_smem(int grp) {
  return static_cast<size_t>(kScW) * kScRing * 16 * kWordsPerRow * 4 + static_cast<size_t>(kScMaxTok) * 4 +
         static_cast<size_t>(grp) * kHistBins * 4;
}

template <int GRP>
__global__ void __launch_bounds__(kScThreads, 2)
attn_score_mma_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                      const uint16_t* __restrict__ k_scale, const uint16_t* __restrict__ k_zero, int T, int S, int tpc,
                      float* __restrict__ score, float* __restrict__ smax, int32_t* __restrict__ hist,
                      uint32_t* __restrict__ amaxu, uint32_t* __restrict__ mkey) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* ring = reinterpret_cast<uint32_t*>(smem);               // [kScW][kScRing][16][8]
  uint32_t* ksz = ring + kScW * kScRing * 16 * kWordsPerRow;         // [tpc] key scale | zero << 16
  int* hs = reinterpret_cast<int*>(ksz + kScMaxTok);                 // [GRP][kHistBins]
  __shared__ int qx[GRP][D];
  __shared__ float qsc[GRP], qsm[GRP];
  __shared__ uint32_t bfr[4 * ((2 * GRP + 7) / 8) * 2][32];  // B fragments of qx, per lane
  const int g = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g8 = lane >> 2, tig = lane & 3;
  const int t0 = blockIdx.x * tpc;
  const int n = max(0, min(tpc, T - t0));
  const int ntile = (n + 15) >> 4;
  const int tpw = (ntile + kScW - 1) / kScW;
  const int tile0 = min(ntile, warp * tpw), tile1 = min(ntile, tile0 + tpw);
  const size_t row0 = static_cast<size_t>(g) * S + t0;  // K rows: the cache's stride
  auto issue = [&](int ti) {
    const int st = (ti - tile0) % kScRing;
    const int row = 16 * ti + (lane >> 1);
    if (row < n)
      cp_async16_attn(ring + ((warp * kScRing + st) * 16 + (lane >> 1)) * kWordsPerRow + (lane & 1) * 4,
                      k_res + (row0 + row) * kWordsPerRow + (lane & 1) * 4);
  };
  for (int i = 0; i < kScRing - 1; ++i) {
    if (tile0 + i < tile1) issue(tile0 + i);
    cp_async_commit_attn();
  }
  // per-head histogram of this CTA's scores over the top 11 bits of the
  // order-preserving key (pass S starts from the sum over all CTAs)
  for (int i = tid; i < GRP * kHistBins; i += kScThreads) hs[i] = 0;
  // the range's key scales and zeros: every load of this thread is issued
  // before the first store
  float smx = 0.0f, szx = 0.0f;
  {
    constexpr int kPer = kScMaxTok / kScThreads;
    uint32_t kzv[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = tid + j * kScThreads;
      kzv[j] = i < n ? static_cast<uint32_t>(k_scale[row0 + i]) | (static_cast<uint32_t>(k_zero[row0 + i]) << 16) : 0u;
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = tid + j * kScThreads;
      if (i < n) {
        ksz[i] = kzv[j];
        const float sv = sfd::half_bits_to_float(static_cast<uint16_t>(kzv[j] & 0xFFFFu));
        const float zv = sfd::half_bits_to_float(static_cast<uint16_t>(kzv[j] >> 16));
        smx = fmaxf(smx, sv);
        szx = fmaxf(szx, __double2float_ru(static_cast<double>(sv) * fabs(1.5 - static_cast<double>(zv))));
      }
    }
  }
  // fixed-point query heads (warp h builds head h, 4 dims per lane) and the
  // sums of q: exact in fp64 (the bf16 exponents span at most 33 binades
  // where the result is used), then one rounding to fp32
  for (int h = warp; h < GRP; h += kScW) {
    float v[4];
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[i] = sfd::bf16_bits_to_float(q[(static_cast<size_t>(g) * GRP + h) * D + 4 * lane + i]);
      am = fmaxf(am, fabsf(v[i]));
    }
    am = warp_max(am);
    double qs_d = (static_cast<double>(v[0]) + v[1]) + (static_cast<double>(v[2]) + v[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qs_d += __shfl_xor_sync(0xffffffffu, qs_d, o);
    const float qs_l = static_cast<float>(qs_d);
    int e = 0;
    if (am > 0.0f) frexpf(am, &e);
#pragma unroll
    for (int i = 0; i < 4; ++i) qx[h][4 * lane + i] = __float2int_rn(ldexpf(v[i], kScQFrac - e));
    if (lane == 0) {
      qsc[h] = ldexpf(1.0f, e - kScQFrac);
      qsm[h] = qs_l;
    }
  }
  __syncthreads();
  // B fragments, built once per CTA: word [ks][nt][half][lane]; column
  // n = lane / 4 of n-tile nt is (head (8 nt + n) / 2, plane n % 2), zero
  // beyond the group
  constexpr int NT = (2 * GRP + 7) / 8;
  for (int e = tid; e < 4 * NT * 2 * 32; e += kScThreads) {
    const int ln = e & 31, f = e >> 5, half = f & 1, nt = (f >> 1) % NT, ks = (f >> 1) / NT;
    const int col = 8 * nt + (ln >> 2), hh = col >> 1, pl = col & 1, tt = ln & 3;
    uint32_t v = 0;
    if (hh < GRP) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int X = qx[hh][16 * (2 * ks + half) + tt + 4 * i];
        const int d0 = ((X + 128) & 255) - 128;
        const int dv = pl == 0 ? d0 : (X - d0) >> 8;
        v |= (static_cast<uint32_t>(dv) & 0xFFu) << (8 * i);
      }
    }
    bfr[f][ln] = v;
  }
  __syncthreads();
  uint32_t bq[4][NT][2];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int half = 0; half < 2; ++half) bq[ks][nt][half] = bfr[(ks * NT + nt) * 2 + half][lane];
  // this lane's head of each n-tile (4 nt + tig): max |score| and the largest
  // score key
  float qscv[NT], qsmv[NT], am[NT];
  uint32_t km[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int h = 4 * nt + tig;
    qscv[nt] = h < GRP ? qsc[h] : 0.0f;
    qsmv[nt] = h < GRP ? qsm[h] : 0.0f;
    am[nt] = 0.0f;
    km[nt] = 0u;
  }
  for (int ti = tile0; ti < tile1; ++ti) {
    if (ti + kScRing - 1 < tile1) issue(ti + kScRing - 1);
    cp_async_commit_attn();
    cp_async_wait_attn<kScRing - 1>();
    __syncwarp();
    const uint32_t* kr = ring + (warp * kScRing + (ti - tile0) % kScRing) * 16 * kWordsPerRow;
    uint32_t wa[8], wb[8];
    {
      const uint4* pa = reinterpret_cast<const uint4*>(kr + g8 * kWordsPerRow);
      const uint4* pb = reinterpret_cast<const uint4*>(kr + (g8 + 8) * kWordsPerRow);
      const uint4 xa0 = pa[0], xa1 = pa[1], xb0 = pb[0], xb1 = pb[1];
      wa[0] = xa0.x; wa[1] = xa0.y; wa[2] = xa0.z; wa[3] = xa0.w;
      wa[4] = xa1.x; wa[5] = xa1.y; wa[6] = xa1.z; wa[7] = xa1.w;
      wb[0] = xb0.x; wb[1] = xb0.y; wb[2] = xb0.z; wb[3] = xb0.w;
      wb[4] = xb1.x; wb[5] = xb1.y; wb[6] = xb1.z; wb[7] = xb1.w;
    }
    __syncwarp();  // the stage is refilled by a later issue
    int d[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const uint32_t a0 = (wa[2 * ks] >> (2 * tig)) & 0x03030303u;
      const uint32_t a1 = (wb[2 * ks] >> (2 * tig)) & 0x03030303u;
      const uint32_t a2 = (wa[2 * ks + 1] >> (2 * tig)) & 0x03030303u;
      const uint32_t a3 = (wb[2 * ks + 1] >> (2 * tig)) & 0x03030303u;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_u8s8(d[nt], a0, a1, a2, a3, bq[ks][nt][0], bq[ks][nt][1]);
    }
    // d[nt][0], [1]: token ta, planes 0 and 1 of head 4 nt + tig; [2], [3]: token tb
    const int ta = 16 * ti + g8, tb = ta + 8;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h = 4 * nt + tig;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int tl = i ? tb : ta;
        if (h < GRP && tl < n) {
          const uint32_t kz = ksz[tl];
          const float sv = sfd::half_bits_to_float(static_cast<uint16_t>(kz & 0xFFFFu));
          const float zv = sfd::half_bits_to_float(static_cast<uint16_t>(kz >> 16));
          // sum_d c_d X_d is below 3 * 128 * 2^14 < 2^23: exact in fp32
          const float P = static_cast<float>(d[nt][2 * i] + 256 * d[nt][2 * i + 1]) * qscv[nt];
          const float E = fmaf(4.0f, P, (1.5f - zv) * qsmv[nt]);
          const float val = (sv * E) * kInvSqrtD;
          score[(static_cast<size_t>(g) * GRP + h) * T + t0 + tl] = val;
          atomicAdd(&hs[h * kHistBins + (okey32(val) >> kHistShift)], 1);
          am[nt] = fmaxf(am[nt], fabsf(val));
          km[nt] = max(km[nt], okey32(val));
        }
      }
    }
  }
  cp_async_wait_attn<0>();
  smx = warp_max(smx);
  szx = warp_max(szx);
  if (lane == 0) {
    atomicMax(reinterpret_cast<unsigned int*>(smax + g), __float_as_uint(smx));
    atomicMax(reinterpret_cast<unsigned int*>(smax + gridDim.y + g), __float_as_uint(szx));
  }
  // lanes with the same tig hold the same heads
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      am[nt] = fmaxf(am[nt], __shfl_xor_sync(0xffffffffu, am[nt], o));
      km[nt] = max(km[nt], __shfl_xor_sync(0xffffffffu, km[nt], o));
    }
    const int h = 4 * nt + tig;
    if (g8 == 0 && h < GRP) {
      atomicMax(amaxu + g * GRP + h, __float_as_uint(am[nt]));
      atomicMax(mkey + g * GRP + h, km[nt]);
    }
  }
  __syncthreads();
  for (int i = tid; i < GRP * kHistBins; i += kScThreads) {
    const int c = hs[i];
    if (c) atomicAdd(hist + static_cast<size_t>(g) * GRP * kHistBins + i, c);
  }
}

// ---- pass S, selection from the score histogram -----------------------------
//
// Pass A left, per query head, a histogram of its fast scores over the top 11
// bits of the order-preserving key, and max |score|.  The bin b1 holding the
// k-th largest score follows from the histogram alone.  Every token whose
// exact key can reach the top k has a fast score >= tau - 2 eps >= (lower
// edge of b1) - 2 eps, so:
//  A  compact: per (4096-token chunk, head), the tokens with fast score >=
//     lower(b1) - 2 eps, appended to the head's list (one atomic per chunk;
//     the list's order does not matter);
//  B  finish (one cluster per KV group, one CTA per query head): find tau
//     exactly by two more radix passes over the listed scores of bin b1,
//     keep the candidates >= tau - 2 eps, re-key them exactly in fp64 and
//     rank them (key desc, token asc); then the group's CTAs build the union
//     of their selections (bitmask and ascending list) through distributed
//     shared memory.

// Per-head threshold of the compaction and the histogram bin: all threads call.
__device__ void select_band(const int32_t* __restrict__ hist_h, int k, double eps_s, int* hsh, int* scan_scratch,
                            int* binfo, uint32_t* b1, int* kk, float* f_low) {
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hsh[i] = hist_h[i];
  __syncthreads();
  find_bin_from_top_block(hsh, kHistBins, k, binfo, scan_scratch);
  *b1 = static_cast<uint32_t>(binfo[0]);
  *kk = binfo[1];
  const float lower = from_okey32(*b1 << kHistShift);
  *f_low = __double2float_rd(static_cast<double>(lower) - 2.0 * eps_s);
}

constexpr int kCompThreads = 256;

template <int GRP>
__global__ void __launch_bounds__(kCompThreads)
attn_select_compact_kernel(const uint16_t* __restrict__ q, int T, int k, const float* __restrict__ score,
                           const float* __restrict__ smax, const int32_t* __restrict__ hist,
                           const uint32_t* __restrict__ amaxu, int32_t* __restrict__ cand,
                           int32_t* __restrict__ ccnt, int32_t* __restrict__ status) {
  const int chunk = blockIdx.x, h = blockIdx.y, g = h / GRP;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ int hsh[kHistBins];
  __shared__ int scan_scratch[64];
  __shared__ int binfo[2];
  __shared__ double qd[D];
  __shared__ double l1_sh, dq_sh;
  __shared__ int qe_sh;
  __shared__ int base_sh;
  select_q_prologue(q, h, g, qd, &l1_sh, &qe_sh, status, nullptr, kScQFrac, &dq_sh);
  const double eps_s = select_eps_pipe(static_cast<double>(smax[g]), static_cast<double>(smax[gridDim.y / GRP + g]),
                                       l1_sh, dq_sh, __uint_as_float(amaxu[h]));
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
    // the chunk's run of the head's list (the list's order does not matter:
    // the finish ranks by key and token)
    if (lane == 31) base_sh = incl ? atomicAdd(ccnt + h, incl) : 0;
  }
  __syncthreads();
  int32_t* out = cand + static_cast<size_t>(h) * T + base_sh;
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
constexpr int kFinList = 4096;     // listed (token, score) pairs cached in shared memory
constexpr size_t kFinDynSmem = static_cast<size_t>(kFinList) * 8 + static_cast<size_t>(kFinKeys) * 4;

template <int GRP>
__global__ void __launch_bounds__(kFinThreads)
attn_select_finish_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                          const uint32_t* __restrict__ k_ref, const uint16_t* __restrict__ k_scale,
                          const uint16_t* __restrict__ k_zero, int T, int k, int S, float* __restrict__ score,
                          const float* __restrict__ smax, const int32_t* __restrict__ hist,
                          const uint32_t* __restrict__ amaxu, const int32_t* __restrict__ cand,
                          const int32_t* __restrict__ ccnt, int32_t* __restrict__ list, double* __restrict__ kap,
                          int32_t* __restrict__ sel_head, uint32_t* __restrict__ umask, int words_t,
                          int32_t* __restrict__ sel_out, int32_t* __restrict__ sel_n, int32_t* __restrict__ status,
                          uint32_t* __restrict__ mkey) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = static_cast<int>(cl.block_rank());
  const int h = blockIdx.x, g = h / GRP;
  const int tid = threadIdx.x;
  __shared__ int hr[2048];
  __shared__ unsigned long long keys[kFinKeys];  // order-preserving exact keys, sorted with the tokens
  __shared__ double qd[D];
  __shared__ int scan_scratch[64];
  __shared__ int binfo[2];
  __shared__ double l1_sh, dq_sh;
  __shared__ int qe_sh, span_sh;
  __shared__ int cnt_sh;  // read remotely
  __shared__ int cntA_sh, cntB_sh;  // outright selections and band candidates listed
  __shared__ uint32_t qpl[3][8][4];  // byte planes of the fixed-point q, in code-extraction order
  __shared__ long long qxsum_sh;
  extern __shared__ int fin_dyn[];
  int* ltok = fin_dyn;                                      // [kFinList]
  float* lsc = reinterpret_cast<float*>(fin_dyn + kFinList);  // [kFinList]
  int* ktok = fin_dyn + 2 * kFinList;                       // [kFinKeys] tokens of the sorted keys
  const float* sc = score + static_cast<size_t>(h) * T;
  const int32_t* L = cand + static_cast<size_t>(h) * T;  // the compaction's list
  int32_t* F = list + static_cast<size_t>(h) * T;        // band candidates
  double* kp = kap + static_cast<size_t>(h) * T;
  const int cap = GRP * k;

  if (tid == 0) cntA_sh = cntB_sh = 0;
  select_q_prologue(q, h, g, qd, &l1_sh, &qe_sh, status, &span_sh, kScQFrac, &dq_sh);
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
  const double eps_s = select_eps_pipe(static_cast<double>(smax[g]), static_cast<double>(smax[gridDim.x / GRP + g]),
                                       l1_sh, dq_sh, __uint_as_float(amaxu[h]));
  uint32_t b1;
  int kk;
  float f_low;
  select_band(hist + static_cast<size_t>(h) * kHistBins, k, eps_s, hr, scan_scratch, binfo, &b1, &kk, &f_low);

  // 1. the compaction's list, with its fast scores in shared memory when it fits
  const int m = min(ccnt[h], T);
  if (m <= kFinList) {
    for (int e = tid; e < m; e += kFinThreads) {
      const int t = L[e];
      ltok[e] = t;
      lsc[e] = sc[t];
    }
  }
  __syncthreads();
  const bool cached = m <= kFinList;
  auto tok_of = [&](int e) { return cached ? ltok[e] : L[e]; };
  auto score_of = [&](int e) { return cached ? lsc[e] : sc[L[e]]; };

  // 2. tau: two radix passes (11 + 10 bits) over the listed scores of bin b1
  uint32_t pre = b1 << kHistShift;
  static_assert(kHistShift == 21, "the two passes cover the 21 key bits below the histogram's");
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? 10 : 0;
    const int nb = pass == 0 ? 2048 : 1024;
    for (int i = tid; i < nb; i += kFinThreads) hr[i] = 0;
    __syncthreads();
    const uint32_t pmask = pass == 0 ? 0xFFE00000u : 0xFFFFFC00u;
    for (int e = tid; e < m; e += kFinThreads) {
      const uint32_t key = okey32(score_of(e));
      if ((key & pmask) == pre) atomicAdd(&hr[(key >> shift) & static_cast<uint32_t>(nb - 1)], 1);
    }
    __syncthreads();
    find_bin_from_top_block(hr, nb, kk, binfo, scan_scratch);
    pre |= static_cast<uint32_t>(binfo[0]) << shift;
    kk = binfo[1];
  }
  const float tau = from_okey32(pre);
  const float fthr = __double2float_ru(static_cast<double>(tau) - 2.0 * eps_s);
  if (tid == 0) {
    // every token left out of the union has a fast score <= tau + 2 eps: pass
    // B's maximum needs no more (the union's resident scores, replaced by
    // refined ones, may lie far above every score pass B uses)
    const uint32_t b = okey32(__double2float_ru(static_cast<double>(tau) + 2.0 * eps_s));
    mkey[h] = min(mkey[h], b);
  }

  // 3. a token whose fast score exceeds tau + 2 eps outranks, by exact key,
  //    every token with fast score <= tau, so fewer than k tokens can rank
  //    above it: it is selected outright.  Only the band [tau - 2 eps,
  //    tau + 2 eps] is re-keyed and ranked (its candidates in token order).
  int32_t* sel = sel_head + static_cast<size_t>(h) * k;
  uint32_t* um = umask + static_cast<size_t>(g) * words_t;
  const double hi_band = static_cast<double>(tau) + 2.0 * eps_s;
  // listed in any order (the ranking orders by key and token): a warp takes
  // its slots with one shared atomic per list
  {
    const int lane = tid & 31;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = 0; base < m; base += kFinThreads) {
      const int e = base + tid;
      const float sv_e = e < m ? score_of(e) : 0.0f;
      const bool inA = e < m && static_cast<double>(sv_e) > hi_band;
      const bool inB = e < m && !inA && sv_e >= fthr;
      const int t = e < m ? tok_of(e) : 0;
      const unsigned bA = __ballot_sync(0xffffffffu, inA), bB = __ballot_sync(0xffffffffu, inB);
      int oA = 0, oB = 0;
      if (lane == 0) {
        if (bA) oA = atomicAdd(&cntA_sh, __popc(bA));
        if (bB) oB = atomicAdd(&cntB_sh, __popc(bB));
      }
      oA = __shfl_sync(0xffffffffu, oA, 0);
      oB = __shfl_sync(0xffffffffu, oB, 0);
      const int pA = oA + __popc(bA & lt);
      if (inA && pA < k) {  // fewer than k by the bound; guarded against corrupt scores
        sel[pA] = t;
        atomicOr(um + (t >> 5), 1u << (t & 31));
      }
      if (inB) F[oB + __popc(bB & lt)] = t;
    }
  }
  __syncthreads();
  const int nA = cntA_sh, ncand = cntB_sh;
  const int kB = max(0, k - nA);  // winners still to pick from the band (>= 1 by the bound)


  // 4. exact keys (four partial sums: exact under the precondition, so the
  //    order does not change the key)
  for (int i = tid; i < ncand; i += kFinThreads) {
    const int t = F[i];
    const size_t row = static_cast<size_t>(g) * S + t;
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

// ---- refined scores of the union --------------------------------------------------
//
// Step R, between the selection and pass B: every token of a group's union
// gets its
// scores for the group's query heads recomputed from the full 4-bit key codes,
// in place in the score buffer, and the largest refined score per head is
// recorded as an order-preserving key.  Pass B then weights every token
// against one fixed maximum per head (the larger of the refined maximum and a
// bound on the resident scores outside the union), so it needs no maximum
// pass and no rescaling.  A thread handles one union token for all the heads
// of the group: one load of the list, one of the token's two code rows.

constexpr int kRefThreads = 256;
// A unit of a KV refinement cache: the token-head's 8 K refinement words,
// then its 8 V refinement words.
constexpr int kCacheUnitWords = 2 * kWordsPerRow;

// The V refinement words of K/V row `row`: from the store (uslot == nullptr)
// or from the cache slot that holds the row's unit.
__device__ __forceinline__ const uint32_t* vref_row(const uint32_t* v_ref, const int32_t* uslot, size_t row) {
  return uslot != nullptr ? v_ref + static_cast<size_t>(uslot[row]) * kCacheUnitWords + kWordsPerRow
                          : v_ref + row * kWordsPerRow;
}

template <int GRP>
__global__ void __launch_bounds__(kRefThreads, 2)
attn_refine_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                   const uint32_t* __restrict__ k_ref, const int32_t* __restrict__ uslot,
                   const uint16_t* __restrict__ k_scale, const uint16_t* __restrict__ k_zero, int T, int S, int cap,
                   const int32_t* __restrict__ sel_out, const int32_t* __restrict__ sel_n, float* __restrict__ score,
                   uint32_t* __restrict__ rkey, uint32_t* __restrict__ umask, int words_t) {
  __shared__ float qs[GRP][D];
  __shared__ float qsum[GRP];
  const int g = blockIdx.y;
  const int lane = threadIdx.x & 31;
  load_q<GRP>(q, g, qs, qsum);  // contains __syncthreads
  const int sn = sel_n[g];
  const int U = min(cap, sn >= 0 ? sn : -1 - sn);
  const int32_t* list = sel_out + static_cast<size_t>(g) * cap;
  const size_t rowg = static_cast<size_t>(g) * S;  // K rows: the cache's stride
  uint32_t mk[GRP];
#pragma unroll
  for (int h = 0; h < GRP; ++h) mk[h] = 0u;
  for (int u0 = blockIdx.x * kRefThreads; u0 < U; u0 += gridDim.x * kRefThreads) {  // uniform over the block
    const int u = u0 + static_cast<int>(threadIdx.x);
    const int t = u < U ? list[u] : 0;
    const size_t row = rowg + t;
    const int slot = (u < U && uslot != nullptr) ? uslot[row] : 0;
    if (u < U && slot < 0) {
      // refinement bits not on the device (a cache miss): the token keeps its
      // resident key and value this step; it leaves the refined set, and its
      // resident scores still bound the weights' maximum
      atomicAnd(umask + static_cast<size_t>(g) * words_t + (t >> 5), ~(1u << (t & 31)));
#pragma unroll
      for (int h = 0; h < GRP; ++h)
        mk[h] = max(mk[h], okey32(score[(static_cast<size_t>(g) * GRP + h) * T + t]));
    } else if (u < U) {
      const uint4* pr = reinterpret_cast<const uint4*>(k_res + row * kWordsPerRow);
      const uint4* pf = reinterpret_cast<const uint4*>(
          uslot != nullptr ? k_ref + static_cast<size_t>(slot) * kCacheUnitWords : k_ref + row * kWordsPerRow);
      const uint4 r0 = pr[0], r1 = pr[1], f0 = pf[0], f1 = pf[1];
      const float sv = sfd::half_bits_to_float(k_scale[row]);
      const float z = sfd::half_bits_to_float(k_zero[row]);
      const uint32_t wr[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
      const uint32_t wf[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
      float P[GRP];
#pragma unroll
      for (int h = 0; h < GRP; ++h) P[h] = 0.0f;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float c = static_cast<float>(((wr[w] >> (2 * j)) & 3u) * 4u + ((wf[w] >> (2 * j)) & 3u));
#pragma unroll
          for (int h = 0; h < GRP; ++h) P[h] = fmaf(qs[h][16 * w + j], c, P[h]);
        }
      }
#pragma unroll
      for (int h = 0; h < GRP; ++h) {
        const float val = (sv * fmaf(-z, qsum[h], P[h])) * kInvSqrtD;
        mk[h] = max(mk[h], okey32(val));
        score[(static_cast<size_t>(g) * GRP + h) * T + t] = val;
      }
    }
  }
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mk[h] = max(mk[h], __shfl_xor_sync(0xffffffffu, mk[h], o));
    if (lane == 0 && mk[h]) atomicMax(rkey + g * GRP + h, mk[h]);
  }
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
// kSub tokens (4096 up to four query heads per group: one sub-chunk per CTA
// up to 128K tokens at 8 KV heads).  Every weight is computed once, by one thread, against the
// head's maximum over all tokens (resident and refined scores, recorded by the
// earlier passes), and stored in shared memory: no maximum pass and no
// rescaling.  The warps then run the MMAs over their tiles of 16 tokens, the
// codes staged by cp.async.

constexpr int kOutThreads = 256;
constexpr int kOW = kOutThreads / 32;
constexpr int kRing = 6;           // cp.async stages per warp
constexpr int kUCap = 384;         // refined rows per sub-chunk staged in shared memory

template <int GRP>
struct OutCfg {
  static constexpr int NC = 2 * GRP;           // weight columns: high parts of the heads, then remainders
  static constexpr int NT = NC <= 8 ? 1 : 2;   // MMA n-tiles of 8 columns
  static constexpr int kSub = NT == 1 ? 4096 : 2048;  // tokens per sub-chunk
  static constexpr int kPerThr = kSub / kOutThreads;  // tokens of a sub-chunk per thread in the weight pass
  static_assert(kPerThr % 4 == 0, "the weight pass loads four tokens per thread at a time");
  static constexpr int kStr = kSub + 8;        // halves per weight row: conflict-free fragment loads
  static constexpr size_t alpha_bytes = static_cast<size_t>(NT) * 8 * kStr * 2;
  static constexpr size_t ring_bytes = static_cast<size_t>(kOW) * kRing * 16 * kWordsPerRow * 4;
  static constexpr size_t ulist_bytes = static_cast<size_t>(kSub) * 2;
  static constexpr size_t vref_bytes = static_cast<size_t>(kUCap) * kWordsPerRow * 4;
  static constexpr size_t smem = alpha_bytes + ring_bytes + ulist_bytes + vref_bytes;
  static_assert(alpha_bytes >= static_cast<size_t>(kOW) * GRP * D * 4, "per-warp output tiles must fit the weight tile");
  static_assert(kSub / 32 <= kOutThreads, "the union scan takes a bitmask word per thread");
};

template <int GRP>
__global__ void __launch_bounds__(kOutThreads)
attn_out_kernel(const uint32_t* __restrict__ v_res,
                const uint32_t* __restrict__ v_ref, const int32_t* __restrict__ uslot,
                const uint16_t* __restrict__ v_scale,
                const uint16_t* __restrict__ v_zero, int T, int S, int tps, int words_t, int splits,
                const float* __restrict__ score, const uint32_t* __restrict__ mkey, const uint32_t* __restrict__ rkey,
                const uint32_t* __restrict__ umask, float* __restrict__ part, int32_t* __restrict__ done,
                float* __restrict__ out) {
  using C = OutCfg<GRP>;
  constexpr int NT = C::NT, kStr = C::kStr, kSub = C::kSub, kPerThr = C::kPerThr;
  extern __shared__ __align__(16) unsigned char smem[];
  __half* as = reinterpret_cast<__half*>(smem);                                      // [NT*8][kStr]
  uint32_t* ring = reinterpret_cast<uint32_t*>(smem + C::alpha_bytes);               // [kOW][kRing][16][8]
  uint16_t* ulist = reinterpret_cast<uint16_t*>(smem + C::alpha_bytes + C::ring_bytes);  // [kSub]
  uint32_t* vrs = reinterpret_cast<uint32_t*>(smem + C::alpha_bytes + C::ring_bytes +
                                              C::ulist_bytes);  // [kUCap][8] refinement rows of listed tokens
  __shared__ float red2[kOW][3 * GRP];
  __shared__ float Msh[GRP];
  __shared__ int ucount;
  __shared__ int uscan[33];

  const int g = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g8 = lane >> 2, tig = lane & 3;
  const int t0s = split * tps, t1s = min(T, t0s + tps);
  const size_t rowg = static_cast<size_t>(g) * S;  // V rows: the cache's stride

  for (int e = tid; e < (NT * 8 - C::NC) * kStr; e += kOutThreads) as[C::NC * kStr + e] = __float2half_rn(0.0f);
  // one maximum per head for every token: the larger of the bound on the
  // resident scores outside the union and the refined maximum (a key of 0:
  // no such token)
  if (tid < GRP) {
    const uint32_t mk = mkey[g * GRP + tid], rk = rkey[g * GRP + tid];
    float m = mk ? from_okey32(mk) : -INFINITY;
    if (rk) m = fmaxf(m, from_okey32(rk));
    Msh[tid] = m;
  }
  __syncthreads();

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
    //    their value refinement rows are staged for step 3 (their scores were
    //    refined in the score buffer before this pass)
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
        ulist[pos++] = static_cast<uint16_t>(32 * tid + b);
      }
      if (tid == 0) ucount = tot;
      __syncthreads();
    }
    const int nu = ucount;
    for (int u = tid; u < min(nu, kUCap); u += kOutThreads) {
      const uint32_t* src = vref_row(v_ref, uslot, rowg + c0 + ulist[u]);
      cp_async16_attn(vrs + u * kWordsPerRow, src);
      cp_async16_attn(vrs + u * kWordsPerRow + 4, src + 4);
    }
    cp_async_commit_attn();
    float M[GRP];
#pragma unroll
    for (int h = 0; h < GRP; ++h) M[h] = Msh[h];

    // 1. weights into shared memory (zero past the end of the last tile) and
    //    sums; the scores, scales and zeros of four of this thread's tokens
    //    are loaded before any is used
#pragma unroll 1
    for (int j0 = 0; j0 < kPerThr; j0 += 4) {
      if (j0 * kOutThreads >= 16 * ntile) break;  // uniform over the block
      float sc4[4][GRP];
      uint16_t vs4[4], vz4[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int i = tid + (j0 + jj) * kOutThreads;
        const bool valid = i < n;
        vs4[jj] = valid ? v_scale[rowg + c0 + i] : 0;
        vz4[jj] = valid ? v_zero[rowg + c0 + i] : 0;
#pragma unroll
        for (int h = 0; h < GRP; ++h) sc4[jj][h] = valid ? score[(static_cast<size_t>(g) * GRP + h) * T + c0 + i] : 0.0f;
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
      const int i = tid + (j0 + jj) * kOutThreads;
      const bool valid = i < n;
      if (i < 16 * ntile) {
        if (valid) {
          const float sv = sfd::half_bits_to_float(vs4[jj]);
          const float zv = sfd::half_bits_to_float(vz4[jj]);
#pragma unroll
          for (int h = 0; h < GRP; ++h) {
            const float p = __expf(sc4[jj][h] - M[h]);
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
    }
    __syncthreads();

    // 2. MMAs over this warp's tiles
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
      // word g8 of token rows 2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9: MMA s
      // covers dims 16 g8 + s and 16 g8 + 8 + s (vfrag)
      uint32_t src[4][4];
      vperm(vr[(2 * tig) * kWordsPerRow + g8], vr[(2 * tig + 1) * kWordsPerRow + g8],
            vr[(2 * tig + 8) * kWordsPerRow + g8], vr[(2 * tig + 9) * kWordsPerRow + g8], src);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        uint32_t a0, a1, a2, a3;
        vfrag(src, s, a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_f16f32(acc[nt][s], a0, a1, a2, a3, b0[nt], b1[nt]);
      }
      __syncwarp();
    }
    cp_async_wait_attn<0>();
    __syncthreads();  // the staged refinement rows come from every thread

    // 3. refined tokens: alpha (c_f - 1.5), lane = dims 4 lane .. 4 lane + 3
    for (int u = warp; u < nu; u += kOW) {
      const int i = ulist[u];
      const uint32_t wrow = u < kUCap ? vrs[u * kWordsPerRow + (lane >> 2)]
                                      : vref_row(v_ref, uslot, rowg + c0 + i)[lane >> 2];
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

  // this warp's output tile ww[head][dim] (in units of the code part, which
  // carries the factor 4^e of the dim's fragment position: uo enters as
  // uo 4^e / 2^b_f) in the dead weight tile, written in three phases whose
  // stores within a warp never collide (high columns, then remainder
  // columns, then the refined corrections); summed over warps below
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
          float* dst = &ww[hh * D + 16 * g8 + w + 8 * (c >> 1)];  // MMA w, row g8 (+ 8)
          *dst = ph == 0 ? acc[nt][w][c] : *dst + acc[nt][w][c];
        }
    __syncwarp();
  }
#pragma unroll
  for (int h = 0; h < GRP; ++h)
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) ww[h * D + 4 * lane + dd] += (0.25f * vpos_mul(4 * lane + dd)) * uo[h][dd];
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
      // resident value s (2^b_f c + m_f - z): code part 4 (acc - 1024 A) 4^-e,
      // offset part Cs
      float o = 0.0f;
      if (j >= 2)
        for (int w = 0; w < kOW; ++w) o += reinterpret_cast<const float*>(smem)[(w * GRP + h) * D + j - 2];
      const float f = j >= 2 ? vpos_inv(j - 2) : 1.0f;
      v = j == 1 ? L : fmaf(4.0f * f, o, fmaf(-4096.0f * f, A, Cs));
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
  // every split weighted its tokens against the same maximum per head: the
  // merge sums the splits' weight sums and outputs; two outputs per thread,
  // eight splits' partials of each in flight at once
  for (int e0 = tid; e0 < GRP * D; e0 += 2 * kOutThreads) {
    const int e1 = e0 + kOutThreads;
    const bool has1 = e1 < GRP * D;
    const int h0 = e0 / D, h1 = has1 ? e1 / D : h0;
    const float* p0 = pg + static_cast<size_t>(h0) * splits * (D + 2);
    const float* p1 = pg + static_cast<size_t>(h1) * splits * (D + 2);
    const int d0 = e0 % D, d1 = has1 ? e1 % D : d0;
    float A0 = 0.0f, A1 = 0.0f, L0 = 0.0f, L1 = 0.0f;
    for (int sp = 0; sp < splits; sp += 8) {
      float v0[8], v1[8], l0[8], l1[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const size_t o = static_cast<size_t>(sp + u) * (D + 2);
        const bool ok = sp + u < splits;
        v0[u] = ok ? __ldcg(p0 + o + 2 + d0) : 0.0f;
        l0[u] = ok ? __ldcg(p0 + o + 1) : 0.0f;
        v1[u] = (ok && has1) ? __ldcg(p1 + o + 2 + d1) : 0.0f;
        l1[u] = (ok && has1) ? __ldcg(p1 + o + 1) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        A0 += v0[u];
        L0 += l0[u];
        A1 += v1[u];
        L1 += l1[u];
      }
    }
    out[(static_cast<size_t>(g) * GRP + h0) * D + d0] = A0 / L0;
    if (has1) out[(static_cast<size_t>(g) * GRP + h1) * D + d1] = A1 / L1;
  }
}

__global__ void fill_all_kernel(int T, int grp, int k, int words_t, uint32_t* umask, int32_t* sel_out,
                                int32_t* sel_n, uint32_t* mkey) {
  const int g = blockIdx.y;
  if (blockIdx.x == 0 && threadIdx.x < grp) mkey[g * grp + threadIdx.x] = 0u;  // no token outside the union
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
  const int S = kv->row_stride > 0 ? kv->row_stride : T;  // rows per KV head in the K/V arrays
  // refinement source: the stores k_ref / v_ref, or a KV refinement cache
  const uint32_t* k_ref = kv->k_ref;
  const uint32_t* v_ref = kv->v_ref;
  const int32_t* uslot = nullptr;
  if (kv->ref_cache) {
    sf::CacheView v{};
    const sf_status cs = sf::cache_view_for_reader(kv->ref_cache, s, &v);
    if (cs != SF_OK) return cs;
    SF_REQUIRE(v.unit_words == kCacheUnitWords, "sf_attn_decode_refine: ref_cache units must be %d bytes",
               4 * kCacheUnitWords);
    SF_REQUIRE(static_cast<long long>(v.num_units) >= static_cast<long long>(Hkv) * S,
               "sf_attn_decode_refine: ref_cache has fewer units than Hkv * row_stride");
    k_ref = v_ref = v.rows;
    uslot = v.unit_slot;
  }
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
  // pass A: about two CTAs per SM, each a contiguous range of <= kScMaxTok tokens
  const int want_a = std::max((2 * sms + Hkv - 1) / Hkv, (T + kScMaxTok - 1) / kScMaxTok);
  const int tpc = ((T + want_a - 1) / want_a + 15) / 16 * 16;
  dim3 ga((T + tpc - 1) / tpc, Hkv);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + L.hist);
  uint32_t* amaxu = reinterpret_cast<uint32_t*>(ws + L.amax);
  uint32_t* mkey = reinterpret_cast<uint32_t*>(ws + L.mkey);
  uint32_t* rkey = reinterpret_cast<uint32_t*>(ws + L.rkey);
  SF_CHECK_CUDA(cudaFuncSetAttribute(attn_score_mma_kernel<GRP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(score_smem(GRP))));
  attn_score_mma_kernel<GRP><<<ga, kScThreads, score_smem(GRP), s>>>(q, kv->k_res, kv->k_scale, kv->k_zero, T, S,
                                                                     tpc, score, smax, hist, amaxu, mkey);
  sf_status st = sf::check_launch("attn_score_mma_kernel");
  if (st != SF_OK) return st;
  if (k > 0 && k < T) {
    int32_t* ccnt = reinterpret_cast<int32_t*>(ws + L.ccnt);
    attn_select_compact_kernel<GRP><<<dim3(L.nchunks, Hq), kCompThreads, 0, s>>>(q, T, k, score, smax, hist, amaxu,
                                                                                cand, ccnt, status);
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
                                     kv->k_zero, T, k, S, score, static_cast<const float*>(smax),
                                     static_cast<const int32_t*>(hist), static_cast<const uint32_t*>(amaxu), cand,
                                     static_cast<const int32_t*>(ccnt), cand2, kap, sel_head, umask, L.words_t,
                                     sel_out, sel_n, status, mkey));
    st = sf::check_launch("attn_select_finish_kernel");
    if (st != SF_OK) return st;
  } else if (k == 0) {  // the token bitmask was cleared with the workspace
    SF_CHECK_CUDA(cudaMemsetAsync(sel_n, 0, sizeof(int32_t) * Hkv, s));
  } else {
    fill_all_kernel<<<dim3(32, Hkv), 256, 0, s>>>(T, grp, k, L.words_t, umask, sel_out, sel_n, mkey);
    st = sf::check_launch("fill_all_kernel");
    if (st != SF_OK) return st;
  }
  if (k > 0) {
    const int cap = grp * k;
    const int nblk = std::max(1, std::min((cap + kRefThreads - 1) / kRefThreads, 2 * sms / Hkv));
    attn_refine_kernel<GRP><<<dim3(nblk, Hkv), kRefThreads, 0, s>>>(q, kv->k_res, k_ref, uslot, kv->k_scale,
                                                                   kv->k_zero, T, S, cap, sel_out, sel_n, score,
                                                                   rkey, umask, L.words_t);
    st = sf::check_launch("attn_refine_kernel");
    if (st != SF_OK) return st;
  }
  dim3 gb(L.splits, Hkv);
  SF_CHECK_CUDA(cudaFuncSetAttribute(attn_out_kernel<GRP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(OutCfg<GRP>::smem)));
  attn_out_kernel<GRP><<<gb, kOutThreads, OutCfg<GRP>::smem, s>>>(kv->v_res, v_ref, uslot, kv->v_scale, kv->v_zero,
                                                                 T, S, L.tps, L.words_t, L.splits, score, mkey, rkey,
                                                                 umask, part, done, out);
  st = sf::check_launch("attn_out_kernel");
  if (st != SF_OK) return st;
  if (kv->ref_cache) return sf::cache_mark_used(kv->ref_cache, s);
  return SF_OK;
}

std::atomic<int> g_attn_path{SF_ATTN_AUTO};

// The cluster kernel where it applies (and is allowed), else the pipeline.
sf_status dispatch(const uint16_t* q, int Hq, int Hkv, int T, const sf_qkv* kv, int k, int32_t* sel_out,
                   int32_t* sel_n, float* out, char* ws, const Layout& L, cudaStream_t s) {
  const int path = g_attn_path.load(std::memory_order_relaxed);
  if (path == SF_ATTN_CLUSTER && kv->ref_cache)
    return sf::fail(SF_ENOTIMPL, "sf_attn_decode_refine: the cluster kernel does not read a ref_cache");
  if (path != SF_ATTN_PIPELINE && !kv->ref_cache) {
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
  SF_REQUIRE(kv->k_res && kv->v_res && kv->k_scale && kv->k_zero && kv->v_scale && kv->v_zero &&
                 (kv->ref_cache || (kv->k_ref && kv->v_ref)),
             "sf_attn_decode_refine: null K/V view");
  SF_REQUIRE(kv->b_r == 2 && kv->b_f == 2, "sf_attn_decode_refine: only 2-bit resident + 2-bit refinement K/V");
  SF_REQUIRE(d == D, "sf_attn_decode_refine: head dim must be %d", D);
  SF_REQUIRE(Hkv >= 1 && Hq >= Hkv && Hq % Hkv == 0, "sf_attn_decode_refine: Hq must be a multiple of Hkv");
  SF_REQUIRE(T >= 1 && T <= (1 << 24), "sf_attn_decode_refine: T out of range");
  SF_REQUIRE(k_tokens >= 0 && k_tokens <= T, "sf_attn_decode_refine: k_tokens must be in [0, T]");
  SF_REQUIRE(kv->row_stride == 0 || kv->row_stride >= T, "sf_attn_decode_refine: row_stride must be 0 or >= T");
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

// ---- units of a KV refinement cache selected by one call -----------------------

namespace {

__global__ void union_units_kernel(const int32_t* __restrict__ sel_out, const int32_t* __restrict__ sel_n, int Hkv,
                                   int cap, int S, int32_t* __restrict__ units, int32_t* __restrict__ n_units) {
  __shared__ int off[65];
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int g = 0; g < Hkv; ++g) {
      off[g] = acc;
      const int n = sel_n[g];
      acc += min(cap, n >= 0 ? n : -1 - n);
    }
    off[Hkv] = acc;
    *n_units = acc;
  }
  __syncthreads();
  for (int g = 0; g < Hkv; ++g) {
    const int n = off[g + 1] - off[g];
    for (int i = threadIdx.x; i < n; i += blockDim.x)
      units[off[g] + i] = g * S + sel_out[static_cast<size_t>(g) * cap + i];
  }
}

}  // namespace

extern "C" sf_status sf_attn_union_units(const int32_t* sel_out, const int32_t* sel_n, int Hkv, int cap, int S,
                                         int32_t* units, int32_t* n_units, sf_stream_t stream) {
  SF_REQUIRE(sel_out && sel_n && units && n_units, "sf_attn_union_units: null pointer");
  SF_REQUIRE(Hkv >= 1 && Hkv <= 64 && cap >= 1 && S >= 1, "sf_attn_union_units: need Hkv in [1, 64], cap, S >= 1");
  SF_REQUIRE(static_cast<long long>(Hkv) * S <= 0x7FFFFFFFLL, "sf_attn_union_units: Hkv * S overflows int32");
  union_units_kernel<<<1, 1024, 0, sf::as_cuda(stream)>>>(sel_out, sel_n, Hkv, cap, S, units, n_units);
  return sf::check_launch("union_units_kernel");
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
  SF_REQUIRE(kv->k_res && kv->v_res && kv->k_scale && kv->k_zero && kv->v_scale && kv->v_zero &&
                 (kv->ref_cache || (kv->k_ref && kv->v_ref)),
             "sf_attn_decode_refine_noalloc: null K/V view");
  SF_REQUIRE(kv->b_r == 2 && kv->b_f == 2, "sf_attn_decode_refine_noalloc: only 2-bit resident + 2-bit refinement K/V");
  SF_REQUIRE(d == D, "sf_attn_decode_refine_noalloc: head dim must be %d", D);
  SF_REQUIRE(Hkv >= 1 && Hq >= Hkv && Hq % Hkv == 0, "sf_attn_decode_refine_noalloc: Hq must be a multiple of Hkv");
  SF_REQUIRE(T >= 1 && T <= (1 << 24), "sf_attn_decode_refine_noalloc: T out of range");
  SF_REQUIRE(k_tokens >= 0 && k_tokens <= T, "sf_attn_decode_refine_noalloc: k_tokens must be in [0, T]");
  SF_REQUIRE(kv->row_stride == 0 || kv->row_stride >= T, "sf_attn_decode_refine_noalloc: row_stride must be 0 or >= T");
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
