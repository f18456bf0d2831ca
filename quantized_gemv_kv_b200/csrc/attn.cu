// sf_attn_decode_refine: decode attention over 2-bit resident K/V with the
// most-attended tokens refined to their full 4-bit codes.
//
// StrataFlux picks KV refinements by the attention weight computed from the
// low-bit keys (rag-lover.com explainer, 解説).  The pass structure:
//
//   A  score   per (KV head, token): resident scores of the Hq/Hkv query
//              heads of the group from the 2-bit keys, fp32, into scratch.
//   S  select  per query head: the k largest scores, exactly.  The fast fp32
//              scores carry a proven error bound eps; every token within
//              2*eps of the k-th largest fast score is a candidate, and the
//              candidates are re-scored exactly in fp64 (the key s*E with
//              E = sum_d q_d (c_d 2^b_f + m_f - z) is exact in fp64 under a
//              precondition on q checked here) and ranked by (key desc, token
//              asc).  So the chosen set equals the exact definition.
//   U  union   per KV head: union of its query heads' choices, ascending,
//              plus a token bitmask.
//   B  output  split over tokens: online softmax over all tokens with the
//              refined (full-code) K and V for tokens in the union and the
//              resident ones elsewhere -- refined tokens are computed directly,
//              never by subtracting their resident contribution.
//   M  merge   per KV group, by the last CTA of pass B to finish: combine the
//              splits' (max, sum, output).
//
// Every scratch array lives in the caller's workspace; nothing is allocated.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "block_scan.cuh"
#include "sf_internal.h"

namespace {

constexpr int D = 128;                 // head dim
constexpr int kWordsPerRow = D * 2 / 32;  // 2-bit codes of one token-head: 8 words
constexpr int kMaxGrp = 8;
constexpr int kMaxSplits = 256;
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1/sqrt(128), rounded to fp32

struct Layout {
  size_t score, cand, cand2, kap, sel, umask, part, smax, status, count, total;
  int splits, tps, words_t;
};

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

Layout make_layout(int Hq, int Hkv, int T, int k, int sms) {
  Layout L{};
  const int want = std::max(1, std::min(kMaxSplits, 2 * sms / Hkv));  // one wave of pass-B CTAs at 2 per SM
  int tps = (T + want - 1) / want;
  tps = std::max(128, (tps + 127) / 128 * 128);
  L.tps = tps;
  L.splits = (T + tps - 1) / tps;
  L.words_t = (T + 31) / 32;
  size_t off = 0;
  L.score = off; off = up256(off + sizeof(float) * Hq * static_cast<size_t>(T));
  L.cand = off; off = up256(off + sizeof(int32_t) * Hq * static_cast<size_t>(T));
  L.cand2 = off; off = up256(off + sizeof(int32_t) * Hq * static_cast<size_t>(T));
  L.kap = off; off = up256(off + sizeof(double) * Hq * static_cast<size_t>(T));
  L.sel = off; off = up256(off + sizeof(int32_t) * Hq * static_cast<size_t>(std::max(k, 1)));
  L.umask = off; off = up256(off + sizeof(uint32_t) * Hkv * static_cast<size_t>(L.words_t));
  L.part = off; off = up256(off + sizeof(float) * Hq * static_cast<size_t>(L.splits) * (D + 2));
  L.smax = off; off = up256(off + sizeof(float) * Hkv);
  L.status = off; off = up256(off + sizeof(int32_t) * std::max(Hkv, 4));
  L.count = off; off = up256(off + sizeof(int32_t) * Hkv);
  L.total = off;
  return L;
}

__device__ __forceinline__ uint32_t okey32(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float from_okey32(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
__device__ __forceinline__ unsigned long long okey64(double x) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x));
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}


__device__ __forceinline__ void cp_async16_attn(void* smem, const void* gmem) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem));
}
__device__ __forceinline__ void cp_async4_attn(void* smem, const void* gmem) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(sa), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit_attn() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait_attn() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

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
__device__ __forceinline__ void mma_u8u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int GRP>
__global__ void __launch_bounds__(128)
attn_score_mma_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                      const uint16_t* __restrict__ k_scale, const uint16_t* __restrict__ k_zero, int T,
                      float* __restrict__ score, float* __restrict__ smax) {
  __shared__ int qx[GRP][D];
  __shared__ float qsc[GRP], qsm[GRP];
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
        score[(static_cast<size_t>(g) * GRP + h) * T + t] = (sv * E) * kInvSqrtD;
      }
    }
    cur = nxt;
  }
  smx = warp_max(smx);
  if (lane == 0) atomicMax(reinterpret_cast<unsigned int*>(smax + g), __float_as_uint(smx));
}

// ---- pass S: exact per-head top-k ------------------------------------------
constexpr int kSelThreads = 1024;

// Finds the bin holding the kk-th largest element of a histogram of nb bins
// (scanning from the top) with warp 0.  Returns via shared out[0] = bin,
// out[1] = kk left inside the bin.
__device__ void find_bin_from_top(const int* hist, int nb, int kk, int* out) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  int above = 0;
  for (int base = nb - 1; base >= 0; base -= 32) {
    const int bin = base - lane;
    const int c = bin >= 0 ? hist[bin] : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const bool hit = (above + incl >= kk) && (above + incl - c < kk);
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (m) {
      const int src = __ffs(m) - 1;
      const int before = __shfl_sync(0xffffffffu, incl - c, src);
      if (lane == 0) { out[0] = base - src; out[1] = kk - (above + before); }
      return;
    }
    above += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) { out[0] = 0; out[1] = kk; }
}

// Block-wide sum of two ints (all threads call; result in every thread).
__device__ __forceinline__ void block_sum2(int& a, int& b, int* scratch /* 64 ints */) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (lane == 0) { scratch[warp] = a; scratch[32 + warp] = b; }
  __syncthreads();
  a = 0;
  b = 0;
  for (int w = 0; w < nw; ++w) { a += scratch[w]; b += scratch[32 + w]; }
  __syncthreads();
}

// Exact per-head top-k (see the pass structure at the top of this file).
//  1. amax over the fast scores and a strided sample of them;
//  2. a threshold theta from the sample such that at least k scores are
//     >= theta + 2 eps (checked by counting; lowered until true, at worst to
//     -inf), so every token whose exact key can reach the top k has a fast
//     score >= theta;
//  3. G = {t : score_t >= theta} in token order, tau = k-th largest score over
//     G by radix select (equal to the k-th largest overall);
//  4. candidates F = {t in G : score_t >= tau - 2 eps}, re-keyed exactly in
//     fp64, ranked by (key desc, token asc).
// Ordered (stable) compaction of the indices i in [0, n) with pred(i), by a
// whole block: warp w owns the contiguous segment [w seg, (w+1) seg) and walks
// it 32 indices at a time (coalesced), with ballots giving positions inside
// the warp; a prefix over the warps' counts gives each warp's offset.
// Writes emit(pos, i) for the kept indices and returns their count.  Every
// thread of the block must call it.
template <class Pred, class Emit>
__device__ int block_ordered_compact(int n, Pred pred, Emit emit, int* wsum /* 33 ints */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int seg = (((n + nw - 1) / nw) + 31) & ~31;
  const int b0 = min(n, warp * seg), b1 = min(n, b0 + seg);
  int cnt = 0;
  for (int base = b0; base < b1; base += 32) {
    const int i = base + lane;
    cnt += __popc(__ballot_sync(0xffffffffu, i < b1 && pred(i)));
  }
  __syncthreads();
  if (lane == 0) wsum[warp] = cnt;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < nw ? wsum[lane] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane < nw) wsum[lane] = incl - v;
    if (lane == 31) wsum[32] = incl;
  }
  __syncthreads();
  int off = wsum[warp];
  const int total = wsum[32];
  const unsigned lt = (1u << lane) - 1u;
  for (int base = b0; base < b1; base += 32) {
    const int i = base + lane;
    const bool p = i < b1 && pred(i);
    const unsigned bal = __ballot_sync(0xffffffffu, p);
    if (p) emit(off + __popc(bal & lt), i);
    off += __popc(bal);
  }
  __syncthreads();
  return total;
}

constexpr int kDirectRank = 1024;  // candidates ranked pairwise (one per thread)

// Query-side setup of pass S (all threads call): q in fp64 into qd, its l1
// norm and the binary exponent of max |q|; flags the KV group when the
// nonzero q exponents span more than the exact-key precondition allows.
__device__ void select_q_prologue(const uint16_t* __restrict__ q, int h, int g, double* qd, double* l1_out,
                                  int* qe_out, int32_t* __restrict__ status) {
  const int tid = threadIdx.x;
  for (int d = tid; d < D; d += blockDim.x)
    qd[d] = static_cast<double>(sfd::bf16_bits_to_float(q[static_cast<size_t>(h) * D + d]));
  __syncthreads();
  if (tid < 32) {
    double l1 = 0.0;
    int emin = 100000, emax = -100000;
    for (int d = tid; d < D; d += 32) {
      const double v = qd[d];
      l1 += fabs(v);
      if (v != 0.0) {
        int e;
        frexp(v, &e);
        emin = min(emin, e);
        emax = max(emax, e);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      emin = min(emin, __shfl_xor_sync(0xffffffffu, emin, o));
      emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
    }
    if (tid == 0) {
      *l1_out = l1;
      *qe_out = emax >= emin ? emax : 0;  // binary exponent of max |q| (frexp convention)
      // 53 - 9 - b - log2(d) with b = 4, d = 128
      if (emax >= emin && emax - emin > 53 - 9 - 4 - 7) atomicOr(status + g, 1);
    }
  }
  __syncthreads();
}

// Error bound of the fast scores (pass A): q rounded to 24-bit fixed point
// (|dq| <= 2^(e-24) per entry), exact integer products and sums, an fp32
// combine of the three plane sums, the fp32 sum of q (<= gamma_128 l1), and
// the roundings of the zero-point term, the fma, the scale and 1/sqrt(d).
// Returns the half-width eps_s of the band; two fast scores whose exact
// values are ordered one way differ by at least -2 eps_s the other way.
__device__ __forceinline__ double select_eps(double s_max, double l1, int qe, float amax) {
  const double u = 5.9604644775390625e-8;  // 2^-24
  const double gam = 130.0 * u / (1.0 - 130.0 * u);
  const double qround = ldexp(1.0, qe - 24);
  const double eps_k = s_max * (4.0 * 3.0 * D * qround + l1 * (136.0 * u + 16.0 * gam));
  return 2.0 * (static_cast<double>(kInvSqrtD) * eps_k + 4.0 * u * static_cast<double>(amax));
}

// Last stage of pass S (all threads call): the candidates F[0..ncand) (token
// order) are re-keyed exactly in fp64 and the k best by (key desc, token asc)
// written to sel (k entries, ascending rank order is not required).
__device__ void select_finish(const uint32_t* __restrict__ k_res, const uint16_t* __restrict__ k_scale,
                              const uint16_t* __restrict__ k_zero, int g, int T, int k, const double* qd,
                              const int32_t* __restrict__ F, int ncand, double* __restrict__ kp, int* hist,
                              int* scan_scratch, int* binfo, int32_t* __restrict__ sel) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  for (int i = tid; i < ncand; i += nthr) {
    const int t = F[i];
    const size_t row = static_cast<size_t>(g) * T + t;
    const uint4* w4 = reinterpret_cast<const uint4*>(k_res + row * kWordsPerRow);
    const uint4 x0 = w4[0], x1 = w4[1];
    const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    const double sv = static_cast<double>(sfd::half_bits_to_float(k_scale[row]));
    const double z = static_cast<double>(sfd::half_bits_to_float(k_zero[row]));
    double E = 0.0;
#pragma unroll
    for (int wi = 0; wi < 8; ++wi) {
      const uint32_t word = w[wi];
#pragma unroll 4
      for (int j = 0; j < 16; ++j) {
        const double c = static_cast<double>((word >> (2 * j)) & 3u);
        E = fma(qd[16 * wi + j], c * 4.0 + 1.5 - z, E);
      }
    }
    kp[i] = sv * E;
  }
  __syncthreads();

  // few candidates (the usual case): rank each one directly against all
  // others by (key desc, token asc) -- no synchronised passes
  if (ncand <= kDirectRank && ncand <= nthr) {
    double* kd = reinterpret_cast<double*>(hist);  // 2048 ints = 1024 doubles of scratch
    for (int i = tid; i < ncand; i += nthr) kd[i] = kp[i];
    __syncthreads();
    int take = 0;
    const int i = tid;
    if (i < ncand) {
      const double ki = kd[i];
      int rank = 0;
      for (int j = 0; j < ncand; ++j) {
        const double kj = kd[j];
        rank += (kj > ki) || (kj == ki && j < i);  // F is in token order
      }
      take = rank < k;
    }
    int tot;
    const int pos = sfd::block_exclusive_scan(take, scan_scratch, &tot);
    if (take) sel[pos] = F[i];
    return;
  }

  // many candidates: exact top-k by an 8-pass radix select on the 64-bit keys
  unsigned long long pre64 = 0, pm64 = 0;
  int kr = k;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = tid; i < 256; i += nthr) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < ncand; i += nthr) {
      const unsigned long long key = okey64(kp[i]);
      if ((key & pm64) == pre64) atomicAdd(&hist[(key >> shift) & 255], 1);
    }
    __syncthreads();
    find_bin_from_top(hist, 256, kr, binfo);
    __syncthreads();
    pre64 |= static_cast<unsigned long long>(binfo[0]) << shift;
    pm64 |= 255ull << shift;
    kr = binfo[1];
    __syncthreads();
  }
  {
    const int chunk = (ncand + nthr - 1) / nthr;
    const int i0 = min(ncand, tid * chunk), i1 = min(ncand, i0 + chunk);
    int eq = 0;
    for (int i = i0; i < i1; ++i) eq += okey64(kp[i]) == pre64;
    int tot;
    int rank = sfd::block_exclusive_scan(eq, scan_scratch, &tot);
    int take = 0;
    {
      int rk = rank;
      for (int i = i0; i < i1; ++i) {
        const unsigned long long key = okey64(kp[i]);
        if (key > pre64) ++take;
        else if (key == pre64) { if (rk < kr) ++take; ++rk; }
      }
    }
    int pos = sfd::block_exclusive_scan(take, scan_scratch, &tot);
    for (int i = i0; i < i1; ++i) {
      const unsigned long long key = okey64(kp[i]);
      bool ok = false;
      if (key > pre64) ok = true;
      else if (key == pre64) { ok = rank < kr; ++rank; }
      if (ok) sel[pos++] = F[i];
    }
  }
}

// Exact per-head top-k for any T, streaming the scores from global memory:
//  1. amax over the fast scores and a strided sample of them;
//  2. a threshold theta from the sample such that at least k scores are
//     >= theta + 2 eps (checked by counting; lowered until true, at worst to
//     -inf), so every token whose exact key can reach the top k has a fast
//     score >= theta;
//  3. G = {t : score_t >= theta} in token order, tau = k-th largest score over
//     G by radix select (equal to the k-th largest overall);
//  4. candidates F = {t in G : score_t >= tau - 2 eps}, re-keyed exactly in
//     fp64, ranked by (key desc, token asc).
template <int GRP>
__global__ void __launch_bounds__(kSelThreads)
attn_select_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                   const uint16_t* __restrict__ k_scale, const uint16_t* __restrict__ k_zero, int T, int k,
                   const float* __restrict__ score, const float* __restrict__ smax, int32_t* __restrict__ cand,
                   int32_t* __restrict__ cand2, double* __restrict__ kap, int32_t* __restrict__ sel_head,
                   int32_t* __restrict__ status) {
  constexpr int kSamples = 512;
  __shared__ __align__(16) int hist[2048];
  __shared__ double qd[D];
  __shared__ float samp[kSamples];
  __shared__ int scan_scratch[64];
  __shared__ int binfo[2];
  __shared__ float red[32];
  __shared__ double l1_sh;
  __shared__ int qe_sh;
  __shared__ float theta_sh;
  const int h = blockIdx.x, g = h / GRP, tid = threadIdx.x;
  const float* sc = score + static_cast<size_t>(h) * T;
  int32_t* G = cand + static_cast<size_t>(h) * T;
  int32_t* F = cand2 + static_cast<size_t>(h) * T;
  double* kp = kap + static_cast<size_t>(h) * T;

  select_q_prologue(q, h, g, qd, &l1_sh, &qe_sh, status);

  // 1. amax and a strided sample
  const int ns = T < kSamples ? T : kSamples;
  const int stride = T / ns;
  float amax = 0.0f;
  for (int t = tid; t < T; t += kSelThreads) amax = fmaxf(amax, fabsf(sc[t]));
  for (int i = tid; i < ns; i += kSelThreads) samp[i] = sc[i * stride];
  {
    const float m = warp_max(amax);
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    if (tid < 32) {
      const float mm = warp_max(red[tid]);
      if (tid == 0) red[0] = mm;
    }
    __syncthreads();
    amax = red[0];
  }
  const double eps_s = select_eps(static_cast<double>(smax[g]), l1_sh, qe_sh, amax);

  // 2. threshold from the sample: aim at ~2k + 64 tokens above it
  double theta = -INFINITY;
  for (int trial = 0; trial < 3; ++trial) {
    int want = static_cast<int>((static_cast<long long>(2 * k + 64) * ns) / T) + 1;
    want <<= (2 * trial);  // lower the threshold on a retry
    if (trial == 2 || want >= ns) break;  // fall back to all tokens
    // the want-th largest sample (rank counted from 1)
    for (int i = tid; i < ns; i += kSelThreads) {
      const float v = samp[i];
      int gt = 0, ge = 0;
      for (int j = 0; j < ns; ++j) {
        const float w = samp[j];
        gt += w > v;
        ge += w >= v;
      }
      if (gt < want && want <= ge) theta_sh = v;
    }
    __syncthreads();
    const double th = static_cast<double>(theta_sh) - 2.0 * eps_s;
    int c1 = 0, dummy = 0;
    for (int t = tid; t < T; t += kSelThreads) c1 += static_cast<double>(sc[t]) >= th + 2.0 * eps_s;
    block_sum2(c1, dummy, scan_scratch);
    if (c1 >= k) { theta = th; break; }
  }

  // 3. G in token order, then tau = k-th largest over G
  const int nG = block_ordered_compact(
      T, [&](int t) { return static_cast<double>(sc[t]) >= theta; }, [&](int pos, int t) { G[pos] = t; },
      scan_scratch);
  uint32_t prefix = 0, pmask = 0;
  int kk = k;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int nb = 1 << widths[pass];
    for (int i = tid; i < nb; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < nG; i += kSelThreads) {
      const uint32_t key = okey32(sc[G[i]]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shifts[pass]) & (nb - 1)], 1);
    }
    __syncthreads();
    find_bin_from_top(hist, nb, kk, binfo);
    __syncthreads();
    prefix |= static_cast<uint32_t>(binfo[0]) << shifts[pass];
    pmask |= static_cast<uint32_t>(nb - 1) << shifts[pass];
    kk = binfo[1];
    __syncthreads();
  }
  const double tau = static_cast<double>(from_okey32(prefix));
  const double thr = tau - 2.0 * eps_s;

  // 4. candidates F (token order), exact keys, ranking
  const int ncand = block_ordered_compact(
      nG, [&](int i) { return static_cast<double>(sc[G[i]]) >= thr; }, [&](int pos, int i) { F[pos] = G[i]; },
      scan_scratch);
  select_finish(k_res, k_scale, k_zero, g, T, k, qd, F, ncand, kp, hist, scan_scratch, binfo,
                sel_head + static_cast<size_t>(h) * k);
}

// Block-parallel search of a histogram from the top (all threads call):
// out[0] = the bin holding the kk-th largest element, out[1] = kk minus the
// elements in higher bins.  Thread t sums its own run of bins, an exclusive
// scan gives the count above each run, and the one thread whose run crosses
// kk walks it.
__device__ void find_bin_from_top_block(const int* hist, int nb, int kk, int* out, int* scratch) {
  const int per = (nb + blockDim.x - 1) / blockDim.x;
  const int hi = nb - static_cast<int>(threadIdx.x) * per;  // exclusive upper bin of this run
  const int lo = max(0, hi - per);
  int c = 0;
  for (int b = hi - 1; b >= lo; --b) c += hist[b];
  int tot;
  const int above = sfd::block_exclusive_scan(c, scratch, &tot);
  if (c > 0 && above < kk && above + c >= kk) {
    int a = above;
    for (int b = hi - 1; b >= lo; --b) {
      const int n = hist[b];
      if (a + n >= kk) { out[0] = b; out[1] = kk - a; break; }
      a += n;
    }
  }
  if (threadIdx.x == 0 && tot < kk) { out[0] = 0; out[1] = kk; }
  __syncthreads();
}

// Exact per-head top-k for T <= kRegKeys * kSelThreads with the scores held
// in registers (one coalesced read of the head's scores):
//  1. tau = the k-th largest fast score, by a 3-pass radix select (11, 11 and
//     10 bits of the order-preserving key) over the register-held keys;
//  2. candidates F = {t : score_t >= tau - 2 eps}, compacted in token order
//     straight from the registers (warp w holds the contiguous token range
//     [w seg, (w+1) seg), row i of it at w seg + 32 i + lane);
//  3. exact fp64 keys and ranking as in the streaming kernel.
constexpr int kRegKeys = 32;

template <int GRP>
__global__ void __launch_bounds__(kSelThreads)
attn_select_reg_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                       const uint16_t* __restrict__ k_scale, const uint16_t* __restrict__ k_zero, int T, int k,
                       const float* __restrict__ score, const float* __restrict__ smax, int32_t* __restrict__ cand2,
                       double* __restrict__ kap, int32_t* __restrict__ sel_head, int32_t* __restrict__ status) {
  __shared__ __align__(16) int hist[2048];
  __shared__ double qd[D];
  __shared__ int scan_scratch[64];
  __shared__ int binfo[2];
  __shared__ float red[32];
  __shared__ double l1_sh;
  __shared__ int qe_sh;
  const int h = blockIdx.x, g = h / GRP, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* sc = score + static_cast<size_t>(h) * T;
  int32_t* F = cand2 + static_cast<size_t>(h) * T;
  double* kp = kap + static_cast<size_t>(h) * T;

  const int seg = (((T + 31) >> 5) + 31) & ~31;  // tokens per warp: a multiple of 32, <= 32 kRegKeys
  const int t0 = warp * seg + lane;
  const int tend = min(T, warp * seg + seg);
  uint32_t key[kRegKeys];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < kRegKeys; ++i) {
    const int t = t0 + 32 * i;
    const float v = t < tend ? sc[t] : 0.0f;
    key[i] = okey32(v);
    amax = fmaxf(amax, fabsf(v));
  }
  for (int i = tid; i < 2048; i += kSelThreads) hist[i] = 0;
  select_q_prologue(q, h, g, qd, &l1_sh, &qe_sh, status);  // ends with __syncthreads
  {
    const float m = warp_max(amax);
    if (lane == 0) red[warp] = m;
  }

  // 1. tau by radix select over the registers
#pragma unroll
  for (int i = 0; i < kRegKeys; ++i)
    if (t0 + 32 * i < tend) atomicAdd(&hist[key[i] >> 21], 1);
  __syncthreads();
  find_bin_from_top_block(hist, 2048, k, binfo, scan_scratch);
  const uint32_t b1 = static_cast<uint32_t>(binfo[0]);
  int kk = binfo[1];
  for (int i = tid; i < 2048; i += kSelThreads) hist[i] = 0;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kRegKeys; ++i)
    if (t0 + 32 * i < tend && (key[i] >> 21) == b1) atomicAdd(&hist[(key[i] >> 10) & 2047u], 1);
  __syncthreads();
  find_bin_from_top_block(hist, 2048, kk, binfo, scan_scratch);
  const uint32_t p2 = (b1 << 11) | static_cast<uint32_t>(binfo[0]);
  kk = binfo[1];
  for (int i = tid; i < 1024; i += kSelThreads) hist[i] = 0;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kRegKeys; ++i)
    if (t0 + 32 * i < tend && (key[i] >> 10) == p2) atomicAdd(&hist[key[i] & 1023u], 1);
  __syncthreads();
  find_bin_from_top_block(hist, 1024, kk, binfo, scan_scratch);
  const float tau = from_okey32((p2 << 10) | static_cast<uint32_t>(binfo[0]));
  if (warp == 0) {
    const float mm = warp_max(red[lane]);
    if (lane == 0) red[0] = mm;
  }
  __syncthreads();
  const double eps_s = select_eps(static_cast<double>(smax[g]), l1_sh, qe_sh, red[0]);
  // smallest float f with f >= tau - 2 eps: (double)x >= tau - 2 eps <=> x >= f
  const float fthr = __double2float_ru(static_cast<double>(tau) - 2.0 * eps_s);

  // 2. candidates in token order
  int cnt = 0;
#pragma unroll
  for (int i = 0; i < kRegKeys; ++i)
    cnt += __popc(__ballot_sync(0xffffffffu, t0 + 32 * i < tend && from_okey32(key[i]) >= fthr));
  if (lane == 0) scan_scratch[warp] = cnt;
  __syncthreads();
  if (warp == 0) {
    const int v = scan_scratch[lane];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    scan_scratch[32 + lane] = incl - v;
    if (lane == 31) binfo[0] = incl;
  }
  __syncthreads();
  int off = scan_scratch[32 + warp];
  const int ncand = binfo[0];
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int i = 0; i < kRegKeys; ++i) {
    const bool p = t0 + 32 * i < tend && from_okey32(key[i]) >= fthr;
    const unsigned bal = __ballot_sync(0xffffffffu, p);
    if (p) F[off + __popc(bal & lt)] = t0 + 32 * i;
    off += __popc(bal);
  }
  __syncthreads();

  // 3. exact keys and ranking
  select_finish(k_res, k_scale, k_zero, g, T, k, qd, F, ncand, kp, hist, scan_scratch, binfo,
                sel_head + static_cast<size_t>(h) * k);
}

// ---- pass U: union per KV head ---------------------------------------------
__global__ void __launch_bounds__(1024)
attn_union_kernel(const int32_t* __restrict__ sel_head, int grp, int T, int k, int words_t,
                  uint32_t* __restrict__ umask, int32_t* __restrict__ sel_out, int32_t* __restrict__ sel_n,
                  const int32_t* __restrict__ status) {
  extern __shared__ uint32_t bits[];  // [words_t]
  __shared__ int scan_scratch[33];
  const int g = blockIdx.x, tid = threadIdx.x;
  for (int i = tid; i < words_t; i += blockDim.x) bits[i] = 0;
  __syncthreads();
  for (int e = tid; e < grp * k; e += blockDim.x) {
    const int t = sel_head[static_cast<size_t>(g) * grp * k + e];
    atomicOr(&bits[t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  const int chunk = (words_t + blockDim.x - 1) / blockDim.x;
  const int w0 = min(words_t, tid * chunk), w1 = min(words_t, w0 + chunk);
  int c = 0;
  for (int w = w0; w < w1; ++w) {
    c += __popc(bits[w]);
    umask[static_cast<size_t>(g) * words_t + w] = bits[w];
  }
  int total;
  int pos = sfd::block_exclusive_scan(c, scan_scratch, &total);
  int32_t* out = sel_out + static_cast<size_t>(g) * grp * k;
  for (int w = w0; w < w1; ++w) {
    uint32_t m = bits[w];
    while (m) {
      const int b = __ffs(m) - 1;
      out[pos++] = w * 32 + b;
      m &= m - 1;
    }
  }
  // a group whose query violated the exact-key precondition reports -1 - n
  if (tid == 0) sel_n[g] = status[g] ? -1 - total : total;
}

// ---- refined scores of the refined tokens ------------------------------------
// For every token in a KV group's union, the scores of the group's query heads
// with the full-code key k' = s (4 c_r + c_f - z) replace the resident scores
// in the score buffer (after the selection has used them).  One warp per token,
// lanes over 4 dims each.
template <int GRP>
__global__ void __launch_bounds__(256)
attn_refine_scores_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                          const uint32_t* __restrict__ k_ref, const uint16_t* __restrict__ k_scale,
                          const uint16_t* __restrict__ k_zero, int T, int cap, const int32_t* __restrict__ sel_out,
                          const int32_t* __restrict__ sel_n, float* __restrict__ score) {
  __shared__ float qs[GRP][D];
  __shared__ float qsum[GRP];
  const int g = blockIdx.y;
  load_q<GRP>(q, g, qs, qsum);
  int n = sel_n[g];
  n = n >= 0 ? n : -1 - n;
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  for (int i = gw; i < n; i += nwarps) {
    const int t = sel_out[static_cast<size_t>(g) * cap + i];
    const size_t row = static_cast<size_t>(g) * T + t;
    const uint32_t wr = k_res[row * kWordsPerRow + (lane >> 2)] >> ((lane & 3) * 8);
    const uint32_t wf = k_ref[row * kWordsPerRow + (lane >> 2)] >> ((lane & 3) * 8);
    float P[GRP];
#pragma unroll
    for (int h = 0; h < GRP; ++h) P[h] = 0.0f;
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) {
      const float c = static_cast<float>(((wr >> (2 * dd)) & 3u) * 4u + ((wf >> (2 * dd)) & 3u));
#pragma unroll
      for (int h = 0; h < GRP; ++h) P[h] = fmaf(qs[h][4 * lane + dd], c, P[h]);
    }
    const float sv = sfd::half_bits_to_float(k_scale[row]);
    const float z = sfd::half_bits_to_float(k_zero[row]);
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const float Ph = warp_sum(P[h]);
      if (lane == 0) score[(static_cast<size_t>(g) * GRP + h) * T + t] = (sv * fmaf(-z, qsum[h], Ph)) * kInvSqrtD;
    }
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
// kSub tokens: the sub-chunk's score maximum per head is found first, so every
// weight is computed once, by one thread, relative to a fixed maximum and
// stored in shared memory (no per-tile online rescaling); the warps then run
// the MMAs over their tiles of 16 tokens, the codes staged by cp.async.
__device__ __forceinline__ void mma_f16f32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

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
  static constexpr size_t wo_bytes = static_cast<size_t>(GRP) * D * 4;
  static constexpr size_t ulist_bytes = static_cast<size_t>(kSub) * 4;
  static constexpr size_t vref_bytes = static_cast<size_t>(kUCap) * kWordsPerRow * 4;
  static constexpr size_t smem = alpha_bytes + ring_bytes + wo_bytes + ulist_bytes + vref_bytes;
  static_assert(alpha_bytes >= static_cast<size_t>(GRP) * kMaxSplits * 4, "merge factors must fit the weight tile");
};

template <int GRP>
__global__ void __launch_bounds__(kOutThreads)
attn_out_kernel(const uint32_t* __restrict__ v_res, const uint32_t* __restrict__ v_ref,
                const uint16_t* __restrict__ v_scale, const uint16_t* __restrict__ v_zero, int T, int tps, int words_t,
                int splits, const float* __restrict__ score, const uint32_t* __restrict__ umask,
                float* __restrict__ part, int32_t* __restrict__ done, float* __restrict__ out) {
  using C = OutCfg<GRP>;
  constexpr int NT = C::NT, kStr = C::kStr;
  extern __shared__ __align__(16) unsigned char smem[];
  __half* as = reinterpret_cast<__half*>(smem);                                      // [NT*8][kStr]
  uint32_t* ring = reinterpret_cast<uint32_t*>(smem + C::alpha_bytes);               // [kOW][kRing][16][8]
  float* wo = reinterpret_cast<float*>(smem + C::alpha_bytes + C::ring_bytes);       // [GRP][D]
  int* ulist = reinterpret_cast<int*>(smem + C::alpha_bytes + C::ring_bytes + C::wo_bytes);  // [kSub]
  uint32_t* vrs = reinterpret_cast<uint32_t*>(smem + C::alpha_bytes + C::ring_bytes + C::wo_bytes +
                                              C::ulist_bytes);  // [kUCap][8] refinement rows of listed tokens
  __shared__ float red[kOW][GRP];
  __shared__ float red2[kOW][3 * GRP];
  __shared__ float Msh[GRP], Fsh[GRP];
  __shared__ int ucount;

  const int g = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g8 = lane >> 2, tig = lane & 3;
  const int t0s = split * tps, t1s = min(T, t0s + tps);
  const size_t rowg = static_cast<size_t>(g) * T;

  for (int e = tid; e < (NT * 8 - C::NC) * kStr; e += kOutThreads) as[C::NC * kStr + e] = __float2half_rn(0.0f);
  for (int e = tid; e < GRP * D; e += kOutThreads) wo[e] = 0.0f;
  if (tid < GRP) Msh[tid] = -INFINITY;

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

    // 1. the sub-chunk's maximum score per head; this thread's tokens'
    //    scale, zero and union bit are fetched meanwhile
    uint32_t svz[kPerThr];
    uint32_t ubits = 0;
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
          const int t = c0 + i;
          ubits |= ((umask[static_cast<size_t>(g) * words_t + (t >> 5)] >> (t & 31)) & 1u) << j;
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
      if (tid == 0) ucount = 0;
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

    // 2. weights into shared memory (zero past the end of the last tile),
    //    sums, and the list of refined tokens
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < kPerThr; ++j) {
      const int i = tid + j * kOutThreads;
      if (j * kOutThreads >= 16 * ntile) break;  // uniform over the block
      const bool valid = i < n;
      bool inU = false;
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
          inU = (ubits >> j) & 1u;
        } else {
#pragma unroll
          for (int h = 0; h < 2 * GRP; ++h) as[h * kStr + i] = __float2half_rn(0.0f);
        }
      }
      const unsigned b = __ballot_sync(0xffffffffu, inU);
      if (b) {
        int pos = 0;
        if (lane == __ffs(b) - 1) pos = atomicAdd(&ucount, __popc(b));
        pos = __shfl_sync(0xffffffffu, pos, __ffs(b) - 1);
        if (inU) ulist[pos + __popc(b & lt)] = i;
      }
    }
    __syncthreads();
    // refinement rows of the listed tokens, staged behind the MMA loop
    const int nu = ucount;
    for (int u = tid; u < min(nu, kUCap); u += kOutThreads) {
      const uint32_t* src = v_ref + (rowg + c0 + ulist[u]) * kWordsPerRow;
      cp_async16_attn(vrs + u * kWordsPerRow, src);
      cp_async16_attn(vrs + u * kWordsPerRow + 4, src + 4);
    }
    cp_async_commit_attn();

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

  // high + remainder columns and the refined corrections into wo[head][dim]
  // (in units of the code part: uo enters divided by 2^b_f = 4)
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int w = 0; w < 8; ++w)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int hh = colh[nt][c & 1];
        if (hh >= 0) atomicAdd(&wo[hh * D + 16 * w + g8 + 8 * (c >> 1)], acc[nt][w][c]);
      }
#pragma unroll
  for (int h = 0; h < GRP; ++h)
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) atomicAdd(&wo[h * D + 4 * lane + dd], 0.25f * uo[h][dd]);
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
      v = j == 1 ? L : fmaf(4.0f, wo[h * D + j - 2], fmaf(-4096.0f, A, Cs));
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
  for (int e = tid; e < GRP * D; e += kOutThreads) {
    const int h = e / D, d = e % D;
    const float* ph = pg + static_cast<size_t>(h) * splits * (D + 2) + 2 + d;
    float O0 = 0.0f, O1 = 0.0f, O2 = 0.0f, O3 = 0.0f;
    int sp = 0;
    for (; sp + 3 < splits; sp += 4) {
      O0 = fmaf(fct[h][sp], __ldcg(ph + sp * (D + 2)), O0);
      O1 = fmaf(fct[h][sp + 1], __ldcg(ph + (sp + 1) * (D + 2)), O1);
      O2 = fmaf(fct[h][sp + 2], __ldcg(ph + (sp + 2) * (D + 2)), O2);
      O3 = fmaf(fct[h][sp + 3], __ldcg(ph + (sp + 3) * (D + 2)), O3);
    }
    for (; sp < splits; ++sp) O0 = fmaf(fct[h][sp], __ldcg(ph + sp * (D + 2)), O0);
    out[(static_cast<size_t>(g) * GRP + h) * D + d] = ((O0 + O1) + (O2 + O3)) / Lh[h];
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
  attn_score_mma_kernel<GRP><<<ga, 128, 0, s>>>(q, kv->k_res, kv->k_scale, kv->k_zero, T, score, smax);
  sf_status st = sf::check_launch("attn_score_mma_kernel");
  if (st != SF_OK) return st;
  const int cap = grp * k;  // row length of sel_out
  if (k > 0 && k < T) {
    if (T <= kRegKeys * kSelThreads) {
      attn_select_reg_kernel<GRP><<<Hq, kSelThreads, 0, s>>>(q, kv->k_res, kv->k_scale, kv->k_zero, T, k, score,
                                                             smax, cand2, kap, sel_head, status);
      st = sf::check_launch("attn_select_reg_kernel");
    } else {
      attn_select_kernel<GRP><<<Hq, kSelThreads, 0, s>>>(q, kv->k_res, kv->k_scale, kv->k_zero, T, k, score, smax,
                                                         cand, cand2, kap, sel_head, status);
      st = sf::check_launch("attn_select_kernel");
    }
    if (st != SF_OK) return st;
    const size_t smem = sizeof(uint32_t) * L.words_t;
    SF_CHECK_CUDA(cudaFuncSetAttribute(attn_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(std::max<size_t>(smem, 1))));
    attn_union_kernel<<<Hkv, 1024, smem, s>>>(sel_head, grp, T, k, L.words_t, umask, sel_out, sel_n, status);
    st = sf::check_launch("attn_union_kernel");
    if (st != SF_OK) return st;
  } else if (k == 0) {
    SF_CHECK_CUDA(cudaMemsetAsync(umask, 0, sizeof(uint32_t) * Hkv * static_cast<size_t>(L.words_t), s));
    SF_CHECK_CUDA(cudaMemsetAsync(sel_n, 0, sizeof(int32_t) * Hkv, s));
  } else {
    fill_all_kernel<<<dim3(32, Hkv), 256, 0, s>>>(T, grp, k, L.words_t, umask, sel_out, sel_n);
    st = sf::check_launch("fill_all_kernel");
    if (st != SF_OK) return st;
  }
  if (k > 0) {
    dim3 gr(std::max(1, std::min((cap + 7) / 8, 128)), Hkv);
    attn_refine_scores_kernel<GRP><<<gr, 256, 0, s>>>(q, kv->k_res, kv->k_ref, kv->k_scale, kv->k_zero, T, cap,
                                                      sel_out, sel_n, score);
    st = sf::check_launch("attn_refine_scores_kernel");
    if (st != SF_OK) return st;
  }
  dim3 gb(L.splits, Hkv);
  SF_CHECK_CUDA(cudaFuncSetAttribute(attn_out_kernel<GRP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(OutCfg<GRP>::smem)));
  attn_out_kernel<GRP><<<gb, kOutThreads, OutCfg<GRP>::smem, s>>>(kv->v_res, kv->v_ref, kv->v_scale, kv->v_zero, T,
                                                                 L.tps, L.words_t, L.splits, score, umask, part,
                                                                 done, out);
  return sf::check_launch("attn_out_kernel");
}

}  // namespace

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
  cudaStream_t s = sf::as_cuda(stream);
  char* ws = static_cast<char*>(workspace);
  switch (Hq / Hkv) {
    case 1: return run<1>(q, Hq, Hkv, T, kv, k_tokens, sel_out, sel_n, out, ws, L, s);
    case 2: return run<2>(q, Hq, Hkv, T, kv, k_tokens, sel_out, sel_n, out, ws, L, s);
    case 4: return run<4>(q, Hq, Hkv, T, kv, k_tokens, sel_out, sel_n, out, ws, L, s);
    case 8: return run<8>(q, Hq, Hkv, T, kv, k_tokens, sel_out, sel_n, out, ws, L, s);
    default: return sf::fail(SF_ENOTIMPL, "sf_attn_decode_refine: Hq/Hkv must be 1, 2, 4 or 8");
  }
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
  cudaStream_t s = sf::as_cuda(stream);
  char* w = static_cast<char*>(ws);
  switch (Hq / Hkv) {
    case 1: return run<1>(q, Hq, Hkv, T, kv, k_tokens, sel_out, sel_n, out, w, L, s);
    case 2: return run<2>(q, Hq, Hkv, T, kv, k_tokens, sel_out, sel_n, out, w, L, s);
    case 4: return run<4>(q, Hq, Hkv, T, kv, k_tokens, sel_out, sel_n, out, w, L, s);
    case 8: return run<8>(q, Hq, Hkv, T, kv, k_tokens, sel_out, sel_n, out, w, L, s);
    default: return sf::fail(SF_ENOTIMPL, "sf_attn_decode_refine_noalloc: Hq/Hkv must be 1, 2, 4 or 8");
  }
}
