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
//              asc).  So the chosen set equals the exact definition.  One
//              cluster per KV group, one CTA per query head, which also forms
//              the group's union (ascending list and token bitmask) and runs
//              step R on it.
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
  pdl_launch_dependents();  // the listing pass may launch; it waits for this grid
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
  pdl_wait();  // the cleared counters (everything read above was final before the clear began)
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

// ---- pass S, listing: the tokens of each head with fast score >= f_low ----------
//
// Per (8192-token chunk, query head), after the head's band from the score
// pass's histogram and maxima (the bin b1 of the k-th largest fast score and
// f_low = lower(b1) - 2 eps; the CTA of chunk 0 records it for the ranking):
// a warp ballots 32 consecutive tokens a row; one atomic per CTA takes the
// chunk's run of the head's list (the list's order does not matter: the
// ranking orders by key and token).  The q terms of eps come first: they need
// no earlier pass.

constexpr int kCompThreads = 256;
constexpr int kChunk = 8192;
constexpr int kCompRows = kChunk / kCompThreads;  // rows of 32 tokens per warp

__global__ void __launch_bounds__(kCompThreads)
attn_compact_kernel(const uint16_t* __restrict__ q, int T, int k, const float* __restrict__ score,
                    const float* __restrict__ smax, const int32_t* __restrict__ hist,
                    const uint32_t* __restrict__ amaxu, SelBand* __restrict__ band, int32_t* __restrict__ cand,
                    int32_t* __restrict__ ccnt, int32_t* __restrict__ status, int grp) {
  const int chunk = blockIdx.x, h = blockIdx.y, g = h / grp;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ int hsh[kHistBins];
  __shared__ int scan_scratch[64];
  __shared__ int binfo[2];
  __shared__ double qd[D];
  __shared__ double l1_sh, dq_sh;
  __shared__ int qe_sh;
  __shared__ int wcnt[kCompThreads / 32], woff[kCompThreads / 32];
  __shared__ int base_sh;
  pdl_launch_dependents();
  select_q_prologue(q, h, g, qd, &l1_sh, &qe_sh, status, nullptr, kScQFrac, &dq_sh);
  pdl_wait();  // the score pass's scores, histogram and maxima
  // the head's histogram, every load in flight
  {
    constexpr int kPer = kHistBins / kCompThreads;
    const int32_t* hg = hist + static_cast<size_t>(h) * kHistBins;
    int hv[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) hv[j] = hg[tid + j * kCompThreads];
#pragma unroll
    for (int j = 0; j < kPer; ++j) hsh[tid + j * kCompThreads] = hv[j];
  }
  // the chunk's scores are loaded while the band is found
  const int t0 = chunk * kChunk + warp * 32 * kCompRows + lane;
  const float* sc = score + static_cast<size_t>(h) * T;
  float v[kCompRows];
#pragma unroll
  for (int i = 0; i < kCompRows; ++i) {
    const int t = t0 + 32 * i;
    v[i] = t < T ? sc[t] : 0.0f;
  }
  const int Hkv = gridDim.y / grp;
  const double eps_s = select_eps_pipe(static_cast<double>(smax[g]), static_cast<double>(smax[Hkv + g]), l1_sh,
                                       dq_sh, __uint_as_float(amaxu[h]));
  __syncthreads();
  find_bin_from_top_block(hsh, kHistBins, k, binfo, scan_scratch);
  const uint32_t b1 = static_cast<uint32_t>(binfo[0]);
  const float f_low = __double2float_rd(static_cast<double>(from_okey32(b1 << kHistShift)) - 2.0 * eps_s);
  if (chunk == 0 && tid == 0) band[h] = SelBand{eps_s, f_low, b1, binfo[1], 0};
  bool p[kCompRows];
  int cnt = 0;
#pragma unroll
  for (int i = 0; i < kCompRows; ++i) {
    p[i] = t0 + 32 * i < T && v[i] >= f_low;
    cnt += __popc(__ballot_sync(0xffffffffu, p[i]));
  }
  if (lane == 0) wcnt[warp] = cnt;
  __syncthreads();
  if (tid == 0) {
    int a = 0;
    for (int w = 0; w < kCompThreads / 32; ++w) {
      woff[w] = a;
      a += wcnt[w];
    }
    base_sh = a ? atomicAdd(ccnt + h, a) : 0;
  }
  __syncthreads();
  int32_t* out = cand + static_cast<size_t>(h) * T + base_sh;
  int o = woff[warp];
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int i = 0; i < kCompRows; ++i) {
    const unsigned bal = __ballot_sync(0xffffffffu, p[i]);
    if (p[i]) out[o + __popc(bal & lt)] = t0 + 32 * i;
    o += __popc(bal);
  }
}

// ---- refined scores of the union --------------------------------------------------
//
// Step R, at the start of pass B: every union token of a CTA's range gets its
// scores for the group's query heads recomputed from the full 4-bit key
// codes, in place in the score buffer.  The CTA then weights its tokens
// against one maximum per head (the larger of its refined maximum and a
// bound on the resident scores outside the union), so it needs no maximum
// pass; the merge rescales the ranges' partials.  A thread handles one union
// token for all the heads of the group: one load of each of the token's two
// code rows.

// A unit of a KV refinement cache: the token-head's 8 K refinement words,
// then its 8 V refinement words.
constexpr int kCacheUnitWords = 2 * kWordsPerRow;

// The V refinement words of K/V row `row`: from the store (uslot == nullptr)
// or from the cache slot that holds the row's unit.
__device__ __forceinline__ const uint32_t* vref_row(const uint32_t* v_ref, const int32_t* uslot, size_t row) {
  return uslot != nullptr ? v_ref + static_cast<size_t>(uslot[row]) * kCacheUnitWords + kWordsPerRow
                          : v_ref + row * kWordsPerRow;
}

// Refines union token t of group g (row = g S + t).  Returns false when its
// refinement bits are not on the device (a cache slot < 0): the token keeps
// its resident key and value this step and leaves the refined set, and its
// resident scores still bound the weights' maximum.  mk[h] takes the max of
// the token's (refined or resident) score keys.
template <int GRP>
__device__ __forceinline__ bool refine_token(const uint32_t* __restrict__ k_res, const uint32_t* __restrict__ k_ref,
                                             const int32_t* __restrict__ uslot, const uint16_t* __restrict__ k_scale,
                                             const uint16_t* __restrict__ k_zero, int T, size_t rowg, int g, int t,
                                             const float (&qs)[GRP][D], const float (&qsum)[GRP],
                                             float* __restrict__ score, uint32_t (&mk)[GRP]) {
  const size_t row = rowg + t;
  const int slot = uslot != nullptr ? uslot[row] : 0;
  float* srow = score + static_cast<size_t>(g) * GRP * T + t;  // head h at srow[h T]
  if (slot < 0) {
#pragma unroll
    for (int h = 0; h < GRP; ++h) mk[h] = max(mk[h], okey32(srow[static_cast<size_t>(h) * T]));
    return false;
  }
  const uint4* pr = reinterpret_cast<const uint4*>(k_res + row * kWordsPerRow);
  const uint4* pf = reinterpret_cast<const uint4*>(
      uslot != nullptr ? k_ref + static_cast<size_t>(slot) * kCacheUnitWords : k_ref + row * kWordsPerRow);
  const uint4 r0 = pr[0], r1 = pr[1], f0 = pf[0], f1 = pf[1];  // both rows in flight at once
  const float sv = sfd::half_bits_to_float(k_scale[row]);
  const float z = sfd::half_bits_to_float(k_zero[row]);
  uint32_t wr[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
  uint32_t wf[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
  float P[GRP];
#pragma unroll
  for (int h = 0; h < GRP; ++h) P[h] = 0.0f;
  // one word per iteration, the words shifted down (static register indices)
#pragma unroll 1
  for (int w = 0; w < 8; ++w) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float c = static_cast<float>(((wr[0] >> (2 * j)) & 3u) * 4u + ((wf[0] >> (2 * j)) & 3u));
#pragma unroll
      for (int h = 0; h < GRP; ++h) P[h] = fmaf(qs[h][16 * w + j], c, P[h]);
    }
#pragma unroll
    for (int i = 0; i < 7; ++i) {
      wr[i] = wr[i + 1];
      wf[i] = wf[i + 1];
    }
  }
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    const float val = (sv * fmaf(-z, qsum[h], P[h])) * kInvSqrtD;
    mk[h] = max(mk[h], okey32(val));
    srow[static_cast<size_t>(h) * T] = val;
  }
  return true;
}

// ---- pass S, ranking: one cluster per KV group, one CTA per query head ----------
//
// The score pass left, per query head, its selection band (the histogram bin
// b1 of the k-th largest fast score and a lower bound f_low of every fast
// score that can reach the top k) and the listing pass the head's tokens with
// fast score >= f_low.  Every token whose exact key can reach the top k has a
// fast score >= tau - 2 eps >= f_low.  Per head:
//  1  the list and its scores into shared memory (beyond kSelList: read in
//     place);
//  2  tau exactly by two more radix passes over the listed scores of b1;
//  3  the tokens above tau + 2 eps selected outright; the band [tau - 2 eps,
//     tau + 2 eps] re-keyed exactly in fp64 and ranked (key desc, token asc);
//  4  the selection marked in the group's token bitmask, whose words are
//     spread over the cluster's shared memory, then the union listed in
//     ascending order (CTA r the words of its range) and the bitmask written
//     for pass B.

constexpr int kSelThreads = 512;
constexpr int kSelKeys = 2048;      // band entries ranked pairwise in shared memory
constexpr int kSelList = 4096;      // listed (token, score) pairs in shared memory
constexpr int kSelMaxWords = 8192;  // bitmask words per CTA held in shared memory (beyond: global atomics)

__host__ __device__ constexpr size_t sel_dyn_smem(int words_sm) {
  return static_cast<size_t>(kSelList) * 8 + static_cast<size_t>(kSelKeys) * 4 + static_cast<size_t>(words_sm) * 4;
}

template <int GRP>
__global__ void __launch_bounds__(kSelThreads)
attn_select_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                   const uint16_t* __restrict__ k_scale, const uint16_t* __restrict__ k_zero, int T, int k, int S,
                   const float* __restrict__ score, const SelBand* __restrict__ band, const int32_t* __restrict__ cand,
                   const int32_t* __restrict__ ccnt, int32_t* __restrict__ list, double* __restrict__ kap,
                   int32_t* __restrict__ sel_head, uint32_t* __restrict__ umask, int words_t, int wper, int dsm,
                   int32_t* __restrict__ sel_out, int32_t* __restrict__ sel_n, int32_t* __restrict__ status,
                   uint32_t* __restrict__ mkey) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = static_cast<int>(cl.block_rank());
  const int h = blockIdx.x, g = h / GRP;
  const int tid = threadIdx.x, lane = tid & 31;
  __shared__ int hr[2048];
  __shared__ unsigned long long keys[kSelKeys];  // order-preserving exact keys, sorted with the tokens
  __shared__ double qd[D];
  __shared__ int scan_scratch[64];
  __shared__ int binfo[2];
  __shared__ double l1_sh;
  __shared__ int qe_sh, span_sh;
  __shared__ int cnt_sh;  // read remotely
  __shared__ int cntA_sh, cntB_sh;  // outright selections and band candidates
  __shared__ uint32_t qpl[3][8][4];  // byte planes of the fixed-point q, in code-extraction order
  __shared__ long long qxsum_sh;
  extern __shared__ __align__(16) int sel_dyn[];
  int* ltok = sel_dyn;                                       // [kSelList]
  float* lsc = reinterpret_cast<float*>(sel_dyn + kSelList);  // [kSelList]
  int* ktok = sel_dyn + 2 * kSelList;                        // [kSelKeys] tokens of the sorted keys
  uint32_t* wsm = reinterpret_cast<uint32_t*>(ktok + kSelKeys);  // [wper] bitmask words of this CTA's range
  const float* sc = score + static_cast<size_t>(h) * T;
  const int32_t* Lg = cand + static_cast<size_t>(h) * T;  // the listing pass's tokens
  int32_t* F = list + static_cast<size_t>(h) * T;         // band candidates beyond kSelKeys
  double* kp = kap + static_cast<size_t>(h) * T;
  uint32_t* um_g = umask + static_cast<size_t>(g) * words_t;
  const int cap = GRP * k;
  const int w0 = min(words_t, rank * wper), w1 = min(words_t, w0 + wper);

  if (tid == 0) cntA_sh = cntB_sh = 0;
  if (dsm)
    for (int w = tid; w < wper; w += kSelThreads) wsm[w] = 0u;
  select_q_prologue(q, h, g, qd, &l1_sh, &qe_sh, status, &span_sh);  // contains __syncthreads
  pdl_wait();  // the listing pass, and through it the score pass
  const SelBand bd = band[h];
  const double eps_s = bd.eps;
  int kk = bd.kk;
  const int m = min(ccnt[h], T);
  // 1. the list with its fast scores: each thread's tokens, then their
  //    scores, every load of a round in flight
  {
    constexpr int kPer = kSelList / kSelThreads;
    const int mm = min(m, kSelList);
    int tv[kPer];
    float sv[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int e = tid + j * kSelThreads;
      tv[j] = e < mm ? Lg[e] : 0;
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int e = tid + j * kSelThreads;
      sv[j] = e < mm ? sc[tv[j]] : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int e = tid + j * kSelThreads;
      if (e < mm) {
        ltok[e] = tv[j];
        lsc[e] = sv[j];
      }
    }
  }
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
    if (tid >= 96 && tid < 128) {
      long long sx = 0;
      for (int d = tid - 96; d < D; d += 32) sx += static_cast<long long>(ldexp(qd[d], 23 - qe_sh));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sx += __shfl_xor_sync(0xffffffffu, sx, o);
      if (tid == 96) qxsum_sh = sx;
    }
  }
  cl.sync();  // 0: every CTA's bitmask words are cleared before any remote update
  auto tok_of = [&](int e) { return e < kSelList ? ltok[e] : Lg[e]; };
  auto score_of = [&](int e) { return e < kSelList ? lsc[e] : sc[Lg[e]]; };
  const unsigned lt = (1u << lane) - 1u;

  // 2. tau: two radix passes (11 + 10 bits) over the listed scores of bin b1
  uint32_t pre = bd.b1 << kHistShift;
  static_assert(kHistShift == 21, "the two passes cover the 21 key bits below the histogram's");
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? 10 : 0;
    const int nb = pass == 0 ? 2048 : 1024;
    for (int i = tid; i < nb; i += kSelThreads) hr[i] = 0;
    __syncthreads();
    const uint32_t pmask = pass == 0 ? 0xFFE00000u : 0xFFFFFC00u;
    for (int e = tid; e < m; e += kSelThreads) {
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

  // the group's token bitmask: words [r wper, (r + 1) wper) in CTA r's shared
  // memory, or the global words
  auto mark = [&](int t) {
    const int w = t >> 5;
    const uint32_t bit = 1u << (t & 31);
    if (dsm) {
      const int r = w / wper;
      atomicOr(cl.map_shared_rank(wsm, r) + (w - r * wper), bit);
    } else {
      atomicOr(um_g + w, bit);
    }
  };

  // 3. a token whose fast score exceeds tau + 2 eps outranks, by exact key,
  //    every token with fast score <= tau, so fewer than k tokens can rank
  //    above it: it is selected outright.  Only the band [tau - 2 eps,
  //    tau + 2 eps] is re-keyed and ranked.
  int32_t* sel = sel_head + static_cast<size_t>(h) * k;
  const double hi_band = static_cast<double>(tau) + 2.0 * eps_s;
  for (int base = 0; base < m; base += kSelThreads) {  // uniform over the block
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
      mark(t);
    }
    if (inB) {
      const int pB = oB + __popc(bB & lt);
      if (pB < kSelKeys) ktok[pB] = t;
      F[pB] = t;
    }
  }
  __syncthreads();
  const int nA = cntA_sh, ncand = cntB_sh;
  const int kB = max(0, k - nA);  // winners still to pick from the band (>= 1 by the bound)

  // 4. exact keys (exact under the precondition, so the summation order does
  //    not change the key)
  for (int i = tid; i < ncand; i += kSelThreads) {
    const int t = i < kSelKeys ? ktok[i] : F[i];
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
      const double qsm = ldexp(static_cast<double>(qxsum_sh), qe_sh - 23);
      key = sv * fma(1.5 - z, qsm, 4.0 * cq);
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
    if (i < kSelKeys) keys[i] = okey64(key);
  }
  __syncthreads();

  // rank the band by (key desc, token asc); its kB winners go to sel_head
  // after the outright ones, and into the bitmask
  if (ncand <= kSelKeys) {
    // bitonic sort of (key desc, token asc) over a power-of-two size,
    // padding with entries that order last; the first kB are the winners
    int n2 = 1;
    while (n2 < ncand) n2 <<= 1;
    for (int i = ncand + tid; i < n2; i += kSelThreads) {
      keys[i] = 0ull;
      ktok[i] = 0x7FFFFFFF;
    }
    __syncthreads();
    for (int size = 2; size <= n2; size <<= 1)
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < (n2 >> 1); i += kSelThreads) {
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
    for (int r = tid; r < kB; r += kSelThreads) {
      const int t = ktok[r];
      sel[nA + r] = t;
      mark(t);
    }
  } else {
    select_rank_radix(F, ncand, kp, kB, hr, scan_scratch, binfo, sel + nA);
    __syncthreads();
    for (int i = tid; i < kB; i += kSelThreads) mark(sel[nA + i]);
  }
  if (!dsm) __threadfence();
  pdl_launch_dependents();  // pass B's CTAs may start their prologue during the union
  cl.sync();  // 1: the group's bitmask is complete

  // 5. union, ascending: CTA r lists the tokens of words [w0, w1)
  auto word = [&](int w) -> uint32_t { return dsm ? wsm[w - w0] : __ldcg(um_g + w); };
  int32_t* uout = sel_out + static_cast<size_t>(g) * cap;
  {
    int off = 0, uloc = 0;
    const int chunk = (w1 - w0 + kSelThreads - 1) / kSelThreads;
    const int a0 = min(w1, w0 + tid * chunk), a1 = min(w1, a0 + chunk);
    int c = 0;
    for (int w = a0; w < a1; ++w) c += __popc(word(w));
    int pos = sfd::block_exclusive_scan(c, scan_scratch, &uloc);
    if (tid == 0) cnt_sh = uloc;
    cl.sync();  // 2: every CTA's count is published
    int U = 0;
    for (int r = 0; r < GRP; ++r) {
      const int cr = *cl.map_shared_rank(&cnt_sh, r);
      if (r < rank) off += cr;
      U += cr;
    }
    cl.barrier_arrive();  // 3 (arrive): no remote shared-memory access by this CTA after this
    for (int w = a0; w < a1; ++w) {
      uint32_t bits = word(w);
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1u;
        const int t = 32 * w + b;
        uout[off + pos] = t;
        ++pos;
      }
    }
    if (rank == 0 && tid == 0) sel_n[g] = status[g] ? -1 - U : U;
  }
  if (dsm) {
    __syncthreads();
    for (int w = w0 + tid; w < w1; w += kSelThreads) um_g[w] = wsm[w - w0];
  }
  cl.barrier_wait();  // 3 (wait): no CTA leaves while another may read its count
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
constexpr int kUMiss = 0x8000;     // union-list flag: refinement bits not on the device
constexpr int kUOff = 0x7FFF;      // union-list offset bits

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
  static_assert(alpha_bytes >= static_cast<size_t>(kOW) * 16 * 8 * NT * 8 * 4, "per-warp output tiles must fit the weight tile");
  static_assert(kSub / 32 <= kOutThreads, "the union scan takes a bitmask word per thread");
};

template <int GRP>
__global__ void __launch_bounds__(kOutThreads, GRP >= 8 ? 1 : 2)
attn_out_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                const uint32_t* __restrict__ k_ref, const uint16_t* __restrict__ k_scale,
                const uint16_t* __restrict__ k_zero, const uint32_t* __restrict__ v_res,
                const uint32_t* __restrict__ v_ref, const int32_t* __restrict__ uslot,
                const uint16_t* __restrict__ v_scale,
                const uint16_t* __restrict__ v_zero, int T, int S, int tps, int words_t, int splits,
                float* __restrict__ score, const uint32_t* __restrict__ mkey,
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
  __shared__ uint32_t mkr_sh[GRP];
  __shared__ int ucount;
  __shared__ int uscan[33];
  __shared__ float qsum[GRP];
  // the group's query heads for step R, in the weight tile (written later)
  float (&qs)[GRP][D] = *reinterpret_cast<float (*)[GRP][D]>(smem);

  const int g = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g8 = lane >> 2, tig = lane & 3;
  const int t0s = split * tps, t1s = min(T, t0s + tps);
  const size_t rowg = static_cast<size_t>(g) * S;  // V rows: the cache's stride

  for (int e = tid; e < (NT * 8 - C::NC) * kStr; e += kOutThreads) as[C::NC * kStr + e] = __float2half_rn(0.0f);
  // a warp's value-code stream of a sub-chunk: 16-token tiles through its
  // ring of kRing cp.async stages (the stage of tile ti is (ti - tile0) mod kRing)
  auto issue_st = [&](int c0, int n, int ti, int st) {
    const int tok = 16 * ti + (lane >> 1);
    if (tok < n)
      cp_async16_attn(ring + ((warp * kRing + st) * 16 + (lane >> 1)) * kWordsPerRow + (lane & 1) * 4,
                      v_res + (rowg + c0 + tok) * kWordsPerRow + (lane & 1) * 4);
  };
  auto issue_at = [&](int c0, int n, int tile0, int ti) { issue_st(c0, n, ti, (ti - tile0) % kRing); };
  auto start_stream = [&](int c0) {
    const int n = min(t1s, c0 + kSub) - c0;
    const int ntile = (n + 15) >> 4;
    const int tpw = (ntile + kOW - 1) / kOW;
    const int tile0 = min(ntile, warp * tpw), tile1 = min(ntile, tile0 + tpw);
    for (int i = 0; i < kRing - 1; ++i) {
      if (tile0 + i < tile1) issue_at(c0, n, tile0, tile0 + i);
      cp_async_commit_attn();
    }
  };
  start_stream(t0s);  // the value codes are inputs: no earlier pass writes them
  if (tid < GRP) mkr_sh[tid] = 0u;
  load_q<GRP>(q, g, qs, qsum);  // contains __syncthreads
  pdl_wait();  // the selection (and every pass before it)

  // the sub-chunk's union tokens (ascending offsets) from the group's bitmask;
  // a token whose refinement bits are not on the device (a cache slot < 0)
  // is flagged kUMiss: it keeps its resident key and value this step
  auto list_union = [&](int c0, int n) {
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
      const int i = 32 * tid + b;
      const bool miss = uslot != nullptr && uslot[rowg + c0 + i] < 0;
      ulist[pos++] = static_cast<uint16_t>(i | (miss ? kUMiss : 0));
    }
    if (tid == 0) ucount = tot;
    __syncthreads();
  };


  // R. the range's union tokens get their refined scores before any weight
  //    is formed: the CTA's maximum per head covers them
  {
    uint32_t mk[GRP];
#pragma unroll
    for (int h = 0; h < GRP; ++h) mk[h] = 0u;
    for (int c0 = t0s; c0 < t1s; c0 += kSub) {
      list_union(c0, min(t1s, c0 + kSub) - c0);
      for (int u = tid; u < ucount; u += kOutThreads)
        refine_token<GRP>(k_res, k_ref, uslot, k_scale, k_zero, T, rowg, g, c0 + (ulist[u] & kUOff), qs, qsum, score,
                          mk);
      __syncthreads();  // the list is rebuilt for the next sub-chunk
    }
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mk[h] = max(mk[h], __shfl_xor_sync(0xffffffffu, mk[h], o));
      if (lane == 0 && mk[h]) atomicMax(&mkr_sh[h], mk[h]);
    }
    __syncthreads();
  }
  // this CTA's maximum per head for every token of its range: the larger of
  // the bound on the resident scores outside the union and the union's
  // (refined or resident) maximum in the range (a key of 0: no such token)
  if (tid < GRP) {
    const uint32_t mk = mkey[g * GRP + tid], rk = mkr_sh[tid];
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
  for (int c0 = t0s; c0 < t1s; c0 += kSub) {
    const int n = min(t1s, c0 + kSub) - c0;
    const int ntile = (n + 15) >> 4;
    const int tpw = (ntile + kOW - 1) / kOW;
    const int tile0 = min(ntile, warp * tpw), tile1 = min(ntile, tile0 + tpw);
    // start the code stream while the weights are being computed (the first
    // sub-chunk's started before step R)
    if (c0 != t0s) start_stream(c0);

    // 0. the sub-chunk's union tokens (the list of step R when the range is
    //    one sub-chunk); the value refinement rows of the refined ones are
    //    staged for step 3
    if (t1s - t0s > kSub) list_union(c0, n);
    const int nu = ucount;
    for (int u = tid; u < min(nu, kUCap); u += kOutThreads) {
      const int e = ulist[u];
      if (e & kUMiss) continue;
      const uint32_t* src = vref_row(v_ref, uslot, rowg + c0 + e);
      cp_async16_attn(vrs + u * kWordsPerRow, src);
      cp_async16_attn(vrs + u * kWordsPerRow + 4, src + 4);
    }
    cp_async_commit_attn();
    float M[GRP];
#pragma unroll
    for (int h = 0; h < GRP; ++h) M[h] = Msh[h];

    // 1. weights into shared memory (zero past the end of the last tile) and
    //    sums; the scores, scales and zeros of kWB of this thread's tokens
    //    are loaded before any is used
    constexpr int kWB = GRP >= 4 ? 4 : 8;
    static_assert(kPerThr % kWB == 0, "whole batches of tokens in the weight pass");
#pragma unroll 1
    for (int j0 = 0; j0 < kPerThr; j0 += kWB) {
      if (j0 * kOutThreads >= 16 * ntile) break;  // uniform over the block
      float scb[kWB][GRP];
      uint16_t vsb[kWB], vzb[kWB];
#pragma unroll
      for (int jj = 0; jj < kWB; ++jj) {
        const int i = tid + (j0 + jj) * kOutThreads;
        const bool valid = i < n;
        vsb[jj] = valid ? v_scale[rowg + c0 + i] : 0;
        vzb[jj] = valid ? v_zero[rowg + c0 + i] : 0;
#pragma unroll
        for (int h = 0; h < GRP; ++h) scb[jj][h] = valid ? score[(static_cast<size_t>(g) * GRP + h) * T + c0 + i] : 0.0f;
      }
#pragma unroll
      for (int jj = 0; jj < kWB; ++jj) {
        const int i = tid + (j0 + jj) * kOutThreads;
        if (i >= 16 * ntile) continue;
        if (i < n) {
          const float sv = sfd::half_bits_to_float(vsb[jj]);
          const float zv = sfd::half_bits_to_float(vzb[jj]);
#pragma unroll
          for (int h = 0; h < GRP; ++h) {
            const float p = __expf(scb[jj][h] - M[h]);
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

    // 2. MMAs over this warp's tiles (stage counters instead of the modulus)
    const uint32_t* ringw = ring + warp * kRing * 16 * kWordsPerRow;
    int st_use = 0, st_iss = kRing - 1;
    for (int ti = tile0; ti < tile1; ++ti) {
      if (ti + kRing - 1 < tile1) issue_st(c0, n, ti + kRing - 1, st_iss);
      st_iss = st_iss == kRing - 1 ? 0 : st_iss + 1;
      cp_async_commit_attn();
      cp_async_wait_attn<kRing - 1>();
      __syncwarp();
      const uint32_t* vr = ringw + st_use * 16 * kWordsPerRow;
      st_use = st_use == kRing - 1 ? 0 : st_use + 1;
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
      const int e = ulist[u];
      if (e & kUMiss) continue;  // uniform over the warp
      const int i = e;
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

  // this warp's output tile (in units of the code part, which carries the
  // factor 4^e of the dim's fragment position: uo enters as uo 4^e / 2^b_f)
  // in the dead weight tile: row (s, g8) for MMA s's rows g8 (s < 8) and
  // g8 + 8 (s + 8), i.e. dims 16 g8 + s and 16 g8 + 8 + s, columns = the
  // MMA's columns (head high parts, then remainders); a lane's two adjacent
  // columns go in one 8-byte store, and a store instruction's 32 lanes
  // cover 64 consecutive words (no bank conflict).  Summed over warps below.
  constexpr int kCols = NT * 8;
  auto tile_row = [](int dim) { return ((dim & 15) << 3) | (dim >> 4); };  // dim = 16 g8 + r -> r * 8 + g8
  __syncthreads();  // every warp is done with the weight tile
  float* ww = reinterpret_cast<float*>(smem) + warp * 16 * 8 * kCols;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int w = 0; w < 8; ++w)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        *reinterpret_cast<float2*>(ww + ((w + 8 * hh) * 8 + g8) * kCols + nt * 8 + 2 * tig) =
            make_float2(acc[nt][w][2 * hh], acc[nt][w][2 * hh + 1]);
  __syncwarp();
#pragma unroll
  for (int h = 0; h < GRP; ++h)
#pragma unroll
    for (int dd = 0; dd < 4; ++dd)
      ww[tile_row(4 * lane + dd) * kCols + h] += (0.25f * vpos_mul(4 * lane + dd)) * uo[h][dd];
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
  if (tid < GRP) {  // the CTA's weight sums per head: L, the offset part Cs and sum(alpha) A
    float L = 0.0f, Cs = 0.0f, A = 0.0f;
    for (int w = 0; w < kOW; ++w) {
      L += red2[w][tid];
      Cs += red2[w][GRP + tid];
      A += red2[w][2 * GRP + tid];
    }
    red2[0][tid] = L;
    red2[0][GRP + tid] = Cs;
    red2[0][2 * GRP + tid] = A;
  }
  __syncthreads();
  float* pg = part + static_cast<size_t>(g) * GRP * splits * (D + 2);
  const float* wt = reinterpret_cast<const float*>(smem);
  for (int e = tid; e < GRP * (D + 2); e += kOutThreads) {
    const int h = e / (D + 2), j = e % (D + 2);
    float v;
    if (j == 0) {
      v = Msh[h];
    } else if (j == 1) {
      v = red2[0][h];
    } else {
      // resident value s (2^b_f c + m_f - z): code part 4 (acc - 1024 A) 4^-e,
      // offset part Cs; acc = the high and remainder columns of head h
      const int r = tile_row(j - 2) * kCols;
      float o = 0.0f;
#pragma unroll
      for (int w = 0; w < kOW; ++w) o += wt[w * 16 * 8 * kCols + r + h] + wt[w * 16 * 8 * kCols + r + GRP + h];
      const float f = vpos_inv(j - 2);
      v = fmaf(4.0f * f, o, fmaf(-4096.0f * f, red2[0][2 * GRP + h], red2[0][GRP + h]));
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
  // every split weighted its tokens against its own maximum per head M_c:
  // factors e^(M_c - M) per head and split (M the largest of the head's),
  // in the dead weight tile
  float* fac = reinterpret_cast<float*>(smem);  // [GRP][splits]
  for (int h = warp; h < GRP; h += kOW) {
    const float* ph = pg + static_cast<size_t>(h) * splits * (D + 2);
    float mx = -INFINITY;
    for (int c = lane; c < splits; c += 32) mx = fmaxf(mx, __ldcg(ph + static_cast<size_t>(c) * (D + 2)));
    mx = warp_max(mx);
    for (int c = lane; c < splits; c += 32) {
      const float mc = __ldcg(ph + static_cast<size_t>(c) * (D + 2));
      fac[h * splits + c] = mc == -INFINITY ? 0.0f : __expf(mc - mx);
    }
  }
  __syncthreads();
  // the merge sums the splits' scaled weight sums and outputs; two outputs
  // per thread, sixteen splits' partials of each in flight at once
  for (int e0 = tid; e0 < GRP * D; e0 += 2 * kOutThreads) {
    const int e1 = e0 + kOutThreads;
    const bool has1 = e1 < GRP * D;
    const int h0 = e0 / D, h1 = has1 ? e1 / D : h0;
    const float* p0 = pg + static_cast<size_t>(h0) * splits * (D + 2);
    const float* p1 = pg + static_cast<size_t>(h1) * splits * (D + 2);
    const int d0 = e0 % D, d1 = has1 ? e1 % D : d0;
    float A0 = 0.0f, A1 = 0.0f, L0 = 0.0f, L1 = 0.0f;
    for (int sp = 0; sp < splits; sp += 16) {
      float v0[16], v1[16], l0[16], l1[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const size_t o = static_cast<size_t>(sp + u) * (D + 2);
        const bool ok = sp + u < splits;
        v0[u] = ok ? __ldcg(p0 + o + 2 + d0) : 0.0f;
        l0[u] = ok ? __ldcg(p0 + o + 1) : 0.0f;
        v1[u] = (ok && has1) ? __ldcg(p1 + o + 2 + d1) : 0.0f;
        l1[u] = (ok && has1) ? __ldcg(p1 + o + 1) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const bool ok = sp + u < splits;
        const float f0 = ok ? fac[h0 * splits + sp + u] : 0.0f, f1 = ok ? fac[h1 * splits + sp + u] : 0.0f;
        A0 = fmaf(f0, v0[u], A0);
        L0 = fmaf(f0, l0[u], L0);
        A1 = fmaf(f1, v1[u], A1);
        L1 = fmaf(f1, l1[u], L1);
      }
    }
    out[(static_cast<size_t>(g) * GRP + h0) * D + d0] = A0 / L0;
    if (has1) out[(static_cast<size_t>(g) * GRP + h1) * D + d1] = A1 / L1;
  }
}

// Clears the workspace's per-call counters and accumulators (a plain launch:
// it starts after the previous kernel of the stream); the score pass, launched
// with programmatic stream serialization, may start meanwhile and waits for
// it only before its first update of the cleared words.
__global__ void ws_clear_kernel(uint4* __restrict__ p, size_t n16) {
  pdl_launch_dependents();
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    p[i] = make_uint4(0u, 0u, 0u, 0u);
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

  {
    const size_t n16 = (L.total - L.smax) / 16;  // offsets are multiples of 256 bytes
    const int blocks = static_cast<int>(std::min<size_t>((n16 + 255) / 256, static_cast<size_t>(2 * sms)));
    ws_clear_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<uint4*>(ws + L.smax), n16);
    const sf_status cs = sf::check_launch("ws_clear_kernel");
    if (cs != SF_OK) return cs;
  }
  // pass A: about two CTAs per SM, each a contiguous range of <= kScMaxTok tokens
  const int want_a = std::max((2 * sms + Hkv - 1) / Hkv, (T + kScMaxTok - 1) / kScMaxTok);
  const int tpc = ((T + want_a - 1) / want_a + 15) / 16 * 16;
  dim3 ga((T + tpc - 1) / tpc, Hkv);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + L.hist);
  uint32_t* amaxu = reinterpret_cast<uint32_t*>(ws + L.amax);
  uint32_t* mkey = reinterpret_cast<uint32_t*>(ws + L.mkey);
  const bool selecting = k > 0 && k < T;
  SelBand* band = reinterpret_cast<SelBand*>(ws + L.band);
  int32_t* ccnt = reinterpret_cast<int32_t*>(ws + L.ccnt);
  SF_CHECK_CUDA(cudaFuncSetAttribute(attn_score_mma_kernel<GRP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(score_smem(GRP))));
  {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = ga;
    cfg.blockDim = dim3(kScThreads);
    cfg.dynamicSmemBytes = score_smem(GRP);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    SF_CHECK_CUDA(cudaLaunchKernelEx(&cfg, attn_score_mma_kernel<GRP>, q, kv->k_res, kv->k_scale, kv->k_zero, T, S,
                                     tpc, score, smax, hist, amaxu, mkey));
  }
  sf_status st = sf::check_launch("attn_score_mma_kernel");
  if (st != SF_OK) return st;
  if (selecting) {
    {
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3(static_cast<unsigned>((T + kChunk - 1) / kChunk), static_cast<unsigned>(Hq));
      cfg.blockDim = dim3(kCompThreads);
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      SF_CHECK_CUDA(cudaLaunchKernelEx(&cfg, attn_compact_kernel, q, T, k, static_cast<const float*>(score),
                                       static_cast<const float*>(smax), static_cast<const int32_t*>(hist),
                                       static_cast<const uint32_t*>(amaxu), band, cand, ccnt, status, grp));
      st = sf::check_launch("attn_compact_kernel");
      if (st != SF_OK) return st;
    }
    // the group's bitmask words in the cluster's shared memory when they fit
    const int wper = (L.words_t + GRP - 1) / GRP;
    const int dsm = wper <= kSelMaxWords ? 1 : 0;
    const size_t dyn = sel_dyn_smem(dsm ? wper : 0);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(Hq));
    cfg.blockDim = dim3(kSelThreads);
    cfg.dynamicSmemBytes = dyn;
    SF_CHECK_CUDA(cudaFuncSetAttribute(attn_select_kernel<GRP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(dyn)));
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = GRP;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    SF_CHECK_CUDA(cudaLaunchKernelEx(&cfg, attn_select_kernel<GRP>, q, kv->k_res, kv->k_scale, kv->k_zero, T, k, S,
                                     static_cast<const float*>(score), static_cast<const SelBand*>(band),
                                     static_cast<const int32_t*>(cand), static_cast<const int32_t*>(ccnt), cand2, kap,
                                     sel_head, umask, L.words_t, wper, dsm, sel_out, sel_n, status, mkey));
    st = sf::check_launch("attn_select_kernel");
    if (st != SF_OK) return st;
  } else if (k == 0) {  // the token bitmask was cleared with the workspace
    SF_CHECK_CUDA(cudaMemsetAsync(sel_n, 0, sizeof(int32_t) * Hkv, s));
  } else {  // every token is in the union
    fill_all_kernel<<<dim3(32, Hkv), 256, 0, s>>>(T, grp, k, L.words_t, umask, sel_out, sel_n, mkey);
    st = sf::check_launch("fill_all_kernel");
    if (st != SF_OK) return st;
  }
  dim3 gb(L.splits, Hkv);
  SF_CHECK_CUDA(cudaFuncSetAttribute(attn_out_kernel<GRP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(OutCfg<GRP>::smem)));
  {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = gb;
    cfg.blockDim = dim3(kOutThreads);
    cfg.dynamicSmemBytes = OutCfg<GRP>::smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    SF_CHECK_CUDA(cudaLaunchKernelEx(&cfg, attn_out_kernel<GRP>, q, kv->k_res, k_ref, kv->k_scale, kv->k_zero,
                                     static_cast<const uint32_t*>(kv->v_res), v_ref, uslot, kv->v_scale, kv->v_zero,
                                     T, S, L.tps, L.words_t, L.splits, score, static_cast<const uint32_t*>(mkey),
                                     static_cast<const uint32_t*>(umask), part, done, out));
  }
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
