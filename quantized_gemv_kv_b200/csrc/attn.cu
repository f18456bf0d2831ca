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
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1/sqrt(128), rounded to fp32

struct Layout {
  size_t score, cand, kap, sel, umask, part, smax, status, count, total;
  int splits, tps, words_t;
};

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

Layout make_layout(int Hq, int Hkv, int T, int k, int sms) {
  Layout L{};
  const int want = std::max(1, (2 * sms + Hkv - 1) / Hkv);
  int tps = (T + want - 1) / want;
  tps = std::max(128, (tps + 127) / 128 * 128);
  L.tps = tps;
  L.splits = (T + tps - 1) / tps;
  L.words_t = (T + 31) / 32;
  size_t off = 0;
  L.score = off; off = up256(off + sizeof(float) * Hq * static_cast<size_t>(T));
  L.cand = off; off = up256(off + sizeof(int32_t) * Hq * static_cast<size_t>(T));
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

// ---- pass A: resident scores --------------------------------------------
template <int GRP>
__global__ void __launch_bounds__(128)
attn_score_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                  const uint16_t* __restrict__ k_scale, const uint16_t* __restrict__ k_zero, int T,
                  float* __restrict__ score, float* __restrict__ smax) {
  __shared__ float qs[GRP][D];
  __shared__ float qsum[GRP];
  const int g = blockIdx.y;
  load_q<GRP>(q, g, qs, qsum);
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  float s = 0.0f;
  if (t < T) {
    const size_t row = static_cast<size_t>(g) * T + t;
    const uint4* kp = reinterpret_cast<const uint4*>(k_res + row * kWordsPerRow);
    const uint4 a = kp[0], b = kp[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    s = sfd::half_bits_to_float(k_scale[row]);
    const float z = sfd::half_bits_to_float(k_zero[row]);
    float P[GRP];
#pragma unroll
    for (int h = 0; h < GRP; ++h) P[h] = 0.0f;
#pragma unroll
    for (int d = 0; d < D; ++d) {
      const float c = static_cast<float>((w[d >> 4] >> ((d & 15) * 2)) & 3u);
#pragma unroll
      for (int h = 0; h < GRP; ++h) P[h] = fmaf(qs[h][d], c, P[h]);
    }
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const float E = fmaf(4.0f, P[h], (1.5f - z) * qsum[h]);
      score[(static_cast<size_t>(g) * GRP + h) * T + t] = (s * E) * kInvSqrtD;
    }
  }
  const float m = warp_max(s);
  if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<unsigned int*>(smax + g), __float_as_uint(m));
}

// Histogram increment with same-bin lanes of a warp merged into one atomic;
// bin < 0 means no increment.  Call with the whole warp.
__device__ __forceinline__ void warp_hist_add(int* hist, int bin) {
  const unsigned peers = __match_any_sync(0xffffffffu, bin);
  const int leader = __ffs(peers) - 1;
  if (bin >= 0 && (threadIdx.x & 31) == leader) atomicAdd(&hist[bin], __popc(peers));
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

template <int GRP>
__global__ void __launch_bounds__(kSelThreads)
attn_select_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                   const uint16_t* __restrict__ k_scale, const uint16_t* __restrict__ k_zero, int T, int k,
                   const float* __restrict__ score, const float* __restrict__ smax, int32_t* __restrict__ cand,
                   double* __restrict__ kap, int32_t* __restrict__ sel_head, int32_t* __restrict__ status) {
  __shared__ int hist[2048];
  __shared__ double qd[D];
  __shared__ int scan_scratch[33];
  __shared__ int binfo[2];
  __shared__ float red[32];
  __shared__ double l1_sh;
  const int h = blockIdx.x, g = h / GRP, tid = threadIdx.x;
  const float* sc = score + static_cast<size_t>(h) * T;
  int32_t* cd = cand + static_cast<size_t>(h) * T;
  double* kp = kap + static_cast<size_t>(h) * T;

  for (int d = tid; d < D; d += kSelThreads) qd[d] = static_cast<double>(sfd::bf16_bits_to_float(q[static_cast<size_t>(h) * D + d]));
  __syncthreads();
  if (tid < 32) {
    // L1 norm (exact in fp64 for 128 bf16 values) and the exponent span check
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
      l1_sh = l1;
      // 53 - 9 - b - log2(d) with b = 4, d = 128
      if (emax >= emin && emax - emin > 53 - 9 - 4 - 7) atomicOr(status + g, 1);
    }
  }

  // 1. radix select of the k-th largest fast score (11 + 11 + 10 bits)
  uint32_t prefix = 0, pmask = 0;
  int kk = k;
  float amax = 0.0f;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int nb = 1 << widths[pass];
    for (int i = tid; i < nb; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int t0 = tid - (tid & 31); t0 < T; t0 += kSelThreads) {
      const int t = t0 + (tid & 31);
      int bin = -1;
      if (t < T) {
        const float v = sc[t];
        if (pass == 0) amax = fmaxf(amax, fabsf(v));
        const uint32_t key = okey32(v);
        if ((key & pmask) == prefix) bin = static_cast<int>((key >> shifts[pass]) & (nb - 1));
      }
      warp_hist_add(hist, bin);
    }
    __syncthreads();
    find_bin_from_top(hist, nb, kk, binfo);
    __syncthreads();
    prefix |= static_cast<uint32_t>(binfo[0]) << shifts[pass];
    pmask |= static_cast<uint32_t>(nb - 1) << shifts[pass];
    kk = binfo[1];
    __syncthreads();
  }
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
  const double tau = static_cast<double>(from_okey32(prefix));

  // 2. error bound of the fast scores (see the pass-A arithmetic): a sum of
  // 128 fp32 FMAs has |error| <= gamma_128 * sum |terms|.
  const double u = 5.9604644775390625e-8;  // 2^-24
  const double gam = 130.0 * u / (1.0 - 130.0 * u);
  const double s_max = static_cast<double>(smax[g]);
  const double l1 = l1_sh;
  const double eps_k = s_max * l1 * (4.0 * 3.0 * gam + 16.0 * gam + 4.0 * 16.0 * u);
  const double eps_s = 2.0 * (static_cast<double>(kInvSqrtD) * eps_k + 4.0 * u * static_cast<double>(amax));
  const double thr = tau - 2.0 * eps_s;

  // 3. candidates (fast score >= thr), ascending token order
  int ncand;
  {
    const int chunk = (T + kSelThreads - 1) / kSelThreads;
    const int t0 = min(T, tid * chunk), t1 = min(T, t0 + chunk);
    int c = 0;
    for (int t = t0; t < t1; ++t) c += static_cast<double>(sc[t]) >= thr;
    int pos = sfd::block_exclusive_scan(c, scan_scratch, &ncand);
    for (int t = t0; t < t1; ++t)
      if (static_cast<double>(sc[t]) >= thr) cd[pos++] = t;
  }
  __syncthreads();

  // 4. exact keys of the candidates
  for (int i = tid; i < ncand; i += kSelThreads) {
    const int t = cd[i];
    const size_t row = static_cast<size_t>(g) * T + t;
    const uint32_t* w = k_res + row * kWordsPerRow;
    const double s = static_cast<double>(sfd::half_bits_to_float(k_scale[row]));
    const double z = static_cast<double>(sfd::half_bits_to_float(k_zero[row]));
    double E = 0.0;
    for (int d = 0; d < D; ++d) {
      const double c = static_cast<double>((w[d >> 4] >> ((d & 15) * 2)) & 3u);
      E = fma(qd[d], c * 4.0 + 1.5 - z, E);
    }
    kp[i] = s * E;
  }
  __syncthreads();

  // 5. exact top-k among the candidates by (key desc, token asc)
  unsigned long long pre64 = 0, pm64 = 0;
  int kr = k;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int i0 = tid - (tid & 31); i0 < ncand; i0 += kSelThreads) {
      const int i = i0 + (tid & 31);
      int bin = -1;
      if (i < ncand) {
        const unsigned long long key = okey64(kp[i]);
        if ((key & pm64) == pre64) bin = static_cast<int>((key >> shift) & 255);
      }
      warp_hist_add(hist, bin);
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
    // keys above the k-th key, plus the first kr equal to it in token order
    const int chunk = (ncand + kSelThreads - 1) / kSelThreads;
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
      if (ok) sel_head[static_cast<size_t>(h) * k + pos++] = cd[i];
    }
  }
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

// ---- pass B: softmax-weighted values over all tokens, refined where selected
template <int GRP>
__global__ void __launch_bounds__(128)
attn_out_kernel(const uint16_t* __restrict__ q, const uint32_t* __restrict__ k_res,
                const uint32_t* __restrict__ k_ref, const uint16_t* __restrict__ k_scale,
                const uint16_t* __restrict__ k_zero, const uint32_t* __restrict__ v_res,
                const uint32_t* __restrict__ v_ref, const uint16_t* __restrict__ v_scale,
                const uint16_t* __restrict__ v_zero, int T, int tps, int words_t, int splits,
                const float* __restrict__ score, const uint32_t* __restrict__ umask, float* __restrict__ part,
                int32_t* __restrict__ done, float* __restrict__ out) {
  __shared__ float qs[GRP][D];
  __shared__ float qsum[GRP];
  __shared__ uint32_t vr[4][32][kWordsPerRow];
  __shared__ uint32_t vf[4][32][kWordsPerRow];
  __shared__ float alpha[4][32][GRP];
  __shared__ float wm[4][GRP];
  __shared__ float wl[4][GRP];
  __shared__ float wo[4][GRP][D];
  const int g = blockIdx.y, split = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  load_q<GRP>(q, g, qs, qsum);
  const int t0 = split * tps, t1 = min(T, t0 + tps);

  float m[GRP], l[GRP], bs[GRP], o[GRP][4];
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.0f;
    bs[h] = 0.0f;
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) o[h][dd] = 0.0f;
  }

  for (int base = t0 + warp * 32; base < t1; base += 4 * 32) {
    const int t = base + lane;
    const bool valid = t < t1;
    const size_t row = static_cast<size_t>(g) * T + (valid ? t : t0);
    bool inU = false;
    float sc[GRP];
    if (valid) {
      inU = (umask[static_cast<size_t>(g) * words_t + (t >> 5)] >> (t & 31)) & 1u;
#pragma unroll
      for (int h = 0; h < GRP; ++h) sc[h] = score[(static_cast<size_t>(g) * GRP + h) * T + t];
      if (inU) {
        // refined key: k' = s (4 c_r + c_f - z)
        const uint32_t* wr = k_res + row * kWordsPerRow;
        const uint32_t* wf = k_ref + row * kWordsPerRow;
        const float s = sfd::half_bits_to_float(k_scale[row]);
        const float z = sfd::half_bits_to_float(k_zero[row]);
        float P[GRP];
#pragma unroll
        for (int h = 0; h < GRP; ++h) P[h] = 0.0f;
        for (int d = 0; d < D; ++d) {
          const uint32_t cr = (wr[d >> 4] >> ((d & 15) * 2)) & 3u;
          const uint32_t cf = (wf[d >> 4] >> ((d & 15) * 2)) & 3u;
          const float c = static_cast<float>(cr * 4u + cf);
#pragma unroll
          for (int h = 0; h < GRP; ++h) P[h] = fmaf(qs[h][d], c, P[h]);
        }
#pragma unroll
        for (int h = 0; h < GRP; ++h) sc[h] = (s * fmaf(-z, qsum[h], P[h])) * kInvSqrtD;
      }
    } else {
#pragma unroll
      for (int h = 0; h < GRP; ++h) sc[h] = -INFINITY;
    }
    // V codes of this token into the warp's staging rows
    {
      const uint4* pr = reinterpret_cast<const uint4*>(v_res + row * kWordsPerRow);
      const uint4 a = pr[0], b = pr[1];
      uint32_t* dst = vr[warp][lane];
      dst[0] = a.x; dst[1] = a.y; dst[2] = a.z; dst[3] = a.w;
      dst[4] = b.x; dst[5] = b.y; dst[6] = b.z; dst[7] = b.w;
      uint32_t* dsf = vf[warp][lane];
      if (inU) {
        const uint4* pf = reinterpret_cast<const uint4*>(v_ref + row * kWordsPerRow);
        const uint4 c = pf[0], e = pf[1];
        dsf[0] = c.x; dsf[1] = c.y; dsf[2] = c.z; dsf[3] = c.w;
        dsf[4] = e.x; dsf[5] = e.y; dsf[6] = e.z; dsf[7] = e.w;
      } else {
#pragma unroll
        for (int i = 0; i < kWordsPerRow; ++i) dsf[i] = 0u;
      }
    }
    const float sv = valid ? sfd::half_bits_to_float(v_scale[row]) : 0.0f;
    const float zv = valid ? sfd::half_bits_to_float(v_zero[row]) : 0.0f;
    const float off = inU ? -zv : 1.5f - zv;  // v = s * (code + off)
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const float mt = warp_max(sc[h]);
      const float nm = fmaxf(m[h], mt);
      const float r = (m[h] == -INFINITY) ? 0.0f : __expf(m[h] - nm);
      m[h] = nm;
      l[h] *= r;
      bs[h] *= r;
#pragma unroll
      for (int dd = 0; dd < 4; ++dd) o[h][dd] *= r;
      const float p = valid ? __expf(sc[h] - nm) : 0.0f;
      l[h] += p;
      bs[h] = fmaf(p * sv, off, bs[h]);
      alpha[warp][lane][h] = p * sv;
    }
    __syncwarp();
    const int wsel = lane >> 2, sh = (lane & 3) * 8;
    for (int tt = 0; tt < 32; ++tt) {
      const uint32_t cr = (vr[warp][tt][wsel] >> sh) & 0xFFu;
      const uint32_t cf = (vf[warp][tt][wsel] >> sh) & 0xFFu;
#pragma unroll
      for (int dd = 0; dd < 4; ++dd) {
        const float code = static_cast<float>(((cr >> (2 * dd)) & 3u) * 4u + ((cf >> (2 * dd)) & 3u));
#pragma unroll
        for (int h = 0; h < GRP; ++h) o[h][dd] = fmaf(alpha[warp][tt][h], code, o[h][dd]);
      }
    }
    __syncwarp();
  }
  // per warp: l and bs are per-lane partials with the warp-uniform max m
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    const float lt = warp_sum(l[h]);
    const float bt = warp_sum(bs[h]);
    if (lane == 0) { wm[warp][h] = m[h]; wl[warp][h] = lt; }
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) wo[warp][h][lane * 4 + dd] = o[h][dd] + bt;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < GRP * (D + 2); e += blockDim.x) {
    const int h = e / (D + 2), j = e % (D + 2);
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w][h]);
    float acc = 0.0f;
    if (j == 0) {
      acc = M;
    } else {
      for (int w = 0; w < 4; ++w) {
        if (wm[w][h] == -INFINITY) continue;
        const float f = __expf(wm[w][h] - M);
        acc += f * (j == 1 ? wl[w][h] : wo[w][h][j - 2]);
      }
    }
    part[((static_cast<size_t>(g) * GRP + h) * splits + split) * (D + 2) + j] = acc;
  }
  // the last CTA of this KV group to finish merges every split's partials
  // (threadfence-then-count, so no CTA ever waits for another)
  __shared__ int last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(done + g, 1) == splits - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int e = threadIdx.x; e < GRP * D; e += blockDim.x) {
    const int h = e / D, d = e % D;
    const float* p = part + (static_cast<size_t>(g) * GRP + h) * splits * (D + 2);
    float M = -INFINITY;
    for (int sp = 0; sp < splits; ++sp) M = fmaxf(M, __ldcg(p + sp * (D + 2)));
    float Lsum = 0.0f, O = 0.0f;
    for (int sp = 0; sp < splits; ++sp) {
      const float ms = __ldcg(p + sp * (D + 2));
      if (ms == -INFINITY) continue;
      const float f = __expf(ms - M);
      Lsum = fmaf(f, __ldcg(p + sp * (D + 2) + 1), Lsum);
      O = fmaf(f, __ldcg(p + sp * (D + 2) + 2 + d), O);
    }
    out[(static_cast<size_t>(g) * GRP + h) * D + d] = O / Lsum;
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
  double* kap = reinterpret_cast<double*>(ws + L.kap);
  int32_t* sel_head = reinterpret_cast<int32_t*>(ws + L.sel);
  uint32_t* umask = reinterpret_cast<uint32_t*>(ws + L.umask);
  float* part = reinterpret_cast<float*>(ws + L.part);
  float* smax = reinterpret_cast<float*>(ws + L.smax);
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  const int grp = GRP;

  SF_CHECK_CUDA(cudaMemsetAsync(ws + L.smax, 0, L.total - L.smax, s));
  if (k > 0 && k < T) {
    dim3 ga((T + 127) / 128, Hkv);
    attn_score_kernel<GRP><<<ga, 128, 0, s>>>(q, kv->k_res, kv->k_scale, kv->k_zero, T, score, smax);
    sf_status st = sf::check_launch("attn_score_kernel");
    if (st != SF_OK) return st;
    attn_select_kernel<GRP><<<Hq, kSelThreads, 0, s>>>(q, kv->k_res, kv->k_scale, kv->k_zero, T, k, score, smax,
                                                       cand, kap, sel_head, status);
    st = sf::check_launch("attn_select_kernel");
    if (st != SF_OK) return st;
    const size_t smem = sizeof(uint32_t) * L.words_t;
    SF_CHECK_CUDA(cudaFuncSetAttribute(attn_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(std::max<size_t>(smem, 1))));
    attn_union_kernel<<<Hkv, 1024, smem, s>>>(sel_head, grp, T, k, L.words_t, umask, sel_out, sel_n, status);
    st = sf::check_launch("attn_union_kernel");
    if (st != SF_OK) return st;
  } else {
    // no selection needed: everything (k == T) or nothing (k == 0) refined,
    // scores still come from pass A
    dim3 ga((T + 127) / 128, Hkv);
    attn_score_kernel<GRP><<<ga, 128, 0, s>>>(q, kv->k_res, kv->k_scale, kv->k_zero, T, score, smax);
    sf_status st = sf::check_launch("attn_score_kernel");
    if (st != SF_OK) return st;
    if (k == 0) {
      SF_CHECK_CUDA(cudaMemsetAsync(umask, 0, sizeof(uint32_t) * Hkv * static_cast<size_t>(L.words_t), s));
      SF_CHECK_CUDA(cudaMemsetAsync(sel_n, 0, sizeof(int32_t) * Hkv, s));
    } else {
      fill_all_kernel<<<dim3(32, Hkv), 256, 0, s>>>(T, grp, k, L.words_t, umask, sel_out, sel_n);
      st = sf::check_launch("fill_all_kernel");
      if (st != SF_OK) return st;
    }
  }
  dim3 gb(L.splits, Hkv);
  int32_t* done = reinterpret_cast<int32_t*>(ws + L.count);
  attn_out_kernel<GRP><<<gb, 128, 0, s>>>(q, kv->k_res, kv->k_ref, kv->k_scale, kv->k_zero, kv->v_res, kv->v_ref,
                                          kv->v_scale, kv->v_zero, T, L.tps, L.words_t, L.splits, score, umask, part,
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
