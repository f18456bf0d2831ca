// Device helpers and the workspace layout shared by the two implementations
// of refined decode attention: the multi-kernel pipeline (attn.cu) and the
// single cluster kernel per KV group (attn_fused.cu).
#pragma once

#include <algorithm>
#include <cmath>

#include "block_scan.cuh"
#include "sf_internal.h"

namespace sf {

// The single cluster kernel per KV group (attn_fused.cu): whether it applies
// to these sizes on the current device, and the launch.  The overflow lists
// (keys, tokens: Hq * T each; winners: Hq * k), the CTAs' partials and
// union counts live in the caller's workspace.
bool attn_fused_eligible(int Hq, int Hkv, int T);
sf_status attn_fused_run(const uint16_t* q, int Hq, int Hkv, int T, const sf_qkv* kv, int k, int32_t* sel_out,
                         int32_t* sel_n, float* out, double* ovf_key, int32_t* ovf_tok, int32_t* ovf_sel,
                         float* gpart, int32_t* gcnt, cudaStream_t s);

}  // namespace sf

namespace {

constexpr int D = 128;                 // head dim
constexpr int kWordsPerRow = D * 2 / 32;  // 2-bit codes of one token-head: 8 words
constexpr int kMaxGrp = 8;
constexpr int kMaxSplits = 256;
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1/sqrt(128), rounded to fp32

constexpr int kHistBits = 11;      // per-head histogram of the fast scores' top 11 key bits
constexpr int kHistBins = 1 << kHistBits;
constexpr int kHistShift = 32 - kHistBits;

// A head's selection band, derived once from the score pass's histogram:
// every token whose exact key can reach the top k has a fast score >= f_low;
// the k-th largest fast score lies in histogram bin b1, kk-th from its top;
// eps bounds |fast score - exact key / sqrt(d)|.
struct SelBand {
  double eps;
  float f_low;
  uint32_t b1;
  int kk;
  int pad;
};

struct Layout {
  // from smax on, everything is cleared at the start of a call
  size_t score, cand, cand2, kap, sel, part, fcnt, smax, status, count, amax, mkey, band, ccnt, hist,
      umask, total;
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
  // split partials of the pipeline, or of the 16 CTAs of a cluster
  L.part = off; off = up256(off + sizeof(float) * Hq * static_cast<size_t>(std::max(L.splits, 16)) * (D + 2));
  L.fcnt = off; off = up256(off + sizeof(int32_t) * Hkv * 16);
  L.smax = off; off = up256(off + sizeof(float) * 2 * Hkv);  // max key scale, then max s |1.5 - z|, per group
  L.status = off; off = up256(off + sizeof(int32_t) * std::max(Hkv, 4));
  L.count = off; off = up256(off + sizeof(int32_t) * Hkv);
  L.amax = off; off = up256(off + sizeof(uint32_t) * Hq);
  L.mkey = off; off = up256(off + sizeof(uint32_t) * Hq);  // max resident score key per head
  L.band = off; off = up256(off + sizeof(SelBand) * Hq);     // selection band per head
  L.ccnt = off; off = up256(off + sizeof(int32_t) * Hq);     // listed candidates per head
  L.hist = off; off = up256(off + sizeof(int32_t) * Hq * static_cast<size_t>(kHistBins));
  L.umask = off; off = up256(off + sizeof(uint32_t) * Hkv * static_cast<size_t>(L.words_t));
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

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while its predecessor runs; pdl_wait() returns once
// the predecessor grid has completed and its memory is visible, and must come
// before the first read of anything the predecessor writes.
// pdl_launch_dependents() lets the next such kernel start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::); }

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
__device__ __forceinline__ void cp_async_commit_attn() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait_attn() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Integer tensor-core MMA over code bytes (m16n8k32, s32 accumulate).
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

// Value codes as f16 MMA fragments.  An MMA row (a dim of the output) need
// not follow the dims' order: lane row g8 (g8 + 8) of MMA s takes dim
// 16 g8 + s (16 g8 + 8 + s), so a lane reads word g8 of its four token rows
// once per 16-token tile; two byte permutes per row pair put dims 0-7 (8-15)
// of the two tokens in the halves of a register, four shifted copies (left
// 6 and 2, right 2 and 6) bring the code of every s to mantissa bits 6-7 or
// 8-9, and each fragment register is one mask and or: the exact f16 pair
// 1024 + c 4^e, e = 3 + (s & 1).  The dim's accumulated code part carries the
// factor 4^e, taken out when the partials are formed; against the 1024
// offset the code part is large (64 c or 256 c), so the offset's removal
// loses little of the fp32 accumulation's precision.
__device__ __forceinline__ int vpos_exp(int dim) { return 3 + (dim & 1); }
// 4^-e for the dim's exponent e (exact)
__device__ __forceinline__ float vpos_inv(int dim) { return __int_as_float((127 - 2 * vpos_exp(dim)) << 23); }
// 4^e
__device__ __forceinline__ float vpos_mul(int dim) { return __int_as_float((127 + 2 * vpos_exp(dim)) << 23); }
// The four fragment registers of MMA s (a constant after unrolling) from the
// shifted permutes src[s / 2] (vperm).
__device__ __forceinline__ void vfrag(const uint32_t (&src)[4][4], int s, uint32_t& a0, uint32_t& a1, uint32_t& a2,
                                      uint32_t& a3) {
  const uint32_t m = (s & 1) ? 0x03000300u : 0x00C000C0u;
  a0 = (src[s >> 1][0] & m) | 0x64006400u;
  a1 = (src[s >> 1][1] & m) | 0x64006400u;
  a2 = (src[s >> 1][2] & m) | 0x64006400u;
  a3 = (src[s >> 1][3] & m) | 0x64006400u;
}
// A lane's words for one tile: word g8 of token rows 2 tig, 2 tig + 1
// (wa, wb: registers 0, 1 = dims 0-7, 8-15) and 2 tig + 8, 2 tig + 9 (wc, wd:
// registers 2, 3), each in the four shifted copies.
__device__ __forceinline__ void vperm(uint32_t wa, uint32_t wb, uint32_t wc, uint32_t wd, uint32_t (&src)[4][4]) {
  const uint32_t p[4] = {__byte_perm(wa, wb, 0x5410), __byte_perm(wa, wb, 0x7632), __byte_perm(wc, wd, 0x5410),
                         __byte_perm(wc, wd, 0x7632)};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    src[0][i] = p[i] << 6;  // s = 0, 1
    src[1][i] = p[i] << 2;  // s = 2, 3
    src[2][i] = p[i] >> 2;  // s = 4, 5
    src[3][i] = p[i] >> 6;  // s = 6, 7
  }
}

// f16 tensor-core MMA with f32 accumulate (m16n8k16).
__device__ __forceinline__ void mma_f16f32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---- pass S: exact per-head top-k ------------------------------------------

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

// Query-side setup of pass S (all threads call): q in fp64 into qd, its l1
// norm and the binary exponent of max |q|; flags the KV group when the
// nonzero q exponents span more than the exact-key precondition allows.
// With dq_out, also the l1 norm of the fixed-point rounding of q with qfrac
// fraction bits (sum_d |q_d - rint(q_d 2^(qfrac - e)) 2^(e - qfrac)|, each
// term exact in fp64; the sum is rounded up by a relative 2^-44).
__device__ void select_q_prologue(const uint16_t* __restrict__ q, int h, int g, double* qd, double* l1_out,
                                  int* qe_out, int32_t* __restrict__ status, int* span_out = nullptr,
                                  int qfrac = 0, double* dq_out = nullptr) {
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
    if (dq_out) {
      const int e = emax >= emin ? emax : 0;
      double dq = 0.0;
      for (int d = tid; d < D; d += 32) {
        const double v = qd[d];
        dq += fabs(v - ldexp(rint(ldexp(v, qfrac - e)), e - qfrac));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dq += __shfl_xor_sync(0xffffffffu, dq, o);
      if (tid == 0) *dq_out = dq * (1.0 + 0x1p-44);
    }
    if (tid == 0) {
      *l1_out = l1;
      *qe_out = emax >= emin ? emax : 0;  // binary exponent of max |q| (frexp convention)
      if (span_out) *span_out = emax >= emin ? emax - emin : 0;  // binades spanned by the nonzero q
      // 53 - 9 - b - log2(d) with b = 4, d = 128
      if (emax >= emin && emax - emin > 53 - 9 - 4 - 7) atomicOr(status + g, 1);
    }
  }
  __syncthreads();
}

// Error bound of the fast scores (pass A): q rounded to fixed point with
// qfrac fraction bits relative to 2^e, X = rint(q 2^(qfrac - e)), so
// |dq| <= 2^(e - qfrac - 1) per entry (the cluster kernel: 23 bits; the
// pipeline's score pass: 14), exact integer products and sums, an fp32
// combine of the plane sums, the fp32 sum of q (<= gamma_128 l1), and the
// roundings of the zero-point term, the fma, the scale and 1/sqrt(d).
// Returns the half-width eps_s of the band; two fast scores whose exact
// values are ordered one way differ by at least -2 eps_s the other way.
__device__ __forceinline__ double select_eps(double s_max, double l1, int qe, float amax, int qfrac) {
  const double u = 5.9604644775390625e-8;  // 2^-24
  const double gam = 130.0 * u / (1.0 - 130.0 * u);
  const double qround = ldexp(1.0, qe - qfrac - 1);
  const double eps_k = s_max * (4.0 * 3.0 * D * qround + l1 * (136.0 * u + 16.0 * gam));
  return 2.0 * (static_cast<double>(kInvSqrtD) * eps_k + 4.0 * u * static_cast<double>(amax));
}

// The same bound for the pipeline's score pass, from the actual rounding of
// q rather than its worst case.  There q~ = X 2^(e - qfrac) (dq = q - q~,
// dq1 = sum |dq|), P = sum_d c_d q~_d exactly, Q = fp32 of the exact sum of
// q (one rounding), a = fl(1.5 - z), b = fl(a Q), E' = fl(4 P + b), score =
// fl(fl(s E') c) with c the fp32 1/sqrt(d); the exact key is s E with E =
// sum_d q_d (4 c_d + 1.5 - z).  Then
//   |4 P - 4 sum c q| <= 12 dq1 (codes <= 3),
//   |b - (1.5 - z) sum q| <= gamma_3 |1.5 - z| l1,
//   the rounding of E' <= u (12 (l1 + dq1) + (1 + gamma_3) |1.5 - z| l1),
//   the two last roundings <= gamma_2 / (1 - u)^2 |score| <= 2.0001 u amax,
// so |score - c s E| <= c (s_max (12 (1 + u) dq1 + 12 u l1) + 4.0002 u
// sz_max l1) + 2.0001 u amax, with s_max = max s and sz_max = max s |1.5 -
// z| over the group's tokens; the result is rounded up by a relative 2^-40.
__device__ __forceinline__ double select_eps_pipe(double s_max, double sz_max, double l1, double dq1, float amax) {
  const double u = 5.9604644775390625e-8;  // 2^-24
  const double inner = s_max * (12.0 * (1.0 + u) * dq1 + 12.0 * u * l1) + 4.0002 * u * sz_max * l1;
  return (static_cast<double>(kInvSqrtD) * inner + 2.0001 * u * static_cast<double>(amax)) * (1.0 + 0x1p-40);
}

// Exact top-k of F[0..ncand) by (key desc, token asc): an 8-pass radix select
// on the 64-bit order-preserving keys kp, then 4 passes on the complemented
// token among the entries tied with the k-th key (F in any order; all threads
// call); the k winners go to sel in no particular order.
__device__ void select_rank_radix(const int32_t* __restrict__ F, int ncand, const double* __restrict__ kp, int k,
                                  int* hist, int* scan_scratch, int* binfo, int32_t* __restrict__ sel) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  unsigned long long pre64 = 0, pm64 = 0;
  uint32_t pt = 0, mt = 0;
  int kr = k;
  for (int pass = 0; pass < 12; ++pass) {
    for (int i = tid; i < 256; i += nthr) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < ncand; i += nthr) {
      const unsigned long long key = okey64(kp[i]);
      const uint32_t nt = ~static_cast<uint32_t>(F[i]);
      if ((key & pm64) != pre64 || (nt & mt) != pt) continue;
      const uint32_t digit = pass < 8 ? static_cast<uint32_t>((key >> (56 - 8 * pass)) & 255u)
                                      : (nt >> (24 - 8 * (pass - 8))) & 255u;
      atomicAdd(&hist[digit], 1);
    }
    __syncthreads();
    find_bin_from_top(hist, 256, kr, binfo);
    __syncthreads();
    if (pass < 8) {
      pre64 |= static_cast<unsigned long long>(binfo[0]) << (56 - 8 * pass);
      pm64 |= 255ull << (56 - 8 * pass);
    } else {
      pt |= static_cast<uint32_t>(binfo[0]) << (24 - 8 * (pass - 8));
      mt |= 255u << (24 - 8 * (pass - 8));
    }
    kr = binfo[1];
    __syncthreads();
  }
  // (key, ~token) pairs are distinct: the winners are those >= the k-th
  int take = 0;
  for (int i = tid; i < ncand; i += nthr) {
    const unsigned long long key = okey64(kp[i]);
    take += (key > pre64 || (key == pre64 && ~static_cast<uint32_t>(F[i]) >= pt)) ? 1 : 0;
  }
  int tot;
  int pos = sfd::block_exclusive_scan(take, scan_scratch, &tot);
  for (int i = tid; i < ncand; i += nthr) {
    const unsigned long long key = okey64(kp[i]);
    if (key > pre64 || (key == pre64 && ~static_cast<uint32_t>(F[i]) >= pt)) sel[pos++] = F[i];
  }
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

// Per-head lower bound of the listed scores and the histogram bin: all threads call.
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

}  // namespace
