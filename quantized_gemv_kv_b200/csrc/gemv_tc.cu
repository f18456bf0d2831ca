// sf_gemv_refine for batches of 2 to 16 rows on the tensor cores.
//
//   y[b][i] = sum_j x[b][j] w_res[i][j] + sum_{j in S} x[b][j] s_{g(j),i} (q_f[i][j] - m_f)
//
// (nested refinement of the columns with the largest activations; the
// selection S is one set for the whole batch, rag-lover.com explainer of
// StrataFlux, 解説).  With eight or more rows the resident part is a dense
// contraction worth the tensor cores, and so is the refinement correction
// once the union of the rows' selections is large.  Below eight rows the
// MMA's unused columns cost nothing that matters: unpacking 2-3-bit codes
// for CUDA-core FMAs is instruction-bound, one MMA per 16x16 codes is not,
// and the bytes read are the same.
//
// Resident part on mma.m16n8k16 (f16 in, f32 accumulate), MMA rows = output
// rows, MMA columns = batch rows (two n-tiles for more than eight):
//  * A: a code c enters as the exact f16 1024 + 64 c (c at mantissa bits
//    6-8), taken from the canonical bitstream with a shift and a mask.  The
//    order of the 16 channels inside one MMA is free (the same permutation on
//    both operands): lane tig's register pairs take channels (tig, tig + 8)
//    and (tig + 4, tig + 12) of the 16-channel block, which sit in the two
//    halves of one 32-bit window of the stream;
//  * B: x of the CTA's K chunk, scaled per batch row by a power of two to
//    max |x~| < 2^15 and converted to f16 (exact for entries within 28
//    binades of the row's maximum in the chunk), stored in shared memory in
//    that permuted fragment order;
//  * per quantization group the MMA sums acc = sum_j x~_j (1024 + 64 c_j)
//    start from zero, and the group's scale and zero point are applied once:
//    sum_j x~_j w_res = s (2^b_f (acc - 1024 X~) / 64 + (m_f - z) X~) with X~
//    the group's sum of x~ (fp32).  The 1024 offset is at most 11x the code
//    part, so its removal costs little of the fp32 accumulation's accuracy.
// A CTA takes 64 output rows (four 16-row tiles) and a K chunk of up to 2048
// channels; two warps per row tile split the chunk's 128-channel units and
// add up in shared memory; with several chunks the CTAs add their sums onto
// a zeroed output.  Codes stream through a per-warp cp.async ring, one unit
// of the warp's 16 rows per stage.  Quantization groups are whole units
// (G a multiple of 128); other shapes take the CUDA-core kernel.
#include <cuda_fp16.h>

#include <algorithm>

#include "sf_internal.h"

namespace {

constexpr int kTcThreads = 256;
constexpr int kTcWarps = kTcThreads / 32;
constexpr int kTcChunk = 2048;    // K channels per CTA at most
template <int BR>
constexpr int tc_ring() { return BR == 2 ? 4 : 3; }  // cp.async stages per warp (one 128-channel unit each)

__device__ __forceinline__ void cp_async16_tc(void* smem, const void* gmem) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit_tc() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait_tc() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// v 2^e exactly for |e| <= 252 and v's range here (two power-of-two factors,
// each a normal fp32)
__device__ __forceinline__ float scale_pow2(float v, int e) {
  const int e1 = e / 2, e2 = e - e1;
  return __fmul_rn(__fmul_rn(v, __int_as_float((127 + e1) << 23)), __int_as_float((127 + e2) << 23));
}

__device__ __forceinline__ void mma_f16_tc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The 32-bit window of a row's code stream that starts at channel 16 q + tig
// (BR bits a code): channel tig + m of the block at bits BR m.  wr: the
// unit's staged words (starting at the unit's first channel, one word of
// padding after them).
template <int BR>
__device__ __forceinline__ uint32_t code_window(const uint32_t* wr, int q, int tig) {
  const int bit = BR * (16 * q + tig);
  const int w = bit >> 5, sh = bit & 31;
  return sh ? __funnelshift_r(wr[w], wr[w + 1], sh) : wr[w];
}

// A-fragment register pair from a window: the codes of window channels 0 and
// 8 (BR = 2: bits 0-1 and 16-17; BR = 3: bits 0-2 and 24-26) as f16 1024 + 64 c.
template <int BR>
__device__ __forceinline__ uint32_t code_pair(uint32_t v) {
  if constexpr (BR == 2) {
    return ((v << 6) & 0x00C000C0u) | 0x64006400u;
  } else {
    const uint32_t t = __byte_perm(v, 0u, 0x4340);  // byte 3 (channel 8's code) to byte 2
    return ((t << 6) & 0x01C001C0u) | 0x64006400u;
  }
}

}  // namespace

namespace {

constexpr int kTcMTiles = 4;                     // 16-row MMA tiles per CTA
constexpr int kTcCtaRows = 16 * kTcMTiles;       // 64 output rows per CTA
constexpr int kTcUnits = kTcChunk / 128;         // 128-channel units per chunk
constexpr int kTcHalves = kTcWarps / kTcMTiles;  // warps per row tile, splitting the chunk's units

template <int BR>
struct TcCfg {
  static constexpr int GW = BR * 4;                 // words of a row's 128-channel unit
  // staged row stride in words: room for the last window's extra word, a
  // multiple of 4 (16-byte cp.async rows) whose multiples by 0..7 fall in
  // eight different banks, so the eight rows a fragment load touches never
  // share a bank
  static constexpr int RS = BR == 2 ? 12 : 20;
  static constexpr int kStage = 16 * RS;            // words per stage: one row tile, one unit
  static constexpr int ring_words = kTcWarps * tc_ring<BR>() * kStage;
};

// The correction's staging, in the ring's space after the resident part:
// per selected channel of the chunk its refinement words for the CTA's rows
// (at most 64 b_f / 32 = 4) and its chunk-relative channel; the k-step table.
constexpr int kTcMaxSel = kTcChunk;
constexpr int kTcMaxKsteps = kTcMaxSel / 16 + kTcUnits;
constexpr int kTcCorrWords = kTcMaxSel * 4 + kTcMaxSel + 2 * kTcMaxKsteps;

template <int NT>
struct TcSmem {
  static constexpr int xs_words = (kTcChunk / 16) * NT * 64;  // f16 pairs in fragment order
  static constexpr int bsum_floats = 16 * (kTcChunk / 16);    // per batch row and 16-channel block
  static constexpr int xsum_floats = 16 * kTcUnits;           // per batch row and unit
  static constexpr int ysm_floats = kTcCtaRows * 16;
  static_assert(ysm_floats <= xs_words, "the output tile lives in the staged fragments' space at the end");
};

// Shared memory: [ring | block sums] (the correction's staging after the
// resident part), the staged x~ fragments (the output tile at the end), the
// unit sums of x~.
template <int BR, int NT>
constexpr int tc_front_words() {
  return TcCfg<BR>::ring_words + TcSmem<NT>::bsum_floats > kTcCorrWords
             ? TcCfg<BR>::ring_words + TcSmem<NT>::bsum_floats
             : kTcCorrWords;
}

template <int BR, int NT>
constexpr size_t tc_smem_bytes() {
  return 4ull * (tc_front_words<BR, NT>() + TcSmem<NT>::xs_words + TcSmem<NT>::xsum_floats);
}

template <int BR, int NT>
__global__ void __launch_bounds__(kTcThreads, 2)
gemv_tc_kernel(const uint32_t* __restrict__ res, const uint16_t* __restrict__ scale,
               const uint16_t* __restrict__ zero, int N, int K, int G, int b_f, const uint16_t* __restrict__ x, int B,
               const int32_t* __restrict__ idx, const int32_t* __restrict__ n_sel,
               const uint32_t* __restrict__ ref_rows, const int32_t* __restrict__ row_of, int unit_words,
               float* __restrict__ y, int accumulate) {
  using C = TcCfg<BR>;
  using M = TcSmem<NT>;
  extern __shared__ __align__(16) uint32_t tsm[];
  uint32_t* ring = tsm;
  float* bsum = reinterpret_cast<float*>(ring + C::ring_words);
  uint32_t* xs = ring + tc_front_words<BR, NT>();
  float* xsum = reinterpret_cast<float*>(xs + M::xs_words);
  float* ysm = reinterpret_cast<float*>(xs);  // [64 rows][16 columns], after the correction
  __shared__ int xsc_sh[16];                     // per batch row: x~ = x 2^xsc

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g8 = lane >> 2, tig = lane & 3;
  const int row0 = blockIdx.x * kTcCtaRows;
  const int k0 = blockIdx.y * kTcChunk, kc = min(kTcChunk, K - k0);
  const int nunits = kc >> 7, nblk = kc >> 4;
  const int rowW = K * BR / 32;  // words per resident row

  // 1. x~ in one pass: batch row b = tid / 16 takes 16 threads, thread j of
  //    them the 16-channel blocks q = j, j + 16, ... of the chunk (every
  //    load in flight at once); the row's scale from the largest exponent
  //    (a 16-lane max); then the f16 pairs in fragment order, (x~[tig],
  //    x~[tig+8]) and (x~[tig+4], x~[tig+12]) for lane (b % 8, tig) of n-tile
  //    b / 8, and each block's sum of x~
  {
    constexpr int kQPer = kTcChunk / 16 / 16;  // blocks per thread
    const int b = tid >> 4, j = tid & 15;
    uint4 raw[kQPer][2];
    int e = 0;
#pragma unroll
    for (int t = 0; t < kQPer; ++t) {
      const int q = j + 16 * t;
      if (b < B && q < nblk) {
        const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(b) * K + k0 + 16 * q);
        raw[t][0] = src[0];
        raw[t][1] = src[1];
      } else {
        raw[t][0] = raw[t][1] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int t = 0; t < kQPer; ++t) {
      const uint32_t w[8] = {raw[t][0].x, raw[t][0].y, raw[t][0].z, raw[t][0].w,
                             raw[t][1].x, raw[t][1].y, raw[t][1].z, raw[t][1].w};
#pragma unroll
      for (int i = 0; i < 8; ++i) e = max(e, static_cast<int>(max((w[i] >> 7) & 0xFFu, (w[i] >> 23) & 0xFFu)));
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) e = max(e, __shfl_xor_sync(0xffffffffu, e, o));
    // max |x~| < 2^15 with x~ = x 2^(141 - e), e the biased exponent (1 for subnormal maxima)
    const int sc = 141 - max(e, 1);
    if (j == 0) xsc_sh[b] = sc;
    if (b < NT * 8) {
#pragma unroll
      for (int t = 0; t < kQPer; ++t) {
        const int q = j + 16 * t;
        if (q >= nblk) continue;
        const uint32_t w[8] = {raw[t][0].x, raw[t][0].y, raw[t][0].z, raw[t][0].w,
                               raw[t][1].x, raw[t][1].y, raw[t][1].z, raw[t][1].w};
        __half hv[16];
        float s = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          hv[2 * i] = __float2half_rn(scale_pow2(__uint_as_float(w[i] << 16), sc));
          hv[2 * i + 1] = __float2half_rn(scale_pow2(__uint_as_float(w[i] & 0xFFFF0000u), sc));
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) s += __half2float(hv[i]);
        uint32_t out[8];
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
          out[2 * tt] = static_cast<uint32_t>(__half_as_ushort(hv[tt])) |
                        (static_cast<uint32_t>(__half_as_ushort(hv[tt + 8])) << 16);
          out[2 * tt + 1] = static_cast<uint32_t>(__half_as_ushort(hv[tt + 4])) |
                            (static_cast<uint32_t>(__half_as_ushort(hv[tt + 12])) << 16);
        }
        uint4* dst = reinterpret_cast<uint4*>(xs + ((q * NT + (b >> 3)) * 32 + (b & 7) * 4) * 2);
        dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
        dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
        bsum[b * (kTcChunk / 16) + q] = s;
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < 16 * nunits; e += kTcThreads) {
    const int b = e / nunits, u = e - b * nunits;
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) s += bsum[b * (kTcChunk / 16) + 8 * u + i];
    xsum[b * kTcUnits + u] = s;
  }
  __syncthreads();

  // 2. resident part: warp (row tile mt, half kh) runs units kh, kh + 2, ...
  const int mt = warp % kTcMTiles, kh = warp / kTcMTiles;
  const int r0 = row0 + 16 * mt;
  float yacc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) yacc[nt][0] = yacc[nt][1] = yacc[nt][2] = yacc[nt][3] = 0.0f;
  const float m_f = static_cast<float>((1 << b_f) - 1) * 0.5f;
  const float coef = static_cast<float>(1 << b_f) * (1.0f / 64.0f);
  if (r0 < N) {
    constexpr int kTcRing = tc_ring<BR>();
    uint32_t* wring = ring + warp * kTcRing * C::kStage;
    const int count = (nunits - kh + kTcHalves - 1) / kTcHalves;  // this warp's units
    auto issue = [&](int i, int st) {
      const int u = kh + kTcHalves * i;
      const size_t col = static_cast<size_t>((k0 >> 7) + u) * C::GW;
      for (int c = lane; c < 16 * BR; c += 32) {
        const int rr = c / BR, part = c - rr * BR;
        cp_async16_tc(wring + st * C::kStage + rr * C::RS + 4 * part,
                      res + static_cast<size_t>(r0 + rr) * rowW + col + 4 * part);
      }
    };
    for (int i = 0; i < kTcRing - 1; ++i) {
      if (i < count) issue(i, i);
      cp_async_commit_tc();
    }
    int st_use = 0, st_iss = kTcRing - 1;
    for (int i = 0; i < count; ++i) {
      if (i + kTcRing - 1 < count) issue(i + kTcRing - 1, st_iss);
      st_iss = st_iss == kTcRing - 1 ? 0 : st_iss + 1;
      cp_async_commit_tc();
      const int u = kh + kTcHalves * i;
      // this unit's scales and zeros for rows g8, g8 + 8 (issued before the wait)
      const int grp = (k0 + 128 * u) / G;
      const float s0 = __half2float(__ushort_as_half(scale[static_cast<size_t>(grp) * N + r0 + g8]));
      const float s1 = __half2float(__ushort_as_half(scale[static_cast<size_t>(grp) * N + r0 + g8 + 8]));
      const float z0 = m_f - __half2float(__ushort_as_half(zero[static_cast<size_t>(grp) * N + r0 + g8]));
      const float z1 = m_f - __half2float(__ushort_as_half(zero[static_cast<size_t>(grp) * N + r0 + g8 + 8]));
      cp_async_wait_tc<kTcRing - 1>();
      __syncwarp();
      const uint32_t* wr0 = wring + st_use * C::kStage + g8 * C::RS;
      const uint32_t* wr1 = wr0 + 8 * C::RS;
      st_use = st_use == kTcRing - 1 ? 0 : st_use + 1;
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t a0 = code_pair<BR>(code_window<BR>(wr0, q, tig));
        const uint32_t a1 = code_pair<BR>(code_window<BR>(wr1, q, tig));
        const uint32_t a2 = code_pair<BR>(code_window<BR>(wr0, q, tig + 4));
        const uint32_t a3 = code_pair<BR>(code_window<BR>(wr1, q, tig + 4));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint2 bb = *reinterpret_cast<const uint2*>(xs + (((8 * u + q) * NT + nt) * 32 + lane) * 2);
          mma_f16_tc(acc[nt], a0, a1, a2, a3, bb.x, bb.y);
        }
      }
      __syncwarp();  // the stage is refilled by a later issue
      // the unit's scale and zero point: s (2^b_f (acc - 1024 X~) / 64 + (m_f - z) X~)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float X = xsum[(nt * 8 + 2 * tig + (c & 1)) * kTcUnits + u];
          const float t = fmaf(-1024.0f, X, acc[nt][c]);
          const float v = fmaf(coef, t, ((c >> 1) ? z1 : z0) * X);
          yacc[nt][c] = fmaf((c >> 1) ? s1 : s0, v, yacc[nt][c]);
        }
    }
    cp_async_wait_tc<0>();
  }
  // 3. refinement correction on the tensor cores, into the same sums: the
  //    chunk's selected channels (one ascending run of the selection) go in
  //    k-steps of 16 that never cross a quantization group (padding: code 0,
  //    x~ 0); A = 1024 + 64 q_f of the k-step's channels, B = their x~
  //    (gathered from the staged fragments), and per k-step
  //    sum_j x~_j s (q_f - m_f) = s ((acc - 1024 X~) / 64 - m_f X~) with X~
  //    the k-step's sum of x~ per batch row.
  if (ref_rows != nullptr) {
    __shared__ int run_sh[2], nks_sh, gks_sh[kTcUnits + 1];
    __syncthreads();  // every warp is done with the ring
    const int ngc = kc / G;  // quantization groups in the chunk
    if (tid <= ngc) {
      // the selection's first entry >= k0 + tid G (tid = ngc: the chunk's end)
      int n = *n_sel;
      n = n < 0 ? 0 : n;
      const int bound = k0 + tid * G;
      int lo = 0, hi = n;
      while (lo < hi) {
        const int m = (lo + hi) >> 1;
        if (idx[m] < bound) lo = m + 1;
        else hi = m;
      }
      gks_sh[tid] = lo;
    }
    __syncthreads();
    const int p0 = gks_sh[0], p1 = gks_sh[ngc];
    const int ns = p1 - p0;
    constexpr int WPC = 4;  // staged words per channel (64 rows x b_f <= 2 bits)
    uint32_t* selw = ring;                                      // [ns][WPC]
    uint16_t* selc = reinterpret_cast<uint16_t*>(ring + kTcMaxSel * WPC);  // [ns] chunk-relative channel
    int* kst = reinterpret_cast<int*>(ring + kTcMaxSel * WPC + kTcMaxSel / 2);  // [k-step]: first entry, group
    const int wrow0 = (row0 * b_f) >> 5;  // the CTA's first refinement word of a unit
    const int nwr = min(WPC, unit_words - wrow0);
    for (int e = tid; e < ns * WPC; e += kTcThreads) {
      const int en = e / WPC, w = e - en * WPC;
      const int p = p0 + en;
      if (w == 0) selc[en] = static_cast<uint16_t>(idx[p] - k0);
      if (w < nwr) {
        const int rid = row_of ? row_of[p] : idx[p];
        selw[e] = ref_rows[static_cast<size_t>(rid) * unit_words + wrow0 + w];
      }
    }
    if (tid == 0) {
      int nk = 0;
      for (int gi = 0; gi < ngc; ++gi)
        for (int st = gks_sh[gi]; st < gks_sh[gi + 1]; st += 16) {
          kst[2 * nk] = st - p0;
          kst[2 * nk + 1] = gi;
          ++nk;
        }
      nks_sh = nk;
    }
    __syncthreads();
    if (r0 < N) {
      const uint32_t fmask = (1u << b_f) - 1u;
      const int lw0 = ((r0 - row0 + g8) * b_f) >> 5, sh0 = ((r0 + g8) * b_f) & 31;
      const int lw1 = ((r0 - row0 + g8 + 8) * b_f) >> 5, sh1 = ((r0 + g8 + 8) * b_f) & 31;
      int cur_g = -1;
      float s0 = 0.0f, s1 = 0.0f;
      for (int ks = kh; ks < nks_sh; ks += kTcHalves) {
        const int e0 = kst[2 * ks], gi = kst[2 * ks + 1];
        const int eend = gks_sh[gi + 1] - p0;
        if (gi != cur_g) {
          cur_g = gi;
          const int grp = k0 / G + gi;
          s0 = __half2float(__ushort_as_half(scale[static_cast<size_t>(grp) * N + r0 + g8]));
          s1 = __half2float(__ushort_as_half(scale[static_cast<size_t>(grp) * N + r0 + g8 + 8]));
        }
        // this lane's channels: k-slots (2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9) = entries tig, tig + 8, tig + 4, tig + 12
        int en[4];
        en[0] = e0 + tig;
        en[1] = e0 + tig + 8;
        en[2] = e0 + tig + 4;
        en[3] = e0 + tig + 12;
        uint32_t q0[4], q1[4];
        int cc[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const bool ok = en[u] < eend;
          const uint32_t* wv = selw + (ok ? en[u] : 0) * WPC;
          q0[u] = ok ? (wv[lw0] >> sh0) & fmask : 0u;
          q1[u] = ok ? (wv[lw1] >> sh1) & fmask : 0u;
          cc[u] = ok ? selc[en[u]] : -1;
        }
        const uint32_t a0 = (q0[0] << 6) | (q0[1] << 22) | 0x64006400u;
        const uint32_t a1 = (q1[0] << 6) | (q1[1] << 22) | 0x64006400u;
        const uint32_t a2 = (q0[2] << 6) | (q0[3] << 22) | 0x64006400u;
        const uint32_t a3 = (q1[2] << 6) | (q1[3] << 22) | 0x64006400u;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int bb = nt * 8 + g8;  // this lane's batch row in the B fragment
          uint16_t xh[4];
          float xsum_l = 0.0f;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            xh[u] = 0;
            if (cc[u] >= 0) {
              const int c = cc[u], q = c >> 4, m = c & 15;
              const uint32_t pr = xs[((q * NT + nt) * 32 + g8 * 4 + (m & 3)) * 2 + ((m >> 2) & 1)];
              xh[u] = static_cast<uint16_t>((m >> 3) ? pr >> 16 : pr & 0xFFFFu);
              xsum_l += __half2float(__ushort_as_half(xh[u]));
            }
          }
          (void)bb;
          const uint32_t b0 = static_cast<uint32_t>(xh[0]) | (static_cast<uint32_t>(xh[1]) << 16);
          const uint32_t b1 = static_cast<uint32_t>(xh[2]) | (static_cast<uint32_t>(xh[3]) << 16);
          float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          mma_f16_tc(acc, a0, a1, a2, a3, b0, b1);
          // the k-step's sum of x~ for batch row nt*8 + g8 (the quad's four lanes), then
          // for this lane's accumulator columns 2 tig, 2 tig + 1 (held by lanes 4 (2 tig + c))
          xsum_l += __shfl_xor_sync(0xffffffffu, xsum_l, 1);
          xsum_l += __shfl_xor_sync(0xffffffffu, xsum_l, 2);
          const float X0 = __shfl_sync(0xffffffffu, xsum_l, 4 * (2 * tig));
          const float X1 = __shfl_sync(0xffffffffu, xsum_l, 4 * (2 * tig + 1));
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float X = (c & 1) ? X1 : X0;
            const float v = fmaf(1.0f / 64.0f, fmaf(-1024.0f, X, acc[c]), -m_f * X);
            yacc[nt][c] = fmaf((c >> 1) ? s1 : s0, v, yacc[nt][c]);
          }
        }
      }
    }
  }
  __syncthreads();  // the staged fragments are read no more: the output tile takes their space
  // the two halves of a row tile add up (half 0 stores, half 1 adds)
  for (int h = 0; h < kTcHalves; ++h) {
    if (kh == h) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int rl = 16 * mt + g8 + 8 * (c >> 1), col = nt * 8 + 2 * tig + (c & 1);
          float* p = ysm + rl * 16 + col;
          *p = h == 0 ? yacc[nt][c] : *p + yacc[nt][c];
        }
    }
    __syncthreads();
  }
  // back to x's units
  for (int e = tid; e < kTcCtaRows * 16; e += kTcThreads) ysm[e] = scale_pow2(ysm[e], -xsc_sh[e & 15]);
  __syncthreads();

  for (int e = tid; e < kTcCtaRows * B; e += kTcThreads) {
    const int b = e / kTcCtaRows, rl = e - b * kTcCtaRows;
    if (row0 + rl >= N) continue;
    float* dst = y + static_cast<size_t>(b) * N + row0 + rl;
    if (accumulate) atomicAdd(dst, ysm[rl * 16 + b]);
    else *dst = ysm[rl * 16 + b];
  }
}

template <int BR, int NT>
sf_status launch_tc(const sf_qweight* W, const uint16_t* x, int B, const int32_t* idx, const int32_t* n,
                    const uint32_t* ref_rows, const int32_t* row_of, int unit_words, float* y, cudaStream_t s) {
  constexpr size_t smem = tc_smem_bytes<BR, NT>();
  SF_CHECK_CUDA(cudaFuncSetAttribute(gemv_tc_kernel<BR, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)));
  const int splits = (W->K + kTcChunk - 1) / kTcChunk;
  if (splits > 1) SF_CHECK_CUDA(cudaMemsetAsync(y, 0, sizeof(float) * B * W->N, s));
  dim3 grid((W->N + kTcCtaRows - 1) / kTcCtaRows, splits);
  gemv_tc_kernel<BR, NT><<<grid, kTcThreads, smem, s>>>(W->res, W->scale, W->zero, W->N, W->K, W->G, W->b_f, x, B,
                                                        idx, n, ref_rows, row_of, unit_words, y, splits > 1);
  return sf::check_launch("gemv_tc_kernel");
}

}  // namespace

namespace sf {

bool gemv_tc_try(const sf_qweight* W, const uint16_t* x, int B, const int32_t* idx, const int32_t* n,
                 const uint32_t* ref_rows, const int32_t* row_of, int unit_words, float* y, cudaStream_t s,
                 sf_status* st) {
  if (B < 2 || B > 16 || W->G % 128 != 0 || W->K % 128 != 0 || !aligned(W->res, 16) || !aligned(x, 16)) return false;
  if (B <= 8)
    *st = W->b_r == 2 ? launch_tc<2, 1>(W, x, B, idx, n, ref_rows, row_of, unit_words, y, s)
                      : launch_tc<3, 1>(W, x, B, idx, n, ref_rows, row_of, unit_words, y, s);
  else
    *st = W->b_r == 2 ? launch_tc<2, 2>(W, x, B, idx, n, ref_rows, row_of, unit_words, y, s)
                      : launch_tc<3, 2>(W, x, B, idx, n, ref_rows, row_of, unit_words, y, s);
  return true;
}

}  // namespace sf
