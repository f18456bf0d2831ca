// Prepared activations for the batch-1 GEMV on the integer tensor cores.
//
// An activation row x[K] (bf16, K a multiple of 256) is cut into 256-channel
// slices, each made of two 128-channel groups (the weight quantization group).
// Per group the activations become exact-as-possible fixed point
//   X_j = rint(x_j 2^(22 - e)),  e = binary exponent of the group's max |x|
// (max |x| in [2^(e-1), 2^e), so |X_j| <= 2^22), split into balanced base-256
// digits X = d0 + 256 d1 + 65536 d2 with every digit in [-128, 127] (|d2| <=
// 65), the signed 8-bit B operand of mma.m16n8k32 (u8 codes x s8 digits).
//
// Per slice, kAct2Words uint32 words:
//   [0, 512)   B fragments of the slice's 8 k-steps: word (m*32 + lane)*2 + r
//              is register b_r of lane `lane` for k-step m.  Column n (= lane
//              / 4) of the MMA is (group slot n / 4, digit plane n % 4); a
//              k-step m belongs to slot m / 4, so only its slot's columns are
//              nonzero (plane 3 is always zero) and the two groups of a slice
//              accumulate into disjoint columns of one accumulator.  Byte b
//              of b_r in lane (n, t) holds the plane's digit of channel
//                256 s + 128 (m/4) + 16 (2t + (m%4)/2) + 4b + 2 (m%2) + r,
//              the channel whose 2-bit code the A fragment extracts as
//              (w >> 2j) & 0x03030303 from weight word 8 (m/4) + 2t + (m%4)/2
//              of the row's slice (j = 2 (m%2) + r).
//   512, 513   group 0: fscale = 2^(e - 22), gsum = fscale * sum_j X_j (fp32)
//   514, 515   group 1: the same
//   516        number of selected channels in slices before this one
//   517        number of selected channels in this slice
//   518, 519   zero
//   [520, 528) selection mask: bit i of word w <=> channel 256 s + 32 w + i
#pragma once

#include <cstdint>

#include "block_scan.cuh"

namespace sfd {

constexpr int kAct2Words = 528;
constexpr int kAct2Frag = 512;
constexpr int kAct2Info = 512;
constexpr int kAct2Mask = 520;

// Binary exponent (frexp convention) of |bf16| given as bits; -1000 for zero.
__device__ __forceinline__ int bf16_exponent(uint32_t b) {
  const uint32_t E = (b >> 7) & 0xFFu;
  const uint32_t m = (b & 0x7Fu) | (E ? 0x80u : 0u);
  const int Ee = E ? static_cast<int>(E) : 1;
  return m ? (32 - __clz(m)) + Ee - 134 : -1000;
}

// X = rint(x 2^(22 - e)) from the bf16 bits with integer operations only
// (ties to even when bits are shifted out).  Valid for e >= the value's own
// exponent; values more than 31 binades below 2^e give 0.
__device__ __forceinline__ int bf16_fixed(uint32_t b, int e) {
  const uint32_t E = (b >> 7) & 0xFFu;
  const uint32_t m = (b & 0x7Fu) | (E ? 0x80u : 0u);
  const int Ee = E ? static_cast<int>(E) : 1;
  const int sh = Ee - 112 - e;  // x = m 2^(Ee - 134), X = m 2^(Ee - 134 + 22 - e)
  int v;
  if (sh >= 0) {
    v = static_cast<int>(m << sh);
  } else if (sh >= -9) {
    const int r = -sh;
    const uint32_t q = m >> r, rem = m & ((1u << r) - 1u), half = 1u << (r - 1);
    v = static_cast<int>(q + ((rem > half || (rem == half && (q & 1u))) ? 1u : 0u));
  } else {
    v = 0;
  }
  return (b & 0x8000u) ? -v : v;
}

// Writes the prepared form of a whole row with one thread block (every thread
// calls; contains __syncthreads).  xs: the row's bf16 bits (shared or global
// memory); flags: one byte per channel, nonzero = selected (nullptr: none);
// eg: K / 128 ints of shared scratch (group exponents); ginfo: 2 * (K / 128)
// floats of shared scratch (fscale, gsum per group); scan: 33 ints of shared
// scratch.
__device__ inline void act2_write_block(const uint16_t* xs, const uint8_t* flags, int K, int* eg, float* ginfo,
                                        int* scan, uint32_t* __restrict__ act) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int ngroups = K >> 7, nslice = K >> 8;
  // 1. per group: exponent, fixed-point values, their sum (one warp a group)
  for (int gi = warp; gi < ngroups; gi += nw) {
    uint32_t b[4];
    int e = -1000;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      b[i] = xs[128 * gi + 32 * i + lane];
      e = max(e, bf16_exponent(b[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e = max(e, __shfl_xor_sync(0xffffffffu, e, o));
    if (e == -1000) e = 0;
    int s = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) s += bf16_fixed(b[i], e);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
      eg[gi] = e;
      const float fscale = ldexpf(1.0f, e - 22);
      ginfo[2 * gi] = fscale;
      ginfo[2 * gi + 1] = static_cast<float>(s) * fscale;
    }
  }
  __syncthreads();
  // 2. B fragments: one task per (slice, k-step m, column tig) converts its 8
  //    channels once and writes their three digit-plane words for b0 and b1;
  //    the other columns' words of the k-step are zero
  for (int task = tid; task < nslice * 32; task += blockDim.x) {
    const int s = task >> 5, m = (task >> 2) & 7, t = task & 3;
    const int slot = m >> 2, mm = m & 3;
    const int ch0 = 256 * s + 128 * slot + 16 * (2 * t + (mm >> 1)) + 2 * (mm & 1);
    const int e = eg[ch0 >> 7];
    uint32_t* o = act + static_cast<size_t>(s) * kAct2Words + m * 64;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      uint32_t w0 = 0, w1 = 0, w2 = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int X = bf16_fixed(xs[ch0 + 4 * b + r], e);
        const int d0 = ((X + 128) & 255) - 128;
        const int X1 = (X - d0) >> 8;
        const int d1 = ((X1 + 128) & 255) - 128;
        const int d2 = (X1 - d1) >> 8;
        w0 |= (static_cast<uint32_t>(d0) & 0xFFu) << (8 * b);
        w1 |= (static_cast<uint32_t>(d1) & 0xFFu) << (8 * b);
        w2 |= (static_cast<uint32_t>(d2) & 0xFFu) << (8 * b);
      }
      // lane (n, t) = 4 n + t; column n = 4 slot + plane
      o[(4 * (4 * slot + 0) + t) * 2 + r] = w0;
      o[(4 * (4 * slot + 1) + t) * 2 + r] = w1;
      o[(4 * (4 * slot + 2) + t) * 2 + r] = w2;
      o[(4 * (4 * slot + 3) + t) * 2 + r] = 0u;
      o[(4 * (4 * (1 - slot) + 0) + t) * 2 + r] = 0u;
      o[(4 * (4 * (1 - slot) + 1) + t) * 2 + r] = 0u;
      o[(4 * (4 * (1 - slot) + 2) + t) * 2 + r] = 0u;
      o[(4 * (4 * (1 - slot) + 3) + t) * 2 + r] = 0u;
    }
  }
  // 3. group scalars, selection masks and counts (one thread a slice)
  int carry = 0;  // selected channels in earlier rounds of slices
  for (int base = 0; base < nslice; base += blockDim.x) {
    const int s = base + tid;
    const bool active = s < nslice;
    uint32_t mw[8];
    int c = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t v = 0;
      if (active && flags != nullptr)
        for (int i = 0; i < 32; ++i) v |= static_cast<uint32_t>(flags[256 * s + 32 * w + i] != 0) << i;
      mw[w] = v;
      c += __popc(v);
    }
    int total;
    const int pre = carry + block_exclusive_scan(c, scan, &total);
    carry += total;
    if (active) {
      uint32_t* o = act + static_cast<size_t>(s) * kAct2Words;
      reinterpret_cast<uint4*>(o + kAct2Info)[0] =
          make_uint4(__float_as_uint(ginfo[4 * s]), __float_as_uint(ginfo[4 * s + 1]),
                     __float_as_uint(ginfo[4 * s + 2]), __float_as_uint(ginfo[4 * s + 3]));
      reinterpret_cast<uint4*>(o + kAct2Info)[1] = make_uint4(static_cast<uint32_t>(pre), static_cast<uint32_t>(c), 0u, 0u);
      reinterpret_cast<uint4*>(o + kAct2Mask)[0] = make_uint4(mw[0], mw[1], mw[2], mw[3]);
      reinterpret_cast<uint4*>(o + kAct2Mask)[1] = make_uint4(mw[4], mw[5], mw[6], mw[7]);
    }
  }
}

}  // namespace sfd
