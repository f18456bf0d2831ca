// Prepared activations for the batch-1 integer GEMV.
//
// Per 32-channel slab s of an activation row x[K] (bf16), 32 uint32 words:
//   [0..24)  fixed-point byte planes: word (wi*4 + k)*3 + p holds, in byte b,
//            byte p of X[16*wi + k + 4*b] -- the order in which a 2-bit code
//            word w_wi yields code bytes via (w_wi >> 2k) & 0x03030303;
//   24       sum_j x_j of the slab as fp32 (from the fixed-point values);
//   25       fscale = 2^(e - 23) as fp32 (x_j ~= X_j * fscale);
//   26       bit j set when channel 32*s + j is in the refined selection;
//   27       number of selected channels in slabs before s;
//   28       sum_j x_j over the slab's 128-channel block, fp32;
//   29..31   zero.
// X_j = rint(x_j * 2^(23 - e)) with e the binary exponent of the largest |x|
// in the slab's 128-channel block (max |x| in [2^(e-1), 2^e)): the four slabs
// of a block share one scale, so their integer dot products can be added
// before any conversion.  |X_j| < 2^23 and every bf16 within 15 binades of
// the block maximum is represented exactly.
#pragma once

#include <cstdint>

namespace sfd {

constexpr int kActWords = 32;

__device__ inline void act_planes_from_floats(const float (&xf)[32], uint32_t (&pl)[24], float* xsum,
                                              float* fscale) {
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(xf[j]));
  int e = 0;
  if (amax > 0.0f) frexpf(amax, &e);
  int X[32];
  int xs = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    X[j] = __float2int_rn(ldexpf(xf[j], 23 - e));
    xs += X[j];
  }
  *fscale = ldexpf(1.0f, e - 23);
  *xsum = static_cast<float>(xs) * *fscale;
#pragma unroll
  for (int wi = 0; wi < 2; ++wi)
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int p = 0; p < 3; ++p) {
        uint32_t v = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b)
          v |= ((static_cast<uint32_t>(X[16 * wi + k + 4 * b]) >> (8 * p)) & 0xFFu) << (8 * b);
        pl[(wi * 4 + k) * 3 + p] = v;
      }
}

// Binary exponent e of the largest |x| of a slab (max |x| in [2^(e-1), 2^e));
// -1000 for an all-zero slab.
__device__ inline int act_slab_exponent(const uint16_t* __restrict__ x32) {
  int e = -1000;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t b = x32[j];
    const uint32_t E = (b >> 7) & 0xFFu;
    const uint32_t m = (b & 0x7Fu) | (E ? 0x80u : 0u);
    const int Ee = E ? static_cast<int>(E) : 1;
    if (m) e = max(e, (32 - __clz(m)) + Ee - 134);
  }
  return e;
}

// Same planes from the bf16 bit patterns with integer operations only
// (identical values: e is the frexp exponent of the largest |x|, and
// X_j = rint(x_j 2^(23-e)) is formed by shifting the 8-bit significand,
// rounding half to even when bits are shifted out).
__device__ inline void act_planes_from_bits(const uint32_t (&xb)[32], int e_block, uint32_t (&pl)[24], float* xsum,
                                            float* fscale) {
  // e_block: exponent shared by the block (>= every element's own exponent)
  int e = e_block;
  int ef[32];
  uint32_t mant[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t E = (xb[j] >> 7) & 0xFFu;
    const uint32_t m = (xb[j] & 0x7Fu) | (E ? 0x80u : 0u);
    const int Ee = E ? static_cast<int>(E) : 1;
    mant[j] = m;
    ef[j] = Ee;
  }
  if (e == -1000) e = 0;
  int X[32];
  int xs = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int sh = ef[j] - 111 - e;  // X = m 2^sh
    int v;
    if (sh >= 0) {
      v = static_cast<int>(mant[j] << sh);
    } else if (sh >= -9) {
      const int r = -sh;
      const uint32_t q = mant[j] >> r, rem = mant[j] & ((1u << r) - 1u), half = 1u << (r - 1);
      v = static_cast<int>(q + ((rem > half || (rem == half && (q & 1u))) ? 1u : 0u));
    } else {
      v = 0;
    }
    X[j] = (xb[j] & 0x8000u) ? -v : v;
    xs += X[j];
  }
  *fscale = ldexpf(1.0f, e - 23);
  *xsum = static_cast<float>(xs) * *fscale;
#pragma unroll
  for (int wi = 0; wi < 2; ++wi)
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int p = 0; p < 3; ++p) {
        uint32_t v = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b)
          v |= ((static_cast<uint32_t>(X[16 * wi + k + 4 * b]) >> (8 * p)) & 0xFFu) << (8 * b);
        pl[(wi * 4 + k) * 3 + p] = v;
      }
}

// Block helper for a warp whose lanes hold consecutive slabs (lane l = slab
// 32*w + l, all 32 lanes calling; inactive lanes pass e = -1000 and xsum = 0):
// the maximum exponent and the sum over each group of 4 lanes (= one block).
__device__ __forceinline__ int act_block_exponent(int e) {
  e = max(e, __shfl_xor_sync(0xffffffffu, e, 1));
  e = max(e, __shfl_xor_sync(0xffffffffu, e, 2));
  return e;
}
__device__ __forceinline__ float act_block_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

// Writes the 32-word prepared form of slab x32[0..32) to out, with the
// block exponent e_block and the block sum of x (filled in by the caller
// once known, see act_write_block_sum).
__device__ inline float act_write_slab(const uint16_t* __restrict__ x32, uint32_t* __restrict__ out, uint32_t selmask,
                                       int selprefix, int e_block) {
  uint32_t xb[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) xb[j] = x32[j];
  uint32_t pl[24];
  float xsum, fscale;
  act_planes_from_bits(xb, e_block, pl, &xsum, &fscale);
  uint4* o = reinterpret_cast<uint4*>(out);
#pragma unroll
  for (int q = 0; q < 6; ++q) o[q] = make_uint4(pl[4 * q], pl[4 * q + 1], pl[4 * q + 2], pl[4 * q + 3]);
  o[6] = make_uint4(__float_as_uint(xsum), __float_as_uint(fscale), selmask, static_cast<uint32_t>(selprefix));
  return xsum;
}

// The whole prepared form of one slab per thread (thread t = slab t of the
// warp-aligned range; every lane of the warp calls, `active` false beyond K):
// block exponent and block sum over groups of 4 lanes.
__device__ inline void act_write_slab_in_block(const uint16_t* __restrict__ x32, uint32_t* __restrict__ out,
                                               bool active, uint32_t selmask, int selprefix) {
  const int e = active ? act_slab_exponent(x32) : -1000;
  const int eb = act_block_exponent(e);
  const float xs = active ? act_write_slab(x32, out, selmask, selprefix, eb) : 0.0f;
  const float bs = act_block_sum(xs);
  if (active) reinterpret_cast<uint4*>(out)[7] = make_uint4(__float_as_uint(bs), 0u, 0u, 0u);
}

}  // namespace sfd
