// The elementwise producers of a GEMV input row (batch-1 decode step), shared
// by the stand-alone producer + selection kernels (decode_fused.cu) and the
// GEMV that computes its own input row (gemv_mma.cu), so both round the same
// values the same way.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace sfd {

__device__ __forceinline__ uint16_t to_bf16(double v) { return __bfloat16_as_ushort(__double2bfloat16(v)); }

// bf16(silu(g) u) rounded once from the exact value.  The fp32 evaluation
// r = fl(fl(g / fl(1 + expf(-g))) u) is within 7 * 2^-24 |r| of the exact
// value (expf within 2 ulp, CUDA math API accuracy table; four correctly
// rounded operations), i.e. within 16 steps of r's fp32 bit pattern even
// across a binade.  RNE to bf16 changes only at the midpoints (low 16 bits
// 0x8000), so when r's low half lies farther than 16 from 0x8000 the exact
// value rounds as r does; otherwise (and for non-normal or huge r) the value
// is recomputed in fp64 and rounded once.
__device__ __forceinline__ uint16_t silu_mul_bf16(float g, float u) {
  const float e = expf(-g);
  const float r = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, e)), u);
  const uint32_t b = __float_as_uint(r) & 0x7FFFFFFFu;
  const int low = static_cast<int>(b & 0xFFFFu);
  if (isfinite(e) && b >= 0x00800000u && b < 0x7E800000u && (low < 0x8000 - 16 || low > 0x8000 + 16))
    return __bfloat16_as_ushort(__float2bfloat16_rn(r));
  const double gv = g;
  return to_bf16(gv / (1.0 + exp(-gv)) * static_cast<double>(u));
}

// The RMSNorm's sum of squares is accumulated as 1024 threads would: thread t
// adds (fp64 fma) the squares of entries t, t + 1024, ... in that order, each
// warp of 32 such threads sums by an xor butterfly (offsets 16 .. 1), and the
// 32 warp totals are added in warp order.  Any block size computes this same
// order, so every kernel that normalises a row gets the same bits.
constexpr int kNormVThreads = 1024;

// RoPE of the pair (i, i + d/2) of one head at position pos: the angle
// pos theta^(-2i/d), its sine and cosine and the rotation in fp64 (each
// result rounded once by the caller).  Shared by every kernel that rotates,
// so a key rotated inside the K/V append equals one rotated on its own.
__device__ __forceinline__ void rope_pair(double lo, double hi, int i, int d, int pos, double theta, double& rlo,
                                          double& rhi) {
  const double ang = static_cast<double>(pos) * pow(theta, -2.0 * i / d);
  double s, c;
  sincos(ang, &s, &c);
  rlo = lo * c - hi * s;
  rhi = hi * c + lo * s;
}

}  // namespace sfd
