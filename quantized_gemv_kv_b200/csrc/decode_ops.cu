// Elementwise operations of a decode step of a Llama-shaped layer: residual
// add with RMSNorm, RoPE of the new token's query and key heads, and the
// SiLU-gated product of the MLP.  The benchmark configuration names the
// shape (Llama-3.1-8B: RMSNorm, RoPE, SiLU MLP); the readings are the
// library's: eps given by the caller, RoPE in the rotate-half pairing with
// base theta and no frequency rescaling.  Each value is computed in fp64 and
// rounded once (to fp32 for the fp32 outputs, to bf16 with ties to even for
// the GEMV and attention inputs), so the results sit within one rounding of
// the exact values.
#include <cuda_bf16.h>

#include "sf_internal.h"

namespace {

constexpr int kNormThreads = 256;

__device__ __forceinline__ uint16_t to_bf16(double v) { return __bfloat16_as_ushort(__double2bfloat16(v)); }

// One CTA per row: x += delta (optional, fp32 written back), then
// y = bf16(x / sqrt(mean(x^2) + eps) * w).
__global__ void __launch_bounds__(kNormThreads)
add_rmsnorm_kernel(float* __restrict__ x, const float* __restrict__ delta, const float* __restrict__ w, int H,
                   float eps, uint16_t* __restrict__ y) {
  __shared__ double part[kNormThreads / 32];
  __shared__ double inv_sh;
  float* xr = x + static_cast<size_t>(blockIdx.x) * H;
  const float* dr = delta ? delta + static_cast<size_t>(blockIdx.x) * H : nullptr;
  uint16_t* yr = y + static_cast<size_t>(blockIdx.x) * H;
  double ss = 0.0;
  for (int i = threadIdx.x; i < H; i += kNormThreads) {
    float v = xr[i];
    if (dr) {
      v = __fadd_rn(v, dr[i]);
      xr[i] = v;
    }
    ss = fma(static_cast<double>(v), static_cast<double>(v), ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < kNormThreads / 32; ++i) t += part[i];
    inv_sh = 1.0 / sqrt(t / H + static_cast<double>(eps));
  }
  __syncthreads();
  const double inv = inv_sh;
  for (int i = threadIdx.x; i < H; i += kNormThreads)
    yr[i] = to_bf16(static_cast<double>(xr[i]) * inv * static_cast<double>(w[i]));
}

// One CTA per head, a thread per pair (i, i + d/2).
__global__ void rope_kernel(float* __restrict__ x, int d, int pos, double theta, uint16_t* __restrict__ y) {
  const int half = d >> 1, i = threadIdx.x;
  if (i >= half) return;
  const double ang = static_cast<double>(pos) * pow(theta, -2.0 * i / d);
  double s, c;
  sincos(ang, &s, &c);
  float* xh = x + static_cast<size_t>(blockIdx.x) * d;
  const double lo = xh[i], hi = xh[i + half];
  const double rlo = lo * c - hi * s, rhi = hi * c + lo * s;
  xh[i] = static_cast<float>(rlo);
  xh[i + half] = static_cast<float>(rhi);
  if (y) {
    uint16_t* yh = y + static_cast<size_t>(blockIdx.x) * d;
    yh[i] = to_bf16(rlo);
    yh[i + half] = to_bf16(rhi);
  }
}

__global__ void silu_mul_kernel(const float* __restrict__ g, const float* __restrict__ u, int n,
                                uint16_t* __restrict__ y) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const double gv = g[i];
    y[i] = to_bf16(gv / (1.0 + exp(-gv)) * static_cast<double>(u[i]));
  }
}

}  // namespace

extern "C" sf_status sf_add_rmsnorm(float* x, const float* delta, const float* w, int B, int H, float eps,
                                    uint16_t* y, sf_stream_t stream) {
  SF_REQUIRE(x && w && y, "sf_add_rmsnorm: null pointer");
  SF_REQUIRE(B >= 1 && H >= 1, "sf_add_rmsnorm: need B >= 1 and H >= 1");
  SF_REQUIRE(eps >= 0.0f, "sf_add_rmsnorm: eps must be >= 0");
  add_rmsnorm_kernel<<<B, kNormThreads, 0, sf::as_cuda(stream)>>>(x, delta, w, H, eps, y);
  return sf::check_launch("add_rmsnorm_kernel");
}

extern "C" sf_status sf_rope(float* x, int H, int d, int pos, double theta, uint16_t* y_bf16, sf_stream_t stream) {
  SF_REQUIRE(x, "sf_rope: null pointer");
  SF_REQUIRE(H >= 1 && d >= 2 && d % 2 == 0 && d <= 2048, "sf_rope: need H >= 1 and an even d in [2, 2048]");
  SF_REQUIRE(pos >= 0 && theta > 0.0, "sf_rope: need pos >= 0 and theta > 0");
  rope_kernel<<<H, ((d / 2 + 31) / 32) * 32, 0, sf::as_cuda(stream)>>>(x, d, pos, theta, y_bf16);
  return sf::check_launch("rope_kernel");
}

extern "C" sf_status sf_silu_mul(const float* g, const float* u, int n, uint16_t* y, sf_stream_t stream) {
  SF_REQUIRE(g && u && y, "sf_silu_mul: null pointer");
  SF_REQUIRE(n >= 1, "sf_silu_mul: n must be >= 1");
  const int blocks = std::min((n + 255) / 256, sf::sm_count() * 8);
  silu_mul_kernel<<<blocks, 256, 0, sf::as_cuda(stream)>>>(g, u, n, y);
  return sf::check_launch("silu_mul_kernel");
}
