// Per-token operations of a decode step of a Llama-shaped layer: residual
// add with RMSNorm, RoPE of the new token's query and key heads, the
// SiLU-gated product of the MLP, and the quantize-and-append of the new
// token's K or V rows into a cache allocated for a larger capacity.  The benchmark configuration names the
// shape (Llama-3.1-8B: RMSNorm, RoPE, SiLU MLP); the readings are the
// library's: eps given by the caller, RoPE in the rotate-half pairing with
// base theta and no frequency rescaling.  Each value is computed in fp64 and
// rounded once (to fp32 for the fp32 outputs, to bf16 with ties to even for
// the GEMV and attention inputs), so the results sit within one rounding of
// the exact values.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "produce.cuh"
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
  float* xh = x + static_cast<size_t>(blockIdx.x) * d;
  double rlo, rhi;
  sfd::rope_pair(xh[i], xh[i + half], i, d, pos, theta, rlo, rhi);
  xh[i] = static_cast<float>(rlo);
  xh[i + half] = static_cast<float>(rhi);
  if (y) {
    uint16_t* yh = y + static_cast<size_t>(blockIdx.x) * d;
    yh[i] = to_bf16(rlo);
    yh[i + half] = to_bf16(rhi);
  }
}

__global__ void round_bf16_kernel(const float* __restrict__ x, int n, uint16_t* __restrict__ y) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    y[i] = __bfloat16_as_ushort(__float2bfloat16_rn(x[i]));
}

__global__ void silu_mul_kernel(const float* __restrict__ g, const float* __restrict__ u, int n,
                                uint16_t* __restrict__ y) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const double gv = g[i];
    y[i] = to_bf16(gv / (1.0 + exp(-gv)) * static_cast<double>(u[i]));
  }
}

constexpr int kAppendMaxD = 512;

// One warp per KV head: the new token's row of d values is quantized as one
// group with the arithmetic of the nested quantizer (min/max, fp32 division,
// fp16 scale, integer zero point, ties to even) and written as cache row
// g * row_stride + t: resident and refinement bitstreams (row-major, little
// endian), fp16 scale and zero.  The refinement words go to ref_row and, when
// crow is not null (the unit is cached), to crow as well, so a cached copy
// never goes stale.  With rope_pos >= 0 the row is first rotated to that
// position (sfd::rope_pair, each value rounded to fp32 once, d a multiple of
// 64 so that a lane holds both dims of its pairs) and written back to rot_out.
// PER: d / 32 known at compile time (the row stays in registers), 0: any d.
template <int PER>
__device__ void append_row(const float* __restrict__ row, int d, int b_r, int b_f, size_t r, uint32_t* __restrict__ res,
                           uint16_t* __restrict__ scale, uint16_t* __restrict__ zero, uint32_t* __restrict__ ref_row,
                           uint32_t* __restrict__ crow, uint8_t* codes, int rope_pos = -1, double theta = 0.0,
                           float* rot_out = nullptr) {
  constexpr int kMax = PER > 0 ? PER : kAppendMaxD / 32;
  const int lane = threadIdx.x & 31;
  const int b = b_r + b_f;
  const float qmax = static_cast<float>((1 << b) - 1);
  const int per_lane = PER > 0 ? PER : d >> 5;
  float v[kMax];
#pragma unroll
  for (int m = 0; m < kMax; ++m)
    if (m < per_lane) v[m] = row[lane + 32 * m];
  if (rope_pos >= 0) {
    const int hm = per_lane >> 1;  // dim lane + 32 m pairs with dim lane + 32 (m + hm)
#pragma unroll
    for (int m = 0; m < kMax / 2; ++m)
      if (m < hm) {
        double rlo, rhi;
        sfd::rope_pair(v[m], v[m + hm], lane + 32 * m, d, rope_pos, theta, rlo, rhi);
        v[m] = static_cast<float>(rlo);
        v[m + hm] = static_cast<float>(rhi);
      }
#pragma unroll
    for (int m = 0; m < kMax; ++m)
      if (m < per_lane) rot_out[lane + 32 * m] = v[m];
  }
  float lo = INFINITY, hi = -INFINITY;
#pragma unroll
  for (int m = 0; m < kMax; ++m)
    if (m < per_lane) {
      lo = fminf(lo, v[m]);
      hi = fmaxf(hi, v[m]);
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  float q32 = __fdiv_rn(__fsub_rn(hi, lo), qmax);
  q32 = fminf(q32, 65504.0f);
  __half s16 = __float2half_rn(q32);
  if (__half2float(s16) == 0.0f) s16 = __float2half_rn(1.0f);
  const float sf = __half2float(s16);
  float zf = rintf(__fdiv_rn(-lo, sf));
  zf = fminf(fmaxf(zf, 0.0f), qmax);
  const int zi = static_cast<int>(zf);
  if (lane == 0) {
    scale[r] = __half_as_ushort(s16);
    zero[r] = __half_as_ushort(__int2half_rn(zi));
  }
#pragma unroll
  for (int m = 0; m < kMax; ++m)
    if (m < per_lane) {
      float qf = rintf(__fdiv_rn(v[m], sf)) + static_cast<float>(zi);
      qf = fminf(fmaxf(qf, 0.0f), qmax);
      codes[lane + 32 * m] = static_cast<uint8_t>(static_cast<int>(qf));
    }
  __syncwarp();
  const uint32_t rmask = (1u << b_r) - 1u, fmask = (1u << b_f) - 1u;
  const int rw = d * b_r / 32, fw = d * b_f / 32;
  for (int ww = lane; ww < rw; ww += 32) {
    uint32_t word = 0;
    for (int bit = 0; bit < 32; ++bit) {
      const int sb = ww * 32 + bit;
      word |= (((static_cast<uint32_t>(codes[sb / b_r]) >> b_f) & rmask) >> (sb % b_r) & 1u) << bit;
    }
    res[r * rw + ww] = word;
  }
  for (int ww = lane; ww < fw; ww += 32) {
    uint32_t word = 0;
    for (int bit = 0; bit < 32; ++bit) {
      const int sb = ww * 32 + bit;
      word |= ((static_cast<uint32_t>(codes[sb / b_f]) & fmask) >> (sb % b_f) & 1u) << bit;
    }
    ref_row[ww] = word;
    if (crow != nullptr) crow[ww] = word;
  }
}

// The refinement words go to ref + r * ref_pitch + ref_off (the store: pitch
// d*b_f/32, offset 0; a KV refinement cache's host master: the unit's pitch
// and the K or V half); unit_slot / crows: the cache's slots and rows.
__global__ void kv_append_kernel(const float* __restrict__ src, int Hkv, int d, int row_stride, int t, int b_r,
                                 int b_f, uint32_t* __restrict__ res, uint32_t* __restrict__ ref, int ref_pitch,
                                 int ref_off, const int32_t* __restrict__ unit_slot, uint32_t* __restrict__ crows,
                                 uint16_t* __restrict__ scale, uint16_t* __restrict__ zero) {
  __shared__ uint8_t codes[4][kAppendMaxD];
  const int warp = threadIdx.x >> 5;
  const int g = blockIdx.x * 4 + warp;
  if (g >= Hkv) return;  // uniform over the warp
  const size_t r = static_cast<size_t>(g) * row_stride + t;
  uint32_t* crow = nullptr;
  if (unit_slot != nullptr) {
    const int slot = unit_slot[r];
    if (slot >= 0) crow = crows + static_cast<size_t>(slot) * ref_pitch + ref_off;
  }
  if (d == 128)
    append_row<4>(src + static_cast<size_t>(g) * d, d, b_r, b_f, r, res, scale, zero, ref + r * ref_pitch + ref_off,
                  crow, codes[warp]);
  else
    append_row<0>(src + static_cast<size_t>(g) * d, d, b_r, b_f, r, res, scale, zero, ref + r * ref_pitch + ref_off,
                  crow, codes[warp]);
}

// The key and value rows of token t in one launch (blockIdx.y: 0 keys, 1
// values); the refinement words go to the device staging rows stage[g] (K
// words, then V words: the unit's layout) and to the cached copy of a cached
// unit.
struct AppendPair {
  const float* src[2];
  uint32_t* res[2];
  uint16_t* scale[2];
  uint16_t* zero[2];
  uint32_t* stage;
  const int32_t* unit_slot;
  uint32_t* crows;
  int Hkv, d, row_stride, t, b_r, b_f;
  // RoPE to position rope_pos (< 0: none) of the keys, rotated in place in
  // src[0] before they are quantized, and of the Hq query heads in q (in
  // place, and as bf16 to q_bf16 when it is not null), by blockIdx.y == 2
  int rope_pos, Hq;
  double theta;
  float* k_rot;
  float* q;
  uint16_t* q_bf16;
};

__global__ void kv_append_pair_kernel(const __grid_constant__ AppendPair A) {
  __shared__ uint8_t codes[4][kAppendMaxD];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, part = blockIdx.y;
  const int g = blockIdx.x * 4 + warp;
  if (part == 2) {  // a warp per query head
    if (g >= A.Hq) return;  // uniform over the warp
    float* xh = A.q + static_cast<size_t>(g) * A.d;
    const int half = A.d >> 1;
    for (int i = lane; i < half; i += 32) {
      double rlo, rhi;
      sfd::rope_pair(xh[i], xh[i + half], i, A.d, A.rope_pos, A.theta, rlo, rhi);
      xh[i] = static_cast<float>(rlo);
      xh[i + half] = static_cast<float>(rhi);
      if (A.q_bf16 != nullptr) {
        uint16_t* yh = A.q_bf16 + static_cast<size_t>(g) * A.d;
        yh[i] = sfd::to_bf16(rlo);
        yh[i + half] = sfd::to_bf16(rhi);
      }
    }
    return;
  }
  if (g >= A.Hkv) return;  // uniform over the warp
  const int fw = A.d * A.b_f / 32;
  const size_t r = static_cast<size_t>(g) * A.row_stride + A.t;
  const int slot = A.unit_slot[r];
  uint32_t* crow = slot >= 0 ? A.crows + static_cast<size_t>(slot) * 2 * fw + part * fw : nullptr;
  const bool rot = part == 0 && A.rope_pos >= 0;
  const float* row = A.src[part] + static_cast<size_t>(g) * A.d;
  uint32_t* stage = A.stage + static_cast<size_t>(g) * 2 * fw + part * fw;
  float* rot_out = rot ? A.k_rot + static_cast<size_t>(g) * A.d : nullptr;
  if (A.d == 128)
    append_row<4>(row, A.d, A.b_r, A.b_f, r, A.res[part], A.scale[part], A.zero[part], stage, crow, codes[warp],
                  rot ? A.rope_pos : -1, A.theta, rot_out);
  else
    append_row<0>(row, A.d, A.b_r, A.b_f, r, A.res[part], A.scale[part], A.zero[part], stage, crow, codes[warp],
                  rot ? A.rope_pos : -1, A.theta, rot_out);
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

extern "C" sf_status sf_round_bf16(const float* x, int n, uint16_t* y, sf_stream_t stream) {
  SF_REQUIRE(x && y, "sf_round_bf16: null pointer");
  SF_REQUIRE(n >= 1, "sf_round_bf16: n must be >= 1");
  const int blocks = std::min((n + 255) / 256, sf::sm_count() * 8);
  round_bf16_kernel<<<blocks, 256, 0, sf::as_cuda(stream)>>>(x, n, y);
  return sf::check_launch("round_bf16_kernel");
}

extern "C" sf_status sf_kv_append(const float* src, int Hkv, int d, int row_stride, int t, int b_r, int b_f,
                                  uint32_t* res, uint32_t* ref, uint16_t* scale, uint16_t* zero, sf_stream_t stream) {
  SF_REQUIRE(src && res && ref && scale && zero, "sf_kv_append: null pointer");
  SF_REQUIRE(Hkv >= 1, "sf_kv_append: Hkv must be >= 1");
  SF_REQUIRE(d >= 32 && d % 32 == 0 && d <= kAppendMaxD, "sf_kv_append: d must be a multiple of 32 in [32, %d]",
             kAppendMaxD);
  SF_REQUIRE(b_r == 2 || b_r == 3, "sf_kv_append: b_r must be 2 or 3");
  SF_REQUIRE(b_f == 1 || b_f == 2, "sf_kv_append: b_f must be 1 or 2");
  SF_REQUIRE(b_r + b_f <= 4, "sf_kv_append: b_r + b_f must be <= 4");
  SF_REQUIRE(row_stride >= 1 && t >= 0 && t < row_stride, "sf_kv_append: need 0 <= t < row_stride");
  kv_append_kernel<<<(Hkv + 3) / 4, 128, 0, sf::as_cuda(stream)>>>(src, Hkv, d, row_stride, t, b_r, b_f, res, ref,
                                                                   d * b_f / 32, 0, nullptr, nullptr, scale, zero);
  return sf::check_launch("kv_append_kernel");
}

namespace {

// The pair append, with RoPE of q and k in the same launch when q is given.
sf_status append_pair(const char* what, float* q, int Hq, uint16_t* q_bf16, int pos, double theta, const float* k_src,
                      const float* v_src, int Hkv, int d, int row_stride, int t, int b_r, int b_f, uint32_t* k_res,
                      uint16_t* k_scale, uint16_t* k_zero, uint32_t* v_res, uint16_t* v_scale, uint16_t* v_zero,
                      sf_refine_cache* ref_cache, sf_stream_t stream, sf_stream_t side) {
  SF_REQUIRE(k_src && v_src && k_res && k_scale && k_zero && v_res && v_scale && v_zero && ref_cache,
             "%s: null pointer", what);
  SF_REQUIRE(Hkv >= 1, "%s: Hkv must be >= 1", what);
  SF_REQUIRE(d >= 32 && d % 32 == 0 && d <= kAppendMaxD, "%s: d must be a multiple of 32 in [32, %d]", what,
             kAppendMaxD);
  SF_REQUIRE(b_r == 2 || b_r == 3, "%s: b_r must be 2 or 3", what);
  SF_REQUIRE(b_f == 1 || b_f == 2, "%s: b_f must be 1 or 2", what);
  SF_REQUIRE(b_r + b_f <= 4, "%s: b_r + b_f must be <= 4", what);
  SF_REQUIRE(row_stride >= 1 && t >= 0 && t < row_stride, "%s: need 0 <= t < row_stride", what);
  if (q != nullptr) {
    SF_REQUIRE(Hq >= 1 && d % 64 == 0, "%s: need Hq >= 1 and d a multiple of 64 for the rotation", what);
    SF_REQUIRE(pos >= 0 && theta > 0.0, "%s: need pos >= 0 and theta > 0", what);
  }
  cudaStream_t s = sf::as_cuda(stream);
  sf::CacheWriteView w{};
  sf_status st = sf::cache_view_for_writer(ref_cache, s, &w);
  if (st != SF_OK) return st;
  const int fw = d * b_f / 32;
  SF_REQUIRE(w.unit_words == 2 * fw, "%s: the cache's units must be %d bytes (K then V words)", what, 8 * fw);
  SF_REQUIRE(static_cast<long long>(w.num_units) >= static_cast<long long>(Hkv) * row_stride,
             "%s: the cache has fewer units than Hkv * row_stride", what);
  uint32_t* stage = nullptr;
  st = sf::cache_append_stage(ref_cache, s, static_cast<size_t>(Hkv) * 2 * fw, &stage);
  if (st != SF_OK) return st;
  AppendPair A{};
  A.src[0] = k_src;
  A.src[1] = v_src;
  A.res[0] = k_res;
  A.res[1] = v_res;
  A.scale[0] = k_scale;
  A.scale[1] = v_scale;
  A.zero[0] = k_zero;
  A.zero[1] = v_zero;
  A.stage = stage;
  A.unit_slot = w.unit_slot;
  A.crows = w.rows;
  A.Hkv = Hkv;
  A.d = d;
  A.row_stride = row_stride;
  A.t = t;
  A.b_r = b_r;
  A.b_f = b_f;
  A.rope_pos = q != nullptr ? pos : -1;
  A.Hq = q != nullptr ? Hq : 0;
  A.theta = theta;
  A.k_rot = const_cast<float*>(k_src);
  A.q = q;
  A.q_bf16 = q_bf16;
  const int gx = std::max((Hkv + 3) / 4, (A.Hq + 3) / 4);
  kv_append_pair_kernel<<<dim3(gx, q != nullptr ? 3 : 2), 128, 0, s>>>(A);
  st = sf::check_launch("kv_append_pair_kernel");
  if (st != SF_OK) return st;
  st = sf::cache_mark_used(ref_cache, s);
  if (st != SF_OK) return st;
  // rows g * row_stride + t of the master, one per KV head
  return sf::cache_append_flush(ref_cache, s, sf::as_cuda(side), static_cast<size_t>(t) * 2 * fw * 4,
                                static_cast<size_t>(row_stride) * 2 * fw * 4, static_cast<size_t>(2 * fw) * 4, Hkv);
}

}  // namespace

extern "C" sf_status sf_kv_append_pair_cached(const float* k_src, const float* v_src, int Hkv, int d, int row_stride,
                                              int t, int b_r, int b_f, uint32_t* k_res, uint16_t* k_scale,
                                              uint16_t* k_zero, uint32_t* v_res, uint16_t* v_scale, uint16_t* v_zero,
                                              sf_refine_cache* ref_cache, sf_stream_t stream, sf_stream_t side) {
  return append_pair("sf_kv_append_pair_cached", nullptr, 0, nullptr, 0, 0.0, k_src, v_src, Hkv, d, row_stride, t,
                     b_r, b_f, k_res, k_scale, k_zero, v_res, v_scale, v_zero, ref_cache, stream, side);
}

extern "C" sf_status sf_rope_kv_append_pair_cached(float* q, int Hq, uint16_t* q_bf16, float* k, const float* v,
                                                   int Hkv, int d, int pos, double theta, int row_stride, int t,
                                                   int b_r, int b_f, uint32_t* k_res, uint16_t* k_scale,
                                                   uint16_t* k_zero, uint32_t* v_res, uint16_t* v_scale,
                                                   uint16_t* v_zero, sf_refine_cache* ref_cache, sf_stream_t stream,
                                                   sf_stream_t side) {
  SF_REQUIRE(q, "sf_rope_kv_append_pair_cached: null pointer");
  return append_pair("sf_rope_kv_append_pair_cached", q, Hq, q_bf16, pos, theta, k, v, Hkv, d, row_stride, t, b_r,
                     b_f, k_res, k_scale, k_zero, v_res, v_scale, v_zero, ref_cache, stream, side);
}

extern "C" sf_status sf_kv_append_cached(const float* src, int Hkv, int d, int row_stride, int t, int b_r, int b_f,
                                         uint32_t* res, uint16_t* scale, uint16_t* zero, sf_refine_cache* ref_cache,
                                         int part, sf_stream_t stream) {
  SF_REQUIRE(src && res && scale && zero && ref_cache, "sf_kv_append_cached: null pointer");
  SF_REQUIRE(Hkv >= 1, "sf_kv_append_cached: Hkv must be >= 1");
  SF_REQUIRE(d >= 32 && d % 32 == 0 && d <= kAppendMaxD,
             "sf_kv_append_cached: d must be a multiple of 32 in [32, %d]", kAppendMaxD);
  SF_REQUIRE(b_r == 2 || b_r == 3, "sf_kv_append_cached: b_r must be 2 or 3");
  SF_REQUIRE(b_f == 1 || b_f == 2, "sf_kv_append_cached: b_f must be 1 or 2");
  SF_REQUIRE(b_r + b_f <= 4, "sf_kv_append_cached: b_r + b_f must be <= 4");
  SF_REQUIRE(row_stride >= 1 && t >= 0 && t < row_stride, "sf_kv_append_cached: need 0 <= t < row_stride");
  SF_REQUIRE(part == 0 || part == 1, "sf_kv_append_cached: part must be 0 (K) or 1 (V)");
  cudaStream_t s = sf::as_cuda(stream);
  sf::CacheWriteView w{};
  sf_status st = sf::cache_view_for_writer(ref_cache, s, &w);
  if (st != SF_OK) return st;
  const int fw = d * b_f / 32;
  SF_REQUIRE(w.unit_words == 2 * fw, "sf_kv_append_cached: the cache's units must be %d bytes (K then V words)",
             8 * fw);
  SF_REQUIRE(static_cast<long long>(w.num_units) >= static_cast<long long>(Hkv) * row_stride,
             "sf_kv_append_cached: the cache has fewer units than Hkv * row_stride");
  kv_append_kernel<<<(Hkv + 3) / 4, 128, 0, s>>>(src, Hkv, d, row_stride, t, b_r, b_f, res, w.master, 2 * fw,
                                                 part * fw, w.unit_slot, w.rows, scale, zero);
  st = sf::check_launch("kv_append_kernel");
  if (st != SF_OK) return st;
  return sf::cache_mark_used(ref_cache, s);
}

