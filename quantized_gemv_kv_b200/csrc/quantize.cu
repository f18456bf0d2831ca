// sf_quantize_nested: nested min-max group quantization and packing.
//
// One CTA owns a tile of 32 rows x one group of G inputs.  Each warp reduces
// min/max of a row's group with shuffles, derives the fp16 scale and integer
// zero point, and writes the b-bit codes to shared memory; the CTA then
// assembles whole uint32 words of the resident stream (row-major) and of the
// refinement stream (column-major for weights, row-major for KV), so every
// word is written exactly once with no atomics.
#include "sf_internal.h"

namespace {

constexpr int kTileRows = 32;
constexpr int kThreads = 256;
constexpr int kMaxG = 512;

__global__ void __launch_bounds__(kThreads)
quantize_nested_kernel(const float* __restrict__ W, int N, int K, int G, int b_r, int b_f, int layout,
                       uint32_t* __restrict__ res, uint32_t* __restrict__ ref,
                       uint16_t* __restrict__ scale, uint16_t* __restrict__ zero) {
  extern __shared__ uint8_t codes[];  // [kTileRows][G]
  const int g = blockIdx.x;
  const int row0 = blockIdx.y * kTileRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = b_r + b_f;
  const float qmax = static_cast<float>((1 << b) - 1);
  const int per_lane = G >> 5;

  for (int rr = warp; rr < kTileRows; rr += kThreads / 32) {
    const int r = row0 + rr;
    if (r >= N) break;
    const float* src = W + static_cast<size_t>(r) * K + static_cast<size_t>(g) * G;
    float v[kMaxG / 32];
    float lo = INFINITY, hi = -INFINITY;
#pragma unroll 4
    for (int m = 0; m < per_lane; ++m) {
      v[m] = src[lane + 32 * m];
      lo = fminf(lo, v[m]);
      hi = fmaxf(hi, v[m]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    // scale: fp32 subtraction and division (IEEE, round to nearest), clamp to
    // the largest finite fp16, round to fp16 (nearest even); 0 -> 1.
    float q32 = __fdiv_rn(__fsub_rn(hi, lo), qmax);
    q32 = fminf(q32, 65504.0f);
    __half s16 = __float2half_rn(q32);
    if (__half2float(s16) == 0.0f) s16 = __float2half_rn(1.0f);
    const float sf = __half2float(s16);
    float zf = rintf(__fdiv_rn(-lo, sf));
    zf = fminf(fmaxf(zf, 0.0f), qmax);
    const int zi = static_cast<int>(zf);
    if (lane == 0) {
      scale[static_cast<size_t>(g) * N + r] = __half_as_ushort(s16);
      zero[static_cast<size_t>(g) * N + r] = __half_as_ushort(__int2half_rn(zi));
    }
    for (int m = 0; m < per_lane; ++m) {
      float qf = rintf(__fdiv_rn(v[m], sf)) + static_cast<float>(zi);
      qf = fminf(fmaxf(qf, 0.0f), qmax);
      codes[rr * G + lane + 32 * m] = static_cast<uint8_t>(static_cast<int>(qf));
    }
  }
  __syncthreads();

  const uint32_t rmask = (1u << b_r) - 1u, fmask = (1u << b_f) - 1u;
  const int rows_here = min(kTileRows, N - row0);
  // resident stream, row-major: a group of G codes is G*b_r/32 whole words
  const int rw = G * b_r / 32;
  const size_t res_row_words = static_cast<size_t>(K) * b_r / 32;
  for (int t = threadIdx.x; t < rows_here * rw; t += kThreads) {
    const int rr = t / rw, ww = t % rw;
    uint32_t word = 0;
    for (int bit = 0; bit < 32; ++bit) {
      const int sb = ww * 32 + bit;
      const uint32_t c = (codes[rr * G + sb / b_r] >> b_f) & rmask;
      word |= ((c >> (sb % b_r)) & 1u) << bit;
    }
    res[static_cast<size_t>(row0 + rr) * res_row_words + static_cast<size_t>(g) * rw + ww] = word;
  }
  if (layout == SF_REF_BY_COLUMN) {
    // column j's stream holds rows; this tile's 32 rows are b_f whole words
    const size_t col_words = static_cast<size_t>(N) * b_f / 32;
    for (int t = threadIdx.x; t < G * b_f; t += kThreads) {
      const int cc = t / b_f, ww = t % b_f;
      uint32_t word = 0;
      for (int bit = 0; bit < 32; ++bit) {
        const int sb = ww * 32 + bit;
        const uint32_t c = codes[(sb / b_f) * G + cc] & fmask;
        word |= ((c >> (sb % b_f)) & 1u) << bit;
      }
      ref[(static_cast<size_t>(g) * G + cc) * col_words + static_cast<size_t>(row0) * b_f / 32 + ww] = word;
    }
  } else {
    const int fw = G * b_f / 32;
    const size_t ref_row_words = static_cast<size_t>(K) * b_f / 32;
    for (int t = threadIdx.x; t < rows_here * fw; t += kThreads) {
      const int rr = t / fw, ww = t % fw;
      uint32_t word = 0;
      for (int bit = 0; bit < 32; ++bit) {
        const int sb = ww * 32 + bit;
        const uint32_t c = codes[rr * G + sb / b_f] & fmask;
        word |= ((c >> (sb % b_f)) & 1u) << bit;
      }
      ref[static_cast<size_t>(row0 + rr) * ref_row_words + static_cast<size_t>(g) * fw + ww] = word;
    }
  }
}

}  // namespace

extern "C" sf_status sf_quantize_nested(const float* W, int N, int K, int G, int b_r, int b_f, int layout,
                                        uint32_t* res_codes, uint32_t* ref_codes, uint16_t* scale,
                                        uint16_t* zero, sf_stream_t stream) {
  SF_REQUIRE(W && res_codes && ref_codes && scale && zero, "sf_quantize_nested: null pointer");
  SF_REQUIRE(b_r == 2 || b_r == 3, "sf_quantize_nested: b_r must be 2 or 3 (got %d)", b_r);
  SF_REQUIRE(b_f == 1 || b_f == 2, "sf_quantize_nested: b_f must be 1 or 2 (got %d)", b_f);
  SF_REQUIRE(b_r + b_f <= 4, "sf_quantize_nested: b_r + b_f must be <= 4");
  SF_REQUIRE(G >= 32 && G % 32 == 0 && G <= kMaxG, "sf_quantize_nested: G must be a multiple of 32 in [32, %d]", kMaxG);
  SF_REQUIRE(N >= 1 && K >= G && K % G == 0, "sf_quantize_nested: need N >= 1 and K a multiple of G");
  SF_REQUIRE(layout == SF_REF_BY_COLUMN || layout == SF_REF_BY_ROW, "sf_quantize_nested: unknown layout %d", layout);
  SF_REQUIRE(layout == SF_REF_BY_ROW || N % 32 == 0, "sf_quantize_nested: column layout needs N %% 32 == 0");
  dim3 grid(K / G, (N + kTileRows - 1) / kTileRows);
  SF_REQUIRE(grid.y <= 65535u, "sf_quantize_nested: N too large");
  const size_t smem = static_cast<size_t>(kTileRows) * G;
  quantize_nested_kernel<<<grid, kThreads, smem, sf::as_cuda(stream)>>>(W, N, K, G, b_r, b_f, layout, res_codes,
                                                                        ref_codes, scale, zero);
  return sf::check_launch("quantize_nested_kernel");
}
