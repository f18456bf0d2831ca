// sf_gemv_refine: refined decode GEMV over packed low-bit resident weights.
//
//   y[b][i] = sum_j x[b][j] w_res[i][j] + sum_{j in S} x[b][j] s_{g(j),i} (q_f[i][j] - m_f)
//
// (nested refinement applied to the columns with the largest activations,
// rag-lover.com explainer of StrataFlux, 解説).  Per 32-column slab of a row
// the resident part is factored as
//   s * (2^b_f * sum_j x_j c_j + (m_f - z) * sum_j x_j),
// so the inner loop is one code unpack and one FMA per weight, and the scale
// and zero point are applied once per slab.  The correction over the
// selected columns runs as an epilogue of the same CTA, reading each column's
// refinement bits from the cache slot (or the HBM store) with lanes mapped to
// the tile's 32 rows.
#include <algorithm>

#include "sf_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTileRows = 32;
constexpr int kXSmemFloats = 24576;  // x chunk budget in shared memory (96 KB)

template <int BR>
__device__ __forceinline__ uint32_t slab_code(const uint32_t (&w)[BR], int j) {
  if constexpr (BR == 2) {
    return (w[j >> 4] >> ((j & 15) * 2)) & 3u;
  } else {
    const int bit = 3 * j, word = bit >> 5, sh = bit & 31;
    uint32_t v = w[word] >> sh;
    if (sh > 29) v |= w[word + 1] << (32 - sh);
    return v & 7u;
  }
}

// MODE 0: refinement bits (ref_rows: rows of N*b_f/32 words); MODE 1: FP16
// fetch, the selected columns' fp16 residuals w - w_res (ref_rows: rows of N
// halves), the comparator of the explainer's 既存手法との違い.
template <int BR, int NB, int MODE>
__global__ void __launch_bounds__(kThreads)
gemv_refine_kernel(const uint32_t* __restrict__ res, const uint16_t* __restrict__ scale,
                   const uint16_t* __restrict__ zero, int N, int K, int G, int b_f, const uint16_t* __restrict__ x,
                   int B, int kc, const int32_t* __restrict__ idx, const int32_t* __restrict__ n_sel,
                   const uint32_t* __restrict__ ref_rows, const int32_t* __restrict__ row_of, int unit_words,
                   float* __restrict__ y, int accumulate) {
  extern __shared__ float smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = blockIdx.x * kTileRows;
  const int k0 = blockIdx.y * kc;
  const int k1 = min(K, k0 + kc);
  const int ncol = k1 - k0;
  const int nslab = ncol >> 5;
  float* xs = smem;                       // [NB][32][nslab]: xs[(b*32+j)*nslab + s] = x[b][k0+32s+j]
  float* xsum = xs + NB * ncol;           // [NB][nslab]
  float* ysm = xsum + NB * nslab;         // [NB][kTileRows]

  for (int e = tid; e < NB * ncol; e += kThreads) {
    const int b = e / ncol, c = e - b * ncol;
    const float v = b < B ? sfd::bf16_bits_to_float(x[static_cast<size_t>(b) * K + k0 + c]) : 0.0f;
    xs[(b * 32 + (c & 31)) * nslab + (c >> 5)] = v;
  }
  for (int e = tid; e < NB * kTileRows; e += kThreads) ysm[e] = 0.0f;
  __syncthreads();
  for (int e = tid; e < NB * nslab; e += kThreads) {
    const int b = e / nslab, s = e - b * nslab;
    float t = 0.0f;
#pragma unroll 8
    for (int j = 0; j < 32; ++j) t += xs[(b * 32 + j) * nslab + s];
    xsum[e] = t;
  }
  __syncthreads();

  const float m_f = static_cast<float>((1 << b_f) - 1) * 0.5f;
  const float two_bf = static_cast<float>(1 << b_f);
  const size_t row_words = static_cast<size_t>(K) * BR / 32;
  const int slab0 = k0 >> 5;

  for (int i = warp; i < kTileRows; i += kWarps) {
    const int r = row0 + i;
    const uint32_t* rrow = res + static_cast<size_t>(r) * row_words;
    float acc[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[b] = 0.0f;
    for (int s = lane; s < nslab; s += 32) {
      const int gs = slab0 + s;
      uint32_t w[BR];
#pragma unroll
      for (int q = 0; q < BR; ++q) w[q] = __ldg(rrow + static_cast<size_t>(gs) * BR + q);
      const int g = (gs * 32) / G;
      const float sc = sfd::half_bits_to_float(__ldg(scale + static_cast<size_t>(g) * N + r));
      const float zz = sfd::half_bits_to_float(__ldg(zero + static_cast<size_t>(g) * N + r));
      float P[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) P[b] = 0.0f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float c = static_cast<float>(slab_code<BR>(w, j));
#pragma unroll
        for (int b = 0; b < NB; ++b) P[b] = fmaf(xs[(b * 32 + j) * nslab + s], c, P[b]);
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[b] = fmaf(sc, fmaf(two_bf, P[b], (m_f - zz) * xsum[b * nslab + s]), acc[b]);
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float v = acc[b];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) ysm[b * kTileRows + i] = v;
    }
  }
  __syncthreads();

  // refinement correction for the selected columns inside this K chunk
  if (ref_rows != nullptr) {
    int n = *n_sel;
    n = n < 0 ? 0 : n;
    const uint32_t fmask = (1u << b_f) - 1u;
    const int i = row0 + lane;
    const int bitpos = i * b_f;
    float corr[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) corr[b] = 0.0f;
    for (int p = warp; p < n; p += kWarps) {
      const int j = idx[p];
      if (j < k0 || j >= k1) continue;
      const int rid = row_of ? row_of[p] : j;
      float d;
      if constexpr (MODE == 0) {
        const uint32_t word = ref_rows[static_cast<size_t>(rid) * unit_words + (bitpos >> 5)];
        const float qf = static_cast<float>((word >> (bitpos & 31)) & fmask);
        const float sc = sfd::half_bits_to_float(scale[static_cast<size_t>(j / G) * N + i]);
        d = sc * (qf - m_f);
      } else {
        d = sfd::half_bits_to_float(reinterpret_cast<const uint16_t*>(ref_rows)[static_cast<size_t>(rid) * N + i]);
      }
      const int c = j - k0;
#pragma unroll
      for (int b = 0; b < NB; ++b) corr[b] = fmaf(xs[(b * 32 + (c & 31)) * nslab + (c >> 5)], d, corr[b]);
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) atomicAdd(&ysm[b * kTileRows + lane], corr[b]);
    __syncthreads();
  }

  for (int e = tid; e < B * kTileRows; e += kThreads) {
    const int b = e / kTileRows, rr = e - b * kTileRows;
    float* dst = y + static_cast<size_t>(b) * N + row0 + rr;
    if (accumulate) atomicAdd(dst, ysm[b * kTileRows + rr]);
    else *dst = ysm[b * kTileRows + rr];
  }
}

template <int BR, int NB, int MODE>
sf_status launch_nb(const sf_qweight* W, const uint16_t* x, int B, const int32_t* idx, const int32_t* n,
                    const uint32_t* ref_rows, const int32_t* row_of, int unit_words, float* y, cudaStream_t s) {
  int kc = kXSmemFloats / NB;
  kc = std::max(W->G, kc / W->G * W->G);
  kc = std::min(kc, W->K);
  const int splits = (W->K + kc - 1) / kc;
  const size_t smem = sizeof(float) * (static_cast<size_t>(NB) * kc + NB * (kc / 32) + NB * kTileRows);
  SF_CHECK_CUDA(cudaFuncSetAttribute(gemv_refine_kernel<BR, NB, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)));
  if (splits > 1) SF_CHECK_CUDA(cudaMemsetAsync(y, 0, sizeof(float) * B * W->N, s));
  dim3 grid(W->N / kTileRows, splits);
  gemv_refine_kernel<BR, NB, MODE><<<grid, kThreads, smem, s>>>(W->res, W->scale, W->zero, W->N, W->K, W->G, W->b_f, x, B,
                                                          kc, idx, n, ref_rows, row_of, unit_words, y, splits > 1);
  return sf::check_launch("gemv_refine_kernel");
}

template <int BR, int MODE>
sf_status launch_br(const sf_qweight* W, const uint16_t* x, int B, const int32_t* idx, const int32_t* n,
                    const uint32_t* ref_rows, const int32_t* row_of, int unit_words, float* y, cudaStream_t s) {
  if (B <= 1) return launch_nb<BR, 1, MODE>(W, x, B, idx, n, ref_rows, row_of, unit_words, y, s);
  if (B <= 2) return launch_nb<BR, 2, MODE>(W, x, B, idx, n, ref_rows, row_of, unit_words, y, s);
  if (B <= 4) return launch_nb<BR, 4, MODE>(W, x, B, idx, n, ref_rows, row_of, unit_words, y, s);
  if (B <= 8) return launch_nb<BR, 8, MODE>(W, x, B, idx, n, ref_rows, row_of, unit_words, y, s);
  return launch_nb<BR, 16, MODE>(W, x, B, idx, n, ref_rows, row_of, unit_words, y, s);
}

// fp16 residual of the fp32 weights against their resident values, one
// thread per weight: the difference is exact in fp64, rounded once.
__global__ void residual_kernel(const float* __restrict__ W, const uint32_t* __restrict__ res,
                               const uint16_t* __restrict__ scale, const uint16_t* __restrict__ zero, int N, int K,
                               int G, int b_r, int b_f, uint16_t* __restrict__ out) {
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= static_cast<long long>(N) * K) return;
  const int j = static_cast<int>(e / N), i = static_cast<int>(e % N);  // out is column-major [K][N]
  const size_t row_words = static_cast<size_t>(K) * b_r / 32;
  const uint32_t c = sfd::read_bits(res + i * row_words, static_cast<uint32_t>(j) * b_r, b_r);
  const double s = sfd::half_bits_to_float(scale[static_cast<size_t>(j / G) * N + i]);
  const double z = sfd::half_bits_to_float(zero[static_cast<size_t>(j / G) * N + i]);
  const double m_f = ((1 << b_f) - 1) * 0.5;
  const double w_res = s * (static_cast<double>(c) * (1 << b_f) + m_f - z);
  out[e] = __half_as_ushort(__double2half(static_cast<double>(W[static_cast<size_t>(i) * K + j]) - w_res));
}

}  // namespace

extern "C" sf_status sf_gemv_refine(const sf_qweight* W, const uint16_t* x, int B, const int32_t* idx,
                                    const int32_t* n, sf_refine_cache* c, float* y, sf_stream_t stream) {
  SF_REQUIRE(W && x && y, "sf_gemv_refine: null pointer");
  SF_REQUIRE(W->res && W->scale && W->zero, "sf_gemv_refine: null weight view");
  SF_REQUIRE(B >= 1 && B <= 16, "sf_gemv_refine: B must be in [1, 16]");
  SF_REQUIRE(W->b_r == 2 || W->b_r == 3, "sf_gemv_refine: b_r must be 2 or 3");
  SF_REQUIRE(W->b_f == 1 || W->b_f == 2, "sf_gemv_refine: b_f must be 1 or 2");
  SF_REQUIRE(W->G >= 32 && W->G % 32 == 0 && W->K % W->G == 0, "sf_gemv_refine: need G %% 32 == 0 and K %% G == 0");
  SF_REQUIRE(W->K >= 32 && W->K <= 32768, "sf_gemv_refine: K must be in [32, 32768]");
  SF_REQUIRE(W->N >= 32 && W->N % 32 == 0, "sf_gemv_refine: N must be a positive multiple of 32");
  cudaStream_t s = sf::as_cuda(stream);
  const uint32_t* ref_rows = nullptr;
  const int32_t* row_of = nullptr;
  int unit_words = W->N * W->b_f / 32;
  int nmax = W->K;  // largest selection the correction may see
  if (c) {
    SF_REQUIRE(idx && n, "sf_gemv_refine: a cache needs the selection (idx, n)");
    sf::CacheView v{};
    sf_status st = sf::cache_view_for_gemv(c, s, &v);
    if (st != SF_OK) return st;
    SF_REQUIRE(v.unit_words == unit_words, "sf_gemv_refine: cache unit size does not match N*b_f/8");
    ref_rows = v.rows;
    row_of = v.row_of;
    nmax = v.max_select;
  } else if (W->ref) {
    SF_REQUIRE(idx && n, "sf_gemv_refine: a refinement store needs the selection (idx, n)");
    ref_rows = W->ref;
  }
  sf_status st = SF_OK;
  if (!(B == 1 && sf::gemv_b1_try(W, x, idx, n, ref_rows, row_of, unit_words, nmax, y, s, &st)) &&
      !(B >= 2 && sf::gemv_tc_try(W, x, B, idx, n, ref_rows, row_of, unit_words, y, s, &st)))
    st = W->b_r == 2 ? launch_br<2, 0>(W, x, B, idx, n, ref_rows, row_of, unit_words, y, s)
                     : launch_br<3, 0>(W, x, B, idx, n, ref_rows, row_of, unit_words, y, s);
  if (st != SF_OK) return st;
  if (c) return sf::cache_mark_used(c, s);
  return SF_OK;
}

extern "C" sf_status sf_quantize_residual(const float* W, const sf_qweight* Wq, uint16_t* out, sf_stream_t stream) {
  SF_REQUIRE(W && Wq && out && Wq->res && Wq->scale && Wq->zero, "sf_quantize_residual: null pointer");
  SF_REQUIRE((Wq->b_r == 2 || Wq->b_r == 3) && (Wq->b_f == 1 || Wq->b_f == 2) && Wq->G >= 32 && Wq->G % 32 == 0 &&
                 Wq->K % Wq->G == 0 && Wq->N >= 1,
             "sf_quantize_residual: shape outside sf_quantize_nested's contract");
  const long long total = static_cast<long long>(Wq->N) * Wq->K;
  residual_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, sf::as_cuda(stream)>>>(
      W, Wq->res, Wq->scale, Wq->zero, Wq->N, Wq->K, Wq->G, Wq->b_r, Wq->b_f, out);
  return sf::check_launch("residual_kernel");
}

extern "C" sf_status sf_gemv_fp16_fetch(const sf_qweight* W, const uint16_t* x, int B, const int32_t* idx,
                                        const int32_t* n, const uint16_t* resid, sf_refine_cache* c, float* y,
                                        sf_stream_t stream) {
  SF_REQUIRE(W && x && y && idx && n, "sf_gemv_fp16_fetch: null pointer");
  SF_REQUIRE(W->res && W->scale && W->zero, "sf_gemv_fp16_fetch: null weight view");
  SF_REQUIRE((resid != nullptr) != (c != nullptr), "sf_gemv_fp16_fetch: give exactly one of resid and c");
  SF_REQUIRE(B >= 1 && B <= 16, "sf_gemv_fp16_fetch: B must be in [1, 16]");
  SF_REQUIRE(W->b_r == 2 || W->b_r == 3, "sf_gemv_fp16_fetch: b_r must be 2 or 3");
  SF_REQUIRE(W->b_f == 1 || W->b_f == 2, "sf_gemv_fp16_fetch: b_f must be 1 or 2");
  SF_REQUIRE(W->G >= 32 && W->G % 32 == 0 && W->K % W->G == 0, "sf_gemv_fp16_fetch: need G %% 32 == 0, K %% G == 0");
  SF_REQUIRE(W->K >= 32 && W->K <= 32768, "sf_gemv_fp16_fetch: K must be in [32, 32768]");
  SF_REQUIRE(W->N >= 32 && W->N % 32 == 0, "sf_gemv_fp16_fetch: N must be a positive multiple of 32");
  cudaStream_t s = sf::as_cuda(stream);
  const uint32_t* rows = reinterpret_cast<const uint32_t*>(resid);
  const int32_t* row_of = nullptr;
  const int unit_words = W->N / 2;
  if (c) {
    sf::CacheView v{};
    const sf_status st = sf::cache_view_for_gemv(c, s, &v);
    if (st != SF_OK) return st;
    SF_REQUIRE(v.unit_words == unit_words, "sf_gemv_fp16_fetch: the cache's units must be N fp16 residuals");
    rows = v.rows;
    row_of = v.row_of;
  }
  const sf_status st = W->b_r == 2 ? launch_br<2, 1>(W, x, B, idx, n, rows, row_of, unit_words, y, s)
                                   : launch_br<3, 1>(W, x, B, idx, n, rows, row_of, unit_words, y, s);
  if (st != SF_OK) return st;
  if (c) return sf::cache_mark_used(c, s);
  return SF_OK;
}
