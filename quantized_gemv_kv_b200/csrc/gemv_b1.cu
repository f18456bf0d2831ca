// Batch-1 refined GEMV for 2-bit resident codes on the integer dot-product
// path.  Same contract as gemv_refine_kernel (y = W_res x + sum_{j in S}
// x_j s (q_f - m_f), nested refinement of the columns with the largest
// activations, rag-lover.com explainer of StrataFlux, 解説); only the
// arithmetic is arranged for the B200's ALU budget.
//
// At batch 1 a 2-bit weight byte holds 4 weights, so streaming at HBM speed
// leaves about one instruction per weight.  Converting codes to floats costs
// more than that; instead each thread owns one 32-column slab of the input:
//
//  * its 32 activations become exact 24-bit fixed point relative to the slab's
//    largest exponent (X_j = rint(x_j 2^(23-e)), |X_j| < 2^23; bf16 inputs
//    within 15 binades of the slab maximum are exact, smaller ones round with
//    error < 2^(e-24)), split into three byte planes and packed to match the
//    byte order of unpacked codes;
//  * a 2-bit code word becomes four code bytes with one shift and one mask,
//    and DP4A multiplies them with the planes: sum_j c_j X_j exactly in int32;
//  * per slab and row: y += s * (2^b_f * P + (m_f - z) * sum_j x_j
//                               + sum_{selected j} x_j (q_f - m_f)),
//    with the refinement correction folded into the same slab sum.
//
// Weight bytes move by per-thread cp.async into a multi-stage shared-memory
// ring (each thread copies exactly the bytes it later reads, so no block-wide
// handshake guards the ring and no thread spins on a flag).  Row partials are
// reduced across lanes with a transposed shuffle reduction and across warps
// through shared memory.
#include <algorithm>

#include "sf_internal.h"

namespace {

constexpr int kNS = 4;  // pipeline stages

// Fixed-point byte planes of one 32-column slab: X_j = rint(x_j 2^(23 - e)),
// e the binary exponent of the slab's largest |x|; word (wi*4 + k)*3 + p holds
// in byte b the byte p of X[16 wi + k + 4 b] (the order in which a code word
// yields code bytes as (w >> 2k) & 0x03030303).  Also the slab sum of the
// fixed-point values and the scale 2^(e - 23).
__device__ inline void slab_planes_from_floats(const float (&xf)[32], uint32_t (&pl)[24], float* xsum,
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

__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

struct B1Args {
  const uint32_t* res;
  const uint16_t* scale;
  const uint16_t* zero;
  int N, K, G, b_f;
  const uint16_t* x;
  const int32_t* idx;
  const int32_t* n_sel;
  const uint32_t* ref_rows;  // nullptr: resident only
  const int32_t* row_of;     // nullptr: row = column index
  int unit_words;
  float* y;
  int ntiles;
  int nmax;  // capacity of the selection list in shared memory
};

template <int R>
struct Smem {
  // byte offsets inside the dynamic shared memory block
  static constexpr int RW = 2;  // refinement words staged per selected column and tile (>= R*b_f/32)
};

template <int R>
__global__ void __launch_bounds__(512)
gemv_b1_dp4a_kernel(B1Args a) {
  extern __shared__ __align__(16) unsigned char sm[];
  const int S = blockDim.x;  // slabs per row (K / 32), a multiple of 32
  const int s = threadIdx.x, lane = s & 31, warp = s >> 5, nw = S >> 5;
  const int spg = a.G >> 5, ng = a.K / a.G, g = s / spg;
  const bool sz_owner = (s % spg) == 0;
  constexpr int RW = Smem<R>::RW;

  uint2* codes = reinterpret_cast<uint2*>(sm);                                   // [kNS][R][S]
  uint16_t* szs = reinterpret_cast<uint16_t*>(codes + kNS * R * S);              // [kNS][ng][2][R]
  int* sel_rid = reinterpret_cast<int*>(szs + kNS * ng * 2 * R);                // [nmax]
  int* sel_col = sel_rid + a.nmax;                                               // [nmax]
  float* sel_x = reinterpret_cast<float*>(sel_col + a.nmax);                     // [nmax]
  uint32_t* refw = reinterpret_cast<uint32_t*>(sel_x + a.nmax);                  // [kNS][nmax][RW]
  float* red = reinterpret_cast<float*>(refw + kNS * a.nmax * RW);               // [2][nw][R]

  // ---- activations of this slab -> fixed point byte planes
  float xf[32];
  {
    const uint4* xp4 = reinterpret_cast<const uint4*>(a.x + 32 * s);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = xp4[q];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        xf[8 * q + 2 * h] = __uint_as_float(w[h] << 16);
        xf[8 * q + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
      }
    }
  }
  uint32_t plf[24];
  float xsum, fscale;
  slab_planes_from_floats(xf, plf, &xsum, &fscale);
  uint32_t pl[2][4][3];
#pragma unroll
  for (int wi = 0; wi < 2; ++wi)
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int p = 0; p < 3; ++p) pl[wi][k][p] = plf[(wi * 4 + k) * 3 + p];

  // ---- selection list (columns ascending) and this thread's part of it
  int n = 0;
  if (a.ref_rows) {
    n = *a.n_sel;
    n = n < 0 ? 0 : (n > a.nmax ? a.nmax : n);
    for (int p = s; p < n; p += S) {
      const int j = a.idx[p];
      sel_col[p] = j;
      sel_rid[p] = a.row_of ? a.row_of[p] : j;
      sel_x[p] = sfd::bf16_bits_to_float(a.x[j]);
    }
  }
  __syncthreads();
  int pb = 0, pe = 0;
  if (n) {
    int lo = 0, hi = n;
    while (lo < hi) { const int m = (lo + hi) >> 1; if (sel_col[m] < 32 * s) lo = m + 1; else hi = m; }
    pb = lo;
    hi = n;
    while (lo < hi) { const int m = (lo + hi) >> 1; if (sel_col[m] < 32 * s + 32) lo = m + 1; else hi = m; }
    pe = lo;
  }

  const size_t row_words = static_cast<size_t>(a.K) / 16;  // 2-bit codes
  const float m_f = static_cast<float>((1 << a.b_f) - 1) * 0.5f;
  const float two_bf = static_cast<float>(1 << a.b_f);
  const uint32_t fmask = (1u << a.b_f) - 1u;
  const int my_tiles = a.ntiles > static_cast<int>(blockIdx.x)
                           ? (a.ntiles - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x
                           : 0;

  auto issue = [&](int i) {
    const int st = i % kNS;
    const int row0 = (blockIdx.x + i * gridDim.x) * R;
    const uint32_t* src = a.res + static_cast<size_t>(row0) * row_words + 2 * s;
    uint2* dst = codes + (st * R) * S + s;
#pragma unroll
    for (int r = 0; r < R; ++r) cp_async8(dst + r * S, src + r * row_words);
    if (sz_owner) {
      uint16_t* d = szs + (st * ng + g) * 2 * R;
      const uint16_t* s0 = a.scale + static_cast<size_t>(g) * a.N + row0;
      const uint16_t* z0 = a.zero + static_cast<size_t>(g) * a.N + row0;
#pragma unroll
      for (int c = 0; c < R / 8; ++c) {
        cp_async16(d + 8 * c, s0 + 8 * c);
        cp_async16(d + R + 8 * c, z0 + 8 * c);
      }
    }
    const int w0 = (row0 * a.b_f) >> 5;
    const int nwords = (R * a.b_f + 31) >> 5;
    for (int p = pb; p < pe; ++p) {
      const uint32_t* col = a.ref_rows + static_cast<size_t>(sel_rid[p]) * a.unit_words + w0;
      uint32_t* d = refw + (st * a.nmax + p) * RW;
      cp_async4(d, col);
      if (nwords > 1) cp_async4(d + 1, col + 1);
    }
  };

#pragma unroll
  for (int i = 0; i < kNS - 1; ++i) {
    if (i < my_tiles) issue(i);
    cp_async_commit();
  }
  for (int i = 0; i < my_tiles; ++i) {
    if (i + kNS - 1 < my_tiles) issue(i + kNS - 1);
    cp_async_commit();
    cp_async_wait<kNS - 1>();
    __syncwarp();
    const int st = i % kNS;
    const int row0 = (blockIdx.x + i * gridDim.x) * R;
    const uint2* cw = codes + (st * R) * S + s;
    const uint16_t* sz = szs + (st * ng + g) * 2 * R;
    const int bitoff = (row0 * a.b_f) & 31;
    float v[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint2 w = cw[r * S];
      uint32_t d0 = 0, d1 = 0;
      int d2 = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t c0 = (w.x >> (2 * k)) & 0x03030303u;
        const uint32_t c1 = (w.y >> (2 * k)) & 0x03030303u;
        d0 = __dp4a(c0, pl[0][k][0], d0);
        d1 = __dp4a(c0, pl[0][k][1], d1);
        d2 = __dp4a(static_cast<int>(c0), static_cast<int>(pl[0][k][2]), d2);
        d0 = __dp4a(c1, pl[1][k][0], d0);
        d1 = __dp4a(c1, pl[1][k][1], d1);
        d2 = __dp4a(static_cast<int>(c1), static_cast<int>(pl[1][k][2]), d2);
      }
      const int pint = d2 * 65536 + static_cast<int>(d1) * 256 + static_cast<int>(d0);
      const float sc = sfd::half_bits_to_float(sz[r]);
      const float zz = sfd::half_bits_to_float(sz[R + r]);
      float t = fmaf(two_bf, static_cast<float>(pint) * fscale, (m_f - zz) * xsum);
      for (int p = pb; p < pe; ++p) {
        const uint32_t* rw = refw + (st * a.nmax + p) * RW;
        const int bit = bitoff + r * a.b_f;
        const uint32_t q = (rw[bit >> 5] >> (bit & 31)) & fmask;
        t = fmaf(sel_x[p], static_cast<float>(q) - m_f, t);
      }
      v[r] = sc * t;
    }
    // reduce v[0..R) over the 32 lanes: lane l ends with row (l mod R)
#pragma unroll
    for (int off = 16; off >= R; off >>= 1)
#pragma unroll
      for (int r = 0; r < R; ++r) v[r] += __shfl_xor_sync(0xffffffffu, v[r], off);
#pragma unroll
    for (int off = R / 2; off >= 1; off >>= 1) {
      const bool up = (lane & off) != 0;
#pragma unroll
      for (int r = 0; r < off; ++r) {
        const float send = up ? v[r] : v[r + off];
        const float keep = up ? v[r + off] : v[r];
        v[r] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
    }
    float* rb = red + (i & 1) * nw * R;
    if (lane < R) rb[warp * R + lane] = v[0];
    __syncthreads();
    if (s < R) {
      float acc = 0.0f;
      for (int w = 0; w < nw; ++w) acc += rb[w * R + s];
      a.y[row0 + s] = acc;
    }
  }
  cp_async_wait<0>();
}

}  // namespace

namespace sf {

// Returns true (and launches) when the batch-1 integer path applies.
bool gemv_b1_try(const sf_qweight* W, const uint16_t* x, const int32_t* idx, const int32_t* n,
                 const uint32_t* ref_rows, const int32_t* row_of, int unit_words, int nmax, float* y,
                 cudaStream_t s, sf_status* st) {
  if (W->b_r != 2 || W->K % 1024 != 0 || W->K > 16384 || W->G > 1024 || W->N % 8 != 0) return false;
  if (!aligned(x, 16) || !aligned(W->res, 16) || !aligned(W->scale, 16) || !aligned(W->zero, 16)) return false;
  if (ref_rows && nmax > 2048) return false;
  if (!ref_rows) nmax = 0;
  const int S = W->K / 32;
  const int ng = W->K / W->G;
  const int sms = sm_count();
  const size_t row_bytes = static_cast<size_t>(W->K) / 4;
  int R = 8;
  if (W->N % 16 == 0 && W->N / 16 >= sms && 16 * row_bytes <= 16384) R = 16;
  const int nw = S / 32;
  auto smem_for = [&](int r) {
    return static_cast<size_t>(kNS) * r * S * 8 + static_cast<size_t>(kNS) * ng * 2 * r * 2 +
           static_cast<size_t>(nmax) * 12 + static_cast<size_t>(kNS) * nmax * 2 * 4 + 2 * nw * r * 4;
  };
  const size_t smem = smem_for(R);
  if (smem > 200 * 1024) return false;
  B1Args a{W->res, W->scale, W->zero, W->N, W->K, W->G, W->b_f, x, idx, n, ref_rows, row_of, unit_words, y,
           W->N / R, nmax};
  auto launch = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) { *st = cuda_fail(e, "gemv_b1 smem attribute"); return; }
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, S, smem);
    if (e != cudaSuccess || occ < 1) occ = 1;
    const int grid = std::min(a.ntiles, occ * sms);
    kern<<<grid, S, smem, s>>>(a);
    *st = check_launch("gemv_b1_dp4a_kernel");
  };
  if (R == 16) launch(gemv_b1_dp4a_kernel<16>);
  else launch(gemv_b1_dp4a_kernel<8>);
  return true;
}

}  // namespace sf
