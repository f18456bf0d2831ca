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

#include "act.cuh"
#include "sf_internal.h"

namespace {

constexpr int kNS = 4;  // pipeline stages

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
  sfd::act_planes_from_floats(xf, plf, &xsum, &fscale);
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

// ---- batch 1 on prepared activations: several matrices sharing x ------------
//
// The activations arrive prepared (fixed-point planes, slab sums, selection
// masks; see act.cuh), so a thread's whole setup is one 128-byte load.  A CTA
// computes one tile of 8 output rows over K/ksplit input channels: every
// thread owns one 32-channel slab and keeps its 8 code words in registers.
// Matrices that read the same x (q/k/v, gate/up) share one launch; each has
// its own weights, refinement rows and output.
namespace {

constexpr int kActR = 8;
constexpr int kMaxJobs = 4;

struct ActJob {
  const uint32_t* res;
  const uint16_t* scale;
  const uint16_t* zero;
  const uint32_t* ref_rows;  // nullptr: resident only
  const int32_t* row_of;     // nullptr: refinement row = channel index
  int unit_words;
  int N;
  float* y;
  int tile_begin;
};

struct ActArgs {
  ActJob job[kMaxJobs];
  int njobs;
  int K, G, b_f, ksplit;
  const uint16_t* x;
  const uint32_t* act;
};

// Persistent CTAs: a CTA keeps one slab range (k-split half) for its whole
// life and walks the row tiles of all jobs, tile c, c + ncta, ...  Per thread
// the slab's prepared activations and up to kSelReg selected channels'
// refinement rows are loaded once; per tile, codes (8 rows x 8 bytes),
// scale/zero (group owners) and the selected columns' refinement words are
// staged with cp.async into a kStages-deep shared-memory ring owned slot by
// slot by the threads that read them.
constexpr int kStages = 4;
constexpr int kSelReg = 4;  // selected channels per slab held in registers

struct PipeCtx {
  int tile_job[kMaxJobs];
};

__device__ __forceinline__ int job_of_tile(const ActArgs& a, int t) {
  int jb = 0;
#pragma unroll
  for (int q = 1; q < kMaxJobs; ++q)
    if (q < a.njobs && t >= a.job[q].tile_begin) jb = q;
  return jb;
}

// fp16 bit pattern -> fp32 with integer/FP32 pipes only (no conversion
// unit): move exponent and mantissa into place and rescale by 2^112, exact for
// every finite fp16 including subnormals.
__device__ __forceinline__ float h2f_bits(uint32_t h) {
  return __uint_as_float((h & 0x7FFFu) << 13) * 5.192296858534828e+33f * ((h & 0x8000u) ? -1.0f : 1.0f);
}

// int -> fp32 for |v| < 2^22 with one integer add and one FP add (no
// conversion unit): 1.5 * 2^23 + v has v in its low mantissa bits.
__device__ __forceinline__ float i2f_small(int v) {
  return __int_as_float(0x4B400000 + v) - 12582912.0f;
}

// Reduce-scatter of 8 rows x (3 integer planes + 1 fp32 correction) over the
// 4 lanes of a 128-channel group: afterwards lane tig owns rows 2 tig and
// 2 tig + 1, summed over the group.
__device__ __forceinline__ void group_reduce_scatter(int (&d0)[8], int (&d1)[8], int (&d2)[8], float (&dc)[8],
                                                     int tig) {
  {
    const bool up = (tig & 2) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int s0 = up ? d0[i] : d0[i + 4], s1 = up ? d1[i] : d1[i + 4], s2 = up ? d2[i] : d2[i + 4];
      float sc = up ? dc[i] : dc[i + 4];
      int k0 = up ? d0[i + 4] : d0[i], k1 = up ? d1[i + 4] : d1[i], k2 = up ? d2[i + 4] : d2[i];
      float kc = up ? dc[i + 4] : dc[i];
      d0[i] = k0 + __shfl_xor_sync(0xffffffffu, s0, 2);
      d1[i] = k1 + __shfl_xor_sync(0xffffffffu, s1, 2);
      d2[i] = k2 + __shfl_xor_sync(0xffffffffu, s2, 2);
      dc[i] = kc + __shfl_xor_sync(0xffffffffu, sc, 2);
    }
  }
  {
    const bool up = (tig & 1) != 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      int s0 = up ? d0[i] : d0[i + 2], s1 = up ? d1[i] : d1[i + 2], s2 = up ? d2[i] : d2[i + 2];
      float sc = up ? dc[i] : dc[i + 2];
      int k0 = up ? d0[i + 2] : d0[i], k1 = up ? d1[i + 2] : d1[i], k2 = up ? d2[i + 2] : d2[i];
      float kc = up ? dc[i + 2] : dc[i];
      d0[i] = k0 + __shfl_xor_sync(0xffffffffu, s0, 1);
      d1[i] = k1 + __shfl_xor_sync(0xffffffffu, s1, 1);
      d2[i] = k2 + __shfl_xor_sync(0xffffffffu, s2, 1);
      dc[i] = kc + __shfl_xor_sync(0xffffffffu, sc, 1);
    }
  }
}

// Persistent CTAs: a CTA keeps one slab range (k-split half) for its whole
// life and walks the row tiles of all jobs, tile c, c + ncta, ...  Per thread
// the slab's prepared activations and up to kSelReg selected channels'
// refinement rows are loaded once; per tile, codes (8 rows x 8 bytes),
// scale/zero (group owners) and the selected columns' refinement words are
// staged with cp.async into a kStages-deep shared-memory ring owned slot by
// slot by the threads that read them.  The four threads of a 128-channel group
// share one fixed-point scale: their integer plane sums are reduce-scattered
// so each converts and scales only two rows.
__global__ void __launch_bounds__(256)
gemv_b1_act_kernel(const __grid_constant__ ActArgs a) {
  constexpr int R = kActR;
  extern __shared__ __align__(16) unsigned char sm[];
  const int nthr = blockDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = nthr >> 5;
  const int tig = lane & 3;
  const int ks = blockIdx.x % a.ksplit;
  const int crow = blockIdx.x / a.ksplit, ncta = gridDim.x / a.ksplit;
  const int s = ks * nthr + tid;  // slab
  const int g = s >> 2;           // 128-channel group (G == 128)
  const int g0 = (ks * nthr) >> 2;
  const int ngc = nthr >> 2;
  const bool sz_owner = tig == 0;
  const size_t row_words = static_cast<size_t>(a.K) / 16;
  const int total_tiles = a.job[a.njobs - 1].tile_begin + a.job[a.njobs - 1].N / R;
  const int my_tiles = crow < total_tiles ? (total_tiles - crow + ncta - 1) / ncta : 0;

  uint2* codes = reinterpret_cast<uint2*>(sm);                                    // [kStages][R][nthr]
  uint16_t* szs = reinterpret_cast<uint16_t*>(codes + kStages * R * nthr);        // [kStages][ngc][2][R]
  uint32_t* refw = reinterpret_cast<uint32_t*>(szs + kStages * ngc * 2 * R);      // [kStages][kSelReg][nthr]
  float* red = reinterpret_cast<float*>(refw + kStages * kSelReg * nthr);         // [2][nw][R]

  // prepared activations of the slab
  const uint4* ap = reinterpret_cast<const uint4*>(a.act + static_cast<size_t>(s) * sfd::kActWords);
  uint32_t pl[24];
#pragma unroll
  for (int q = 0; q < 6; ++q) {
    const uint4 v = ap[q];
    pl[4 * q] = v.x; pl[4 * q + 1] = v.y; pl[4 * q + 2] = v.z; pl[4 * q + 3] = v.w;
  }
  const uint4 meta = ap[6];
  const float fscale = __uint_as_float(meta.y);
  const uint32_t mask = meta.z;
  const int prefix = static_cast<int>(meta.w);
  const float gsum = __uint_as_float(ap[7].x);  // sum of x over the 128-channel group
  const int nsel = __popc(mask);
  int selj[kSelReg];
  float selx[kSelReg];
  {
    uint32_t mm = mask;
#pragma unroll
    for (int i = 0; i < kSelReg; ++i) {
      selj[i] = 0;
      selx[i] = 0.0f;
      if (mm) {
        const int j = __ffs(mm) - 1;
        mm &= mm - 1u;
        selj[i] = j;
        selx[i] = sfd::bf16_bits_to_float(a.x[32 * s + j]);
      }
    }
  }
  const float m_f = static_cast<float>((1 << a.b_f) - 1) * 0.5f;
  const float two_bf = static_cast<float>(1 << a.b_f);
  const uint32_t fmask = (1u << a.b_f) - 1u;

  int issue_job = -1;
  int rid[kSelReg];
#pragma unroll
  for (int i = 0; i < kSelReg; ++i) rid[i] = 0;

  auto issue = [&](int i) {
    const int st = i % kStages;
    const int t = crow + i * ncta;
    const int jb = job_of_tile(a, t);
    const ActJob& J = a.job[jb];
    const int row0 = (t - J.tile_begin) * R;
    if (jb != issue_job) {
      issue_job = jb;
#pragma unroll
      for (int q = 0; q < kSelReg; ++q)
        if (q < nsel && J.ref_rows) rid[q] = J.row_of ? J.row_of[prefix + q] : 32 * s + selj[q];
    }
    const uint32_t* src = J.res + static_cast<size_t>(row0) * row_words + 2 * s;
    uint2* dst = codes + (st * R) * nthr + tid;
#pragma unroll
    for (int r = 0; r < R; ++r) cp_async8(dst + r * nthr, src + r * row_words);
    if (sz_owner) {
      uint16_t* d = szs + ((st * ngc) + (g - g0)) * 2 * R;
      cp_async16(d, J.scale + static_cast<size_t>(g) * J.N + row0);
      cp_async16(d + R, J.zero + static_cast<size_t>(g) * J.N + row0);
    }
    if (J.ref_rows) {
      const int w0 = (row0 * a.b_f) >> 5;
#pragma unroll
      for (int q = 0; q < kSelReg; ++q)
        if (q < nsel) cp_async4(refw + (st * kSelReg + q) * nthr + tid,
                                J.ref_rows + static_cast<size_t>(rid[q]) * J.unit_words + w0);
    }
  };

#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (i < my_tiles) issue(i);
    cp_async_commit();
  }
  for (int i = 0; i < my_tiles; ++i) {
    if (i + kStages - 1 < my_tiles) issue(i + kStages - 1);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const int st = i % kStages;
    const int t = crow + i * ncta;
    const int jb = job_of_tile(a, t);
    const ActJob& J = a.job[jb];
    const int row0 = (t - J.tile_begin) * R;
    const uint2* cw = codes + (st * R) * nthr + tid;
    const int bitoff = (row0 * a.b_f) & 31;
    // per row: integer plane sums of this slab, and the refinement correction
    int d0[R], d1[R], d2[R];
    float dc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint2 w = cw[r * nthr];
      uint32_t u0 = 0, u1 = 0;
      int u2 = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t c0 = (w.x >> (2 * k)) & 0x03030303u;
        const uint32_t c1 = (w.y >> (2 * k)) & 0x03030303u;
        u0 = __dp4a(c0, pl[k * 3 + 0], u0);
        u1 = __dp4a(c0, pl[k * 3 + 1], u1);
        u2 = __dp4a(static_cast<int>(c0), static_cast<int>(pl[k * 3 + 2]), u2);
        u0 = __dp4a(c1, pl[(4 + k) * 3 + 0], u0);
        u1 = __dp4a(c1, pl[(4 + k) * 3 + 1], u1);
        u2 = __dp4a(static_cast<int>(c1), static_cast<int>(pl[(4 + k) * 3 + 2]), u2);
      }
      d0[r] = static_cast<int>(u0);
      d1[r] = static_cast<int>(u1);
      d2[r] = u2;
      dc[r] = 0.0f;
    }
    if (J.ref_rows) {
#pragma unroll
      for (int q = 0; q < kSelReg; ++q)
        if (q < nsel) {
          const uint32_t word = refw[(st * kSelReg + q) * nthr + tid];
#pragma unroll
          for (int r = 0; r < R; ++r)
            dc[r] = fmaf(selx[q], static_cast<float>((word >> (bitoff + r * a.b_f)) & fmask) - m_f, dc[r]);
        }
      if (nsel > kSelReg) {  // rare: more selected channels than held in registers
        uint32_t mm = mask;
        for (int q = 0; q < kSelReg; ++q) mm &= mm - 1u;
        int p = prefix + kSelReg;
        while (mm) {
          const int j = __ffs(mm) - 1;
          mm &= mm - 1u;
          const int rr = J.row_of ? J.row_of[p] : 32 * s + j;
          const uint32_t word = J.ref_rows[static_cast<size_t>(rr) * J.unit_words + ((row0 * a.b_f) >> 5)];
          const float xj = sfd::bf16_bits_to_float(a.x[32 * s + j]);
#pragma unroll
          for (int r = 0; r < R; ++r)
            dc[r] = fmaf(xj, static_cast<float>((word >> (bitoff + r * a.b_f)) & fmask) - m_f, dc[r]);
          ++p;
        }
      }
    }
    group_reduce_scatter(d0, d1, d2, dc, tig);
    // this lane's two rows of the group: 2 tig, 2 tig + 1
    const uint16_t* sz = szs + ((st * ngc) + (g - g0)) * 2 * R;
    const uint32_t sw = reinterpret_cast<const uint32_t*>(sz)[tig];      // scales of rows 2tig, 2tig+1
    const uint32_t zw = reinterpret_cast<const uint32_t*>(sz + R)[tig];  // zeros
    float v[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      // |d2| <= 128*3*128, |d1|, |d0| <= 128*3*255 after the group sum: exact
      // small-integer conversions
      const float P = fmaf(i2f_small(d2[q]), 65536.0f, fmaf(i2f_small(d1[q]), 256.0f, i2f_small(d0[q])));
      const float sc = h2f_bits(q ? (sw >> 16) : (sw & 0xFFFFu));
      const float zz = h2f_bits(q ? (zw >> 16) : (zw & 0xFFFFu));
      v[q] = sc * (fmaf(two_bf, P * fscale, (m_f - zz) * gsum) + dc[q]);
    }
    // sum over the warp's 8 groups (lanes with equal tig), then across warps
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
      v[1] += __shfl_xor_sync(0xffffffffu, v[1], off);
    }
    float* rb = red + (i & 1) * nw * R;
    if (lane < 4) {
      rb[warp * R + 2 * lane] = v[0];
      rb[warp * R + 2 * lane + 1] = v[1];
    }
    __syncthreads();
    if (tid < R) {
      float acc = 0.0f;
      for (int q = 0; q < nw; ++q) acc += rb[q * R + tid];
      float* dst = J.y + row0 + tid;
      if (a.ksplit > 1) atomicAdd(dst, acc);  // two contributions onto zero: order-independent
      else *dst = acc;
    }
  }
  cp_async_wait<0>();
}

}  // namespace

extern "C" sf_status sf_gemv_refine_batch1(const sf_gemv_job* jobs, int count, const uint16_t* x, const void* act,
                                           sf_stream_t stream) {
  SF_REQUIRE(jobs && x && act, "sf_gemv_refine_batch1: null pointer");
  SF_REQUIRE(count >= 1 && count <= kMaxJobs, "sf_gemv_refine_batch1: count must be in [1, %d]", kMaxJobs);
  SF_REQUIRE(sf::aligned(act, 16) && sf::aligned(x, 4), "sf_gemv_refine_batch1: act must be 16-byte aligned");
  const sf_qweight* W0 = jobs[0].W;
  SF_REQUIRE(W0, "sf_gemv_refine_batch1: null weight");
  const int K = W0->K, G = W0->G, b_f = W0->b_f;
  SF_REQUIRE(W0->b_r == 2, "sf_gemv_refine_batch1: 2-bit resident codes only");
  SF_REQUIRE(b_f == 1 || b_f == 2, "sf_gemv_refine_batch1: b_f must be 1 or 2");
  SF_REQUIRE(G == 128 && K % G == 0, "sf_gemv_refine_batch1: group size must be 128 (the prepared activations' block)");
  const int S = K / 32;
  int ksplit = 0;
  if (K % 1024 == 0 && S <= 256) ksplit = 1;
  else if (K % 2048 == 0 && S <= 512) ksplit = 2;
  SF_REQUIRE(ksplit, "sf_gemv_refine_batch1: K must be a multiple of 1024 up to 8192, or of 2048 up to 16384");
  SF_REQUIRE((S / ksplit * 32) % G == 0, "sf_gemv_refine_batch1: each K half must hold whole groups");
  cudaStream_t s = sf::as_cuda(stream);
  ActArgs a{};
  a.njobs = count;
  a.K = K;
  a.G = G;
  a.b_f = b_f;
  a.ksplit = ksplit;
  a.x = x;
  a.act = static_cast<const uint32_t*>(act);
  int tiles = 0;
  for (int i = 0; i < count; ++i) {
    const sf_qweight* W = jobs[i].W;
    SF_REQUIRE(W && W->res && W->scale && W->zero && jobs[i].y, "sf_gemv_refine_batch1: job %d incomplete", i);
    SF_REQUIRE(W->K == K && W->G == G && W->b_f == b_f && W->b_r == 2,
               "sf_gemv_refine_batch1: jobs must share K, G and bit widths");
    SF_REQUIRE(W->N >= kActR && W->N % kActR == 0, "sf_gemv_refine_batch1: N must be a multiple of %d", kActR);
    SF_REQUIRE(sf::aligned(W->res, 16) && sf::aligned(W->scale, 16) && sf::aligned(W->zero, 16),
               "sf_gemv_refine_batch1: weight arrays must be 16-byte aligned");
    ActJob& J = a.job[i];
    J.res = W->res;
    J.scale = W->scale;
    J.zero = W->zero;
    J.N = W->N;
    J.y = jobs[i].y;
    J.unit_words = W->N * b_f / 32;
    J.tile_begin = tiles / ksplit;
    tiles += (W->N / kActR) * ksplit;
    if (jobs[i].cache) {
      sf::CacheView v{};
      const sf_status st = sf::cache_view_for_gemv(jobs[i].cache, s, &v);
      if (st != SF_OK) return st;
      SF_REQUIRE(v.unit_words == J.unit_words, "sf_gemv_refine_batch1: cache unit size does not match N*b_f/8");
      J.ref_rows = v.rows;
      J.row_of = v.row_of;
    } else if (jobs[i].use_ref_store) {
      SF_REQUIRE(W->ref, "sf_gemv_refine_batch1: use_ref_store without W->ref");
      J.ref_rows = W->ref;
      J.row_of = nullptr;
    }
    if (ksplit > 1) SF_CHECK_CUDA(cudaMemsetAsync(jobs[i].y, 0, sizeof(float) * W->N, s));
  }
  const int nthr = S / ksplit;
  const int ngc = nthr / 4;
  const size_t smem = static_cast<size_t>(kStages) * kActR * nthr * 8 + static_cast<size_t>(kStages) * ngc * 2 * kActR * 2 +
                      static_cast<size_t>(kStages) * kSelReg * nthr * 4 + 2 * (nthr / 32) * kActR * 4;
  SF_CHECK_CUDA(cudaFuncSetAttribute(gemv_b1_act_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)));
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gemv_b1_act_kernel, nthr, smem) != cudaSuccess || occ < 1)
    occ = 1;
  const int row_tiles = tiles / ksplit;
  const int ncta = std::max(1, std::min(row_tiles, occ * sf::sm_count() / ksplit));
  gemv_b1_act_kernel<<<ncta * ksplit, nthr, smem, s>>>(a);
  const sf_status st = sf::check_launch("gemv_b1_act_kernel");
  if (st != SF_OK) return st;
  for (int i = 0; i < count; ++i)
    if (jobs[i].cache) {
      const sf_status m = sf::cache_mark_used(jobs[i].cache, s);
      if (m != SF_OK) return m;
    }
  return SF_OK;
}
