// sf_gemv_refine_batch1: batch-1 refined GEMV on the integer tensor cores.
//
//   y_i = sum_j x_j w_res[i][j] + sum_{j in S} x_j s_{g(j),i} (q_f[i][j] - m_f)
//
// (nested refinement applied to the columns with the largest activations,
// rag-lover.com explainer of StrataFlux, 解説), for up to four matrices that
// read the same activation row (q/k/v, gate/up), with x prepared once
// (act.cuh: per-group fixed point in signed 8-bit digits, laid out as MMA B
// fragments, plus the selection mask).
//
// Tiles are 16 output rows; a CTA walks a contiguous block of them.  A warp
// owns SPW 256-channel slices of K for the whole kernel; their B fragments
// stay in registers.  Per tile and slice:
//  * resident part: 8 mma.m16n8k32 (u8 codes x s8 digits, s32 accumulate,
//    two independent chains); a code word becomes four A-fragment bytes with
//    one shift and one mask.  The slice's two groups land in disjoint
//    accumulator columns (three digit planes each), so after one lane swap
//    each lane owns one (row, group) pair and applies its scale and zero point;
//  * refinement correction: the 2-bit q_f of the 16 rows for the slice's
//    selected channels (one staged word per channel) become f16 A fragments
//    (1024 + q_f, exact) against the channels' x split into f16 high and low
//    parts, on mma.m16n8k16; the 1024 offset and m_f are removed with
//    per-group sums of x.
// The warps of a CTA cover consecutive slices of one tile and add up in
// shared memory; with two K halves (ksplit = 2) the halves add their partial
// sums onto a zeroed output (two terms onto zero: the result does not depend
// on their order).
//
// Each warp streams its own codes (16 rows x 64 or 96 bytes per slice; the
// 2-bit rows' 16-byte chunks XOR-swizzled, the 3-bit rows' 24-word stride
// already conflict-free, so the fragment loads never collide on a bank),
// scale/zero and refinement words through a cp.async ring in shared memory
// and waits only for its own copies.
//
// 3-bit resident codes are read from a split layout written once by
// sf_gemv_pack_batch1 (a 3-bit code straddles bytes in the canonical
// bitstream, so it cannot become an A-fragment byte with one shift and one
// mask).  Per row and 256-channel slice, 24 words:
//   words 0-15  the low 2 bits of the codes, arranged as 2-bit codes are
//               (word w, byte b, bits 2j..2j+1: channel 16 w + 4 b + j);
//   words 16-23 the high bits: word 16 + 2 t + slot covers the low words
//               8 slot + 2 t + h (h = 0, 1), bit 4 h + j of its byte b holding
//               the high bit of channel 16 (8 slot + 2 t + h) + 4 b + j.
// A fragment byte is then ((w >> 2j) & 0x03030303) | (high bit moved to bit
// 2 of each byte): two shifts and two logic operations per register.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <type_traits>
#include <utility>

#include "act.cuh"  // bf16_exponent, bf16_fixed
#include "produce.cuh"
#include "select_row.cuh"
#include "sf_internal.h"

namespace {

constexpr int kMaxJobs = 4;
constexpr int kRows = 16;          // output rows per tile
constexpr int kMaxWarps = 16;      // warps per CTA
constexpr int kCorrList = 32;      // selected channels per slice handled on the tensor cores
// selected x at or above this magnitude would overflow the f16 (high, low)
// split of the correction MMA: such a slice takes the fp32 correction loop
constexpr float kCorrXMax = 32768.0f;

struct MJob {
  const uint32_t* res;       // resident codes in the batch-1 layout
  const uint16_t* scale;
  const uint16_t* zero;
  const uint32_t* ref_rows;  // nullptr: resident only
  const int32_t* row_of;     // nullptr: refinement row = channel index
  const int32_t* unit_slot;  // deadline reading: refinement row of channel j = unit_slot[j] (-1: not refined)
  float* y;
  int N, unit_words, tile_begin;
};

// The input row made inside the launch (sf_gemv_refine_batch1_produce): every
// CTA computes the row and its selection itself, in the ring stage that the
// weight stream does not use before the main loop.
enum ProdOp { kProdNone = -1, kProdNorm = 0, kProdRound = 1, kProdSilu = 2 };

struct MProd {
  int op, k, hrows;  // hrows: histogram rows of the selection (warps share them)
  float eps;
  const float* x;      // kProdNorm: the residual; kProdRound: the row; kProdSilu: the gate
  const float* delta;  // kProdNorm: added to x first (may be null)
  const float* w;      // kProdNorm: RMSNorm weights
  const float* u;      // kProdSilu: the up projection
  float* x_out;        // kProdNorm: x + delta, written by CTA 0 (may be null)
  uint16_t* y;         // the bf16 row: written by every CTA (identical values)
  int32_t* idx;        // its selection and length: likewise
  int32_t* n;
};

struct MArgs {
  MJob job[kMaxJobs];
  MProd prod;
  const uint16_t* x;     // the row (with a producer: prod.y, read back by the fp32 correction)
  const int32_t* idx;    // the selection: ascending channels (nullptr: none)
  const int32_t* n_sel;  // its length (negative counts as 0)
  int njobs, K, ksplit;
};

__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
// Programmatic dependent launch: returns once the preceding kernel (the
// producer of x and the selection) has completed and its writes are visible.
__device__ __forceinline__ void pdl_wait_gemv() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// fp16 bit pattern -> fp32 with integer/FP32 pipes only: move exponent and
// mantissa into place and rescale by 2^112, exact for every finite fp16
// including subnormals.
__device__ __forceinline__ float h2f_bits(uint32_t h) {
  return __uint_as_float((h & 0x7FFFu) << 13) * 5.192296858534828e+33f * ((h & 0x8000u) ? -1.0f : 1.0f);
}
// int -> fp32 for |v| < 2^22 with one integer add and one FP add.
__device__ __forceinline__ float i2f_small(int v) { return __int_as_float(0x4B400000 + v) - 12582912.0f; }

__device__ __forceinline__ int job_of(const MArgs& a, int t) {
  int jb = 0;
#pragma unroll
  for (int q = 1; q < kMaxJobs; ++q)
    if (q < a.njobs && t >= a.job[q].tile_begin) jb = q;
  return jb;
}

// Word offset of 16-byte chunk c of staged code row r.  2-bit rows (64 bytes,
// chunks 0..3): rows 2, 3 (mod 4) swap chunk pairs, so the rows read by one
// half-warp's 8-byte fragment loads fall on distinct banks.  3-bit rows (96
// bytes, chunks 0..5): a 24-word row stride already spreads them.
template <int BR>
__device__ __forceinline__ int code_off(int r, int c) {
  if constexpr (BR == 2) return r * 16 + ((c ^ (((r >> 1) & 1) << 1)) << 2);
  else return r * 24 + 4 * c;
}

// Bit s of every byte of h moved to bit 2 (the high bit of a 3-bit code).
template <int S>
__device__ __forceinline__ uint32_t hi_bit(uint32_t h) {
  if constexpr (S >= 2) return (h >> (S - 2)) & 0x04040404u;
  else return (h << (2 - S)) & 0x04040404u;
}

// f16 (1024 + q_f) pairs for rows g8 (lo_row) / g8 + 8 (hi_row) of two
// channels whose refinement words are wa, wb (bits b_f*r + off hold row r).
template <int BF>
__device__ __forceinline__ void qf_frag(uint32_t wa, uint32_t wb, int g8, int off, uint32_t& lo_row,
                                        uint32_t& hi_row) {
  if constexpr (BF == 2) {
    const uint32_t xa = wa >> (2 * g8 + off), xb = wb >> (2 * g8 + off);
    lo_row = (__byte_perm(xa, xb, 0x5410) & 0x00030003u) | 0x64006400u;  // row g8: bits 0-1 of each half
    hi_row = (__byte_perm(xa, xb, 0x7632) & 0x00030003u) | 0x64006400u;  // row g8 + 8: bits 16-17
  } else {
    const uint32_t xa = wa >> (g8 + off), xb = wb >> (g8 + off);
    const uint32_t p = __byte_perm(xa, xb, 0x5410);  // row g8 at bit 0, row g8 + 8 at bit 8 of each half
    lo_row = (p & 0x00010001u) | 0x64006400u;
    hi_row = ((p >> 8) & 0x00010001u) | 0x64006400u;
  }
}

// The producer's row into xs (bf16 bits), with the arithmetic of
// produce_select_kernel (decode_fused.cu): kProdNorm y = bf16(RMSNorm(x +
// delta) w) (fp32 add, fp64 sum of squares in the order of 1024 threads,
// fp64 scaling, one rounding), kProdRound y = bf16(x), kProdSilu y =
// bf16(silu(x) u).  A thread's entries are i = tid + j blockDim.x, loaded
// kProdBatch at a time with every load in flight (the weight stream keeps
// the memory system busy, so each round trip is long).  vbuf (vcap floats of
// scratch) holds x + delta for the fp64 sum when the row fits (else the sum
// re-reads x and delta).  Every CTA writes y to global memory (the same
// values) and CTA 0 the updated residual.  Ends with a barrier.
constexpr int kProdBatch = 12;

__device__ void produce_row(const MProd& P, int K, uint16_t* xs, float* vbuf, int vcap, double* part,
                            double* inv_sh) {
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5, nw = nthr >> 5;
  if (P.op == kProdNorm) {
    const bool keep = K <= vcap;
    // one load round for x, delta and w when a thread's entries fit one batch
    const bool one = keep && K <= kProdBatch * nthr;
    const bool cta0 = blockIdx.x == 0 && P.x_out != nullptr;
    float wv[kProdBatch];
    if (keep) {
      for (int i0 = 0; i0 < K; i0 += kProdBatch * nthr) {
        float xv[kProdBatch], dv[kProdBatch];
#pragma unroll
        for (int j = 0; j < kProdBatch; ++j) {
          const int i = i0 + tid + j * nthr;
          xv[j] = i < K ? P.x[i] : 0.0f;
          dv[j] = i < K && P.delta ? P.delta[i] : 0.0f;
          wv[j] = one && i < K ? P.w[i] : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < kProdBatch; ++j) {
          const int i = i0 + tid + j * nthr;
          if (i < K) {
            const float v = P.delta ? __fadd_rn(xv[j], dv[j]) : xv[j];
            vbuf[i] = v;
            if (cta0) P.x_out[i] = v;
          }
        }
      }
      __syncthreads();
    }
    // virtual warp vw (threads 32 vw .. 32 vw + 31 of the 1024) is taken by
    // warp vw % nw, whose lanes coincide with the virtual lanes
    for (int vw = warp; vw < 32; vw += nw) {
      const int vt = 32 * vw + lane;
      double ss = 0.0;
      for (int i = vt; i < K; i += sfd::kNormVThreads) {
        float v;
        if (keep) {
          v = vbuf[i];
        } else {
          v = P.x[i];
          if (P.delta) v = __fadd_rn(v, P.delta[i]);
        }
        ss = fma(static_cast<double>(v), static_cast<double>(v), ss);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) part[vw] = ss;
    }
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int i = 0; i < sfd::kNormVThreads / 32; ++i) t += part[i];
      *inv_sh = 1.0 / sqrt(t / K + static_cast<double>(P.eps));
    }
    __syncthreads();
    const double inv = *inv_sh;
    for (int i0 = 0; i0 < K; i0 += kProdBatch * nthr) {
      float xv[kProdBatch], dv[kProdBatch];
      if (!one) {
#pragma unroll
        for (int j = 0; j < kProdBatch; ++j) {
          const int i = i0 + tid + j * nthr;
          wv[j] = i < K ? P.w[i] : 0.0f;
          if (!keep) {
            xv[j] = i < K ? P.x[i] : 0.0f;
            dv[j] = i < K && P.delta ? P.delta[i] : 0.0f;
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kProdBatch; ++j) {
        const int i = i0 + tid + j * nthr;
        if (i < K) {
          float v;
          if (keep) {
            v = vbuf[i];
          } else {
            v = P.delta ? __fadd_rn(xv[j], dv[j]) : xv[j];
            if (cta0) P.x_out[i] = v;
          }
          const uint16_t y = sfd::to_bf16(static_cast<double>(v) * inv * static_cast<double>(wv[j]));
          xs[i] = y;
          P.y[i] = y;
        }
      }
    }
  } else {
    const bool silu = P.op == kProdSilu;
    for (int i0 = 0; i0 < K; i0 += kProdBatch * nthr) {
      float av[kProdBatch], uv[kProdBatch];
#pragma unroll
      for (int j = 0; j < kProdBatch; ++j) {
        const int i = i0 + tid + j * nthr;
        av[j] = i < K ? P.x[i] : 0.0f;
        uv[j] = i < K && silu ? P.u[i] : 0.0f;
      }
#pragma unroll
      for (int j = 0; j < kProdBatch; ++j) {
        const int i = i0 + tid + j * nthr;
        if (i < K) {
          const uint16_t y = silu ? sfd::silu_mul_bf16(av[j], uv[j])
                                  : __bfloat16_as_ushort(__float2bfloat16_rn(av[j]));
          xs[i] = y;
          P.y[i] = y;
        }
      }
    }
  }
  __syncthreads();
}

// Words of the producer's scratch (the last ring stage of every warp) taken
// before the selection list: the row, the histogram rows, scan and info.
__host__ __device__ constexpr int prod_row_words(int K) { return (K / 2 + 3) & ~3; }
__host__ __device__ constexpr int prod_fixed_words(int K, int hrows) { return prod_row_words(K) + hrows * 256 + 48; }

template <int SPW, int BR>
struct MCfg {
  static constexpr int kCodeWords = 128 * BR;              // 16 rows x 8 BR words
  static constexpr int kSZ = kCodeWords;                   // scale/zero: 32 words
  static constexpr int kRF = kCodeWords + 32;              // refinement: 32 words
  static constexpr int kSliceWords = kCodeWords + 64;      // words per slice and stage
  // 16 warps (14 of two slices) fit 227 KB
  static constexpr int kStages = SPW == 1 ? (BR == 2 ? 8 : 7) : (BR == 2 ? 5 : 4);
  static constexpr int kRedTiles = SPW == 1 ? 16 : 4;  // tiles whose warp partials wait for one reduction
  static constexpr int SW = SPW * kSliceWords;  // ring words per warp and stage
  static size_t smem_bytes(int W) {
    return sizeof(uint32_t) * (static_cast<size_t>(W) * kStages * SW           // rings
                               + static_cast<size_t>(W) * SPW * kCorrList / 2   // listed channels (u16)
                               + static_cast<size_t>(kRedTiles) * W * kRows);   // row partials of the warps
  }
};

// PROD: the launch makes its own input row and selection (a.prod); the
// plain instantiation reads them from a.x, a.idx, a.n_sel.
template <int SPW, int BF, int BR, bool PROD>
__global__ void __launch_bounds__(kMaxWarps * 32, 1)
gemv_mma_kernel(const __grid_constant__ MArgs a) {
  using C = MCfg<SPW, BR>;
  constexpr int kStages = C::kStages, SW = C::SW, kRedTiles = C::kRedTiles;
  constexpr int kSliceWords = C::kSliceWords, kSZ = C::kSZ, kRF = C::kRF;
  extern __shared__ __align__(16) uint32_t sm[];
  const int W = blockDim.x >> 5;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g8 = lane >> 2, tig = lane & 3;
  const int ks = blockIdx.x % a.ksplit, crow = blockIdx.x / a.ksplit, ncta = gridDim.x / a.ksplit;
  // ring stage s of warp w at sm + (s W + w) SW: the last stage of all warps
  // is one contiguous block, the producer's scratch until the main loop
  auto stage_base = [&](int st) { return sm + (st * W + warp) * SW; };
  uint16_t* mylist = reinterpret_cast<uint16_t*>(sm + W * kStages * SW) + warp * SPW * kCorrList;  // [SPW][32]
  float* red = reinterpret_cast<float*>(sm + W * kStages * SW + W * SPW * kCorrList / 2);

  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const bool pair = a.ksplit > 1;  // launched as clusters of the two K halves
  const int slice0 = (ks * W + warp) * SPW;
  const int myslot = tig >> 1, myrow = g8 + 8 * (tig & 1);
  const bool even = (tig & 1) == 0;
  const float m_f = static_cast<float>((1 << BF) - 1) * 0.5f;
  const uint32_t fmask = (1u << BF) - 1u;

  const size_t row_words = static_cast<size_t>(a.K) * BR / 32;
  const int last = a.njobs - 1;
  const int total_tiles = a.job[last].tile_begin + a.job[last].N / kRows;
  // a contiguous block of tiles per CTA: consecutive tiles read consecutive
  // words of each selected channel's refinement row (one sector serves 8 or 16)
  const int per_cta = (total_tiles + ncta - 1) / ncta;
  const int t_begin = crow * per_cta;
  const int my_tiles = max(0, min(total_tiles, t_begin + per_cta) - t_begin);
  // per-warp state filled by the setup below (issued after the first code copies)
  uint32_t bf[SPW][8][2];
  uint32_t cb[SPW][2][2];
  float fsc[SPW], gsm[SPW], cconst[SPW];
  int nsl[SPW], psl[SPW];
  int ntc[SPW];  // selected channels of the slice corrected on the tensor cores (the rest in fp32)
  uint32_t hl_l[SPW];  // lane k < ntc: (high, low) halves of x of listed channel k
  int grp_l[SPW];      // and its group inside the slice (-1: none)

  // Copies are issued tile by tile in order, so their addresses advance by
  // fixed strides and are recomputed only where the next matrix begins.
  // Code cursor: codes and scale/zero (they depend on nothing the previous
  // kernel writes); ref cursor: the refinement words of the listed channels.
  // this lane's BR code chunks of a tile's slice: chunk lane + 32 i of the
  // slice's 16 rows x 2 BR chunks
  int c_soff[BR];      // word offset in the stage
  size_t c_goff[BR];   // word offset from the tile's first row in the matrix
#pragma unroll
  for (int i = 0; i < BR; ++i) {
    const int c = lane + 32 * i, r = c / (2 * BR), ch = c % (2 * BR);
    c_soff[i] = code_off<BR>(r, ch);
    c_goff[i] = static_cast<size_t>(r) * row_words + 4 * ch;
  }
  const int sz_grp = lane >> 2, sz_arr = (lane >> 1) & 1, sz_hf = lane & 1;  // lanes 0-7
  int c_t = t_begin, c_jb = my_tiles > 0 ? job_of(a, t_begin) : 0, c_next = 0;
  const uint32_t* c_code = nullptr;  // the tile's first row, slice0
  const uint16_t* c_sz = nullptr;    // lanes 0-7: scale or zero of (slice0, group), rows row0 + 8 hf
  size_t c_szs = 0;                  // elements between consecutive slices' scale rows
  auto c_seek = [&]() {              // the cursor's tile starts (or the job changes)
    const MJob& J = a.job[c_jb];
    const int row0 = (c_t - J.tile_begin) * kRows;
    c_next = c_jb + 1 < a.njobs ? a.job[c_jb + 1].tile_begin : 0x7FFFFFFF;
    c_code = J.res + static_cast<size_t>(row0) * row_words + 8 * BR * slice0;
    c_szs = 2 * static_cast<size_t>(J.N);
    c_sz = (sz_arr ? J.zero : J.scale) + static_cast<size_t>(2 * slice0 + sz_grp) * J.N + row0 + 8 * sz_hf;
  };
  if (my_tiles > 0) c_seek();
  const int c_jb0 = c_jb;
  auto issue_codes = [&](int i) {
    if (c_t == c_next) {
      ++c_jb;
      c_seek();
    }
    uint32_t* stage = stage_base(i % kStages);
#pragma unroll
    for (int sp = 0; sp < SPW; ++sp) {
      uint32_t* base = stage + sp * kSliceWords;
#pragma unroll
      for (int q = 0; q < BR; ++q) cp_async16(base + c_soff[q], c_code + c_goff[q] + 8 * BR * sp);
      if (lane < 8)
        cp_async16(reinterpret_cast<uint16_t*>(base + kSZ) + (sz_grp * 2 + sz_arr) * 16 + 8 * sz_hf,
                   c_sz + sp * c_szs);
    }
    c_code += kRows * row_words;
    c_sz += kRows;
    ++c_t;
  };
  int r_t = t_begin, r_jb = c_jb0, r_next = 0, r_tb = 0;
  bool r_has = false;
  const uint32_t* r_row[SPW];  // lanes below the list length: refinement row of listed channel lane
  auto r_seek = [&]() {
    const MJob& J = a.job[r_jb];
    r_next = r_jb + 1 < a.njobs ? a.job[r_jb + 1].tile_begin : 0x7FFFFFFF;
    r_tb = J.tile_begin;
    r_has = J.ref_rows != nullptr;
#pragma unroll
    for (int sp = 0; sp < SPW; ++sp) {
      r_row[sp] = J.ref_rows;
      if (r_has && lane < ntc[sp]) {
        const int ch = 256 * (slice0 + sp) + mylist[sp * kCorrList + lane];
        int rr = J.unit_slot ? J.unit_slot[ch] : (J.row_of ? J.row_of[psl[sp] + lane] : ch);
        rr = rr < 0 ? 0 : rr;  // not cached (deadline reading): any row; its B column is zero
        r_row[sp] = J.ref_rows + static_cast<size_t>(rr) * J.unit_words;
      }
    }
  };
  auto issue_refs = [&](int i) {
    if (r_t == r_next) {
      ++r_jb;
      r_seek();
    }
    if (r_has) {
      const int woff = ((r_t - r_tb) * kRows * BF) >> 5;
      uint32_t* stage = stage_base(i % kStages);
#pragma unroll
      for (int sp = 0; sp < SPW; ++sp)
        if (lane < ntc[sp]) cp_async4(stage + sp * kSliceWords + kRF + lane, r_row[sp] + woff);
    }
    ++r_t;
  };

#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (i < my_tiles) issue_codes(i);
    cp_async_commit();
  }
  // ---- per-warp setup, from x and the selection list: the B fragments of
  // the slice's fixed-point activations, the group scalars, the slice's
  // selected channels, the correction MMA's B fragments (x of the listed
  // channels, high and low).  Launched with programmatic stream
  // serialization, the kernel may have started before the producer of x and
  // the selection finished: the code copies above need nothing it writes.
  pdl_wait_gemv();
  constexpr bool produce = PROD;
  const uint16_t* xrow = a.x;  // the row and its selection for the setup below
  const int32_t* sel = a.idx;
  int n_all;
  if constexpr (PROD) {
    // the row and its selection, computed by this CTA in the last ring stage
    __shared__ double part[sfd::kNormVThreads / 32];
    __shared__ double inv_sh;
    uint32_t* scr = sm + (kStages - 1) * W * SW;
    uint16_t* xs = reinterpret_cast<uint16_t*>(scr);
    int* whist = reinterpret_cast<int*>(scr + prod_row_words(a.K));
    int* sscan = whist + a.prod.hrows * 256;
    int* info = sscan + 40;
    int32_t* list = reinterpret_cast<int32_t*>(scr + prod_fixed_words(a.K, a.prod.hrows));
    // x + delta kept between the producer's sweeps in the rest of the scratch
    produce_row(a.prod, a.K, xs, reinterpret_cast<float*>(whist), W * SW - prod_row_words(a.K), part, &inv_sh);
    sfd::select_row_cta(xs, a.K, a.prod.k, list, whist, a.prod.hrows, sscan, info, nullptr);
    // every CTA writes the same selection; the fp32 correction reads it back
    const int taken = info[6];
    for (int i = tid; i < taken; i += blockDim.x) a.prod.idx[i] = list[i];
    if (tid == 0) *a.prod.n = info[5];
    n_all = info[5] < 0 ? 0 : info[5];
    xrow = xs;
    sel = list;
  } else {
    n_all = a.idx != nullptr ? *a.n_sel : 0;
    n_all = n_all < 0 ? 0 : n_all;
  }
#pragma unroll
  for (int sp = 0; sp < SPW; ++sp) {
    const int slice = slice0 + sp;
    {
      // lane (col n, t): group slot_b = n / 4, digit plane n % 4 (3: zero);
      // its B registers hold that plane's digits of channels
      // 128 slot_b + 32 t + [0, 32) of the slice.  The four lanes of one
      // (slot_b, t) share those channels: lane plane q converts channels
      // 8q .. 8q + 7 and the lanes swap digit bytes by shuffles.
      const int bn = lane >> 2, slot_b = bn >> 2, plane = bn & 3;
      const uint4 v = *reinterpret_cast<const uint4*>(xrow + 256 * static_cast<size_t>(slice) + 128 * slot_b +
                                                     32 * tig + 8 * plane);
      const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
      // the group's largest |x| (15-bit magnitude keys order as |x| does):
      // lanes of one slot_b hold its 128 channels
      uint32_t kmax = 0u;
#pragma unroll
      for (int w = 0; w < 4; ++w) kmax = max(kmax, max(xw[w] & 0x7FFFu, (xw[w] >> 16) & 0x7FFFu));
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
      int e = sfd::bf16_exponent(kmax);
      if (e == -1000) e = 0;
      // X = rint(x 2^(22 - e)): exact power-of-two factors (two, so a group
      // of bf16 subnormals does not overflow one), rounding to nearest even
      const int s1 = min(22 - e, 126);
      const float sc1 = ldexpf(1.0f, s1), sc2 = ldexpf(1.0f, 22 - e - s1);
      int gs = 0;
      // pk[p][h]: plane-p digits of my channels 8 plane + 4 h + [0, 4): bytes
      // in channel order
      uint32_t pk[3][2] = {{0u, 0u}, {0u, 0u}, {0u, 0u}};
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int X = __float2int_rn(__uint_as_float(((xw[c >> 1] >> (16 * (c & 1))) & 0xFFFFu) << 16) * sc1 * sc2);
        gs += X;
        const int d0 = ((X + 128) & 255) - 128;
        const int X1 = (X - d0) >> 8;
        const int d1 = ((X1 + 128) & 255) - 128;
        const int d2 = (X1 - d1) >> 8;
        pk[0][c >> 2] |= (static_cast<uint32_t>(d0) & 0xFFu) << (8 * (c & 3));
        pk[1][c >> 2] |= (static_cast<uint32_t>(d1) & 0xFFu) << (8 * (c & 3));
        pk[2][c >> 2] |= (static_cast<uint32_t>(d2) & 0xFFu) << (8 * (c & 3));
      }
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) gs += __shfl_xor_sync(0xffffffffu, gs, o);  // the group's 128
      // channel c of my run -> k-step 4 slot_b + mm, register r, byte b:
      // mm = 2 (c >> 4) + ((c >> 1) & 1), b = (c >> 2) & 3, r = c & 1.  The
      // channels 8q + [0, 8) of lane plane q fill bytes 2 (q & 1) + {0, 1} of
      // the words (mm, r) with mm >> 1 = q >> 1.
      uint32_t dg[4][2] = {{0u, 0u}, {0u, 0u}, {0u, 0u}, {0u, 0u}};
#pragma unroll
      for (int d = 0; d < 4; ++d) {
        const int q = plane ^ d;  // the lane I receive from (and send to)
        // send the digits of the receiver's plane (plane ^ d == q's plane)
        const int rp = q;         // receiver of my data has plane q
        const uint32_t s0 = rp == 0 ? pk[0][0] : (rp == 1 ? pk[1][0] : (rp == 2 ? pk[2][0] : 0u));
        const uint32_t s1w = rp == 0 ? pk[0][1] : (rp == 1 ? pk[1][1] : (rp == 2 ? pk[2][1] : 0u));
        const uint32_t r0 = __shfl_xor_sync(0xffffffffu, s0, 4 * d);
        const uint32_t r1 = __shfl_xor_sync(0xffffffffu, s1w, 4 * d);
        // r0 bytes: channels 8q + {0..3} = (mm = 2 (q >> 1) + 0/1 by bit 1 of c, r by bit 0, b = 2 (q & 1))
        //   c = 8q + i, i = 0..3: (c >> 1) & 1 = i >> 1, r = i & 1, b = 2 (q & 1)
        // r1 bytes: channels 8q + 4 + i: b = 2 (q & 1) + 1
        const bool upper = (q >> 1) != 0;  // k-steps mm = 2, 3 (else 0, 1): selects keep dg in registers
        const int bb = 2 * (q & 1);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = i & 1;
          const uint32_t bits = (((r0 >> (8 * i)) & 0xFFu) << (8 * bb)) | (((r1 >> (8 * i)) & 0xFFu) << (8 * (bb + 1)));
          dg[(i >> 1)][r] |= upper ? 0u : bits;
          dg[2 + (i >> 1)][r] |= upper ? bits : 0u;
        }
      }
#pragma unroll
      for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int r = 0; r < 2; ++r) bf[sp][m][r] = (m >> 2) == slot_b ? dg[m & 3][r] : 0u;
      // the epilogue's lane (row, group myslot) takes its group's scalars
      const float fs = ldexpf(1.0f, e - 22);
      const float gsum = static_cast<float>(gs) * fs;
      fsc[sp] = __shfl_sync(0xffffffffu, fs, 16 * myslot);
      gsm[sp] = __shfl_sync(0xffffffffu, gsum, 16 * myslot);
    }
    {
      // the slice's run of the ascending selection: two rounds of a 32-way
      // search (the first on every ceil(n / 32)-th entry, the second inside
      // the segment it finds), for both ends of the slice
      const int lo = 256 * slice, hi = lo + 256;
      const int step = (n_all + 31) >> 5;
      int c_lo = 0, c_hi = 0;
      if (step > 32) {  // more than 1024 selected: count by a plain sweep
        for (int i = lane; i < n_all; i += 32) {
          const int w = sel[i];
          c_lo += w < lo;
          c_hi += w < hi;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          c_lo += __shfl_xor_sync(0xffffffffu, c_lo, o);
          c_hi += __shfl_xor_sync(0xffffffffu, c_hi, o);
        }
      } else if (n_all > 0) {
        const int p1 = min(n_all - 1, lane * step);
        const int v1 = sel[p1];
        const bool in1 = lane * step < n_all;
        const int seg_lo = __popc(__ballot_sync(0xffffffffu, in1 && v1 < lo));  // segments entirely below lo
        const int seg_hi = __popc(__ballot_sync(0xffffffffu, in1 && v1 < hi));
        // entries before segment seg - 1 are all below the bound; search it
        const int b_lo = max(seg_lo - 1, 0) * step, b_hi = max(seg_hi - 1, 0) * step;
        const bool ok_lo = lane < step && b_lo + lane < n_all, ok_hi = lane < step && b_hi + lane < n_all;
        const int w_lo = ok_lo ? sel[b_lo + lane] : 0x7FFFFFFF;
        const int w_hi = ok_hi ? sel[b_hi + lane] : 0x7FFFFFFF;
        c_lo = b_lo + __popc(__ballot_sync(0xffffffffu, ok_lo && w_lo < lo));
        c_hi = b_hi + __popc(__ballot_sync(0xffffffffu, ok_hi && w_hi < hi));
      }
      psl[sp] = c_lo;
      nsl[sp] = c_hi - c_lo;
      if (lane < min(nsl[sp], kCorrList)) mylist[sp * kCorrList + lane] = static_cast<uint16_t>(sel[c_lo + lane] - lo);
    }
    __syncwarp();
    int nl = min(nsl[sp], kCorrList);
    float xv = 0.0f;
    if (lane < nl) xv = sfd::bf16_bits_to_float(xrow[256 * slice + mylist[sp * kCorrList + lane]]);
    // a listed |x| at or above 2^15 would overflow the f16 split: the whole
    // slice is then corrected by the fp32 loop
    if (__any_sync(0xffffffffu, !(fabsf(xv) < kCorrXMax))) nl = 0;
    ntc[sp] = nl;
    uint32_t hl = 0;
    int grp = -1;
    if (lane < nl) {
      const int ch = mylist[sp * kCorrList + lane];
      const __half hi = __float2half_rn(xv);
      const __half lo = __float2half_rn(xv - __half2float(hi));
      hl = static_cast<uint32_t>(__half_as_ushort(hi)) | (static_cast<uint32_t>(__half_as_ushort(lo)) << 16);
      grp = ch >> 7;
    }
    hl_l[sp] = hl;
    grp_l[sp] = grp;
  }
  if constexpr (PROD) __syncthreads();  // every warp is done with the scratch before the main loop refills it
  // the correction MMA's B fragments and offset constant for the job the
  // compute cursor is in: a job reading a cache in the deadline reading drops
  // the listed channels not cached (their x becomes 0)
  auto build_corr = [&](const MJob& J) {
#pragma unroll
    for (int sp = 0; sp < SPW; ++sp) {
      const int nl = ntc[sp];
      uint32_t hl = hl_l[sp];
      const int grp = grp_l[sp];
      if (J.unit_slot != nullptr && lane < nl && J.unit_slot[256 * (slice0 + sp) + mylist[sp * kCorrList + lane]] < 0)
        hl = 0u;
      const float part = lane < nl ? __half2float(__ushort_as_half(static_cast<unsigned short>(hl & 0xFFFFu))) +
                                         __half2float(__ushort_as_half(static_cast<unsigned short>(hl >> 16)))
                                   : 0.0f;
      float x0 = grp == 0 ? part : 0.0f, x1 = grp == 1 ? part : 0.0f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        x0 += __shfl_xor_sync(0xffffffffu, x0, o);
        x1 += __shfl_xor_sync(0xffffffffu, x1, o);
      }
      cconst[sp] = -(1024.0f + m_f) * (myslot ? x1 : x0);
      // column n of the correction MMA = (group n / 2, part n % 2)
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          uint32_t v = 0;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int k = 16 * kb + 2 * tig + 8 * r + h;  // < 32: a lane of the warp
            const uint32_t hk = __shfl_sync(0xffffffffu, hl, k);
            const int gk = __shfl_sync(0xffffffffu, grp, k);
            if (g8 < 4 && k < nl && gk == (g8 >> 1)) v |= ((g8 & 1) ? (hk >> 16) : (hk & 0xFFFFu)) << (16 * h);
          }
          cb[sp][kb][r] = v;
        }
    }
  };
  if (my_tiles > 0) build_corr(a.job[c_jb0]);

  if (my_tiles > 0) r_seek();
  for (int i = 0; i < kStages - 1 && i < my_tiles; ++i) issue_refs(i);
  cp_async_commit();
  int k_jb = c_jb0, k_next = c_jb0 + 1 < a.njobs ? a.job[c_jb0 + 1].tile_begin : 0x7FFFFFFF;  // compute cursor
  for (int i = 0; i < my_tiles; ++i) {
    if (i + kStages - 1 < my_tiles) {
      issue_codes(i + kStages - 1);
      issue_refs(i + kStages - 1);
    }
    cp_async_commit();
    // tile i needs its code group and the prologue's refinement group, which
    // has i + 1 newer groups while i + 1 < kStages - 1
    switch (min(i + 1, kStages - 1)) {
      case 1: cp_async_wait<1>(); break;
      case 2: cp_async_wait<2>(); break;
      case 3: cp_async_wait<3>(); break;
      case 4: cp_async_wait<4>(); break;
      case 5: cp_async_wait<5>(); break;
      case 6: cp_async_wait<6>(); break;
      default: cp_async_wait<kStages - 1>(); break;
    }
    __syncwarp();
    const int st = i % kStages;
    const int t = t_begin + i;
    if (t == k_next) {
      ++k_jb;
      k_next = k_jb + 1 < a.njobs ? a.job[k_jb + 1].tile_begin : 0x7FFFFFFF;
      build_corr(a.job[k_jb]);
    }
    const MJob& J = a.job[k_jb];
    const int row0 = (t - J.tile_begin) * kRows;
    const int roff = (row0 * BF) & 31;
    float v = 0.0f;
#pragma unroll
    for (int sp = 0; sp < SPW; ++sp) {
      const uint32_t* base = stage_base(st) + sp * kSliceWords;
      // (low) code words: rows g8 and g8 + 8, words 2 tig, 2 tig + 1 of each group
      const uint2 r0a = *reinterpret_cast<const uint2*>(base + code_off<BR>(g8, tig >> 1) + 2 * (tig & 1));
      const uint2 r0b = *reinterpret_cast<const uint2*>(base + code_off<BR>(g8, 2 + (tig >> 1)) + 2 * (tig & 1));
      const uint2 r1a = *reinterpret_cast<const uint2*>(base + code_off<BR>(g8 + 8, tig >> 1) + 2 * (tig & 1));
      const uint2 r1b = *reinterpret_cast<const uint2*>(base + code_off<BR>(g8 + 8, 2 + (tig >> 1)) + 2 * (tig & 1));
      // 3-bit: the high-bit words of both groups (.x group 0, .y group 1)
      uint2 h0 = make_uint2(0u, 0u), h1 = make_uint2(0u, 0u);
      if constexpr (BR == 3) {
        h0 = *reinterpret_cast<const uint2*>(base + g8 * 24 + 16 + 2 * tig);
        h1 = *reinterpret_cast<const uint2*>(base + (g8 + 8) * 24 + 16 + 2 * tig);
      }
      int d[4] = {0, 0, 0, 0}, e[4] = {0, 0, 0, 0};
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int slot = m >> 2, hi = (m >> 1) & 1, j = 2 * (m & 1);
        const uint32_t w0 = slot ? (hi ? r0b.y : r0b.x) : (hi ? r0a.y : r0a.x);
        const uint32_t w1 = slot ? (hi ? r1b.y : r1b.x) : (hi ? r1a.y : r1a.x);
        uint32_t a0 = (w0 >> (2 * j)) & 0x03030303u;
        uint32_t a1 = (w1 >> (2 * j)) & 0x03030303u;
        uint32_t a2 = (w0 >> (2 * j + 2)) & 0x03030303u;
        uint32_t a3 = (w1 >> (2 * j + 2)) & 0x03030303u;
        if constexpr (BR == 3) {
          const uint32_t x0 = slot ? h0.y : h0.x, x1 = slot ? h1.y : h1.x;
          // channel offset j (j + 1) of low word `hi`: bit 4 hi + j (+ 1)
          switch (4 * hi + j) {
            case 0: a0 |= hi_bit<0>(x0); a1 |= hi_bit<0>(x1); a2 |= hi_bit<1>(x0); a3 |= hi_bit<1>(x1); break;
            case 2: a0 |= hi_bit<2>(x0); a1 |= hi_bit<2>(x1); a2 |= hi_bit<3>(x0); a3 |= hi_bit<3>(x1); break;
            case 4: a0 |= hi_bit<4>(x0); a1 |= hi_bit<4>(x1); a2 |= hi_bit<5>(x0); a3 |= hi_bit<5>(x1); break;
            default: a0 |= hi_bit<6>(x0); a1 |= hi_bit<6>(x1); a2 |= hi_bit<7>(x0); a3 |= hi_bit<7>(x1); break;
          }
        }
        if (m & 1) mma_u8s8(e, a0, a1, a2, a3, bf[sp][m][0], bf[sp][m][1]);
        else mma_u8s8(d, a0, a1, a2, a3, bf[sp][m][0], bf[sp][m][1]);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) d[c] += e[c];
      // even lanes: d0, d1 = planes 0, 1 of row g8 and d2, d3 = planes 0, 1 of
      // row g8 + 8; odd lanes: d0, d2 = plane 2 of rows g8, g8 + 8.  Plane sums
      // are below 7 * 128 * 128 < 2^17 in magnitude: exact small-integer
      // conversions.
      const float f0 = i2f_small(d[0]), f1 = i2f_small(d[1]), f2 = i2f_small(d[2]), f3 = i2f_small(d[3]);
      const float send = even ? fmaf(f3, 256.0f, f2) : 65536.0f * f0;
      const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
      const float P = even ? fmaf(f1, 256.0f, f0) + recv : fmaf(65536.0f, f2, recv);
      const uint16_t* szs = reinterpret_cast<const uint16_t*>(base + kSZ);
      const float sc = h2f_bits(szs[(myslot * 2) * 16 + myrow]);
      const float zz = h2f_bits(szs[(myslot * 2 + 1) * 16 + myrow]);
      float tsum = fmaf(static_cast<float>(1 << BF) * fsc[sp], P, (m_f - zz) * gsm[sp]);
      if (J.ref_rows && nsl[sp] > 0) {
        const uint32_t* refw = base + kRF;
        float c4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const int nl = ntc[sp];
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          if (16 * kb < nl) {  // uniform over the warp
            // entries at or beyond nl hold stale words: their B columns are zero
            const int k0 = 16 * kb + 2 * tig;
            uint32_t qa0, qa1, qa2, qa3;
            qf_frag<BF>(refw[k0], refw[k0 + 1], g8, roff, qa0, qa1);
            qf_frag<BF>(refw[k0 + 8], refw[k0 + 9], g8, roff, qa2, qa3);
            mma_f16(c4, qa0, qa1, qa2, qa3, cb[sp][kb][0], cb[sp][kb][1]);
          }
        }
        // lane (g8, t), t < 2, holds group t's (high, low) columns for rows g8 and g8 + 8
        const float u0 = __shfl_sync(0xffffffffu, c4[0] + c4[1], 4 * g8 + myslot);
        const float u1 = __shfl_sync(0xffffffffu, c4[2] + c4[3], 4 * g8 + myslot);
        float corr = nl > 0 ? ((tig & 1) ? u1 : u0) + cconst[sp] : 0.0f;
        // channels beyond the tensor-core list (more than kCorrList selected in
        // the slice, or every selected channel of a slice with a huge |x|)
        for (int k = nl; k < nsl[sp]; ++k) {
          const int ch = a.idx[psl[sp] + k];  // the slice's k-th selected channel (global)
          if (((ch >> 7) & 1) != myslot) continue;
          const int rr = J.unit_slot ? J.unit_slot[ch] : (J.row_of ? J.row_of[psl[sp] + k] : ch);
          if (rr < 0) continue;  // not cached at the step's start (deadline reading): resident precision
          const uint32_t word = J.ref_rows[static_cast<size_t>(rr) * J.unit_words + ((row0 * BF) >> 5)];
          const float xv = sfd::bf16_bits_to_float(a.x[ch]);
          corr = fmaf(xv, i2f_small(static_cast<int>((word >> (roff + BF * myrow)) & fmask)) - m_f, corr);
        }
        tsum += corr;
      }
      v = fmaf(sc, tsum, v);
    }
    // lanes tig and tig ^ 2 hold the same row for the two groups; the warps'
    // partials of up to kRedTiles tiles are summed together (no barrier per tile)
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    if (tig < 2) red[((i % kRedTiles) * W + warp) * kRows + myrow] = v;
    if (i % kRedTiles == kRedTiles - 1 || i == my_tiles - 1) {
      // with two K halves the CTAs of a cluster pair hold the same tiles:
      // each writes half of the rows, summing both CTAs' warp partials
      // through distributed shared memory (half 0's sum plus half 1's)
      if (pair) cl.sync();
      else __syncthreads();
      const int i0 = i - i % kRedTiles, nt = i - i0 + 1;
      const int rows = pair ? kRows / 2 : kRows, r0 = ks * rows;
      const float* red0 = pair ? cl.map_shared_rank(red, 0) : red;
      const float* red1 = pair ? cl.map_shared_rank(red, 1) : red;
      // every partial of a row is loaded before the sum (the partner's are
      // remote loads), then added in warp order
      auto sum_warps = [&](const float* rd, int ti, int rr) {
        float t[kMaxWarps];
#pragma unroll
        for (int w = 0; w < kMaxWarps; ++w) t[w] = w < W ? rd[(ti * W + w) * kRows + rr] : 0.0f;
        float acc = 0.0f;
#pragma unroll
        for (int w = 0; w < kMaxWarps; ++w)
          if (w < W) acc += t[w];
        return acc;
      };
      for (int e = tid; e < nt * rows; e += blockDim.x) {
        const int ti = e / rows, rr = r0 + e % rows;
        float acc = sum_warps(red0, ti, rr);
        if (pair) acc += sum_warps(red1, ti, rr);
        const int tt = t_begin + i0 + ti;
        const MJob& Jt = a.job[job_of(a, tt)];
        Jt.y[(tt - Jt.tile_begin) * kRows + rr] = acc;
      }
      if (pair) cl.sync();  // the partner has read this CTA's partials
      else __syncthreads();
    }
  }
  cp_async_wait<0>();
}

std::atomic<int> g_gemv_overlap{0};

// (slices per warp, K halves) for K / 256 slices: at most 16 warps per CTA.
bool pick_split(int nslice, int* spw, int* ksplit) {
  const int cand[4][2] = {{1, 1}, {1, 2}, {2, 1}, {2, 2}};
  for (const auto& c : cand) {
    if (nslice % (c[0] * c[1])) continue;
    const int w = nslice / (c[0] * c[1]);
    if (w >= 1 && w <= kMaxWarps) {
      *spw = c[0];
      *ksplit = c[1];
      return true;
    }
  }
  return false;
}


// Canonical 3-bit rows -> the split batch-1 layout: one thread per (row,
// 256-channel slice); the slice's 256 codes are 24 whole words in both.
__global__ void pack_res3_kernel(const uint32_t* __restrict__ res, int nrows, int nslice,
                                 uint32_t* __restrict__ out) {
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= static_cast<long long>(nrows) * nslice) return;
  const uint32_t* src = res + e * 24;
  uint32_t lo[16], hb[8];
#pragma unroll
  for (int w = 0; w < 16; ++w) lo[w] = 0u;
#pragma unroll
  for (int w = 0; w < 8; ++w) hb[w] = 0u;
  for (int c = 0; c < 256; ++c) {
    const int bit = 3 * c, wd = bit >> 5, sh = bit & 31;
    uint32_t v = src[wd] >> sh;
    if (sh > 29) v |= src[wd + 1] << (32 - sh);
    v &= 7u;
    const int w = c >> 4, b = (c >> 2) & 3, j = c & 3;
    lo[w] |= (v & 3u) << (8 * b + 2 * j);
    const int slot = w >> 3, t = (w & 7) >> 1, h = w & 1;
    hb[2 * t + slot] |= (v >> 2) << (8 * b + 4 * h + j);
  }
  uint32_t* dst = out + e * 24;
#pragma unroll
  for (int w = 0; w < 16; ++w) dst[w] = lo[w];
#pragma unroll
  for (int w = 0; w < 8; ++w) dst[16 + w] = hb[w];
}

}  // namespace

extern "C" sf_status sf_gemv_pack_batch1(const uint32_t* res, int N, int K, int b_r, uint32_t* out,
                                         sf_stream_t stream) {
  SF_REQUIRE(res && out, "sf_gemv_pack_batch1: null pointer");
  SF_REQUIRE(b_r == 2 || b_r == 3, "sf_gemv_pack_batch1: b_r must be 2 or 3");
  SF_REQUIRE(N >= 1 && K >= 256 && K % 256 == 0, "sf_gemv_pack_batch1: need N >= 1 and K a positive multiple of 256");
  cudaStream_t s = sf::as_cuda(stream);
  const size_t words = static_cast<size_t>(N) * K / 32 * b_r;
  if (b_r == 2) {
    if (out != res) SF_CHECK_CUDA(cudaMemcpyAsync(out, res, words * 4, cudaMemcpyDeviceToDevice, s));
    return SF_OK;
  }
  SF_REQUIRE(out != res, "sf_gemv_pack_batch1: the 3-bit layout cannot be written in place");
  const long long n = static_cast<long long>(N) * (K / 256);
  const int threads = 128;
  pack_res3_kernel<<<static_cast<unsigned>((n + threads - 1) / threads), threads, 0, s>>>(res, N, K / 256, out);
  return sf::check_launch("pack_res3_kernel");
}

namespace {

// Clusters of two K halves that can be resident at once (cached per kernel
// and shared-memory size): the grid never holds more pairs than that, so no
// pair waits for a second wave.
int max_pairs(const void* kern, size_t smem, int block) {
  static std::mutex mu;
  static std::map<std::pair<const void*, size_t>, int> known;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(kern, smem);
  const auto it = known.find(key);
  if (it != known.end()) return it->second;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * sf::sm_count());
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = sf::sm_count() / 2;
  }
  known[key] = n;
  return n;
}

sf_status run_batch1(const char* what, const sf_gemv_job* jobs, int count, const uint16_t* x, const int32_t* idx,
                     const int32_t* n, const sf_gemv_producer* p, cudaStream_t s) {
  SF_REQUIRE(jobs, "%s: null pointer", what);
  SF_REQUIRE(count >= 1 && count <= kMaxJobs, "%s: count must be in [1, %d]", what, kMaxJobs);
  const sf_qweight* W0 = jobs[0].W;
  SF_REQUIRE(W0, "%s: null weight", what);
  const int K = W0->K, G = W0->G, b_f = W0->b_f, b_r = W0->b_r;
  SF_REQUIRE(b_r == 2 || b_r == 3, "%s: b_r must be 2 or 3", what);
  SF_REQUIRE(b_f == 1 || b_f == 2, "%s: b_f must be 1 or 2", what);
  SF_REQUIRE(b_r + b_f <= 4, "%s: b_r + b_f must be at most 4", what);
  SF_REQUIRE(G == 128, "%s: group size must be 128 (the prepared activations' group)", what);
  SF_REQUIRE(K >= 256 && K % 256 == 0, "%s: K must be a positive multiple of 256", what);
  int spw = 0, ksplit = 0;
  SF_REQUIRE(pick_split(K / 256, &spw, &ksplit),
             "%s: K/256 must split into at most 16 warps of 1 or 2 slices, in 1 or 2 halves", what);
  const int warps = K / 256 / (spw * ksplit);
  MArgs a{};
  a.njobs = count;
  a.K = K;
  a.ksplit = ksplit;
  a.prod.op = kProdNone;
  if (p == nullptr) {
    SF_REQUIRE(x, "%s: null pointer", what);
    SF_REQUIRE((idx == nullptr) == (n == nullptr), "%s: idx and n go together", what);
    SF_REQUIRE(sf::aligned(x, 16), "%s: x must be 16-byte aligned", what);
    a.x = x;
    a.idx = idx;
    a.n_sel = n;
  } else {
    SF_REQUIRE(p->op == SF_PRODUCE_NORM || p->op == SF_PRODUCE_ROUND || p->op == SF_PRODUCE_SILU_MUL,
               "%s: unknown producer op %d", what, p->op);
    SF_REQUIRE(p->x && p->y && p->idx && p->n, "%s: null producer pointer", what);
    SF_REQUIRE(p->op != SF_PRODUCE_NORM || p->w, "%s: SF_PRODUCE_NORM needs w", what);
    SF_REQUIRE(p->op != SF_PRODUCE_SILU_MUL || p->u, "%s: SF_PRODUCE_SILU_MUL needs u", what);
    SF_REQUIRE(p->op != SF_PRODUCE_NORM || p->eps >= 0.0f, "%s: eps must be >= 0", what);
    SF_REQUIRE(sf::aligned(p->y, 16), "%s: y must be 16-byte aligned", what);
    SF_REQUIRE(K <= sfd::kSelRowMaxK, "%s: K must be at most %d with a producer", what, sfd::kSelRowMaxK);
    // the selection list shares the last ring stage with the row and the histograms
    const size_t stage_words = static_cast<size_t>(warps) * (b_r == 2 ? (spw == 1 ? MCfg<1, 2>::SW : MCfg<2, 2>::SW)
                                                                      : (spw == 1 ? MCfg<1, 3>::SW : MCfg<2, 3>::SW));
    // histogram rows: one per warp while the list still fits, else shared
    int hrows = warps;
    auto cap = [&](int h) { return static_cast<long long>(stage_words) - prod_fixed_words(K, h); };
    while (hrows > 1 && cap(hrows) < p->k) hrows = (hrows + 1) / 2;
    SF_REQUIRE(p->k >= 0 && p->k <= K && p->k <= cap(hrows), "%s: k must be in [0, min(K, %lld)]", what,
               std::max(0LL, std::min(static_cast<long long>(K), cap(hrows))));
    a.prod.hrows = hrows;
    if (p->op == SF_PRODUCE_NORM && p->x_out) {
      auto overlaps = [&](const float* q) {
        return q != nullptr && p->x_out < q + K && q < p->x_out + K;
      };
      SF_REQUIRE(!overlaps(p->x) && !overlaps(p->delta), "%s: x_out must not overlap x or delta", what);
    }
    a.prod.op = p->op;
    a.prod.k = p->k;
    a.prod.eps = p->eps;
    a.prod.x = p->x;
    a.prod.delta = p->op == SF_PRODUCE_NORM ? p->delta : nullptr;
    a.prod.w = p->w;
    a.prod.u = p->u;
    a.prod.x_out = p->op == SF_PRODUCE_NORM ? p->x_out : nullptr;
    a.prod.y = p->y;
    a.prod.idx = p->idx;
    a.prod.n = p->n;
    a.x = p->y;
    a.idx = p->idx;
    a.n_sel = p->n;
  }
  int row_tiles = 0;
  for (int i = 0; i < count; ++i) {
    const sf_qweight* W = jobs[i].W;
    SF_REQUIRE(W && W->scale && W->zero && jobs[i].y, "%s: job %d incomplete", what, i);
    SF_REQUIRE(W->K == K && W->G == G && W->b_f == b_f && W->b_r == b_r,
               "%s: jobs must share K, G and bit widths", what);
    const uint32_t* res = jobs[i].res_b1 ? jobs[i].res_b1 : W->res;
    SF_REQUIRE(res, "%s: job %d has no resident codes", what, i);
    SF_REQUIRE(b_r == 2 || jobs[i].res_b1,
               "%s: 3-bit codes must be given in the batch-1 layout (res_b1, sf_gemv_pack_batch1)", what);
    SF_REQUIRE(W->N >= kRows && W->N % kRows == 0, "%s: N must be a multiple of %d", what, kRows);
    SF_REQUIRE(sf::aligned(res, 16) && sf::aligned(W->scale, 16) && sf::aligned(W->zero, 16),
               "%s: weight arrays must be 16-byte aligned", what);
    MJob& J = a.job[i];
    J.res = res;
    J.scale = W->scale;
    J.zero = W->zero;
    J.N = W->N;
    J.y = jobs[i].y;
    J.unit_words = W->N * b_f / 32;
    J.tile_begin = row_tiles;
    row_tiles += W->N / kRows;
    if (jobs[i].cache) {
      sf::CacheView v{};
      const bool deadline = sf::cache_deadline(jobs[i].cache);
      SF_REQUIRE(deadline || p == nullptr,
                 "%s: a producer needs caches in the deadline reading (a blocking prefetch needs the selection "
                 "before the launch)", what);
      const sf_status st = deadline ? sf::cache_view_for_reader(jobs[i].cache, s, &v)
                                    : sf::cache_view_for_gemv(jobs[i].cache, s, &v);
      if (st != SF_OK) return st;
      SF_REQUIRE(v.unit_words == J.unit_words, "%s: cache unit size does not match N*b_f/8", what);
      SF_REQUIRE(!deadline || v.num_units == K, "%s: a deadline cache must have K units", what);
      J.ref_rows = v.rows;
      J.row_of = deadline ? nullptr : v.row_of;
      J.unit_slot = deadline ? v.unit_slot : nullptr;
    } else if (jobs[i].use_ref_store) {
      SF_REQUIRE(W->ref, "%s: use_ref_store without W->ref", what);
      J.ref_rows = W->ref;
      J.row_of = nullptr;
    }
  }
  const int sms = sf::sm_count();
  auto launch = [&](auto kern, size_t smem) -> sf_status {
    SF_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
    // row blocks (pairs with two K halves) with work only: ceil(tiles / per)
    // blocks of per = ceil(tiles / cap) tiles, so no block idles and the SMs
    // left over stay free (for a producer that the launch overlaps)
    int cap = std::max(1, sms / ksplit);
    if (ksplit > 1) cap = std::max(1, std::min(cap, max_pairs(reinterpret_cast<const void*>(kern), smem, 32 * warps)));
    const int per = (row_tiles + cap - 1) / cap;
    const int nrow_cta = (row_tiles + per - 1) / per;
    // programmatic stream serialization: the CTAs may start streaming codes
    // while the previous kernel (typically the producer of x) runs
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(nrow_cta * ksplit);
    cfg.blockDim = dim3(32 * warps);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (g_gemv_overlap.load(std::memory_order_relaxed)) {
      attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[na].val.programmaticStreamSerializationAllowed = 1;
      ++na;
    }
    if (ksplit > 1) {  // the two K halves of a row block form a cluster
      attr[na].id = cudaLaunchAttributeClusterDimension;
      attr[na].val.clusterDim.x = 2;
      attr[na].val.clusterDim.y = 1;
      attr[na].val.clusterDim.z = 1;
      ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    SF_CHECK_CUDA(cudaLaunchKernelEx(&cfg, kern, a));
    return sf::check_launch("gemv_mma_kernel");
  };
  auto dispatch = [&](auto prod) -> sf_status {
    constexpr bool P = decltype(prod)::value;
    if (b_r == 2) {
      if (spw == 1) {
        const size_t smem = MCfg<1, 2>::smem_bytes(warps);
        return b_f == 2 ? launch(gemv_mma_kernel<1, 2, 2, P>, smem) : launch(gemv_mma_kernel<1, 1, 2, P>, smem);
      }
      const size_t smem = MCfg<2, 2>::smem_bytes(warps);
      return b_f == 2 ? launch(gemv_mma_kernel<2, 2, 2, P>, smem) : launch(gemv_mma_kernel<2, 1, 2, P>, smem);
    }
    // b_r == 3, b_f == 1
    return spw == 1 ? launch(gemv_mma_kernel<1, 1, 3, P>, MCfg<1, 3>::smem_bytes(warps))
                    : launch(gemv_mma_kernel<2, 1, 3, P>, MCfg<2, 3>::smem_bytes(warps));
  };
  const sf_status st = p != nullptr ? dispatch(std::true_type{}) : dispatch(std::false_type{});
  if (st != SF_OK) return st;
  for (int i = 0; i < count; ++i)
    if (jobs[i].cache) {
      const sf_status m = sf::cache_mark_used(jobs[i].cache, s);
      if (m != SF_OK) return m;
    }
  return SF_OK;
}

}  // namespace

extern "C" sf_status sf_gemv_refine_batch1(const sf_gemv_job* jobs, int count, const uint16_t* x, const int32_t* idx,
                                           const int32_t* n, sf_stream_t stream) {
  return run_batch1("sf_gemv_refine_batch1", jobs, count, x, idx, n, nullptr, sf::as_cuda(stream));
}

extern "C" sf_status sf_gemv_refine_batch1_produce(const sf_gemv_job* jobs, int count, const sf_gemv_producer* p,
                                                   sf_stream_t stream) {
  SF_REQUIRE(p, "sf_gemv_refine_batch1_produce: null producer");
  return run_batch1("sf_gemv_refine_batch1_produce", jobs, count, nullptr, nullptr, nullptr, p,
                    sf::as_cuda(stream));
}

extern "C" sf_status sf_gemv_set_launch_overlap(int on) {
  g_gemv_overlap.store(on != 0 ? 1 : 0, std::memory_order_relaxed);
  return SF_OK;
}
