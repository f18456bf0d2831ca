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
// Tiles are 16 output rows.  A warp owns SPW 256-channel slices of K for the
// whole kernel; their B fragments stay in registers.  Per tile and slice the
// 16 rows x 256 codes go through 8 mma.m16n8k32 (u8 codes x s8 digits, s32
// accumulate); a code word becomes four A-fragment bytes with one shift and
// one mask.  The two 128-channel groups of a slice accumulate into disjoint
// columns (three digit planes each), so after the 8 MMAs each pair of lanes
// holds the plane sums of two (row, group) pairs and one swap gives each
// lane one pair: it applies that pair's scale and zero point,
//   s (2^b_f fscale P + (m_f - z) gsum + sum_{j in S, j in group} x_j (q_f - m_f)),
// so the scale/zero arithmetic and the refinement correction are spread over
// all 32 lanes.  The warps of a CTA cover consecutive slices of one tile and
// add up in shared memory; with two K halves (ksplit = 2) the halves add
// their partial sums onto a zeroed output (two terms onto zero: the result
// does not depend on their order).
//
// Each warp streams its own codes, scale/zero and refinement words through a
// cp.async ring in shared memory; a warp waits only for its own copies.
#include <algorithm>

#include "act.cuh"
#include "sf_internal.h"

namespace {

constexpr int kMaxJobs = 4;
constexpr int kRows = 16;       // output rows per tile
constexpr int kCodeStr = 24;    // words per staged code row (16 used): conflict-free fragment loads
constexpr int kRefSlot = 16;    // refinement words staged per (slice, group) and tile
constexpr int kSelCap = 128;    // list capacity per (slice, group): the whole group
constexpr int kSzWords = 32;    // scale, zero of 2 groups x 16 rows (fp16)
constexpr int kSliceStage = kRows * kCodeStr + kSzWords + 2 * kRefSlot;  // words per slice and stage
constexpr int kMaxWarps = 16;

struct MJob {
  const uint32_t* res;
  const uint16_t* scale;
  const uint16_t* zero;
  const uint32_t* ref_rows;  // nullptr: resident only
  const int32_t* row_of;     // nullptr: refinement row = channel index
  float* y;
  int N, unit_words, tile_begin;
};

struct MArgs {
  MJob job[kMaxJobs];
  const uint16_t* x;
  const uint32_t* act;
  int njobs, K, b_f, ksplit;
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
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// fp16 bit pattern -> fp32 with integer/FP32 pipes only: move exponent and
// mantissa into place and rescale by 2^112, exact for every finite fp16
// including subnormals.
__device__ __forceinline__ float h2f_bits(uint32_t h) {
  return __uint_as_float((h & 0x7FFFu) << 13) * 5.192296858534828e+33f * ((h & 0x8000u) ? -1.0f : 1.0f);
}

// int -> fp32 for |v| < 2^22 with one integer add and one FP add: 1.5 * 2^23
// + v has v in its low mantissa bits.
__device__ __forceinline__ float i2f_small(int v) { return __int_as_float(0x4B400000 + v) - 12582912.0f; }

__device__ __forceinline__ int job_of(const MArgs& a, int t) {
  int jb = 0;
#pragma unroll
  for (int q = 1; q < kMaxJobs; ++q)
    if (q < a.njobs && t >= a.job[q].tile_begin) jb = q;
  return jb;
}

template <int SPW>
struct MCfg {
  static constexpr int kStages = SPW == 1 ? 4 : 3;
  static constexpr int SW = SPW * kSliceStage;  // ring words per warp and stage
  static size_t smem_bytes(int W) {
    return sizeof(uint32_t) * (static_cast<size_t>(W) * kStages * SW + 2 * static_cast<size_t>(W) * SPW * 2 * kSelCap +
                               static_cast<size_t>(W) * SPW * 2 * kRefSlot + 2 * static_cast<size_t>(W) * kRows);
  }
};

template <int SPW>
__global__ void __launch_bounds__(512, 1)
gemv_mma_kernel(const __grid_constant__ MArgs a) {
  using C = MCfg<SPW>;
  constexpr int kStages = C::kStages, SW = C::SW;
  extern __shared__ __align__(16) uint32_t sm[];
  const int W = blockDim.x >> 5;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g8 = lane >> 2, tig = lane & 3;
  const int ks = blockIdx.x % a.ksplit, crow = blockIdx.x / a.ksplit, ncta = gridDim.x / a.ksplit;
  uint32_t* ring = sm + warp * kStages * SW;
  uint32_t* after_ring = sm + W * kStages * SW;
  float* selx = reinterpret_cast<float*>(after_ring) + warp * SPW * 2 * kSelCap;      // [SPW][2][kSelCap]
  int* selp = reinterpret_cast<int*>(after_ring + W * SPW * 2 * kSelCap) + warp * SPW * 2 * kSelCap;
  int* selr = reinterpret_cast<int*>(after_ring + 2 * W * SPW * 2 * kSelCap) + warp * SPW * 2 * kRefSlot;
  float* red = reinterpret_cast<float*>(after_ring + 2 * W * SPW * 2 * kSelCap + W * SPW * 2 * kRefSlot);  // [2][W][16]

  const int slice0 = (ks * W + warp) * SPW;
  const int myslot = tig >> 1, myrow = g8 + 8 * (tig & 1);
  const bool even = (tig & 1) == 0;

  // ---- per-warp setup: B fragments, group scalars, selection lists
  uint32_t bf[SPW][8][2];
  float fsc[SPW], gsm[SPW];
  int ns[SPW][2];
#pragma unroll
  for (int sp = 0; sp < SPW; ++sp) {
    const uint32_t* A = a.act + static_cast<size_t>(slice0 + sp) * sfd::kAct2Words;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const uint2 v = reinterpret_cast<const uint2*>(A)[m * 32 + lane];
      bf[sp][m][0] = v.x;
      bf[sp][m][1] = v.y;
    }
    fsc[sp] = __uint_as_float(A[sfd::kAct2Info + 2 * myslot]);
    gsm[sp] = __uint_as_float(A[sfd::kAct2Info + 2 * myslot + 1]);
    const int prefix = static_cast<int>(A[sfd::kAct2Info + 4]);
    // lanes 0..7 own one mask word each (32 channels); words 0..3 = group 0
    const uint32_t mw = lane < 8 ? A[sfd::kAct2Mask + lane] : 0u;
    const int c = __popc(mw);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int n0 = __shfl_sync(0xffffffffu, incl, 3);
    const int nall = __shfl_sync(0xffffffffu, incl, 7);
    ns[sp][0] = n0;
    ns[sp][1] = nall - n0;
    if (lane < 8) {
      const int slot = lane >> 2;
      int r = incl - c - (slot ? n0 : 0);  // rank inside the group's list
      int p = prefix + incl - c;           // position in the selection (idx order)
      uint32_t mm = mw;
      while (mm) {
        const int bit = __ffs(mm) - 1;
        mm &= mm - 1u;
        const int ch = 32 * lane + bit;  // channel inside the slice
        const int e = (sp * 2 + slot) * kSelCap + r;
        selx[e] = sfd::bf16_bits_to_float(a.x[256 * (slice0 + sp) + ch]);
        selp[e] = (p << 8) | ch;
        ++r;
        ++p;
      }
    }
  }
  __syncwarp();

  const float m_f = static_cast<float>((1 << a.b_f) - 1) * 0.5f;
  const float two_bf = static_cast<float>(1 << a.b_f);
  const uint32_t fmask = (1u << a.b_f) - 1u;
  const size_t row_words = static_cast<size_t>(a.K) / 16;
  const int last = a.njobs - 1;
  const int total_tiles = a.job[last].tile_begin + a.job[last].N / kRows;
  const int my_tiles = crow < total_tiles ? (total_tiles - crow + ncta - 1) / ncta : 0;
  int issue_job = -1;

  auto issue = [&](int i) {
    const int st = i % kStages;
    const int t = crow + i * ncta;
    const int jb = job_of(a, t);
    const MJob& J = a.job[jb];
    const int row0 = (t - J.tile_begin) * kRows;
    if (jb != issue_job) {  // refinement rows of the staged list entries, for this matrix
      issue_job = jb;
      if (J.ref_rows) {
#pragma unroll
        for (int sp = 0; sp < SPW; ++sp)
#pragma unroll
          for (int slot = 0; slot < 2; ++slot)
            if (lane < kRefSlot && lane < ns[sp][slot]) {
              const int pc = selp[(sp * 2 + slot) * kSelCap + lane];
              selr[(sp * 2 + slot) * kRefSlot + lane] =
                  J.row_of ? J.row_of[pc >> 8] : 256 * (slice0 + sp) + (pc & 255);
            }
      }
      __syncwarp();
    }
#pragma unroll
    for (int sp = 0; sp < SPW; ++sp) {
      uint32_t* base = ring + st * SW + sp * kSliceStage;
      const int slice = slice0 + sp;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = (lane >> 2) + 8 * h;
        cp_async16(base + row * kCodeStr + 4 * (lane & 3),
                   J.res + static_cast<size_t>(row0 + row) * row_words + 16 * slice + 4 * (lane & 3));
      }
      if (lane < 8) {  // (group, scale|zero, half of the 16 rows)
        const int grp = lane >> 2, arr = (lane >> 1) & 1, hf = lane & 1;
        const uint16_t* src = (arr ? J.zero : J.scale) + static_cast<size_t>(2 * slice + grp) * J.N + row0 + 8 * hf;
        cp_async16(reinterpret_cast<uint16_t*>(base + kRows * kCodeStr) + (grp * 2 + arr) * 16 + 8 * hf, src);
      }
      if (J.ref_rows) {
        const int slot = lane >> 4, q = lane & (kRefSlot - 1);
        const int n = slot ? ns[sp][1] : ns[sp][0];
        if (q < n)
          cp_async4(base + kRows * kCodeStr + kSzWords + lane,
                    J.ref_rows + static_cast<size_t>(selr[(sp * 2 + slot) * kRefSlot + q]) * J.unit_words +
                        ((row0 * a.b_f) >> 5));
      }
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
    const int jb = job_of(a, t);
    const MJob& J = a.job[jb];
    const int row0 = (t - J.tile_begin) * kRows;
    const int sh = ((row0 * a.b_f) & 31) + a.b_f * myrow;  // this lane's row in a refinement word
    float v = 0.0f;
#pragma unroll
    for (int sp = 0; sp < SPW; ++sp) {
      const uint32_t* base = ring + st * SW + sp * kSliceStage;
      // code words: rows g8 and g8 + 8, words 2 tig, 2 tig + 1 of each group
      const uint2 r0a = *reinterpret_cast<const uint2*>(base + g8 * kCodeStr + 2 * tig);
      const uint2 r0b = *reinterpret_cast<const uint2*>(base + g8 * kCodeStr + 8 + 2 * tig);
      const uint2 r1a = *reinterpret_cast<const uint2*>(base + (g8 + 8) * kCodeStr + 2 * tig);
      const uint2 r1b = *reinterpret_cast<const uint2*>(base + (g8 + 8) * kCodeStr + 8 + 2 * tig);
      // two independent accumulator chains (even / odd k-steps), added at the end
      int d[4] = {0, 0, 0, 0}, e[4] = {0, 0, 0, 0};
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int slot = m >> 2, hi = (m >> 1) & 1, j = 2 * (m & 1);
        const uint32_t w0 = slot ? (hi ? r0b.y : r0b.x) : (hi ? r0a.y : r0a.x);
        const uint32_t w1 = slot ? (hi ? r1b.y : r1b.x) : (hi ? r1a.y : r1a.x);
        const uint32_t a0 = (w0 >> (2 * j)) & 0x03030303u;
        const uint32_t a1 = (w1 >> (2 * j)) & 0x03030303u;
        const uint32_t a2 = (w0 >> (2 * j + 2)) & 0x03030303u;
        const uint32_t a3 = (w1 >> (2 * j + 2)) & 0x03030303u;
        if (m & 1) mma_u8s8(e, a0, a1, a2, a3, bf[sp][m][0], bf[sp][m][1]);
        else mma_u8s8(d, a0, a1, a2, a3, bf[sp][m][0], bf[sp][m][1]);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) d[c] += e[c];
      // even lanes: d0, d1 = planes 0, 1 of row g8 and d2, d3 = planes 0, 1 of
      // row g8 + 8; odd lanes: d0, d2 = plane 2 of rows g8, g8 + 8.  Plane sums
      // are below 2^17 in magnitude: exact small-integer conversions.
      const float f0 = i2f_small(d[0]), f1 = i2f_small(d[1]), f2 = i2f_small(d[2]), f3 = i2f_small(d[3]);
      const float send = even ? fmaf(f3, 256.0f, f2) : 65536.0f * f0;
      const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
      const float P = even ? fmaf(f1, 256.0f, f0) + recv : fmaf(65536.0f, f2, recv);
      const uint16_t* szs = reinterpret_cast<const uint16_t*>(base + kRows * kCodeStr);
      const float sc = h2f_bits(szs[(myslot * 2) * 16 + myrow]);
      const float zz = h2f_bits(szs[(myslot * 2 + 1) * 16 + myrow]);
      float tsum = fmaf(two_bf * fsc[sp], P, (m_f - zz) * gsm[sp]);
      if (J.ref_rows) {
        // sum_j x_j (q_f - m_f) over the group's selected channels: the staged
        // entries two at a time (a missing second entry has x = 0 and reads a
        // staged word that is never used), the rest from the refinement rows
        const int n = myslot ? ns[sp][1] : ns[sp][0];
        const int nst = min(max(ns[sp][0], ns[sp][1]), kRefSlot);
        const float* lx = selx + (sp * 2 + myslot) * kSelCap;
        const uint32_t* rw = base + kRows * kCodeStr + kSzWords + myslot * kRefSlot;
        float c0 = 0.0f, c1 = 0.0f;
        for (int q = 0; q < nst; q += 2) {
          const float x0 = q < n ? lx[q] : 0.0f, x1 = q + 1 < n ? lx[q + 1] : 0.0f;
          const uint32_t w0 = rw[q], w1 = rw[q + 1];
          c0 = fmaf(x0, i2f_small(static_cast<int>((w0 >> sh) & fmask)) - m_f, c0);
          c1 = fmaf(x1, i2f_small(static_cast<int>((w1 >> sh) & fmask)) - m_f, c1);
        }
        tsum += c0 + c1;
        for (int q = kRefSlot; q < n; ++q) {  // beyond the staged entries (rare)
          const int pc = selp[(sp * 2 + myslot) * kSelCap + q];
          const int rid = J.row_of ? J.row_of[pc >> 8] : 256 * (slice0 + sp) + (pc & 255);
          const uint32_t word = J.ref_rows[static_cast<size_t>(rid) * J.unit_words + ((row0 * a.b_f) >> 5)];
          tsum = fmaf(lx[q], i2f_small(static_cast<int>((word >> sh) & fmask)) - m_f, tsum);
        }
      }
      v = fmaf(sc, tsum, v);
    }
    // lanes tig and tig ^ 2 hold the same row for the two groups
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    float* rb = red + (i & 1) * W * kRows;
    if (tig < 2) rb[warp * kRows + myrow] = v;
    __syncthreads();
    if (tid < kRows) {
      float acc = 0.0f;
      for (int w = 0; w < W; ++w) acc += rb[w * kRows + tid];
      float* dst = J.y + row0 + tid;
      if (a.ksplit > 1) atomicAdd(dst, acc);
      else *dst = acc;
    }
  }
  cp_async_wait<0>();
}

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
  SF_REQUIRE(G == 128, "sf_gemv_refine_batch1: group size must be 128 (the prepared activations' group)");
  SF_REQUIRE(K >= 256 && K % 256 == 0, "sf_gemv_refine_batch1: K must be a positive multiple of 256");
  int spw = 0, ksplit = 0;
  SF_REQUIRE(pick_split(K / 256, &spw, &ksplit),
             "sf_gemv_refine_batch1: K/256 must split into at most 16 warps of 1 or 2 slices, in 1 or 2 halves");
  cudaStream_t s = sf::as_cuda(stream);
  MArgs a{};
  a.njobs = count;
  a.K = K;
  a.b_f = b_f;
  a.ksplit = ksplit;
  a.x = x;
  a.act = static_cast<const uint32_t*>(act);
  int row_tiles = 0;
  for (int i = 0; i < count; ++i) {
    const sf_qweight* W = jobs[i].W;
    SF_REQUIRE(W && W->res && W->scale && W->zero && jobs[i].y, "sf_gemv_refine_batch1: job %d incomplete", i);
    SF_REQUIRE(W->K == K && W->G == G && W->b_f == b_f && W->b_r == 2,
               "sf_gemv_refine_batch1: jobs must share K, G and bit widths");
    SF_REQUIRE(W->N >= kRows && W->N % kRows == 0, "sf_gemv_refine_batch1: N must be a multiple of %d", kRows);
    SF_REQUIRE(sf::aligned(W->res, 16) && sf::aligned(W->scale, 16) && sf::aligned(W->zero, 16),
               "sf_gemv_refine_batch1: weight arrays must be 16-byte aligned");
    MJob& J = a.job[i];
    J.res = W->res;
    J.scale = W->scale;
    J.zero = W->zero;
    J.N = W->N;
    J.y = jobs[i].y;
    J.unit_words = W->N * b_f / 32;
    J.tile_begin = row_tiles;
    row_tiles += W->N / kRows;
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
  const int warps = K / 256 / (spw * ksplit);
  const int threads = 32 * warps;
  const int sms = sf::sm_count();
  const int nrow_cta = std::max(1, std::min(row_tiles, std::max(1, sms / ksplit)));
  sf_status st = SF_OK;
  if (spw == 1) {
    const size_t smem = MCfg<1>::smem_bytes(warps);
    SF_CHECK_CUDA(cudaFuncSetAttribute(gemv_mma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)));
    gemv_mma_kernel<1><<<nrow_cta * ksplit, threads, smem, s>>>(a);
    st = sf::check_launch("gemv_mma_kernel");
  } else {
    const size_t smem = MCfg<2>::smem_bytes(warps);
    SF_CHECK_CUDA(cudaFuncSetAttribute(gemv_mma_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)));
    gemv_mma_kernel<2><<<nrow_cta * ksplit, threads, smem, s>>>(a);
    st = sf::check_launch("gemv_mma_kernel");
  }
  if (st != SF_OK) return st;
  for (int i = 0; i < count; ++i)
    if (jobs[i].cache) {
      const sf_status m = sf::cache_mark_used(jobs[i].cache, s);
      if (m != SF_OK) return m;
    }
  return SF_OK;
}
