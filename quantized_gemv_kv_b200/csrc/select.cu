// sf_select_topk: top-k input channels by |x| per batch row, union over rows.
//
// |x| of a bf16 value is its 15 low bits read as an unsigned integer (sign
// dropped, so +0 and -0 tie and larger magnitudes give larger keys), which
// makes the selection exact integer work.  One CTA of 1024 threads; each of
// the B rows owns a contiguous slice of the threads and all rows advance
// together through a two-pass radix select (8 high bits, then 7 low bits)
// that finds the k-th largest key tau.  Keys above tau are taken; keys equal
// to tau are taken in ascending channel order until k are chosen (an ordered
// scan), which is the "ties to the lower index" rule.  A final ordered
// compaction writes the union in ascending order.
#include <cooperative_groups.h>

#include "act.cuh"
#include "block_scan.cuh"
#include "select_row.cuh"
#include "sf_internal.h"

namespace {

constexpr int kThreads = 1024;
constexpr int kMaxRows = 16;
constexpr int kActMaxK = 32768;
constexpr int kActMaxGroups = kActMaxK / 128;

// Histogram increment with the lanes of a warp that hit the same bin merged
// into one atomic (keys cluster in few bins, so plain atomics serialise).
// bin < 0 means "no increment".  Call with the whole warp.
__device__ __forceinline__ void warp_hist_add(int* hist, int bin) {
  const unsigned peers = __match_any_sync(0xffffffffu, bin);
  const int leader = __ffs(peers) - 1;
  if (bin >= 0 && (threadIdx.x & 31) == leader) atomicAdd(&hist[bin], __popc(peers));
}

struct RowState {
  int b1, k1;      // high-byte bin of the k-th key, rank left inside it
  int tau, r;      // k-th largest key, how many keys equal to tau to take
};

__global__ void __launch_bounds__(kThreads)
select_topk_kernel(const uint16_t* __restrict__ x, int B, int K, int k, int32_t* __restrict__ idx_out,
                   int32_t* __restrict__ n_out, uint32_t* __restrict__ act) {
  extern __shared__ uint8_t smem[];
  uint8_t* flags = smem;                                                   // [K]
  int* hist1 = reinterpret_cast<int*>(smem + ((K + 15) & ~15));           // [kMaxRows][256]
  int* hist2 = hist1 + kMaxRows * 256;                                     // [kMaxRows][128]
  __shared__ RowState st[kMaxRows];
  __shared__ int scan_scratch[33];
  __shared__ int bad;
  __shared__ int eg[kActMaxGroups];
  __shared__ float ginfo[2 * kActMaxGroups];

  const int tid = threadIdx.x;
  int rb = 1;
  while (rb < B) rb <<= 1;
  const int tpr = kThreads / rb;  // threads per row
  const int row = tid / tpr, lid = tid % tpr;
  const bool active = row < B;
  const uint16_t* xr = x + static_cast<size_t>(row) * K;

  for (int j = tid; j < K; j += kThreads) flags[j] = 0;
  for (int j = tid; j < kMaxRows * 256; j += kThreads) hist1[j] = 0;
  for (int j = tid; j < kMaxRows * 128; j += kThreads) hist2[j] = 0;
  if (tid == 0) bad = 0;
  __syncthreads();

  // pass 1: histogram of the high 8 bits of the 15-bit magnitude key
  if (active) {
    int* h = hist1 + row * 256;
    // trip count is uniform across a warp (tpr is a multiple of 32), so the
    // whole warp takes part in each aggregation round
    for (int j0 = lid - (lid & 31); j0 < K; j0 += tpr) {
      const int j = j0 + (lid & 31);
      const bool in = j < K;
      const uint32_t v = in ? xr[j] : 0u;
      if (in && (v & 0x7F80u) == 0x7F80u) bad = 1;  // Inf or NaN
      warp_hist_add(h, in ? static_cast<int>((v & 0x7FFFu) >> 7) : -1);
    }
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  if (warp < B) {
    // find the bin holding the k-th largest key: scan bins from the top
    const int* h = hist1 + warp * 256;
    int above = 0, b1 = -1, k1 = 0;
    for (int base = 255; base >= 0 && b1 < 0; base -= 32) {
      const int bin = base - lane;
      const int c = h[bin];
      int incl = c;  // inclusive prefix from the top within this chunk
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const bool hit = (above + incl >= k) && (above + incl - c < k);
      const unsigned m = __ballot_sync(0xffffffffu, hit && k > 0);
      if (m) {
        const int src = __ffs(m) - 1;
        b1 = base - src;
        k1 = k - (above + __shfl_sync(0xffffffffu, incl - c, src));
      }
      above += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) { st[warp].b1 = b1; st[warp].k1 = k1; }
  }
  __syncthreads();
  // pass 2: histogram of the low 7 bits inside that bin
  if (active && st[row].b1 >= 0) {
    int* h = hist2 + row * 128;
    const int b1 = st[row].b1;
    for (int j0 = lid - (lid & 31); j0 < K; j0 += tpr) {
      const int j = j0 + (lid & 31);
      const uint32_t v = j < K ? (xr[j] & 0x7FFFu) : 0xFFFFu;
      warp_hist_add(h, (j < K && static_cast<int>(v >> 7) == b1) ? static_cast<int>(v & 0x7Fu) : -1);
    }
  }
  __syncthreads();
  if (warp < B) {
    const int* h = hist2 + warp * 128;
    const int b1 = st[warp].b1, kk = st[warp].k1;
    int above = 0, tau = -1, r = 0;
    if (b1 >= 0) {
      for (int base = 127; base >= 0 && tau < 0; base -= 32) {
        const int bin = base - lane;
        const int c = h[bin];
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const bool hit = (above + incl >= kk) && (above + incl - c < kk);
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
          const int src = __ffs(m) - 1;
          tau = (b1 << 7) | (base - src);
          r = kk - (above + __shfl_sync(0xffffffffu, incl - c, src));
        }
        above += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    if (lane == 0) { st[warp].tau = tau; st[warp].r = r; }
  }
  __syncthreads();

  // ordered pass: keys > tau always; keys == tau for the first r in index order
  {
    const int chunk = (K + tpr - 1) / tpr;
    const int j0 = min(K, lid * chunk), j1 = min(K, j0 + chunk);
    const int tau = active ? st[row].tau : -1;
    int eq = 0;
    if (active && tau >= 0)
      for (int j = j0; j < j1; ++j) eq += ((xr[j] & 0x7FFF) == tau);
    int total;
    const int pre = sfd::block_exclusive_scan(eq, scan_scratch, &total);
    // the row's threads are contiguous: subtract the prefix at its first thread
    __shared__ int row_base[kMaxRows];
    if (lid == 0 && active) row_base[row] = pre;
    __syncthreads();
    if (active && tau >= 0) {
      int rank = pre - row_base[row];
      const int r = st[row].r;
      for (int j = j0; j < j1; ++j) {
        const int key = xr[j] & 0x7FFF;
        if (key > tau) {
          flags[j] = 1;
        } else if (key == tau) {
          if (rank < r) flags[j] = 1;
          ++rank;
        }
      }
    }
  }
  __syncthreads();

  // ordered compaction of the union
  {
    const int chunk = (K + kThreads - 1) / kThreads;
    const int j0 = min(K, tid * chunk), j1 = min(K, j0 + chunk);
    int c = 0;
    for (int j = j0; j < j1; ++j) c += flags[j];
    int total;
    int pos = sfd::block_exclusive_scan(c, scan_scratch, &total);
    for (int j = j0; j < j1; ++j)
      if (flags[j]) idx_out[pos++] = j;
    if (tid == 0) *n_out = bad ? -1 : total;
  }

  // prepared activations (batch 1): digit planes as MMA fragments, group
  // scalars, the selection mask and counts (act.cuh)
  if (act != nullptr) {
    __syncthreads();
    sfd::act2_write_block(x, flags, K, eg, ginfo, scan_scratch, act);
  }
}

__global__ void __launch_bounds__(kThreads)
act_prepare_kernel(const uint16_t* __restrict__ x, int K, uint32_t* __restrict__ act) {
  __shared__ int eg[kActMaxGroups];
  __shared__ float ginfo[2 * kActMaxGroups];
  __shared__ int scan_scratch[33];
  sfd::act2_write_block(x, nullptr, K, eg, ginfo, scan_scratch, act);
}

// ---- several single-row selections in one launch (one CTA each) -------------
// The row is read once into shared memory; the histograms, the ordered
// tie pass, the compaction and the prepared activations all work from there.
constexpr int kMaxSelJobs = 8;
struct SelJobDev {
  const uint16_t* x;
  int K, k;
  int32_t* idx;
  int32_t* n;
  uint32_t* act;
};
struct SelManyArgs {
  SelJobDev job[kMaxSelJobs];
};

__global__ void __launch_bounds__(kThreads)
select_act_many_kernel(const __grid_constant__ SelManyArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const SelJobDev& J = a.job[blockIdx.x];
  const int K = J.K, tid = threadIdx.x;
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);  // [K]
  uint8_t* flags = smem + 2 * K;                     // [K]
  {
    const uint4* src = reinterpret_cast<const uint4*>(J.x);
    uint4* dst = reinterpret_cast<uint4*>(xs);
    for (int i = tid; i < K / 8; i += kThreads) dst[i] = src[i];
  }
  __syncthreads();
  sfd::select_row_block(xs, flags, K, J.k, J.idx, J.n, J.act);
}
// ---- random selection (the comparator of the explainer's 既存手法との違い) -----
// key_j = (splitmix64(seed + K step + j) >> 49) mod 32640 (Steele, Lea and
// Flood's finalizer: a counter-based generator, so every channel's key is
// drawn on its own), read as a finite positive bf16 magnitude; the k largest
// keys (ties to the lower channel) are the selection.
__device__ __forceinline__ uint64_t splitmix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void __launch_bounds__(kThreads)
select_random_kernel(int K, int k, uint64_t seed, uint64_t step, int32_t* __restrict__ idx, int32_t* __restrict__ n) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);  // [K], padded to sel_row_bytes(K)
  uint8_t* flags = smem + sfd::sel_row_bytes(K);     // [K]
  const uint64_t base = seed + static_cast<uint64_t>(K) * step;
  for (int j = threadIdx.x; j < K; j += kThreads)
    xs[j] = static_cast<uint16_t>((splitmix64(base + static_cast<uint64_t>(j)) >> 49) % 0x7F80u);
  __syncthreads();
  sfd::select_row_block(xs, flags, K, k, idx, n, nullptr);
}

// ---- the union over a batch, one CTA per row in one thread-block cluster ---
//
// CTA b selects row b's top k (select_row_block, its list in idx_out's row b
// as scratch) and marks them in the union bitmask held in rank 0's shared
// memory (distributed-shared-memory atomics); rank 0 then lists the union in
// ascending order into idx_out (the rows' scratch lists are read before).
constexpr int kUnionMaxWords = kActMaxK / 32;

__global__ void __launch_bounds__(kThreads)
select_union_cluster_kernel(const uint16_t* __restrict__ x, int K, int k, int32_t* __restrict__ idx_out,
                            int32_t* __restrict__ n_out) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);  // [K], padded to sel_row_bytes(K)
  uint8_t* flags = smem + sfd::sel_row_bytes(K);     // [K]
  __shared__ uint32_t mask[kUnionMaxWords];          // rank 0's: the union
  __shared__ int nrow, bad_any, scan_scratch[33];
  const int b = static_cast<int>(cl.block_rank()), tid = threadIdx.x;
  const int nw = (K + 31) >> 5;
  if (b == 0) {
    for (int w = tid; w < nw; w += kThreads) mask[w] = 0u;
    if (tid == 0) bad_any = 0;
  }
  const uint16_t* xr = x + static_cast<size_t>(b) * K;
  for (int j = tid; j < K; j += kThreads) xs[j] = xr[j];
  __syncthreads();
  int32_t* mine = idx_out + static_cast<size_t>(b) * k;
  sfd::select_row_block(xs, flags, K, k, mine, &nrow, nullptr);
  __syncthreads();  // this row's list (global) and count are complete
  cl.sync();        // rank 0's bitmask is cleared
  uint32_t* m0 = cl.map_shared_rank(mask, 0);
  const int nr = nrow;
  if (nr < 0) {
    if (tid == 0) atomicOr(cl.map_shared_rank(&bad_any, 0), 1);
  } else {
    for (int e = tid; e < nr; e += kThreads) {
      const int j = mine[e];
      atomicOr(m0 + (j >> 5), 1u << (j & 31));
    }
  }
  cl.sync();  // the union is complete; every row's scratch list has been read
  if (b != 0) return;
  const int per = (nw + kThreads - 1) / kThreads;
  const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
  int c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(mask[w]);
  int total;
  int pos = sfd::block_exclusive_scan(c, scan_scratch, &total);
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = mask[w];
    while (bits) {
      const int bi = __ffs(bits) - 1;
      bits &= bits - 1u;
      idx_out[pos++] = 32 * w + bi;
    }
  }
  if (tid == 0) *n_out = bad_any ? -1 : total;
}

}  // namespace

extern "C" sf_status sf_select_random(int K, int k, uint64_t seed, uint64_t step, int32_t* idx_out, int32_t* n_out,
                                      sf_stream_t stream) {
  SF_REQUIRE(idx_out && n_out, "sf_select_random: null pointer");
  SF_REQUIRE(K >= 1 && K <= 32768 && k >= 0 && k <= K, "sf_select_random: need 1 <= K <= 32768, 0 <= k <= K");
  const size_t smem = sfd::sel_row_bytes(K) + static_cast<size_t>(K);
  SF_CHECK_CUDA(cudaFuncSetAttribute(select_random_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)));
  select_random_kernel<<<1, kThreads, smem, sf::as_cuda(stream)>>>(K, k, seed, step, idx_out, n_out);
  return sf::check_launch("select_random_kernel");
}

extern "C" sf_status sf_select_topk(const uint16_t* x, int B, int K, int k, int32_t* idx_out, int32_t* n_out,
                                    sf_stream_t stream) {
  SF_REQUIRE(x && idx_out && n_out, "sf_select_topk: null pointer");
  SF_REQUIRE(B >= 1 && B <= kMaxRows, "sf_select_topk: B must be in [1, %d]", kMaxRows);
  SF_REQUIRE(K >= 1 && K <= 65536, "sf_select_topk: K must be in [1, 65536]");
  SF_REQUIRE(k >= 0 && k <= K, "sf_select_topk: k must be in [0, K]");
  if (B >= 2 && K <= kActMaxK && k >= 1) {
    // one CTA per row, the union through a thread-block cluster
    const size_t smem = sfd::sel_row_bytes(K) + static_cast<size_t>(K);
    SF_CHECK_CUDA(cudaFuncSetAttribute(select_union_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)));
    SF_CHECK_CUDA(cudaFuncSetAttribute(select_union_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(B));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = sf::as_cuda(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(B);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    SF_CHECK_CUDA(cudaLaunchKernelEx(&cfg, select_union_cluster_kernel, x, K, k, idx_out, n_out));
    return sf::check_launch("select_union_cluster_kernel");
  }
  const size_t smem = static_cast<size_t>((K + 15) & ~15) + sizeof(int) * kMaxRows * (256 + 128);
  SF_CHECK_CUDA(cudaFuncSetAttribute(select_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024));
  select_topk_kernel<<<1, kThreads, smem, sf::as_cuda(stream)>>>(x, B, K, k, idx_out, n_out, nullptr);
  return sf::check_launch("select_topk_kernel");
}

extern "C" size_t sf_act_bytes(int K) {
  return (K > 0 && K % 256 == 0) ? static_cast<size_t>(K / 256) * sfd::kAct2Words * sizeof(uint32_t) : 0;
}

extern "C" sf_status sf_select_topk_act(const uint16_t* x, int K, int k, int32_t* idx_out, int32_t* n_out, void* act,
                                        sf_stream_t stream) {
  SF_REQUIRE(x && idx_out && n_out && act, "sf_select_topk_act: null pointer");
  SF_REQUIRE(K >= 256 && K <= kActMaxK && K % 256 == 0,
             "sf_select_topk_act: K must be a multiple of 256 in [256, %d]", kActMaxK);
  SF_REQUIRE(k >= 0 && k <= K, "sf_select_topk_act: k must be in [0, K]");
  SF_REQUIRE(sf::aligned(act, 16), "sf_select_topk_act: act must be 16-byte aligned");
  const size_t smem = static_cast<size_t>((K + 15) & ~15) + sizeof(int) * kMaxRows * (256 + 128);
  SF_CHECK_CUDA(cudaFuncSetAttribute(select_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024));
  select_topk_kernel<<<1, kThreads, smem, sf::as_cuda(stream)>>>(x, 1, K, k, idx_out, n_out,
                                                                 static_cast<uint32_t*>(act));
  return sf::check_launch("select_topk_kernel");
}

extern "C" sf_status sf_act_prepare(const uint16_t* x, int K, void* act, sf_stream_t stream) {
  SF_REQUIRE(x && act, "sf_act_prepare: null pointer");
  SF_REQUIRE(K >= 256 && K <= kActMaxK && K % 256 == 0,
             "sf_act_prepare: K must be a multiple of 256 in [256, %d]", kActMaxK);
  SF_REQUIRE(sf::aligned(act, 16), "sf_act_prepare: act must be 16-byte aligned");
  act_prepare_kernel<<<1, kThreads, 0, sf::as_cuda(stream)>>>(x, K, static_cast<uint32_t*>(act));
  return sf::check_launch("act_prepare_kernel");
}

extern "C" sf_status sf_select_topk_act_many(const sf_select_job* jobs, int count, sf_stream_t stream) {
  SF_REQUIRE(jobs, "sf_select_topk_act_many: null pointer");
  SF_REQUIRE(count >= 1 && count <= kMaxSelJobs, "sf_select_topk_act_many: count must be in [1, %d]", kMaxSelJobs);
  SelManyArgs a{};
  int kmax = 0;
  for (int i = 0; i < count; ++i) {
    const sf_select_job& j = jobs[i];
    SF_REQUIRE(j.x && j.idx_out && j.n_out, "sf_select_topk_act_many: job %d has a null pointer", i);
    SF_REQUIRE(j.K >= 32 && j.K <= 32768 && j.K % 32 == 0,
               "sf_select_topk_act_many: K must be a multiple of 32 in [32, 32768] (job %d)", i);
    SF_REQUIRE(j.k >= 0 && j.k <= j.K, "sf_select_topk_act_many: k out of range (job %d)", i);
    SF_REQUIRE(j.act == nullptr || j.K % 256 == 0,
               "sf_select_topk_act_many: prepared activations need K a multiple of 256 (job %d)", i);
    SF_REQUIRE(sf::aligned(j.x, 16) && (j.act == nullptr || sf::aligned(j.act, 16)),
               "sf_select_topk_act_many: x and act must be 16-byte aligned (job %d)", i);
    a.job[i] = SelJobDev{j.x, j.K, j.k, j.idx_out, j.n_out, static_cast<uint32_t*>(j.act)};
    kmax = j.K > kmax ? j.K : kmax;
  }
  const size_t smem = static_cast<size_t>(kmax) * 3;
  SF_CHECK_CUDA(cudaFuncSetAttribute(select_act_many_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)));
  select_act_many_kernel<<<count, kThreads, smem, sf::as_cuda(stream)>>>(a);
  return sf::check_launch("select_act_many_kernel");
}
