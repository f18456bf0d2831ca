// Refinement cache: an LRU set of refinement units (weight columns) kept in
// device memory and refilled from a host-resident master copy.
//
// StrataFlux reuses fetched precision across decode steps and hides transfer
// behind compute (arXiv 2611.08363 abstract; rag-lover.com explainer, 解説:
// fetch lead and caching).  Everything that decides hits, misses, slots and
// the LRU order runs on the device in one CTA (no host round trip), so a
// step can be enqueued ahead of time and captured in a CUDA graph.  Misses
// are copied by a gather kernel that reads the page-locked, device-mapped
// host master directly over the host link, on a side stream.
//
// LRU bookkeeping: `order` lists the cached units from least to most
// recently used, ties (units touched in the same step) in ascending unit
// order.  A step removes the hits from it, takes victims from its front,
// and appends the units touched this step (hits and inserted misses) in
// ascending order -- which keeps it sorted by (last use, unit) without
// storing the last-use stamps.  Slots are never freed except by reset, so
// the free slots are always the suffix [occupied, capacity).
#include <algorithm>
#include <cstring>
#include <vector>

#include "block_scan.cuh"
#include "sf_internal.h"

namespace {

constexpr int kIndexThreads = 1024;
constexpr int kGatherThreads = 128;

enum Meta { kOcc = 0, kStep, kHits, kMisses, kBypass, kGather, kMetaCount };
enum Stat { kStSteps = 0, kStHits, kStMisses, kStBypass, kStBytes, kStLate, kStatCount };

// Largest capacity: the index step keeps one byte per slot in shared memory.
constexpr int kMaxCapacity = 196608;

// Everything one cache step touches on the device.
struct CacheDev {
  const int32_t* S;      // selection (ascending units)
  const int32_t* n_ptr;  // its length
  int max_select, capacity;
  int budget;            // misses fetched per step at most (the rest are late)
  int slot_base;         // global slot number of this LRU's slot 0 (parts: p * capacity)
  int bypass_base;       // global row of this LRU's first bypass row
  int unit_lo, unit_hi;  // a part's unit range: its selection is the sub-range of S in it (unit_lo < 0: all of S)
  int64_t unit_bytes;
  int32_t *unit_slot, *slot_unit, *order, *order_tmp, *row_of, *hits_out, *misses_out, *bypass_out, *victim_unit,
      *victim_slot, *gather_unit, *gather_row, *meta;
  int64_t* stats;
  const uint4* master;  // device view of the host master
  uint4* rows;
  int unit_vec;         // unit_bytes / 16
};

// One cache step.  S = idx[0..n) ascending.  Runs in one CTA of
// kIndexThreads threads with `capacity` bytes of dynamic shared memory.
__device__ void cache_step(const CacheDev& d) {
  const int32_t* __restrict__ S = d.S;  // shifted to a part's sub-range below
  const int max_select = d.max_select, capacity = d.capacity;
  int32_t* __restrict__ unit_slot = d.unit_slot;
  int32_t* __restrict__ slot_unit = d.slot_unit;
  int32_t* __restrict__ order = d.order;
  int32_t* __restrict__ order_tmp = d.order_tmp;
  int32_t* __restrict__ row_of = d.row_of;
  int32_t* __restrict__ hits_out = d.hits_out;
  int32_t* __restrict__ misses_out = d.misses_out;
  int32_t* __restrict__ bypass_out = d.bypass_out;
  int32_t* __restrict__ victim_unit = d.victim_unit;
  int32_t* __restrict__ victim_slot = d.victim_slot;
  int32_t* __restrict__ gather_unit = d.gather_unit;
  int32_t* __restrict__ gather_row = d.gather_row;
  int32_t* __restrict__ meta = d.meta;
  int64_t* __restrict__ stats = d.stats;
  const int64_t unit_bytes = d.unit_bytes;
  extern __shared__ uint8_t slot_hit[];  // [capacity]
  __shared__ int scratch[33];
  const int tid = threadIdx.x;
  int n = *d.n_ptr;
  const int slot_base = d.slot_base;
  if (d.unit_lo >= 0) {
    // a part of a partitioned cache: its units form one contiguous run of
    // the ascending selection, found by binary search
    __shared__ int range[2];
    n = n < 0 ? 0 : n;
    if (tid < 2) {
      const int key = tid == 0 ? d.unit_lo : d.unit_hi;
      int a = 0, b = n;  // first position with S[pos] >= key
      while (a < b) {
        const int m = (a + b) >> 1;
        if (S[m] < key) a = m + 1; else b = m;
      }
      range[tid] = a;
    }
    __syncthreads();
    S += range[0];
    row_of += range[0];
    n = range[1] - range[0];
  }
  n = n < 0 ? 0 : (n > max_select ? max_select : n);
  const int occ = meta[kOcc];

  for (int i = tid; i < capacity; i += kIndexThreads) slot_hit[i] = 0;
  __syncthreads();

  // 1. hits and misses of S, in ascending order (ordered scan over chunks)
  const int chunk = (n + kIndexThreads - 1) / kIndexThreads;
  const int p0 = min(n, tid * chunk), p1 = min(n, p0 + chunk);
  int h = 0;
  for (int p = p0; p < p1; ++p) {
    const int sl = unit_slot[S[p]];
    if (sl >= 0) { ++h; slot_hit[sl - slot_base] = 1; }
  }
  int H;
  const int h_before = sfd::block_exclusive_scan(h, scratch, &H);
  {
    int hh = h_before, mm = p0 - h_before;
    for (int p = p0; p < p1; ++p) {
      const int u = S[p];
      if (unit_slot[u] >= 0) hits_out[hh++] = u; else misses_out[mm++] = u;
    }
  }
  const int mi = n - H;
  const int fetch = min(mi, d.budget);  // the misses after these are late: not fetched, not cached
  const int avail = capacity - H;
  const int ins = min(fetch, avail);
  const int use_free = min(ins, capacity - occ);
  const int v = ins - use_free;

  // 2. LRU order without the hits; its first v entries are the victims
  const int ochunk = (occ + kIndexThreads - 1) / kIndexThreads;
  const int o0 = min(occ, tid * ochunk), o1 = min(occ, o0 + ochunk);
  int keep = 0;
  for (int i = o0; i < o1; ++i) keep += !slot_hit[unit_slot[order[i]] - slot_base];
  int F;
  int fpos = sfd::block_exclusive_scan(keep, scratch, &F);
  for (int i = o0; i < o1; ++i) {
    const int u = order[i];
    const int sl = unit_slot[u] - slot_base;  // local slot
    if (slot_hit[sl]) continue;
    if (fpos < v) { victim_unit[fpos] = u; victim_slot[fpos] = sl; }
    else order_tmp[fpos - v] = u;
    ++fpos;
  }
  __syncthreads();

  // 3. place the fetched misses: free slots first, then victims, then bypass rows
  for (int r = tid; r < fetch; r += kIndexThreads) {
    const int u = misses_out[r];
    int row;
    if (r < use_free) {
      row = slot_base + occ + r;
    } else if (r < ins) {
      row = slot_base + victim_slot[r - use_free];
      unit_slot[victim_unit[r - use_free]] = -1;
    } else {
      row = d.bypass_base + (r - ins);
      bypass_out[r - ins] = u;
    }
    if (r < ins) { unit_slot[u] = row; slot_unit[row - slot_base] = u; }
    gather_unit[r] = u;
    gather_row[r] = row;
  }
  __syncthreads();

  // 4. row of every selected position; 5. append touched units to the order
  int touched = 0;
  {
    int mm = p0 - h_before;
    for (int p = p0; p < p1; ++p) {
      const int u = S[p];
      // a unit is a hit iff it is not in the miss list; misses are ranked mm
      // in ascending order, so compare with the miss list entry at rank mm
      const bool is_miss = (mm < mi) && (misses_out[mm] == u);
      if (is_miss) {
        row_of[p] = mm < fetch ? gather_row[mm] : -1;
        if (mm < ins) ++touched;
        ++mm;
      } else {
        row_of[p] = unit_slot[u];
        ++touched;
      }
    }
  }
  int T_all;
  int tpos = sfd::block_exclusive_scan(touched, scratch, &T_all);
  const int base = (occ - H) - v;
  {
    int mm = p0 - h_before;
    for (int p = p0; p < p1; ++p) {
      const int u = S[p];
      const bool is_miss = (mm < mi) && (misses_out[mm] == u);
      bool t_here = true;
      if (is_miss) { t_here = mm < ins; ++mm; }
      if (t_here) order_tmp[base + tpos++] = u;
    }
  }
  __syncthreads();
  const int new_occ = occ + use_free;
  for (int i = tid; i < new_occ; i += kIndexThreads) order[i] = order_tmp[i];
  if (tid == 0) {
    meta[kOcc] = new_occ;
    meta[kStep] += 1;
    meta[kHits] = H;
    meta[kMisses] = mi;
    meta[kBypass] = fetch - ins;
    meta[kGather] = fetch;
    stats[kStSteps] += 1;
    stats[kStHits] += H;
    stats[kStMisses] += mi;
    stats[kStBypass] += fetch - ins;
    stats[kStBytes] += static_cast<int64_t>(fetch) * unit_bytes;
    stats[kStLate] += mi - fetch;
  }
}

__global__ void __launch_bounds__(kIndexThreads) cache_index_kernel(CacheDev d) { cache_step(d); }

// One CTA per cache of a group.
__global__ void __launch_bounds__(kIndexThreads) cache_index_many_kernel(const CacheDev* __restrict__ table) {
  cache_step(table[blockIdx.x]);
}

// The parts of a partitioned cache, one CTA each, on the selection (S, n).
__global__ void __launch_bounds__(kIndexThreads)
cache_index_parts_kernel(const CacheDev* __restrict__ table, const int32_t* S, const int32_t* n) {
  CacheDev d = table[blockIdx.x];
  d.S = S;
  d.n_ptr = n;
  cache_step(d);
}

// Copy the missed units of `count` caches: one warp per unit, every lane
// keeping several 16-byte loads from the host link in flight.
__global__ void __launch_bounds__(256)
cache_gather_many_kernel(const CacheDev* __restrict__ table, int count) {
  __shared__ int offs[65];
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int c = 0; c < count; ++c) { offs[c] = acc; acc += table[c].meta[kGather]; }
    offs[count] = acc;
  }
  __syncthreads();
  const int total = offs[count];
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  for (int e = gw; e < total; e += nwarps) {
    int c = 0;
    while (offs[c + 1] <= e) ++c;
    const CacheDev& d = table[c];
    const int i = e - offs[c];
    const uint4* src = d.master + static_cast<size_t>(d.gather_unit[i]) * d.unit_vec;
    uint4* dst = d.rows + static_cast<size_t>(d.gather_row[i]) * d.unit_vec;
    for (int w = lane; w < d.unit_vec; w += 4 * 32) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (w + 32 * u < d.unit_vec) v[u] = src[w + 32 * u];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (w + 32 * u < d.unit_vec) dst[w + 32 * u] = v[u];
    }
  }
}

// Copy every missed unit of one cache (descriptor by value).
__global__ void __launch_bounds__(256) cache_gather_kernel(CacheDev d) {
  const int n = d.meta[kGather];
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  for (int i = gw; i < n; i += nwarps) {
    const uint4* src = d.master + static_cast<size_t>(d.gather_unit[i]) * d.unit_vec;
    uint4* dst = d.rows + static_cast<size_t>(d.gather_row[i]) * d.unit_vec;
    for (int w = lane; w < d.unit_vec; w += 4 * 32) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (w + 32 * u < d.unit_vec) v[u] = src[w + 32 * u];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (w + 32 * u < d.unit_vec) dst[w + 32 * u] = v[u];
    }
  }
}

// Preload: units[i] goes to slot i; copies its bytes too.
__global__ void cache_preload_kernel(const int32_t* __restrict__ units, int n, const uint4* __restrict__ master,
                                     uint4* __restrict__ rows, int unit_vec, int32_t* __restrict__ unit_slot,
                                     int32_t* __restrict__ slot_unit, int32_t* __restrict__ order,
                                     int32_t* __restrict__ meta) {
  for (int e = blockIdx.x; e < n; e += gridDim.x) {
    const int u = units[e];
    if (threadIdx.x == 0) {
      unit_slot[u] = e;
      slot_unit[e] = u;
      order[e] = u;
    }
    const uint4* src = master + static_cast<size_t>(u) * unit_vec;
    uint4* dst = rows + static_cast<size_t>(e) * unit_vec;
    for (int w = threadIdx.x; w < unit_vec; w += blockDim.x) dst[w] = src[w];
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) meta[kOcc] = n;
}

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    cudaGetDevice(&prev);
    if (prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur = -1;
    cudaGetDevice(&cur);
    if (prev >= 0 && cur != prev) cudaSetDevice(prev);
  }
};

unsigned long long capture_id(cudaStream_t s) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  unsigned long long id = 0;
  if (cudaStreamGetCaptureInfo(s, &st, &id) != cudaSuccess) return 0;
  return st == cudaStreamCaptureStatusActive ? id : 0;
}

}  // namespace

struct sf_refine_cache {
  int device = 0;
  int num_units = 0;
  size_t unit_bytes = 0;
  int parts = 1;       // independent LRUs over consecutive unit ranges of part_units units
  int part_units = 0;
  int capacity = 0;    // slots per part
  int max_select = 0;  // selected units per part and step at most
  int budget = 0;  // per-step fetch limit; max_select = no limit
  bool deadline = false;  // GEMVs refine only the selected units cached when they run
  const void* host_master = nullptr;
  const void* master_dev = nullptr;
  bool registered_here = false;
  uint32_t* rows = nullptr;
  int32_t* ints = nullptr;  // one allocation for every int32 array below
  int32_t *unit_slot = nullptr, *slot_unit = nullptr, *order = nullptr, *order_tmp = nullptr, *row_of = nullptr,
          *hits = nullptr, *misses = nullptr, *bypass = nullptr, *victim_unit = nullptr, *victim_slot = nullptr,
          *gather_unit = nullptr, *gather_row = nullptr, *meta = nullptr;
  int64_t* stats = nullptr;
  CacheDev* table = nullptr;  // parts > 1: the parts' descriptors on the device
  cudaEvent_t ev_idx = nullptr, ev_ready = nullptr, ev_used = nullptr;
  cudaStream_t aux = nullptr;
  bool ready_pending = false, used_pending = false;
  unsigned long long ready_capture = 0, used_capture = 0;
  // a writer's staging area for the host master (sf_kv_append_pair_cached)
  uint32_t* stage = nullptr;
  size_t stage_words = 0;
  cudaEvent_t ev_staged = nullptr, ev_flushed = nullptr;
  bool flush_pending = false;
  unsigned long long flush_capture = 0;
};

namespace {

// Descriptor of part `p` (parts == 1: the whole cache).  Per-part arrays are
// laid out part after part; slot numbers and rows are global.
CacheDev make_dev(const sf_refine_cache* c, const int32_t* S, const int32_t* n, int p = 0) {
  CacheDev d{};
  const size_t cap1 = std::max(c->capacity, 1), ms = c->max_select;
  d.S = S;
  d.n_ptr = n;
  d.max_select = c->max_select;
  d.capacity = c->capacity;
  d.budget = c->budget;
  d.slot_base = p * c->capacity;
  d.bypass_base = c->parts * c->capacity + p * c->max_select;
  d.unit_lo = c->parts > 1 ? p * c->part_units : -1;
  d.unit_hi = c->parts > 1 ? (p + 1) * c->part_units : -1;
  d.unit_bytes = static_cast<int64_t>(c->unit_bytes);
  d.unit_slot = c->unit_slot;
  d.slot_unit = c->slot_unit + p * cap1;
  d.order = c->order + p * cap1;
  d.order_tmp = c->order_tmp + p * cap1;
  d.row_of = c->row_of;
  d.hits_out = c->hits + p * ms;
  d.misses_out = c->misses + p * ms;
  d.bypass_out = c->bypass + p * ms;
  d.victim_unit = c->victim_unit + p * ms;
  d.victim_slot = c->victim_slot + p * ms;
  d.gather_unit = c->gather_unit + p * ms;
  d.gather_row = c->gather_row + p * ms;
  d.meta = c->meta + p * kMetaCount;
  d.stats = c->stats + p * kStatCount;
  d.master = static_cast<const uint4*>(c->master_dev);
  d.rows = reinterpret_cast<uint4*>(c->rows);
  d.unit_vec = static_cast<int>(c->unit_bytes / 16);
  return d;
}

sf_status cache_free(sf_refine_cache* c) {
  if (!c) return SF_OK;
  DeviceGuard g(c->device);
  if (c->aux) cudaStreamSynchronize(c->aux);
  if (c->ev_ready) cudaEventSynchronize(c->ev_ready);
  if (c->ev_used) cudaEventSynchronize(c->ev_used);
  if (c->rows) cudaFree(c->rows);
  if (c->ints) cudaFree(c->ints);
  if (c->table) cudaFree(c->table);
  if (c->stats) cudaFree(c->stats);
  if (c->ev_idx) cudaEventDestroy(c->ev_idx);
  if (c->ev_ready) cudaEventDestroy(c->ev_ready);
  if (c->ev_used) cudaEventDestroy(c->ev_used);
  if (c->stage) cudaFree(c->stage);
  if (c->ev_staged) cudaEventDestroy(c->ev_staged);
  if (c->ev_flushed) cudaEventDestroy(c->ev_flushed);
  if (c->aux) cudaStreamDestroy(c->aux);
  if (c->registered_here) cudaHostUnregister(const_cast<void*>(c->host_master));
  delete c;
  cudaGetLastError();  // teardown is best effort: leave no error for the next launch check
  return SF_OK;
}

sf_status cache_clear(sf_refine_cache* c, cudaStream_t s) {
  SF_CHECK_CUDA(cudaMemsetAsync(c->unit_slot, 0xFF, sizeof(int32_t) * c->num_units, s));
  SF_CHECK_CUDA(cudaMemsetAsync(c->slot_unit, 0xFF, sizeof(int32_t) * std::max(c->capacity, 1) * c->parts, s));
  SF_CHECK_CUDA(cudaMemsetAsync(c->meta, 0, sizeof(int32_t) * kMetaCount * c->parts, s));
  SF_CHECK_CUDA(cudaMemsetAsync(c->stats, 0, sizeof(int64_t) * kStatCount * c->parts, s));
  return SF_OK;
}

// Host wait for the last prefetch.  Once it has completed, later GEMVs need
// not wait for it on the device any more (so a GEMV captured into a graph
// after this point may consume an eager prefetch).
// A prefetch captured into a graph has no event to wait on from the host:
// the caller synchronizes the stream the graph was launched on first.
sf_status wait_ready(sf_refine_cache* c) {
  if (c->ready_pending) {
    if (c->ready_capture == 0) SF_CHECK_CUDA(cudaEventSynchronize(c->ev_ready));
    c->ready_pending = false;
  }
  SF_CHECK_CUDA(cudaStreamSynchronize(c->aux));
  return SF_OK;
}

// parts > 1: the parts' descriptors (selection pointers filled per prefetch
// by the kernel's arguments) on the device.
sf_status upload_table(sf_refine_cache* c) {
  std::vector<CacheDev> host(c->parts);
  for (int q = 0; q < c->parts; ++q) host[q] = make_dev(c, nullptr, nullptr, q);
  if (!c->table) SF_CHECK_CUDA(cudaMalloc(&c->table, sizeof(CacheDev) * c->parts));
  SF_CHECK_CUDA(cudaMemcpy(c->table, host.data(), sizeof(CacheDev) * c->parts, cudaMemcpyHostToDevice));
  return SF_OK;
}

}  // namespace

namespace sf {

sf_status cache_view_for_gemv(sf_refine_cache* c, cudaStream_t stream, CacheView* v) {
  SF_REQUIRE(c->budget >= c->max_select,
             "sf_gemv_refine: a GEMV needs every selected column fetched; this cache has a fetch budget "
             "(use the deadline reading, sf_refine_cache_set_deadline)");
  SF_REQUIRE(!c->deadline, "sf_gemv_refine: only the batch-1 GEMV reads a cache in the deadline reading");
  return cache_view_for_reader(c, stream, v);
}

sf_status cache_view_for_reader(sf_refine_cache* c, cudaStream_t stream, CacheView* v) {
  if (c->ready_pending) {
    const unsigned long long cid = capture_id(stream);
    SF_REQUIRE(cid == c->ready_capture,
               "sf_gemv_refine: the cache's last prefetch and this GEMV must both be inside the same stream "
               "capture, or both outside one");
    SF_CHECK_CUDA(cudaStreamWaitEvent(stream, c->ev_ready, 0));
  }
  v->rows = c->rows;
  v->row_of = c->row_of;
  v->unit_slot = c->unit_slot;
  v->num_units = c->num_units;
  v->unit_words = static_cast<int>(c->unit_bytes / 4);
  v->max_select = c->max_select * c->parts;
  return SF_OK;
}

sf_status cache_view_for_writer(sf_refine_cache* c, cudaStream_t stream, CacheWriteView* w) {
  CacheView v{};
  const sf_status st = cache_view_for_reader(c, stream, &v);
  if (st != SF_OK) return st;
  w->master = static_cast<uint32_t*>(const_cast<void*>(c->master_dev));
  w->rows = c->rows;
  w->unit_slot = c->unit_slot;
  w->num_units = c->num_units;
  w->unit_words = static_cast<int>(c->unit_bytes / 4);
  return SF_OK;
}

bool cache_deadline(const sf_refine_cache* c) { return c->deadline; }

sf_status cache_append_stage(sf_refine_cache* c, cudaStream_t stream, size_t words, uint32_t** stage) {
  if (c->stage_words < words) {
    SF_REQUIRE(capture_id(stream) == 0,
               "sf_kv_append_pair_cached: the first call per cache must not be under stream capture");
    DeviceGuard guard(c->device);
    if (c->stage) {
      SF_CHECK_CUDA(cudaStreamSynchronize(stream));
      cudaFree(c->stage);
      c->stage = nullptr;
      c->stage_words = 0;
    }
    SF_CHECK_CUDA(cudaMalloc(&c->stage, words * 4));
    c->stage_words = words;
    if (!c->ev_staged) SF_CHECK_CUDA(cudaEventCreateWithFlags(&c->ev_staged, cudaEventDisableTiming));
    if (!c->ev_flushed) SF_CHECK_CUDA(cudaEventCreateWithFlags(&c->ev_flushed, cudaEventDisableTiming));
  }
  // the last flush read the staging area: the next write waits for it
  if (c->flush_pending && c->flush_capture == capture_id(stream))
    SF_CHECK_CUDA(cudaStreamWaitEvent(stream, c->ev_flushed, 0));
  *stage = c->stage;
  return SF_OK;
}

sf_status cache_append_flush(sf_refine_cache* c, cudaStream_t stream, cudaStream_t side, size_t dst_off,
                             size_t dpitch, size_t width, int height) {
  if (side != stream) {
    SF_CHECK_CUDA(cudaEventRecord(c->ev_staged, stream));
    SF_CHECK_CUDA(cudaStreamWaitEvent(side, c->ev_staged, 0));
  }
  char* dst = static_cast<char*>(const_cast<void*>(c->host_master)) + dst_off;
  SF_CHECK_CUDA(cudaMemcpy2DAsync(dst, dpitch, c->stage, width, width, static_cast<size_t>(height),
                                  cudaMemcpyDeviceToHost, side));
  SF_CHECK_CUDA(cudaEventRecord(c->ev_flushed, side));
  c->flush_pending = true;
  c->flush_capture = capture_id(side);
  return SF_OK;
}

sf_status cache_mark_used(sf_refine_cache* c, cudaStream_t stream) {
  SF_CHECK_CUDA(cudaEventRecord(c->ev_used, stream));
  c->used_pending = true;
  c->used_capture = capture_id(stream);
  return SF_OK;
}

}  // namespace sf

extern "C" {

sf_status sf_refine_cache_create_parts(sf_refine_cache** out, int num_units, size_t unit_bytes, int parts,
                                       int capacity, int max_select, const void* host_master, int device) {
  SF_REQUIRE(out && host_master, "sf_refine_cache_create: null pointer");
  *out = nullptr;
  SF_REQUIRE(num_units >= 1, "sf_refine_cache_create: num_units must be >= 1");
  SF_REQUIRE(parts >= 1 && parts <= 64 && num_units % parts == 0,
             "sf_refine_cache_create: parts must be in [1, 64] and divide num_units");
  const int part_units = num_units / parts;
  SF_REQUIRE(unit_bytes >= 16 && unit_bytes % 16 == 0, "sf_refine_cache_create: unit_bytes must be a positive multiple of 16");
  SF_REQUIRE(capacity >= 0 && capacity <= part_units && capacity <= kMaxCapacity,
             "sf_refine_cache_create: capacity must be in [0, min(units per part, %d)]", kMaxCapacity);
  SF_REQUIRE(max_select >= 1 && max_select <= 1 << 20, "sf_refine_cache_create: max_select out of range");
  SF_REQUIRE(static_cast<long long>(parts) * (capacity + max_select) < (1LL << 31),
             "sf_refine_cache_create: too many rows");
  SF_REQUIRE(sf::aligned(host_master, 16), "sf_refine_cache_create: host_master must be 16-byte aligned");
  DeviceGuard g(device);
  auto* c = new sf_refine_cache();
  c->device = device;
  c->num_units = num_units;
  c->unit_bytes = unit_bytes;
  c->parts = parts;
  c->part_units = part_units;
  c->capacity = capacity;
  c->max_select = max_select;
  c->budget = max_select;
  c->host_master = host_master;
  const size_t master_bytes = static_cast<size_t>(num_units) * unit_bytes;

  cudaPointerAttributes attr{};
  cudaError_t e = cudaPointerGetAttributes(&attr, host_master);
  if (e != cudaSuccess) cudaGetLastError();
  if (e != cudaSuccess || attr.type == cudaMemoryTypeUnregistered) {
    e = cudaHostRegister(const_cast<void*>(host_master), master_bytes, cudaHostRegisterMapped);
    if (e != cudaSuccess) { cache_free(c); return sf::cuda_fail(e, "cudaHostRegister(host_master)"); }
    c->registered_here = true;
  } else if (attr.type != cudaMemoryTypeHost) {
    cache_free(c);
    return sf::fail(SF_EINVAL, "sf_refine_cache_create: host_master must be host memory");
  }
  void* dptr = nullptr;
  e = cudaHostGetDevicePointer(&dptr, const_cast<void*>(host_master), 0);
  if (e != cudaSuccess) { cache_free(c); return sf::cuda_fail(e, "cudaHostGetDevicePointer(host_master)"); }
  c->master_dev = dptr;

  const size_t P = parts;
  const size_t rows_bytes = P * (static_cast<size_t>(capacity) + max_select) * unit_bytes;
  e = cudaMalloc(&c->rows, rows_bytes);
  if (e != cudaSuccess) { cache_free(c); return sf::fail(SF_ENOMEM, "sf_refine_cache_create: cudaMalloc rows: %s", cudaGetErrorString(e)); }
  const size_t cap1 = std::max(capacity, 1), ms = max_select;
  const size_t n_ints = static_cast<size_t>(num_units) + P * (3 * cap1 + 8 * ms + kMetaCount);
  e = cudaMalloc(&c->ints, n_ints * sizeof(int32_t));
  if (e != cudaSuccess) { cache_free(c); return sf::fail(SF_ENOMEM, "sf_refine_cache_create: cudaMalloc index: %s", cudaGetErrorString(e)); }
  e = cudaMalloc(&c->stats, P * kStatCount * sizeof(int64_t));
  if (e != cudaSuccess) { cache_free(c); return sf::fail(SF_ENOMEM, "sf_refine_cache_create: cudaMalloc stats: %s", cudaGetErrorString(e)); }
  int32_t* p = c->ints;
  c->unit_slot = p; p += num_units;
  c->slot_unit = p; p += P * cap1;
  c->order = p; p += P * cap1;
  c->order_tmp = p; p += P * cap1;
  c->row_of = p; p += P * ms;
  c->hits = p; p += P * ms;
  c->misses = p; p += P * ms;
  c->bypass = p; p += P * ms;
  c->victim_unit = p; p += P * ms;
  c->victim_slot = p; p += P * ms;
  c->gather_unit = p; p += P * ms;
  c->gather_row = p; p += P * ms;
  c->meta = p;
  if ((e = cudaEventCreateWithFlags(&c->ev_idx, cudaEventDisableTiming)) != cudaSuccess ||
      (e = cudaEventCreateWithFlags(&c->ev_ready, cudaEventDisableTiming)) != cudaSuccess ||
      (e = cudaEventCreateWithFlags(&c->ev_used, cudaEventDisableTiming)) != cudaSuccess ||
      (e = cudaStreamCreateWithFlags(&c->aux, cudaStreamNonBlocking)) != cudaSuccess) {
    cache_free(c);
    return sf::cuda_fail(e, "sf_refine_cache_create: events/stream");
  }
  sf_status st = cache_clear(c, c->aux);
  if (st == SF_OK && parts > 1) st = upload_table(c);
  if (st == SF_OK) {
    e = cudaStreamSynchronize(c->aux);
    if (e != cudaSuccess) st = sf::cuda_fail(e, "sf_refine_cache_create: init");
  }
  if (st != SF_OK) { cache_free(c); return st; }
  *out = c;
  return SF_OK;
}

sf_status sf_refine_cache_create(sf_refine_cache** out, int num_units, size_t unit_bytes, int capacity,
                                 int max_select, const void* host_master, int device) {
  return sf_refine_cache_create_parts(out, num_units, unit_bytes, 1, capacity, max_select, host_master, device);
}

sf_status sf_refine_cache_preload(sf_refine_cache* c, const int32_t* units, int n, sf_stream_t stream) {
  SF_REQUIRE(c, "sf_refine_cache_preload: null cache");
  SF_REQUIRE(c->parts == 1, "sf_refine_cache_preload: not available for a partitioned cache");
  SF_REQUIRE(n >= 0 && n <= c->capacity, "sf_refine_cache_preload: n must be in [0, capacity]");
  SF_REQUIRE(n == 0 || units, "sf_refine_cache_preload: null units");
  DeviceGuard g(c->device);
  if (n == 0) return SF_OK;
  cudaStream_t s = sf::as_cuda(stream);
  const int grid = std::min(n, 4 * sf::sm_count());
  cache_preload_kernel<<<grid, kGatherThreads, 0, s>>>(units, n, static_cast<const uint4*>(c->master_dev),
                                                        reinterpret_cast<uint4*>(c->rows),
                                                        static_cast<int>(c->unit_bytes / 16), c->unit_slot,
                                                        c->slot_unit, c->order, c->meta);
  return sf::check_launch("cache_preload_kernel");
}

sf_status sf_refine_cache_prefetch(sf_refine_cache* c, const int32_t* idx, const int32_t* n, sf_stream_t producer,
                                   sf_stream_t side) {
  SF_REQUIRE(c && idx && n, "sf_refine_cache_prefetch: null pointer");
  DeviceGuard g(c->device);
  cudaStream_t ps = sf::as_cuda(producer), ss = sf::as_cuda(side);
  // when the producer is being captured, waiting on its event forks the side
  // stream into the same capture
  const unsigned long long cid = capture_id(ps);
  SF_CHECK_CUDA(cudaEventRecord(c->ev_idx, ps));
  SF_CHECK_CUDA(cudaStreamWaitEvent(ss, c->ev_idx, 0));
  // the previous step's GEMV must have read the rows before they change
  if (c->used_pending && c->used_capture == cid) SF_CHECK_CUDA(cudaStreamWaitEvent(ss, c->ev_used, 0));
  const size_t smem = std::max(c->capacity, 1);
  sf_status st;
  if (c->parts == 1) {
    const CacheDev d = make_dev(c, idx, n);
    SF_CHECK_CUDA(cudaFuncSetAttribute(cache_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)));
    cache_index_kernel<<<1, kIndexThreads, smem, ss>>>(d);
    st = sf::check_launch("cache_index_kernel");
    if (st != SF_OK) return st;
    const int grid = std::min((c->max_select + 7) / 8, 2 * sf::sm_count());
    cache_gather_kernel<<<grid, 256, 0, ss>>>(d);
    st = sf::check_launch("cache_gather_kernel");
  } else {  // one CTA per part, then one gather over every part's misses
    SF_CHECK_CUDA(cudaFuncSetAttribute(cache_index_parts_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)));
    cache_index_parts_kernel<<<c->parts, kIndexThreads, smem, ss>>>(c->table, idx, n);
    st = sf::check_launch("cache_index_parts_kernel");
    if (st != SF_OK) return st;
    const int grid = std::min((c->parts * c->max_select + 7) / 8, 4 * sf::sm_count());
    cache_gather_many_kernel<<<grid, 256, 0, ss>>>(c->table, c->parts);
    st = sf::check_launch("cache_gather_many_kernel");
  }
  if (st != SF_OK) return st;
  SF_CHECK_CUDA(cudaEventRecord(c->ev_ready, ss));
  c->ready_pending = true;
  c->ready_capture = cid;
  c->used_pending = false;
  return SF_OK;
}

sf_status sf_refine_cache_sets(sf_refine_cache* c, int32_t* hits, int32_t* misses, int32_t* bypass,
                               int32_t counts[3]) {
  SF_REQUIRE(c && counts, "sf_refine_cache_sets: null pointer");
  DeviceGuard g(c->device);
  sf_status st = wait_ready(c);
  if (st != SF_OK) return st;
  // the parts' lists, concatenated in part order (so each stays ascending)
  std::vector<int32_t> meta(static_cast<size_t>(kMetaCount) * c->parts);
  SF_CHECK_CUDA(cudaMemcpy(meta.data(), c->meta, sizeof(int32_t) * meta.size(), cudaMemcpyDeviceToHost));
  counts[0] = counts[1] = counts[2] = 0;
  const size_t ms = c->max_select;
  for (int q = 0; q < c->parts; ++q) {
    const int32_t* m = meta.data() + q * kMetaCount;
    if (hits && m[kHits])
      SF_CHECK_CUDA(cudaMemcpy(hits + counts[0], c->hits + q * ms, sizeof(int32_t) * m[kHits], cudaMemcpyDeviceToHost));
    if (misses && m[kMisses])
      SF_CHECK_CUDA(cudaMemcpy(misses + counts[1], c->misses + q * ms, sizeof(int32_t) * m[kMisses],
                               cudaMemcpyDeviceToHost));
    if (bypass && m[kBypass])
      SF_CHECK_CUDA(cudaMemcpy(bypass + counts[2], c->bypass + q * ms, sizeof(int32_t) * m[kBypass],
                               cudaMemcpyDeviceToHost));
    counts[0] += m[kHits];
    counts[1] += m[kMisses];
    counts[2] += m[kBypass];
  }
  return SF_OK;
}

sf_status sf_refine_cache_slots(sf_refine_cache* c, int32_t* slot_units) {
  SF_REQUIRE(c && slot_units, "sf_refine_cache_slots: null pointer");
  DeviceGuard g(c->device);
  sf_status st = wait_ready(c);
  if (st != SF_OK) return st;
  for (int q = 0; q < c->parts && c->capacity; ++q)
    SF_CHECK_CUDA(cudaMemcpy(slot_units + static_cast<size_t>(q) * c->capacity,
                             c->slot_unit + static_cast<size_t>(q) * std::max(c->capacity, 1),
                             sizeof(int32_t) * c->capacity, cudaMemcpyDeviceToHost));
  return SF_OK;
}

sf_status sf_refine_cache_stats(sf_refine_cache* c, sf_cache_stats* out) {
  SF_REQUIRE(c && out, "sf_refine_cache_stats: null pointer");
  DeviceGuard g(c->device);
  sf_status st = wait_ready(c);
  if (st != SF_OK) return st;
  std::vector<int64_t> all(static_cast<size_t>(kStatCount) * c->parts);
  SF_CHECK_CUDA(cudaMemcpy(all.data(), c->stats, sizeof(int64_t) * all.size(), cudaMemcpyDeviceToHost));
  int64_t s[kStatCount] = {};
  for (int q = 0; q < c->parts; ++q)
    for (int k = 0; k < kStatCount; ++k) s[k] += all[q * kStatCount + k];
  s[kStSteps] /= c->parts;  // every part counts each step
  out->steps = s[kStSteps];
  out->hits = s[kStHits];
  out->misses = s[kStMisses];
  out->bypass = s[kStBypass];
  out->h2d_bytes = s[kStBytes];
  out->late = s[kStLate];
  return SF_OK;
}

sf_status sf_refine_cache_reset(sf_refine_cache* c) {
  SF_REQUIRE(c, "sf_refine_cache_reset: null cache");
  DeviceGuard g(c->device);
  sf_status st = wait_ready(c);
  if (st != SF_OK) return st;
  if (c->used_pending) SF_CHECK_CUDA(cudaEventSynchronize(c->ev_used));
  st = cache_clear(c, c->aux);
  if (st != SF_OK) return st;
  SF_CHECK_CUDA(cudaStreamSynchronize(c->aux));
  c->ready_pending = c->used_pending = false;
  return SF_OK;
}

sf_status sf_refine_cache_destroy(sf_refine_cache* c) { return cache_free(c); }

sf_status sf_refine_cache_set_deadline(sf_refine_cache* c, int on) {
  SF_REQUIRE(c, "sf_refine_cache_set_deadline: null cache");
  SF_REQUIRE(c->parts == 1, "sf_refine_cache_set_deadline: for the cache of one weight matrix (parts = 1)");
  c->deadline = on != 0;
  return SF_OK;
}

sf_status sf_refine_cache_set_budget(sf_refine_cache* c, int budget) {
  SF_REQUIRE(c, "sf_refine_cache_set_budget: null cache");
  SF_REQUIRE(budget >= -1, "sf_refine_cache_set_budget: budget must be >= 0, or -1 for none");
  c->budget = budget < 0 || budget > c->max_select ? c->max_select : budget;
  if (c->parts > 1) return upload_table(c);
  return SF_OK;
}

// ---- groups: one index launch and one gather launch for several caches ----

}  // extern "C"

struct sf_refine_group {
  int device = 0;
  int count = 0;
  std::vector<sf_refine_cache*> caches;
  CacheDev* table = nullptr;  // device copy of the descriptors
  int max_capacity = 1;
  int total_select = 0;
  cudaEvent_t ev_idx = nullptr;
};

extern "C" {

sf_status sf_refine_group_create(sf_refine_group** out, sf_refine_cache* const* caches, const int32_t* const* idx,
                                 const int32_t* const* n, int count) {
  SF_REQUIRE(out && caches && idx && n, "sf_refine_group_create: null pointer");
  *out = nullptr;
  SF_REQUIRE(count >= 1 && count <= 64, "sf_refine_group_create: count must be in [1, 64]");
  for (int i = 0; i < count; ++i) {
    SF_REQUIRE(caches[i] && idx[i] && n[i], "sf_refine_group_create: null entry %d", i);
    SF_REQUIRE(caches[i]->parts == 1, "sf_refine_group_create: a partitioned cache cannot join a group");
    SF_REQUIRE(caches[i]->device == caches[0]->device, "sf_refine_group_create: caches on different devices");
    for (int j = 0; j < i; ++j) SF_REQUIRE(caches[j] != caches[i], "sf_refine_group_create: cache listed twice");
  }
  DeviceGuard g(caches[0]->device);
  auto* grp = new sf_refine_group();
  grp->device = caches[0]->device;
  grp->count = count;
  std::vector<CacheDev> host(count);
  for (int i = 0; i < count; ++i) {
    grp->caches.push_back(caches[i]);
    host[i] = make_dev(caches[i], idx[i], n[i]);
    grp->max_capacity = std::max(grp->max_capacity, caches[i]->capacity);
    grp->total_select += caches[i]->max_select;
  }
  cudaError_t e = cudaMalloc(&grp->table, sizeof(CacheDev) * count);
  if (e == cudaSuccess) e = cudaMemcpy(grp->table, host.data(), sizeof(CacheDev) * count, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&grp->ev_idx, cudaEventDisableTiming);
  if (e != cudaSuccess) {
    if (grp->table) cudaFree(grp->table);
    delete grp;
    return sf::cuda_fail(e, "sf_refine_group_create");
  }
  *out = grp;
  return SF_OK;
}

sf_status sf_refine_group_prefetch(sf_refine_group* grp, sf_stream_t producer, sf_stream_t side) {
  SF_REQUIRE(grp, "sf_refine_group_prefetch: null group");
  DeviceGuard g(grp->device);
  cudaStream_t ps = sf::as_cuda(producer), ss = sf::as_cuda(side);
  const unsigned long long cid = capture_id(ps);
  SF_CHECK_CUDA(cudaEventRecord(grp->ev_idx, ps));
  SF_CHECK_CUDA(cudaStreamWaitEvent(ss, grp->ev_idx, 0));
  for (sf_refine_cache* c : grp->caches)
    if (c->used_pending && c->used_capture == cid) SF_CHECK_CUDA(cudaStreamWaitEvent(ss, c->ev_used, 0));
  SF_CHECK_CUDA(cudaFuncSetAttribute(cache_index_many_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     grp->max_capacity));
  cache_index_many_kernel<<<grp->count, kIndexThreads, grp->max_capacity, ss>>>(grp->table);
  sf_status st = sf::check_launch("cache_index_many_kernel");
  if (st != SF_OK) return st;
  const int grid = std::min((grp->total_select + 7) / 8, 4 * sf::sm_count());
  cache_gather_many_kernel<<<grid, 256, 0, ss>>>(grp->table, grp->count);
  st = sf::check_launch("cache_gather_many_kernel");
  if (st != SF_OK) return st;
  for (sf_refine_cache* c : grp->caches) {
    SF_CHECK_CUDA(cudaEventRecord(c->ev_ready, ss));
    c->ready_pending = true;
    c->ready_capture = cid;
    c->used_pending = false;
  }
  return SF_OK;
}

sf_status sf_refine_group_destroy(sf_refine_group* grp) {
  if (!grp) return SF_OK;
  DeviceGuard g(grp->device);
  cudaDeviceSynchronize();
  if (grp->table) cudaFree(grp->table);
  if (grp->ev_idx) cudaEventDestroy(grp->ev_idx);
  delete grp;
  cudaGetLastError();  // teardown is best effort: leave no error for the next launch check
  return SF_OK;
}

}  // extern "C"
