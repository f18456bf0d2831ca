// Top-k channel selection of one activation row by one thread block, from
// the row's bf16 bits in shared memory (the explainer of StrataFlux, 解説:
// weights are refined where the input activation is large).
//
// |x| of a bf16 value is its 15 low bits read as an unsigned integer (+0 and
// -0 tie, larger magnitudes give larger keys), so the selection is exact
// integer work: a two-pass radix select (8 high bits, then 7 low bits) finds
// the k-th largest key tau; keys above tau are taken and keys equal to tau in
// ascending channel order until k are chosen (ties to the lower index); an
// ordered compaction writes the ascending list.  The prepared activations of
// the batch-1 GEMV (act.cuh) are written from the same shared row.
#pragma once

#include <cstdint>

#include "act.cuh"
#include "block_scan.cuh"

namespace sfd {

constexpr int kSelRowMaxK = 32768;

// The selection of one row by the calling block, with scratch provided by the
// caller (so a kernel can place it where it has room).  xs: the row's K bf16
// bits (shared memory, 16-byte aligned, written and synchronized by the
// caller, readable up to the next multiple of 8 entries: sel_row_bytes(K));
// whist: hrows x 256 ints (warp w counts into row
// w % hrows); scan: 33 ints; info: 8 ints; flags: K bytes set to 1 for the
// selected channels (nullptr: not written).  Writes list[0..n) ascending
// (shared or global memory) and leaves n in info[5] (-1 if the row holds a
// NaN or Inf) and the number of list entries written in info[6], visible to
// every thread on return.  All threads of the block call; blockDim.x is a
// multiple of 32 up to 1024.
//
// Two radix passes (the high byte of the key, the bf16 exponent; then its
// low 7 bits inside the bin holding the k-th key) over 16-byte units of 8 keys
// taken by consecutive threads (no bank conflicts), counted into per-warp rows;
// then one block scan of packed
// (above, tied) counts over contiguous chunks of units gives every selected
// channel its position directly, ties taken in ascending channel order.  A
// chunk's units are read in an order rotated by the thread index, so the
// threads of a warp spread over the banks.
__device__ __forceinline__ uint32_t sel_key(const uint4& q, int e) {
  const uint32_t w = e < 2 ? q.x : (e < 4 ? q.y : (e < 6 ? q.z : q.w));
  return (w >> (16 * (e & 1))) & 0x7FFFu;
}

__host__ __device__ constexpr int sel_row_bytes(int K) { return (2 * K + 15) & ~15; }

// One warp: the bin b (counting from the top of hist[0..NB)) that holds the
// k-th largest key and the key's rank k' inside it; lane l sums the NB/32
// bins just below the top l NB/32, one inclusive scan over the lanes finds
// the lane, which walks its bins.  Writes out[0] = b (-1: fewer than k
// keys), out[1] = k'.
template <int NB>
__device__ __forceinline__ void sel_find_bin(const int* hist, int k, int* out) {
  constexpr int kPer = NB / 32;
  const int lane = threadIdx.x & 31;
  const int hi = NB - kPer * lane;  // this lane's bins: [hi - kPer, hi)
  int c[kPer];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    c[i] = hist[hi - 1 - i];  // descending
    sum += c[i];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned m = __ballot_sync(0xffffffffu, incl >= k);
  if (m == 0u) {
    if (lane == 0) {
      out[0] = -1;
      out[1] = 0;
    }
    return;
  }
  if (lane == __ffs(m) - 1) {
    int a = incl - sum;  // keys in the bins above this lane's
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      if (a + c[i] >= k) {
        out[0] = hi - 1 - i;
        out[1] = k - a;
        break;
      }
      a += c[i];
    }
  }
}

__device__ inline void select_row_cta(const uint16_t* xs, int K, int k, int32_t* list, int* whist, int hrows,
                                      int* scan, int* info, uint8_t* flags) {
  constexpr int kGrp = 4;  // units of a chunk held in registers at a time (a power of two)
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const uint4* xu = reinterpret_cast<const uint4*>(xs);
  const int nunits = (K + 7) >> 3;
  // contiguous chunks of units per thread (the ordered pass walks them in order)
  const int cu = (nunits + nthr - 1) / nthr;
  const int u0 = min(nunits, tid * cu), u1 = min(nunits, u0 + cu);
  int mybad = 0;
  if (k <= 0) {
    for (int u = tid; u < nunits; u += nthr) {
      const uint4 q = xu[u];
#pragma unroll
      for (int e = 0; e < 8; ++e) mybad |= 8 * u + e < K && (sel_key(q, e) & 0x7F80u) == 0x7F80u;
    }
    if (flags != nullptr)
      for (int j = tid; j < K; j += nthr) flags[j] = 0;
    const int bad = __syncthreads_or(mybad);
    if (tid == 0) {
      info[5] = bad ? -1 : 0;
      info[6] = 0;
    }
    __syncthreads();
    return;
  }
  int* hist = whist;  // row 0 doubles as the summed histogram
  int* wh = whist + (warp % hrows) * 256;
  // pass 1: high byte
  for (int b = tid; b < hrows * 256; b += nthr) whist[b] = 0;
  __syncthreads();
  for (int ub = 0; ub < nunits; ub += nthr) {
    const int u = ub + tid;
    const bool ok = u < nunits;
    const uint4 q = ok ? xu[u] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t v = sel_key(q, e);
      const bool in = ok && 8 * u + e < K;
      mybad |= in && (v & 0x7F80u) == 0x7F80u;
      if (in) atomicAdd(&wh[v >> 7], 1);
    }
  }
  const int bad = __syncthreads_or(mybad);
  for (int b = tid; b < 256; b += nthr) {  // column b is read and written by this thread only
    int c = 0;
#pragma unroll 4
    for (int w = 0; w < hrows; ++w) c += whist[w * 256 + b];
    hist[b] = c;
  }
  __syncthreads();
  if (warp == 0) sel_find_bin<256>(hist, k, info + 1);  // info[1] = b1, info[2] = k1
  // pass 2: low 7 bits inside bin b1 (few keys: plain atomics)
  __syncthreads();
  for (int b = tid; b < hrows * 128; b += nthr) whist[(b >> 7) * 256 + (b & 127)] = 0;
  __syncthreads();
  const int b1 = info[1];
  if (b1 >= 0)
    for (int u = tid; u < nunits; u += nthr) {
      const uint4 q = xu[u];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t v = sel_key(q, e);
        if (8 * u + e < K && static_cast<int>(v >> 7) == b1) atomicAdd(&wh[v & 0x7Fu], 1);
      }
    }
  __syncthreads();
  for (int b = tid; b < 128; b += nthr) {
    int c = 0;
#pragma unroll 4
    for (int w = 0; w < hrows; ++w) c += whist[w * 256 + b];
    hist[b] = c;
  }
  __syncthreads();
  if (warp == 0) {
    if (b1 >= 0) {
      sel_find_bin<128>(hist, info[2], info + 3);  // the low 7 bits, and the rank among equal keys
      __syncwarp();
      if (lane == 0 && info[3] >= 0) info[3] |= b1 << 7;
    } else if (lane == 0) {
      info[3] = -1;
      info[4] = 0;
    }
  }
  __syncthreads();
  // ordered pass: channel j is taken if key > tau, or key == tau and fewer
  // than r keys equal to tau precede it; its position is the number of taken
  // channels before it = (keys > tau before j) + min(ties before j, r)
  const int tau = info[3], r = info[4];
  const int kt = tau < 0 ? 0x10000 : tau;  // no key reaches it: nothing taken
  // a group's units, read in an order rotated by the thread index (a warp's
  // threads spread over the banks) into fixed registers (no local memory)
  auto load_group = [&](int g0, uint4 (&q)[kGrp]) {
    const int n = min(kGrp, u1 - g0);
#pragma unroll
    for (int s = 0; s < kGrp; ++s) {
      const int e = (s + tid) & (kGrp - 1);
      const uint4 v = e < n ? xu[g0 + e] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int c = 0; c < kGrp; ++c)
        if (c == e) q[c] = v;
    }
  };
  int gt = 0, eq = 0;
  for (int g0 = u0; g0 < u1; g0 += kGrp) {
    uint4 q[kGrp];
    load_group(g0, q);
    const int n = min(kGrp, u1 - g0);
#pragma unroll
    for (int uu = 0; uu < kGrp; ++uu)
      if (uu < n)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int key = 8 * (g0 + uu) + e < K ? static_cast<int>(sel_key(q[uu], e)) : -1;
          gt += key > kt;
          eq += key == kt;
        }
  }
  int total;
  const int pre = block_exclusive_scan((gt << 16) | eq, scan, &total);  // K <= 32768 fits 16 bits
  int gt_b = pre >> 16, eq_b = pre & 0xFFFF;
  for (int g0 = u0; g0 < u1; g0 += kGrp) {
    uint4 q[kGrp];
    load_group(g0, q);
    const int n = min(kGrp, u1 - g0);
#pragma unroll
    for (int uu = 0; uu < kGrp; ++uu)
      if (uu < n)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = 8 * (g0 + uu) + e;
          const int key = j < K ? static_cast<int>(sel_key(q[uu], e)) : -1;
          const bool take = key > kt || (key == kt && eq_b < r);
          if (take) list[gt_b + min(eq_b, r)] = j;
          if (flags != nullptr && j < K) flags[j] = take ? 1 : 0;
          gt_b += key > kt;
          eq_b += key == kt;
        }
  }
  if (tid == 0) {
    const int taken = tau >= 0 ? (total >> 16) + min(total & 0xFFFF, r) : 0;
    info[5] = bad ? -1 : taken;
    info[6] = taken;  // entries written to list, also when the row is bad
  }
  __syncthreads();
}

// The selection with the block's own scratch (static shared memory), for
// blocks of up to 1024 threads over one row: xs as above; flags: K bytes of
// shared scratch (used only when act is given).  Writes idx[0..n) ascending
// and *n_out (-1 if the row holds a NaN or Inf) to global memory, and the
// prepared activations of the batch-1 GEMV (act.cuh) to act when it is not
// null.  Same radix passes as select_row_cta, with one histogram row per warp
// and each thread walking one contiguous chunk of channels throughout.
__device__ inline void select_row_block(const uint16_t* xs, uint8_t* flags, int K, int k, int32_t* idx,
                                        int32_t* n_out, uint32_t* act) {
  constexpr int kMaxWarps = 32;
  __shared__ int whist[kMaxWarps][256];
  __shared__ int hist[256];
  __shared__ int scan_scratch[33];
  __shared__ int info[8];
  __shared__ int eg[kSelRowMaxK / 128];
  __shared__ float ginfo[2 * (kSelRowMaxK / 128)];
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5, nw = nthr >> 5;
  // contiguous chunks per thread (the ordered pass below walks them in order)
  const int chunk = (K + nthr - 1) / nthr;
  const int j0 = min(K, tid * chunk), j1 = min(K, j0 + chunk);
  int mybad = 0;
  if (k <= 0) {
    for (int j = j0; j < j1; ++j) mybad |= (xs[j] & 0x7F80u) == 0x7F80u;
    if (act != nullptr)
      for (int j = tid; j < K; j += nthr) flags[j] = 0;
    const int bad = __syncthreads_or(mybad);
    if (tid == 0) *n_out = bad ? -1 : 0;
    if (act != nullptr) act2_write_block(xs, flags, K, eg, ginfo, scan_scratch, act);
    return;
  }
  // pass 1: high byte
  for (int b = lane; b < 256; b += 32) whist[warp][b] = 0;
  __syncwarp();
  for (int j = j0; j < j1; ++j) {
    const uint32_t v = xs[j];
    mybad |= (v & 0x7F80u) == 0x7F80u;
    atomicAdd(&whist[warp][(v & 0x7FFFu) >> 7], 1);
  }
  const int bad = __syncthreads_or(mybad);
  for (int b = tid; b < 256; b += nthr) {
    int c = 0;
    for (int w = 0; w < nw; ++w) c += whist[w][b];
    hist[b] = c;
  }
  __syncthreads();
  if (warp == 0) sel_find_bin<256>(hist, k, info + 1);  // info[1] = b1, info[2] = k1
  // pass 2: low 7 bits inside bin b1
  for (int b = lane; b < 128; b += 32) whist[warp][b] = 0;
  __syncthreads();
  const int b1 = info[1];
  if (b1 >= 0)
    for (int j = j0; j < j1; ++j) {
      const uint32_t v = xs[j] & 0x7FFFu;
      if (static_cast<int>(v >> 7) == b1) atomicAdd(&whist[warp][v & 0x7Fu], 1);
    }
  __syncthreads();
  for (int b = tid; b < 128; b += nthr) {
    int c = 0;
    for (int w = 0; w < nw; ++w) c += whist[w][b];
    hist[b] = c;
  }
  __syncthreads();
  if (warp == 0) {
    if (b1 >= 0) {
      sel_find_bin<128>(hist, info[2], info + 3);
      __syncwarp();
      if (lane == 0 && info[3] >= 0) info[3] |= b1 << 7;
    } else if (lane == 0) {
      info[3] = -1;
      info[4] = 0;
    }
  }
  __syncthreads();
  // ordered pass, as in select_row_cta
  const int tau = info[3], r = info[4];
  int gt = 0, eq = 0;
  if (tau >= 0)
    for (int j = j0; j < j1; ++j) {
      const int key = xs[j] & 0x7FFF;
      gt += key > tau;
      eq += key == tau;
    }
  int total;
  const int pre = block_exclusive_scan((gt << 16) | eq, scan_scratch, &total);  // K <= 32768 fits 16 bits
  int gt_b = pre >> 16, eq_b = pre & 0xFFFF;
  for (int j = j0; j < j1; ++j) {
    const int key = xs[j] & 0x7FFF;
    const bool take = tau >= 0 && (key > tau || (key == tau && eq_b < r));
    if (take) idx[gt_b + min(eq_b, r)] = j;
    if (act != nullptr) flags[j] = take ? 1 : 0;
    gt_b += key > tau;
    eq_b += key == tau;
  }
  if (tid == 0) *n_out = bad ? -1 : (tau >= 0 ? (total >> 16) + min(total & 0xFFFF, r) : 0);
  if (act != nullptr) {
    __syncthreads();
    act2_write_block(xs, flags, K, eg, ginfo, scan_scratch, act);
  }
}

}  // namespace sfd
