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

// Histogram increment with the lanes of a warp that hit the same bin merged
// into one atomic (keys cluster in few bins, so plain atomics serialise).
// bin < 0 means "no increment".  Call with the whole warp.
__device__ __forceinline__ void sel_hist_add(int* hist, int bin) {
  const unsigned peers = __match_any_sync(0xffffffffu, bin);
  const int leader = __ffs(peers) - 1;
  if (bin >= 0 && (threadIdx.x & 31) == leader) atomicAdd(&hist[bin], __popc(peers));
}

// xs: the row's K bf16 bits (shared memory, written and synchronized by the
// caller); flags: K bytes of shared scratch.  Writes idx[0..n) ascending and
// *n_out (-1 if the row holds a NaN or Inf), and the prepared form to act
// when it is not null.  All threads of the block call; blockDim.x is a
// multiple of 32 up to 1024.
__device__ inline void select_row_block(const uint16_t* xs, uint8_t* flags, int K, int k, int32_t* idx,
                                        int32_t* n_out, uint32_t* act) {
  __shared__ int hist1[256], hist2[128];
  __shared__ int scan_scratch[33];
  __shared__ int b1_sh, k1_sh, tau_sh, r_sh, bad;
  __shared__ int eg[kSelRowMaxK / 128];
  __shared__ float ginfo[2 * (kSelRowMaxK / 128)];
  const int tid = threadIdx.x, nthr = blockDim.x;
  for (int j = tid; j < K; j += nthr) flags[j] = 0;
  for (int j = tid; j < 256; j += nthr) hist1[j] = 0;
  for (int j = tid; j < 128; j += nthr) hist2[j] = 0;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int j0 = 0; j0 < K; j0 += nthr) {  // uniform trip count: whole warps call sel_hist_add
    const int j = j0 + tid;
    int bin = -1;
    if (j < K) {
      const uint32_t v = xs[j];
      if ((v & 0x7F80u) == 0x7F80u) bad = 1;
      bin = static_cast<int>((v & 0x7FFFu) >> 7);
    }
    sel_hist_add(hist1, bin);
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  if (warp == 0) {
    int above = 0, b1 = -1, k1 = 0;
    for (int base = 255; base >= 0 && b1 < 0; base -= 32) {
      const int c = hist1[base - lane];
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned m = __ballot_sync(0xffffffffu, k > 0 && above + incl >= k && above + incl - c < k);
      if (m) {
        const int src = __ffs(m) - 1;
        b1 = base - src;
        k1 = k - (above + __shfl_sync(0xffffffffu, incl - c, src));
      }
      above += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) { b1_sh = b1; k1_sh = k1; }
  }
  __syncthreads();
  const int b1 = b1_sh;
  if (b1 >= 0)
    for (int j0 = 0; j0 < K; j0 += nthr) {
      const int j = j0 + tid;
      int bin = -1;
      if (j < K) {
        const uint32_t v = xs[j] & 0x7FFFu;
        if (static_cast<int>(v >> 7) == b1) bin = static_cast<int>(v & 0x7Fu);
      }
      sel_hist_add(hist2, bin);
    }
  __syncthreads();
  if (warp == 0) {
    const int kk = k1_sh;
    int above = 0, tau = -1, r = 0;
    if (b1 >= 0) {
      for (int base = 127; base >= 0 && tau < 0; base -= 32) {
        const int c = hist2[base - lane];
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const unsigned m = __ballot_sync(0xffffffffu, above + incl >= kk && above + incl - c < kk);
        if (m) {
          const int src = __ffs(m) - 1;
          tau = (b1 << 7) | (base - src);
          r = kk - (above + __shfl_sync(0xffffffffu, incl - c, src));
        }
        above += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    if (lane == 0) { tau_sh = tau; r_sh = r; }
  }
  __syncthreads();
  const int tau = tau_sh;
  // ordered tie pass over contiguous chunks, then the compaction
  const int chunk = (K + nthr - 1) / nthr;
  const int j0 = min(K, tid * chunk), j1 = min(K, j0 + chunk);
  {
    int eq = 0;
    if (tau >= 0)
      for (int j = j0; j < j1; ++j) eq += ((xs[j] & 0x7FFF) == tau);
    int total;
    int rank = block_exclusive_scan(eq, scan_scratch, &total);
    if (tau >= 0)
      for (int j = j0; j < j1; ++j) {
        const int key = xs[j] & 0x7FFF;
        if (key > tau) flags[j] = 1;
        else if (key == tau) { if (rank < r_sh) flags[j] = 1; ++rank; }
      }
  }
  __syncthreads();
  {
    int c = 0;
    for (int j = j0; j < j1; ++j) c += flags[j];
    int total;
    int pos = block_exclusive_scan(c, scan_scratch, &total);
    for (int j = j0; j < j1; ++j)
      if (flags[j]) idx[pos++] = j;
    if (tid == 0) *n_out = bad ? -1 : total;
  }
  __syncthreads();
  if (act != nullptr) act2_write_block(xs, flags, K, eg, ginfo, scan_scratch, act);
}

}  // namespace sfd
