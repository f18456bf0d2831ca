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
// caller); flags: K bytes of shared scratch (used only when act is given).
// Writes idx[0..n) ascending and *n_out (-1 if the row holds a NaN or Inf),
// and the prepared form to act when it is not null.  All threads of the block
// call; blockDim.x is a multiple of 32 up to 1024.
//
// Two radix passes with warp-private histograms (no atomics between warps):
// the high byte of the key (the bf16 exponent), then its low 7 bits inside
// the bin holding the k-th key; then one block scan of packed (above, tied)
// counts over contiguous chunks gives every selected channel its position
// directly, ties taken in ascending channel order.
__device__ inline void select_row_block(const uint16_t* xs, uint8_t* flags, int K, int k, int32_t* idx,
                                        int32_t* n_out, uint32_t* act) {
  constexpr int kMaxWarps = 32;
  __shared__ int whist[kMaxWarps][256];
  __shared__ int hist[256];
  __shared__ int scan_scratch[33];
  __shared__ int b1_sh, k1_sh, tau_sh, r_sh, bad;
  __shared__ int eg[kSelRowMaxK / 128];
  __shared__ float ginfo[2 * (kSelRowMaxK / 128)];
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5, nw = nthr >> 5;
  if (tid == 0) bad = 0;
  // contiguous chunks per thread (the ordered pass below walks them in order)
  const int chunk = (K + nthr - 1) / nthr;
  const int j0 = min(K, tid * chunk), j1 = min(K, j0 + chunk);
  if (k <= 0) {
    if (tid == 0) *n_out = 0;
    for (int j = j0; j < j1; ++j)
      if ((xs[j] & 0x7F80u) == 0x7F80u) bad = 1;
    __syncthreads();
    if (tid == 0 && bad) *n_out = -1;
    if (act != nullptr) {
      for (int j = tid; j < K; j += nthr) flags[j] = 0;
      __syncthreads();
      act2_write_block(xs, flags, K, eg, ginfo, scan_scratch, act);
    }
    return;
  }
  // pass 1: high byte
  for (int b = lane; b < 256; b += 32) whist[warp][b] = 0;
  __syncwarp();
  for (int j = j0; j < j1; ++j) {
    const uint32_t v = xs[j];
    if ((v & 0x7F80u) == 0x7F80u) bad = 1;
    atomicAdd(&whist[warp][(v & 0x7FFFu) >> 7], 1);
  }
  __syncthreads();
  for (int b = tid; b < 256; b += nthr) {
    int c = 0;
    for (int w = 0; w < nw; ++w) c += whist[w][b];
    hist[b] = c;
  }
  __syncthreads();
  if (warp == 0) {
    int above = 0, b1 = -1, k1 = 0;
    for (int base = 255; base >= 0 && b1 < 0; base -= 32) {
      const int c = hist[base - lane];
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned m = __ballot_sync(0xffffffffu, above + incl >= k && above + incl - c < k);
      if (m) {
        const int src = __ffs(m) - 1;
        b1 = base - src;
        k1 = k - (above + __shfl_sync(0xffffffffu, incl - c, src));
      }
      above += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) { b1_sh = b1; k1_sh = k1; }
  }
  // pass 2: low 7 bits inside bin b1
  for (int b = lane; b < 128; b += 32) whist[warp][b] = 0;
  __syncthreads();
  const int b1 = b1_sh;
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
    const int kk = k1_sh;
    int above = 0, tau = -1, r = 0;
    if (b1 >= 0) {
      for (int base = 127; base >= 0 && tau < 0; base -= 32) {
        const int c = hist[base - lane];
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
  // ordered pass: channel j is taken if key > tau, or key == tau and fewer
  // than r keys equal to tau precede it; its position is the number of taken
  // channels before it = (keys > tau before j) + min(ties before j, r)
  const int tau = tau_sh, r = r_sh;
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
  if (tau >= 0)
    for (int j = j0; j < j1; ++j) {
      const int key = xs[j] & 0x7FFF;
      const bool take = key > tau || (key == tau && eq_b < r);
      if (take) idx[gt_b + min(eq_b, r)] = j;
      if (act != nullptr) flags[j] = take ? 1 : 0;
      gt_b += key > tau;
      eq_b += key == tau;
    }
  if (tid == 0) *n_out = bad ? -1 : (total >> 16) + min(total & 0xFFFF, r);
  if (act != nullptr) {
    __syncthreads();
    act2_write_block(xs, flags, K, eg, ginfo, scan_scratch, act);
  }
}

}  // namespace sfd
