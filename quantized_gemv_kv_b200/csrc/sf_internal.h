// Internal helpers shared by the CUDA translation units of libsf.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include <cstdint>
#include <cstdio>
#include <string>

#include "sf.h"

namespace sf {

// Thread-local last error message (set on every non-OK return).
void set_error(const std::string& msg);
sf_status fail(sf_status st, const char* fmt, ...);
sf_status cuda_fail(cudaError_t e, const char* what);

inline cudaStream_t as_cuda(sf_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

#define SF_CHECK_CUDA(call)                                 \
  do {                                                      \
    cudaError_t e__ = (call);                               \
    if (e__ != cudaSuccess) return ::sf::cuda_fail(e__, #call); \
  } while (0)

#define SF_REQUIRE(cond, ...)                                   \
  do {                                                          \
    if (!(cond)) return ::sf::fail(SF_EINVAL, __VA_ARGS__);     \
  } while (0)

// After a kernel launch: report launch-configuration errors.
inline sf_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return SF_OK;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Number of SMs of the current device (cached per device).
int sm_count();

// Device view of a refinement cache for the GEMV: where the rows live and
// which row serves each selected position of the last prefetch.
struct CacheView {
  const uint32_t* rows;     // [(capacity + max_select)][unit_words]
  const int32_t* row_of;    // [max_select]
  const int32_t* unit_slot; // [num_units]: slot of a cached unit, -1 if not cached
  int num_units;
  int unit_words;
  int max_select;
};
// For a GEMV: refuses a cache with a fetch budget (every selected column must
// be fetched); makes `stream` wait for the last prefetch.
sf_status cache_view_for_gemv(sf_refine_cache* c, cudaStream_t stream, CacheView* v);
// For a reader that looks units up by unit_slot (the cached set as the last
// prefetch left it); makes `stream` wait for that prefetch.
sf_status cache_view_for_reader(sf_refine_cache* c, cudaStream_t stream, CacheView* v);
sf_status cache_mark_used(sf_refine_cache* c, cudaStream_t stream);
// Whether the cache is read in the deadline reading (sf_refine_cache_set_deadline).
bool cache_deadline(const sf_refine_cache* c);

// For a writer of units (the KV append): the host master's device-mapped
// address and the device rows, so a new unit's bytes go to both; makes
// `stream` wait for the last prefetch.
struct CacheWriteView {
  uint32_t* master;          // device address of the host master [num_units][unit_words]
  uint32_t* rows;            // cache rows
  const int32_t* unit_slot;  // [num_units]
  int num_units;
  int unit_words;
};
sf_status cache_view_for_writer(sf_refine_cache* c, cudaStream_t stream, CacheWriteView* v);
// A writer's device staging area of at least `words` words (allocated on the
// first call, which must not be under stream capture); makes `stream` wait
// for the last flush of the staging area when that flush is visible to it.
sf_status cache_append_stage(sf_refine_cache* c, cudaStream_t stream, size_t words, uint32_t** stage);
// Copies `height` rows of `width` bytes from the staging area (packed) to the
// host master at byte offset dst_off with pitch dpitch, on `side` after the
// work enqueued so far on `stream` (side == stream: in order).
sf_status cache_append_flush(sf_refine_cache* c, cudaStream_t stream, cudaStream_t side, size_t dst_off,
                             size_t dpitch, size_t width, int height);

// Batch 2-16 GEMV on the tensor cores (gemv_tc.cu).
// Returns false when the shape is outside that kernel's range (the caller
// then runs the CUDA-core kernel); otherwise launches it and reports through
// *st.
bool gemv_tc_try(const sf_qweight* W, const uint16_t* x, int B, const int32_t* idx, const int32_t* n,
                 const uint32_t* ref_rows, const int32_t* row_of, int unit_words, float* y, cudaStream_t s,
                 sf_status* st);

// Batch-1 2-bit GEMV on the integer dot-product path (gemv_b1.cu).  Returns
// false when the shape is outside that kernel's range (the caller then runs
// the generic kernel); otherwise launches it and reports through *st.
bool gemv_b1_try(const sf_qweight* W, const uint16_t* x, const int32_t* idx, const int32_t* n,
                 const uint32_t* ref_rows, const int32_t* row_of, int unit_words, int nmax, float* y,
                 cudaStream_t s, sf_status* st);

}  // namespace sf

// -------- device helpers ------------------------------------------------
namespace sfd {

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

// Read `bits` bits starting at stream bit `pos` of a little-endian uint32
// bitstream (bits <= 8; may straddle a word boundary).
__device__ __forceinline__ uint32_t read_bits(const uint32_t* s, uint32_t pos, int bits) {
  uint32_t w = pos >> 5, sh = pos & 31;
  uint64_t v = s[w];
  if (sh + bits > 32) v |= static_cast<uint64_t>(s[w + 1]) << 32;
  return static_cast<uint32_t>(v >> sh) & ((1u << bits) - 1u);
}

}  // namespace sfd
