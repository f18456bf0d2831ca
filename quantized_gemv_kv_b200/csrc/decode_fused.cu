// Producer + selection in one launch for the batch-1 decode step: the op that
// makes a GEMV's input row (residual add and RMSNorm, the bf16 rounding of
// the attention output, the SiLU-gated product of the MLP) runs in the same
// thread block as the top-k channel selection of that row and the prepared
// activations of the tensor-core GEMV, so the row never leaves the block
// between the two and one launch replaces two on the step's critical path.
// The arithmetic of each producer is that of its stand-alone entry point in
// decode_ops.cu (fp64, one rounding to bf16 with ties to even); the selection
// is select_row_block (ties to the lower channel).  Also here: RoPE of the
// query and key heads in one launch.
#include <cuda_bf16.h>

#include "produce.cuh"
#include "select_row.cuh"
#include "sf_internal.h"

namespace {

constexpr int kThreads = sfd::kNormVThreads;  // the RMSNorm sum order is that of 1024 threads

using sfd::silu_mul_bf16;
using sfd::to_bf16;

// Writes the producer's row to xs (shared) and y (global), then selects.
enum Producer { kNorm = 0, kRound = 1, kSilu = 2 };

struct FusedArgs {
  int op, K, k;
  float eps;
  float* x;            // kNorm: residual, updated by += delta
  const float* delta;  // kNorm: may be null
  const float* w;      // kNorm: RMSNorm weights
  const float* a;      // kRound: the fp32 row; kSilu: the gate
  const float* b;      // kSilu: the up projection
  uint16_t* y;         // the bf16 row (the GEMV's x)
  int32_t* idx;
  int32_t* n;
  uint32_t* act;
};

__global__ void __launch_bounds__(kThreads) produce_select_kernel(const __grid_constant__ FusedArgs A) {
  // a GEMV launched after this kernel with programmatic stream serialization
  // may start streaming its weight codes now; it waits for this grid before
  // it reads the row or the selection
  asm volatile("griddepcontrol.launch_dependents;\n" ::);
  extern __shared__ __align__(16) uint8_t smem[];
  const int K = A.K, tid = threadIdx.x;
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);  // [K]
  uint8_t* flags = smem + 2 * K;                     // [K]
  if (A.op == kNorm) {
    __shared__ double part[kThreads / 32];
    __shared__ double inv_sh;
    // up to kPer entries of x, delta and w per thread in registers, every
    // load in flight; longer rows take a second sweep over x and w
    constexpr int kPer = 8;
    const bool in_regs = K <= kPer * kThreads;
    float xv[kPer], wv[kPer];
    double ss = 0.0;
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = tid + j * kThreads;
        xv[j] = i < K ? A.x[i] : 0.0f;
        wv[j] = i < K ? A.w[i] : 0.0f;
        if (A.delta && i < K) xv[j] = __fadd_rn(xv[j], A.delta[i]);
      }
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = tid + j * kThreads;
        if (i < K) {
          if (A.delta) A.x[i] = xv[j];
          ss = fma(static_cast<double>(xv[j]), static_cast<double>(xv[j]), ss);
        }
      }
    } else {
      for (int i = tid; i < K; i += kThreads) {
        float v = A.x[i];
        if (A.delta) {
          v = __fadd_rn(v, A.delta[i]);
          A.x[i] = v;
        }
        ss = fma(static_cast<double>(v), static_cast<double>(v), ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((tid & 31) == 0) part[tid >> 5] = ss;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int i = 0; i < kThreads / 32; ++i) t += part[i];
      inv_sh = 1.0 / sqrt(t / K + static_cast<double>(A.eps));
    }
    __syncthreads();
    const double inv = inv_sh;
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = tid + j * kThreads;
        if (i < K) {
          const uint16_t v = to_bf16(static_cast<double>(xv[j]) * inv * static_cast<double>(wv[j]));
          xs[i] = v;
          A.y[i] = v;
        }
      }
    } else {
      for (int i = tid; i < K; i += kThreads) {
        const uint16_t v = to_bf16(static_cast<double>(A.x[i]) * inv * static_cast<double>(A.w[i]));
        xs[i] = v;
        A.y[i] = v;
      }
    }
  } else if (A.op == kRound) {
    constexpr int kPer = 16;
    for (int i0 = 0; i0 < K; i0 += kPer * kThreads) {
      float av[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = i0 + tid + j * kThreads;
        av[j] = i < K ? A.a[i] : 0.0f;
      }
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = i0 + tid + j * kThreads;
        if (i < K) {
          const uint16_t v = __bfloat16_as_ushort(__float2bfloat16_rn(av[j]));
          xs[i] = v;
          A.y[i] = v;
        }
      }
    }
  } else {
    // eight entries of g and u per thread in flight at a time
    constexpr int kPer = 8;
    for (int i0 = 0; i0 < K; i0 += kPer * kThreads) {
      float gv[kPer], uv[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = i0 + tid + j * kThreads;
        gv[j] = i < K ? A.a[i] : 0.0f;
        uv[j] = i < K ? A.b[i] : 0.0f;
      }
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = i0 + tid + j * kThreads;
        if (i < K) {
          const uint16_t v = silu_mul_bf16(gv[j], uv[j]);
          xs[i] = v;
          A.y[i] = v;
        }
      }
    }
  }
  __syncthreads();
  sfd::select_row_block(xs, flags, K, A.k, A.idx, A.n, A.act);
}

// One block per head: q heads [0, Hq) rotated in place and written as bf16,
// k heads [Hq, Hq + Hkv) rotated in place; a thread per pair (i, i + d/2).
__global__ void rope_qk_kernel(float* __restrict__ q, int Hq, float* __restrict__ kk, int d, int pos, double theta,
                               uint16_t* __restrict__ q_bf16) {
  const int half = d >> 1, i = threadIdx.x;
  if (i >= half) return;
  const bool is_q = static_cast<int>(blockIdx.x) < Hq;
  float* xh = is_q ? q + static_cast<size_t>(blockIdx.x) * d : kk + static_cast<size_t>(blockIdx.x - Hq) * d;
  double rlo, rhi;
  sfd::rope_pair(xh[i], xh[i + half], i, d, pos, theta, rlo, rhi);
  xh[i] = static_cast<float>(rlo);
  xh[i + half] = static_cast<float>(rhi);
  if (is_q && q_bf16) {
    uint16_t* yh = q_bf16 + static_cast<size_t>(blockIdx.x) * d;
    yh[i] = to_bf16(rlo);
    yh[i + half] = to_bf16(rhi);
  }
}

sf_status launch_fused(const FusedArgs& A, cudaStream_t s, const char* what) {
  SF_REQUIRE(A.y && A.idx && A.n, "%s: null pointer", what);
  SF_REQUIRE(A.K >= 256 && A.K % 256 == 0 && A.K <= sfd::kSelRowMaxK,
             "%s: K must be a multiple of 256 up to %d", what, sfd::kSelRowMaxK);
  SF_REQUIRE(A.k >= 0 && A.k <= A.K, "%s: k must be in [0, K]", what);
  SF_REQUIRE(!A.act || sf::aligned(A.act, 16), "%s: act must be 16-byte aligned", what);
  const size_t smem = 3 * static_cast<size_t>(A.K);
  SF_CHECK_CUDA(cudaFuncSetAttribute(produce_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)));
  produce_select_kernel<<<1, kThreads, smem, s>>>(A);
  return sf::check_launch("produce_select_kernel");
}

}  // namespace

extern "C" sf_status sf_norm_select(float* x, const float* delta, const float* w, int H, float eps, uint16_t* y,
                                    int k, int32_t* idx_out, int32_t* n_out, void* act, sf_stream_t stream) {
  SF_REQUIRE(x && w, "sf_norm_select: null pointer");
  SF_REQUIRE(eps >= 0.0f, "sf_norm_select: eps must be >= 0");
  FusedArgs A{};
  A.op = kNorm;
  A.K = H;
  A.k = k;
  A.eps = eps;
  A.x = x;
  A.delta = delta;
  A.w = w;
  A.y = y;
  A.idx = idx_out;
  A.n = n_out;
  A.act = static_cast<uint32_t*>(act);
  return launch_fused(A, sf::as_cuda(stream), "sf_norm_select");
}

extern "C" sf_status sf_round_select(const float* a, int K, uint16_t* y, int k, int32_t* idx_out, int32_t* n_out,
                                     void* act, sf_stream_t stream) {
  SF_REQUIRE(a, "sf_round_select: null pointer");
  FusedArgs A{};
  A.op = kRound;
  A.K = K;
  A.k = k;
  A.a = a;
  A.y = y;
  A.idx = idx_out;
  A.n = n_out;
  A.act = static_cast<uint32_t*>(act);
  return launch_fused(A, sf::as_cuda(stream), "sf_round_select");
}

extern "C" sf_status sf_silu_mul_select(const float* g, const float* u, int K, uint16_t* y, int k, int32_t* idx_out,
                                        int32_t* n_out, void* act, sf_stream_t stream) {
  SF_REQUIRE(g && u, "sf_silu_mul_select: null pointer");
  FusedArgs A{};
  A.op = kSilu;
  A.K = K;
  A.k = k;
  A.a = g;
  A.b = u;
  A.y = y;
  A.idx = idx_out;
  A.n = n_out;
  A.act = static_cast<uint32_t*>(act);
  return launch_fused(A, sf::as_cuda(stream), "sf_silu_mul_select");
}

extern "C" sf_status sf_rope_qk(float* q, int Hq, float* k, int Hkv, int d, int pos, double theta, uint16_t* q_bf16,
                                sf_stream_t stream) {
  SF_REQUIRE(q && k, "sf_rope_qk: null pointer");
  SF_REQUIRE(Hq >= 1 && Hkv >= 0 && d >= 2 && d % 2 == 0 && d <= 2048 && pos >= 0 && theta > 0.0,
             "sf_rope_qk: need Hq >= 1, Hkv >= 0, d even in [2, 2048], pos >= 0, theta > 0");
  rope_qk_kernel<<<Hq + Hkv, d / 2, 0, sf::as_cuda(stream)>>>(q, Hq, k, d, pos, theta, q_bf16);
  return sf::check_launch("rope_qk_kernel");
}
