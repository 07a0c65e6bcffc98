// Weighted combine: out[t, :] = sum_k w[t, k] * Y[pos[t, k], :].
//
// "Mixture-of-Experts FFN" (crackedaicode.com Flax exercise), section
// "Weight the selected outputs": each token sums its own K selected expert
// outputs weighted by its routing weights.  Y holds one row per (token,
// slot) in expert order; pos maps a slot to its row.  Each output element
// is written exactly once, the K terms are summed in fp32 in slot order and
// rounded once to the output dtype: no atomics, bitwise repeatable.
//
// HBM-bound gather: one CTA per (token, 1024-column chunk), 16-byte loads
// and stores, so small batches still spread over the SMs.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 128;

// Slots are read in batches of kBatch: all loads of a batch are issued
// before the first is used, so each thread keeps several rows in flight.
constexpr int kBatch = 8;

__global__ void __launch_bounds__(kThreads) combine_bf16_kernel(const __nv_bfloat16* __restrict__ Y,
                                                                const float* __restrict__ w,
                                                                const int* __restrict__ pos, int K,
                                                                int D,
                                                                __nv_bfloat16* __restrict__ out) {
  __shared__ int sp[kMaxExperts];
  __shared__ float sw[kMaxExperts];
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x;
  for (int k = threadIdx.x; k < K; k += kThreads) {
    sp[k] = pos[static_cast<size_t>(t) * K + k];
    sw[k] = w[static_cast<size_t>(t) * K + k];
  }
  __syncthreads();
  const int d_hi = min(D, static_cast<int>(blockIdx.y + 1) * kThreads * 8);
  for (int d = blockIdx.y * kThreads * 8 + threadIdx.x * 8; d < d_hi; d += kThreads * 8) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int k0 = 0; k0 < K; k0 += kBatch) {
      uint4 q[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int k = k0 + j;
        if (k < K && sp[k] >= 0)
          q[j] = __ldg(reinterpret_cast<const uint4*>(Y + static_cast<size_t>(sp[k]) * D + d));
      }
      // accumulate in slot order; a dropped slot adds nothing
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int k = k0 + j;
        if (k < K && sp[k] >= 0) {
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q[j]);
          const float wk = sw[k];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h[i]);
            acc[2 * i] = fmaf(wk, f.x, acc[2 * i]);
            acc[2 * i + 1] = fmaf(wk, f.y, acc[2 * i + 1]);
          }
        }
      }
    }
    uint4 o;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    *reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * D + d) = o;
  }
}

__global__ void __launch_bounds__(kThreads) combine_f32_kernel(const float* __restrict__ Y,
                                                               const float* __restrict__ w,
                                                               const int* __restrict__ pos, int K,
                                                               int D, float* __restrict__ out) {
  __shared__ int sp[kMaxExperts];
  __shared__ float sw[kMaxExperts];
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x;
  for (int k = threadIdx.x; k < K; k += kThreads) {
    sp[k] = pos[static_cast<size_t>(t) * K + k];
    sw[k] = w[static_cast<size_t>(t) * K + k];
  }
  __syncthreads();
  const int d_hi = min(D, static_cast<int>(blockIdx.y + 1) * kThreads * 8);
  for (int d = blockIdx.y * kThreads * 8 + threadIdx.x; d < d_hi; d += kThreads) {
    float acc = 0.f;
    for (int k0 = 0; k0 < K; k0 += kBatch) {
      float q[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int k = k0 + j;
        if (k < K && sp[k] >= 0) q[j] = __ldg(Y + static_cast<size_t>(sp[k]) * D + d);
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int k = k0 + j;
        if (k < K && sp[k] >= 0) acc = fmaf(sw[k], q[j], acc);
      }
    }
    out[static_cast<size_t>(t) * D + d] = acc;
  }
}

}  // namespace

cudaError_t launch_combine(const void* Y, const float* w32, const int* pos, int T, int K, int D,
                           int dt, void* out, cudaStream_t s) {
  const dim3 grid(T, (D + kThreads * 8 - 1) / (kThreads * 8));
  if (dt == kBF16) {
    return launch_k(combine_bf16_kernel, grid, dim3(kThreads), 0, s, pdl_enabled(), 1,
                    static_cast<const __nv_bfloat16*>(Y), w32, pos, K, D,
                    static_cast<__nv_bfloat16*>(out));
  } else {
    return launch_k(combine_f32_kernel, grid, dim3(kThreads), 0, s, pdl_enabled(), 1,
                    static_cast<const float*>(Y), w32, pos, K, D, static_cast<float*>(out));
  }
  return cudaGetLastError();
}

}  // namespace moe
