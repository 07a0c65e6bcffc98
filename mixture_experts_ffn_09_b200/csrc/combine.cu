// Weighted combine: out[t, :] = sum_k w[t, k] * Y[pos[t, k], :].
//
// "Mixture-of-Experts FFN" (crackedaicode.com Flax exercise), section
// "Weight the selected outputs": each token sums its own K selected expert
// outputs weighted by its routing weights.  Y holds one row per (token,
// slot) in expert order; pos maps a slot to its row.  Each output element
// is written exactly once, the K terms are summed in fp32 in slot order and
// rounded once to the output dtype: no atomics, bitwise repeatable.
//
// HBM-bound gather: one CTA per (token, 1024 x C-column chunk), 16-byte
// loads and stores, so small batches still spread over the SMs.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 128;

// Slots are read in batches of kBatch: all loads of a batch are issued
// before the first is used, so each thread keeps several rows in flight.
constexpr int kBatch = 8;

// A thread handles C 8-column chunks, kThreads * 8 columns apart (so each
// warp's loads stay coalesced), and issues the loads of all its chunks for
// a batch of slots before using any: with few slots (K = 2 on the Mixtral
// layer) that keeps C * K rows in flight instead of K.
template <int C>
__global__ void __launch_bounds__(kThreads) combine_bf16_kernel(const __nv_bfloat16* __restrict__ Y,
                                                                const float* __restrict__ w,
                                                                const int* __restrict__ pos, int K,
                                                                int D,
                                                                __nv_bfloat16* __restrict__ out) {
  constexpr int kB = kBatch / C > 0 ? kBatch / C : 1;    // slots per batch
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
  const int d0 = blockIdx.y * (kThreads * 8 * C) + threadIdx.x * 8;
  float acc[C][8];
#pragma unroll
  for (int c = 0; c < C; ++c)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[c][i] = 0.f;
  for (int k0 = 0; k0 < K; k0 += kB) {
    uint4 q[C][kB];
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      const int k = k0 + j;
      if (k < K && sp[k] >= 0) {
        const __nv_bfloat16* row = Y + static_cast<size_t>(sp[k]) * D;
#pragma unroll
        for (int c = 0; c < C; ++c) {
          const int d = d0 + c * kThreads * 8;
          if (d < D) q[c][j] = __ldg(reinterpret_cast<const uint4*>(row + d));
        }
      }
    }
    // accumulate in slot order; a dropped slot adds nothing
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      const int k = k0 + j;
      if (k < K && sp[k] >= 0) {
        const float wk = sw[k];
#pragma unroll
        for (int c = 0; c < C; ++c) {
          if (d0 + c * kThreads * 8 >= D) continue;
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q[c][j]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h[i]);
            acc[c][2 * i] = fmaf(wk, f.x, acc[c][2 * i]);
            acc[c][2 * i + 1] = fmaf(wk, f.y, acc[c][2 * i + 1]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int c = 0; c < C; ++c) {
    const int d = d0 + c * kThreads * 8;
    if (d < D) {
      uint4 o;
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[c][2 * i], acc[c][2 * i + 1]);
      *reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * D + d) = o;
    }
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
    // chunks per thread: about kBatch rows in flight whatever K is, as long
    // as the grid still has a few CTAs per SM (a decode step has 32 tokens)
    int C = K <= 2 ? 4 : (K <= 4 ? 2 : 1);
    while (C > 1 && static_cast<long long>(T) * ((D + kThreads * 8 * C - 1) / (kThreads * 8 * C)) <
                        4LL * num_sms())
      C >>= 1;
    const dim3 g(T, (D + kThreads * 8 * C - 1) / (kThreads * 8 * C));
    const auto* Yb = static_cast<const __nv_bfloat16*>(Y);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    if (C == 4)
      return launch_k(combine_bf16_kernel<4>, g, dim3(kThreads), 0, s, pdl_enabled(), 1, Yb, w32, pos,
                      K, D, ob);
    if (C == 2)
      return launch_k(combine_bf16_kernel<2>, g, dim3(kThreads), 0, s, pdl_enabled(), 1, Yb, w32, pos,
                      K, D, ob);
    return launch_k(combine_bf16_kernel<1>, g, dim3(kThreads), 0, s, pdl_enabled(), 1, Yb, w32, pos,
                    K, D, ob);
  } else {
    return launch_k(combine_f32_kernel, grid, dim3(kThreads), 0, s, pdl_enabled(), 1,
                    static_cast<const float*>(Y), w32, pos, K, D, static_cast<float*>(out));
  }
  return cudaGetLastError();
}

}  // namespace moe
