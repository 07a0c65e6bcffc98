// float32 grouped GEMMs on the CUDA cores, for the float32 path.
//
// Experts of "Mixture-of-Experts FFN" (crackedaicode.com, "Compute the
// experts and router": Dense(F) -> ReLU -> Dense(D) with biases) and of
// mojolearn.MoEBlock (down_proj(silu(gate) * up), HF layout).  The float32
// path keeps true fp32 products and sums (fmaf): TF32 tensor cores round the
// operands to 10 mantissa bits, which cannot hold a 1e-4 relative bound.
//
// Grid (row tiles, N tiles, experts); a CTA whose row tile lies past its
// expert's row count exits at once.  32 x 32 output tile, 16 x 16 threads,
// 2 x 2 outputs per thread, K staged through shared memory in steps of 32.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BT = 32;

template <int ACT>
__global__ void __launch_bounds__(256) gemm_simt_f32_kernel(const float* __restrict__ A,
                                                            const float* __restrict__ W,
                                                            const int* __restrict__ offsets,
                                                            int Kdim, int N, int w_rows,
                                                            const float* __restrict__ bias,
                                                            float* __restrict__ C) {
  __shared__ float As[BT][BT + 1];
  __shared__ float Gs[BT][BT + 1];
  __shared__ float Us[ACT == 0 ? BT : 1][BT + 1];
  pdl_trigger();
  pdl_wait();
  const int e = blockIdx.z;
  const int r0 = offsets[e];
  const int cnt = offsets[e + 1] - r0;
  const int m0 = blockIdx.x * BT;
  if (m0 >= cnt) return;
  const int n0 = blockIdx.y * BT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float* We = W + static_cast<size_t>(e) * w_rows * Kdim;

  float g[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  float u[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  for (int k0 = 0; k0 < Kdim; k0 += BT) {
    for (int i = threadIdx.x; i < BT * BT; i += 256) {
      const int r = i / BT, kk = i % BT;
      const int k = k0 + kk;
      As[r][kk] = (m0 + r < cnt && k < Kdim) ? A[static_cast<size_t>(r0 + m0 + r) * Kdim + k] : 0.f;
      Gs[r][kk] = (n0 + r < N && k < Kdim) ? We[static_cast<size_t>(n0 + r) * Kdim + k] : 0.f;
      if (ACT == 0)
        Us[r][kk] = (n0 + r < N && k < Kdim) ? We[static_cast<size_t>(N + n0 + r) * Kdim + k] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < BT; ++kk) {
      const float a0 = As[ty * 2][kk], a1 = As[ty * 2 + 1][kk];
      const float b0 = Gs[tx * 2][kk], b1 = Gs[tx * 2 + 1][kk];
      g[0][0] = fmaf(a0, b0, g[0][0]);
      g[0][1] = fmaf(a0, b1, g[0][1]);
      g[1][0] = fmaf(a1, b0, g[1][0]);
      g[1][1] = fmaf(a1, b1, g[1][1]);
      if (ACT == 0) {
        const float c0 = Us[tx * 2][kk], c1 = Us[tx * 2 + 1][kk];
        u[0][0] = fmaf(a0, c0, u[0][0]);
        u[0][1] = fmaf(a0, c1, u[0][1]);
        u[1][0] = fmaf(a1, c0, u[1][0]);
        u[1][1] = fmaf(a1, c1, u[1][1]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = m0 + ty * 2 + i;
    if (r >= cnt) continue;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int c = n0 + tx * 2 + j;
      if (c >= N) continue;
      float h;
      if (ACT == 0) {
        const float z = g[i][j];
        h = z / (1.f + expf(-z)) * u[i][j];
      } else if (ACT == 1) {
        h = fmaxf(g[i][j] + bias[static_cast<size_t>(e) * N + c], 0.f);
      } else {
        h = g[i][j] + (bias ? bias[static_cast<size_t>(e) * N + c] : 0.f);
      }
      C[static_cast<size_t>(r0 + r) * N + c] = h;
    }
  }
}

}  // namespace

cudaError_t launch_gemm_simt_f32(int act, const float* A, const float* W, const int* offsets, int E,
                                 int T, int Kdim, int N, int w_rows_per_expert, const float* bias,
                                 float* C, cudaStream_t s) {
  const dim3 grid((T + BT - 1) / BT, (N + BT - 1) / BT, E);
  if (act == 0)
    return launch_k(gemm_simt_f32_kernel<0>, grid, dim3(256), 0, s, pdl_enabled(), 1, A, W, offsets,
                    Kdim, N, w_rows_per_expert, bias, C);
  else if (act == 1)
    return launch_k(gemm_simt_f32_kernel<1>, grid, dim3(256), 0, s, pdl_enabled(), 1, A, W, offsets,
                    Kdim, N, w_rows_per_expert, bias, C);
  else
    return launch_k(gemm_simt_f32_kernel<2>, grid, dim3(256), 0, s, pdl_enabled(), 1, A, W, offsets,
                    Kdim, N, w_rows_per_expert, bias, C);
  return cudaGetLastError();
}

}  // namespace moe
