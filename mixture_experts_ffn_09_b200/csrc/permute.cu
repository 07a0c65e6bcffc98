// Expert permutation: sorts the (token, slot) pairs into expert order so the
// experts can run as one grouped matrix multiplication over contiguous rows
// ("Mixture of experts", dewml.dev, section "Expert computation and
// placement": tokens are sorted into expert order).
//
// The order is stable: rows of one expert are listed by (token, slot), so
// the result is deterministic and independent of scheduling.  Two kernels:
//   scan    - one CTA turns the router's per-block histograms into expert
//             offsets and each block's first row per expert;
//   scatter - each router block ranks its own slots within their expert
//             (warp match + per-warp counts), writes perm / pos, and copies
//             the token rows into the expert-sorted x_perm.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

__device__ __forceinline__ unsigned int lanemask_lt() {
  unsigned int m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) permute_scan_kernel(const int* __restrict__ bc,
                                                                    int B, int E,
                                                                    int* __restrict__ offsets,
                                                                    int* __restrict__ blockbase) {
  __shared__ int tot[kMaxExperts + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = warp; e < E; e += kScanThreads / 32) {
    int running = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      const int c = (b < B) ? bc[static_cast<size_t>(b) * E + e] : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      if (b < B) blockbase[static_cast<size_t>(b) * E + e] = running + incl - c;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) tot[e] = running;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      const int c = tot[e];
      tot[e] = acc;
      offsets[e] = acc;
      acc += c;
    }
    tot[E] = acc;
    offsets[E] = acc;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < B * E; i += kScanThreads) blockbase[i] += tot[i % E];
}

constexpr int kScatterThreads = 256;
constexpr int kScatterWarps = kScatterThreads / 32;

__global__ void __launch_bounds__(kScatterThreads) permute_scatter_kernel(
    const int* __restrict__ idx32, const int* __restrict__ blockbase, int T, int K, int E,
    const uint8_t* __restrict__ x, int row_bytes, int* __restrict__ perm, int* __restrict__ pos,
    uint8_t* __restrict__ x_perm) {
  __shared__ int run[kMaxExperts];
  __shared__ int wc[kScatterWarps][kMaxExperts];
  __shared__ int rowbuf[kScatterThreads];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += kScatterThreads) {
    run[e] = blockbase[static_cast<size_t>(b) * E + e];
#pragma unroll
    for (int w = 0; w < kScatterWarps; ++w) wc[w][e] = 0;
  }
  __syncthreads();

  const int t_lo = b * kRouterTokensPerCta;
  const int t_hi = min(T, t_lo + kRouterTokensPerCta);
  const int s_lo = t_lo * K, s_hi = t_hi * K;
  const bool vec = (row_bytes % 16) == 0;

  for (int c0 = s_lo; c0 < s_hi; c0 += kScatterThreads) {
    const int s = c0 + threadIdx.x;
    const bool valid = s < s_hi;
    const int e = valid ? idx32[s] : -1;
    const unsigned int mask = __match_any_sync(0xffffffffu, e);
    const int wrank = __popc(mask & lanemask_lt());
    if (valid && lane == __ffs(mask) - 1) wc[warp][e] = __popc(mask);
    __syncthreads();
    if (valid) {
      int r = run[e] + wrank;
      for (int w = 0; w < warp; ++w) r += wc[w][e];
      perm[r] = s;
      pos[s] = r;
      rowbuf[threadIdx.x] = r;
    }
    __syncthreads();
    for (int ee = threadIdx.x; ee < E; ee += kScatterThreads) {
      int add = 0;
#pragma unroll
      for (int w = 0; w < kScatterWarps; ++w) {
        add += wc[w][ee];
        wc[w][ee] = 0;
      }
      run[ee] += add;
    }
    // gather the token rows of this chunk, one warp per row
    const int nvalid = min(kScatterThreads, s_hi - c0);
    for (int j = warp; j < nvalid; j += kScatterWarps) {
      const int r = rowbuf[j];
      const int t = (c0 + j) / K;
      const uint8_t* src = x + static_cast<size_t>(t) * row_bytes;
      uint8_t* dst = x_perm + static_cast<size_t>(r) * row_bytes;
      if (vec) {
        const uint4* s4 = reinterpret_cast<const uint4*>(src);
        uint4* d4 = reinterpret_cast<uint4*>(dst);
        for (int i = lane; i < row_bytes / 16; i += 32) d4[i] = __ldg(s4 + i);
      } else {
        for (int i = lane; i < row_bytes / 4; i += 32)
          reinterpret_cast<uint32_t*>(dst)[i] = reinterpret_cast<const uint32_t*>(src)[i];
      }
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_permute_scan(const int* blockcounts, int B, int E, int* offsets, int* blockbase,
                                cudaStream_t s) {
  permute_scan_kernel<<<1, kScanThreads, 0, s>>>(blockcounts, B, E, offsets, blockbase);
  return cudaGetLastError();
}

cudaError_t launch_permute_scatter(const int* idx32, const int* blockbase, int T, int K, int E,
                                   const void* x, int D, int elem_bytes, int* perm, int* pos,
                                   void* x_perm, cudaStream_t s) {
  const int B = (T + kRouterTokensPerCta - 1) / kRouterTokensPerCta;
  permute_scatter_kernel<<<B, kScatterThreads, 0, s>>>(
      idx32, blockbase, T, K, E, static_cast<const uint8_t*>(x), D * elem_bytes, perm, pos,
      static_cast<uint8_t*>(x_perm));
  return cudaGetLastError();
}

}  // namespace moe
