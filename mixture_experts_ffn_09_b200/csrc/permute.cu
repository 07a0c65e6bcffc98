// Expert permutation: sorts the (token, slot) pairs into expert order so the
// experts can run as one grouped matrix multiplication over contiguous rows
// ("Mixture of experts", dewml.dev, section "Expert computation and
// placement": tokens are sorted into expert order).
//
// The order is stable: rows of one expert are listed by (token, slot), so
// the result is deterministic and independent of scheduling.  Three kernels:
//   scan    - one CTA per expert scans that expert's column of the router's
//             32-token histograms: each block's first row within the expert
//             and the expert's total (for a small table the scatter blocks
//             scan it themselves and this kernel does not run);
//   scatter - one CTA per 32-token block ranks its slots within their
//             expert (warp match + per-warp counts) and writes perm / pos;
//             slots the router dropped, or past a capacity, get no row;
//   gather  - copies the token rows into x_perm: one warp per sorted row
//             while x fits in L2, else one warp per token, which reads each
//             row of x once and stores it to all of the token's rows.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

__device__ __forceinline__ unsigned int lanemask_lt() {
  unsigned int m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

constexpr int kScanThreads = 512;

__global__ void __launch_bounds__(kScanThreads) permute_scan_kernel(const int* __restrict__ bc,
                                                                    int B, int E,
                                                                    int* __restrict__ blockbase,
                                                                    int* __restrict__ totals) {
  __shared__ int wsum[kScanThreads / 32];
  __shared__ int carry;
  pdl_trigger();
  pdl_wait();
  const int e = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int b0 = 0; b0 < B; b0 += kScanThreads) {
    const int b = b0 + threadIdx.x;
    const int c = (b < B) ? bc[static_cast<size_t>(b) * E + e] : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = carry;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    if (b < B) blockbase[static_cast<size_t>(b) * E + e] = before + incl - c;
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) carry = before + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) totals[e] = carry;
}

constexpr int kScatterThreads = 256;
constexpr int kScatterWarps = kScatterThreads / 32;

// One CTA per 32-token block.  A slot's row is its expert's offset + the
// rows of that expert in earlier blocks + its rank among the block's slots
// of the same expert (token order).  When the block counts were clamped by
// a capacity, slots ranked at or past the clamped count get no row.
__global__ void __launch_bounds__(kScatterThreads) permute_scatter_kernel(
    const int* __restrict__ idx32, const int* __restrict__ blockbase, const int* __restrict__ totals,
    const int* __restrict__ blockcounts, int T, int K, int E, int* __restrict__ offsets,
    int* __restrict__ perm, int* __restrict__ pos, uint8_t* __restrict__ slot_kept,
    int* __restrict__ sched) {
  __shared__ int off[kMaxExperts + 1];
  __shared__ int base[kMaxExperts];
  __shared__ int kept[kMaxExperts];
  __shared__ int run[kMaxExperts];
  __shared__ int wc[kScatterWarps][kMaxExperts];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  if (!blockbase) {
    // no scan kernel ran (small block-count table): each block scans the
    // expert columns itself - the expert totals and the rows of each expert
    // in earlier blocks, both in block order
    // one warp per expert, lanes striding over the blocks
    for (int e = warp; e < E; e += kScatterWarps) {
      int before = 0, total = 0;
      for (int b2 = lane; b2 < static_cast<int>(gridDim.x); b2 += 32) {
        const int c = blockcounts[static_cast<size_t>(b2) * E + e];
        before += b2 < b ? c : 0;
        total += c;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        before += __shfl_xor_sync(0xffffffffu, before, o);
        total += __shfl_xor_sync(0xffffffffu, total, o);
      }
      if (lane == 0) {
        base[e] = before;
        run[e] = total;                    // borrowed until the offsets exist
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      off[e] = acc;
      acc += blockbase ? totals[e] : run[e];
    }
    off[E] = acc;
  }
  __syncthreads();
  if (b == 0) {
    for (int e = threadIdx.x; e <= E; e += kScatterThreads) offsets[e] = off[e];
    // the grouped GEMMs' tile counters start this forward at zero
    if (sched)
      for (int i = threadIdx.x; i < kSchedInts; i += kScatterThreads) sched[i] = 0;
  }
  for (int e = threadIdx.x; e < E; e += kScatterThreads) {
    base[e] = off[e] + (blockbase ? blockbase[static_cast<size_t>(b) * E + e] : base[e]);
    kept[e] = blockcounts[static_cast<size_t>(b) * E + e];
    run[e] = 0;
#pragma unroll
    for (int w = 0; w < kScatterWarps; ++w) wc[w][e] = 0;
  }
  __syncthreads();

  const int t_lo = b * kRouterTokensPerCta;
  const int t_hi = min(T, t_lo + kRouterTokensPerCta);
  const int s_lo = t_lo * K, s_hi = t_hi * K;

  for (int c0 = s_lo; c0 < s_hi; c0 += kScatterThreads) {
    const int s = c0 + threadIdx.x;
    const bool in_range = s < s_hi;
    int e = in_range ? idx32[s] : -1;
    if (e >= E) e = -1;                       // dropped by the router: no row, no rank
    const unsigned int mask = __match_any_sync(0xffffffffu, e);
    const int wrank = __popc(mask & lanemask_lt());
    if (e >= 0 && lane == __ffs(mask) - 1) wc[warp][e] = __popc(mask);
    __syncthreads();
    if (in_range) {
      bool has_row = false;
      if (e >= 0) {
        int q = run[e] + wrank;
        for (int w = 0; w < warp; ++w) q += wc[w][e];
        if (q < kept[e]) {
          const int r = base[e] + q;
          perm[r] = s;
          pos[s] = r;
          has_row = true;
        }
      }
      if (!has_row) {
        pos[s] = -1;
        if (slot_kept) slot_kept[s] = 0;
      }
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
    __syncthreads();
  }
}

constexpr int kGatherThreads = 256;
constexpr int kGatherBatch = 8;   // 16-byte vectors each lane holds per chunk of a row

// Row order: one warp per sorted row copies x[perm[row] / K].  Every lane
// issues its whole batch of loads before its stores.  A row of x chosen by
// several experts is read once per copy; that is cheap while x sits in L2.
__global__ void __launch_bounds__(kGatherThreads) gather_by_row_kernel(
    const int* __restrict__ perm, const int* __restrict__ offsets, int E, int K,
    const uint8_t* __restrict__ x, int row_bytes, uint8_t* __restrict__ x_perm) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * (kGatherThreads / 32) + warp;
  if (r >= offsets[E]) return;
  const int t = perm[r] / K;
  const uint8_t* src = x + static_cast<size_t>(t) * row_bytes;
  uint8_t* dst = x_perm + static_cast<size_t>(r) * row_bytes;
  if ((row_bytes & 15) == 0) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    const int n16 = row_bytes >> 4;
    for (int i0 = 0; i0 < n16; i0 += 32 * kGatherBatch) {
      uint4 v[kGatherBatch];
#pragma unroll
      for (int j = 0; j < kGatherBatch; ++j) {
        const int i = i0 + j * 32 + lane;
        if (i < n16) v[j] = __ldg(s4 + i);
      }
#pragma unroll
      for (int j = 0; j < kGatherBatch; ++j) {
        const int i = i0 + j * 32 + lane;
        if (i < n16) d4[i] = v[j];
      }
    }
  } else {
    for (int i = lane; i < row_bytes / 4; i += 32)
      reinterpret_cast<uint32_t*>(dst)[i] = reinterpret_cast<const uint32_t*>(src)[i];
  }
}

// Token order: one warp per token reads its row of x once, a chunk of
// 32 x kGatherBatch 16-byte vectors at a time, and stores each chunk to
// every sorted row the token's slots were given (pos; a dropped slot has
// none).  Each x row leaves HBM once however many experts chose it, which
// matters once x no longer fits in L2.
__global__ void __launch_bounds__(kGatherThreads) gather_by_token_kernel(
    const int* __restrict__ pos, int T, int K, const uint8_t* __restrict__ x, int row_bytes,
    uint8_t* __restrict__ x_perm) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (kGatherThreads / 32) + warp;
  if (t >= T) return;
  const int* tp = pos + static_cast<size_t>(t) * K;
  const int my_row = lane < K ? tp[lane] : -1;     // slots 0..31, shared by shuffle
  auto row_of = [&](int k) { return k < 32 ? __shfl_sync(0xffffffffu, my_row, k) : __ldg(tp + k); };
  const uint8_t* src = x + static_cast<size_t>(t) * row_bytes;
  if ((row_bytes & 15) == 0) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    const int n16 = row_bytes >> 4;
    for (int i0 = 0; i0 < n16; i0 += 32 * kGatherBatch) {
      uint4 v[kGatherBatch];
#pragma unroll
      for (int j = 0; j < kGatherBatch; ++j) {
        const int i = i0 + j * 32 + lane;
        if (i < n16) v[j] = __ldg(s4 + i);
      }
      for (int k = 0; k < K; ++k) {
        const int r = row_of(k);
        if (r < 0) continue;
        uint4* d4 = reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(r) * row_bytes);
#pragma unroll
        for (int j = 0; j < kGatherBatch; ++j) {
          const int i = i0 + j * 32 + lane;
          if (i < n16) d4[i] = v[j];
        }
      }
    }
  } else {
    for (int k = 0; k < K; ++k) {
      const int r = row_of(k);
      if (r < 0) continue;
      uint32_t* dst = reinterpret_cast<uint32_t*>(x_perm + static_cast<size_t>(r) * row_bytes);
      for (int i = lane; i < row_bytes / 4; i += 32)
        dst[i] = reinterpret_cast<const uint32_t*>(src)[i];
    }
  }
}

}  // namespace

cudaError_t launch_permute_scan(const int* blockcounts, int B, int E, int* blockbase, int* totals,
                                cudaStream_t s) {
  return launch_k(permute_scan_kernel, dim3(E), dim3(kScanThreads), 0, s, pdl_enabled(), 1,
                  blockcounts, B, E, blockbase, totals);
}

cudaError_t launch_permute_scatter(const int* idx32, const int* blockbase, const int* totals,
                                   const int* blockcounts, int T, int K, int E, int* offsets,
                                   int* perm, int* pos, uint8_t* slot_kept, int* sched,
                                   cudaStream_t s) {
  const int B = (T + kRouterTokensPerCta - 1) / kRouterTokensPerCta;
  return launch_k(permute_scatter_kernel, dim3(B), dim3(kScatterThreads), 0, s, pdl_enabled(), 1,
                  idx32, blockbase, totals, blockcounts, T, K, E, offsets, perm, pos, slot_kept,
                  sched);
}

cudaError_t launch_gather_rows(const int* perm, const int* offsets, const int* pos, int T, int E,
                               int K, const void* x, int row_bytes, void* x_perm, cudaStream_t s) {
  constexpr size_t kL2ResidentBytes = 48u << 20;   // x read per copy while it stays in L2
  const int warps = kGatherThreads / 32;
  if (static_cast<size_t>(T) * row_bytes <= kL2ResidentBytes) {
    const long long rows = static_cast<long long>(T) * K;
    return launch_k(gather_by_row_kernel, dim3(static_cast<unsigned>((rows + warps - 1) / warps)),
                    dim3(kGatherThreads), 0, s, pdl_enabled(), 1, perm, offsets, E, K,
                    static_cast<const uint8_t*>(x), row_bytes, static_cast<uint8_t*>(x_perm));
  }
  return launch_k(gather_by_token_kernel, dim3((T + warps - 1) / warps), dim3(kGatherThreads), 0, s,
                  pdl_enabled(), 1, pos, T, K, static_cast<const uint8_t*>(x), row_bytes,
                  static_cast<uint8_t*>(x_perm));
}

}  // namespace moe
