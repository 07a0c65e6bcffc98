// Routing extensions that act between the router and the permutation:
//
// capacity - "Mixture of experts" (dewml.dev), "Expert computation and
//   placement", capacity_factor: each sequence keeps
//   floor(max(ceil(L*K/E)*cf, cf)) slots per expert, taken in token order,
//   and a dropped slot adds nothing.  Applied to the router's 32-token block
//   histograms: for every (sequence, expert) the blocks are scanned in token
//   order and each block's count is clamped to what the capacity still
//   allows.  The stable scatter then keeps, in each block, exactly the first
//   slots of each expert up to the clamped count.
//
// balance - ES-MoE API page, "Balancing objectives": switch, gshard, master
//   and gshard_probs of the batch, from the router's per-tile sums of the
//   scores, the gate and gate > 0, added in fixed order.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kClampWarps = 8;

__global__ void __launch_bounds__(kClampWarps * 32) capacity_clamp_kernel(int* __restrict__ bc,
                                                                        int B, int E, int T, int K,
                                                                        int blocks_per_seq,
                                                                        float cf) {
  pdl_trigger();
  pdl_wait();
  const int seq = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b_lo = seq * blocks_per_seq;
  const int b_hi = min(B, b_lo + blocks_per_seq);
  const int t_lo = b_lo * kRouterTokensPerCta;
  const int t_hi = min(T, b_hi * kRouterTokensPerCta);
  const int len = t_hi - t_lo;
  const double c = fmax(ceil(static_cast<double>(len) * K / E) * static_cast<double>(cf),
                        static_cast<double>(cf));
  const int cap = static_cast<int>(floor(c));
  for (int e = warp; e < E; e += kClampWarps) {
    int running = 0;   // slots of expert e in earlier blocks of this sequence
    for (int b0 = b_lo; b0 < b_hi; b0 += 32) {
      const int b = b0 + lane;
      const int cnt = (b < b_hi) ? bc[static_cast<size_t>(b) * E + e] : 0;
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      const int before = running + incl - cnt;
      const int keep = max(0, min(cnt, cap - before));
      if (b < b_hi) bc[static_cast<size_t>(b) * E + e] = keep;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
}

__global__ void __launch_bounds__(256) balance_finalize_kernel(const float* __restrict__ part,
                                                               int parts, int E, int T,
                                                               float* __restrict__ out) {
  __shared__ float mp[kMaxExperts], mg[kMaxExperts], fr[kMaxExperts];
  pdl_trigger();
  pdl_wait();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float P = 0.f, G = 0.f, C = 0.f;
    for (int i = 0; i < parts; ++i) {
      const float* q = part + static_cast<size_t>(i) * 3 * E;
      P += q[e];
      G += q[E + e];
      C += q[2 * E + e];
    }
    mp[e] = P / T;
    mg[e] = G / T;
    fr[e] = C / T;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float smp = 0.f, smg = 0.f, sw = 0.f;
    for (int e = 0; e < E; ++e) {
      smp += mp[e];
      smg += mg[e];
      sw += mp[e] * fr[e];
    }
    float gs = 0.f, ms = 0.f, gp = 0.f;
    for (int e = 0; e < E; ++e) {
      const float u = mg[e] / smg;
      const float v = mp[e] / smp;
      gs += u * u;
      ms += (u - 1.f / E) * (u - 1.f / E);
      gp += v * v;
    }
    out[0] = E * sw;        // switch
    out[1] = E * gs;        // gshard
    out[2] = ms / E;        // master
    out[3] = E * gp;        // gshard_probs
  }
}

// The bounded wait of the GEMM and router kernels, on a barrier that never
// completes: it must give up, record the timeout and let the kernel return.
__global__ void bounded_wait_probe_kernel(unsigned long long timeout_ns, unsigned int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort, err, SITE_PROBE, timeout_ns);
  __syncthreads();
}

}  // namespace

cudaError_t launch_bounded_wait_probe(unsigned long long timeout_ns, unsigned int* err,
                                      cudaStream_t s) {
  bounded_wait_probe_kernel<<<1, 32, 0, s>>>(timeout_ns, err);
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) note_launch();
  return e;
}

cudaError_t launch_capacity_clamp(int* blockcounts, int B, int E, int T, int K, int seq_len,
                                  float capacity_factor, cudaStream_t s) {
  const int bps = seq_len > 0 ? seq_len / kRouterTokensPerCta : B;
  const int seqs = (B + bps - 1) / bps;
  return launch_k(capacity_clamp_kernel, dim3(seqs), dim3(kClampWarps * 32), 0, s, pdl_enabled(),
                  1, blockcounts, B, E, T, K, bps, capacity_factor);
}

cudaError_t launch_balance_finalize(const float* partial, int parts, int E, int T, float* out4,
                                    cudaStream_t s) {
  return launch_k(balance_finalize_kernel, dim3(1), dim3(256), 0, s, pdl_enabled(), 1, partial,
                  parts, E, T, out4);
}

}  // namespace moe
