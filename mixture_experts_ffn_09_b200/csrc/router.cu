// Router: logits = x router^T (+ bias) in fp32, softmax over the experts,
// top-k with lower-index tie-breaking, renormalised weights, and the
// per-block expert histogram the permutation needs.
//
// Follows "Mixture-of-Experts FFN" (crackedaicode.com Flax exercise),
// sections "Compute the experts and router" (Dense(E) router, softmax,
// jax.lax.top_k order: descending, equal scores to the lower index) and
// "Weight the selected outputs" (weights = sel / (sum(sel) + 1e-9)); and
// mojolearn.MoEBlock (router (E, D) without bias, norm_topk_prob).
//
// One warp per token.  Lanes stride over D with 16-byte loads and keep 8
// expert partial sums at a time; the logits of a token then live one per
// lane (E <= 256: up to 8 per lane).  Ranking uses the fp32 logits, which
// orders the experts exactly as their probabilities do (softmax is
// monotone), so ties in the logits are ties in the probabilities.
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kPerLane = kMaxExperts / 32;

template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void load(const float* p, float (&v)[4]) {
    const float4 q = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
};

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }

// True when (v, e) ranks before (bv, be): larger value, then lower index.
__device__ __forceinline__ bool ranks_before(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

template <typename Tin, bool kVec>
__global__ void __launch_bounds__(kWarps * 32) router_topk_kernel(RouteArgs a) {
  extern __shared__ float sm[];
  const int E = a.E, K = a.K, D = a.D;
  int* hist = reinterpret_cast<int*>(sm);                      // E
  float* lg_all = sm + E;                                      // kWarps * E
  int* sel_all = reinterpret_cast<int*>(lg_all + kWarps * E);  // kWarps * K
  float* selv_all = reinterpret_cast<float*>(sel_all + kWarps * K);
  float* bal_all = selv_all + kWarps * K;                      // kWarps * 3 * E (balance only)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  if (a.bal_partial)
    for (int i = threadIdx.x; i < kWarps * 3 * E; i += blockDim.x) bal_all[i] = 0.f;
  __syncthreads();

  const Tin* X = static_cast<const Tin*>(a.x);
  const Tin* W = static_cast<const Tin*>(a.router);
  float* lg = lg_all + warp * E;
  int* sel = sel_all + warp * K;
  float* selv = selv_all + warp * K;
  float* bal = bal_all + warp * 3 * E;

  for (int j = 0; j < kRouterTokensPerCta / kWarps; ++j) {
    const int t = blockIdx.x * kRouterTokensPerCta + j * kWarps + warp;
    if (t >= a.T) break;
    const Tin* xr = X + static_cast<size_t>(t) * D;

    // ---- logits, 8 experts at a time
    for (int e0 = 0; e0 < E; e0 += 8) {
      const int ne = min(8, E - e0);
      float acc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = 0.f;
      if (kVec) {
        constexpr int V = Vec<Tin>::N;
        for (int d = lane * V; d < D; d += 32 * V) {
          float xv[V];
          Vec<Tin>::load(xr + d, xv);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (q < ne) {
              float wv[V];
              Vec<Tin>::load(W + static_cast<size_t>(e0 + q) * D + d, wv);
#pragma unroll
              for (int v = 0; v < V; ++v) acc[q] = fmaf(xv[v], wv[v], acc[q]);
            }
          }
        }
      } else {
        for (int d = lane; d < D; d += 32) {
          const float xv = to_f(xr[d]);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (q < ne) acc[q] = fmaf(xv, to_f(W[static_cast<size_t>(e0 + q) * D + d]), acc[q]);
        }
      }
      float mine = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float s = warp_sum(acc[q]);
        if (lane == q) mine = s;
      }
      if (lane < ne) lg[e0 + lane] = mine;
    }
    __syncwarp();

    // ---- bias, logits out, softmax statistics, scores and ranking keys
    float l[kPerLane], sc[kPerLane], key[kPerLane];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int e = lane + 32 * i;
      l[i] = -INFINITY;
      if (e < E) {
        float v = lg[e];
        if (a.router_bias) v += __ldg(a.router_bias + e);
        if (a.logits) a.logits[static_cast<size_t>(t) * E + e] = v;
        l[i] = isnan(v) ? -INFINITY : v;
        m = fmaxf(m, l[i]);
      }
    }
    m = warp_max(m);
    float s = 0.f;
    if (a.score == 0) {
#pragma unroll
      for (int i = 0; i < kPerLane; ++i)
        if (lane + 32 * i < E) s += expf(l[i] - m);
      s = warp_sum(s);
    }
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int e = lane + 32 * i;
      sc[i] = 0.f;
      key[i] = -INFINITY;
      if (e < E) {
        sc[i] = a.score == 0 ? expf(l[i] - m) / s : 1.f / (1.f + expf(-l[i]));
        const float kb = a.sel_bias ? sc[i] + __ldg(a.sel_bias + e) : l[i];
        key[i] = isnan(kb) ? -INFINITY : kb;   // NaN never ranks: keep every key orderable
        if (a.bal_partial) bal[e] += sc[i];
      }
    }

    // ---- top-k: K rounds of a warp-wide argmax over the untaken experts
    unsigned int taken = 0u;
    for (int k = 0; k < K; ++k) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < kPerLane; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !(taken & (1u << i)) && ranks_before(key[i], e, bv, be)) {
          bv = key[i];
          be = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (ranks_before(ov, oe, bv, be)) {
          bv = ov;
          be = oe;
        }
      }
      if ((be & 31) == lane) {
        taken |= 1u << (be >> 5);
        float own = 0.f;
#pragma unroll
        for (int i = 0; i < kPerLane; ++i)
          if (i == (be >> 5)) own = sc[i];
        sel[k] = be;
        selv[k] = own;       // the unbiased score
      }
    }
    __syncwarp();

    // ---- weights: renormalised scores, then the optional dynamic threshold
    float psum = 0.f;
    for (int k = 0; k < K; ++k) psum += selv[k];
    float ksum = 0.f;
    if (a.dyn_threshold > 0.f)
      for (int k = 0; k < K; ++k) {
        const float sh = selv[k] / psum;
        if (k == 0 || sh >= a.dyn_threshold) ksum += sh;
      }
    const float denom = a.norm ? (psum + 1e-9f) : 1.f;
    auto weight = [&](int k, bool& keep) {
      const float p = selv[k];
      float w = a.norm ? p / denom : p;
      keep = true;
      if (a.dyn_threshold > 0.f) {
        const float sh = p / psum;
        keep = k == 0 || sh >= a.dyn_threshold;
        w = keep ? sh / ksum : 0.f;
      }
      return w;
    };
    // the balance statistics read the selection renormalised to sum to one
    // (whether or not the output weights are): gate = w / sum of the kept w
    float wsum = 0.f;
    if (a.bal_partial)
      for (int k = 0; k < K; ++k) {
        bool kk;
        wsum += weight(k, kk);
      }
    for (int k = lane; k < K; k += 32) {
      const int e = sel[k];
      bool keep;
      const float w = weight(k, keep);
      const size_t o = static_cast<size_t>(t) * K + k;
      if (a.sel64) a.sel64[o] = e;
      if (a.wout) a.wout[o] = w;
      if (a.idx32) a.idx32[o] = keep ? e : E;
      if (a.w32) a.w32[o] = w;
      if (a.slot_kept) a.slot_kept[o] = keep ? 1 : 0;
      if (keep && a.blockcounts) atomicAdd(&hist[e], 1);
      if (a.bal_partial) {
        const float g = wsum > 0.f ? w / wsum : 0.f;
        bal[E + e] += g;
        bal[2 * E + e] += g > 0.f ? 1.f : 0.f;
      }
    }
    __syncwarp();
  }

  if (a.blockcounts || a.bal_partial) {
    __syncthreads();
    if (a.blockcounts)
      for (int e = threadIdx.x; e < E; e += blockDim.x)
        a.blockcounts[static_cast<size_t>(blockIdx.x) * E + e] = hist[e];
    if (a.bal_partial)
      for (int i = threadIdx.x; i < 3 * E; i += blockDim.x) {
        float acc = 0.f;
        for (int w = 0; w < kWarps; ++w) acc += bal_all[w * 3 * E + i];   // fixed warp order
        a.bal_partial[static_cast<size_t>(blockIdx.x) * 3 * E + i] = acc;
      }
  }
}

template <typename Tin, bool kVec>
cudaError_t launch_typed(const RouteArgs& a, cudaStream_t s) {
  const int blocks = (a.T + kRouterTokensPerCta - 1) / kRouterTokensPerCta;
  size_t smem = sizeof(float) * (a.E + kWarps * a.E) + sizeof(int) * kWarps * a.K +
                sizeof(float) * kWarps * a.K;
  if (a.bal_partial) smem += sizeof(float) * kWarps * 3 * a.E;
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64 || !done[dev]) {
      err = cudaFuncSetAttribute(router_topk_kernel<Tin, kVec>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
      if (err != cudaSuccess) return err;
      if (dev >= 0 && dev < 64) done[dev] = true;
    }
  }
  return launch_k(router_topk_kernel<Tin, kVec>, dim3(blocks), dim3(kWarps * 32), smem, s,
                  pdl_enabled(), 1, a);
}

}  // namespace

int router_simt_parts(int T) { return (T + kRouterTokensPerCta - 1) / kRouterTokensPerCta; }

cudaError_t launch_router(const RouteArgs& a, cudaStream_t s) {
  if (a.dt == kBF16) {
    const bool vec = (a.D % 8 == 0);
    return vec ? launch_typed<__nv_bfloat16, true>(a, s) : launch_typed<__nv_bfloat16, false>(a, s);
  }
  const bool vec = (a.D % 4 == 0);
  return vec ? launch_typed<float, true>(a, s) : launch_typed<float, false>(a, s);
}

}  // namespace moe
