// The whole forward of a small float32 layer in one launch.
//
// The layers of the Flax exercise "Mixture-of-Experts FFN" (crackedaicode.com,
// "Problem": T=64 tokens, D=32, F=64, E=4 Dense/ReLU experts with biases) and
// of mojolearn.MoEBlock's example (64 tokens, D=64, F=128, E=8, SiLU-gated)
// are a few MFLOP: the six kernels of the general path cost far more in
// launches than in work.  Here one thread-block cluster with one CTA per
// expert does everything:
//
//   1. every CTA computes the router for all tokens - logits (+ bias),
//      softmax, top-k (descending, equal logits to the lower index, as the
//      exercise's "Compute the experts and router" and mojolearn state) and
//      the weights of "Weight the selected outputs" - with the same code on
//      the same data, so all CTAs agree on the selection bit for bit; CTA 0
//      writes the routing outputs;
//   2. CTA e lists the tokens that chose expert e in token order, stages
//      that expert's weights in shared memory and computes its rows:
//      H = silu(x Wg^T) * (x Wu^T), or relu(x W1^T + b1), then Y = H Wd^T
//      (+ b2), in fp32 FMA;
//   3. after a cluster barrier each CTA combines a slice of the tokens:
//      out[t] = sum_k w[t, k] * Y_{e_k}[row of t in e_k], the k-th term read
//      from expert e_k's CTA through distributed shared memory, summed in
//      slot order and written once.
//
// Same results as the general path up to fp32 summation order (the same
// definitions, fp32 accumulation throughout); deterministic, no atomics.

#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 512;
constexpr int kRowGroup = 4;      // rows of one expert computed together by a thread

struct SmallParams {
  const float* x;
  const float* router;
  const float* rb;
  const float* gu;
  const float* dn;
  const float* b1;
  const float* b2;
  float* out;
  int64_t* sel64;
  float* wout;
  float* logits;
  int T, D, F, E, K, norm, gated;
};

// Shared-memory layout (floats / ints), the same in every CTA of the
// cluster so that a remote Y row is at the same offset as a local one.
struct SmallLayout {
  int xs, wr, lg, sel, w, rank, tok, wcnt, w1, w2, h, y, total;   // offsets in 4-byte words
  int ldx, ldw1, ldw2, ldh;                                       // padded row lengths
};

__host__ __device__ constexpr int round4(int v) { return (v + 3) & ~3; }

// Rows read whole by every lane at once (x, the router, H) are padded to a
// multiple of 4 floats, so they are read 16 bytes at a time (one wavefront
// serves all lanes); x and router rows get 4 more so that a warp reading 4
// different rows at once hits different banks.  Weight rows, read one
// element per lane along a column, keep an odd length: conflict-free.
// Every region starts on a 16-byte boundary.
__host__ __device__ inline SmallLayout small_layout(int T, int D, int F, int E, int K, int gated) {
  SmallLayout L;
  const int gu_rows = gated ? 2 * F : F;
  L.ldx = round4(D) + 4;
  L.ldw1 = D + 1;
  L.ldw2 = F + 1;
  L.ldh = round4(F);
  int o = 0;
  L.xs = o;   o += round4(T * L.ldx);
  L.wr = o;   o += round4(E * L.ldx);
  L.lg = o;   o += round4(T * E);
  L.sel = o;  o += round4(T * K);
  L.w = o;    o += round4(T * K);
  L.rank = o; o += round4(T * K);
  L.tok = o;  o += round4(T);
  L.wcnt = o; o += round4((kThreads / 32) * kSmallMaxExperts);
  L.w1 = o;   o += round4(gu_rows * L.ldw1);
  L.w2 = o;   o += round4(D * L.ldw2);
  L.h = o;    o += round4(T * L.ldh);
  L.y = o;    o += round4(T * D);
  L.total = o;
  return L;
}

__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ float ld_remote_f32(const float* local_addr, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local_addr)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ unsigned int lanemask_lt() {
  unsigned int m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Asynchronous 4-byte copies from global into shared memory: every copy of
// a matrix is in flight at once and no registers hold the data.
__device__ __forceinline__ void cp_async4(float* dst, const float* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Starts copying a rows x cols row-major matrix into shared rows of length
// ld: a warp per row, lanes along the row (coalesced).
__device__ __forceinline__ void stage_async(float* dst, int ld, const float* __restrict__ src,
                                            int rows, int cols) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < rows; r += kThreads / 32)
    for (int c = lane; c < cols; c += 32) cp_async4(dst + r * ld + c, src + static_cast<size_t>(r) * cols + c);
}

// True when (v, e) ranks before (bv, be): larger value, then lower index.
__device__ __forceinline__ bool ranks_before(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

template <bool kGated>
__global__ void __launch_bounds__(kThreads, 1) small_layer_f32_kernel(const SmallParams p) {
  extern __shared__ __align__(16) float sm[];
  const int T = p.T, D = p.D, F = p.F, E = p.E, K = p.K;
  const SmallLayout L = small_layout(T, D, F, E, K, kGated);
  float* xs = sm + L.xs;
  float* wr = sm + L.wr;
  float* lg = sm + L.lg;
  int* sel = reinterpret_cast<int*>(sm + L.sel);
  float* wsel = sm + L.w;
  int* rank = reinterpret_cast<int*>(sm + L.rank);
  int* tok = reinterpret_cast<int*>(sm + L.tok);
  int* wcnt = reinterpret_cast<int*>(sm + L.wcnt);
  float* w1 = sm + L.w1;
  float* w2 = sm + L.w2;
  float* hs = sm + L.h;
  float* ys = sm + L.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int me = static_cast<int>(cta_rank());      // this CTA's expert
  const int gu_rows = kGated ? 2 * F : F;

  pdl_trigger();
  pdl_wait();
  // ---- stage x and the router (group 0), then this expert's weights
  // (group 1), which land while the router runs
  stage_async(xs, L.ldx, p.x, T, D);
  stage_async(wr, L.ldx, p.router, E, D);
  cp_async_commit();
  stage_async(w1, L.ldw1, p.gu + static_cast<size_t>(me) * gu_rows * D, gu_rows, D);
  stage_async(w2, L.ldw2, p.dn + static_cast<size_t>(me) * D * F, D, F);
  cp_async_commit();
  cp_async_wait<1>();
  __syncthreads();

  // ---- router: logits of every (token, expert), four partial sums each
  for (int i = tid; i < T * E; i += kThreads) {
    const int t = i / E, e = i % E;
    const float* xr = xs + t * L.ldx;
    const float* rr = wr + e * L.ldx;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int d = 0;
    for (; d + 4 <= D; d += 4) {
      const float4 xv = *reinterpret_cast<const float4*>(xr + d);
      const float4 rv = *reinterpret_cast<const float4*>(rr + d);
      a0 = fmaf(xv.x, rv.x, a0);
      a1 = fmaf(xv.y, rv.y, a1);
      a2 = fmaf(xv.z, rv.z, a2);
      a3 = fmaf(xv.w, rv.w, a3);
    }
    for (; d < D; ++d) a0 = fmaf(xr[d], rr[d], a0);
    float acc = (a0 + a1) + (a2 + a3);
    if (p.rb) acc += __ldg(p.rb + e);
    lg[i] = acc;
    if (me == 0 && p.logits) p.logits[i] = acc;
  }
  __syncthreads();
  // ---- softmax, top-k and weights, one thread per token (T <= kThreads)
  const int t = tid;
  unsigned int member = 0u;                    // experts token t chose
  if (t < T) {
    const float* l = lg + t * E;
    float m = -INFINITY;
    for (int e = 0; e < E; ++e) m = fmaxf(m, isnan(l[e]) ? -INFINITY : l[e]);
    float s = 0.f;
    for (int e = 0; e < E; ++e) s += isnan(l[e]) ? 0.f : expf(l[e] - m);
    // the K best by logit (softmax is monotone), a NaN logit ranking last
    float psum = 0.f;
    for (int k = 0; k < K; ++k) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
      for (int e = 0; e < E; ++e) {
        const float v = isnan(l[e]) ? -INFINITY : l[e];
        if (!(member & (1u << e)) && ranks_before(v, e, bv, be)) {
          bv = v;
          be = e;
        }
      }
      member |= 1u << be;
      const float pk = isnan(l[be]) ? 0.f : expf(l[be] - m) / s;
      sel[t * K + k] = be;
      wsel[t * K + k] = pk;
      psum += pk;
    }
    const float denom = psum + 1e-9f;
    for (int k = 0; k < K; ++k) {
      const float w = p.norm ? wsel[t * K + k] / denom : wsel[t * K + k];
      wsel[t * K + k] = w;
      if (me == 0) {
        if (p.sel64) p.sel64[static_cast<size_t>(t) * K + k] = sel[t * K + k];
        if (p.wout) p.wout[static_cast<size_t>(t) * K + k] = w;
      }
    }
  }
  // ---- each slot's row within its expert = the earlier tokens that chose
  // the same expert (an expert's rows are listed in token order): per expert
  // a warp ballot over the tokens, then the counts of the earlier warps
  int below[kSmallMaxExperts];
#pragma unroll
  for (int e = 0; e < kSmallMaxExperts; ++e) {
    const unsigned int b = __ballot_sync(0xffffffffu, (member >> e) & 1u);
    below[e] = __popc(b & lanemask_lt());
    if (lane == 0) wcnt[warp * kSmallMaxExperts + e] = __popc(b);
  }
  __syncthreads();
  int rows = 0;                                // rows of expert `me`
  for (int w = 0; w < kThreads / 32; ++w) rows += wcnt[w * kSmallMaxExperts + me];
  if (t < T) {
    for (int k = 0; k < K; ++k) {
      const int e = sel[t * K + k];
      int r = 0;
#pragma unroll
      for (int ee = 0; ee < kSmallMaxExperts; ++ee)
        if (ee == e) r = below[ee];
      for (int w = 0; w < warp; ++w) r += wcnt[w * kSmallMaxExperts + e];
      rank[t * K + k] = r;
      if (e == me) tok[r] = t;
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- expert `me` on its rows: H, then Y (fp32 FMA from shared memory)
  const int groups = (rows + kRowGroup - 1) / kRowGroup;
  for (int item = tid; item < F * groups; item += kThreads) {
    const int f = item % F, g = item / F;
    float a[kRowGroup], b[kRowGroup];
#pragma unroll
    for (int j = 0; j < kRowGroup; ++j) a[j] = b[j] = 0.f;
    const float* wa = w1 + f * L.ldw1;                         // gate row (or W1 row)
    const float* wb = w1 + (kGated ? F + f : f) * L.ldw1;     // up row
    const float* xr[kRowGroup];
#pragma unroll
    for (int j = 0; j < kRowGroup; ++j) {
      const int r = g * kRowGroup + j;
      xr[j] = xs + (r < rows ? tok[r] : 0) * L.ldx;
    }
    // x rows four columns at a time (16-byte reads every lane shares)
    int d = 0;
#pragma unroll 2
    for (; d + 4 <= D; d += 4) {
      float4 xv[kRowGroup];
#pragma unroll
      for (int j = 0; j < kRowGroup; ++j) xv[j] = *reinterpret_cast<const float4*>(xr[j] + d);
      const float va[4] = {wa[d], wa[d + 1], wa[d + 2], wa[d + 3]};
      float vb[4] = {0.f, 0.f, 0.f, 0.f};
      if (kGated) {
        vb[0] = wb[d];
        vb[1] = wb[d + 1];
        vb[2] = wb[d + 2];
        vb[3] = wb[d + 3];
      }
#pragma unroll
      for (int j = 0; j < kRowGroup; ++j) {
        a[j] = fmaf(xv[j].x, va[0], a[j]);
        a[j] = fmaf(xv[j].y, va[1], a[j]);
        a[j] = fmaf(xv[j].z, va[2], a[j]);
        a[j] = fmaf(xv[j].w, va[3], a[j]);
        if (kGated) {
          b[j] = fmaf(xv[j].x, vb[0], b[j]);
          b[j] = fmaf(xv[j].y, vb[1], b[j]);
          b[j] = fmaf(xv[j].z, vb[2], b[j]);
          b[j] = fmaf(xv[j].w, vb[3], b[j]);
        }
      }
    }
    for (; d < D; ++d) {
      const float va = wa[d];
      const float vb = kGated ? wb[d] : 0.f;
#pragma unroll
      for (int j = 0; j < kRowGroup; ++j) {
        const float xv = xr[j][d];
        a[j] = fmaf(xv, va, a[j]);
        if (kGated) b[j] = fmaf(xv, vb, b[j]);
      }
    }
    const float bias = (!kGated && p.b1) ? __ldg(p.b1 + static_cast<size_t>(me) * F + f) : 0.f;
#pragma unroll
    for (int j = 0; j < kRowGroup; ++j) {
      const int r = g * kRowGroup + j;
      if (r < rows)
        hs[r * L.ldh + f] = kGated ? a[j] / (1.f + expf(-a[j])) * b[j] : fmaxf(a[j] + bias, 0.f);
    }
  }
  __syncthreads();
  for (int item = tid; item < D * groups; item += kThreads) {
    const int d = item % D, g = item / D;
    float a[kRowGroup];
#pragma unroll
    for (int j = 0; j < kRowGroup; ++j) a[j] = 0.f;
    const float* wd = w2 + d * L.ldw2;
    const float* hr[kRowGroup];
#pragma unroll
    for (int j = 0; j < kRowGroup; ++j) hr[j] = hs + min(g * kRowGroup + j, rows - 1) * L.ldh;
    int f = 0;
#pragma unroll 2
    for (; f + 4 <= F; f += 4) {
      const float v[4] = {wd[f], wd[f + 1], wd[f + 2], wd[f + 3]};
#pragma unroll
      for (int j = 0; j < kRowGroup; ++j) {
        const float4 h4 = *reinterpret_cast<const float4*>(hr[j] + f);
        a[j] = fmaf(h4.x, v[0], a[j]);
        a[j] = fmaf(h4.y, v[1], a[j]);
        a[j] = fmaf(h4.z, v[2], a[j]);
        a[j] = fmaf(h4.w, v[3], a[j]);
      }
    }
    for (; f < F; ++f) {
      const float v = wd[f];
#pragma unroll
      for (int j = 0; j < kRowGroup; ++j) a[j] = fmaf(hr[j][f], v, a[j]);
    }
    const float bias = p.b2 ? __ldg(p.b2 + static_cast<size_t>(me) * D + d) : 0.f;
#pragma unroll
    for (int j = 0; j < kRowGroup; ++j) {
      const int r = g * kRowGroup + j;
      if (r < rows) ys[r * D + d] = a[j] + bias;
    }
  }

  // ---- combine: every expert's rows are in its CTA's shared memory
  cluster_barrier();
  const int t_lo = me * T / E, t_hi = (me + 1) * T / E;
  for (int i = tid; i < (t_hi - t_lo) * D; i += kThreads) {
    const int tt = t_lo + i / D, d = i % D;
    float acc = 0.f;
    for (int k = 0; k < K; ++k) {
      const int e = sel[tt * K + k];
      acc = fmaf(wsel[tt * K + k], ld_remote_f32(ys + rank[tt * K + k] * D + d, e), acc);
    }
    p.out[static_cast<size_t>(tt) * D + d] = acc;
  }
  // no CTA leaves while another may still read its rows
  cluster_barrier();
}

size_t small_smem_bytes(int T, int D, int F, int E, int K, int gated) {
  return sizeof(float) * static_cast<size_t>(small_layout(T, D, F, E, K, gated).total);
}

}  // namespace

bool small_layer_fits(int T, int D, int F, int E, int K, int gated) {
  if (E < 1 || E > kSmallMaxExperts || K < 1 || K > E) return false;
  if (static_cast<long long>(T) * K > kSmallMaxRows || D > 1024 || F > 1024) return false;
  return small_smem_bytes(T, D, F, E, K, gated) <= kSmallMaxSmem;
}

cudaError_t launch_small_layer_f32(const float* x, const float* router, const float* rb,
                                   const float* gu, const float* dn, const float* b1,
                                   const float* b2, int T, int D, int F, int E, int K, int norm,
                                   int gated, float* out, int64_t* sel64, float* wout,
                                   float* logits, cudaStream_t s) {
  if (!small_layer_fits(T, D, F, E, K, gated)) return cudaErrorInvalidValue;
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64 || !done[dev]) {
      for (auto fn : {small_layer_f32_kernel<true>, small_layer_f32_kernel<false>}) {
        err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(kSmallMaxSmem));
        if (err != cudaSuccess) return err;
      }
      if (dev >= 0 && dev < 64) done[dev] = true;
    }
  }
  SmallParams p;
  p.x = x;
  p.router = router;
  p.rb = rb;
  p.gu = gu;
  p.dn = dn;
  p.b1 = b1;
  p.b2 = b2;
  p.out = out;
  p.sel64 = sel64;
  p.wout = wout;
  p.logits = logits;
  p.T = T;
  p.D = D;
  p.F = F;
  p.E = E;
  p.K = K;
  p.norm = norm;
  p.gated = gated;
  return launch_k(gated ? small_layer_f32_kernel<true> : small_layer_f32_kernel<false>, dim3(E),
                  dim3(kThreads), small_smem_bytes(T, D, F, E, K, gated), s, pdl_enabled(), E, p);
}

}  // namespace moe
