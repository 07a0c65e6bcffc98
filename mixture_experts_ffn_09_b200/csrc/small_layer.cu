// The whole forward of a small float32 layer in one launch.
//
// The layers of the Flax exercise "Mixture-of-Experts FFN" (crackedaicode.com,
// "Problem": T=64 tokens, D=32, F=64, E=4 Dense/ReLU experts with biases) and
// of mojolearn.MoEBlock's example (64 tokens, D=64, F=128, E=8, SiLU-gated)
// are a few MFLOP: the six kernels of the general path cost far more in
// launches than in work.  Here one thread-block cluster of C CTAs (16 where
// the GPU can co-schedule them, else 8) does everything:
//
//   1. every CTA computes the router for all tokens - logits (+ bias),
//      softmax, top-k (descending, equal logits to the lower index, as the
//      exercise's "Compute the experts and router" and mojolearn state) and
//      the weights of "Weight the selected outputs" - with the same code on
//      the same data, so all CTAs agree on the selection bit for bit; CTA 0
//      writes the routing outputs;
//   2. from the rows each expert received, every CTA derives the same
//      assignment of the C CTAs to experts: each expert with rows gets one
//      CTA plus its proportional share of the rest (rounded down), and each
//      CTA still free goes to the expert with the most rows per CTA (lower
//      index on ties).  An expert's s CTAs split its hidden
//      columns F into s slices of whole 4-column groups, so the routing skew
//      of a real batch (one expert can take almost half of all rows) is
//      spread over several SMs instead of setting the time of the launch;
//   3. the CTA holding slice [f0, f1) of expert e stages that slice of the
//      weights (gate and up rows f0..f1-1 of gate_up_proj[e], columns
//      f0..f1-1 of down_proj[e]), lists the tokens that chose e in token
//      order, and computes H[:, f0:f1] = silu(x Wg^T) * (x Wu^T), or
//      relu(x W1^T + b1), then the slice's share of Y = H Wd^T (+ b2 in the
//      first slice), in fp32 FMA;
//   4. after a cluster barrier each CTA combines a range of tokens:
//      out[t] = sum_k w[t, k] * (sum over the slices of expert e_k of that
//      slice's share of Y), each share read from its CTA through distributed
//      shared memory, summed in slot order and slice order and written once.
//
// Same results as the general path up to fp32 summation order (the same
// definitions, fp32 accumulation throughout); deterministic, no atomics.
// At entry every CTA also asks L2 to prefetch its share of all experts'
// weights, so that weights not yet in L2 come from DRAM while the router
// runs.

#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kRowGroup = 4;      // rows of one expert computed together by a thread
constexpr int kLogitT = 2;        // router: a block of kLogitT tokens ...
constexpr int kLogitE = 4;        // ... x kLogitE experts ...
constexpr int kSplit = 8;         // ... computed by kSplit lanes that split D between them

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
  int T, D, F, E, K, norm;
  int C;      // CTAs in the cluster
  int vec;    // D and F multiples of 4: 16-byte copies
};

__host__ __device__ constexpr int round4(int v) { return (v + 3) & ~3; }
// Length of rows that the lanes of a warp read 16 bytes at a time, each lane
// from its own row: a multiple of 4 floats with an odd number of 16-byte
// units, so the 8 lanes of a quarter warp fall in 8 different bank groups.
__host__ __device__ constexpr int ld_odd4(int v) {
  return ((round4(v) >> 2) & 1) ? round4(v) : round4(v) + 4;
}

// Shared-memory layout (offsets in 4-byte words), the same in every CTA of
// the cluster so that a remote Y row is at the same offset as a local one.
// The weight, H and Y regions are sized for the largest case: one slice of
// all F columns, an expert chosen by all T tokens.
struct SmallLayout {
  int xs, wr, rbs, lg, sel, w, rank, tok, wcnt, cnt, cfirst, scount, w1, w2, b1s, b2s, h, y, total;
  int ldx;    // rows of x, of the router and of the staged gate/up weights
};

// Row counts are kept per group of 4 tokens (the tokens of one warp in the
// top-k, 8 lanes per token).
__host__ __device__ constexpr int token_quads(int T) { return (T + 3) / 4; }

__host__ __device__ inline SmallLayout small_layout(int T, int D, int F, int E, int K, int gated) {
  SmallLayout L;
  L.ldx = ld_odd4(D);
  const int fmax = round4(F);
  int o = 0;
  L.xs = o;     o += round4(T * L.ldx);
  L.wr = o;     o += round4(E * L.ldx);
  L.rbs = o;    o += kSmallMaxExperts;
  L.lg = o;     o += round4(T * E);
  L.sel = o;    o += round4(T * K);
  L.w = o;      o += round4(T * K);
  L.rank = o;   o += round4(T * K);
  L.tok = o;    o += round4(T);
  L.wcnt = o;   o += token_quads(T) * kSmallMaxExperts;
  L.cnt = o;    o += kSmallMaxExperts;
  L.cfirst = o; o += kSmallMaxExperts;
  L.scount = o; o += kSmallMaxExperts;
  L.w1 = o;     o += (gated ? 2 : 1) * fmax * L.ldx;
  L.w2 = o;     o += D * ld_odd4(F);
  L.b1s = o;    o += fmax;
  L.b2s = o;    o += round4(D);
  L.h = o;      o += T * fmax;
  L.y = o;      o += round4(T * D);
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

// Asynchronous copies from global into shared memory: every copy of a
// matrix is in flight at once and no registers hold the data.
__device__ __forceinline__ void cp_async4(float* dst, const float* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(float* dst, const float* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Starts copying a rows x cols block (source rows src_ld floats apart) into
// shared rows of length ld.  vec: cols, src_ld, ld and both addresses are
// multiples of 4 floats (16-byte copies); otherwise 4-byte copies.
__device__ __forceinline__ void stage_async(float* dst, int ld, const float* __restrict__ src,
                                            int src_ld, int rows, int cols, bool vec) {
  if (vec) {
    const int c4 = cols >> 2;
    for (int i = threadIdx.x; i < rows * c4; i += kThreads) {
      const int r = i / c4, c = (i - r * c4) << 2;
      cp_async16(dst + r * ld + c, src + static_cast<size_t>(r) * src_ld + c);
    }
  } else {
    for (int i = threadIdx.x; i < rows * cols; i += kThreads) {
      const int r = i / cols, c = i - r * cols;
      cp_async4(dst + r * ld + c, src + static_cast<size_t>(r) * src_ld + c);
    }
  }
}

// Asks L2 to fetch bytes [lo, hi) of the buffer at base (base, lo and hi
// multiples of 16), in pieces of at most 16 KB spread over the warp's lanes.
__device__ __forceinline__ void prefetch_l2(const void* base, size_t lo, size_t hi, int lane) {
  constexpr size_t kPiece = 16384;
  for (size_t off = lo + static_cast<size_t>(lane) * kPiece; off < hi; off += 32 * kPiece) {
    const size_t n = hi - off < kPiece ? hi - off : kPiece;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(static_cast<const char*>(base) + off),
                 "r"(static_cast<uint32_t>(n))
                 : "memory");
  }
}

// This CTA's share [lo, hi) of a buffer of `bytes` bytes (a multiple of
// 16) split into C shares of whole 16-byte units; empty when lo >= hi.
__device__ __forceinline__ void share_of(size_t bytes, int C, int me, size_t& lo, size_t& hi) {
  const size_t units = bytes >> 4;
  const size_t per = (units + C - 1) / C;
  lo = per * me * 16;
  hi = per * (me + 1) * 16;
  if (hi > bytes) hi = bytes;
}

// True when (v, e) ranks before (bv, be): larger value, then lower index.
__device__ __forceinline__ bool ranks_before(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

template <bool kGated>
__global__ void __launch_bounds__(kThreads, 1) small_layer_f32_kernel(const SmallParams p) {
  extern __shared__ __align__(16) float sm[];
  const int T = p.T, D = p.D, F = p.F, E = p.E, K = p.K, C = p.C;
  const bool vec = p.vec != 0;
  const SmallLayout L = small_layout(T, D, F, E, K, kGated);
  float* xs = sm + L.xs;
  float* wr = sm + L.wr;
  float* rbs = sm + L.rbs;
  float* lg = sm + L.lg;
  int* sel = reinterpret_cast<int*>(sm + L.sel);
  float* wsel = sm + L.w;
  int* rank = reinterpret_cast<int*>(sm + L.rank);
  int* tok = reinterpret_cast<int*>(sm + L.tok);
  int* wcnt = reinterpret_cast<int*>(sm + L.wcnt);
  int* cnt = reinterpret_cast<int*>(sm + L.cnt);
  int* cfirst = reinterpret_cast<int*>(sm + L.cfirst);
  int* scount = reinterpret_cast<int*>(sm + L.scount);
  float* w1 = sm + L.w1;
  float* w2 = sm + L.w2;
  float* b1s = sm + L.b1s;
  float* b2s = sm + L.b2s;
  float* hs = sm + L.h;
  float* ys = sm + L.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const unsigned full = 0xffffffffu;
  const int me = static_cast<int>(cta_rank());
  const int gu_rows = kGated ? 2 * F : F;

  pdl_trigger();
  pdl_wait();
  // ---- x, the router and its bias into shared memory; this CTA's share of
  // every expert's weights into L2
  stage_async(xs, L.ldx, p.x, D, T, D, vec);
  stage_async(wr, L.ldx, p.router, D, E, D, vec);
  if (p.rb) stage_async(rbs, E, p.rb, E, 1, E, false);
  cp_async_commit();
  if (vec && warp == kWarps - 1) {
    size_t lo, hi;
    share_of(static_cast<size_t>(E) * gu_rows * D * sizeof(float), C, me, lo, hi);
    if (lo < hi) prefetch_l2(p.gu, lo, hi, lane);
    share_of(static_cast<size_t>(E) * D * F * sizeof(float), C, me, lo, hi);
    if (lo < hi) prefetch_l2(p.dn, lo, hi, lane);
  }
  cp_async_wait_all();
  __syncthreads();

  // ---- router: logits of every (token, expert).  Eight consecutive lanes
  // share 2 tokens x 4 experts and split D between them (lane c takes the
  // 4-float chunks c, c + 8, ...), so every x and router value a lane reads
  // feeds 4 or 2 FMAs; the eight partial sums are added by a butterfly of
  // shuffles.  Every CTA runs the same code on the same data.
  {
    const int nq = (E + kLogitE - 1) / kLogitE;
    const int items = ((T + kLogitT - 1) / kLogitT) * nq;
    const int c = lane & (kSplit - 1);
    for (int it = 0; it < (items + kThreads / kSplit - 1) / (kThreads / kSplit); ++it) {
      const int item = it * (kThreads / kSplit) + tid / kSplit;    // the same in all 8 lanes
      const bool ok = item < items;
      const int t0 = ok ? (item / nq) * kLogitT : 0, e0 = ok ? (item % nq) * kLogitE : 0;
      const float* xr[kLogitT];
      const float* rr[kLogitE];
#pragma unroll
      for (int u = 0; u < kLogitT; ++u) xr[u] = xs + min(t0 + u, T - 1) * L.ldx;
#pragma unroll
      for (int v = 0; v < kLogitE; ++v) rr[v] = wr + min(e0 + v, E - 1) * L.ldx;
      float a[kLogitT][kLogitE];
#pragma unroll
      for (int u = 0; u < kLogitT; ++u)
#pragma unroll
        for (int v = 0; v < kLogitE; ++v) a[u][v] = 0.f;
      if (ok) {
        int d = 4 * c;
        for (; d + 4 <= D; d += 4 * kSplit) {
          float4 xv[kLogitT];
#pragma unroll
          for (int u = 0; u < kLogitT; ++u) xv[u] = *reinterpret_cast<const float4*>(xr[u] + d);
#pragma unroll
          for (int v = 0; v < kLogitE; ++v) {
            const float4 rv = *reinterpret_cast<const float4*>(rr[v] + d);
#pragma unroll
            for (int u = 0; u < kLogitT; ++u) {
              a[u][v] = fmaf(xv[u].x, rv.x, a[u][v]);
              a[u][v] = fmaf(xv[u].y, rv.y, a[u][v]);
              a[u][v] = fmaf(xv[u].z, rv.z, a[u][v]);
              a[u][v] = fmaf(xv[u].w, rv.w, a[u][v]);
            }
          }
        }
        // D not a multiple of 4: the last D % 4 columns, in the lane whose
        // next chunk would have held them
        if (d < D && d + 4 > D)
          for (; d < D; ++d)
#pragma unroll
            for (int u = 0; u < kLogitT; ++u)
#pragma unroll
              for (int v = 0; v < kLogitE; ++v) a[u][v] = fmaf(xr[u][d], rr[v][d], a[u][v]);
      }
#pragma unroll
      for (int o = 1; o < kSplit; o <<= 1)
#pragma unroll
        for (int u = 0; u < kLogitT; ++u)
#pragma unroll
          for (int v = 0; v < kLogitE; ++v) a[u][v] += __shfl_xor_sync(full, a[u][v], o);
      if (ok && c == 0) {
#pragma unroll
        for (int u = 0; u < kLogitT; ++u)
#pragma unroll
          for (int v = 0; v < kLogitE; ++v) {
            const int t = t0 + u, e = e0 + v;
            if (t < T && e < E) {
              const float acc = p.rb ? a[u][v] + rbs[e] : a[u][v];
              lg[t * E + e] = acc;
              if (me == 0 && p.logits) p.logits[t * E + e] = acc;
            }
          }
      }
    }
  }
  __syncthreads();

  // ---- softmax, top-k and weights: eight lanes per token, lane e holding
  // expert e (lanes e >= E hold nothing and rank after every expert).  The
  // K best by logit (softmax is monotone; a NaN logit ranks last, equal
  // logits to the lower index) are the lanes with fewer than K lanes ranking
  // before them; lane rank k writes slot k.  One ballot per warp then gives,
  // for each selected slot, the earlier tokens of the warp that chose the
  // same expert, and per expert the count of the warp's 4 tokens.
  for (int it = 0; it < (T + kThreads / 8 - 1) / (kThreads / 8); ++it) {
    const int t = it * (kThreads / 8) + tid / 8, e = lane & 7;
    const bool valid = t < T && e < E;
    const float l = valid ? lg[t * E + e] : NAN;
    const float v = isnan(l) ? -INFINITY : l;
    float m = v;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(full, m, o));
    const float ex = (valid && !isnan(l)) ? expf(l - m) : 0.f;
    float s = ex;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) s += __shfl_xor_sync(full, s, o);
    int k = 0;                                 // lanes of this token ranking before e
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float vj = __shfl_sync(full, v, (lane & ~7) | j);
      k += ranks_before(vj, j, v, e) ? 1 : 0;
    }
    const bool chosen = valid && k < K;
    const float pk = chosen ? (isnan(l) ? 0.f : ex / s) : 0.f;
    float psum = pk;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) psum += __shfl_xor_sync(full, psum, o);
    const unsigned int b = __ballot_sync(full, chosen);
    const unsigned int col = 0x01010101u << e;     // expert e's lane in each of the 4 tokens
    if (chosen) {
      const float w = p.norm ? pk / (psum + 1e-9f) : pk;
      sel[t * K + k] = e;
      wsel[t * K + k] = w;
      rank[t * K + k] = __popc(b & col & lanemask_lt());   // completed below
      if (me == 0) {
        if (p.sel64) p.sel64[static_cast<size_t>(t) * K + k] = e;
        if (p.wout) p.wout[static_cast<size_t>(t) * K + k] = w;
      }
    }
    const int quad = it * (kThreads / 32) + warp;
    if (lane < 8 && quad < token_quads(T)) wcnt[quad * kSmallMaxExperts + lane] = __popc(b & col);
  }
  __syncthreads();
  // ---- per expert (warp e), the exclusive prefix of the quads' counts, in
  // place, and the expert's total rows
  if (warp < E) {
    const int e = warp, nquads = token_quads(T);
    int total = 0;
    for (int q0 = 0; q0 < nquads; q0 += 32) {
      const int q = q0 + lane;
      const int c0 = q < nquads ? wcnt[q * kSmallMaxExperts + e] : 0;
      int inc = c0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(full, inc, o);
        if (lane >= o) inc += y;
      }
      if (q < nquads) wcnt[q * kSmallMaxExperts + e] = total + inc - c0;
      total += __shfl_sync(full, inc, 31);
    }
    if (lane == 0) cnt[e] = total;
  }
  __syncthreads();
  // ---- the assignment of CTAs to (expert, slice), computed by every warp
  // with lane e standing for expert e, so all threads of all CTAs agree.
  // Each expert with rows gets one CTA plus its proportional share of the
  // other C - A (rounded down; at most one CTA per 4-column group of F);
  // each CTA still free then goes to the expert with the most rows per CTA
  // (lower index on ties) that can still be split.  The comparison uses
  // n * 65536 / s, exact for these sizes: two different ratios n/s with
  // s <= 16 differ by at least 1/256.
  const int groups4 = (F + 3) >> 2;
  int my_e, my_j, my_s, my_n;
  {
    const int ne = lane < E ? cnt[lane] : 0;
    const int R = __reduce_add_sync(full, ne);
    const int A = __popc(__ballot_sync(full, ne > 0));
    int se = ne > 0 ? 1 + min(groups4 - 1, ne * (C - A) / R) : 0;
    for (int used = __reduce_add_sync(full, se); used < C; ++used) {
      const bool can = se > 0 && se < groups4;
      const unsigned int key =
          can ? (((static_cast<unsigned int>(ne) << 16) / static_cast<unsigned int>(se)) << 3) |
                    static_cast<unsigned int>(7 - lane)
              : 0u;
      const unsigned int best = __reduce_max_sync(full, key);
      if (best == 0u) break;
      if (lane == 7 - static_cast<int>(best & 7u)) ++se;
    }
    int cf = se;                               // inclusive scan over the experts
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      const int y = __shfl_up_sync(full, cf, o);
      if (lane >= o) cf += y;
    }
    cf -= se;
    const unsigned int hit = __ballot_sync(full, lane < 8 && se > 0 && me >= cf && me < cf + se);
    my_e = hit ? __ffs(hit) - 1 : -1;
    const int src = my_e >= 0 ? my_e : 0;
    my_j = me - __shfl_sync(full, cf, src);
    my_s = __shfl_sync(full, se, src);
    my_n = __shfl_sync(full, ne, src);
    if (tid < kSmallMaxExperts) {
      cfirst[tid] = cf;
      scount[tid] = se;
    }
  }
  // this CTA's columns [f0, f1): slices of whole 4-column groups (a CTA
  // left over when every expert is split to single groups has none)
  const int f0 = my_e >= 0 ? 4 * (groups4 * my_j / my_s) : 0;
  const int f1 = my_e >= 0 ? min(F, 4 * (groups4 * (my_j + 1) / my_s)) : 0;
  const int wdt = f1 - f0;
  const int ld2 = ld_odd4(wdt);
  // ---- stage the slice's weights and biases while the rows are listed
  if (my_e >= 0) {
    const float* gu_e = p.gu + static_cast<size_t>(my_e) * gu_rows * D;
    stage_async(w1, L.ldx, gu_e + static_cast<size_t>(f0) * D, D, wdt, D, vec);
    if (kGated)
      stage_async(w1 + wdt * L.ldx, L.ldx, gu_e + static_cast<size_t>(F + f0) * D, D, wdt, D, vec);
    stage_async(w2, ld2, p.dn + static_cast<size_t>(my_e) * D * F + f0, F, D, wdt, vec);
    if (!kGated && p.b1) stage_async(b1s, wdt, p.b1 + static_cast<size_t>(my_e) * F + f0, wdt, 1, wdt, vec);
    if (p.b2 && my_j == 0) stage_async(b2s, D, p.b2 + static_cast<size_t>(my_e) * D, D, 1, D, vec);
  }
  cp_async_commit();
  // each slot's row within its expert: earlier tokens of its warp (above)
  // plus the expert's rows in earlier quads
  for (int i = tid; i < T * K; i += kThreads) {
    const int t = i / K, e = sel[i];
    const int r = rank[i] + wcnt[(t >> 2) * kSmallMaxExperts + e];
    rank[i] = r;
    if (e == my_e) tok[r] = t;
  }
  cp_async_wait_all();
  __syncthreads();

  const int rows = my_n;
  const int groups = (rows + kRowGroup - 1) / kRowGroup;
  const int ldh = round4(wdt);
  // ---- H[:, f0:f1] of expert my_e on its rows (fp32 FMA from shared memory)
  for (int item = tid; item < wdt * groups; item += kThreads) {
    const int f = item % wdt, g = item / wdt;
    float a[kRowGroup], b[kRowGroup];
#pragma unroll
    for (int j = 0; j < kRowGroup; ++j) a[j] = b[j] = 0.f;
    const float* wa = w1 + f * L.ldx;                          // gate row (or W1 row)
    const float* wb = w1 + (kGated ? wdt + f : f) * L.ldx;     // up row
    const float* xr[kRowGroup];
#pragma unroll
    for (int j = 0; j < kRowGroup; ++j) {
      const int r = g * kRowGroup + j;
      xr[j] = xs + (r < rows ? tok[r] : 0) * L.ldx;
    }
    int d = 0;
#pragma unroll 2
    for (; d + 4 <= D; d += 4) {
      float4 xv[kRowGroup];
#pragma unroll
      for (int j = 0; j < kRowGroup; ++j) xv[j] = *reinterpret_cast<const float4*>(xr[j] + d);
      const float4 va = *reinterpret_cast<const float4*>(wa + d);
      const float4 vb = kGated ? *reinterpret_cast<const float4*>(wb + d) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < kRowGroup; ++j) {
        a[j] = fmaf(xv[j].x, va.x, a[j]);
        a[j] = fmaf(xv[j].y, va.y, a[j]);
        a[j] = fmaf(xv[j].z, va.z, a[j]);
        a[j] = fmaf(xv[j].w, va.w, a[j]);
        if (kGated) {
          b[j] = fmaf(xv[j].x, vb.x, b[j]);
          b[j] = fmaf(xv[j].y, vb.y, b[j]);
          b[j] = fmaf(xv[j].z, vb.z, b[j]);
          b[j] = fmaf(xv[j].w, vb.w, b[j]);
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
    const float bias = (!kGated && p.b1) ? b1s[f] : 0.f;
#pragma unroll
    for (int j = 0; j < kRowGroup; ++j) {
      const int r = g * kRowGroup + j;
      if (r < rows)
        hs[r * ldh + f] = kGated ? a[j] / (1.f + expf(-a[j])) * b[j] : fmaxf(a[j] + bias, 0.f);
    }
  }
  __syncthreads();
  // ---- this slice's share of Y = H Wd^T (+ b2 once, in the first slice)
  for (int item = tid; item < D * groups; item += kThreads) {
    const int d = item % D, g = item / D;
    float a[kRowGroup];
#pragma unroll
    for (int j = 0; j < kRowGroup; ++j) a[j] = 0.f;
    const float* wd = w2 + d * ld2;
    const float* hr[kRowGroup];
#pragma unroll
    for (int j = 0; j < kRowGroup; ++j) hr[j] = hs + min(g * kRowGroup + j, rows - 1) * ldh;
    int f = 0;
#pragma unroll 2
    for (; f + 4 <= wdt; f += 4) {
      const float4 v = *reinterpret_cast<const float4*>(wd + f);
#pragma unroll
      for (int j = 0; j < kRowGroup; ++j) {
        const float4 h4 = *reinterpret_cast<const float4*>(hr[j] + f);
        a[j] = fmaf(h4.x, v.x, a[j]);
        a[j] = fmaf(h4.y, v.y, a[j]);
        a[j] = fmaf(h4.z, v.z, a[j]);
        a[j] = fmaf(h4.w, v.w, a[j]);
      }
    }
    for (; f < wdt; ++f) {
      const float v = wd[f];
#pragma unroll
      for (int j = 0; j < kRowGroup; ++j) a[j] = fmaf(hr[j][f], v, a[j]);
    }
    const float bias = (p.b2 && my_j == 0) ? b2s[d] : 0.f;
#pragma unroll
    for (int j = 0; j < kRowGroup; ++j) {
      const int r = g * kRowGroup + j;
      if (r < rows) ys[r * D + d] = a[j] + bias;
    }
  }

  // ---- combine: every slice's share of Y is in its CTA's shared memory
  cluster_barrier();
  const int t_lo = me * T / C, t_hi = (me + 1) * T / C;
  for (int i = tid; i < (t_hi - t_lo) * D; i += kThreads) {
    const int tt = t_lo + i / D, d = i % D;
    float acc = 0.f;
    for (int k = 0; k < K; ++k) {
      const int e = sel[tt * K + k];
      const float* yrow = ys + rank[tt * K + k] * D + d;
      const int c0 = cfirst[e], ns = scount[e];
      float y = 0.f;
      for (int j = 0; j < ns; ++j) y += ld_remote_f32(yrow, static_cast<uint32_t>(c0 + j));
      acc = fmaf(wsel[tt * K + k], y, acc);
    }
    p.out[static_cast<size_t>(tt) * D + d] = acc;
  }
  // no CTA leaves while another may still read its rows
  cluster_barrier();
}

size_t small_smem_bytes(int T, int D, int F, int E, int K, int gated) {
  return sizeof(float) * static_cast<size_t>(small_layout(T, D, F, E, K, gated).total);
}

// The automatic cluster size of a device: 16 CTAs when a cluster of 16 of
// these CTAs (512 threads, the largest shared-memory size this kernel is
// launched with) can be resident at once, else the portable 8.
int auto_cluster(int dev) {
  static std::mutex mu;
  static int cached[64] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  int c = kSmallMinCluster;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kSmallMaxCluster);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmallMaxSmem;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = kSmallMaxCluster;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int nclusters = 0;
  if (cudaOccupancyMaxActiveClusters(&nclusters, small_layer_f32_kernel<true>, &cfg) == cudaSuccess &&
      nclusters >= 1)
    c = kSmallMaxCluster;
  (void)cudaGetLastError();   // a refused query leaves no error behind
  if (dev >= 0 && dev < 64) cached[dev] = c;
  return c;
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
                                   float* logits, int cluster, cudaStream_t s) {
  if (!small_layer_fits(T, D, F, E, K, gated)) return cudaErrorInvalidValue;
  if (cluster != 0 && cluster != kSmallMinCluster && cluster != kSmallMaxCluster)
    return cudaErrorInvalidValue;
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
        err = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (err != cudaSuccess) return err;
      }
      if (dev >= 0 && dev < 64) done[dev] = true;
    }
  }
  const int C = cluster ? cluster : auto_cluster(dev);
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
  p.C = C;
  p.vec = (D % 4 == 0 && F % 4 == 0) ? 1 : 0;
  return launch_k(gated ? small_layer_f32_kernel<true> : small_layer_f32_kernel<false>, dim3(C),
                  dim3(kThreads), small_smem_bytes(T, D, F, E, K, gated), s, pdl_enabled(), C, p);
}

}  // namespace moe
