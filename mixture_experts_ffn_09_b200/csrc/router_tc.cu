// bf16 router on the sm_100a tensor cores: logits = x router^T in fp32 via
// tcgen05.mma (TMA-fed, accumulator in TMEM), then one thread per token
// reads its row of logits from TMEM and does bias, softmax statistics,
// top-k and the renormalised weights in registers.
//
// Same definitions as the CUDA-core router (router.cu): "Mixture-of-Experts
// FFN" (crackedaicode.com), "Compute the experts and router" and "Weight the
// selected outputs"; mojolearn.MoEBlock (router (E, D), lower-index ties,
// norm_topk_prob).  The logits are a dense (T x D) x (D x E) contraction, so
// they go to the tensor cores; everything after is per token.
//
// CTA = 128 tokens (one MMA tile of M = 128), N = E rounded up to 16..256.
// warp 0: TMA producer (x tile 128 x 64 and router tile N x 64 per k-block)
// warp 1: TMEM allocation and the MMA issue
// warps 2..5: one token per thread (TMEM lane = row).  Each warp also counts
// the experts chosen by its 32 tokens: the per-32-token histograms the
// stable permutation uses.
//
// Streaming x is latency-bound per SM, so few row tiles (small T) would use
// few SMs: the D axis is then split over a thread-block cluster of S <= 8
// CTAs.  Each CTA accumulates its share of D in TMEM and stores the partial
// logits into its own slot of rank 0's shared memory (remote stores through
// distributed shared memory); after a cluster barrier rank 0 adds the S
// slots in rank order (fixed order: deterministic, no atomics, no global
// workspace) and runs the per-token epilogue.
//
// Top-k: for K <= 8 one pass over the experts keeps a sorted register list
// of the best K; for larger K, the k-th choice is the best entry that ranks
// strictly after the (k-1)-th in the order (value descending, index
// ascending), one scan over the row per round.
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kSlices = 4;                      // epilogue threads per token
constexpr int kEpiThreads = kSlices * BM;       // warps 2.. (4 per TMEM lane quadrant)
constexpr int THREADS = 64 + kEpiThreads;
constexpr int kDroppedBit = 1 << 30;              // marks a slot the threshold dropped
constexpr int A_BYTES = BM * BK * 2;

template <int NPAD>
struct Cfg {
  static constexpr int B_BYTES = NPAD * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (196 * 1024 / STAGE_BYTES) > 12 ? 12 : (196 * 1024 / STAGE_BYTES);
  static constexpr uint32_t TMEM_COLS = NPAD < 32 ? 32 : NPAD;
  static constexpr int PART_STRIDE = NPAD + 1;   // padded rows: conflict-free column access
  // after the partial logits: the slices' maxima and sums, their candidate
  // lists (value and index, 8 each), then the token's final choices
  static constexpr int SCRATCH_BYTES = (2 * kSlices * BM + 2 * kSlices * 8 * BM + 2 * 8 * BM) * 4;
  static_assert(BM * PART_STRIDE * 4 + SCRATCH_BYTES <= STAGES * STAGE_BYTES,
                "partials and scratch must fit the ring");
};

struct Params {
  int T, E, K, norm, num_kb;
  int S;                  // CTAs per cluster splitting the k-blocks (power of 2, <= num_kb)
  const float* bias;
  float* logits;
  int64_t* sel64;
  float* wout;
  int* idx32;
  float* w32;
  int* blockcounts;   // (ceil(T/32), E) or null
  unsigned int* err;
  int score;               // 0 softmax, 1 sigmoid
  const float* sel_bias;   // (E) or null
  float dyn_threshold;     // > 0: on
  uint8_t* slot_kept;      // (T, K) or null
  float* bal_partial;      // (m_tiles, 3, E) or null
};

template <int NPAD>
struct Tail {
  uint64_t full[Cfg<NPAD>::STAGES];
  uint64_t empty[Cfg<NPAD>::STAGES];
  uint64_t tfull;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int hist[4][kMaxExperts];
};

template <int NPAD>
constexpr size_t smem_bytes() {
  return 1024 + Cfg<NPAD>::STAGES * Cfg<NPAD>::STAGE_BYTES + sizeof(Tail<NPAD>);
}

__device__ __forceinline__ bool ranks_before(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Address of the same shared-memory offset in cluster rank 0.
__device__ __forceinline__ uint32_t map_to_rank0(const void* local) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(smem_u32(local)));
  return r;
}
__device__ __forceinline__ void st_dsmem(uint32_t cluster_addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(v) : "memory");
}


template <int NPAD>
__global__ void __launch_bounds__(THREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const Params p) {
  using C = Cfg<NPAD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * A_BYTES;
  Tail<NPAD>* st = reinterpret_cast<Tail<NPAD>*>(smem + C::STAGES * C::STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = p.S > 1 ? cluster_rank() : 0u;
  const int m0 = (blockIdx.x / p.S) * BM;
  const int E = p.E;
  const int kb_lo = static_cast<int>(rank) * p.num_kb / p.S;         // balanced, never empty
  const int kb_hi = (static_cast<int>(rank) + 1) * p.num_kb / p.S;
  float* part = reinterpret_cast<float*>(sA);   // reuses the ring once the MMAs are done

  pdl_trigger();
  for (int i = threadIdx.x; i < 4 * kMaxExperts; i += THREADS) (&st->hist[0][0])[i] = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], 1);
    }
    mbar_init(&st->tfull, 1);
    mbar_init(&st->mma_done, 1);
    st->abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&st->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the previous forward's kernels may still read this call's outputs
  pdl_wait();
  const uint32_t tmem = st->tmem_base;
  volatile int* abort = &st->abort;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmW);
      int stage = 0;
      uint32_t phase = 0, used = 0, last_parity = 0;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(&st->empty[stage], phase ^ 1u, abort, p.err, SITE_ROUTER_PRODUCER)) break;
        mbar_arrive_expect_tx(&st->full[stage], C::STAGE_BYTES);
        tma_load_2d(&tmX, &st->full[stage], sA + stage * A_BYTES, kb * BK, m0);
        tma_load_2d(&tmW, &st->full[stage], sB + stage * C::B_BYTES, kb * BK, 0);
        used |= 1u << stage;
        last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      int dummy = 0;
      for (int s = 0; s < C::STAGES; ++s)
        if (used & (1u << s))
          mbar_wait(&st->full[s], (last_parity >> s) & 1u, &dummy, p.err, SITE_ROUTER_PRODUCER);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, NPAD);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(&st->full[stage], phase, abort, p.err, SITE_ROUTER_MMA)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
        const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          umma_bf16(tmem, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), idesc,
                    (kb != kb_lo || k != 0) ? 1u : 0u);
        umma_commit(&st->empty[stage]);
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (ok) umma_commit(&st->tfull);
      umma_commit(&st->mma_done);
      int dummy = 0;
      mbar_wait(&st->mma_done, 0, &dummy, p.err, SITE_ROUTER_MMA);
    }
  }
  // Partial logits of this CTA's k-blocks: warps 2..5 (one per TMEM lane
  // quadrant) wait for the MMAs; once every CTA of the cluster is past its
  // MMAs (barrier A, taken by all threads, so rank 0's ring is free) they
  // store the partials of the valid token rows into slot `rank` of rank 0's
  // shared memory - remote stores for the other ranks - and barrier B
  // publishes them to rank 0.
  const int wq = warp & 3;
  const int row = wq * 32 + lane;
  const int slice = warp >= 2 ? (warp - 2) >> 2 : 0;   // which quarter of the experts
  const int t = m0 + row;
  const bool valid = t < p.T;
  bool have = false;
  if (warp >= 2 && slice == 0) {
    // warp-uniform: the TMEM loads below are warp-collective
    have = __all_sync(0xffffffffu, mbar_wait(&st->tfull, 0, abort, p.err, SITE_ROUTER_EPILOGUE));
    if (have) {
      tc_fence_after();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
  }
  __syncwarp();
  if (p.S > 1) cluster_sync_all();                                   // A
  if (have) {
    const uint32_t tb = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    float* dst = part + (static_cast<int>(rank) * BM + row) * C::PART_STRIDE;
    for (int c0 = 0; c0 < E; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tb + c0, r);
      tmem_ld_wait();
      if (!valid) continue;                 // padding rows: nothing to reduce
      if (rank == 0) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j < E) dst[c0 + j] = __uint_as_float(r[j]);
      } else {
        const uint32_t d0 = map_to_rank0(dst + c0);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j < E) st_dsmem(d0 + 4u * j, __uint_as_float(r[j]));
      }
    }
  }
  __syncwarp();
  if (p.S > 1) cluster_sync_all(); else __syncthreads();            // B

  if (warp >= 2 && rank == 0 && !*abort) {
    // ------------------------------------------- kSlices threads per token
    // Thread `slice` of a token owns experts [e_lo, e_hi); the 16 epilogue
    // warps meet at named barrier 1.  The row's logits live in lrow
    // (shared memory), updated in place by the slice owners.
    auto epi_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); };
    int* hist = st->hist[wq];
    float* lrow = part + row * C::PART_STRIDE;
    float* red = part + p.S * BM * C::PART_STRIDE;           // [2][kSlices][BM]
    float* cand_v = red + 2 * kSlices * BM;                  // [kSlices][8][BM]
    int* cand_e = reinterpret_cast<int*>(cand_v + kSlices * 8 * BM);
    int* sel_e = cand_e + kSlices * 8 * BM;                  // [8][BM] final choices
    float* sel_p = reinterpret_cast<float*>(sel_e + 8 * BM);  // [8][BM] their weights
    constexpr int CW = NPAD / kSlices;
    const int e_lo = slice * CW;
    const int e_hi = min(E, e_lo + CW);
    // sum the split partials in rank order, add the bias, write the logits
    float lmax = -INFINITY;
    for (int e = e_lo; e < e_hi; ++e) {
      // padding rows were not copied: they reduce to zeros (their results
      // are never stored, but must stay well defined)
      float v = valid ? lrow[e] : 0.f;
      for (int q = 1; q < p.S; ++q)
        if (valid) v += part[(q * BM + row) * C::PART_STRIDE + e];
      if (p.bias) v += __ldg(p.bias + e);
      if (valid && p.logits) p.logits[static_cast<size_t>(t) * E + e] = v;
      if (isnan(v)) v = -INFINITY;
      lrow[e] = v;
      lmax = fmaxf(lmax, v);
    }
    red[slice * BM + row] = lmax;
    epi_sync();
    float m = red[row];
#pragma unroll
    for (int j = 1; j < kSlices; ++j) m = fmaxf(m, red[j * BM + row]);
    float s = 0.f;
    if (p.score == 0) {
      float ls = 0.f;
      for (int e = e_lo; e < e_hi; ++e) ls += expf(lrow[e] - m);
      red[(kSlices + slice) * BM + row] = ls;
      epi_sync();
#pragma unroll
      for (int j = 0; j < kSlices; ++j) s += red[(kSlices + j) * BM + row];   // fixed order
    }
    // score of expert e: softmax probability or sigmoid of the logit
    auto score = [&](int e) {
      const float l = e < E ? lrow[e] : -INFINITY;
      return p.score == 0 ? expf(l - m) / s : 1.f / (1.f + expf(-l));
    };
    // ranking key: the logit (monotone in either score) unless a selection
    // bias is added to the score; a NaN key (from NaN inputs) ranks as -inf,
    // so every expert stays orderable and a choice is always a real expert
    auto key = [&](int e) {
      const float k = p.sel_bias ? score(e) + __ldg(p.sel_bias + e) : lrow[e];
      return isnan(k) ? -INFINITY : k;
    };
    if (p.K <= 8) {
      // each slice keeps a sorted list of its best entries (value
      // descending, index ascending: a later equal value never overtakes, so
      // the lower index stays ahead); the list holds 8 and only its first K
      // are used.  Thread 0 of the token merges the slices' lists, whose
      // index ranges are disjoint and ascending in slice order.
      float tv[8];
      int te[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        tv[k] = -INFINITY;
        te[k] = 0x7fffffff;
      }
      for (int e = e_lo; e < e_hi; ++e) {
        // insert e into the sorted list: the list is sorted, so "e ranks
        // before entry k" holds from some k on; every entry is then a select
        // from the old list (no chain of dependent swaps)
        const float v = key(e);
        bool b[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) b[k] = ranks_before(v, e, tv[k], te[k]);
#pragma unroll
        for (int k = 7; k > 0; --k) {
          tv[k] = b[k] ? (b[k - 1] ? tv[k - 1] : v) : tv[k];
          te[k] = b[k] ? (b[k - 1] ? te[k - 1] : e) : te[k];
        }
        tv[0] = b[0] ? v : tv[0];
        te[0] = b[0] ? e : te[0];
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        cand_v[(slice * 8 + k) * BM + row] = tv[k];
        cand_e[(slice * 8 + k) * BM + row] = te[k];
      }
      epi_sync();
      if (slice == 0) {
        // Short rolled loops from here on: each router CTA runs this code
        // once per launch with a cold instruction cache, so code size costs
        // more than the few extra shared-memory accesses.  The choices go to
        // sel_e / sel_p (index, unbiased score; the index's top bit marks a
        // slot the threshold dropped).
        int head0 = 0, head1 = 0, head2 = 0, head3 = 0;
        float psum = 0.f;
#pragma unroll 1
        for (int k = 0; k < p.K; ++k) {
          float bv = cand_v[(0 * 8 + head0) * BM + row];
          int be = cand_e[(0 * 8 + head0) * BM + row];
          int bj = 0;
          const float v1 = cand_v[(1 * 8 + head1) * BM + row];
          const int e1 = cand_e[(1 * 8 + head1) * BM + row];
          if (ranks_before(v1, e1, bv, be)) { bv = v1; be = e1; bj = 1; }
          const float v2 = cand_v[(2 * 8 + head2) * BM + row];
          const int e2 = cand_e[(2 * 8 + head2) * BM + row];
          if (ranks_before(v2, e2, bv, be)) { bv = v2; be = e2; bj = 2; }
          const float v3 = cand_v[(3 * 8 + head3) * BM + row];
          const int e3 = cand_e[(3 * 8 + head3) * BM + row];
          if (ranks_before(v3, e3, bv, be)) { bv = v3; be = e3; bj = 3; }
          head0 += bj == 0;
          head1 += bj == 1;
          head2 += bj == 2;
          head3 += bj == 3;
          const float pk = score(be);
          sel_e[k * BM + row] = be;
          sel_p[k * BM + row] = pk;
          psum += pk;
        }
        float ksum = 0.f;
        if (p.dyn_threshold > 0.f) {
#pragma unroll 1
          for (int k = 0; k < p.K; ++k) {
            const float sh = sel_p[k * BM + row] / psum;
            if (k == 0 || sh >= p.dyn_threshold) ksum += sh;
          }
        }
        const float denom = p.norm ? (psum + 1e-9f) : 1.f;
#pragma unroll 1
        for (int k = 0; k < p.K; ++k) {
          const float pk = sel_p[k * BM + row];
          const int e = sel_e[k * BM + row];
          float w = p.norm ? pk / denom : pk;
          bool keep = true;
          if (p.dyn_threshold > 0.f) {
            const float sh = pk / psum;
            keep = k == 0 || sh >= p.dyn_threshold;
            w = keep ? sh / ksum : 0.f;
          }
          sel_p[k * BM + row] = w;                 // the final weight from here on
          if (!keep) sel_e[k * BM + row] = e | kDroppedBit;
          if (valid) {
            const size_t o = static_cast<size_t>(t) * p.K + k;
            if (p.sel64) p.sel64[o] = e;
            if (p.wout) p.wout[o] = w;
            if (p.w32) p.w32[o] = w;
            if (p.idx32) p.idx32[o] = keep ? e : E;   // dropped: no row
            if (p.slot_kept) p.slot_kept[o] = keep ? 1 : 0;
          }
          // per-warp expert counts: one shared atomic per distinct expert
          if (p.blockcounts) {
            const int ek = (valid && keep) ? e : -1;
            const unsigned int same = __match_any_sync(0xffffffffu, ek);
            if (ek >= 0 && lane == __ffs(same) - 1) atomicAdd(&hist[ek], __popc(same));
          }
        }
      }
    } else if (slice == 0) {
      // K > 8: the k-th choice is the best entry that ranks strictly after
      // the (k-1)-th, one scan over the row per round; the chosen index goes
      // to sel64 / idx32 and the unbiased score to the weight buffer until
      // the weights are final
      float* tmpw = p.w32 ? p.w32 : p.wout;
      float lv = INFINITY;
      int le = -1;
      float psum = 0.f;
      for (int k = 0; k < p.K; ++k) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
        for (int e = 0; e < E; ++e) {
          const float v = key(e);
          if (ranks_before(lv, le, v, e) && ranks_before(v, e, bv, be)) {
            bv = v;
            be = e;
          }
        }
        lv = bv;
        le = be;
        const float pk = score(be);
        psum += pk;
        if (valid) {
          const size_t o = static_cast<size_t>(t) * p.K + k;
          tmpw[o] = pk;
          if (p.sel64) p.sel64[o] = be;
          if (p.idx32) p.idx32[o] = be;
        }
      }
      // weights: renormalised scores, then the optional dynamic threshold
      // (the leader stays; the kept shares are renormalised to sum to one)
      float ksum = 0.f;
      if (valid && p.dyn_threshold > 0.f) {
        for (int k = 0; k < p.K; ++k) {
          const float sh = tmpw[static_cast<size_t>(t) * p.K + k] / psum;
          if (k == 0 || sh >= p.dyn_threshold) ksum += sh;
        }
      }
      const float denom = p.norm ? (psum + 1e-9f) : 1.f;
      for (int k = 0; k < p.K; ++k) {
        const size_t o = static_cast<size_t>(t) * p.K + k;
        int ek = -1;
        if (valid) {
          const float pk = tmpw[o];
          const int e = p.idx32 ? p.idx32[o] : static_cast<int>(p.sel64[o]);
          float w = p.norm ? pk / denom : pk;
          bool keep = true;
          if (p.dyn_threshold > 0.f) {
            const float sh = pk / psum;
            keep = k == 0 || sh >= p.dyn_threshold;
            w = keep ? sh / ksum : 0.f;
          }
          if (p.wout) p.wout[o] = w;
          if (p.w32) p.w32[o] = w;
          if (p.slot_kept) p.slot_kept[o] = keep ? 1 : 0;
          if (!keep && p.idx32) p.idx32[o] = E;           // dropped: no row
          if (keep) ek = e;
        }
        if (p.blockcounts) {
          const unsigned int same = __match_any_sync(0xffffffffu, ek);
          if (ek >= 0 && lane == __ffs(same) - 1) atomicAdd(&hist[ek], __popc(same));
        }
      }
    }
    if (slice == 0 && p.blockcounts) {
      __syncwarp();
      const int b = (m0 + wq * 32) / 32;
      if (m0 + wq * 32 < p.T)
        for (int e = lane; e < E; e += 32) p.blockcounts[static_cast<size_t>(b) * E + e] = hist[e];
    }
    if (slice == 0 && p.bal_partial) {
      // per-tile column sums of the scores, the gate and gate > 0, each in
      // row order (deterministic); the 128 threads of slice 0 meet at
      // named barrier 2
      const int tid = row;
      float* bp = p.bal_partial + static_cast<size_t>(blockIdx.x / p.S) * 3 * E;
      // the row's scores replace its logits (score(e) reads only lrow[e])
      for (int e = 0; e < E; ++e) lrow[e] = valid ? score(e) : 0.f;
      asm volatile("bar.sync 2, 128;" ::: "memory");
      for (int e = tid; e < E; e += BM) {
        float acc = 0.f;
        for (int r = 0; r < BM; ++r) acc += part[r * C::PART_STRIDE + e];
        bp[e] = acc;
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");
      // the row's gate: its kept weights renormalised to sum to one (the
      // selection renormalised, whether or not the output weights are)
      for (int e = 0; e < E; ++e) lrow[e] = 0.f;
      if (valid) {
        if (p.K <= 8) {
          float wsum = 0.f;
          for (int k = 0; k < p.K; ++k)
            if (!(sel_e[k * BM + row] & kDroppedBit)) wsum += sel_p[k * BM + row];
          for (int k = 0; k < p.K; ++k) {
            const int e = sel_e[k * BM + row];
            if (!(e & kDroppedBit)) lrow[e] = wsum > 0.f ? sel_p[k * BM + row] / wsum : 0.f;
          }
        } else {
          const float* wk = (p.w32 ? p.w32 : p.wout) + static_cast<size_t>(t) * p.K;
          float wsum = 0.f;
          for (int k = 0; k < p.K; ++k) wsum += wk[k];   // dropped slots hold 0
          for (int k = 0; k < p.K; ++k) {
            const size_t o = static_cast<size_t>(t) * p.K + k;
            const int e = p.idx32 ? p.idx32[o] : static_cast<int>(p.sel64[o]);
            if (e < E) lrow[e] = wsum > 0.f ? wk[k] / wsum : 0.f;
          }
        }
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");
      for (int e = tid; e < E; e += BM) {
        float g = 0.f, c = 0.f;
        for (int r = 0; r < BM; ++r) {
          const float v = part[r * C::PART_STRIDE + e];
          g += v;
          c += v > 0.f ? 1.f : 0.f;
        }
        bp[E + e] = g;
        bp[2 * E + e] = c;
      }
    }
  }
  __syncwarp();

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NPAD>
cudaError_t launch_npad(const RouteArgs& a, cudaStream_t s) {
  CUtensorMap mx, mw;
  if (!make_map(&mx, a.x, static_cast<uint64_t>(a.T), static_cast<uint64_t>(a.D), BM) ||
      !make_map(&mw, a.router, static_cast<uint64_t>(a.E), static_cast<uint64_t>(a.D), NPAD))
    return cudaErrorInvalidValue;
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64 || !done[dev]) {
      err = cudaFuncSetAttribute(router_tc_kernel<NPAD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem_bytes<NPAD>()));
      if (err != cudaSuccess) return err;
      if (dev >= 0 && dev < 64) done[dev] = true;
    }
  }
  Params p;
  p.T = a.T;
  p.E = a.E;
  p.K = a.K;
  p.norm = a.norm;
  p.num_kb = (a.D + BK - 1) / BK;
  p.bias = a.router_bias;
  p.logits = a.logits;
  p.sel64 = a.sel64;
  p.wout = a.wout;
  p.idx32 = a.idx32;
  p.w32 = a.w32;
  p.blockcounts = a.blockcounts;
  p.err = a.err;
  p.score = a.score;
  p.sel_bias = a.sel_bias;
  p.dyn_threshold = a.dyn_threshold;
  p.slot_kept = a.slot_kept;
  p.bal_partial = a.bal_partial;
  const int m_tiles = (a.T + BM - 1) / BM;
  // split D over a cluster when the row tiles alone would leave SMs idle
  int S = 1;
  constexpr int kMaxSlots = (Cfg<NPAD>::STAGES * Cfg<NPAD>::STAGE_BYTES - Cfg<NPAD>::SCRATCH_BYTES) /
                            (BM * Cfg<NPAD>::PART_STRIDE * 4);
  while (S < 8 && m_tiles * S * 2 <= num_sms() && S * 2 <= p.num_kb && S * 2 <= kMaxSlots) S *= 2;
  p.S = S;
  return launch_k(router_tc_kernel<NPAD>, dim3(m_tiles * p.S), dim3(THREADS), smem_bytes<NPAD>(), s,
                  pdl_enabled(), p.S, mx, mw, p);
}

}  // namespace

int router_tc_parts(int T) { return (T + BM - 1) / BM; }

cudaError_t launch_router_tc(const RouteArgs& a, cudaStream_t s) {
  if (a.E <= 16) return launch_npad<16>(a, s);
  if (a.E <= 32) return launch_npad<32>(a, s);
  if (a.E <= 64) return launch_npad<64>(a, s);
  if (a.E <= 128) return launch_npad<128>(a, s);
  return launch_npad<256>(a, s);
}

}  // namespace moe
