// bf16 grouped GEMM on CTA pairs: tcgen05.mma.cta_group::2, M = 256 rows
// (128 per CTA) x N = 256, fp32 accumulators in both CTAs' TMEM.
//
// Same computation and epilogues as the one-CTA kernel in gemm_tc.cu (the
// experts of mojolearn.MoEBlock / the Flax exercise, run as one grouped
// matrix multiplication over the expert-sorted rows; "Mixture of experts",
// dewml.dev, "Expert computation and placement": fp32 accumulation, one
// rounding to bf16).  What changes is the operand traffic: each CTA of a
// pair stages its own 128 rows of A and HALF of the 256 B rows, and the pair's
// MMA reads both CTAs' shared memory, so a CTA moves 32 KB per k-block for
// the same 128 x 256 x 64 product that costs 48 KB on one CTA.  The saved
// shared memory buys a 6-stage ring (192 KB: the ring starts at the
// 1024-byte-aligned base of dynamic shared memory, and the tile table keeps
// only the per-expert tile starts and row offsets) and 8 KB of output
// staging per epilogue warp.
//
// Cluster of 2 CTAs (rank 0 = leader), 192 threads each:
//   warp 0 (both)   TMA producer for this CTA's A rows and B half; the loads
//                   complete on the LEADER's full barrier, whose expected
//                   bytes the leader's producer posts for the pair;
//   warp 1 (both)   allocates 512 TMEM columns for the pair
//                   (tcgen05.alloc.cta_group::2); in the leader one lane
//                   issues the pair's MMAs and commits, multicast to both
//                   CTAs, the stage releases and accumulator completions;
//   warps 2..5      epilogue of this CTA's 128 rows; each warp's release of
//                   an accumulator arrives on the leader's barrier (8
//                   arrivals per tile).  A warp converts 128 columns of its
//                   32 rows (a row per lane, as TMEM hands them out) into
//                   its staging area, then stores them as whole 256-byte
//                   row runs, two rows per instruction: 4 full lines per
//                   store instead of 32 scattered 16-byte pieces.
// For the gated expert the leader stages the 128 gate rows and the peer the
// matching 128 up rows, so accumulator columns [0,128) are gate and
// [128,256) up in both CTAs, exactly as in the one-CTA kernel.
//
// The last wave is split: when fewer tiles are left than pairs, the last
// `pairs` tiles each run as two work items over the two halves of the
// k-blocks.  The first half stores its fp32 accumulator to a scratch area
// and sets one flag per epilogue warp; the second half waits (bounded) for
// the flag of its warp and adds the stored partial before its own epilogue.
// The two halves are consecutive items, so the first is always handed out
// before the second, and the sum is always (second half) + (first half):
// deterministic.  Pairs that would have idled through a mostly empty last
// wave take half tiles instead.
//
// Tiles are handed out dynamically, in order: the leader's producer takes
// the next tile index from a global counter (zeroed each forward by the
// scatter kernel) and publishes it through a small ring in shared memory to
// the leader's MMA issuer and epilogue warps and, by a store into the peer's
// shared memory and a remote barrier arrival, to the peer's producer and
// epilogue warps.  Row blocks that share a weight tile are then taken within
// a few tiles of each other wherever the pairs stand, so the weight tile is
// read from DRAM once and served from L2 to the others; and pairs that draw
// cheap tiles (swapped tails) simply take more of them.
//
// A pair tile covers 256 rows of one expert; rows past the expert's end are
// computed and not stored.  The exception is an expert's last row block when
// it holds at most `swap_max` rows (a short tail): that tile runs with the
// operands swapped.  The weight rows become the MMA's M = 256 and the tail's
// token rows its N (16, 32, 64 or 128; half from each CTA), so the tensor
// cores do not spend a full 256-row tile on a few rows.  For the gated
// expert each CTA stages its 64 gate rows and the matching 64 up rows
// interleaved in groups of 16, so the gate and up values of one feature land
// in TMEM lanes i and i^16 of the same warp and meet through one shuffle.
// The epilogue writes the transposed result straight to the row-major output.
// A swapped k-block takes two copies per CTA, as a regular one does: the
// token rows in one box of 8, 16, 32 or 64 rows (N = 16..128), and the
// interleaved gate/up rows through one 4-D view of the weights.
// No load uses cluster multicast.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BMC = 128;                      // rows per CTA
constexpr int BMP = 256;                      // rows per pair
constexpr int BK = 64;
constexpr int BN_MMA = 256;
constexpr int STAGES = 6;
constexpr int A_BYTES = BMC * BK * 2;         // 16 KB
constexpr int B_BYTES = (BN_MMA / 2) * BK * 2;  // 16 KB (this CTA's half)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int WB_BOX = 16;      // gate (then up) rows per group of the interleaved staging
constexpr int kSwapMax = 128;   // longest tail that may run swapped (N = 128)
constexpr int SCHED = 8;        // tile indices in flight from the scheduler to the roles
// Readers of each published tile index, who release its slot: the leader's
// MMA issuer and 4 epilogue warps, the peer's producer and 4 epilogue warps.
constexpr int SCHED_READERS = 10;

// Token-row views for swapped tails: box heights 8, 16, 32 and 64 rows.
struct TokMaps {
  CUtensorMap m[4];
};

enum { kSiluGated = 0, kReluBias = 1, kBias = 2 };

struct Params {
  const int* perm;    // gathered A: sorted row -> (token, slot); null otherwise
  int K;
  const int* offsets;
  int E;
  int n_out;
  int num_kb;
  int b_rows;
  int up_off;
  __nv_bfloat16* out;
  const float* bias;
  unsigned int* err;
  int swap_max;       // an expert's last block of at most this many rows runs swapped (0: never)
  int* tile_counter;  // next tile to hand out; zero at launch
  float* split_partial;   // first halves' fp32 accumulators (split last wave), or null
  int* split_flags;       // one per split unit, CTA and epilogue warp; zero at launch
  int split_cap;          // split units the scratch holds
};

// One scheduled work item: tile t over k-blocks [kb0, kb1); half -1 for a
// whole tile, else 0 / 1 for the halves of split unit `slot`.
struct Item {
  int t, kb0, kb1, half, slot;
};

// The first `total - S` items are whole tiles; the last S tiles follow as
// pairs of half items.
__device__ __forceinline__ Item decode_item(int w, int total, int S, int num_kb) {
  Item it;
  const int first = total - S;
  if (w < first) {
    it.t = w;
    it.kb0 = 0;
    it.kb1 = num_kb;
    it.half = -1;
    it.slot = 0;
    return it;
  }
  const int j = w - first;
  const int mid = num_kb / 2;
  it.t = first + (j >> 1);
  it.half = j & 1;
  it.slot = j >> 1;
  it.kb0 = it.half ? mid : 0;
  it.kb1 = it.half ? num_kb : mid;
  return it;
}

__device__ __forceinline__ void flag_release(int* f) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(f), "r"(1) : "memory");
}
__device__ __forceinline__ int flag_acquire(const int* f) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
  return v;
}

struct Tail {
  uint64_t full[STAGES];     // leader: both CTAs' loads of a stage
  uint64_t empty[STAGES];    // both: the pair's MMAs have read the stage
  uint64_t tfull[2];         // both: accumulator ready
  uint64_t tempty[2];        // leader: 8 epilogue warps released the accumulator
  uint64_t mma_done;
  uint64_t sfull[SCHED];     // both: the slot holds the next tile index for this CTA
  uint64_t sempty[SCHED];    // leader: every reader of the slot has taken it
  int sched_tile[SCHED];     // tile index, -1 = no more tiles
  uint32_t tmem_base;
  int abort;
  int total_tiles;
  int tile_start[kMaxExperts + 1];
  int off[kMaxExperts + 1];
  uint32_t wfast[(kMaxExperts + 31) / 32];   // bit e: expert e's tiles go weight block fastest
};

constexpr size_t kTailBytes = (sizeof(Tail) + 127) & ~size_t(127);
constexpr int kEpiStageBytes = 32 * 256;      // per epilogue warp: 32 rows x 256 B
constexpr size_t kSmemBytes = STAGES * STAGE_BYTES + kTailBytes + 4 * kEpiStageBytes;

// Rows of 256 B staged by the epilogue warp, 16-byte unit u of row r at
// unit u ^ (r & 7): the row-per-lane writes and the run-per-half-warp reads
// are both free of bank conflicts.
__device__ __forceinline__ void epi_put(uint8_t* stg, int r, int u, const uint32_t* w) {
  *reinterpret_cast<uint4*>(stg + r * 256 + ((u ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
}
// Stores the staged 32 x 128 block: each instruction writes two 256-byte row
// runs.  Rows at or beyond row_end and columns at or beyond n_out are skipped.
__device__ __forceinline__ void epi_flush(const uint8_t* stg, int lane, __nv_bfloat16* out, int grow0,
                                          int row_end, int col_base, int n_out) {
  __syncwarp();
  const int u = lane & 15;
  const int col = col_base + u * 8;
#pragma unroll 4
  for (int i = 0; i < 16; ++i) {
    const int r = 2 * i + (lane >> 4);
    const uint4 v = *reinterpret_cast<const uint4*>(stg + r * 256 + ((u ^ (r & 7)) << 4));
    const int grow = grow0 + r;
    if (grow < row_end && col < n_out)
      *reinterpret_cast<uint4*>(out + static_cast<size_t>(grow) * n_out + col) = v;
  }
  __syncwarp();
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void st_cluster_s32(uint32_t cluster_addr, int v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
// Reads the index of the i-th tile this CTA works on from the scheduler
// ring and releases the slot on the leader (any role but the leader's
// producer, which writes it).  -1: no more tiles, or the wait gave up.
__device__ __forceinline__ int sched_take(Tail* st, int i, volatile int* abort, unsigned int* err,
                                          unsigned int site) {
  const int slot = i % SCHED;
  if (!mbar_wait_cluster(&st->sfull[slot], (i / SCHED) & 1u, abort, err, site)) return -1;
  const int t = st->sched_tile[slot];
  mbar_arrive_cluster(map_to_rank(&st->sempty[slot], 0));
  return t;
}
// TMA load into this CTA's shared memory whose completion is counted on the
// barrier at `bar_cluster_addr` (the leader's, for a pair).
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* map, uint32_t bar_cluster_addr,
                                                 void* dst, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d_pair(const CUtensorMap* map, uint32_t bar_cluster_addr,
                                                 void* dst, int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(c0), "r"(c1), "r"(c2),
      "r"(c3)
      : "memory");
}
// Gathered variant: 4 token rows of x (box 64 x 1) into 512 bytes of this
// CTA's shared memory, completing on the leader's barrier.
__device__ __forceinline__ void tma_gather4_pair(const CUtensorMap* map, uint32_t bar_cluster_addr,
                                                 void* dst, int c0, int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4"
      ".mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(c0), "r"(r0), "r"(r1),
      "r"(r2), "r"(r3)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives once on the barrier at this offset in both CTAs of the pair when
// the pair's MMAs issued so far have completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}

// Expert, row block and weight block of tile t.  An expert's tiles are
// ordered with the row block fastest (consecutive tiles share a weight
// block, and the expert's token rows are re-read for every weight block),
// or, for an expert with more token rows than weight rows, with the weight
// block fastest (consecutive tiles share the token rows, and the smaller
// weights are the operand re-read).  Either way the operand that must stay
// in L2 between its uses is the smaller one.
__device__ __forceinline__ void decode_tile(const Tail* st, int E, int n_tiles, int t, int& e,
                                            int& m_blk, int& n_blk) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (st->tile_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  e = lo;
  const int local = t - st->tile_start[e];
  if ((st->wfast[e >> 5] >> (e & 31)) & 1u) {
    m_blk = local / n_tiles;
    n_blk = local - m_blk * n_tiles;
  } else {
    const int mt = (st->tile_start[e + 1] - st->tile_start[e]) / n_tiles;
    n_blk = local / mt;
    m_blk = local - n_blk * mt;
  }
}

// Rows of a swapped tail tile (1..255), or 0 for a regular tile.  Every row
// block but an expert's last has more than 255 rows left, so only the last
// can qualify.
__device__ __forceinline__ int swap_rows(const Tail* st, int swap_max, int e, int m_blk) {
  const int left = st->off[e + 1] - st->off[e] - m_blk * BMP;
  return left <= swap_max ? left : 0;
}
// The swapped tile's N: 16, 32, 64 or 128 (index 0..3 of the token views).
__device__ __forceinline__ int swap_idx(int rows) {
  return rows <= 16 ? 0 : rows <= 32 ? 1 : rows <= 64 ? 2 : 3;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int EPI, bool GATHER>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmGU,
                             const __grid_constant__ TokMaps tmT, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if ((smem_u32(smem_raw) & 1023u) != 0) {   // the ring needs 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(p.err, DEVERR_BOUNDS);
    return;
  }
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  Tail* st = reinterpret_cast<Tail*>(smem + STAGES * STAGE_BYTES);
  uint8_t* epi_stage = smem + STAGES * STAGE_BYTES + kTailBytes;

  constexpr int BN_OUT = (EPI == kSiluGated) ? 128 : 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int E = p.E;
  const int n_tiles = (p.n_out + BN_OUT - 1) / BN_OUT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&st->tfull[a], 1);
      mbar_init(&st->tempty[a], 8);
    }
    mbar_init(&st->mma_done, 1);
    for (int j = 0; j < SCHED; ++j) {
      mbar_init(&st->sfull[j], 1);
      mbar_init(&st->sempty[j], SCHED_READERS);
    }
    st->abort = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (!GATHER && p.swap_max > 0) {
      for (int j = 0; j < 4; ++j) tma_prefetch_desc(&tmT.m[j]);
      if (EPI == kSiluGated) tma_prefetch_desc(&tmGU);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(&st->tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  pdl_trigger();
  // the expert offsets come from the permutation kernel
  pdl_wait();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int j = 0; j < (kMaxExperts + 31) / 32; ++j) st->wfast[j] = 0u;
    for (int e = 0; e < E; ++e) {
      const int o0 = p.offsets[e], o1 = p.offsets[e + 1];
      const int mt = (o1 - o0 + BMP - 1) / BMP;
      st->off[e] = o0;
      st->tile_start[e] = acc;
      acc += mt * n_tiles;
      if (o1 - o0 > p.b_rows) st->wfast[e >> 5] |= 1u << (e & 31);
    }
    st->off[E] = p.offsets[E];
    st->tile_start[E] = acc;
    st->total_tiles = acc;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();     // the leader's barriers exist before the peer signals them
  tc_fence_after();

  const uint32_t tmem = st->tmem_base;
  const int total = st->total_tiles;
  volatile int* abort = &st->abort;
  // the last min(pairs, tiles) tiles run as k-halves when scratch is given
  const int n_pairs = static_cast<int>(gridDim.x >> 1);
  const int S = (p.split_partial && p.num_kb >= 2)
                    ? min(min(n_pairs, total), p.split_cap)
                    : 0;
  const int total_items = total + S;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Lane 0 waits for free stages (and, in the leader, posts the pair's
    // expected bytes); with a gathered A every lane fetches 4 of this CTA's
    // 128 token rows.
    int stage = 0;
    uint32_t phase = 0, used = 0, last_parity = 0;
    const int rows_live = st->off[E];
    for (int i = 0;; ++i) {
      // the next tile: the leader takes it from the counter and publishes it
      // to both CTAs; the peer reads it from its own ring
      int t = -1;
      if (lane == 0) {
        if (leader) {
          const int slot = i % SCHED;
          if (mbar_wait(&st->sempty[slot], ((i / SCHED) & 1u) ^ 1u, abort, p.err,
                        SITE_PAIR_PRODUCER)) {
            t = atomicAdd(p.tile_counter, 1);
            if (t >= total_items) t = -1;
          }
          st->sched_tile[slot] = t;
          st_cluster_s32(map_to_rank(&st->sched_tile[slot], 1), t);
          mbar_arrive(&st->sfull[slot]);
          mbar_arrive_cluster(map_to_rank(&st->sfull[slot], 1));
        } else {
          t = sched_take(st, i, abort, p.err, SITE_PAIR_PRODUCER);
        }
      }
      t = __shfl_sync(0xffffffffu, t, 0);
      if (t < 0) break;
      if (!__shfl_sync(0xffffffffu, lane == 0 ? static_cast<int>(!*abort) : 0, 0)) break;
      const Item it = decode_item(t, total, S, p.num_kb);
      int e, m_blk, n_blk;
      decode_tile(st, E, n_tiles, it.t, e, m_blk, n_blk);
      const int rowA = st->off[e] + m_blk * BMP + static_cast<int>(rank) * BMC;
      const int rowB = (EPI == kSiluGated)
                           ? e * p.b_rows + n_blk * 128 + (leader ? 0 : p.up_off)
                           : e * p.b_rows + n_blk * 256 + static_cast<int>(rank) * 128;
      int tok[4] = {0, 0, 0, 0};
      if (GATHER) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = rowA + 4 * lane + q;
          tok[q] = r < rows_live ? __ldg(p.perm + r) / p.K : 0;
        }
      }
      bool ok = true;
      const int sw = GATHER ? 0 : swap_rows(st, p.swap_max, e, m_blk);
      if (sw) {
        // swapped tail: this CTA's weight rows into the B slot, its half of
        // the tail's token rows (nt/2) into the A slot
        const int si = swap_idx(sw);
        const int nt = 16 << si;
        const int row_tok = st->off[e] + m_blk * BMP + static_cast<int>(rank) * (nt / 2);
        // gated: the first 16-row group of this CTA's 64 features, counted in
        // the weights' 16-row groups (the gated swap requires F % 16 == 0)
        const int g0 = (e * p.b_rows + n_blk * 128 + static_cast<int>(rank) * 64) / WB_BOX;
        for (int kb = it.kb0; kb < it.kb1; ++kb) {
          int good = 1;
          if (lane == 0) {
            good = mbar_wait(&st->empty[stage], phase ^ 1u, abort, p.err, SITE_PAIR_PRODUCER) ? 1 : 0;
            if (good && leader) mbar_arrive_expect_tx(&st->full[stage], 2 * B_BYTES + nt * BK * 2);
          }
          if (!__shfl_sync(0xffffffffu, good, 0)) { ok = false; break; }
          const uint32_t fb = map_to_rank(&st->full[stage], 0);
          if (lane == 0) {
            // box (64 k, 16 rows, gate/up, 4 groups) lands as smem rows
            // 32q + i (gate) and 32q + 16 + i (up) of group q
            if (EPI == kSiluGated)
              tma_load_4d_pair(&tmGU, fb, sB + stage * B_BYTES, kb * BK, 0, 0, g0);
            else
              tma_load_2d_pair(&tmB, fb, sB + stage * B_BYTES, kb * BK, rowB);
            tma_load_2d_pair(&tmT.m[si], fb, sA + stage * A_BYTES, kb * BK, row_tok);
            used |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        continue;
      }
      for (int kb = it.kb0; kb < it.kb1; ++kb) {
        int good = 1;
        if (lane == 0) {
          good = mbar_wait(&st->empty[stage], phase ^ 1u, abort, p.err, SITE_PAIR_PRODUCER) ? 1 : 0;
          if (good && leader) mbar_arrive_expect_tx(&st->full[stage], 2 * STAGE_BYTES);
        }
        if (!__shfl_sync(0xffffffffu, good, 0)) { ok = false; break; }
        const uint32_t fb = map_to_rank(&st->full[stage], 0);
        if (GATHER)
          tma_gather4_pair(&tmA, fb, sA + stage * A_BYTES + lane * 512, kb * BK, tok[0], tok[1],
                           tok[2], tok[3]);
        if (lane == 0) {
          if (!GATHER) tma_load_2d_pair(&tmA, fb, sA + stage * A_BYTES, kb * BK, rowA);
          tma_load_2d_pair(&tmB, fb, sB + stage * B_BYTES, kb * BK, rowB);
          used |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
    // Let issued loads land before the CTA can leave: the leader sees them
    // on its full barriers; the peer's complete on the leader's, so the
    // peer waits for the pair's MMAs to have released its stages.
    if (lane == 0) {
      int dummy = 0;
      for (int s = 0; s < STAGES; ++s)
        if (used & (1u << s)) {
          const uint32_t par = (last_parity >> s) & 1u;
          if (leader) mbar_wait(&st->full[s], par, &dummy, p.err, SITE_PAIR_PRODUCER);
          else mbar_wait(&st->empty[s], par, &dummy, p.err, SITE_PAIR_PRODUCER);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA (leader)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = idesc_bf16_f32(BMP, BN_MMA);
      int stage = 0;
      uint32_t phase = 0;
      for (int i = 0;; ++i) {
        const int t = sched_take(st, i, abort, p.err, SITE_PAIR_MMA);
        if (t < 0) break;
        const int acc = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        if (!mbar_wait(&st->tempty[acc], aph ^ 1u, abort, p.err, SITE_PAIR_MMA)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN_MMA;
        bool ok = true;
        int sw = 0;
        const Item it = decode_item(t, total, S, p.num_kb);
        if (!GATHER && p.swap_max > 0) {
          int e, m_blk, n_blk;
          decode_tile(st, E, n_tiles, it.t, e, m_blk, n_blk);
          sw = swap_rows(st, p.swap_max, e, m_blk);
        }
        if (sw) {
          // swapped tail: A = the weight rows (B slot), B = the token rows (A slot)
          const uint32_t idesc_sw = idesc_bf16_f32(BMP, 16 << swap_idx(sw));
          for (int kb = it.kb0; kb < it.kb1; ++kb) {
            if (!mbar_wait(&st->full[stage], phase, abort, p.err, SITE_PAIR_MMA)) { ok = false; break; }
            tc_fence_after();
            const uint32_t w0 = smem_u32(sB + stage * B_BYTES);
            const uint32_t x0 = smem_u32(sA + stage * A_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_bf16_pair(d, sw128_kmajor_desc(w0 + k * 32), sw128_kmajor_desc(x0 + k * 32),
                             idesc_sw, (kb != it.kb0 || k != 0) ? 1u : 0u);
            umma_commit_pair(&st->empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
        } else {
          for (int kb = it.kb0; kb < it.kb1; ++kb) {
            if (!mbar_wait(&st->full[stage], phase, abort, p.err, SITE_PAIR_MMA)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
            const uint32_t b0 = smem_u32(sB + stage * B_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_bf16_pair(d, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), idesc,
                             (kb != it.kb0 || k != 0) ? 1u : 0u);
            umma_commit_pair(&st->empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
        }
        if (!ok) break;
        umma_commit_pair(&st->tfull[acc]);
      }
      umma_commit_pair(&st->mma_done);
      int dummy = 0;
      mbar_wait(&st->mma_done, 0, &dummy, p.err, SITE_PAIR_MMA);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int lane_base = (warp & 3) * 32;
    const uint32_t tempty_leader0 = map_to_rank(&st->tempty[0], 0);
    const uint32_t tempty_leader1 = map_to_rank(&st->tempty[1], 0);
    for (int i = 0;; ++i) {
      int t = lane == 0 ? sched_take(st, i, abort, p.err, SITE_PAIR_EPILOGUE) : -1;
      t = __shfl_sync(0xffffffffu, t, 0);
      if (t < 0) break;
      const Item it = decode_item(t, total, S, p.num_kb);
      int e, m_blk, n_blk;
      decode_tile(st, E, n_tiles, it.t, e, m_blk, n_blk);
      const int acc = i & 1;
      const uint32_t aph = (i >> 1) & 1;
      // every lane must agree before the warp-collective TMEM loads
      const bool got = mbar_wait(&st->tfull[acc], aph, abort, p.err, SITE_PAIR_EPILOGUE);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tb = tmem + (static_cast<uint32_t>(lane_base) << 16) + acc * BN_MMA;
      // split last wave: this warp's slice of the unit's partial accumulator,
      // column-major over its 128 rows (column c of row r at c * 128 + r)
      const int prow = lane_base + lane;
      float* part = it.half >= 0
                        ? p.split_partial + (static_cast<size_t>(it.slot) * 2 + rank) * (256 * 128)
                        : nullptr;
      int* flag = it.half >= 0 ? p.split_flags + (it.slot * 2 + static_cast<int>(rank)) * 4 + (warp & 3)
                               : nullptr;
      if (it.half == 0) {
        // first half: hand the raw accumulator to the second half
#pragma unroll 1
        for (int c = 0; c < BN_MMA / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tb + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) part[(c * 32 + j) * 128 + prow] = __uint_as_float(v[j]);
        }
        __threadfence();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          flag_release(flag);
          mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        }
        continue;
      }
      if (it.half == 1) {
        // second half: wait (bounded) for the first half's partial
        int ready = 1;
        if (lane == 0) {
          const unsigned long long t0 = globaltimer();
          while (flag_acquire(flag) == 0) {
            if (*abort || globaltimer() - t0 > kWaitTimeoutNs) {
              if (!*abort) atomicOr(p.err, DEVERR_TIMEOUT | SITE_PAIR_EPILOGUE);
              *abort = 1;
              ready = 0;
              break;
            }
            __nanosleep(256);
          }
        }
        if (!__shfl_sync(0xffffffffu, ready, 0)) break;
        __threadfence();
      }
      // adds the first half's partial to columns [c0, c0 + 32) of this row
      auto add_partial = [&](uint32_t (&v)[32], int c0) {
        if (it.half == 1) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            v[j] = __float_as_uint(__uint_as_float(v[j]) + __ldcg(part + (c0 + j) * 128 + prow));
        }
      };
      const int sw = GATHER ? 0 : swap_rows(st, p.swap_max, e, m_blk);
      if (sw) {
        // swapped tail: this thread's TMEM lane is one weight row (an output
        // feature), its columns the tail's token rows
        const int row0 = st->off[e] + m_blk * BMP;
        const int nchunks = (sw + 31) >> 5;
        if (EPI == kSiluGated) {
          // lane i < 16 holds gate, lane i + 16 up, of the same feature f
          const bool hi = lane >= 16;
          const int f = n_blk * 128 + static_cast<int>(rank) * 64 + (warp & 3) * WB_BOX + (lane & 15);
          const bool fvalid = f < p.n_out;
#pragma unroll 1
          for (int c = 0; c < nchunks; ++c) {
            uint32_t v[32];
            tmem_ld32(tb + c * 32, v);
            tmem_ld_wait();
            add_partial(v, c * 32);
            // the low lane finishes tokens 32c..32c+15, the high lane 32c+16..32c+31
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float give = __uint_as_float(hi ? v[j] : v[16 + j]);
              const float got = __shfl_xor_sync(0xffffffffu, give, 16);
              const float g = hi ? got : __uint_as_float(v[j]);
              const float u = hi ? __uint_as_float(v[16 + j]) : got;
              const int tok = c * 32 + (hi ? 16 : 0) + j;
              if (fvalid && tok < sw)
                p.out[static_cast<size_t>(row0 + tok) * p.n_out + f] =
                    __float2bfloat16_rn(silu_bf16_epilogue(g) * u);
            }
          }
        } else {
          const int dcol = n_blk * 256 + static_cast<int>(rank) * 128 + lane_base + lane;
          const bool dvalid = dcol < p.n_out;
          const float b =
              (p.bias && dvalid) ? __ldg(p.bias + static_cast<size_t>(e) * p.n_out + dcol) : 0.f;
#pragma unroll 1
          for (int c = 0; c < nchunks; ++c) {
            uint32_t v[32];
            tmem_ld32(tb + c * 32, v);
            tmem_ld_wait();
            add_partial(v, c * 32);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int tok = c * 32 + j;
              if (dvalid && tok < sw) {
                float a = __uint_as_float(v[j]) + b;
                if (EPI == kReluBias) a = fmaxf(a, 0.f);
                p.out[static_cast<size_t>(row0 + tok) * p.n_out + dcol] = __float2bfloat16_rn(a);
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        continue;
      }
      const int grow0 = st->off[e] + m_blk * BMP + static_cast<int>(rank) * BMC + lane_base;
      const int row_end = st->off[e + 1];
      uint8_t* stg = epi_stage + (warp - 2) * kEpiStageBytes;
      if (EPI == kSiluGated) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(tb + c * 32, g);
          tmem_ld32(tb + 128 + c * 32, u);
          tmem_ld_wait();
          add_partial(g, c * 32);
          add_partial(u, 128 + c * 32);
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float g0 = __uint_as_float(g[2 * j]), g1 = __uint_as_float(g[2 * j + 1]);
            const float u0 = __uint_as_float(u[2 * j]), u1 = __uint_as_float(u[2 * j + 1]);
            w[j] = pack_bf16x2(silu_bf16_epilogue(g0) * u0, silu_bf16_epilogue(g1) * u1);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) epi_put(stg, lane, c * 4 + q, w + 4 * q);
        }
        epi_flush(stg, lane, p.out, grow0, row_end, n_blk * 128, p.n_out);
      } else {
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            const int c = h * 4 + cc;
            uint32_t v[32];
            tmem_ld32(tb + c * 32, v);
            tmem_ld_wait();
            add_partial(v, c * 32);
            const int col0 = n_blk * 256 + c * 32;
            const float* bias = p.bias ? p.bias + static_cast<size_t>(e) * p.n_out + col0 : nullptr;
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float a0 = __uint_as_float(v[2 * j]), a1 = __uint_as_float(v[2 * j + 1]);
              if (bias) {
                if (col0 + 2 * j < p.n_out) a0 += __ldg(bias + 2 * j);
                if (col0 + 2 * j + 1 < p.n_out) a1 += __ldg(bias + 2 * j + 1);
              }
              if (EPI == kReluBias) {
                a0 = fmaxf(a0, 0.f);
                a1 = fmaxf(a1, 0.f);
              }
              w[j] = pack_bf16x2(a0, a1);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) epi_put(stg, lane, cc * 4 + q, w + 4 * q);
          }
          epi_flush(stg, lane, p.out, grow0, row_end, n_blk * 256 + h * 128, p.n_out);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
    }
  }

  tc_fence_before();
  __syncwarp();
  __syncthreads();
  cluster_sync_all();     // neither CTA frees TMEM while its peer may still use it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
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

bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
              uint32_t box_rows = 128u) {
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

// The gated weights (E x [F gate rows; F up rows] x Kdim) seen as 4-D:
// (k, row in a 16-row group, gate or up (F rows apart), group).  Only gate
// groups are addressed, so the last group plus F stays inside the tensor.
bool make_gate_up_map(CUtensorMap* m, const void* W, int E, int F, int Kdim) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || F % WB_BOX != 0) return false;
  const uint64_t row = static_cast<uint64_t>(Kdim) * 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(Kdim), static_cast<cuuint64_t>(WB_BOX), 2,
                              static_cast<cuuint64_t>(F) * (2 * E - 1) / WB_BOX};
  const cuuint64_t strides[3] = {row, row * F, row * WB_BOX};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(WB_BOX), 2u,
                             static_cast<cuuint32_t>(BMC / (2 * WB_BOX))};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(W), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, bool GATHER>
cudaError_t launch_epi(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& gu,
                       const TokMaps& tok, const Params& p, int clusters, cudaStream_t s) {
  static std::mutex mu;
  static int resident[64] = {};    // pairs that fit on the device at once (0: not asked yet)
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  int fit = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64 || resident[dev] == 0) {
      err = cudaFuncSetAttribute(grouped_gemm_pair_kernel<EPI, GATHER>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kSmemBytes));
      if (err != cudaSuccess) return err;
      // the grid is persistent: every pair should be resident from the start
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * clusters);
      cfg.blockDim = dim3(THREADS);
      cfg.dynamicSmemBytes = kSmemBytes;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 2;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_pair_kernel<EPI, GATHER>, &cfg) !=
              cudaSuccess ||
          n <= 0) {
        cudaGetLastError();            // the query is advisory: fall back to one pair per 2 SMs
        n = num_sms() / 2;
      }
      fit = n;
      if (dev >= 0 && dev < 64) resident[dev] = n;
    } else {
      fit = resident[dev];
    }
  }
  if (clusters > fit) clusters = fit;
  return launch_k(grouped_gemm_pair_kernel<EPI, GATHER>, dim3(2 * clusters), dim3(THREADS),
                  kSmemBytes, s, pdl_enabled(), 2, a, b, gu, tok, p);
}

}  // namespace

cudaError_t launch_gemm_tc_pair(int act, const void* A, int a_rows, const void* W,
                                const int* offsets, int E, int Kdim, int N, int w_rows_per_expert,
                                const float* bias, void* C, unsigned int* err, int* tile_counter,
                                cudaStream_t s, const int* gather_perm, int gather_K,
                                int gather_rows, int swap_max, float* split_partial,
                                int* split_flags) {
  CUtensorMap ma, mb, mgu;
  TokMaps tok;
  const bool gather = gather_perm != nullptr;
  if (swap_max < 0 || swap_max > kSwapMax || !tile_counter) return cudaErrorInvalidValue;
  if (!make_map(&ma, A, static_cast<uint64_t>(gather ? gather_rows : a_rows),
                static_cast<uint64_t>(Kdim), gather ? 1u : 128u) ||
      !make_map(&mb, W, static_cast<uint64_t>(E) * w_rows_per_expert, static_cast<uint64_t>(Kdim)))
    return cudaErrorInvalidValue;
  // swapped tails: the gated staging needs F % 16 == 0 (whole 16-row groups)
  if (gather || (act == kSiluGated && N % WB_BOX != 0)) swap_max = 0;
  mgu = mb;
  for (int j = 0; j < 4; ++j) tok.m[j] = ma;
  if (swap_max > 0) {
    for (int j = 0; j < 4; ++j)
      if (!make_map(&tok.m[j], A, static_cast<uint64_t>(a_rows), static_cast<uint64_t>(Kdim),
                    8u << j))
        return cudaErrorInvalidValue;
    if (act == kSiluGated && !make_gate_up_map(&mgu, W, E, N, Kdim)) return cudaErrorInvalidValue;
  }
  Params p;
  p.perm = gather_perm;
  p.K = gather_K;
  p.offsets = offsets;
  p.E = E;
  p.n_out = N;
  p.num_kb = (Kdim + BK - 1) / BK;
  p.b_rows = w_rows_per_expert;
  p.up_off = (act == kSiluGated) ? N : 0;
  p.out = static_cast<__nv_bfloat16*>(C);
  p.bias = bias;
  p.err = err;
  p.swap_max = swap_max;
  p.tile_counter = tile_counter;
  p.split_partial = split_flags ? split_partial : nullptr;
  p.split_flags = split_flags;
  p.split_cap = kSplitMaxCtas / 2;
  const int bn_out = (act == kSiluGated) ? 128 : 256;
  const long long tiles_bound =
      (static_cast<long long>(a_rows) / BMP + E) * ((N + bn_out - 1) / bn_out);
  const int max_clusters = num_sms() / 2;
  const int clusters = static_cast<int>(tiles_bound < max_clusters ? tiles_bound : max_clusters);
  if (gather) {
    if (act == kSiluGated) return launch_epi<kSiluGated, true>(ma, mb, mgu, tok, p, clusters, s);
    if (act == kReluBias) return launch_epi<kReluBias, true>(ma, mb, mgu, tok, p, clusters, s);
    return cudaErrorInvalidValue;
  }
  if (act == kSiluGated) return launch_epi<kSiluGated, false>(ma, mb, mgu, tok, p, clusters, s);
  if (act == kReluBias) return launch_epi<kReluBias, false>(ma, mb, mgu, tok, p, clusters, s);
  return launch_epi<kBias, false>(ma, mb, mgu, tok, p, clusters, s);
}

}  // namespace moe
