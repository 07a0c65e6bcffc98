// bf16 grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// The experts run as one grouped matrix multiplication over the rows sorted
// into expert order ("Mixture of experts", dewml.dev, "Expert computation
// and placement"); every contraction accumulates in fp32 and is rounded
// once to bf16 in the epilogue (same section, its precision rules).  The
// expert maths is mojolearn.MoEBlock's down_proj(silu(gate) * up) with the
// Hugging Face layout, or the exercise's Dense -> ReLU -> Dense with
// biases ("Mixture-of-Experts FFN", "Compute the experts and router").
//
// One persistent CTA per SM, 192 threads:
//   warp 0      TMA producer: A tile 128 x 64 and B tile 256 x 64 (two
//               128-row boxes) per k-block into a 4-stage ring;
//   warp 1      allocates 512 TMEM columns; one lane issues
//               tcgen05.mma M=128 N=256 K=16 into one of two 256-column fp32
//               accumulators and commits stage releases / tile completion;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (each warp its 32
//               TMEM lanes = 32 rows), activation, bf16 rounding, stores.
// Epilogue of tile i overlaps the MMAs of tile i+1 (double-buffered TMEM).
//
// Tiles: for expert e with n_e rows, ceil(n_e / 128) row blocks times
// ceil(N / BN) column blocks; within an expert the row block varies
// fastest, so CTAs running side by side share one weight tile through L2.
// Rows of a tile past the expert's last row belong to the next expert (or
// lie past the end and read as zeros); they are computed and not stored.
//
// Epilogues (BN = output columns per tile):
//   kSiluGated  B = 128 gate rows + the matching 128 up rows; the
//               accumulator's columns [0,128) are gate, [128,256) up;
//               H = silu(gate) * up, BN = 128.
//   kReluBias   B = 256 rows of W1; H = relu(acc + b1), BN = 256.
//   kBias       B = 256 rows; Y = acc (+ b2), BN = 256.
//
// Every mbarrier wait is bounded (common.cuh): on a timeout the kernel sets
// the device error word, the roles stop, outstanding TMA loads and MMAs are
// waited for (bounded), TMEM is freed and the CTA returns.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int BN_MMA = 256;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_BYTES = BN_MMA * BK * 2;      // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;

enum { kSiluGated = 0, kReluBias = 1, kBias = 2 };

struct Params {
  const int* perm;      // gathered A: sorted row -> (token, slot); null otherwise
  int K;                // slots per token (gathered A)
  const int* offsets;   // (E + 1) first sorted row of each expert
  int E;
  int n_out;            // output columns
  int num_kb;           // k-blocks of 64
  int b_rows;           // weight rows per expert
  int up_off;           // row offset of the up half (gated)
  __nv_bfloat16* out;   // (rows, n_out)
  const float* bias;    // (E, n_out) or null
  unsigned int* err;
};

struct Tail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int total_tiles;
  int tile_start[kMaxExperts + 1];
  int mt[kMaxExperts];
  int off[kMaxExperts + 1];
};

constexpr size_t kSmemBytes = 1024 + STAGES * STAGE_BYTES + sizeof(Tail);

__device__ __forceinline__ void decode_tile(const Tail* st, int E, int t, int& e, int& m_blk,
                                            int& n_blk) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (st->tile_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  e = lo;
  const int local = t - st->tile_start[e];
  const int mt = st->mt[e];
  n_blk = local / mt;
  m_blk = local - n_blk * mt;
}

// Bounded wait that ignores the abort flag: used only on the way out, to let
// copies and MMAs already in flight land before the CTA leaves.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, unsigned int* err,
                                           unsigned int site) {
  int dummy = 0;
  mbar_wait(bar, parity, &dummy, err, site);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Stores 32 bf16 values (16 packed words) at out[row, col0 .. col0+32),
// dropping 8-column groups at or past n_out (n_out is a multiple of 8).
__device__ __forceinline__ void store_row32(__nv_bfloat16* rowp, int col0, int n_out,
                                            const uint32_t (&w)[16]) {
  uint4* dst = reinterpret_cast<uint4*>(rowp + col0);
  if (col0 + 32 <= n_out) {
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (col0 + 8 * q < n_out) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

// Four rows of x (token indices r0..r3), 64 columns from c0, into 512
// contiguous bytes of shared memory with the same 128-byte swizzle as a
// tiled load (the tensor map's box is 64 x 1).
__device__ __forceinline__ void tma_gather4(const CUtensorMap* map, uint64_t* bar, void* dst, int c0,
                                            int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(r0), "r"(r1), "r"(r2),
      "r"(r3)
      : "memory");
}

template <int EPI, bool GATHER>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  Tail* st = reinterpret_cast<Tail*>(smem + STAGES * STAGE_BYTES);

  constexpr int BN_OUT = (EPI == kSiluGated) ? 128 : 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;
  const int n_tiles = (p.n_out + BN_OUT - 1) / BN_OUT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&st->tfull[a], 1);
      mbar_init(&st->tempty[a], 4);
    }
    mbar_init(&st->mma_done, 1);
    st->abort = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&st->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  pdl_trigger();
  // the expert offsets come from the permutation kernel
  pdl_wait();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      const int o0 = p.offsets[e], o1 = p.offsets[e + 1];
      const int mt = (o1 - o0 + BM - 1) / BM;
      st->off[e] = o0;
      st->mt[e] = mt;
      st->tile_start[e] = acc;
      acc += mt * n_tiles;
    }
    st->off[E] = p.offsets[E];
    st->tile_start[E] = acc;
    st->total_tiles = acc;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = st->tmem_base;
  const int total = st->total_tiles;
  volatile int* abort = &st->abort;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Lane 0 waits for free stages and posts the expected bytes; with a
    // gathered A every lane then fetches 4 of the tile's 128 token rows.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t used = 0, last_parity = 0;   // per stage: ever filled / parity of last fill
    const int rows_live = st->off[E];
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      if (!__shfl_sync(0xffffffffu, lane == 0 ? static_cast<int>(!*abort) : 0, 0)) break;
      int e, m_blk, n_blk;
      decode_tile(st, E, t, e, m_blk, n_blk);
      const int rowA = st->off[e] + m_blk * BM;
      int rowB0, rowB1;
      if (EPI == kSiluGated) {
        rowB0 = e * p.b_rows + n_blk * 128;
        rowB1 = rowB0 + p.up_off;
      } else {
        rowB0 = e * p.b_rows + n_blk * 256;
        rowB1 = rowB0 + 128;
      }
      int tok[4] = {0, 0, 0, 0};
      // gathered A: only the lanes whose 4 rows hold some of this expert's
      // rows fetch them; the other rows of the stage are padding (computed,
      // never stored) and keep whatever the stage held
      int gather_lanes = 32;
      if (GATHER) {
        const int valid = min(BM, st->off[e + 1] - rowA);
        gather_lanes = (valid + 3) >> 2;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = rowA + 4 * lane + i;
          tok[i] = r < rows_live ? __ldg(p.perm + r) / p.K : 0;   // rows past the end: any row
        }
      }
      const uint32_t stage_tx = STAGE_BYTES - static_cast<uint32_t>(32 - gather_lanes) * 512u;
      bool ok = true;
      for (int kb = 0; kb < p.num_kb; ++kb) {
        int good = 1;
        if (lane == 0) {
          good = mbar_wait(&st->empty[stage], phase ^ 1u, abort, p.err, SITE_GEMM_PRODUCER) ? 1 : 0;
          if (good) mbar_arrive_expect_tx(&st->full[stage], stage_tx);
        }
        if (!__shfl_sync(0xffffffffu, good, 0)) { ok = false; break; }
        if (GATHER && lane < gather_lanes)
          tma_gather4(&tmA, &st->full[stage], sA + stage * A_BYTES + lane * 512, kb * BK, tok[0],
                      tok[1], tok[2], tok[3]);
        if (lane == 0) {
          if (!GATHER) tma_load_2d(&tmA, &st->full[stage], sA + stage * A_BYTES, kb * BK, rowA);
          tma_load_2d(&tmB, &st->full[stage], sB + stage * B_BYTES, kb * BK, rowB0);
          tma_load_2d(&tmB, &st->full[stage], sB + stage * B_BYTES + B_BYTES / 2, kb * BK, rowB1);
          used |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
    // let every issued load land before the CTA can leave
    if (lane == 0)
      for (int s = 0; s < STAGES; ++s)
        if (used & (1u << s)) drain_wait(&st->full[s], (last_parity >> s) & 1u, p.err, SITE_GEMM_PRODUCER);
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN_MMA);
      int stage = 0;
      uint32_t phase = 0;
      int i = 0;
      for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
        const int acc = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        if (!mbar_wait(&st->tempty[acc], aph ^ 1u, abort, p.err, SITE_GEMM_MMA)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN_MMA;
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&st->full[stage], phase, abort, p.err, SITE_GEMM_MMA)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16(d, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), idesc,
                      (kb | k) != 0 ? 1u : 0u);
          umma_commit(&st->empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&st->tfull[acc]);
      }
      // all MMAs issued by this thread complete before TMEM / smem go away
      umma_commit(&st->mma_done);
      drain_wait(&st->mma_done, 0, p.err, SITE_GEMM_MMA);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int lane_base = (warp & 3) * 32;   // TMEM lanes this warp may access
    int i = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
      int e, m_blk, n_blk;
      decode_tile(st, E, t, e, m_blk, n_blk);
      const int acc = i & 1;
      const uint32_t aph = (i >> 1) & 1;
      // every lane must agree before the warp-collective TMEM loads
      const bool got = mbar_wait(&st->tfull[acc], aph, abort, p.err, SITE_GEMM_EPILOGUE);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int grow = st->off[e] + m_blk * BM + lane_base + lane;
      const bool rvalid = grow < st->off[e + 1];
      __nv_bfloat16* rowp = p.out + static_cast<size_t>(rvalid ? grow : 0) * p.n_out;
      const uint32_t tb = tmem + (static_cast<uint32_t>(lane_base) << 16) + acc * BN_MMA;
      if (EPI == kSiluGated) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(tb + c * 32, g);
          tmem_ld32(tb + 128 + c * 32, u);
          tmem_ld_wait();
          const int col0 = n_blk * 128 + c * 32;
          if (rvalid && col0 < p.n_out) {
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float g0 = __uint_as_float(g[2 * j]), g1 = __uint_as_float(g[2 * j + 1]);
              const float u0 = __uint_as_float(u[2 * j]), u1 = __uint_as_float(u[2 * j + 1]);
              const float h0 = silu_bf16_epilogue(g0) * u0;
              const float h1 = silu_bf16_epilogue(g1) * u1;
              w[j] = pack_bf16x2(h0, h1);
            }
            store_row32(rowp, col0, p.n_out, w);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t v[32];
          tmem_ld32(tb + c * 32, v);
          tmem_ld_wait();
          const int col0 = n_blk * 256 + c * 32;
          if (rvalid && col0 < p.n_out) {
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
            store_row32(rowp, col0, p.n_out, w);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&st->tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
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

// Row-major (rows, cols) bf16 matrix, boxes of 128 rows x 64 columns with
// the 128-byte swizzle; out-of-range elements read as zero.
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

template <int EPI, bool GATHER>
cudaError_t launch_epi(const CUtensorMap& a, const CUtensorMap& b, const Params& p, int grid,
                       cudaStream_t s) {
  // the shared-memory opt-in is a per-device function attribute
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64 || !done[dev]) {
      err = cudaFuncSetAttribute(grouped_gemm_tc_kernel<EPI, GATHER>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kSmemBytes));
      if (err != cudaSuccess) return err;
      if (dev >= 0 && dev < 64) done[dev] = true;
    }
  }
  return launch_k(grouped_gemm_tc_kernel<EPI, GATHER>, dim3(grid), dim3(THREADS), kSmemBytes, s,
                  pdl_enabled(), 1, a, b, p);
}

}  // namespace

cudaError_t launch_gemm_tc(int act, const void* A, int a_rows, const void* W, const int* offsets,
                           int E, long long rows, int Kdim, int N, int w_rows_per_expert,
                           const float* bias,
                           void* C, unsigned int* err, cudaStream_t s, const int* gather_perm,
                           int gather_K, int gather_rows) {
  CUtensorMap ma, mb;
  const bool gather = gather_perm != nullptr;
  if (!make_map(&ma, A, static_cast<uint64_t>(gather ? gather_rows : a_rows),
                static_cast<uint64_t>(Kdim), gather ? 1u : 128u) ||
      !make_map(&mb, W, static_cast<uint64_t>(E) * w_rows_per_expert, static_cast<uint64_t>(Kdim)))
    return cudaErrorInvalidValue;
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
  const int bn_out = (act == kSiluGated) ? 128 : 256;
  const long long n_tiles = (N + bn_out - 1) / bn_out;
  // upper bound on the tile count: every expert may add one partial row block
  const long long tiles_bound = (static_cast<long long>(a_rows) / BM + E) * n_tiles;
  // With at most 128 rows per expert on average (weight streaming) each
  // touched expert has one row block and, rows >= E, all experts are
  // likely touched: size the grid so that every CTA takes the same number of
  // tiles.  A last wave of a few CTAs would stream its weight tiles at
  // single-SM bandwidth while the rest of HBM sits idle.
  long long tiles = tiles_bound;
  if (rows <= 128LL * E) tiles = (rows < E ? rows : E) * n_tiles;
  const long long sms = num_sms();
  const long long waves = (tiles + sms - 1) / sms;
  const int grid = static_cast<int>(waves > 0 ? (tiles + waves - 1) / waves : 1);
  if (gather) {
    if (act == kSiluGated) return launch_epi<kSiluGated, true>(ma, mb, p, grid, s);
    if (act == kReluBias) return launch_epi<kReluBias, true>(ma, mb, p, grid, s);
    return cudaErrorInvalidValue;
  }
  if (act == kSiluGated) return launch_epi<kSiluGated, false>(ma, mb, p, grid, s);
  if (act == kReluBias) return launch_epi<kReluBias, false>(ma, mb, p, grid, s);
  return launch_epi<kBias, false>(ma, mb, p, grid, s);
}

}  // namespace moe
