// Internal launch interface between the C ABI (moe_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kMaxExperts = 256;
constexpr int kRouterTokensPerCta = 32;   // tokens per router CTA = per permute block
constexpr int kTileM = 128;               // rows of one grouped-GEMM tile
// Tile counters of the grouped GEMMs' dynamic schedulers, one per GEMM of a
// forward, each on its own 128-byte line, then each GEMM's flags of the
// split last wave (one per split unit, CTA and epilogue warp): kSchedInts
// ints in the workspace, zeroed by the scatter kernel of the same forward.
constexpr int kSplitMaxCtas = 148;           // CTAs whose partial tiles the scratch holds
constexpr int kSplitFlags = kSplitMaxCtas * 4;
constexpr int kSchedGateUp = 0;
constexpr int kSchedDown = 32;
constexpr int kSchedFlagsGateUp = 64;
constexpr int kSchedFlagsDown = kSchedFlagsGateUp + kSplitFlags;
constexpr int kSchedInts = kSchedFlagsDown + kSplitFlags;
// fp32 partial accumulators of the split last wave: 128 rows x 256 columns
// per CTA of a split unit
constexpr size_t kSplitCtaBytes = 128u * 256u * 4u;
constexpr size_t kSplitBytes = kSplitMaxCtas * kSplitCtaBytes;

enum DType : int { kF32 = 0, kBF16 = 1 };

struct RouteArgs {
  const void* x;            // (T, D) f32 or bf16
  const void* router;       // (E, D)
  const float* router_bias; // (E) or null
  int T, D, E, K, norm, dt;
  float* logits;            // (T, E) or null
  int64_t* sel64;           // (T, K) or null
  float* wout;              // (T, K) or null
  int* idx32;               // (T, K) or null
  float* w32;               // (T, K) or null
  int* blockcounts;         // (ceil(T / kRouterTokensPerCta), E) or null
  unsigned int* err;        // device error word (bounded waits)
  // routing extensions (all off when zero / null)
  int score;                // 0: softmax over experts, 1: sigmoid per expert
  const float* sel_bias;    // (E): added to the scores only to choose the experts
  float dyn_threshold;      // > 0: drop kept experts whose renormalised share is below it
  uint8_t* slot_kept;       // (T, K): 1 where the slot's expert output enters out
  float* bal_partial;       // (parts, 3, E): per-CTA sums of scores, gate, gate > 0
};

// Slots the router dropped carry this expert index in idx32 (= E).
// Parts of the balance partials each router flavour writes.
int router_tc_parts(int T);
int router_simt_parts(int T);

// Balancing statistics {switch, gshard, master, gshard_probs} from the
// router's partial sums, in fixed order.
cudaError_t launch_balance_finalize(const float* partial, int parts, int E, int T, float* out4,
                                    cudaStream_t s);

// Capacity: clamps the 32-token block histograms in place so that each
// sequence keeps at most floor(max(ceil(L*K/E)*cf, cf)) slots per expert,
// the first in token order.  L is a multiple of 32 (0: one sequence).
cudaError_t launch_capacity_clamp(int* blockcounts, int B, int E, int T, int K, int seq_len,
                                  float capacity_factor, cudaStream_t s);

// CUDA-core router (any dtype; used for float32).
cudaError_t launch_router(const RouteArgs& a, cudaStream_t s);
// Tensor-core router (bf16, E <= 256): same outputs.
cudaError_t launch_router_tc(const RouteArgs& a, cudaStream_t s);

// Per-expert column scans of the router's 32-token histograms (B, E):
// blockbase[b, e] = rows of expert e in blocks before b; totals[e].
cudaError_t launch_permute_scan(const int* blockcounts, int B, int E, int* blockbase,
                                int* totals, cudaStream_t s);

// Stable scatter of the (token, slot) pairs into expert order: perm[row] =
// slot, pos[slot] = row; block 0 also writes offsets (E + 1).
// Slots whose in-block rank reaches the (clamped) block count, and slots
// with the sentinel expert, get no row: pos = -1, slot_kept = 0.
// blockbase / totals null: the kernel scans the block counts itself.
// sched (kSchedInts, or null): block 0 zeroes the GEMMs' tile counters.
cudaError_t launch_permute_scatter(const int* idx32, const int* blockbase, const int* totals,
                                   const int* blockcounts, int T, int K, int E, int* offsets,
                                   int* perm, int* pos, uint8_t* slot_kept, int* sched,
                                   cudaStream_t s);

// x_perm[pos[t, k], :] = x[t, :] for every slot that was given a row
// (pos >= 0; perm is the inverse map, offsets[E] the live row count): by
// sorted row while x fits in L2, else by token with each row of x read once.
cudaError_t launch_gather_rows(const int* perm, const int* offsets, const int* pos, int T, int E,
                               int K, const void* x, int row_bytes, void* x_perm, cudaStream_t s);

// out[t, :] = sum_k w[t, k] * Y[pos[t, k], :], fp32 sum in k order; slots
// with pos < 0 (dropped) add nothing.
cudaError_t launch_combine(const void* Y, const float* w32, const int* pos, int T, int K, int D,
                           int dt, void* out, cudaStream_t s);

// fp32 grouped GEMMs on CUDA cores (the float32 path).
//   act 0: H = silu(A W_gate^T) * (A W_up^T)   (W rows [0,N) gate, [N,2N) up)
//   act 1: H = relu(A W^T + bias)
//   act 2: H = A W^T (+ bias)
cudaError_t launch_gemm_simt_f32(int act, const float* A, const float* W, const int* offsets,
                                 int E, int T, int Kdim, int N, int w_rows_per_expert,
                                 const float* bias, float* C, cudaStream_t s);

// bf16 grouped GEMMs on the tcgen05 tensor cores (same three epilogues).
// A: (a_rows, Kdim) bf16 sorted rows; W: (E * w_rows_per_expert, Kdim) bf16.
// With gather_perm set, A is x itself (gather_rows = T rows) and each tile's
// rows are fetched by token index perm[row] / gather_K (TMA tile::gather4),
// so the expert-sorted copy of x is never written.
// rows = routed rows T*K (sizes the persistent grid).
cudaError_t launch_gemm_tc(int act, const void* A, int a_rows, const void* W, const int* offsets,
                           int E, long long rows, int Kdim, int N, int w_rows_per_expert,
                           const float* bias, void* C, unsigned int* err, cudaStream_t s,
                           const int* gather_perm = nullptr, int gather_K = 0,
                           int gather_rows = 0);

// Same GEMM on CTA pairs (tcgen05 cta_group::2, 256-row tiles).  An expert's
// last row block of at most swap_max rows (0..255; 0: never) runs as a
// swapped-operand tile whose N is the block's rows rounded up to 16.  The
// persistent pairs take tiles in order from *tile_counter, which must be
// zero when the kernel starts (the scatter kernel zeroes it each forward).
// split_partial (kSplitBytes) / split_flags (kSplitFlags, zero at start):
// the last wave's units run as two halves of the k-blocks, the first
// handing its fp32 accumulator to the second; null: no split.
cudaError_t launch_gemm_tc_pair(int act, const void* A, int a_rows, const void* W,
                                const int* offsets, int E, int Kdim, int N, int w_rows_per_expert,
                                const float* bias, void* C, unsigned int* err, int* tile_counter,
                                cudaStream_t s, const int* gather_perm = nullptr,
                                int gather_K = 0, int gather_rows = 0, int swap_max = 0,
                                float* split_partial = nullptr, int* split_flags = nullptr);

// The whole float32 forward of a small layer in one launch: a cluster of
// 8 or 16 CTAs (router in every CTA; each expert's hidden columns split
// over CTAs in proportion to its rows; the combine over distributed shared
// memory).  For layers within these limits and no routing options.
constexpr int kSmallMaxExperts = 8;
constexpr int kSmallMinCluster = 8;             // the portable cluster size
constexpr int kSmallMaxCluster = 16;            // where the GPU co-schedules 16 CTAs
constexpr int kSmallMaxRows = 256;              // routed rows T*K
constexpr size_t kSmallMaxSmem = 200u << 10;    // x, router, one expert's weights, H, Y
bool small_layer_fits(int T, int D, int F, int E, int K, int gated);
// cluster: 0 = automatic (16 where possible, else 8), or 8 / 16.
cudaError_t launch_small_layer_f32(const float* x, const float* router, const float* rb,
                                   const float* gu, const float* dn, const float* b1,
                                   const float* b2, int T, int D, int F, int E, int K, int norm,
                                   int gated, float* out, int64_t* sel64, float* wout,
                                   float* logits, int cluster, cudaStream_t s);

int num_sms();
unsigned long long kernel_launches();   // accepted launches so far (note_launch)

// One CTA waiting (bounded) on an mbarrier nothing arrives at.
cudaError_t launch_bounded_wait_probe(unsigned long long timeout_ns, unsigned int* err,
                                      cudaStream_t s);

// Sets the message moe_last_error() returns on this host thread.
void set_last_error(const char* msg);

// The whole forward behind moe_ffn_forward_ex.  with_aux = false skips the
// per-device host bookkeeping (a stream, an event and a pinned host word
// for reading the error word during a stall), so the call allocates
// nothing; the no-allocation entry point uses that.
moe_status_t ffn_forward_impl(const void* x, const void* router, const void* gate_up_proj,
                              const void* down_proj, int E, int K, int norm_topk_prob,
                              moe_act_t act, void* out, int64_t* selected_experts,
                              float* routing_weights, int64_t T, int64_t D, int64_t F,
                              moe_dtype_t dt, const float* router_bias, const float* b1,
                              const float* b2, float* router_logits, void* workspace,
                              size_t workspace_bytes, const moe_route_opts_t* opts, void* stream,
                              bool with_aux);

}  // namespace moe
