/*
 * libmoe — forward pass of a top-k mixture-of-experts feed-forward layer on
 * one NVIDIA B200 (sm_100a).  Plain C ABI: device pointers, sizes, a stream
 * handle passed as void* (a cudaStream_t, NULL = the legacy default stream).
 *
 * What is computed (for each token t of x, flattened to (T, D)):
 *
 *   logits[t, e] = sum_d x[t, d] * router[e, d] (+ router_bias[e])
 *   p[t, :]      = softmax(logits[t, :]) over the E experts
 *   idx[t, 0..K) = the K largest p, in descending order, equal scores going
 *                  to the lower expert index
 *   w[t, k]      = p[t, idx[t, k]] / (sum_j p[t, idx[t, j]] + 1e-9)
 *                  when norm_topk_prob, else p[t, idx[t, k]]
 *   out[t, :]    = sum_k w[t, k] * expert_{idx[t, k]}(x[t, :])
 *
 * with expert_e either
 *   MOE_ACT_SILU_GATED:  down_e(silu(gate_e x) * up_e x)   (no biases), or
 *   MOE_ACT_RELU:        W2_e relu(W1_e x + b1_e) + b2_e.
 *
 * Sources, by page and section:
 *   - "Mixture-of-Experts FFN" (crackedaicode.com Flax exercise): "Compute
 *     the experts and router" (Dense/ReLU experts, biased Dense(E) router,
 *     softmax, top_k order and ties), "Weight the selected outputs" (the
 *     1e-9 renormalisation and the per-token gather), "Problem" (shapes,
 *     1 <= K <= E, positive dimensions, features fastest).
 *   - "mojolearn.MoEBlock": class description (SiLU-gated Mixtral expert,
 *     lower-index ties, forward only), "Variables" (router (E, D),
 *     gate_up_proj (E, 2F, D), down_proj (E, D, F), selected_experts int64),
 *     "Parameters" (top_k range -> error, hidden_act other than silu ->
 *     error, norm_topk_prob), forward(x) (float64 input -> error, output
 *     with the shape of x).
 *   - "Mixture of experts" (dewml.dev), "Expert computation and placement":
 *     tokens are sorted into expert order and the experts run as one grouped
 *     matrix multiplication; each contraction accumulates in at least fp32
 *     and rounds once to the compute dtype.
 *
 * Only the selected experts are computed.  Work runs asynchronously on the
 * given stream; results are deterministic (bitwise repeatable run to run:
 * no floating-point atomics anywhere).  The library allocates nothing and
 * keeps no state between calls except the optional stage profiler and a
 * per-device error word written by bounded waits (see moe_device_status).
 */
#ifndef LIBMOE_MOE_H
#define LIBMOE_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 1

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,      /* K outside [1, E], a dimension <= 0, a required pointer NULL
                                   ("Problem": positive dimensions, 1 <= K <= E;
                                   mojolearn "Parameters": top_k range -> ValueError) */
  MOE_ERR_UNSUPPORTED_ACT = 2,  /* act is neither SiLU-gated nor ReLU (mojolearn "Parameters":
                                   hidden_act other than silu -> NotImplementedError) */
  MOE_ERR_DTYPE = 3,            /* dtype other than f32 / bf16, e.g. MOE_F64 (mojolearn
                                   forward(x): float64 input -> TypeError) */
  MOE_ERR_SHAPE = 4,            /* a size the kernels cannot index (E > MOE_MAX_EXPERTS,
                                   T*K or T*max(D,F) beyond 2^31-1) */
  MOE_ERR_ALIGNMENT = 5,        /* a device pointer not 16-byte aligned, or on the bf16 path D or F
                                   not a multiple of 8 (tensor-memory-access rows need 16-byte
                                   strides) */
  MOE_ERR_WORKSPACE = 6,        /* workspace NULL or smaller than moe_ffn_workspace_size() */
  MOE_ERR_CUDA = 7,             /* a CUDA runtime call failed (a launch error, or a sticky error
                                   from earlier work on the device); see moe_last_error() */
  MOE_ERR_TIMEOUT = 8,          /* a bounded wait inside a kernel gave up (reported by
                                   moe_device_status); outputs of that call are undefined */
  MOE_ERR_DEVICE = 9            /* the current device is not sm_100 (B200 / GB200) */
} moe_status_t;

typedef enum {
  MOE_ACT_SILU_GATED = 0,  /* Mixtral expert: gate_up_proj (E, 2F, D), rows [0,F) gate, [F,2F) up;
                              down_proj (E, D, F); b1, b2 must be NULL */
  MOE_ACT_RELU = 1         /* exercise expert: gate_up_proj slot holds W1 (E, F, D), down_proj slot
                              holds W2 (E, D, F); b1 (E, F) and b2 (E, D) required */
} moe_act_t;

typedef enum {
  MOE_F32 = 0,   /* float32 x / weights / out; experts in fp32 FMA on CUDA cores */
  MOE_BF16 = 1,  /* bfloat16 x / weights / out; tensor cores, fp32 accumulation, the
                    intermediate H = act(...) rounded once to bf16 */
  MOE_F64 = 2    /* not supported: always MOE_ERR_DTYPE */
} moe_dtype_t;

/* Largest expert count the router kernel holds in registers. */
#define MOE_MAX_EXPERTS 256

/*
 * Bytes of device workspace moe_ffn_forward needs for these sizes (0 when
 * the sizes are invalid).  Holds the token permutation, the expert-sorted
 * copy of x, the intermediate H (T*K, F) and per-slot expert outputs
 * (T*K, D).  The caller allocates it; contents need not be initialised and
 * are garbage after the call.  Calls that share a workspace must not
 * overlap on the GPU.
 */
MOE_API size_t moe_ffn_workspace_size(int64_t T, int64_t D, int64_t F, int E, int K,
                              moe_dtype_t dt, moe_act_t act);

/*
 * The whole forward.  All pointers are device pointers owned by the caller,
 * 16-byte aligned, row-major with the last dimension contiguous:
 *
 *   x                (T, D)            dt    tokens; any leading shape flattened to T
 *   router           (E, D)            dt    router weight, one row per expert
 *   gate_up_proj     (E, 2F, D) / (E, F, D)  dt   see moe_act_t
 *   down_proj        (E, D, F)         dt
 *   out              (T, D)            dt    written once per element (must not alias inputs)
 *   selected_experts (T, K)            int64 may be NULL
 *   routing_weights  (T, K)            f32   may be NULL
 *   router_bias      (E)               f32   may be NULL for SiLU; required for ReLU
 *   b1               (E, F)            f32   ReLU only
 *   b2               (E, D)            f32   ReLU only
 *   router_logits    (T, E)            f32   may be NULL
 *   workspace        workspace_bytes         >= moe_ffn_workspace_size(...)
 *
 * Host-side validation happens before any launch; on an error nothing is
 * launched and no output is touched.  Returns MOE_OK once all kernels are
 * enqueued on `stream`; inputs must stay valid until the stream reaches
 * that point.
 *
 * A forward makes no synchronising call, so it can be recorded into a CUDA
 * graph by stream capture.  The first call of a kernel variant on a device
 * sets that kernel's attributes (and, for the one-kernel small layer,
 * queries how large a cluster the device can co-schedule); make one call of
 * the same shape outside capture first.
 */
MOE_API moe_status_t moe_ffn_forward(const void* x, const void* router, const void* gate_up_proj,
                             const void* down_proj, int E, int K, int norm_topk_prob,
                             moe_act_t act, void* out, int64_t* selected_experts,
                             float* routing_weights, int64_t T, int64_t D, int64_t F,
                             moe_dtype_t dt, const float* router_bias, const float* b1,
                             const float* b2, float* router_logits, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * Router only: logits, softmax, top-k selection and weights (the first half
 * of moe_ffn_forward, same definitions).  router_logits may be NULL;
 * selected_experts and routing_weights are required.  Needs no workspace.
 */
MOE_API moe_status_t moe_route(const void* x, const void* router, const float* router_bias, int64_t T,
                       int64_t D, int E, int K, int norm_topk_prob, moe_dtype_t dt,
                       float* router_logits, int64_t* selected_experts, float* routing_weights,
                       void* stream);

/*
 * Routing options (all off when zeroed; a NULL options pointer is the same
 * as zeroed options, i.e. exactly moe_ffn_forward / moe_route).
 *
 *   score             MOE_SCORE_SOFTMAX (default): softmax over the experts;
 *                     MOE_SCORE_SIGMOID: each expert scored by sigmoid(logit)
 *                     on its own ("Mixture of experts", dewml.dev, "Router
 *                     behavior": softmax or sigmoid scores).
 *   selection_bias    (E) f32 device pointer or NULL: added to the scores
 *                     only to choose the top-k; the weights come from the
 *                     unbiased scores (same section: a per-expert bias that
 *                     changes which experts are picked).
 *   dynamic_threshold > 0: after the weights, a kept expert whose share of
 *                     the mixture (renormalised weight) is below the
 *                     threshold is dropped, the first (leader) always stays,
 *                     and the kept shares are renormalised to sum to one
 *                     (ES-MoE API page, "ESMoE" settings, dynamic_threshold).
 *                     Dropped slots get weight 0 and no expert work.
 *   capacity_factor   > 0: each sequence of seq_len tokens keeps
 *                     floor(max(ceil(seq_len*K/E)*cf, cf)) slots per expert,
 *                     the first in token order; a dropped slot adds nothing
 *                     and no weight is renormalised ("Expert computation and
 *                     placement", capacity_factor).  Forward only.
 *   seq_len           tokens per sequence for the capacity; 0 = the whole
 *                     batch is one sequence; otherwise a multiple of 32.
 *   slot_kept         (T, K) u8 device out or NULL: 1 where the slot's
 *                     expert output enters out, 0 where it was dropped.
 *   balance           4 f32 device out or NULL: the batch's balancing
 *                     statistics {switch, gshard, master, gshard_probs}
 *                     (ES-MoE API page, "Balancing objectives"), from the
 *                     scores and the final routing weights.  Forward only.
 *
 * selected_experts keeps the router's top-k choice even for dropped slots;
 * routing_weights holds the final weights (0 where the threshold dropped).
 */
typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score_t;

typedef struct moe_route_opts {
  moe_score_t score;
  const float* selection_bias;
  float dynamic_threshold;
  float capacity_factor;
  int64_t seq_len;
  uint8_t* slot_kept;
  float* balance;
} moe_route_opts_t;

MOE_API moe_status_t moe_ffn_forward_ex(const void* x, const void* router,
                                        const void* gate_up_proj, const void* down_proj, int E,
                                        int K, int norm_topk_prob, moe_act_t act, void* out,
                                        int64_t* selected_experts, float* routing_weights,
                                        int64_t T, int64_t D, int64_t F, moe_dtype_t dt,
                                        const float* router_bias, const float* b1,
                                        const float* b2, float* router_logits, void* workspace,
                                        size_t workspace_bytes, const moe_route_opts_t* opts,
                                        void* stream);

/* Router only with options (capacity_factor and balance need the forward:
 * MOE_ERR_INVALID_ARG here). */
MOE_API moe_status_t moe_route_ex(const void* x, const void* router, const float* router_bias,
                                  int64_t T, int64_t D, int E, int K, int norm_topk_prob,
                                  moe_dtype_t dt, float* router_logits, int64_t* selected_experts,
                                  float* routing_weights, const moe_route_opts_t* opts,
                                  void* stream);

/*
 * Forward pass that allocates nothing, for callers that cannot obtain device
 * memory at call time: code running where a device allocation is not
 * permitted or not available to it, such as a plugin or callback of another
 * runtime that owns all device memory and hands the plugin only its inputs
 * and outputs.  The cited descriptions of the layer have no counterpart;
 * it is an addition of this library.
 *
 * Same arguments and results as moe_ffn_forward, without the workspace:
 * the scratch lives in one static device array of
 * MOE_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * this part of the library keeps until the process exits.  Sizes whose
 * moe_ffn_workspace_size exceeds it are rejected with MOE_ERR_WORKSPACE
 * before anything is launched (for bf16 that covers e.g. T=32 tokens with
 * D=4096, F=14336, E=8, K=8).  No cudaMalloc / cudaFree is called.
 *
 * The first call on a device does a one-time host-side set-up with that
 * device current: it reads the device's attributes and looks up the device
 * addresses of the array and of the library's error word
 * (cudaGetSymbolAddress).  If the CUDA runtime loads modules lazily, that
 * lookup is what loads the library's device code, and with it the driver
 * places the 32 MiB array in device memory.  Later calls reuse what the first
 * one found.  So make the first call on each device part of the caller's
 * initialisation, before any stream capture.  This entry point creates no
 * stream, event or pinned host memory (the other entry points create one
 * each per device on their first call, for reading the error word during a
 * stall); the first moe_set_debug_sync wait or moe_device_error_peek on a
 * device creates them.  A cudaDeviceReset discards what the set-up found:
 * calls after one, in the same process, are not supported.
 *
 * All calls share the one array and it keeps the previous call's contents;
 * no part of it has to start at zero, since each call writes every scratch
 * element it later reads (pad rows only feed rows that are never stored).
 * Calls whose work overlaps on the GPU (e.g. on two streams at once) race
 * on the array: order them on one stream or with events.
 */
#define MOE_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
MOE_API moe_status_t moe_ffn_forward_noalloc(const void* x, const void* router,
                                             const void* gate_up_proj, const void* down_proj,
                                             int E, int K, int norm_topk_prob, moe_act_t act,
                                             void* out, int64_t* selected_experts,
                                             float* routing_weights, int64_t T, int64_t D,
                                             int64_t F, moe_dtype_t dt, const float* router_bias,
                                             const float* b1, const float* b2,
                                             float* router_logits, void* stream);

/*
 * Which tensor-core grouped GEMM the bf16 path uses (process-wide setting):
 *   MOE_GEMM_AUTO  - CTA pairs when the average expert has >= 512 routed
 *                    rows (large batches), one CTA per tile otherwise;
 *   MOE_GEMM_1SM   - always one CTA per 128 x 256 tile;
 *   MOE_GEMM_2SM   - always CTA pairs (tcgen05 cta_group::2, 256 x 256).
 * Both give identical results up to fp32 summation order inside the MMA.
 * Returns the previous mode, or -1 for an unknown mode (nothing changes).
 */
#define MOE_GEMM_AUTO 0
#define MOE_GEMM_1SM 1
#define MOE_GEMM_2SM 2
MOE_API int moe_set_gemm_mode(int mode);

/*
 * Short expert tails on the CTA-pair GEMM (process-wide setting).  An
 * expert's routed rows fill 256-row tiles; when its last tile holds at most
 * max_rows rows, that tile runs with the operands swapped: 256 weight rows
 * as the MMA's M and the tail's rows (rounded up to 16, 32, 64 or 128) as
 * its N, instead of a full 256-row tile that is mostly padding.  max_rows in
 * 0..MOE_TAIL_SWAP_MAX; 0 turns it off.  The SiLU-gated GEMM swaps only when
 * F is a multiple of 16.  Results agree with the unswapped tile up to fp32
 * summation order.  Returns the previous setting, or -1 if max_rows is out
 * of range (nothing changes).
 */
#define MOE_TAIL_SWAP_DEFAULT 128
#define MOE_TAIL_SWAP_MAX 128
MOE_API int moe_set_tail_swap(int max_rows);

/*
 * Cluster size of the one-kernel float32 small layer (process-wide
 * setting).  A small float32 layer (E <= 8, T*K <= 256, no routing
 * options, the kernel's shared memory within 200 KB) runs as one cluster
 * of CTAs; each expert's hidden columns are split over CTAs in proportion
 * to the rows it received.  ctas: MOE_SMALL_CLUSTER_AUTO (16 where the GPU
 * can co-schedule a cluster of 16 such CTAs, else 8), 8 or 16.  A forced
 * 16 on a GPU that cannot co-schedule it makes the forward fail with
 * MOE_ERR_CUDA.  Results agree across sizes up to fp32 summation order.
 * Returns the previous setting, or -1 for any other value (nothing
 * changes).
 */
#define MOE_SMALL_CLUSTER_AUTO 0
MOE_API int moe_set_small_cluster(int ctas);

/*
 * Whether the bf16 gate_up GEMM fetches its token rows from x by index
 * (TMA tile::gather4, four rows per copy, only for the rows a tile holds)
 * instead of from an expert-sorted copy written by a separate gather
 * kernel.  Results are bit-identical either way.  Process-wide setting:
 *   MOE_FUSED_GATHER_OFF  - always the expert-sorted copy;
 *   MOE_FUSED_GATHER_ON   - always by index;
 *   MOE_FUSED_GATHER_AUTO - (default) by index when the one-CTA GEMM runs
 *                           and experts average at most 16 routed rows
 *                           (decode steps): the few copies hide under the
 *                           weight stream and the gather kernel is saved.
 *                           With full tiles the four-row copies deliver A
 *                           far slower than the tensor cores consume it
 *                           (gate_up about 3x slower on the Mixtral layer).
 * Returns the previous setting, or -1 for another value (nothing changes).
 */
#define MOE_FUSED_GATHER_OFF 0
#define MOE_FUSED_GATHER_ON 1
#define MOE_FUSED_GATHER_AUTO 2
MOE_API int moe_set_fused_gather(int mode);

/*
 * Whether the kernels of one forward are launched with programmatic
 * dependent launch (OFF by default): each kernel's set-up (barriers, tensor
 * memory, descriptor prefetch) then overlaps the end of the previous kernel,
 * and it waits for that kernel before reading or writing shared buffers.
 * Same results either way; it saves 0-2% of a forward.  Off by default
 * because, with it on, back-to-back forwards of the 64-expert fine-grained
 * layer were seen to stall on B200 (no cause found; none with it off).
 * Returns the previous setting.
 */
MOE_API int moe_set_pdl(int on);

/*
 * Debug-sync mode (process wide, off by default): with timeout_ms > 0,
 * moe_ffn_forward waits after every kernel it launches, polling for at most
 * timeout_ms, and returns MOE_ERR_TIMEOUT naming the first kernel that did
 * not finish (with the device error word) in moe_last_error().  Kernels then
 * never overlap and each call is synchronous: for locating a stall, not for
 * timing.  timeout_ms <= 0 turns it off.  Returns the previous setting.
 */
MOE_API int moe_set_debug_sync(int timeout_ms);

/* Short English description of a status code (static storage). */
MOE_API const char* moe_status_string(moe_status_t status);

/* Detail of the last error returned on this host thread ("" if none). */
MOE_API const char* moe_last_error(void);

/* MOE_ABI_VERSION of the built library. */
MOE_API int moe_abi_version(void);

/*
 * Synchronises `stream`, then reads and clears the current device's error
 * word, which kernels set when a bounded wait gives up instead of hanging.
 * Returns MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_CUDA; on MOE_ERR_TIMEOUT,
 * moe_last_error() names the kernels and roles whose waits gave up.
 */
MOE_API moe_status_t moe_device_status(void* stream);

/*
 * Reads the current device's error word into *word WITHOUT waiting for any
 * caller stream (a copy on a private stream), and does not clear it: for a
 * host watchdog that wants to know, while kernels may still be running,
 * whether and where a bounded wait has given up.  Bit 0 = a wait timed out;
 * bits 8.. = the site (router / grouped GEMM / CTA-pair GEMM, each as
 * producer, MMA issuer or epilogue, then the test probe).  *word is host
 * memory.  Returns MOE_OK, MOE_ERR_INVALID_ARG (word NULL) or MOE_ERR_CUDA.
 */
MOE_API moe_status_t moe_device_error_peek(unsigned int* word);

/* Number of kernels this library has launched in the process so far (all
   devices, all entry points; launches the CUDA runtime accepted).  A forward
   launches 6 to 9 kernels depending on its size and options, or one for a
   small float32 layer (E <= 8, T*K <= 256, no routing options). */
MOE_API unsigned long long moe_kernel_launches(void);

/* Comma-separated names of the sites set in an error word (static storage
   of the calling thread, overwritten by the next call). */
MOE_API const char* moe_error_sites(unsigned int word);

/*
 * Test hook for failure detection: launches one CTA that waits, through the
 * same bounded mbarrier wait the kernels use, on a barrier nothing ever
 * arrives at.  The wait gives up after timeout_ms, sets the device error
 * word and the kernel returns; moe_device_status then reports
 * MOE_ERR_TIMEOUT and clears the word, and the context stays usable.
 * timeout_ms must be in [1, 2000].
 */
MOE_API moe_status_t moe_debug_bounded_wait(int timeout_ms, void* stream);

/*
 * Stage profiler.  While enabled, moe_ffn_forward records CUDA events
 * around each of its kernels on the caller's stream (router, permute,
 * gate_up, down, combine; a small float32 layer that runs as one kernel
 * records it as small_layer).  moe_profile_read synchronises on the
 * recorded events, adds their durations (milliseconds) into
 * ms[0..n_stages) and returns the number of forward calls covered, then
 * resets the counters.
 */
#define MOE_NUM_STAGES 6
MOE_API moe_status_t moe_profile_enable(int enable);
MOE_API int moe_profile_read(float* ms, int n_stages);
MOE_API const char* moe_stage_name(int stage);

#ifdef __cplusplus
}
#endif
#endif /* LIBMOE_MOE_H */
