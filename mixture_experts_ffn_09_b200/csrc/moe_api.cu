// libmoe C ABI: argument validation, workspace layout, the launch sequence
// of one forward, device status and the optional stage profiler.
//
// One forward = five stages on the caller's stream:
//   router   logits, softmax, top-k, weights, per-block expert histogram
//   permute  expert offsets (1-CTA scan) + stable scatter and row gather
//   gate_up  grouped GEMM 1 with the activation fused in its epilogue
//   down     grouped GEMM 2 (+ b2 for the Dense/ReLU expert)
//   combine  weighted gather back to token order, one write per element
#include <limits.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <chrono>
#include <thread>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/moe.h"
#include "internal.h"

namespace {

thread_local std::string g_last_error;

std::atomic<int> g_gemm_mode{MOE_GEMM_AUTO};
std::atomic<int> g_tail_swap{MOE_TAIL_SWAP_DEFAULT};
std::atomic<int> g_small_cluster{MOE_SMALL_CLUSTER_AUTO};
std::atomic<int> g_fused_gather{MOE_FUSED_GATHER_AUTO};
std::atomic<int> g_pdl{0};   // programmatic dependent launch: opt-in
std::atomic<int> g_debug_sync_ms{0};   // > 0: bounded wait after every kernel of a forward
// Block-count tables up to this many entries (blocks x experts) are scanned
// inside the scatter kernel: each of its blocks reads the whole table.
constexpr long long kScatterScansItself = 4096;

// The tensor-core GEMM for one launch: CTA pairs pay off when experts have
// enough rows to fill 256-row tiles.  With gather_perm the A rows are read
// from x by token index inside the GEMM.
cudaError_t launch_gemm_bf16(int act, const void* A, int a_rows, const void* W,
                             const int* offsets, int E, int T, int K, int Kdim, int N,
                             int w_rows, const float* bias, void* C, unsigned int* err,
                             int* tile_counter, float* split_partial, int* split_flags,
                             cudaStream_t s, const int* gather_perm = nullptr) {
  const int mode = g_gemm_mode.load();
  const bool pair = mode == MOE_GEMM_2SM ||
                    (mode == MOE_GEMM_AUTO && static_cast<long long>(T) * K >= 512LL * E);
  if (pair)
    return moe::launch_gemm_tc_pair(act, A, a_rows, W, offsets, E, Kdim, N, w_rows, bias, C, err,
                                    tile_counter, s, gather_perm, K, T, g_tail_swap.load(),
                                    split_partial, split_flags);
  return moe::launch_gemm_tc(act, A, a_rows, W, offsets, E, static_cast<long long>(T) * K, Kdim, N,
                             w_rows, bias, C, err, s, gather_perm, K, T);
}

__device__ unsigned int g_device_error;   // per device: bounded waits that gave up

moe_status_t fail(moe_status_t s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
moe_status_t fail(moe_status_t s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

moe_status_t cuda_fail(cudaError_t e, const char* where) {
  return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ------------------------------------------------------------ device info
struct DevInfo {
  bool init = false;
  int sms = 0;
  int major = 0, minor = 0;
  unsigned int* err = nullptr;
  // Host-side bookkeeping for reading the error word while kernels may be
  // stalled, made once per device so that such a read needs no call that
  // could wait for the device.  The ordinary entry points create it on
  // their first call; the no-allocation entry point never does (it holds a
  // pinned host word), and the readers create it on first use.
  bool aux = false;
  cudaStream_t peek_stream = nullptr;
  unsigned int* peek_host = nullptr;
  cudaEvent_t dbg_event = nullptr;
};
std::mutex g_dev_mu;
DevInfo g_dev[64];

// Creates the device's stream, event and pinned word (g_dev_mu held).
moe_status_t make_aux(DevInfo& d) {
  if (d.aux) return MOE_OK;
  cudaError_t e;
  if ((e = cudaStreamCreateWithFlags(&d.peek_stream, cudaStreamNonBlocking)) != cudaSuccess ||
      (e = cudaMallocHost(&d.peek_host, sizeof(unsigned int))) != cudaSuccess ||
      (e = cudaEventCreateWithFlags(&d.dbg_event, cudaEventDisableTiming)) != cudaSuccess)
    return cuda_fail(e, "device bookkeeping");
  d.aux = true;
  return MOE_OK;
}

// The current device's attributes and error-word address, checked to be an
// sm_100 part; with_aux also sets up the bookkeeping above.
moe_status_t device_info(DevInfo** out, bool with_aux = true) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_DEVICE, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.init) {
    if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) !=
            cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev)) !=
            cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_device_error)) != cudaSuccess)
      return cuda_fail(e, "cudaGetSymbolAddress(error word)");
    d.err = static_cast<unsigned int*>(p);
    d.init = true;
  }
  if (d.major != 10 || d.minor != 0)
    return fail(MOE_ERR_DEVICE, "device %d is sm_%d%d; libmoe is built for sm_100a", dev, d.major,
                d.minor);
  if (with_aux) {
    const moe_status_t st = make_aux(d);
    if (st != MOE_OK) return st;
  }
  *out = &d;
  return MOE_OK;
}

// The bookkeeping of a device whose DevInfo exists already (made on first use).
bool ensure_aux(DevInfo* d) {
  std::lock_guard<std::mutex> lock(g_dev_mu);
  return make_aux(*d) == MOE_OK;
}

// Polls until `done()` or `ms` milliseconds have passed.
template <typename Done>
bool poll_ms(int ms, Done done) {
  const auto t0 = std::chrono::steady_clock::now();
  while (!done()) {
    if (std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(ms)) return false;
    std::this_thread::sleep_for(std::chrono::microseconds(200));
  }
  return true;
}

// Copies the error word to the host on the private stream; false when the
// copy does not finish within `ms` (the device is not answering).
bool peek_word(DevInfo* dev, unsigned int* word, int ms) {
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (!ensure_aux(dev)) return false;
  if (cudaMemcpyAsync(dev->peek_host, dev->err, sizeof(unsigned int), cudaMemcpyDeviceToHost,
                      dev->peek_stream) != cudaSuccess)
    return false;
  if (!poll_ms(ms, [&] { return cudaStreamQuery(dev->peek_stream) != cudaErrorNotReady; }))
    return false;
  *word = *dev->peek_host;
  return true;
}

// Debug-sync mode: waits, bounded, for the kernels launched so far on `s`.
// False (with the error set) when they do not finish in time.
bool debug_wait(DevInfo* dev, cudaStream_t s, const char* stage) {
  const int ms = g_debug_sync_ms.load();
  if (ms <= 0) return true;
  if (!ensure_aux(dev)) {
    fail(MOE_ERR_CUDA, "debug sync after %s: could not create its event", stage);
    return false;
  }
  if (cudaEventRecord(dev->dbg_event, s) == cudaSuccess &&
      poll_ms(ms, [&] { return cudaEventQuery(dev->dbg_event) != cudaErrorNotReady; }))
    return true;
  unsigned int word = 0;
  const bool got = peek_word(dev, &word, 1000);
  fail(MOE_ERR_TIMEOUT, "%s did not finish within %d ms (device error word %s0x%x: %s)", stage, ms,
       got ? "" : "unreadable, ", word, got ? moe_error_sites(word) : "");
  return false;
}

// --------------------------------------------------------------- profiler
struct ProfState {
  bool enabled = false;
  int calls = 0;
  std::vector<cudaEvent_t> pool;
  std::vector<std::pair<int, std::pair<cudaEvent_t, cudaEvent_t>>> recs;   // stage, (start, end)
  size_t next = 0;
};
std::mutex g_prof_mu;
ProfState g_prof;

cudaEvent_t prof_event() {
  if (g_prof.next == g_prof.pool.size()) {
    cudaEvent_t ev;
    if (cudaEventCreate(&ev) != cudaSuccess) return nullptr;
    g_prof.pool.push_back(ev);
  }
  return g_prof.pool[g_prof.next++];
}

struct StageTimer {
  bool on;
  cudaStream_t s;
  explicit StageTimer(cudaStream_t st) : on(false), s(st) {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    on = g_prof.enabled;
    if (on) g_prof.calls++;
  }
  // Records an event pair around fn() on the stream when profiling.
  template <typename Fn>
  cudaError_t run(int stage, Fn fn) {
    if (!on) return fn();
    cudaEvent_t a, b;
    {
      std::lock_guard<std::mutex> lock(g_prof_mu);
      a = prof_event();
      b = prof_event();
      if (a && b) g_prof.recs.push_back({stage, {a, b}});
    }
    if (a) cudaEventRecord(a, s);
    cudaError_t e = fn();
    if (b) cudaEventRecord(b, s);
    return e;
  }
};

// ------------------------------------------------------ workspace layout
struct Layout {
  size_t idx32, w32, bcount, bbase, totals, offsets, sched, perm, pos, bal, part, xperm, h, y,
      total;
  bool split;     // the CTA-pair GEMMs may split their last wave (scratch reserved)
  int B, Rpad;
};

Layout layout(int64_t T, int64_t D, int64_t F, int E, int K, int elem) {
  Layout L{};
  const int64_t R = T * K;
  L.B = static_cast<int>((T + moe::kRouterTokensPerCta - 1) / moe::kRouterTokensPerCta);
  L.Rpad = static_cast<int>(align_up(static_cast<size_t>(R), moe::kTileM));
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 1024);
    return at;
  };
  L.idx32 = take(sizeof(int) * R);
  L.w32 = take(sizeof(float) * R);
  L.bcount = take(sizeof(int) * static_cast<size_t>(L.B) * E);
  L.bbase = take(sizeof(int) * static_cast<size_t>(L.B) * E);
  L.totals = take(sizeof(int) * E);
  L.offsets = take(sizeof(int) * (E + 1));
  L.sched = take(sizeof(int) * moe::kSchedInts);
  L.perm = take(sizeof(int) * R);
  L.pos = take(sizeof(int) * R);
  {
    const int parts = moe::router_simt_parts(static_cast<int>(T)) > moe::router_tc_parts(static_cast<int>(T))
                          ? moe::router_simt_parts(static_cast<int>(T))
                          : moe::router_tc_parts(static_cast<int>(T));
    L.bal = take(sizeof(float) * 3 * static_cast<size_t>(parts) * E);
  }
  // the split last wave's partial tiles, for layers whose automatic choice
  // is the CTA-pair GEMM (bf16, at least 512 routed rows per expert)
  L.split = elem == 2 && R >= 512LL * E;
  L.part = take(L.split ? moe::kSplitBytes : 0);
  L.xperm = take(static_cast<size_t>(elem) * L.Rpad * D);
  L.h = take(static_cast<size_t>(elem) * L.Rpad * F);
  L.y = take(static_cast<size_t>(elem) * L.Rpad * D);
  L.total = o;
  return L;
}

moe_status_t check_common(int64_t T, int64_t D, int E, int K, moe_dtype_t dt) {
  if (dt != MOE_F32 && dt != MOE_BF16)
    return fail(MOE_ERR_DTYPE, "dtype %d not supported (f32 or bf16; float64 is rejected)",
                static_cast<int>(dt));
  if (T <= 0 || D <= 0 || E <= 0)
    return fail(MOE_ERR_INVALID_ARG, "dimensions must be positive (T=%lld D=%lld E=%d)",
                static_cast<long long>(T), static_cast<long long>(D), E);
  if (K < 1 || K > E) return fail(MOE_ERR_INVALID_ARG, "top_k=%d outside [1, E=%d]", K, E);
  if (E > MOE_MAX_EXPERTS)
    return fail(MOE_ERR_SHAPE, "E=%d exceeds MOE_MAX_EXPERTS=%d", E, MOE_MAX_EXPERTS);
  if (T * K > INT_MAX - moe::kTileM || T > INT_MAX || D > INT_MAX)
    return fail(MOE_ERR_SHAPE, "T*K=%lld exceeds the 32-bit row index", static_cast<long long>(T * K));
  return MOE_OK;
}

// Row coordinates of the weight matrices are 32-bit in the kernels.
bool shapes_ok(int64_t T, int64_t D, int64_t F, int E, int K, moe_act_t act) {
  (void)T;
  (void)K;
  const int64_t wrows = static_cast<int64_t>(E) * (act == MOE_ACT_SILU_GATED ? 2 * F : F);
  return F <= INT_MAX / 2 && wrows + 256 <= INT_MAX && static_cast<int64_t>(E) * D + 256 <= INT_MAX;
}

moe_status_t check_opts(const moe_route_opts_t* o, bool forward) {
  if (!o) return MOE_OK;
  if (o->score != MOE_SCORE_SOFTMAX && o->score != MOE_SCORE_SIGMOID)
    return fail(MOE_ERR_INVALID_ARG, "unknown score function %d", static_cast<int>(o->score));
  if (!(o->dynamic_threshold >= 0.f) || !(o->capacity_factor >= 0.f) ||
      !(o->dynamic_threshold < 1e30f) || !(o->capacity_factor < 1e30f))
    return fail(MOE_ERR_INVALID_ARG, "dynamic_threshold and capacity_factor must be finite and >= 0");
  if (o->seq_len < 0 || (o->seq_len > 0 && o->seq_len % moe::kRouterTokensPerCta != 0))
    return fail(MOE_ERR_INVALID_ARG, "seq_len must be 0 or a multiple of %d (got %lld)",
                moe::kRouterTokensPerCta, static_cast<long long>(o->seq_len));
  if (!forward && (o->capacity_factor > 0.f || o->balance))
    return fail(MOE_ERR_INVALID_ARG, "capacity_factor and balance need moe_ffn_forward_ex");
  if (o->selection_bias && !aligned16(o->selection_bias))
    return fail(MOE_ERR_ALIGNMENT, "selection_bias must be 16-byte aligned");
  if (o->balance && (reinterpret_cast<uintptr_t>(o->balance) & 3u))
    return fail(MOE_ERR_ALIGNMENT, "balance must be 4-byte aligned");
  return MOE_OK;
}

// True when any routing option differs from its default (off).
bool opts_active(const moe_route_opts_t* o) {
  return o && (o->score != MOE_SCORE_SOFTMAX || o->selection_bias || o->dynamic_threshold > 0.f ||
               o->capacity_factor > 0.f || o->slot_kept || o->balance);
}

void apply_opts(moe::RouteArgs& a, const moe_route_opts_t* o) {
  if (!o) return;
  a.score = o->score == MOE_SCORE_SIGMOID ? 1 : 0;
  a.sel_bias = o->selection_bias;
  a.dyn_threshold = o->dynamic_threshold;
  a.slot_kept = o->slot_kept;
}

}  // namespace

extern "C" {

int moe_abi_version(void) { return MOE_ABI_VERSION; }

int moe_set_fused_gather(int mode) {
  if (mode != MOE_FUSED_GATHER_OFF && mode != MOE_FUSED_GATHER_ON && mode != MOE_FUSED_GATHER_AUTO)
    return -1;
  return g_fused_gather.exchange(mode);
}

int moe_set_pdl(int on) { return g_pdl.exchange(on ? 1 : 0); }

int moe_set_gemm_mode(int mode) {
  if (mode != MOE_GEMM_AUTO && mode != MOE_GEMM_1SM && mode != MOE_GEMM_2SM) return -1;
  return g_gemm_mode.exchange(mode);
}

int moe_set_tail_swap(int max_rows) {
  if (max_rows < 0 || max_rows > MOE_TAIL_SWAP_MAX) return -1;
  return g_tail_swap.exchange(max_rows);
}

int moe_set_small_cluster(int ctas) {
  if (ctas != MOE_SMALL_CLUSTER_AUTO && ctas != 8 && ctas != 16) return -1;
  return g_small_cluster.exchange(ctas);
}

const char* moe_last_error(void) { return g_last_error.c_str(); }

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_ACT: return "unsupported activation";
    case MOE_ERR_DTYPE: return "unsupported dtype";
    case MOE_ERR_SHAPE: return "unsupported shape";
    case MOE_ERR_ALIGNMENT: return "misaligned pointer or size";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "a bounded wait in a kernel timed out";
    case MOE_ERR_DEVICE: return "unsupported device";
  }
  return "unknown status";
}

const char* moe_stage_name(int stage) {
  static const char* names[MOE_NUM_STAGES] = {"router", "permute", "gate_up", "down", "combine",
                                              "small_layer"};
  return (stage >= 0 && stage < MOE_NUM_STAGES) ? names[stage] : "";
}

size_t moe_ffn_workspace_size(int64_t T, int64_t D, int64_t F, int E, int K, moe_dtype_t dt,
                              moe_act_t act) {
  if (check_common(T, D, E, K, dt) != MOE_OK || F <= 0) return 0;
  if (act != MOE_ACT_SILU_GATED && act != MOE_ACT_RELU) return 0;
  if (!shapes_ok(T, D, F, E, K, act)) return 0;
  return layout(T, D, F, E, K, dt == MOE_BF16 ? 2 : 4).total;
}

moe_status_t moe_route(const void* x, const void* router, const float* router_bias, int64_t T,
                       int64_t D, int E, int K, int norm_topk_prob, moe_dtype_t dt,
                       float* router_logits, int64_t* selected_experts, float* routing_weights,
                       void* stream) {
  return moe_route_ex(x, router, router_bias, T, D, E, K, norm_topk_prob, dt, router_logits,
                      selected_experts, routing_weights, nullptr, stream);
}

moe_status_t moe_route_ex(const void* x, const void* router, const float* router_bias, int64_t T,
                          int64_t D, int E, int K, int norm_topk_prob, moe_dtype_t dt,
                          float* router_logits, int64_t* selected_experts, float* routing_weights,
                          const moe_route_opts_t* opts, void* stream) {
  g_last_error.clear();
  moe_status_t st = check_common(T, D, E, K, dt);
  if (st != MOE_OK) return st;
  if ((st = check_opts(opts, false)) != MOE_OK) return st;
  if (!x || !router || !selected_experts || !routing_weights)
    return fail(MOE_ERR_INVALID_ARG, "x, router, selected_experts and routing_weights are required");
  const void* ptrs[] = {x, router, router_bias, router_logits, selected_experts, routing_weights};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(MOE_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
  DevInfo* dev = nullptr;
  if ((st = device_info(&dev)) != MOE_OK) return st;
  moe::RouteArgs a{};
  a.x = x;
  a.router = router;
  a.router_bias = router_bias;
  a.T = static_cast<int>(T);
  a.D = static_cast<int>(D);
  a.E = E;
  a.K = K;
  a.norm = norm_topk_prob ? 1 : 0;
  a.dt = dt == MOE_BF16 ? moe::kBF16 : moe::kF32;
  a.logits = router_logits;
  a.sel64 = selected_experts;
  a.wout = routing_weights;
  a.err = dev->err;
  apply_opts(a, opts);
  cudaError_t e = dt == MOE_BF16 ? moe::launch_router_tc(a, static_cast<cudaStream_t>(stream))
                                 : moe::launch_router(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "router launch");
  return MOE_OK;
}

moe_status_t moe_ffn_forward(const void* x, const void* router, const void* gate_up_proj,
                             const void* down_proj, int E, int K, int norm_topk_prob,
                             moe_act_t act, void* out, int64_t* selected_experts,
                             float* routing_weights, int64_t T, int64_t D, int64_t F,
                             moe_dtype_t dt, const float* router_bias, const float* b1,
                             const float* b2, float* router_logits, void* workspace,
                             size_t workspace_bytes, void* stream) {
  return moe_ffn_forward_ex(x, router, gate_up_proj, down_proj, E, K, norm_topk_prob, act, out,
                            selected_experts, routing_weights, T, D, F, dt, router_bias, b1, b2,
                            router_logits, workspace, workspace_bytes, nullptr, stream);
}

moe_status_t moe_ffn_forward_ex(const void* x, const void* router, const void* gate_up_proj,
                                const void* down_proj, int E, int K, int norm_topk_prob,
                                moe_act_t act, void* out, int64_t* selected_experts,
                                float* routing_weights, int64_t T, int64_t D, int64_t F,
                                moe_dtype_t dt, const float* router_bias, const float* b1,
                                const float* b2, float* router_logits, void* workspace,
                                size_t workspace_bytes, const moe_route_opts_t* opts,
                                void* stream) {
  return moe::ffn_forward_impl(x, router, gate_up_proj, down_proj, E, K, norm_topk_prob, act, out,
                               selected_experts, routing_weights, T, D, F, dt, router_bias, b1, b2,
                               router_logits, workspace, workspace_bytes, opts, stream, true);
}

}  // extern "C"

namespace moe {
moe_status_t ffn_forward_impl(const void* x, const void* router, const void* gate_up_proj,
                              const void* down_proj, int E, int K, int norm_topk_prob,
                              moe_act_t act, void* out, int64_t* selected_experts,
                              float* routing_weights, int64_t T, int64_t D, int64_t F,
                              moe_dtype_t dt, const float* router_bias, const float* b1,
                              const float* b2, float* router_logits, void* workspace,
                              size_t workspace_bytes, const moe_route_opts_t* opts, void* stream,
                              bool with_aux) {
  g_last_error.clear();
  moe_status_t st = check_common(T, D, E, K, dt);
  if (st != MOE_OK) return st;
  if ((st = check_opts(opts, true)) != MOE_OK) return st;
  if (act != MOE_ACT_SILU_GATED && act != MOE_ACT_RELU)
    return fail(MOE_ERR_UNSUPPORTED_ACT, "activation %d not supported (SiLU-gated or ReLU)",
                static_cast<int>(act));
  if (F <= 0) return fail(MOE_ERR_INVALID_ARG, "F=%lld must be positive", static_cast<long long>(F));
  if (!shapes_ok(T, D, F, E, K, act)) return fail(MOE_ERR_SHAPE, "sizes exceed 32-bit indexing");
  if (!x || !router || !gate_up_proj || !down_proj || !out)
    return fail(MOE_ERR_INVALID_ARG, "x, router, gate_up_proj, down_proj and out are required");
  if (act == MOE_ACT_RELU && (!b1 || !b2 || !router_bias))
    return fail(MOE_ERR_INVALID_ARG, "the ReLU expert needs router_bias, b1 and b2");
  if (act == MOE_ACT_SILU_GATED && (b1 || b2))
    return fail(MOE_ERR_INVALID_ARG, "the SiLU-gated expert has no b1/b2");
  const void* ptrs[] = {x, router, gate_up_proj, down_proj, out, selected_experts, routing_weights,
                        router_bias, b1, b2, router_logits, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(MOE_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
  if (dt == MOE_BF16 && (D % 8 != 0 || F % 8 != 0))
    return fail(MOE_ERR_ALIGNMENT, "bf16 path needs D and F multiples of 8 (D=%lld F=%lld)",
                static_cast<long long>(D), static_cast<long long>(F));
  const int elem = dt == MOE_BF16 ? 2 : 4;
  const Layout L = layout(T, D, F, E, K, elem);
  if (!workspace || workspace_bytes < L.total)
    return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", L.total,
                workspace ? workspace_bytes : static_cast<size_t>(0));
  DevInfo* dev = nullptr;
  if ((st = device_info(&dev, with_aux)) != MOE_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* idx32 = reinterpret_cast<int*>(ws + L.idx32);
  float* w32 = reinterpret_cast<float*>(ws + L.w32);
  int* bcount = reinterpret_cast<int*>(ws + L.bcount);
  int* bbase = reinterpret_cast<int*>(ws + L.bbase);
  int* totals = reinterpret_cast<int*>(ws + L.totals);
  int* offsets = reinterpret_cast<int*>(ws + L.offsets);
  int* sched = reinterpret_cast<int*>(ws + L.sched);
  int* perm = reinterpret_cast<int*>(ws + L.perm);
  int* pos = reinterpret_cast<int*>(ws + L.pos);
  void* xperm = ws + L.xperm;
  void* H = ws + L.h;
  void* Y = ws + L.y;
  float* bal = reinterpret_cast<float*>(ws + L.bal);
  float* part = L.split ? reinterpret_cast<float*>(ws + L.part) : nullptr;
  const float cap = opts ? opts->capacity_factor : 0.f;
  const int seq_len = opts ? static_cast<int>(opts->seq_len) : 0;
  float* balance_out = opts ? opts->balance : nullptr;
  uint8_t* slot_kept = opts ? opts->slot_kept : nullptr;
  // bf16: gate_up reads the token rows of x directly (TMA gather), so the
  // expert-sorted copy is not materialised; automatically for layers on the
  // one-CTA GEMM whose experts average at most 16 routed rows
  const int fg_mode = g_fused_gather.load();
  const bool pair_gemm = g_gemm_mode.load() == MOE_GEMM_2SM ||
                         (g_gemm_mode.load() == MOE_GEMM_AUTO && T * K >= 512LL * E);
  const bool fused_gather =
      dt == MOE_BF16 && (fg_mode == MOE_FUSED_GATHER_ON ||
                         (fg_mode == MOE_FUSED_GATHER_AUTO && !pair_gemm && T * K <= 16LL * E));
  const int Ti = static_cast<int>(T), Di = static_cast<int>(D), Fi = static_cast<int>(F);
  const int gu_act = act == MOE_ACT_SILU_GATED ? 0 : 1;
  const int gu_rows = act == MOE_ACT_SILU_GATED ? 2 * Fi : Fi;

  StageTimer timer(s);
  cudaError_t e;
  if (dt == MOE_F32 && !opts_active(opts) && moe::small_layer_fits(Ti, Di, Fi, E, K, gu_act == 0)) {
    // a small float32 layer: the whole forward in one launch
    e = timer.run(5, [&] {
      return moe::launch_small_layer_f32(
          static_cast<const float*>(x), static_cast<const float*>(router), router_bias,
          static_cast<const float*>(gate_up_proj), static_cast<const float*>(down_proj), b1, b2,
          Ti, Di, Fi, E, K, norm_topk_prob ? 1 : 0, gu_act == 0 ? 1 : 0, static_cast<float*>(out),
          selected_experts, routing_weights, router_logits, g_small_cluster.load(), s);
    });
    if (e != cudaSuccess) return cuda_fail(e, "small-layer launch");
    if (!debug_wait(dev, s, "small layer")) return MOE_ERR_TIMEOUT;
    return MOE_OK;
  }
  e = timer.run(0, [&] {
    moe::RouteArgs a{};
    a.x = x;
    a.router = router;
    a.router_bias = router_bias;
    a.T = Ti;
    a.D = Di;
    a.E = E;
    a.K = K;
    a.norm = norm_topk_prob ? 1 : 0;
    a.dt = dt == MOE_BF16 ? moe::kBF16 : moe::kF32;
    a.logits = router_logits;
    a.sel64 = selected_experts;
    a.wout = routing_weights;
    a.idx32 = idx32;
    a.w32 = w32;
    a.blockcounts = bcount;
    a.err = dev->err;
    apply_opts(a, opts);
    a.bal_partial = balance_out ? bal : nullptr;
    cudaError_t r = dt == MOE_BF16 ? moe::launch_router_tc(a, s) : moe::launch_router(a, s);
    if (r != cudaSuccess || !balance_out) return r;
    const int parts = dt == MOE_BF16 ? moe::router_tc_parts(Ti) : moe::router_simt_parts(Ti);
    return moe::launch_balance_finalize(bal, parts, E, Ti, balance_out, s);
  });
  if (e != cudaSuccess) return cuda_fail(e, "router launch");
  if (!debug_wait(dev, s, "router")) return MOE_ERR_TIMEOUT;
  e = timer.run(1, [&] {
    cudaError_t r = cudaSuccess;
    if (cap > 0.f) {
      r = moe::launch_capacity_clamp(bcount, L.B, E, Ti, K, seq_len, cap, s);
      if (r != cudaSuccess) return r;
      if (!debug_wait(dev, s, "capacity clamp")) return cudaErrorTimeout;
    }
    // a small block-count table is scanned by the scatter blocks themselves
    const bool own_scan = static_cast<long long>(L.B) * E <= kScatterScansItself;
    if (!own_scan) {
      r = moe::launch_permute_scan(bcount, L.B, E, bbase, totals, s);
      if (r != cudaSuccess) return r;
      if (!debug_wait(dev, s, "permute scan")) return cudaErrorTimeout;
    }
    r = moe::launch_permute_scatter(idx32, own_scan ? nullptr : bbase, own_scan ? nullptr : totals,
                                    bcount, Ti, K, E, offsets, perm, pos, slot_kept, sched, s);
    if (r != cudaSuccess) return r;
    if (!debug_wait(dev, s, "permute scatter")) return cudaErrorTimeout;
    if (fused_gather) return r;
    r = moe::launch_gather_rows(perm, offsets, pos, Ti, E, K, x, Di * elem, xperm, s);
    if (r != cudaSuccess) return r;
    return debug_wait(dev, s, "row gather") ? cudaSuccess : cudaErrorTimeout;
  });
  if (e == cudaErrorTimeout) return MOE_ERR_TIMEOUT;
  if (e != cudaSuccess) return cuda_fail(e, "permute launch");
  if (dt == MOE_BF16) {
    e = timer.run(2, [&] {
      return launch_gemm_bf16(gu_act, fused_gather ? x : xperm, L.Rpad, gate_up_proj, offsets, E,
                              Ti, K, Di, Fi, gu_rows, b1, H, dev->err, sched + moe::kSchedGateUp,
                              part, part ? sched + moe::kSchedFlagsGateUp : nullptr, s,
                              fused_gather ? perm : nullptr);
    });
    if (e != cudaSuccess) return cuda_fail(e, "gate_up launch");
    if (!debug_wait(dev, s, "gate_up GEMM")) return MOE_ERR_TIMEOUT;
    e = timer.run(3, [&] {
      return launch_gemm_bf16(2, H, L.Rpad, down_proj, offsets, E, Ti, K, Fi, Di, Di, b2, Y,
                              dev->err, sched + moe::kSchedDown, part,
                              part ? sched + moe::kSchedFlagsDown : nullptr, s);
    });
    if (e != cudaSuccess) return cuda_fail(e, "down launch");
    if (!debug_wait(dev, s, "down GEMM")) return MOE_ERR_TIMEOUT;
  } else {
    e = timer.run(2, [&] {
      return moe::launch_gemm_simt_f32(gu_act, static_cast<const float*>(xperm),
                                       static_cast<const float*>(gate_up_proj), offsets, E, Ti, Di,
                                       Fi, gu_rows, b1, static_cast<float*>(H), s);
    });
    if (e != cudaSuccess) return cuda_fail(e, "gate_up launch");
    e = timer.run(3, [&] {
      return moe::launch_gemm_simt_f32(2, static_cast<const float*>(H),
                                       static_cast<const float*>(down_proj), offsets, E, Ti, Fi, Di,
                                       Di, b2, static_cast<float*>(Y), s);
    });
    if (e != cudaSuccess) return cuda_fail(e, "down launch");
  }
  e = timer.run(4, [&] {
    return moe::launch_combine(Y, w32, pos, Ti, K, Di, dt == MOE_BF16 ? moe::kBF16 : moe::kF32, out,
                               s);
  });
  if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  if (!debug_wait(dev, s, "combine")) return MOE_ERR_TIMEOUT;
  return MOE_OK;
}
}  // namespace moe

extern "C" {

moe_status_t moe_debug_bounded_wait(int timeout_ms, void* stream) {
  g_last_error.clear();
  if (timeout_ms < 1 || timeout_ms > 2000)
    return fail(MOE_ERR_INVALID_ARG, "timeout_ms=%d outside [1, 2000]", timeout_ms);
  DevInfo* dev = nullptr;
  moe_status_t st = device_info(&dev);
  if (st != MOE_OK) return st;
  cudaError_t e = moe::launch_bounded_wait_probe(static_cast<unsigned long long>(timeout_ms) * 1000000ull,
                                                 dev->err, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "bounded wait launch");
  return MOE_OK;
}

const char* moe_error_sites(unsigned int word) {
  static const char* const kNames[] = {"router producer", "router mma", "router epilogue",
                                       "gemm producer", "gemm mma", "gemm epilogue",
                                       "pair gemm producer", "pair gemm mma",
                                       "pair gemm epilogue", "bounded-wait probe"};
  thread_local std::string out;
  out.clear();
  for (int b = 0; b < static_cast<int>(sizeof(kNames) / sizeof(kNames[0])); ++b)
    if (word & (1u << (8 + b))) {
      if (!out.empty()) out += ", ";
      out += kNames[b];
    }
  return out.c_str();
}

moe_status_t moe_device_error_peek(unsigned int* word) {
  g_last_error.clear();
  if (!word) return fail(MOE_ERR_INVALID_ARG, "word is NULL");
  DevInfo* dev = nullptr;
  moe_status_t st = device_info(&dev);
  if (st != MOE_OK) return st;
  if (!peek_word(dev, word, 1000))
    return fail(MOE_ERR_TIMEOUT, "the device did not answer a 4-byte copy within 1 s");
  return MOE_OK;
}

unsigned long long moe_kernel_launches(void) { return moe::kernel_launches(); }

int moe_set_debug_sync(int timeout_ms) { return g_debug_sync_ms.exchange(timeout_ms > 0 ? timeout_ms : 0); }

moe_status_t moe_device_status(void* stream) {
  g_last_error.clear();
  DevInfo* dev = nullptr;
  moe_status_t st = device_info(&dev);
  if (st != MOE_OK) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int word = 0;
  e = cudaMemcpy(&word, dev->err, sizeof word, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the error word");
  if (word != 0) {
    const unsigned int zero = 0;
    cudaMemcpy(dev->err, &zero, sizeof zero, cudaMemcpyHostToDevice);
    return fail(MOE_ERR_TIMEOUT, "device error word 0x%x (1 = a bounded wait timed out; in: %s)",
                word, moe_error_sites(word));
  }
  return MOE_OK;
}

moe_status_t moe_profile_enable(int enable) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  g_prof.enabled = enable != 0;
  g_prof.recs.clear();
  g_prof.next = 0;
  g_prof.calls = 0;
  return MOE_OK;
}

int moe_profile_read(float* ms, int n_stages) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  for (int i = 0; i < n_stages; ++i) ms[i] = 0.f;
  for (auto& r : g_prof.recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.second.second) == cudaSuccess &&
        cudaEventElapsedTime(&t, r.second.first, r.second.second) == cudaSuccess &&
        r.first < n_stages)
      ms[r.first] += t;
  }
  const int calls = g_prof.calls;
  g_prof.recs.clear();
  g_prof.next = 0;
  g_prof.calls = 0;
  return calls;
}

}  // extern "C"

namespace moe {
bool pdl_enabled() { return g_pdl.load() != 0; }

std::atomic<unsigned long long> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
unsigned long long kernel_launches() { return g_launches.load(); }

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_dev_mu);
  if (dev >= 0 && dev < 64 && g_dev[dev].init) return g_dev[dev].sms;
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}
}  // namespace moe

namespace moe {
void set_last_error(const char* msg) { g_last_error = msg ? msg : ""; }
}  // namespace moe
