// moe_ffn_forward_noalloc: the forward for callers that cannot allocate
// device memory when they call us (for example a plugin or callback inside
// another runtime that owns all device memory and passes only the tensors
// the layer reads and writes).  Instead of a caller-provided workspace it
// uses one static device array, sized MOE_NOALLOC_SCRATCH_BYTES, that each
// GPU loading this file's module keeps until the process exits.
//
// No call here allocates: the array is static, its device address is looked
// up once per device with cudaGetSymbolAddress, and the work itself is the
// ordinary forward with that address as its workspace, run without the host
// bookkeeping (stream, event, pinned word) the other entry points set up.
// The addresses cached per device belong to the process's CUDA context: a
// cudaDeviceReset invalidates them, and calls after one are not supported.
#include <stdio.h>

#include <mutex>

#include "../../include/moe.h"
#include "internal.h"

namespace {

// Scratch of the no-allocation entry point.  In host code this name is only
// a stand-in for the symbol; its device address comes from
// cudaGetSymbolAddress below and is what the kernels receive.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
void* g_scratch_ptr[64];

// Device address of the scratch on the current device, looked up on the
// first call for that device.
moe_status_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    moe::set_last_error(cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  if (dev < 0 || dev >= 64) {
    moe::set_last_error("device ordinal out of range");
    return MOE_ERR_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char buf[256];
      snprintf(buf, sizeof buf, "cudaGetSymbolAddress(no-allocation scratch): %s",
               cudaGetErrorString(e));
      moe::set_last_error(buf);
      return MOE_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_ffn_forward_noalloc(const void* x, const void* router,
                                                const void* gate_up_proj, const void* down_proj,
                                                int E, int K, int norm_topk_prob, moe_act_t act,
                                                void* out, int64_t* selected_experts,
                                                float* routing_weights, int64_t T, int64_t D,
                                                int64_t F, moe_dtype_t dt,
                                                const float* router_bias, const float* b1,
                                                const float* b2, float* router_logits,
                                                void* stream) {
  const size_t need = moe_ffn_workspace_size(T, D, F, E, K, dt, act);
  if (need == 0) {
    // invalid sizes: let the ordinary entry point report exactly which
    // argument is wrong (it validates before touching the workspace)
    return moe::ffn_forward_impl(x, router, gate_up_proj, down_proj, E, K, norm_topk_prob, act,
                                 out, selected_experts, routing_weights, T, D, F, dt, router_bias,
                                 b1, b2, router_logits, nullptr, 0, nullptr, stream, false);
  }
  if (need > MOE_NOALLOC_SCRATCH_BYTES) {
    char buf[256];
    snprintf(buf, sizeof buf,
             "these sizes need %zu bytes of scratch; the static scratch holds %zu "
             "(use moe_ffn_forward with a caller workspace)",
             need, static_cast<size_t>(MOE_NOALLOC_SCRATCH_BYTES));
    moe::set_last_error(buf);
    return MOE_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  const moe_status_t st = scratch_address(&scratch);
  if (st != MOE_OK) return st;
  return moe::ffn_forward_impl(x, router, gate_up_proj, down_proj, E, K, norm_topk_prob, act, out,
                               selected_experts, routing_weights, T, D, F, dt, router_bias, b1, b2,
                               router_logits, scratch, MOE_NOALLOC_SCRATCH_BYTES, nullptr, stream,
                               false);
}
