// cca_prefill_noalloc: the prefill of one block with its workspace in memory
// the library owns, for callers that cannot allocate device memory.
//
// Why: some callers may not call cudaMalloc at all once they are running.
// cudaMalloc can synchronize the device and stall every stream of the
// process, so latency-bound serving loops avoid it; runtimes that own the
// whole device memory pool (and plugins hosted by them) forbid it; and a
// caller that already holds all the memory it was given has no way to get a
// workspace of the size cca_workspace_size asks for. Such callers pass only
// their inputs and outputs; the intermediates go to a fixed device array
// declared in this file.
//
// Limits and sharing: the array holds CCA_NOALLOC_WORKSPACE_BYTES (64 MiB);
// every GPU on which this entry point runs keeps that much memory until the
// process exits. That holds under lazy module loading (CUDA_MODULE_LOADING=LAZY,
// the default of recent CUDA runtimes); with CUDA_MODULE_LOADING=EAGER every
// device on which the library is loaded reserves the 64 MiB, used or not.
// Larger blocks are rejected with CCA_ERR_WORKSPACE. All calls
// share the one array: two calls whose work overlaps on the GPU (different
// streams, or different host threads on the same device) race on it, so they
// must be ordered by the caller. No part of the workspace has to start at
// zero: every byte a call reads was written earlier in the same call.
#include <stdio.h>

#include <mutex>

#include "../../include/cca.h"
#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

// The workspace of cca_prefill_noalloc. In host code this name is only a
// stand-in for the device symbol; its device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_workspace[CCA_NOALLOC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
void* g_ws_ptr[kMaxDevices] = {};
std::mutex g_ws_mu;

// Device address of the array on the current device, looked up once per device.
cudaError_t workspace_ptr(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_ws_mu);
  if (g_ws_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_workspace);
    if (e != cudaSuccess) return e;
    g_ws_ptr[dev] = p;
  }
  *out = g_ws_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace cca

extern "C" cca_status_t cca_prefill_noalloc(const cca_config_t* cfg, const void* x, const void* W_q,
                                            const void* W_k, const void* W_v, const void* convq_seq,
                                            const void* convq_chan, const void* convk_seq,
                                            const void* convk_chan, const void* W_o, void* y, void* k_cache,
                                            void* v_cache, void* conv_state, void* stream) {
  const size_t need = cca_workspace_size(cfg);
  if (need == 0) return cca_validate(cfg);  // invalid configuration: its own status and message
  if (need > (size_t)CCA_NOALLOC_WORKSPACE_BYTES) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "this block needs a %zu-byte workspace; the library's static workspace holds %zu bytes "
             "(use cca_prefill with a caller-allocated workspace)",
             need, (size_t)CCA_NOALLOC_WORKSPACE_BYTES);
    return (cca_status_t)cca::set_last_error(CCA_ERR_WORKSPACE, msg);
  }
  void* ws = nullptr;
  const cudaError_t e = cca::workspace_ptr(&ws);
  if (e != cudaSuccess) {
    char msg[200];
    snprintf(msg, sizeof(msg), "cudaGetSymbolAddress of the static workspace: %s", cudaGetErrorString(e));
    return (cca_status_t)cca::set_last_error(CCA_ERR_CUDA, msg);
  }
  return cca_prefill(cfg, x, W_q, W_k, W_v, convq_seq, convq_chan, convk_seq, convk_chan, W_o, y, k_cache,
                     v_cache, conv_state, ws, (size_t)CCA_NOALLOC_WORKSPACE_BYTES, stream);
}
