// coli_static.cu -- a layer forward whose scratch lives in a fixed device
// array inside the library, for callers that cannot allocate device memory.
//
// Who needs it: hosts that own every device allocation and hand a plugin no
// allocator (nothing to pass as `workspace`), and serving loops that may not
// call cudaMalloc after start-up because cudaMalloc can synchronise the
// device and stall every stream in flight.  Such callers still pass their
// own inputs and outputs; only the scratch comes from here.
#include <cstdio>
#include <mutex>

#include "../../include/coli.h"
#include "coli_launch.h"

#define COLI_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB

// The scratch.  Every GPU that loads this library holds these 8 MiB until
// the process exits.  Host code must not use the symbol as an address: it is
// a host-side stand-in, so its device address is looked up per device below.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device (looked up once per
// device, with that device current).  The cached address assumes that the
// device's primary context lives as long as the process: after
// cudaDeviceReset the module is loaded afresh, so a process that resets a
// device must not call the no-allocation forward on it again.
cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

cudaError_t coli::noalloc_scratch(void** out) { return scratch_on_current_device(out); }

COLI_EXPORT coli_status coli_moe_layer_forward_noalloc(const coli_moe_layer* layer, const float* x, int64_t n_tok,
                                                       float* out, void* stream) {
  char msg[320];
  if (layer == nullptr) {
    coli::set_error_message("coli_moe_layer_forward_noalloc: null layer");
    return COLI_EINVAL;
  }
  // the token range of coli_moe_layer_forward, checked before the scratch
  // need is computed (its size arithmetic is only meaningful inside it)
  if (n_tok < 0 || n_tok > (int64_t(1) << 24)) {
    snprintf(msg, sizeof msg, "coli_moe_layer_forward_noalloc: n_tok=%lld outside [0, 2^24]", (long long)n_tok);
    coli::set_error_message(msg);
    return COLI_EINVAL;
  }
  const size_t need = coli_moe_workspace_bytes(&layer->cfg, n_tok);
  if (need == 0) return coli_moe_layer_forward(layer, x, n_tok, out, nullptr, 0, stream);  // reports the cfg error
  if (need > kStaticScratchBytes) {
    snprintf(msg, sizeof msg,
             "coli_moe_layer_forward_noalloc: %lld tokens need %zu bytes of scratch, more than the fixed %zu; "
             "use coli_moe_layer_forward with a workspace",
             (long long)n_tok, need, kStaticScratchBytes);
    coli::set_error_message(msg);
    return COLI_EINVAL;
  }
  if (n_tok == 0) return COLI_OK;
  void* ws = nullptr;
  const cudaError_t e = scratch_on_current_device(&ws);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof msg, "coli_moe_layer_forward_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    coli::set_error_message(msg);
    return COLI_ECUDA;
  }
  // Nothing in the scratch has to start at zero: every kernel of the forward
  // writes each scratch word before it reads it.
  return coli_moe_layer_forward(layer, x, n_tok, out, ws, kStaticScratchBytes, stream);
}
