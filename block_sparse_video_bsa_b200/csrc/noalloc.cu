// bsa_forward_noalloc: the whole forward path for callers that cannot
// allocate device memory.
//
// bsa_forward needs a caller-provided workspace for the intermediates of its
// four stages (pooled Q/K, anchor, summaries, bias, block lists).  Some hosts
// cannot provide one: a plugin running inside a framework whose memory pool
// owns the device (a cudaMalloc there bypasses the pool's accounting or is
// forbidden by its policy), a server that reserves all device memory at
// start-up and treats any later allocation as a fault, or latency-critical
// code that cannot afford cudaMalloc's implicit device-wide synchronisation.
// For them this file keeps the workspace in a fixed-size static device array
// instead, and the entry point never calls cudaMalloc, cudaFree or any
// allocating library routine.
#include <mutex>

#include "bsa.h"
#include <cuda_runtime.h>

namespace {

// The scratch area.  Every GPU on which the library is used holds these
// BSA_NOALLOC_SCRATCH_BYTES from module load until the process exits.
__device__ __align__(256) unsigned char g_noalloc_scratch[BSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_dev_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the name g_noalloc_scratch is only a host-side stand-in; the real address
// comes from cudaGetSymbolAddress, looked up once per device with that
// device current (the first call on a device does this set-up).
int scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_dev_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();   // clear it, so a later call's launch check does not report it
      return BSA_ERR_CUDA;
    }
    g_scratch_dev_ptr[dev] = p;
  }
  *out = g_scratch_dev_ptr[dev];
  return BSA_OK;
}

}  // namespace

extern "C" int bsa_forward_noalloc(const bsa_params* p, const void* Q, const void* K,
                                   const void* V, void* O, float* lse, void* stream) {
  const size_t need = bsa_workspace_bytes(p);
  if (need == 0) return BSA_ERR_INVALID;
  if (need > static_cast<size_t>(BSA_NOALLOC_SCRATCH_BYTES)) return BSA_ERR_SCRATCH;
  void* ws = nullptr;
  const int rc = scratch_on_current_device(&ws);
  if (rc != BSA_OK) return rc;
  // Nothing in the scratch has to start at zero: each stage writes every
  // intermediate it produces in full before the next stage reads it, so the
  // previous call's leftovers are never read.
  return bsa_forward(p, Q, K, V, O, lse, ws, static_cast<size_t>(BSA_NOALLOC_SCRATCH_BYTES),
                     stream);
}
