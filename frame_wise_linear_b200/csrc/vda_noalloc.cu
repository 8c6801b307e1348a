// vda_forward_noalloc: the forward with a scratch array owned by the library,
// for callers that cannot allocate device memory (see include/vda.h).
//
// The scratch is a file-scope __device__ array.  In host code its name is only
// a host-side stand-in, not a device address, so the device address is looked
// up with cudaGetSymbolAddress once per device (with that device current) and
// cached; the workspace pointer handed to the kernels is that address.
#include <stdio.h>

#include <mutex>

#include "vda_internal.cuh"

namespace {

constexpr size_t kScratchBytes = VDA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 128;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up on first use).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" vda_status vda_forward_noalloc(const vda_problem* p, const void* Q, const void* K,
                                          const void* V, const void* G, const void* K_txt,
                                          const void* V_txt, void* O, void* stream) {
  size_t need = 0;
  vda_status s = vda_workspace_size(p, &need);
  if (s != VDA_OK) return s;
  if (need > kScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "vda_forward_noalloc: the problem needs %zu bytes of workspace, above the library's "
             "static scratch of %zu bytes; use vda_forward with a caller-provided workspace",
             need, kScratchBytes);
    vda::set_error_message(msg);
    return VDA_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  cudaError_t e = scratch_address(&ws);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "vda_forward_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    vda::set_error_message(msg);
    return VDA_ERR_CUDA;
  }
  return vda_forward(p, Q, K, V, G, K_txt, V_txt, O, ws, kScratchBytes, stream);
}
