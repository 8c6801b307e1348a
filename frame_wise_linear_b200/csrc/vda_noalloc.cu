// vda_forward_noalloc: the forward with a scratch array owned by the library,
// for callers that cannot allocate device memory (see include/vda.h).
//
// The scratch is a file-scope __device__ array.  In host code its name is only
// a host-side stand-in, not a device address, so the device address is looked
// up with cudaGetSymbolAddress (with the device current) and the workspace
// pointer handed to the kernels is that address.
//
// That address belongs to a CUDA context, not to a device ordinal: the module
// holding the array is loaded once per context.  The lookup is therefore
// cached per context, keyed by the context's process-unique ID.  A device that
// was reset (cudaDeviceReset) gets a new primary context with a new ID, and a
// context a driver-API caller made current gets its own entry, so neither can
// be handed the address of another context's scratch.
#include <cudaTypedefs.h>
#include <stdio.h>

#include <mutex>

#include "vda_internal.cuh"

namespace {

constexpr size_t kScratchBytes = VDA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxContexts = 256;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

struct CachedAddress {
  unsigned long long ctx_id;
  void* addr;
};

std::mutex g_mu;
CachedAddress g_cache[kMaxContexts];
int g_cached = 0;
int g_next = 0;   // the entry a full cache replaces next

PFN_cuCtxGetCurrent_v4000 g_get_current = nullptr;
PFN_cuCtxGetId_v12000 g_get_id = nullptr;

// Driver entry points through the runtime (the library does not link libcuda).
bool driver_entry_points() {
  if (g_get_current && g_get_id) return true;
  void* a = nullptr;
  void* b = nullptr;
  cudaDriverEntryPointQueryResult qa, qb;
  if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &a, 4000, cudaEnableDefault, &qa) != cudaSuccess ||
      qa != cudaDriverEntryPointSuccess ||
      cudaGetDriverEntryPointByVersion("cuCtxGetId", &b, 12000, cudaEnableDefault, &qb) != cudaSuccess ||
      qb != cudaDriverEntryPointSuccess)
    return false;
  g_get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(a);
  g_get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(b);
  return true;
}

// ID of the context current on this thread (0 when none is).
cudaError_t current_context_id(unsigned long long* id) {
  *id = 0;
  CUcontext ctx = nullptr;
  if (g_get_current(&ctx) != CUDA_SUCCESS) return cudaErrorContextIsDestroyed;
  if (!ctx) return cudaSuccess;
  if (g_get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorContextIsDestroyed;
  return cudaSuccess;
}

// Device address of g_scratch in the context current on this thread.  The
// first call in a context makes the runtime's primary context current if no
// context is, and looks the address up.
cudaError_t scratch_address(void** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!driver_entry_points()) return cudaErrorNotSupported;
  unsigned long long id = 0;
  cudaError_t e = current_context_id(&id);
  if (e != cudaSuccess) return e;
  for (int i = 0; id && i < g_cached; ++i)
    if (g_cache[i].ctx_id == id) {
      *out = g_cache[i].addr;
      return cudaSuccess;
    }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_scratch);   // initialises the primary context if none is current
  if (e != cudaSuccess) return e;
  if (!id && (e = current_context_id(&id)) != cudaSuccess) return e;
  if (id) {
    const int slot = g_cached < kMaxContexts ? g_cached++ : g_next;
    g_next = (slot + 1) % kMaxContexts;
    g_cache[slot] = CachedAddress{id, p};
  }
  *out = p;
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
    snprintf(msg, sizeof(msg), "vda_forward_noalloc: looking up the scratch address: %s", cudaGetErrorString(e));
    vda::set_error_message(msg);
    return VDA_ERR_CUDA;
  }
  return vda_forward(p, Q, K, V, G, K_txt, V_txt, O, ws, kScratchBytes, stream);
}
