// gdn_prefill_noalloc: gdn_prefill with the scratch held inside the library.
//
// gdn_prefill needs a device workspace for the normalised q, k, v and the
// gates that pass between its two kernels.  Some callers cannot provide one:
// an operator plugin that is handed only its input and output tensors, with
// no allocator to ask for temporary memory, or a runtime that has divided up
// all device memory in advance and allows no allocation (and no implicit
// device synchronisation of cudaMalloc / cudaFree) while it serves requests.
// For them this file keeps one fixed scratch array in device memory, sized
// for up to GDN_NOALLOC_SCRATCH_BYTES of workspace, and runs the ordinary
// gdn_prefill path on it.  Nothing here allocates.
#include <stdint.h>

#include <atomic>

#include <cuda.h>

#include "gdn_internal.h"

namespace {

// The scratch itself (64 MiB per device, held until the process exits).
// With CUDA's lazy module loading (the default) the device memory behind it is
// committed when this module is first loaded on a device, which is the first
// gdn_prefill_noalloc call there (its cudaGetSymbolAddress).  In host code
// this name is only a host-side stand-in for the symbol: its device address
// comes from cudaGetSymbolAddress (scratch_on_current_device).
__device__ __align__(256) unsigned char g_gdn_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Process-unique id of the current CUDA context (0 when there is none or it
// cannot be read).  A context made after cudaDeviceReset gets a new id.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!get_current || !get_id) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess || qb != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return 0;
    }
    get_current = reinterpret_cast<CtxGetCurrentFn>(a);
    get_id = reinterpret_cast<CtxGetIdFn>(b);
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

constexpr int kMaxDevices = 64;
struct CachedAddress {
  std::atomic<unsigned long long> ctx_id{0};
  std::atomic<void*> addr{nullptr};
};
CachedAddress g_scratch[kMaxDevices];

// Device address of the scratch on the current device.  It is looked up with
// cudaGetSymbolAddress on the first call for that device and cached together
// with the id of the context it belongs to; a call in a different context (the
// device was reset with cudaDeviceReset since) looks it up again.  Returns
// nullptr if the lookup fails.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  const unsigned long long id = current_context_id();
  void* p = g_scratch[dev].addr.load(std::memory_order_acquire);
  if (p && id != 0 && g_scratch[dev].ctx_id.load(std::memory_order_acquire) == id) return p;
  p = nullptr;
  if (cudaGetSymbolAddress(&p, g_gdn_noalloc_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();  // do not leave this error for an unrelated later call to find
    return nullptr;
  }
  // the lookup created the context if there was none: take its id now
  g_scratch[dev].ctx_id.store(id != 0 ? id : current_context_id(), std::memory_order_release);
  g_scratch[dev].addr.store(p, std::memory_order_release);
  return p;
}

}  // namespace

extern "C" gdn_status gdn_prefill_noalloc(const gdn_dims* dims, const gdn_prefill_args* args,
                                          void* stream) {
  if (!dims || !args) return GDN_ERR_NULL;
  if (args->reuse_workspace) return GDN_ERR_UNSUPPORTED;  // the scratch holds no state map's records
  const size_t need = gdn_prefill_workspace_size(dims, args->T_tot, args->dtype);
  if (args->T_tot > 0 && need == 0) return gdn_prefill(dims, args, stream);  // reports the bad size
  if (need > (size_t)GDN_NOALLOC_SCRATCH_BYTES) return GDN_ERR_WORKSPACE;
  void* scratch = scratch_on_current_device();
  if (!scratch) return GDN_ERR_CUDA;
  gdn_prefill_args a = *args;
  a.workspace = scratch;
  a.workspace_bytes = (size_t)GDN_NOALLOC_SCRATCH_BYTES;
  return gdn_prefill(dims, &a, stream);
}
