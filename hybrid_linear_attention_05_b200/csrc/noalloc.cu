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

#include "gdn_internal.h"

namespace {

// The scratch itself.  Every device that loads this library holds it (64 MiB)
// until the process exits.  In host code this name is only a host-side
// stand-in for the symbol: its device address comes from
// cudaGetSymbolAddress, once per device (scratch_on_current_device).
__device__ __align__(256) unsigned char g_gdn_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of the scratch on the current device, looked up on the first
// call for that device and cached.  Returns nullptr if the lookup fails.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p) return p;
  if (cudaGetSymbolAddress(&p, g_gdn_noalloc_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();  // do not leave this error for an unrelated later call to find
    return nullptr;
  }
  g_scratch_addr[dev].store(p, std::memory_order_release);
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
