// fathom_scan_topk_noalloc: the scan for callers that cannot allocate device
// memory (see include/fathom.h).  The scan's workspace is a fixed array in
// the library's own device memory instead of a caller buffer; the kernels
// and launch sequence are those of fathom_scan_topk.
#include <cuda_runtime.h>
#include <stdio.h>

#include <mutex>

#include "fathom.h"

namespace fathom {
void set_error_message(const char *msg);
}

namespace {

// The scratch every call uses.  Each device that loads the library holds one
// copy of it until the process exits.
static __device__ __align__(256) unsigned char g_fathom_noalloc_scratch[FATHOM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device.  In host code the array's name only stands for the symbol; the
// kernels must be given this address.
fathom_status scratch_on_current_device(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "no current device: %s", cudaGetErrorString(e));
    fathom::set_error_message(msg);
    return FATHOM_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    fathom::set_error_message("device index beyond the no-alloc scratch table");
    return FATHOM_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fathom_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[256];
      snprintf(msg, sizeof(msg), "cudaGetSymbolAddress of the scratch failed: %s",
               cudaGetErrorString(e));
      fathom::set_error_message(msg);
      return FATHOM_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FATHOM_OK;
}

}  // namespace

extern "C" fathom_status fathom_scan_topk_noalloc(const fathom_scan_args *args, void *stream) {
  const size_t need = fathom_scan_topk_workspace_size(args);
  if (need == 0) return fathom_scan_topk(args, nullptr, 0, stream);  // reports the bad argument
  if (need > FATHOM_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "this scan needs %zu bytes of scratch; the built-in scratch holds %zu "
             "(use fathom_scan_topk with a caller workspace)",
             need, (size_t)FATHOM_NOALLOC_SCRATCH_BYTES);
    fathom::set_error_message(msg);
    return FATHOM_ERR_WORKSPACE_TOO_SMALL;
  }
  void *scratch = nullptr;
  const fathom_status st = scratch_on_current_device(&scratch);
  if (st != FATHOM_OK) return st;
  return fathom_scan_topk(args, scratch, FATHOM_NOALLOC_SCRATCH_BYTES, stream);
}
