// fathom_scan_topk_noalloc: the scan for callers that cannot allocate device
// memory (see include/fathom.h).  The scan's workspace is a fixed array in
// the library's own device memory instead of a caller buffer; the kernels
// and launch sequence are those of fathom_scan_topk.
#include <cuda.h>
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

// The scratch's device address, per device, with the id of the context it
// was looked up in.  A device reset (cudaDeviceReset) destroys that context
// and the module holding the array; the next call finds a new context id and
// looks the address up again instead of handing the kernels a stale one.
struct ScratchAddr {
  void *ptr;
  unsigned long long ctx_id;
};
std::mutex g_scratch_mu;
ScratchAddr g_scratch[kMaxDevices] = {};

typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

fathom_status fail_cuda(const char *what, cudaError_t e) {
  char msg[256];
  snprintf(msg, sizeof(msg), "%s: %s", what, cudaGetErrorString(e));
  fathom::set_error_message(msg);
  return FATHOM_ERR_CUDA;
}

// Id of the current context (unique for the life of the process), through
// the driver entry point the runtime hands out (no link against libcuda).
fathom_status current_context_id(unsigned long long *id) {
  static CtxGetIdFn fn = nullptr;
  if (fn == nullptr) {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    const cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || f == nullptr)
      return fail_cuda("driver entry point cuCtxGetId", e != cudaSuccess ? e : cudaErrorNotSupported);
    fn = reinterpret_cast<CtxGetIdFn>(f);
  }
  if (fn(nullptr, id) != CUDA_SUCCESS) {
    fathom::set_error_message("no current CUDA context for the no-alloc scratch");
    return FATHOM_ERR_CUDA;
  }
  return FATHOM_OK;
}

// Device address of the scratch array on the current device.  Set-up, once
// per device (and again after a reset of it): with that device current,
// cudaGetSymbolAddress, whose return code is checked.  In host code the
// array's name only stands for the symbol; the kernels must be given this
// address.
fathom_status scratch_on_current_device(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda("no current device", e);
  if (dev < 0 || dev >= kMaxDevices) {
    fathom::set_error_message("device index beyond the no-alloc scratch table");
    return FATHOM_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  unsigned long long ctx = 0;
  // the first call on a device may find no context yet: the symbol lookup
  // below creates the device's primary context, and the id is read after it
  const bool have_ctx = current_context_id(&ctx) == FATHOM_OK;
  if (!have_ctx || g_scratch[dev].ptr == nullptr || g_scratch[dev].ctx_id != ctx) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fathom_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail_cuda("cudaGetSymbolAddress of the scratch", e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    fathom_status st = current_context_id(&ctx);
    if (st != FATHOM_OK) return st;
    g_scratch[dev].ptr = p;
    g_scratch[dev].ctx_id = ctx;
  }
  *out = g_scratch[dev].ptr;
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

extern "C" fathom_status fathom_scan_read_report_noalloc(fathom_scan_report *report,
                                                         void *stream) {
  if (report == nullptr) {
    fathom::set_error_message("report is NULL");
    return FATHOM_ERR_INVALID_ARGUMENT;
  }
  void *scratch = nullptr;
  const fathom_status st = scratch_on_current_device(&scratch);
  if (st != FATHOM_OK) return st;
  return fathom_scan_read_report(scratch, report, stream);
}
