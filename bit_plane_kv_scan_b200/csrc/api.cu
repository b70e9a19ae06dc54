// Host side of the C ABI declared in include/fathom.h: argument checks,
// workspace layout and the launch sequence.  Every check runs before any
// launch; a failed check launches nothing and returns a status.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <cmath>

#include <nvtx3/nvToolsExt.h>

#include "fathom_internal.cuh"

namespace fathom {
cudaError_t launch_pack(const uint8_t *codes, int64_t n, int d, int h_kv, uint32_t *planes,
                        cudaStream_t stream);
cudaError_t launch_allocate_uniform(int h_q, int d, int budget, uint8_t *alloc,
                                    cudaStream_t stream);
cudaError_t launch_append(const uint8_t *codes, int64_t n, int64_t m, int d, int h_kv,
                          const uint32_t *planes_in, uint32_t *planes_out, cudaStream_t stream);
cudaError_t launch_attention(const void *q, int q_bf16, const uint16_t *k_rows,
                             const uint8_t *k_codes, const float *k_qmin, const float *k_qscale,
                             const uint16_t *v_rows, const int32_t *idx, int64_t n, int d,
                             int h_q, int h_kv, int k, float scale, float *out, float *lse,
                             cudaStream_t stream);
cudaError_t launch_allocate(const void *q, int q_bf16, const float *sigma, int h_q, int h_kv, int d,
                            int budget, uint8_t *alloc, cudaStream_t stream);
cudaError_t launch_scan_pipeline(const ScanParams &p, bool any_sampling, cudaStream_t stream);
cudaError_t launch_merge_parts(const int32_t *in_idx, const float *in_score, int parts,
                               const int64_t *offsets, int h_q, int k_in, int k, int32_t *out_idx,
                               float *out_score, cudaStream_t stream);
int tc_plan_bytes(int d);
}  // namespace fathom

using namespace fathom;

namespace {

thread_local char g_err[512] = "";
thread_local cudaEvent_t g_prof_begin = nullptr;
thread_local cudaEvent_t g_prof_end = nullptr;

fathom_status fail(fathom_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

fathom_status cuda_fail(cudaError_t e, const char *what) {
  return fail(FATHOM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

fathom_status ok() {
  g_err[0] = 0;
  return FATHOM_OK;
}

// Pointer kinds.  A device pointer is device or managed memory; a host-mapped
// pointer is pinned host memory the device can address.
enum PtrKind { kPtrDevice, kPtrHostMapped, kPtrOther };

PtrKind ptr_kind(const void *p) {
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return kPtrOther;
  }
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return kPtrDevice;
  if (a.type == cudaMemoryTypeHost && a.devicePointer == p) return kPtrHostMapped;
  return kPtrOther;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

#define REQUIRE(cond, ...)                                            \
  do {                                                                \
    if (!(cond)) return fail(FATHOM_ERR_INVALID_ARGUMENT, __VA_ARGS__); \
  } while (0)
#define REQUIRE_DEV(ptr, name)                                                           \
  do {                                                                                   \
    if ((ptr) == nullptr) return fail(FATHOM_ERR_INVALID_ARGUMENT, "%s is NULL", name);   \
    if (ptr_kind(ptr) != kPtrDevice)                                                     \
      return fail(FATHOM_ERR_INVALID_ARGUMENT, "%s is not a device pointer", name);      \
  } while (0)

fathom_status check_shape(int d, int h_q, int h_kv) {
  if (d < 32 || d > FATHOM_MAX_D || d % 32 != 0)
    return fail(FATHOM_ERR_UNSUPPORTED, "d=%d: need a multiple of 32 in [32, %d]", d, FATHOM_MAX_D);
  if (h_kv < 1 || h_q < 1) return fail(FATHOM_ERR_INVALID_ARGUMENT, "h_q=%d h_kv=%d: need >= 1", h_q, h_kv);
  if (h_q % h_kv != 0)
    return fail(FATHOM_ERR_INVALID_ARGUMENT, "h_q=%d is not a multiple of h_kv=%d", h_q, h_kv);
  return FATHOM_OK;
}

// Workspace layout of one scan launch set.
struct WsLayout {
  size_t off_counts, off_tau, off_plans, off_sample, off_cand, total;
  size_t zero_bytes;  // prefix cleared before every scan
  int64_t cap, m_max;
  int sample_rank;
};

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

WsLayout ws_layout(int S, int64_t n_max, int d, int h_q, int h_kv, int k, uint32_t flags,
                   int n_tgroups = 1) {
  WsLayout L;
  const int64_t heads = (int64_t)S * h_q;
  const int64_t groups = (int64_t)S * h_kv * n_tgroups;  // one plan each
  L.sample_rank = sample_rank_for(k);
  int64_t cap = 8 * (int64_t)k;
  if (cap < 512 * (int64_t)L.sample_rank) cap = 512 * (int64_t)L.sample_rank;
  if (flags & FATHOM_FLAG_NO_SAMPLING) cap = cap > n_max ? cap : n_max;
  L.cap = cap + kFallbackSlack;
  L.m_max = sampling_on(n_max, L.sample_rank, flags) ? sampled_sectors(n_max) * 256 : 0;
  size_t o = sizeof(WsStatus);
  L.off_counts = o;
  o = up256(o + 4 * heads);
  L.off_tau = o;
  o = up256(o + 4 * heads);
  L.zero_bytes = o;
  L.off_plans = o;
  const size_t plan_bytes = (size_t)(tc_plan_bytes(d) > plan_layout(d).bytes ? tc_plan_bytes(d)
                                                                              : plan_layout(d).bytes);
  o = up256(o + (size_t)groups * plan_bytes);
  L.off_sample = o;
  o = up256(o + (size_t)heads * L.m_max * 4);
  L.off_cand = o;
  o = up256(o + (size_t)heads * L.cap * 8);
  L.total = o;
  return L;
}

void fill_ws(ScanParams &p, const WsLayout &L, void *ws) {
  unsigned char *b = static_cast<unsigned char *>(ws);
  p.zero = reinterpret_cast<uint32_t *>(b);
  p.zero_words = (int)(L.zero_bytes / 4);
  p.plan_stride = (p.flags & FATHOM_FLAG_CUDA_CORES) ? plan_layout(p.d).bytes : tc_plan_bytes(p.d);
  p.status = reinterpret_cast<WsStatus *>(b);
  p.counts = reinterpret_cast<uint32_t *>(b + L.off_counts);
  p.tau = reinterpret_cast<uint32_t *>(b + L.off_tau);
  p.plans = b + L.off_plans;
  p.sample = reinterpret_cast<uint32_t *>(b + L.off_sample);
  p.cand = reinterpret_cast<unsigned long long *>(b + L.off_cand);
  p.cap = L.cap;
  p.m_max = L.m_max;
  p.sample_rank = L.sample_rank;
}

fathom_status check_scan_common(int64_t n, int d, int h_q, int h_kv, int k, int q_dtype,
                                int planes_location) {
  fathom_status st = check_shape(d, h_q, h_kv);
  if (st != FATHOM_OK) return st;
  const int G = h_q / h_kv;
  if (G != 1 && G != 2 && G != 4)
    return fail(FATHOM_ERR_UNSUPPORTED, "query heads per KV head G=%d: need 1, 2 or 4", G);
  REQUIRE(n >= 0 && n < ((int64_t)1 << 31), "n=%lld out of range [0, 2^31)", (long long)n);
  REQUIRE(k >= 1 && k <= FATHOM_MAX_K, "k=%d out of range [1, %d]", k, FATHOM_MAX_K);
  REQUIRE(q_dtype == FATHOM_F32 || q_dtype == FATHOM_BF16, "q_dtype=%d unknown", q_dtype);
  REQUIRE(planes_location == FATHOM_PLANES_DEVICE || planes_location == FATHOM_PLANES_HOST_MAPPED,
          "planes_location=%d unknown", planes_location);
  return FATHOM_OK;
}

}  // namespace

namespace fathom {
// Lets other translation units of the library report an error message.
void set_error_message(const char *msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }
}  // namespace fathom

// An NVTX range over one ABI call, so that a trace (nsys, ncu's NVTX
// filters) shows each call's launches under its name.  Without a tool
// attached the push and pop do nothing.
struct CallRange {
  explicit CallRange(const char *name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
};

extern "C" {

const char *fathom_last_error(void) { return g_err; }

void fathom_profile_scan_kernel(void *begin, void *end) {
  g_prof_begin = (cudaEvent_t)begin;
  g_prof_end = (cudaEvent_t)end;
}

int64_t fathom_plane_words(int64_t n) { return n < 0 ? 0 : plane_words(n); }

size_t fathom_planes_bytes(int64_t n, int d, int h_kv) {
  if (n < 0 || d < 0 || h_kv < 0) return 0;
  return (size_t)h_kv * d * 4 * plane_words(n) * 4;
}

fathom_status fathom_pack_planes(const uint8_t *codes, int64_t n, int d, int h_kv, uint32_t *planes,
                                 void *stream) {
  const CallRange range("fathom_pack_planes");
  fathom_status st = check_shape(d, h_kv, h_kv);
  if (st != FATHOM_OK) return st;
  REQUIRE(n >= 0 && n < ((int64_t)1 << 31), "n=%lld out of range [0, 2^31)", (long long)n);
  if (n == 0) return ok();
  REQUIRE_DEV(codes, "codes");
  REQUIRE_DEV(planes, "planes");
  REQUIRE(aligned(codes, 16) && aligned(planes, 16), "codes and planes must be 16-byte aligned");
  cudaError_t e = launch_pack(codes, n, d, h_kv, planes, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  return ok();
}

fathom_status fathom_append_planes(const uint8_t *codes, int64_t n, int64_t m, int d, int h_kv,
                                   const uint32_t *planes_in, uint32_t *planes_out, void *stream) {
  const CallRange range("fathom_append_planes");
  fathom_status st = check_shape(d, h_kv, h_kv);
  if (st != FATHOM_OK) return st;
  REQUIRE(n >= 0 && m >= 0 && n + m < ((int64_t)1 << 31), "n=%lld m=%lld out of range",
          (long long)n, (long long)m);
  if (n + m == 0) return ok();  // nothing stored, nothing to add
  REQUIRE_DEV(planes_out, "planes_out");
  if (m > 0) REQUIRE_DEV(codes, "codes");
  const bool same = planes_in == planes_out;
  if (!same && plane_words(n) > 0) REQUIRE_DEV(planes_in, "planes_in");
  REQUIRE(!same || plane_words(n) == plane_words(n + m),
          "in place needs fathom_plane_words(n + m) == fathom_plane_words(n) (%lld != %lld)",
          (long long)plane_words(n + m), (long long)plane_words(n));
  if (!same) {
    const int64_t bytes_in = (int64_t)h_kv * d * 4 * plane_words(n) * 4;
    const int64_t bytes_out = (int64_t)h_kv * d * 4 * plane_words(n + m) * 4;
    const uintptr_t a = (uintptr_t)planes_in, b = (uintptr_t)planes_out;
    REQUIRE(a + (uintptr_t)bytes_in <= b || b + (uintptr_t)bytes_out <= a,
            "planes_in and planes_out overlap");
  }
  cudaError_t e = launch_append(codes, n, m, d, h_kv, planes_in, planes_out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  return ok();
}

fathom_status fathom_allocate(const void *q, fathom_dtype q_dtype, const float *sigma, int h_q,
                              int h_kv, int d, int budget_bits, uint8_t *alloc, void *stream) {
  const CallRange range("fathom_allocate");
  fathom_status st = check_shape(d, h_q, h_kv);
  if (st != FATHOM_OK) return st;
  REQUIRE(q_dtype == FATHOM_F32 || q_dtype == FATHOM_BF16, "q_dtype=%d unknown", (int)q_dtype);
  REQUIRE(budget_bits >= 0 && budget_bits <= 4 * d, "budget_bits=%d out of range [0, 4d=%d]",
          budget_bits, 4 * d);
  REQUIRE_DEV(q, "q");
  REQUIRE_DEV(sigma, "sigma");
  REQUIRE_DEV(alloc, "alloc");
  cudaError_t e = launch_allocate(q, q_dtype == FATHOM_BF16, sigma, h_q, h_kv, d, budget_bits,
                                  alloc, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "allocate launch");
  return ok();
}

fathom_status fathom_allocate_uniform(int h_q, int d, int budget_bits, uint8_t *alloc,
                                      void *stream) {
  const CallRange range("fathom_allocate_uniform");
  fathom_status st = check_shape(d, h_q, 1);
  if (st != FATHOM_OK) return st;
  REQUIRE((int64_t)h_q * d < ((int64_t)1 << 30), "h_q=%d too large", h_q);
  REQUIRE(budget_bits >= 0 && budget_bits <= 4 * d, "budget_bits=%d out of range [0, 4d=%d]",
          budget_bits, 4 * d);
  REQUIRE_DEV(alloc, "alloc");
  cudaError_t e = launch_allocate_uniform(h_q, d, budget_bits, alloc, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "allocate_uniform launch");
  return ok();
}

fathom_status fathom_sparse_attention(const fathom_attention_args *a, void *stream) {
  const CallRange range("fathom_sparse_attention");
  REQUIRE(a != nullptr, "args is NULL");
  fathom_status st = check_shape(a->d, a->h_q, a->h_kv);
  if (st != FATHOM_OK) return st;
  REQUIRE(a->q_dtype == FATHOM_F32 || a->q_dtype == FATHOM_BF16, "q_dtype=%d unknown",
          (int)a->q_dtype);
  REQUIRE(a->n >= 0 && a->n < ((int64_t)1 << 31), "n=%lld out of range [0, 2^31)",
          (long long)a->n);
  REQUIRE(a->k >= 0, "k=%d is negative", a->k);
  REQUIRE(std::isfinite(a->softmax_scale), "softmax_scale is not finite");
  REQUIRE(a->kv_location == FATHOM_PLANES_DEVICE || a->kv_location == FATHOM_PLANES_HOST_MAPPED,
          "kv_location=%d unknown", a->kv_location);
  REQUIRE_DEV(a->q, "q");
  if (a->k > 0) REQUIRE_DEV(a->idx, "idx");
  REQUIRE_DEV(a->out, "out");
  if (a->lse) REQUIRE_DEV(a->lse, "lse");
  if (a->n > 0 && a->k > 0) {
    const PtrKind want = a->kv_location == FATHOM_PLANES_DEVICE ? kPtrDevice : kPtrHostMapped;
    const char *where = a->kv_location == FATHOM_PLANES_DEVICE
                            ? "not a device pointer (kv_location=DEVICE)"
                            : "not pinned, mapped host memory (kv_location=HOST_MAPPED)";
    auto check_kv = [&](const void *ptr, const char *name) -> fathom_status {
      if (ptr == nullptr) return fail(FATHOM_ERR_INVALID_ARGUMENT, "%s is NULL", name);
      if (ptr_kind(ptr) != want) return fail(FATHOM_ERR_INVALID_ARGUMENT, "%s is %s", name, where);
      return FATHOM_OK;
    };
    fathom_status st2 = a->k_codes ? check_kv(a->k_codes, "k_codes") : check_kv(a->k_rows, "k_rows");
    if (st2 != FATHOM_OK) return st2;
    st2 = check_kv(a->v_rows, "v_rows");
    if (st2 != FATHOM_OK) return st2;
    if (a->k_codes) {
      REQUIRE_DEV(a->k_qmin, "k_qmin");
      REQUIRE_DEV(a->k_qscale, "k_qscale");
      REQUIRE(aligned(a->k_codes, 16), "k_codes not 16-byte aligned");
    } else {
      REQUIRE(aligned(a->k_rows, 16), "k_rows not 16-byte aligned");
    }
    REQUIRE(aligned(a->v_rows, 16), "v_rows not 16-byte aligned");
  }
  cudaError_t e = launch_attention(a->q, a->q_dtype == FATHOM_BF16, a->k_rows, a->k_codes,
                                   a->k_qmin, a->k_qscale, a->v_rows, a->idx, a->n, a->d, a->h_q,
                                   a->h_kv, a->k, a->softmax_scale, a->out, a->lse,
                                   (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return ok();
}

// Plans per KV head of a single-session call: one per token group.
static int tgroups_of(const fathom_scan_args *a) {
  if (a->token_group <= 0 || a->n <= 0) return 1;
  return (int)((a->n + a->token_group - 1) / a->token_group);
}

static fathom_status check_token_group(const fathom_scan_args *a) {
  REQUIRE(a->token_group >= 0 && a->token_group % FATHOM_TOKEN_GROUP_QUANTUM == 0,
          "token_group=%lld: need 0 or a positive multiple of %d", (long long)a->token_group,
          FATHOM_TOKEN_GROUP_QUANTUM);
  if (a->token_group > 0 && (a->flags & FATHOM_FLAG_CUDA_CORES))
    return fail(FATHOM_ERR_UNSUPPORTED,
                "per-token-group statistics are supported by the tensor-core scan only");
  return FATHOM_OK;
}

static fathom_status check_scan_args(const fathom_scan_args *a) {
  REQUIRE(a != nullptr, "args is NULL");
  fathom_status st = check_scan_common(a->n, a->d, a->h_q, a->h_kv, a->k, a->q_dtype,
                                       a->planes_location);
  if (st != FATHOM_OK) return st;
  st = check_token_group(a);
  if (st != FATHOM_OK) return st;
  REQUIRE_DEV(a->qmin, "qmin");
  REQUIRE_DEV(a->qscale, "qscale");
  REQUIRE_DEV(a->q, "q");
  REQUIRE_DEV(a->alloc, "alloc");
  REQUIRE_DEV(a->out_idx, "out_idx");
  REQUIRE_DEV(a->out_score, "out_score");
  if (a->debug_scores) REQUIRE_DEV(a->debug_scores, "debug_scores");
  if (a->n > 0) {
    REQUIRE(a->planes != nullptr, "planes is NULL");
    const PtrKind kind = ptr_kind(a->planes);
    if (a->planes_location == FATHOM_PLANES_DEVICE)
      REQUIRE(kind == kPtrDevice, "planes is not a device pointer (planes_location=DEVICE)");
    else
      REQUIRE(kind == kPtrHostMapped,
              "planes is not pinned, mapped host memory (planes_location=HOST_MAPPED)");
    REQUIRE(aligned(a->planes, 16), "planes must be 16-byte aligned");
  }
  return FATHOM_OK;
}

size_t fathom_scan_topk_workspace_size(const fathom_scan_args *a) {
  if (a == nullptr || check_scan_common(a->n, a->d, a->h_q, a->h_kv, a->k, a->q_dtype,
                                        a->planes_location) != FATHOM_OK ||
      check_token_group(a) != FATHOM_OK)
    return 0;
  return ws_layout(1, a->n, a->d, a->h_q, a->h_kv, a->k, a->flags, tgroups_of(a)).total;
}

fathom_status fathom_scan_topk(const fathom_scan_args *a, void *ws, size_t ws_bytes, void *stream) {
  const CallRange range("fathom_scan_topk");
  fathom_status st = check_scan_args(a);
  if (st != FATHOM_OK) return st;
  const WsLayout L = ws_layout(1, a->n, a->d, a->h_q, a->h_kv, a->k, a->flags, tgroups_of(a));
  REQUIRE_DEV(ws, "workspace");
  REQUIRE(aligned(ws, 256), "workspace must be 256-byte aligned");
  if (ws_bytes < L.total)
    return fail(FATHOM_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu needed", ws_bytes,
                L.total);
  ScanParams p;
  memset(&p, 0, sizeof(p));
  p.sessions = nullptr;
  p.one.planes = a->planes;
  p.one.qmin = a->qmin;
  p.one.qscale = a->qscale;
  p.one.q = a->q;
  p.one.alloc = a->alloc;
  p.one.n = a->n;
  p.n_max = a->n;
  p.token_group = a->token_group;
  p.n_tgroups = tgroups_of(a);
  p.one.out_idx = a->out_idx;
  p.one.out_score = a->out_score;
  p.batched = 0;
  p.S = 1;
  p.d = a->d;
  p.h_q = a->h_q;
  p.h_kv = a->h_kv;
  p.G = a->h_q / a->h_kv;
  p.k = a->k;
  p.q_bf16 = a->q_dtype == FATHOM_BF16;
  p.planes_host = a->planes_location == FATHOM_PLANES_HOST_MAPPED;
  p.flags = a->flags;
  p.debug_scores = a->debug_scores;
  fill_ws(p, L, ws);
  p.prof_begin = g_prof_begin;
  p.prof_end = g_prof_end;
  cudaStream_t s = (cudaStream_t)stream;
  // the plan kernel clears the workspace's status, counters and thresholds
  cudaError_t e = launch_scan_pipeline(p, sampling_on(a->n, L.sample_rank, a->flags), s);
  if (e != cudaSuccess) return cuda_fail(e, "scan launch");
  return ok();
}

static fathom_status check_batched_args(const fathom_batched_args *a) {
  REQUIRE(a != nullptr, "args is NULL");
  REQUIRE(a->num_sessions >= 1 && a->num_sessions <= 1024, "num_sessions=%d out of range [1, 1024]",
          a->num_sessions);
  fathom_status st = check_scan_common(a->n_max, a->d, a->h_q, a->h_kv, a->k, a->q_dtype,
                                       a->planes_location);
  if (st != FATHOM_OK) return st;
  REQUIRE_DEV(a->sessions, "sessions");
  return FATHOM_OK;
}

size_t fathom_scan_topk_batched_workspace_size(const fathom_batched_args *a) {
  if (a == nullptr || a->num_sessions < 1 || a->num_sessions > 1024 ||
      check_scan_common(a->n_max, a->d, a->h_q, a->h_kv, a->k, a->q_dtype, a->planes_location) !=
          FATHOM_OK)
    return 0;
  return ws_layout(a->num_sessions, a->n_max, a->d, a->h_q, a->h_kv, a->k, a->flags).total;
}

fathom_status fathom_scan_topk_batched(const fathom_batched_args *a, void *ws, size_t ws_bytes,
                                       void *stream) {
  const CallRange range("fathom_scan_topk_batched");
  fathom_status st = check_batched_args(a);
  if (st != FATHOM_OK) return st;
  const WsLayout L = ws_layout(a->num_sessions, a->n_max, a->d, a->h_q, a->h_kv, a->k, a->flags);
  REQUIRE_DEV(ws, "workspace");
  REQUIRE(aligned(ws, 256), "workspace must be 256-byte aligned");
  if (ws_bytes < L.total)
    return fail(FATHOM_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu needed", ws_bytes,
                L.total);
  ScanParams p;
  memset(&p, 0, sizeof(p));
  p.sessions = a->sessions;
  p.n_max = a->n_max;
  p.token_group = 0;
  p.n_tgroups = 1;
  p.batched = 1;
  p.S = a->num_sessions;
  p.d = a->d;
  p.h_q = a->h_q;
  p.h_kv = a->h_kv;
  p.G = a->h_q / a->h_kv;
  p.k = a->k;
  p.q_bf16 = a->q_dtype == FATHOM_BF16;
  p.planes_host = a->planes_location == FATHOM_PLANES_HOST_MAPPED;
  p.flags = a->flags;
  p.debug_scores = nullptr;
  fill_ws(p, L, ws);
  p.prof_begin = g_prof_begin;
  p.prof_end = g_prof_end;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = launch_scan_pipeline(p, L.m_max > 0, s);
  if (e != cudaSuccess) return cuda_fail(e, "scan launch");
  return ok();
}

fathom_status fathom_merge_topk(const int32_t *in_idx, const float *in_score, int parts,
                                const int64_t *offsets, int h_q, int k_in, int k, int32_t *out_idx,
                                float *out_score, void *stream) {
  const CallRange range("fathom_merge_topk");
  REQUIRE(parts >= 1 && parts <= FATHOM_MAX_MERGE_PARTS, "parts=%d out of range [1, %d]", parts,
          FATHOM_MAX_MERGE_PARTS);
  REQUIRE(h_q >= 1, "h_q=%d: need >= 1", h_q);
  REQUIRE(k_in >= 1 && k_in <= FATHOM_MAX_K, "k_in=%d out of range [1, %d]", k_in, FATHOM_MAX_K);
  REQUIRE(k >= 1 && k <= FATHOM_MAX_K, "k=%d out of range [1, %d]", k, FATHOM_MAX_K);
  REQUIRE(offsets != nullptr, "offsets is NULL");
  for (int b = 0; b < parts; ++b)
    REQUIRE(offsets[b] >= 0 && offsets[b] < ((int64_t)1 << 31), "offsets[%d]=%lld out of range",
            b, (long long)offsets[b]);
  REQUIRE_DEV(in_idx, "in_idx");
  REQUIRE_DEV(in_score, "in_score");
  REQUIRE_DEV(out_idx, "out_idx");
  REQUIRE_DEV(out_score, "out_score");
  cudaError_t e = launch_merge_parts(in_idx, in_score, parts, offsets, h_q, k_in, k, out_idx,
                                     out_score, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return ok();
}

fathom_status fathom_scan_read_report(const void *ws, fathom_scan_report *report, void *stream) {
  REQUIRE(report != nullptr, "report is NULL");
  REQUIRE_DEV(ws, "workspace");
  WsStatus hs;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(&hs, ws, sizeof(hs), cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "report copy");
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "report sync");
  report->fallback_heads = hs.fallback_heads;
  report->device_faults = hs.device_faults;
  report->max_candidates = hs.max_candidates;
  report->union_planes = hs.union_planes;
  if (hs.device_faults) return fail(FATHOM_ERR_DEVICE_CHECK, "device checks recorded %u faults",
                                    hs.device_faults);
  return ok();
}

fathom_status fathom_check_device_status(const void *ws, void *stream) {
  fathom_scan_report r;
  return fathom_scan_read_report(ws, &r, stream);
}

}  // extern "C"
