// Internal definitions shared by the Fathom sm_100a kernels and their host
// launchers.  Not part of the ABI (include/fathom.h is).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "fathom.h"

namespace fathom {

// ---------------------------------------------------------------- geometry --
// A scan tile is 2048 tokens of one (session, KV head): 64 plane words per
// plane row.  A 128-thread block gives every word two threads, 16 tokens each
// (warps 2w and 2w+1 share the words 32w .. 32w+31).
constexpr int kTileWords = 64;
constexpr int kTileTokens = kTileWords * 32;
constexpr int kScanThreads = 128;
// Plane rows staged in shared memory per pipeline stage, and the stage width
// used to cut a KV head's union prefixes into stages (an entry of at most 4
// planes that ends inside a 29-plane window starts at most 3 planes before
// it, so a stage never holds more than 32 rows).
constexpr int kStageRows = 32;
constexpr int kStageSpan = 29;
constexpr int kStageBytes = kStageRows * kTileWords * 4;  // 8 KiB
constexpr int kNumBuf = 3;                                  // stage buffers in flight
constexpr int kNumPlanSlots = 4;                            // resident KV-head plans
// Threshold sampling: one 256-token sector (8 words) in every 64.
constexpr int kSectorWords = 8;
constexpr int kSampleStride = 64;
constexpr int kSampleSectorsPerTile = kTileWords / kSectorWords;  // 8
constexpr int kMergeThreads = 1024;
constexpr int kFallbackSlack = 2048;

enum ScanMode { kModeSample = 0, kModeFilter = 1 };

// Device status block at the start of every scan workspace.
struct WsStatus {
  uint32_t fallback_heads;
  uint32_t device_faults;
  uint32_t max_candidates;
  uint32_t union_planes;
  uint32_t pad[60];
};
static_assert(sizeof(WsStatus) == 256, "status block is 256 bytes");

// ------------------------------------------------------------------- plans --
// A plan is everything a scan block needs for one (session, KV head): the
// union plane prefixes, the per-channel features of its G query heads, their
// weights and constants, and how the prefixes are cut into staged copies.
//   entry  = one channel with union prefix t* > 0, in channel order;
//   info   = c | t* << 8 | slot0 << 11 | nfeat << 16 (slot0: first staged row);
//   feat   = up to 4 bytes, each (tf | mask << 3): the query heads in `mask`
//            read the first tf planes of this channel;
//   W      = per query head 32 q_c s_c (0 where that head reads nothing).
struct PlanHeader {
  int nent;
  int nstage;
  int union_planes;
  int pad0;
  float K[4];    // per query head constant: C_h - sum of W/2 over the channels it reads
  float tau[4];  // per query head candidate threshold (filled when a scan block loads it)
  int pad1[4];
};
static_assert(sizeof(PlanHeader) == 64, "plan header is 64 bytes");

struct PlanLayout {
  int maxst;
  int off_stage_begin;  // uint16 [maxst + 1]
  int off_stage_nrows;  // uint8  [maxst]
  int off_stage_rows;   // uint16 [maxst][32]: c * 4 + j of each staged row
  int off_info;         // uint32 [d]
  int off_feat;         // uint32 [d]
  int off_w;            // float4 [d]
  int bytes;
};

__host__ __device__ inline int align16(int x) { return (x + 15) & ~15; }

__host__ __device__ inline PlanLayout plan_layout(int d) {
  PlanLayout L;
  L.maxst = (4 * d + kStageSpan - 1) / kStageSpan + 1;
  int o = (int)sizeof(PlanHeader);
  L.off_stage_begin = o;
  o = align16(o + 2 * (L.maxst + 1));
  L.off_stage_nrows = o;
  o = align16(o + L.maxst);
  L.off_stage_rows = o;
  o = align16(o + 2 * kStageRows * L.maxst);
  L.off_info = o;
  o = align16(o + 4 * d);
  L.off_feat = o;
  o = align16(o + 4 * d);
  L.off_w = o;
  o = align16(o + 16 * d);
  L.bytes = o;
  return L;
}

// --------------------------------------------------------------- sessions --
// Per-launch parameters.  A single-session call carries its descriptor by
// value; a batched call points at the caller's device array.
struct ScanParams {
  const fathom_session *sessions;
  fathom_session one;
  int batched;
  int S;
  int d, h_q, h_kv, G, k;
  int q_bf16;
  int planes_host;  // planes in pinned, mapped host memory
  uint32_t flags;
  int sample_rank;  // r: threshold = r-th largest sampled score
  int64_t cap;      // candidate capacity per query head
  int64_t m_max;    // sample slots per query head
  int64_t n_max;    // the workspace's bound on every session's n
  int64_t token_group;  // keys per quantiser group (0: per channel over the context)
  int n_tgroups;        // plans per (session, KV head): ceil(n / token_group), or 1
  // workspace
  uint32_t *zero;    // prefix of the workspace the plan kernel clears (status, counts, tau)
  int zero_words;
  int plan_stride;   // bytes between consecutive plans
  WsStatus *status;
  uint32_t *counts;  // [S * h_q] candidate counts
  uint32_t *tau;     // [S * h_q] threshold keys (0 = keep every key)
  unsigned char *plans;  // [S * h_kv * n_tgroups] plans
  uint32_t *sample;      // [S * h_q][m_max] sampled keys
  unsigned long long *cand;  // [S * h_q][cap] composite (key << 32 | ~index)
  float *debug_scores;       // single session only
  cudaEvent_t prof_begin;    // optional events around the filtering scan
  cudaEvent_t prof_end;
};

// Device bounds checks of the checked build (compiled with
// -DFATHOM_DEVICE_CHECKS into libfathom_checked.so).  In_bounds(ok, st) is
// true in the normal build, where the index arithmetic is trusted; in the
// checked build an index that fails its bound is counted in the workspace
// status (device_faults, read by fathom_scan_read_report) and the caller
// skips the access.
#ifdef FATHOM_DEVICE_CHECKS
__device__ __forceinline__ bool in_bounds(bool ok, WsStatus *st) {
  if (!ok) atomicAdd(&st->device_faults, 1u);
  return ok;
}
#else
__device__ __forceinline__ bool in_bounds(bool, WsStatus *) { return true; }
#endif

__device__ __forceinline__ const fathom_session &session_of(const ScanParams &p, int s) {
  return p.batched ? p.sessions[s] : p.one;
}

// Keys of session s as the kernels use them.  A batched descriptor is read
// from device memory that the host never checked: an n outside [0, n_max]
// (the bound the workspace was sized for) makes the session empty, so that no
// kernel reads or writes past its buffers; the plan kernel records it as a
// device fault.
__device__ __forceinline__ bool session_n_valid(const ScanParams &p, int64_t n) {
  return n >= 0 && n <= p.n_max;
}
__device__ __forceinline__ int64_t session_n(const ScanParams &p, int s) {
  const int64_t n = session_of(p, s).n;
  return session_n_valid(p, n) ? n : 0;
}

__host__ __device__ inline int64_t plane_words(int64_t n) { return ((n + 127) / 128) * 4; }
__host__ __device__ inline int64_t filter_tiles(int64_t n) {
  return (plane_words(n) + kTileWords - 1) / kTileWords;
}
__host__ __device__ inline int64_t sectors(int64_t n) {
  return (plane_words(n) + kSectorWords - 1) / kSectorWords;
}
__host__ __device__ inline int64_t sampled_sectors(int64_t n) {
  return (sectors(n) + kSampleStride - 1) / kSampleStride;
}
__host__ __device__ inline int sample_rank_for(int k) {
  int r = (k + 31) / 32;
  return r < 16 ? 16 : r;
}
// A session is sampled when its sample holds at least 8 r keys.
__host__ __device__ inline bool sampling_on(int64_t n, int r, uint32_t flags) {
  return !(flags & FATHOM_FLAG_NO_SAMPLING) && n >= (int64_t)512 * r;
}
__host__ __device__ inline int64_t sample_tiles(int64_t n, int r, uint32_t flags) {
  if (!sampling_on(n, r, flags)) return 0;
  return (sampled_sectors(n) + kSampleSectorsPerTile - 1) / kSampleSectorsPerTile;
}

// ------------------------------------------------------------------ keys ---
// Order-preserving map of a float to uint32 (larger float, larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}
// Composite ordering of (score desc, index asc) as one descending uint64.
__device__ __forceinline__ unsigned long long composite(float s, uint32_t idx) {
  return ((unsigned long long)float_key(s) << 32) | (unsigned long long)(0xffffffffu - idx);
}

__device__ __forceinline__ float load_q(const void *q, int q_bf16, int64_t i) {
  if (q_bf16) {
    uint16_t b = reinterpret_cast<const uint16_t *>(q)[i];
    return __uint_as_float((uint32_t)b << 16);
  }
  return reinterpret_cast<const float *>(q)[i];
}

// ------------------------------------------------------- dependent launch --
// The step's kernels run back to back on one stream.  Each is launched with
// programmatic stream serialisation: it may be scheduled while its
// predecessor finishes, and waits (grid_dependency_wait) before it touches
// anything the predecessor wrote.  Each lets its successor launch early
// (allow_dependent_launch) as soon as it starts.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

template <typename... Params, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace fathom
