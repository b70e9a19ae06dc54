/*
 * fathom.h -- C ABI of the B200 (sm_100a) Fathom query-adaptive key scan.
 *
 * Fathom ("Fathom: Per-Query Read Depth for Sparse Decoding over Offloaded
 * KV Caches", arXiv 2609.17652; summarised in "Fathom Makes KV-Cache Scans
 * Query-Adaptive for Long-Context Decoding", cctest.ai) ranks all n cached
 * keys for each decode step's top-k.  Its 4-bit K cache is stored as
 * channel-major bit planes, so a channel's first t planes are that
 * channel's t-bit quantiser; each query spends a budget of B bits per key
 * over its channels by reverse water-filling, and only the allocated plane
 * prefixes are read.
 *
 * The hot path is four steps in three calls:
 *   fathom_pack_planes   4-bit codes -> bit planes (once per cache, off the
 *                        per-step path);
 *   fathom_allocate      per query head, bits per channel (the allocation);
 *   fathom_scan_topk     scores of all n keys from the allocated prefixes and
 *                        the per-head top-k (one session);
 *   fathom_scan_topk_batched   the same for many sessions in one launch set.
 * Around it:
 *   fathom_append_planes       adds decoded tokens to a packed store;
 *   fathom_allocate_uniform    the same B bits per key for every query head,
 *                        spread evenly over the channels (the fixed-depth
 *                        read that the adaptive allocation is compared with);
 *   fathom_sparse_attention    after the scan: each query head's attention
 *                        over only its selected keys;
 *   fathom_merge_topk          token-range sharding: the top-k of the ranges'
 *                        top-k lists;
 *   fathom_scan_topk_noalloc   fathom_scan_topk on built-in scratch, for
 *                        callers that cannot allocate;
 *   fathom_scan_read_report, fathom_check_device_status    what the last
 *                        scan on a workspace recorded (faults, fallbacks).
 * fathom_scan_args.token_group selects the quantiser variant with (m, s) per
 * run of token_group keys instead of per channel over the whole context.
 *
 * Conventions shared by every call
 *   - The caller owns every buffer.  The library never allocates or frees;
 *     scans take a caller-sized workspace (see *_workspace_size).
 *   - Pointers are CUDA device pointers unless a parameter says otherwise.
 *     Plane stores may instead live in pinned, mapped host memory
 *     (FATHOM_PLANES_HOST_MAPPED): the scan then reads only the allocated
 *     prefixes across the host link.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     stream-ordered and asynchronous: none synchronises the host except
 *     the report and status reads.  Kernels are launched with programmatic
 *     stream serialisation: one may be scheduled while the stream's previous
 *     kernel finishes, but waits for that kernel to complete before it reads
 *     or writes anything; ordering with the caller's own work is unchanged.
 *   - Every call validates its arguments on the host before any launch and
 *     returns a status; on error nothing is launched and
 *     fathom_last_error() holds a message.  No C++ exception crosses the ABI.
 *   - Notation: KV heads g < h_kv, query heads h < h_q with G = h_q / h_kv
 *     query heads per KV head (head h reads KV head h / G), channels c < d,
 *     tokens i < n, plane j < 4 (j = 0 is the code's most significant bit).
 */
#ifndef FATHOM_H
#define FATHOM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FATHOM_API __attribute__((visibility("default")))
#else
#define FATHOM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fathom_status {
  FATHOM_OK = 0,
  FATHOM_ERR_INVALID_ARGUMENT = 1,     /* bad size, null or wrong-kind pointer */
  FATHOM_ERR_UNSUPPORTED = 2,          /* valid but outside this build's limits */
  FATHOM_ERR_WORKSPACE_TOO_SMALL = 3,  /* ws_bytes below *_workspace_size */
  FATHOM_ERR_CUDA = 4,                 /* a CUDA runtime call or launch failed */
  FATHOM_ERR_DEVICE_CHECK = 5          /* a device-side check recorded a fault */
} fathom_status;

typedef enum fathom_dtype { FATHOM_F32 = 0, FATHOM_BF16 = 1 } fathom_dtype;

typedef enum fathom_planes_location {
  FATHOM_PLANES_DEVICE = 0,      /* planes in device memory (HBM) */
  FATHOM_PLANES_HOST_MAPPED = 1  /* planes in pinned host memory mapped into the device */
} fathom_planes_location;

/* Limits of this build. */
#define FATHOM_MAX_D 256    /* d is a multiple of 32, 32 <= d <= 256 */
#define FATHOM_MAX_GROUP 4  /* G = h_q / h_kv is 1, 2 or 4 */
#define FATHOM_MAX_K 8192   /* 1 <= k <= 8192 */
#define FATHOM_MAX_MERGE_PARTS 64  /* partial lists one fathom_merge_topk call merges */

/* Test knobs for fathom_scan_args.flags (0 in normal use). */
#define FATHOM_FLAG_NO_SAMPLING 1u     /* skip the threshold sample: every key is a candidate */
#define FATHOM_FLAG_FORCE_FALLBACK 2u  /* take the exact single-block fallback for every head */
/* Run the scan on the CUDA-core kernel (fp32 FMAs on per-channel prefix codes)
 * instead of the default tcgen05 tensor-core kernel (int8 MMAs into tensor
 * memory).  Same results; kept as a second, independent implementation. */
#define FATHOM_FLAG_CUDA_CORES 4u

/* Last error message of the calling thread ("" if none). */
FATHOM_API const char *fathom_last_error(void);

/* ---------------------------------------------------------------------------
 * Bit-plane store layout (method paragraph 2: the K cache is kept as
 * channel-major bit planes; abstract: a channel's first t planes are
 * precisely its t-bit quantiser):
 *   planes[g][c][j][w], uint32, w < W = fathom_plane_words(n);
 *   bit b of word w of plane j holds bit (3 - j) of the code of token
 *   32 w + b; rows are padded to a multiple of 128 tokens (16 bytes) and
 *   every bit of a token >= n is 0.
 * The t planes of a channel's prefix are one contiguous run of t*W words.
 */
FATHOM_API int64_t fathom_plane_words(int64_t n);
FATHOM_API size_t fathom_planes_bytes(int64_t n, int d, int h_kv);

/* fathom_pack_planes -- build the bit-plane store from a 4-bit K cache.
 *   codes   [h_kv][n][d/2] uint8, token-major, two channels per byte, low
 *           nibble = even channel: the per-channel asymmetric 4-bit codes a
 *           quantised serving stack holds (abstract: the store is the
 *           4-bit copy of K that such a stack keeps anyway).  Read only.
 *   planes  [h_kv][d][4][fathom_plane_words(n)] uint32, written in full
 *           (padding zeroed).  16-byte aligned.
 * n >= 0 (n = 0 writes nothing), d as FATHOM_MAX_D, h_kv >= 1.
 */
FATHOM_API fathom_status fathom_pack_planes(const uint8_t *codes, int64_t n, int d, int h_kv,
                                 uint32_t *planes, void *stream);

/* fathom_append_planes -- add m decoded tokens to a store of n tokens
 * (decoding grows the cache a token at a time).
 *   codes       [h_kv][m][d/2] uint8: the new tokens' 4-bit codes, laid out as
 *               for fathom_pack_planes.  The codes come from the caller's
 *               quantiser with the store's existing per-channel m_c, s_c,
 *               clamped to 0..15: the scan's dequantisation stays that of
 *               the store.  Requantising for a new min/max means packing
 *               anew.
 *   planes_in   [h_kv][d][4][fathom_plane_words(n)], the store of tokens
 *               0 .. n - 1 (padding bits zero, as fathom_pack_planes leaves
 *               them).
 *   planes_out  [h_kv][d][4][fathom_plane_words(n + m)].  It may be planes_in
 *               itself when the row length does not change
 *               (fathom_plane_words(n + m) == fathom_plane_words(n)); then only
 *               the words holding the new tokens are touched.  Otherwise it
 *               must not overlap planes_in, which is copied into it first.
 * The result equals fathom_pack_planes of all n + m tokens' codes.
 */
FATHOM_API fathom_status fathom_append_planes(const uint8_t *codes, int64_t n, int64_t m, int d,
                                   int h_kv, const uint32_t *planes_in, uint32_t *planes_out,
                                   void *stream);

/* fathom_allocate -- per-query bit allocation by reverse water-filling
 * (method paragraph 3: reverse water-filling gives more bits to the
 * channels that weigh most for the query at hand, in closed form;
 * abstract: the weights are the channels' variance-weighted importance).
 *   q       [h_q][d], FATHOM_BF16 or FATHOM_F32.
 *   sigma   [h_kv][d] float, the channel statistics sigma_c (head h uses row
 *           h / G).  Importance w_c = q_c^2 sigma_c^2 (fp64).
 *   alloc   [h_q][d] uint8 out: t_c in 0..4 with sum_c t_c = budget_bits.
 * The continuous rule is b_c = clip(log2(w_c / theta) / 2, 0, 4) with theta
 * set so that sum_c b_c = B.  Its integer form, computed exactly: take the B
 * largest of the 4d slot keys w_c 4^-tau (tau = 0..3), ties broken by lower
 * channel then lower tau, and let t_c count channel c's slots.  This is the
 * exact optimum of sum_c w_c 4^-t_c subject to sum_c t_c = B and equals the
 * largest-remainder rounding of the closed form.  0 <= budget_bits <= 4d.
 * For many sessions pass them concatenated: h_q = S*H_q, sigma [S*H_kv][d].
 */
FATHOM_API fathom_status fathom_allocate(const void *q, fathom_dtype q_dtype, const float *sigma, int h_q,
                              int h_kv, int d, int budget_bits, uint8_t *alloc, void *stream);

/* fathom_allocate_uniform -- a query-independent allocation of the same
 * budget: the fixed-depth read that the pages' measurements set the
 * adaptive read against (findings: GPU time against scans that read 136
 * bits per key; abstract: comparisons at the same number of bytes read).
 *   alloc   [h_q][d] uint8 out: t_c = budget_bits / d for every channel,
 *           plus one for channels c < budget_bits % d; the same row for
 *           every head, so sum_c t_c = budget_bits.
 * This is fathom_allocate's rule with every channel equally important (its
 * tie-break takes lower channels first), so a GQA group's union prefix is
 * one head's read.  The result feeds fathom_scan_topk unchanged.
 * Requires d a multiple of 32 in [32, 256], h_q >= 1 and
 * 0 <= budget_bits <= 4d.
 */
FATHOM_API fathom_status fathom_allocate_uniform(int h_q, int d, int budget_bits, uint8_t *alloc,
                                      void *stream);

/* fathom_scan_topk -- score all n keys of one session from the allocated
 * plane prefixes and return each query head's top-k (method paragraph 1:
 * sparse decoding finds its top-k candidates by scanning many keys;
 * abstract: the scan ranks every one of the n keys for each top-k step).
 *
 * Score of key i for query head h (KV head g = h / G):
 *   s_h(i) = sum_c q_c * deq_{t_c}(v_{t_c}(i, c)),
 * v_t the value of the first t planes of channel c and
 * deq_t(v) = m_c + s_c (2^(4-t) v + (2^(4-t) - 1) / 2), the centre of the
 * t-bit cell (t = 0: the constant m_c + 7.5 s_c).  Scores are formed in
 * fp32: the tensor-core kernel sums the plane bits against 30-bit fixed-point
 * weights exactly in int32 and converts once, the CUDA-core kernel
 * accumulates fp32 FMAs.
 * Output per head: the k keys with the largest s_h, ordered by score
 * descending then index ascending; if k > n the tail is index -1, score -inf.
 * Per KV head the scan reads, for each channel, the longest prefix any of its
 * G query heads was allocated (the union); each head uses only its own.
 */
typedef struct fathom_scan_args {
  const uint32_t *planes;  /* [h_kv][d][4][W] (device, or host-mapped pinned) */
  int planes_location;     /* fathom_planes_location */
  const float *qmin;       /* [h_kv][d] m_c, float ([h_kv][groups][d] with token_group) */
  const float *qscale;     /* [h_kv][d] s_c, float ([h_kv][groups][d] with token_group) */
  const void *q;           /* [h_q][d], q_dtype */
  int q_dtype;             /* fathom_dtype */
  const uint8_t *alloc;    /* [h_q][d] from fathom_allocate */
  int64_t n;               /* keys, 0 <= n < 2^31 */
  int d, h_q, h_kv, k;
  int32_t *out_idx;        /* [h_q][k] out */
  float *out_score;        /* [h_q][k] out */
  float *debug_scores;     /* optional [h_q][n] out: every score (tests); NULL normally */
  uint32_t flags;          /* FATHOM_FLAG_* test knobs, 0 normally */
  int64_t token_group;     /* 0: qmin/qscale are one (m, s) per channel over the whole
                            * context (the default reading).  Else the quantiser variant
                            * with statistics per run of token_group keys: a positive
                            * multiple of FATHOM_TOKEN_GROUP_QUANTUM, qmin/qscale
                            * [h_kv][ceil(n / token_group)][d], key i dequantised with row
                            * i / token_group.  The tensor-core scan only:
                            * FATHOM_ERR_UNSUPPORTED with FATHOM_FLAG_CUDA_CORES. */
} fathom_scan_args;

/* Token groups hold whole sample tiles (the sample pass reads one 256-key
 * sector in 64 and four of those per 1024-key tile): 65536 keys. */
#define FATHOM_TOKEN_GROUP_QUANTUM 65536

/* Bytes of workspace fathom_scan_topk needs for these arguments (0 on bad
 * arguments).  The workspace is device memory, 256-byte aligned, owned by the
 * caller, reused across calls; calls sharing one workspace must not overlap. */
FATHOM_API size_t fathom_scan_topk_workspace_size(const fathom_scan_args *args);
FATHOM_API fathom_status fathom_scan_topk(const fathom_scan_args *args, void *workspace,
                               size_t workspace_bytes, void *stream);

/* Batched ragged sessions (abstract: many sessions are resident together): one
 * set of launches scores every session; sessions share d, h_q, h_kv, k and
 * the dtype and differ in n and buffers.  `sessions` is a DEVICE array of S
 * descriptors, which the host never reads: its pointers are not checked.
 * The kernels check each descriptor's n against n_max (the bound the
 * workspace was sized for): a session with n < 0 or n > n_max is scanned as
 * empty (its heads get index -1, score -inf) and counted in the report's
 * device_faults, so fathom_scan_read_report returns FATHOM_ERR_DEVICE_CHECK. */
typedef struct fathom_session {
  const uint32_t *planes;  /* [h_kv][d][4][fathom_plane_words(n)] */
  const float *qmin;       /* [h_kv][d] */
  const float *qscale;     /* [h_kv][d] */
  const void *q;           /* [h_q][d] */
  const uint8_t *alloc;    /* [h_q][d] */
  int64_t n;               /* 0 <= n <= n_max */
  int32_t *out_idx;        /* [h_q][k] */
  float *out_score;        /* [h_q][k] */
} fathom_session;

typedef struct fathom_batched_args {
  const fathom_session *sessions; /* device array [num_sessions] */
  int num_sessions;               /* 1 <= S <= 1024 */
  int64_t n_max;                  /* an upper bound on every session's n */
  int d, h_q, h_kv, k;
  int q_dtype;                    /* fathom_dtype */
  int planes_location;            /* fathom_planes_location, all sessions */
  uint32_t flags;                 /* FATHOM_FLAG_* */
} fathom_batched_args;

FATHOM_API size_t fathom_scan_topk_batched_workspace_size(const fathom_batched_args *args);
FATHOM_API fathom_status fathom_scan_topk_batched(const fathom_batched_args *args, void *workspace,
                                       size_t workspace_bytes, void *stream);

/* fathom_scan_topk_noalloc -- fathom_scan_topk for callers that cannot
 * allocate device memory.  The paper has no counterpart; this is a service of
 * this library.
 *
 * Some callers may not call cudaMalloc: a plugin running inside an inference
 * server that owns all device memory through its own pool and forbids
 * plugins from allocating, or a latency-critical decode loop where an
 * allocation can block or synchronise the device.  They still provide the
 * inputs and outputs in `args`, but no workspace: this entry point uses a
 * fixed scratch array compiled into the library, FATHOM_NOALLOC_SCRATCH_BYTES
 * (16 MiB) of device memory that every GPU which loads the library holds
 * until the process exits.
 *   - Sizes whose workspace (fathom_scan_topk_workspace_size) exceeds the
 *     scratch are rejected with FATHOM_ERR_WORKSPACE_TOO_SMALL; nothing is
 *     launched.  The 1M-token, 32-query-head, k = 2048 step fits.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.  The
 *     first call on each device looks up the scratch array's device address
 *     (cudaGetSymbolAddress, which may load the library's kernels onto that
 *     device); make that first call before any stream capture.  The address
 *     is kept per device together with the id of the CUDA context it belongs
 *     to: after a device reset (cudaDeviceReset) the next call runs that
 *     set-up again, so it too should come before any capture.
 *   - All calls share the one array, which keeps the previous call's data;
 *     each call clears the counters that must start at zero.  Calls whose
 *     work overlaps on the GPU (different streams, or different host threads
 *     without ordering) race on the scratch: order them.
 *   - Results are those of fathom_scan_topk on the same arguments.
 */
#define FATHOM_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
FATHOM_API fathom_status fathom_scan_topk_noalloc(const fathom_scan_args *args, void *stream);

/* Profiling hook: while set, every scan launch set of the calling thread
 * records `begin` (a cudaEvent_t) on its stream just before the filtering scan
 * kernel -- the kernel that streams the union plane prefixes -- and `end`
 * just after it, so a caller can time that kernel alone with
 * cudaEventElapsedTime.  Pass NULL, NULL to clear.  Never synchronises.
 * The two events stop the kernels around the filtering scan from overlapping
 * it, so time whole steps without them. */
FATHOM_API void fathom_profile_scan_kernel(void *begin, void *end);

/* What the last scan on a workspace recorded.  Synchronises `stream`. */
typedef struct fathom_scan_report {
  uint32_t fallback_heads;  /* heads whose sampled threshold failed; answered exactly by the fallback */
  uint32_t device_faults;   /* device-side check failures (0 expected) */
  uint32_t max_candidates;  /* largest per-head candidate count */
  uint32_t union_planes;    /* sum over sessions and KV heads of the union prefix planes */
} fathom_scan_report;

FATHOM_API fathom_status fathom_scan_read_report(const void *workspace, fathom_scan_report *report,
                                      void *stream);

/* fathom_check_device_status -- FATHOM_OK when the last scan on `workspace`
 * recorded no device-side fault, else FATHOM_ERR_DEVICE_CHECK with the count
 * in fathom_last_error().  Faults are bounded mbarrier waits that gave up
 * and, in the checked build (libfathom_checked.so, FATHOM_DEVICE_CHECKS),
 * every guarded global or shared access that was out of range and skipped.
 * Synchronises `stream`; FATHOM_ERR_INVALID_ARGUMENT for a workspace that is
 * not device memory. */
FATHOM_API fathom_status fathom_check_device_status(const void *workspace, void *stream);

/* fathom_scan_read_report_noalloc -- the report of the last
 * fathom_scan_topk_noalloc on the current device (its status block lives in
 * the built-in scratch, whose address the caller never sees).  Same fields
 * and status as fathom_scan_read_report; synchronises `stream`.  Like the
 * scan itself it allocates nothing; no counterpart in the paper. */
FATHOM_API fathom_status fathom_scan_read_report_noalloc(fathom_scan_report *report, void *stream);

/* fathom_merge_topk -- the top-k of a scan whose keys were split into token
 * ranges: the last step of token-range sharding, where each GPU scans the
 * planes of its own range of the context (fathom_scan_topk, local indices)
 * and the per-range lists are gathered (one all-gather of parts x k
 * (index, score) pairs per head over NVLink).  The pages rank every key of
 * the context for each top-k step (abstract); the k best of the context are
 * the k best of the union of every range's k best, so the merged answer is
 * the unsplit scan's.
 *   in_idx     int32 [parts][h_q][k_in], in_score float [parts][h_q][k_in]:
 *              each part's fathom_scan_topk output for its range -- sorted by
 *              score descending then index ascending, -1 padding at the tail;
 *              indices local to the range.
 *   offsets    HOST array int64 [parts]: first token of each range, so that
 *              a part's global index is offsets[p] + local index.  Ranges
 *              must not overlap; global indices must stay below 2^31 - 1
 *              (larger ones are dropped).
 *   out_idx    int32 [h_q][k], out_score float [h_q][k]: the k best by score
 *              descending then global index ascending; -1 / -inf past the
 *              number of entries.
 * Requires 1 <= parts <= FATHOM_MAX_MERGE_PARTS, 1 <= k_in, k <= FATHOM_MAX_K,
 * h_q >= 1.  Device pointers; no workspace.  An input list that is not
 * sorted gives an unspecified (but in-bounds) result.
 */
FATHOM_API fathom_status fathom_merge_topk(const int32_t *in_idx, const float *in_score, int parts,
                                           const int64_t *offsets, int h_q, int k_in, int k,
                                           int32_t *out_idx, float *out_score, void *stream);

/* fathom_sparse_attention -- the step after the scan: each query head's
 * attention over only the keys its top-k selected (method paragraph 1: the
 * scan finds the top-k candidates, and only the few KV rows that win are
 * then fetched).  For head h (KV head
 * g = h / G) and its entries idx[h][r] in [0, n):
 *   s_r = softmax_scale * <q[h], k_rows[g][idx[h][r]]>,
 *   out[h] = sum_r softmax(s)_r v_rows[g][idx[h][r]],
 *   lse[h] = log(sum_r exp(s_r))   (natural log).
 * Entries outside [0, n) (the -1 padding of fathom_scan_topk) are skipped; a
 * head with none gets out = 0 and lse = -inf.  fp32 arithmetic.
 *   q        [h_q][d], FATHOM_BF16 or FATHOM_F32.
 *   k_rows, v_rows   bf16 [h_kv][n][d]: the serving stack's keys and values
 *            (16-byte aligned).
 *   k_codes  optional uint8 [h_kv][n][d/2]: the 4-bit key codes (the layout
 *            fathom_pack_planes reads) with k_qmin, k_qscale float [h_kv][d];
 *            when set, key row i is k_qmin + k_qscale * code (the 4-bit
 *            dequantisation, a quarter of a bf16 row's bytes per gathered
 *            key) and k_rows is not read (it may be NULL).
 *   kv_location  FATHOM_PLANES_DEVICE, or FATHOM_PLANES_HOST_MAPPED when
 *            k_rows / k_codes and v_rows are pinned host memory mapped into
 *            the device (the pages' offloaded KV cache, whose title names it):
 *            only the selected rows cross the host link.
 *   idx      int32 [h_q][k], e.g. fathom_scan_topk's out_idx.
 *   out      float [h_q][d]; lse float [h_q] or NULL.
 * Requires d as FATHOM_MAX_D, h_q a multiple of h_kv, k >= 0, 0 <= n < 2^31
 * and a finite softmax_scale (1/sqrt(d) is the usual one).  No workspace.
 */
typedef struct fathom_attention_args {
  const void *q;
  fathom_dtype q_dtype;
  const uint16_t *k_rows;
  const uint16_t *v_rows;
  const int32_t *idx;
  int64_t n;
  int d, h_q, h_kv, k;
  float softmax_scale;
  float *out;
  float *lse;
  int kv_location;          /* fathom_planes_location of the K and V rows */
  const uint8_t *k_codes;   /* optional 4-bit keys (then k_rows is unused) */
  const float *k_qmin;      /* [h_kv][d], with k_codes */
  const float *k_qscale;    /* [h_kv][d], with k_codes */
} fathom_attention_args;

FATHOM_API fathom_status fathom_sparse_attention(const fathom_attention_args *args, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* FATHOM_H */
