// fathom_merge_topk: the top-k of several partial top-k lists per query
// head, for a scan whose keys are split into token ranges (one range per
// GPU, each scanned with fathom_scan_topk, the lists gathered over NVLink).
//
// The pages rank every key of the context for each top-k step (arXiv
// 2609.17652 abstract; "Fathom Makes KV-Cache Scans Query-Adaptive for
// Long-Context Decoding", method paragraph 1).  The k best keys of the whole
// context are the k best of the union of every range's k best, so a split
// scan returns exactly the unsplit one's answer once the partial lists are
// merged.
//
// One block per query head.  Each list arrives sorted by (score desc,
// index asc) with -1 padding at its tail, which is the order of the
// composite (float key << 32 | ~global index) descending.  The rank of an
// entry in the merged order is its position in its own list plus, for every
// other list, the number of entries that order before it there (a binary
// search); an entry whose rank is below k is written at that rank.  Every
// global index is distinct, so the ranks are too.
#include "fathom_internal.cuh"

namespace fathom {

constexpr int kMergePartsThreads = 1024;

struct MergePartsParams {
  const int32_t *in_idx;   // [parts][h_q][k_in]
  const float *in_score;   // [parts][h_q][k_in]
  int parts, h_q, k_in, k;
  int staged;              // 1: the block's composites fit in shared memory
  int32_t *out_idx;        // [h_q][k]
  float *out_score;        // [h_q][k]
  int64_t offset[FATHOM_MAX_MERGE_PARTS];
};

// Composite of entry j of part b's list for head h (0 = no entry).
__device__ __forceinline__ unsigned long long merge_entry(const MergePartsParams &m, int b, int h,
                                                          int j) {
  const int64_t at = ((int64_t)b * m.h_q + h) * m.k_in + j;
  const int32_t li = m.in_idx[at];
  if (li < 0) return 0ull;
  const int64_t gi = m.offset[b] + li;
  if (gi >= 0x7fffffffll) return 0ull;
  return composite(m.in_score[at], (uint32_t)gi);
}

__global__ void __launch_bounds__(kMergePartsThreads) merge_parts_kernel(MergePartsParams m) {
  grid_dependency_wait();
  allow_dependent_launch();
  extern __shared__ unsigned long long s_c[];  // [parts][k_in] when staged
  const int h = blockIdx.x;
  const int cnt = m.parts * m.k_in;
  if (m.staged) {
    for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
      const int b = i / m.k_in;
      s_c[i] = merge_entry(m, b, h, i - b * m.k_in);
    }
  }
  for (int r = threadIdx.x; r < m.k; r += blockDim.x) {
    m.out_idx[(int64_t)h * m.k + r] = -1;
    m.out_score[(int64_t)h * m.k + r] = -INFINITY;
  }
  __syncthreads();
  auto get = [&](int b, int j) -> unsigned long long {
    return m.staged ? s_c[b * m.k_in + j] : merge_entry(m, b, h, j);
  };
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
    const int a = i / m.k_in;
    const int pos = i - a * m.k_in;
    const unsigned long long x = get(a, pos);
    if (x == 0ull) continue;
    int64_t rank = pos;
    for (int b = 0; b < m.parts && rank < m.k; ++b) {
      if (b == a) continue;
      // entries of list b that order before x: the first j with get(b, j) < x
      int lo = 0, hi = m.k_in;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (get(b, mid) > x) lo = mid + 1; else hi = mid;
      }
      rank += lo;
    }
    if (rank < m.k) {
      m.out_idx[(int64_t)h * m.k + rank] = (int32_t)(0xffffffffu - (uint32_t)(x & 0xffffffffull));
      m.out_score[(int64_t)h * m.k + rank] = key_float((uint32_t)(x >> 32));
    }
  }
}

cudaError_t launch_merge_parts(const int32_t *in_idx, const float *in_score, int parts,
                               const int64_t *offsets, int h_q, int k_in, int k, int32_t *out_idx,
                               float *out_score, cudaStream_t stream) {
  MergePartsParams m;
  m.in_idx = in_idx;
  m.in_score = in_score;
  m.parts = parts;
  m.h_q = h_q;
  m.k_in = k_in;
  m.k = k;
  m.out_idx = out_idx;
  m.out_score = out_score;
  for (int b = 0; b < FATHOM_MAX_MERGE_PARTS; ++b) m.offset[b] = b < parts ? offsets[b] : 0;
  const size_t bytes = (size_t)parts * k_in * 8;
  m.staged = bytes <= (size_t)200 * 1024 ? 1 : 0;
  const size_t smem = m.staged ? bytes : 0;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(merge_parts_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_dependent(merge_parts_kernel, dim3(h_q), dim3(kMergePartsThreads), smem, stream, m);
}

}  // namespace fathom
