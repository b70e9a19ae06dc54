// Sparse attention over the selected keys: the step after the scan ("Fathom
// Makes KV-Cache Scans Query-Adaptive for Long-Context Decoding", method
// paragraph 1: the scan finds the top-k candidates, and only the few KV rows
// that win are then fetched).
//
// For query head h (KV head g = h / G) and its selected keys idx_r >= 0:
//   s_r = scale <q_h, K[g][idx_r]>,  o_h = sum_r softmax(s)_r V[g][idx_r],
//   lse_h = log sum_r exp(s_r).
// A decode query is one vector per head, so this is a gather of k rows of K
// and V followed by matrix-vector work: bound by the gathered bytes, not by
// arithmetic, and kept on the CUDA cores.
//
// A cluster of 8 CTAs of 256 threads per query head, so that the gather
// runs on 8 SMs per head.  Warp w of the head's 64 takes the selected rows
// w * U .. w * U + U - 1, then the next 64 U, ...; each lane holds d / 32
// consecutive dimensions of q, of the running output and of every row it
// loads.  A warp first issues the loads (K and V) of its U rows (U = 8 up to
// d = 128, else 4), reduces their U dot products across the warp together,
// then folds them into an online softmax in base 2 with one rescale per pass
// (q pre-scaled by scale * log2 e).  Each CTA merges its 8 warps' partial
// (max, sum, output) in shared memory; CTA 0 of the cluster merges the 8 CTA
// partials through distributed shared memory and writes the result.
// Indices outside [0, n) are skipped, as are -1 entries.
//
// Keys come either as bf16 rows or as the 4-bit codes the scan's store is
// packed from (k = m_c + s_c u, dequantised in the gather: a quarter of the
// bytes of a bf16 row).  Keys and values may live in device memory or in
// pinned host memory mapped into the device (the pages' offloaded cache,
// "Fathom: Per-Query Read Depth for Sparse Decoding over Offloaded KV
// Caches", abstract): then only the selected rows cross the host link.
#include <cooperative_groups.h>

#include "fathom_internal.cuh"

namespace cg = cooperative_groups;

namespace fathom {

constexpr int kAttnSplit = 8;  // CTAs per query head: one cluster
constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;            // per CTA
constexpr int kAttnHeadWarps = kAttnSplit * kAttnWarps;  // per head
// rows a warp has in flight (a pass): their loads are issued together, and
// their scores reduced and folded into the online softmax together
__host__ __device__ constexpr int attn_rows(int dpl) { return dpl <= 4 ? 8 : 4; }

struct AttnParams {
  const void *q;
  int q_bf16;
  const uint16_t *k_rows;
  const uint8_t *k_codes;  // when set: 4-bit keys [h_kv][n][d/2], k = m + s u
  const float *k_qmin;
  const float *k_qscale;
  const uint16_t *v_rows;
  const int32_t *idx;
  int64_t n;
  int d, G, k;
  float qscale;  // softmax scale * log2(e)
  float *out;
  float *lse;
};

__device__ __forceinline__ float bf16_float(uint16_t x) {
  return __uint_as_float((uint32_t)x << 16);
}

// DPL consecutive bf16 values starting at p (p aligned to 2 DPL bytes when
// DPL is a power of two, else to 4 bytes when DPL is even).
template <int DPL>
__device__ __forceinline__ void load_row_part(const uint16_t *p, uint32_t (&w)[(DPL + 1) / 2]) {
  if (DPL == 8) {
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if (DPL == 4) {
    const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
    w[0] = v.x; w[1] = v.y;
  } else if (DPL % 2 == 0) {
#pragma unroll
    for (int i = 0; i < DPL / 2; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t *>(p) + i);
  } else {
#pragma unroll
    for (int i = 0; i < (DPL + 1) / 2; ++i) {
      const uint32_t lo = __ldg(p + 2 * i);
      const uint32_t hi = 2 * i + 1 < DPL ? (uint32_t)__ldg(p + 2 * i + 1) : 0u;
      w[i] = lo | (hi << 16);
    }
  }
}

__device__ __forceinline__ float part_value(const uint32_t *w, int i) {
  return bf16_float((uint16_t)(w[i >> 1] >> (16 * (i & 1))));
}

// The DPL 4-bit codes of dimensions c0 .. c0 + DPL - 1 of a code row (two
// channels per byte, low nibble = even channel), packed in order from bit 0.
template <int DPL>
__device__ __forceinline__ uint32_t load_codes_part(const uint8_t *row, int c0) {
  if (DPL == 8) return __ldg(reinterpret_cast<const uint32_t *>(row + c0 / 2));
  if (DPL == 4) return __ldg(reinterpret_cast<const uint16_t *>(row + c0 / 2));
  if (DPL == 2) return __ldg(row + c0 / 2);
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    const int c = c0 + i;
    w |= (uint32_t)((__ldg(row + c / 2) >> (4 * (c & 1))) & 15u) << (4 * i);
  }
  return w;
}

template <int DPL, bool CODES>
__global__ void __cluster_dims__(kAttnSplit, 1, 1) __launch_bounds__(kAttnThreads)
    attention_kernel(AttnParams a) {
  grid_dependency_wait();
  allow_dependent_launch();
  constexpr int D = 32 * DPL;
  constexpr int NW = (DPL + 1) / 2;
  constexpr int kAttnRows = attn_rows(DPL);
  __shared__ float s_m[kAttnWarps], s_l[kAttnWarps];
  __shared__ float s_o[kAttnWarps][D];
  __shared__ float s_pm, s_pl;  // this CTA's partial: max, sum
  __shared__ float s_po[D];     // and output
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int h = blockIdx.x / kAttnSplit;
  const int g = h / a.G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c0 = lane * DPL;

  float qv[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    const int64_t at = (int64_t)h * D + c0 + i;
    const float x = a.q_bf16 ? bf16_float(reinterpret_cast<const uint16_t *>(a.q)[at])
                             : reinterpret_cast<const float *>(a.q)[at];
    qv[i] = x * a.qscale;
  }
  const int32_t *ix = a.idx + (int64_t)h * a.k;
  const uint16_t *Kg = CODES ? nullptr : a.k_rows + (int64_t)g * a.n * D + c0;
  const uint8_t *Cg = CODES ? a.k_codes + (int64_t)g * a.n * (D / 2) : nullptr;
  const uint16_t *Vg = a.v_rows + (int64_t)g * a.n * D + c0;
  float km[DPL], ks[DPL];  // dequantisation of this lane's dimensions (4-bit keys)
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    km[i] = CODES ? a.k_qmin[(int64_t)g * D + c0 + i] : 0.0f;
    ks[i] = CODES ? a.k_qscale[(int64_t)g * D + c0 + i] : 0.0f;
  }

  float m = -INFINITY, l = 0.0f, o[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) o[i] = 0.0f;

  // A pass: kAttnRows rows of this warp, their loads issued together.  Two
  // passes are in flight: the loads of the next pass are issued before the
  // current one is folded in, so their latency overlaps its arithmetic.
  struct Pass {
    int row[kAttnRows];  // -1: no selected row (n < 2^31)
    uint32_t kw[kAttnRows][CODES ? 1 : NW], vw[kAttnRows][NW];
  };
  auto load_pass = [&](int r0, Pass &ps) {
#pragma unroll
    for (int u = 0; u < kAttnRows; ++u) {
      const int r = r0 + u;
      const int32_t x = r < a.k ? __ldg(ix + r) : -1;
      ps.row[u] = (x >= 0 && (int64_t)x < a.n) ? x : -1;
      if (ps.row[u] >= 0) {
        if constexpr (CODES)
          ps.kw[u][0] = load_codes_part<DPL>(Cg + (int64_t)ps.row[u] * (D / 2), c0);
        else
          load_row_part<DPL>(Kg + (int64_t)ps.row[u] * D, ps.kw[u]);
        load_row_part<DPL>(Vg + (int64_t)ps.row[u] * D, ps.vw[u]);
      } else {
#pragma unroll
        for (int i = 0; i < (CODES ? 1 : NW); ++i) ps.kw[u][i] = 0u;
#pragma unroll
        for (int i = 0; i < NW; ++i) ps.vw[u][i] = 0u;
      }
    }
  };
  auto fold_pass = [&](const Pass &ps) {
    // the pass's dot products: lane partials, then all kAttnRows warp sums at
    // once (independent shuffles), so the rows share the reduction latency
    float sc[kAttnRows];
#pragma unroll
    for (int u = 0; u < kAttnRows; ++u) {
      float s = 0.0f;
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        float kv;
        if constexpr (CODES)
          kv = fmaf(ks[i], (float)((ps.kw[u][0] >> (4 * i)) & 15u), km[i]);
        else
          kv = part_value(ps.kw[u], i);
        s = fmaf(qv[i], kv, s);
      }
      sc[u] = s;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int u = 0; u < kAttnRows; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], off);
    // one rescale per pass: the pass's largest score joins the running max
    float mb = -INFINITY;
#pragma unroll
    for (int u = 0; u < kAttnRows; ++u)
      if (ps.row[u] >= 0) mb = fmaxf(mb, sc[u]);  // the same for every lane of the warp
    if (mb == -INFINITY) return;                  // no selected row in this pass
    const float mn = fmaxf(m, mb);
    const float corr = exp2f(m - mn);  // 0 while m = -inf
    l *= corr;
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[i] *= corr;
#pragma unroll
    for (int u = 0; u < kAttnRows; ++u) {
      if (ps.row[u] < 0) continue;
      const float pr = exp2f(sc[u] - mn);
      l += pr;
#pragma unroll
      for (int i = 0; i < DPL; ++i) o[i] = fmaf(pr, part_value(ps.vw[u], i), o[i]);
    }
    m = mn;
  };
  const int rstep = kAttnHeadWarps * kAttnRows;
  int r0 = (rank * kAttnWarps + warp) * kAttnRows;
  Pass pa, pb;
  if (r0 < a.k) load_pass(r0, pa);
  while (r0 < a.k) {
    if (r0 + rstep < a.k) load_pass(r0 + rstep, pb);
    fold_pass(pa);
    r0 += rstep;
    if (r0 >= a.k) break;
    if (r0 + rstep < a.k) load_pass(r0 + rstep, pa);
    fold_pass(pb);
    r0 += rstep;
  }

  if (lane == 0) {
    s_m[warp] = m;
    s_l[warp] = l;
  }
#pragma unroll
  for (int i = 0; i < DPL; ++i) s_o[warp][c0 + i] = o[i];
  __syncthreads();
  float M = -INFINITY;
  for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, s_m[w]);
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    float L = 0.0f, O = 0.0f;
    if (M != -INFINITY) {
      for (int w = 0; w < kAttnWarps; ++w) {
        if (s_m[w] == -INFINITY) continue;
        const float f = exp2f(s_m[w] - M);
        L = fmaf(s_l[w], f, L);
        O = fmaf(s_o[w][c], f, O);
      }
    }
    s_po[c] = O;
    if (c == 0) {
      s_pm = M;
      s_pl = L;
    }
  }
  cluster.sync();  // every CTA's partial is in its shared memory
  if (rank == 0 && threadIdx.x < D) {
    const int c = threadIdx.x;
    float MM = -INFINITY;
    for (int r = 0; r < kAttnSplit; ++r) MM = fmaxf(MM, *cluster.map_shared_rank(&s_pm, r));
    float L = 0.0f, O = 0.0f;
    if (MM != -INFINITY) {
      for (int r = 0; r < kAttnSplit; ++r) {
        const float pm = *cluster.map_shared_rank(&s_pm, r);
        if (pm == -INFINITY) continue;
        const float f = exp2f(pm - MM);
        L = fmaf(*cluster.map_shared_rank(&s_pl, r), f, L);
        O = fmaf(*cluster.map_shared_rank(&s_po[c], r), f, O);
      }
    }
    a.out[(int64_t)h * D + c] = L > 0.0f ? O / L : 0.0f;
    if (c == 0 && a.lse) a.lse[h] = L > 0.0f ? (MM + log2f(L)) * 0.6931471805599453f : -INFINITY;
  }
  cluster.sync();  // CTA 0 has read the others' shared memory
}

template <bool CODES>
static cudaError_t launch_attention_d(const AttnParams &a, int d, dim3 grid, dim3 block,
                                     cudaStream_t stream) {
  switch (d / 32) {
    case 1: return launch_dependent(attention_kernel<1, CODES>, grid, block, 0, stream, a);
    case 2: return launch_dependent(attention_kernel<2, CODES>, grid, block, 0, stream, a);
    case 3: return launch_dependent(attention_kernel<3, CODES>, grid, block, 0, stream, a);
    case 4: return launch_dependent(attention_kernel<4, CODES>, grid, block, 0, stream, a);
    case 5: return launch_dependent(attention_kernel<5, CODES>, grid, block, 0, stream, a);
    case 6: return launch_dependent(attention_kernel<6, CODES>, grid, block, 0, stream, a);
    case 7: return launch_dependent(attention_kernel<7, CODES>, grid, block, 0, stream, a);
    case 8: return launch_dependent(attention_kernel<8, CODES>, grid, block, 0, stream, a);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attention(const void *q, int q_bf16, const uint16_t *k_rows,
                             const uint8_t *k_codes, const float *k_qmin, const float *k_qscale,
                             const uint16_t *v_rows, const int32_t *idx, int64_t n, int d,
                             int h_q, int h_kv, int k, float scale, float *out, float *lse,
                             cudaStream_t stream) {
  AttnParams a;
  a.q = q;
  a.q_bf16 = q_bf16;
  a.k_rows = k_rows;
  a.k_codes = k_codes;
  a.k_qmin = k_qmin;
  a.k_qscale = k_qscale;
  a.v_rows = v_rows;
  a.idx = idx;
  a.n = n;
  a.d = d;
  a.G = h_q / h_kv;
  a.k = k;
  a.qscale = scale * 1.4426950408889634f;
  a.out = out;
  a.lse = lse;
  const dim3 grid(h_q * kAttnSplit), block(kAttnThreads);
  return k_codes ? launch_attention_d<true>(a, d, grid, block, stream)
                 : launch_attention_d<false>(a, d, grid, block, stream);
}

}  // namespace fathom
