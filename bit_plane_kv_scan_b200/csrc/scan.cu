// The Fathom query-adaptive key scan and its top-k, for sm_100a.
//
// What is computed ("Fathom Makes KV-Cache Scans Query-Adaptive for
// Long-Context Decoding", method paragraphs 1-3; arXiv 2609.17652
// abstract): for every query head h and key i,
//   s_h(i) = sum_c q_c * deq_{t_c}(v_{t_c}(i, c)),
// v_t the value of the first t bit planes of channel c and deq_t the centre
// of the t-bit cell, followed by the k largest s_h per head.
//
// How (B200 design, not the pages' A100 one):
//  * plan_kernel, one block per (session, KV head): the union prefix
//    t*_c = max over the G query heads of t_c, and per channel the distinct
//    prefix lengths ("features") with the heads that use each.  Per head the
//    score is rewritten as
//        s_h(i) = K_h + sum_{c: t_c > 0} W_c * x_{t_c}(i, c),
//        W_c = 32 q_c s_c,  x_t = 1/2 + y_t / 32,
//    y_t the code's top t bits left-aligned in 4 bits (y_t = 2^(4-t) v_t),
//    K_h = sum_c q_c (m_c + s_c (2^(4-t_c) - 1) / 2) - sum_{c: t_c > 0} W_c / 2.
//    x_t is an exact fp32 bit pattern (exponent -1, y_t in the top four
//    fraction bits), so one byte permute per (token, channel, feature) and
//    one packed FMA per (token pair, head) replace t_c conditional adds.
//  * scan_kernel, persistent blocks of 128 threads over 2048-token tiles:
//    the union plane rows of a tile are staged into shared memory with
//    16-byte cp.async copies, three stages in flight; two threads share a
//    plane word and each keeps 16 tokens x G heads of scores in registers
//    (fp32x2 FMAs); the filtering pass writes the tokens whose score clears
//    the head's sampled threshold as (score, index) candidates.
//  * A sample pass of the same kernel scores one 256-token sector in 64 and
//    threshold_kernel takes the r-th largest sampled score per head as that
//    threshold (expected ~2k candidates per head, no dense score write).
//  * merge_kernel, one block per head: exact radix select of the k-th
//    largest (score, -index) composite among the candidates, then a sort.
//    When a threshold turns out invalid (fewer than k candidates, or more
//    than the buffer holds) the block recomputes that head exactly with a
//    streaming single-block scan.
#include <float.h>

#include <atomic>

#include "fathom_internal.cuh"

namespace fathom {

// ------------------------------------------------------------ utilities --

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// x shifted right by S (S > 0) or left by -S.  Right shifts are written as
// the high half of a multiply and left shifts as a multiply, so that they
// may issue on the FMA pipe rather than the busier integer ALU pipe.
// Call sites pass compile-time shifts (unrolled loops), so the branches fold.
__device__ __forceinline__ uint32_t shift_by(uint32_t x, int s) {
  if (s > 0) return __umulhi(x, 1u << (32 - s));
  if (s < 0) return x * (1u << (-s));
  return x;
}

// Block-wide inclusive scan of one int per thread (blockDim.x <= 1024).
__device__ int block_inclusive_scan(int v, int *s_tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  if (lane == 31) s_tmp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    const int nw = (blockDim.x + 31) >> 5;
    int x = lane < nw ? s_tmp[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int o = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += o;
    }
    if (lane < nw) s_tmp[lane] = x;
  }
  __syncthreads();
  if (warp > 0) v += s_tmp[warp - 1];
  __syncthreads();
  return v;
}

// Adds one to hist[digit] for every lane with digit >= 0.
__device__ __forceinline__ void hist_add(unsigned *hist, int digit) {
  if (digit >= 0) atomicAdd(&hist[digit], 1u);
}

// ------------------------------------------------------------ plan kernel --

__global__ void __launch_bounds__(256) plan_kernel(ScanParams p) {
  grid_dependency_wait();
  allow_dependent_launch();
  // clear the workspace's status, counters and thresholds (read by the
  // kernels after this one)
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.zero_words; i += gridDim.x * blockDim.x)
    p.zero[i] = 0u;
  const int gid = blockIdx.x;
  const int s = gid / p.h_kv;
  const int g = gid - s * p.h_kv;
  const fathom_session &se = session_of(p, s);
  const int d = p.d, G = p.G;
  const int c = threadIdx.x;
  const PlanLayout L = plan_layout(d);
  unsigned char *plan = p.plans + (size_t)gid * L.bytes;
  PlanHeader *hdr = reinterpret_cast<PlanHeader *>(plan);
  uint16_t *stage_begin = reinterpret_cast<uint16_t *>(plan + L.off_stage_begin);
  uint8_t *stage_nrows = plan + L.off_stage_nrows;
  uint16_t *stage_rows = reinterpret_cast<uint16_t *>(plan + L.off_stage_rows);
  uint32_t *info = reinterpret_cast<uint32_t *>(plan + L.off_info);
  uint32_t *feat = reinterpret_cast<uint32_t *>(plan + L.off_feat);
  float4 *wts = reinterpret_cast<float4 *>(plan + L.off_w);

  __shared__ int s_tmp[32];
  __shared__ double s_k[4][8];
  __shared__ int s_stage_base[64];
  __shared__ int s_total[2];

  int tstar = 0, nfeat = 0;
  uint32_t fbits = 0;
  float W[4] = {0.f, 0.f, 0.f, 0.f};
  double kpart[4] = {0.0, 0.0, 0.0, 0.0};
  if (c < d) {
    const float m = se.qmin[(int64_t)g * d + c];
    const float sc = se.qscale[(int64_t)g * d + c];
    int t[4] = {0, 0, 0, 0};
    for (int hh = 0; hh < G; ++hh) {
      const int64_t hq = (int64_t)(g * G + hh) * d + c;
      t[hh] = se.alloc[hq];
      const float qv = load_q(se.q, p.q_bf16, hq);
      tstar = max(tstar, t[hh]);
      W[hh] = t[hh] > 0 ? (qv * sc) * 32.0f : 0.0f;
      const double cell = (double)(1 << (4 - t[hh]));
      kpart[hh] =
          (double)qv * ((double)m + (double)sc * ((cell - 1.0) * 0.5)) - 0.5 * (double)W[hh];
    }
    for (int tf = 1; tf <= 4; ++tf) {
      uint32_t mask = 0;
      for (int hh = 0; hh < G; ++hh) mask |= (t[hh] == tf ? 1u : 0u) << hh;
      if (mask) {
        fbits |= ((uint32_t)tf | (mask << 3)) << (8 * nfeat);
        ++nfeat;
      }
    }
  }
  // per-head constants
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int hh = 0; hh < G; ++hh) {
    double v = kpart[hh];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) s_k[hh][warp] = v;
  }
  // entry index and first plane of every channel with t* > 0
  const int packed = (tstar > 0 ? 1 : 0) | (tstar << 12);
  const int incl = block_inclusive_scan(packed, s_tmp);
  const int e = (incl & 0xfff) - 1;  // entry index if tstar > 0
  const int p_incl = incl >> 12;     // planes up to and including c
  const int p_excl = p_incl - tstar;
  if (threadIdx.x == blockDim.x - 1) {
    s_total[0] = incl & 0xfff;  // entries
    s_total[1] = incl >> 12;    // union planes
  }
  const int stage = tstar > 0 ? (p_incl - 1) / kStageSpan : -1;
  const int prev_stage = tstar > 0 ? (p_excl > 0 ? (p_excl - 1) / kStageSpan : -1) : -1;
  // the first entry of a stage is the one whose previous plane lies in an earlier stage
  if (tstar > 0 && (p_excl == 0 || prev_stage != stage)) {
    s_stage_base[stage] = p_excl;
    stage_begin[stage] = (uint16_t)e;
  }
  __syncthreads();
  const int nent = s_total[0];
  const int nplanes = s_total[1];
  const int nstage = nplanes > 0 ? (nplanes - 1) / kStageSpan + 1 : 1;
  if (tstar > 0) {
    const int slot0 = p_excl - s_stage_base[stage];
    info[e] = (uint32_t)c | ((uint32_t)tstar << 8) | ((uint32_t)slot0 << 11) |
              ((uint32_t)nfeat << 16);
    feat[e] = fbits;
    wts[e] = make_float4(W[0], W[1], W[2], W[3]);
    for (int j = 0; j < tstar; ++j)
      stage_rows[stage * kStageRows + slot0 + j] = (uint16_t)(c * 4 + j);
  }
  if (threadIdx.x < nstage) {
    const int st = threadIdx.x;
    const int base = nplanes > 0 ? s_stage_base[st] : 0;
    const int end = (st + 1 < nstage) ? s_stage_base[st + 1] : nplanes;
    stage_nrows[st] = (uint8_t)(end - base);
  }
  if (threadIdx.x == 0) {
    if (nplanes == 0) stage_begin[0] = 0;
    stage_begin[nstage] = (uint16_t)nent;
    hdr->nent = nent;
    hdr->nstage = nstage;
    hdr->union_planes = nplanes;
    const int nw = (blockDim.x + 31) >> 5;
    for (int hh = 0; hh < 4; ++hh) {
      double sum = 0.0;
      if (hh < G)
        for (int w = 0; w < nw; ++w) sum += s_k[hh][w];
      hdr->K[hh] = (float)sum;
      hdr->tau[hh] = -INFINITY;
    }
  }
}

// ------------------------------------------------------------ scan kernel --

struct TileLoc {
  int s, g, ti;  // session, KV head, tile within (session, KV head)
  int64_t n, W;  // session keys and plane words
  const uint32_t *planes;
};

struct Item {
  int t;     // tile index in the launch's tile space (-1 = none)
  int st;    // stage within the tile
  int slot;  // plan slot in shared memory
  int nst;   // stages of this tile
};

template <int MODE>
__device__ __forceinline__ int64_t tiles_per_group(int64_t n, const ScanParams &p) {
  return MODE == kModeSample ? sample_tiles(n, p.sample_rank, p.flags) : filter_tiles(n);
}

template <int MODE>
__device__ __forceinline__ TileLoc locate(const ScanParams &p, const int *s_tprefix, int t) {
  int lo = 0, hi = p.S;  // find s with prefix[s] <= t < prefix[s+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_tprefix[mid] <= t) lo = mid; else hi = mid;
  }
  TileLoc L;
  L.s = lo;
  const fathom_session &se = session_of(p, lo);
  L.n = session_n(p, lo);
  L.W = plane_words(L.n);
  L.planes = se.planes;
  const int per = (int)tiles_per_group<MODE>(L.n, p);
  const int r = t - s_tprefix[lo];
  L.g = r / per;
  L.ti = r - L.g * per;
  return L;
}

// One channel of the plan for this thread's 16 tokens (bit positions
// 8 kk + r of its word, r = HALF .. HALF + 3).
//  R[i], byte kk = y << 3 for token 8 kk + HALF + i, y = the union prefix
//  code left-aligned in 4 bits (plane j lands on bit 6 - j).
//  Each feature masks R to its prefix length, turns every byte into the
//  fp32 x = 1/2 + y/32 with one byte permute ([0x3f][byte][0][0]), and adds
//  W_h x to the scores of the heads that read it.
template <int G, int HALF>
__device__ __forceinline__ void scan_entry(const uint32_t *src, int tstar, int nfeat, uint32_t fb,
                                           const float4 w4, float2 (&acc)[G][4][2]) {
  uint32_t R[4];
  const uint32_t p0 = src[0];
#pragma unroll
  for (int i = 0; i < 4; ++i) R[i] = shift_by(p0, HALF + i - 6) & 0x40404040u;
  if (tstar > 1) {
    const uint32_t p1 = src[kTileWords];
#pragma unroll
    for (int i = 0; i < 4; ++i) R[i] |= shift_by(p1, HALF + i - 5) & 0x20202020u;
    if (tstar > 2) {
      const uint32_t p2 = src[2 * kTileWords];
#pragma unroll
      for (int i = 0; i < 4; ++i) R[i] |= shift_by(p2, HALF + i - 4) & 0x10101010u;
      if (tstar > 3) {
        const uint32_t p3 = src[3 * kTileWords];
#pragma unroll
        for (int i = 0; i < 4; ++i) R[i] |= shift_by(p3, HALF + i - 3) & 0x08080808u;
      }
    }
  }
  const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
  for (int f = 0; f < nfeat; ++f) {
    const uint32_t byte = (fb >> (8 * f)) & 0xffu;
    const int tf = byte & 7;
    const uint32_t mask = byte >> 3;
    uint32_t Rf[4];
    if (tf == tstar) {
#pragma unroll
      for (int i = 0; i < 4; ++i) Rf[i] = R[i];
    } else {
      // keep planes j < tf: bits 6 .. 7 - tf of every byte
      const uint32_t keep = (((1u << tf) - 1u) << (7 - tf)) * 0x01010101u;
#pragma unroll
      for (int i = 0; i < 4; ++i) Rf[i] = R[i] & keep;
    }
    float2 xx[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int pp = 0; pp < 2; ++pp)
        xx[i][pp] = make_float2(
            __uint_as_float(__byte_perm(Rf[i], 0x3f000000u, 0x7054u | ((2 * pp) << 8))),
            __uint_as_float(__byte_perm(Rf[i], 0x3f000000u, 0x7054u | ((2 * pp + 1) << 8))));
#pragma unroll
    for (int h = 0; h < G; ++h) {
      if (mask & (1u << h)) {
        const float2 ww = make_float2(wv[h], wv[h]);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int pp = 0; pp < 2; ++pp) acc[h][i][pp] = __ffma2_rn(xx[i][pp], ww, acc[h][i][pp]);
      }
    }
  }
}

template <int G, int MODE>
__global__ void __launch_bounds__(kScanThreads, 4) scan_kernel(ScanParams p) {
  grid_dependency_wait();
  allow_dependent_launch();
  extern __shared__ __align__(16) unsigned char smem[];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int half = warp & 1;                 // which 16 tokens of the word
  const int word = (warp >> 1) * 32 + lane;  // word of the tile this thread reads
  const PlanLayout PL = plan_layout(p.d);
  uint32_t *sbuf = reinterpret_cast<uint32_t *>(smem);
  unsigned char *splans = smem + kNumBuf * kStageBytes;
  int *s_tprefix = reinterpret_cast<int *>(splans + kNumPlanSlots * PL.bytes);
  __shared__ int s_tmp[32];
  __shared__ int s_slot_gid[kNumPlanSlots];

  // ---- tile space: every (session, KV head) contributes its tiles --------
  for (int base = 0; base < p.S; base += kScanThreads) {
    const int s = base + tid;
    int v = 0;
    if (s < p.S) v = (int)(tiles_per_group<MODE>(session_n(p, s), p) * p.h_kv);
    const int carry = base > 0 ? s_tprefix[base] : 0;
    __syncthreads();
    const int incl = block_inclusive_scan(v, s_tmp);
    if (s < p.S) s_tprefix[s + 1] = carry + incl;
    if (base == 0 && tid == 0) s_tprefix[0] = 0;
    __syncthreads();
  }
  const int total = s_tprefix[p.S];
  const int t_begin = (int)(((int64_t)blockIdx.x * total) / gridDim.x);
  const int t_end = (int)(((int64_t)(blockIdx.x + 1) * total) / gridDim.x);
  if (t_begin >= t_end) return;
  if (tid < kNumPlanSlots) s_slot_gid[tid] = -1;
  __syncthreads();

  // ---- plan slots ---------------------------------------------------------
  // Loads the plan of (session s, KV head g) into a slot not used by the two
  // items ahead of it, unless it is resident already.  Called uniformly.
  auto ensure_plan = [&](int gid, int busy0, int busy1) -> int {
    int slot = -1;
#pragma unroll
    for (int i = 0; i < kNumPlanSlots; ++i)
      if (s_slot_gid[i] == gid) slot = i;
    if (slot >= 0) return slot;
#pragma unroll
    for (int i = kNumPlanSlots - 1; i >= 0; --i)
      if (i != busy0 && i != busy1) slot = i;
    __syncthreads();
    const uint4 *src = reinterpret_cast<const uint4 *>(p.plans + (size_t)gid * PL.bytes);
    uint4 *dst = reinterpret_cast<uint4 *>(splans + slot * PL.bytes);
    for (int i = tid; i < PL.bytes / 16; i += kScanThreads) dst[i] = src[i];
    __syncthreads();
    if (tid < G) {
      PlanHeader *hdr = reinterpret_cast<PlanHeader *>(splans + slot * PL.bytes);
      float tau = -INFINITY;
      if (MODE == kModeFilter) {
        const int s = gid / p.h_kv, g = gid - s * p.h_kv;
        const uint32_t key = p.tau[(int64_t)s * p.h_q + g * G + tid];
        tau = key == 0u ? -INFINITY : key_float(key);
      }
      hdr->tau[tid] = tau;
    }
    if (tid == 0) s_slot_gid[slot] = gid;
    __syncthreads();
    return slot;
  };

  auto first_item = [&](int t, int busy0, int busy1) -> Item {
    Item it;
    it.t = t;
    it.st = 0;
    if (t >= t_end) {
      it.t = -1;
      it.slot = -1;
      it.nst = 0;
      return it;
    }
    const TileLoc L = locate<MODE>(p, s_tprefix, t);
    it.slot = ensure_plan(L.s * p.h_kv + L.g, busy0, busy1);
    it.nst = reinterpret_cast<const PlanHeader *>(splans + it.slot * PL.bytes)->nstage;
    return it;
  };
  auto next_item = [&](const Item &a, int busy0, int busy1) -> Item {
    if (a.t < 0) return a;
    if (a.st + 1 < a.nst) {
      Item b = a;
      b.st += 1;
      return b;
    }
    return first_item(a.t + 1, busy0, busy1);
  };

  // ---- staged copies of one item's plane rows -----------------------------
  constexpr int kChunks = kTileWords / 4;  // 16-byte copies per staged row
  auto issue = [&](const Item &it, int buf) {
    if (it.t < 0) return;
    const TileLoc L = locate<MODE>(p, s_tprefix, it.t);
    const unsigned char *plan = splans + it.slot * PL.bytes;
    const int nrows = plan[PL.off_stage_nrows + it.st];
    const uint16_t *rows =
        reinterpret_cast<const uint16_t *>(plan + PL.off_stage_rows) + it.st * kStageRows;
    uint32_t *dst_base = sbuf + buf * (kStageBytes / 4);
    const uint32_t *gbase = L.planes + (int64_t)L.g * p.d * 4 * L.W;
    for (int id = tid; id < nrows * kChunks; id += kScanThreads) {
      const int slot = id / kChunks, q = id % kChunks;
      const uint32_t *row = gbase + (int64_t)rows[slot] * L.W;
      int64_t gw;
      bool ok;
      if (MODE == kModeSample) {
        const int64_t sj = (int64_t)L.ti * kSampleSectorsPerTile + (q >> 1);
        gw = sj * kSampleStride * kSectorWords + (q & 1) * 4;
        ok = sj < sampled_sectors(L.n) && gw < L.W;
      } else {
        gw = (int64_t)L.ti * kTileWords + q * 4;
        ok = gw < L.W;
      }
      ok = ok && in_bounds(rows[slot] < 4 * p.d && gw >= 0 && gw + 4 <= L.W, p.status);
      cp_async16(dst_base + slot * kTileWords + q * 4,
                 ok ? (const void *)(row + gw) : (const void *)gbase, ok ? 16u : 0u);
    }
  };

  // ---- per-thread scores: 16 tokens x G heads -----------------------------
  // acc[h][i][pp]: .x is byte 2pp and .y byte 2pp+1 of register i, i.e. the
  // tokens at bits 8 (2pp) + 4 half + i and 8 (2pp + 1) + 4 half + i of the word.
  float2 acc[G][4][2];

  auto compute = [&](const Item &it, int buf) {
    const unsigned char *plan = splans + it.slot * PL.bytes;
    const PlanHeader *hdr = reinterpret_cast<const PlanHeader *>(plan);
    if (it.st == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float k0 = hdr->K[h];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[h][i][0] = make_float2(k0, k0);
          acc[h][i][1] = make_float2(k0, k0);
        }
      }
    }
    const uint16_t *stage_begin = reinterpret_cast<const uint16_t *>(plan + PL.off_stage_begin);
    const uint32_t *sb = sbuf + buf * (kStageBytes / 4) + word;
    const int e0 = stage_begin[it.st], e1 = stage_begin[it.st + 1];
    const uint32_t *info = reinterpret_cast<const uint32_t *>(plan + PL.off_info);
    const uint32_t *feats = reinterpret_cast<const uint32_t *>(plan + PL.off_feat);
    const float4 *wts = reinterpret_cast<const float4 *>(plan + PL.off_w);
    for (int e = e0; e < e1; ++e) {
      const uint32_t inf = info[e];
      const int tstar = (inf >> 8) & 7;
      const int slot0 = (inf >> 11) & 31;
      const int nfeat = (inf >> 16) & 7;
      const uint32_t *src = sb + slot0 * kTileWords;
      if (half)
        scan_entry<G, 4>(src, tstar, nfeat, feats[e], wts[e], acc);
      else
        scan_entry<G, 0>(src, tstar, nfeat, feats[e], wts[e], acc);
    }
  };

  auto score_of = [&](int h, int i, int kk) -> float {
    return (kk & 1) ? acc[h][i][kk >> 1].y : acc[h][i][kk >> 1].x;
  };

  // ---- results of a finished tile -------------------------------------------
  auto emit = [&](const Item &it) {
    const TileLoc L = locate<MODE>(p, s_tprefix, it.t);
    const PlanHeader *hdr = reinterpret_cast<const PlanHeader *>(splans + it.slot * PL.bytes);
    const int64_t head0 = (int64_t)L.s * p.h_q + L.g * G;
    const int r0 = 4 * half;
    if (MODE == kModeSample) {
      const int64_t sj = (int64_t)L.ti * kSampleSectorsPerTile + (word >> 3);
      if (sj >= sampled_sectors(L.n)) return;
      const int64_t tok0 = (sj * kSampleStride * kSectorWords + (word & 7)) * 32;
      const int64_t slot0 = sj * 256 + (word & 7) * 32;
      if (!in_bounds(slot0 + 32 <= p.m_max && head0 + G <= (int64_t)p.S * p.h_q, p.status)) return;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        uint32_t *dst = p.sample + (head0 + h) * p.m_max + slot0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int b = 8 * kk + r0 + i;
            dst[b] = (tok0 + b < L.n) ? float_key(score_of(h, i, kk)) : 0u;
          }
      }
      return;
    }
    const int64_t tok0 = ((int64_t)L.ti * kTileWords + word) * 32;
    if (p.debug_scores) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int64_t tok = tok0 + 8 * kk + r0 + i;
            if (tok < L.n) p.debug_scores[(head0 + h) * L.n + tok] = score_of(h, i, kk);
          }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float tau = hdr->tau[h];
      uint32_t m = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int b = 8 * kk + r0 + i;
          m |= ((tok0 + b < L.n) && (score_of(h, i, kk) >= tau) ? 1u : 0u) << (4 * kk + i);
        }
      const int cnt = __popc(m);
      if (__any_sync(0xffffffffu, cnt != 0)) {
        int incl = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int o = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += o;
        }
        unsigned base = 0;
        if (lane == 31) base = atomicAdd(&p.counts[head0 + h], (unsigned)incl);
        base = __shfl_sync(0xffffffffu, base, 31);
        if (cnt) {
          int64_t pos = (int64_t)base + (incl - cnt);
          unsigned long long *dst = p.cand + (head0 + h) * p.cap;
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              if ((m >> (4 * kk + i)) & 1u) {
                if (pos < p.cap)
                  dst[pos] = composite(score_of(h, i, kk), (uint32_t)(tok0 + 8 * kk + r0 + i));
                ++pos;
              }
            }
        }
      }
    }
  };

  // ---- software pipeline over (tile, stage) items ---------------------------
  Item cur = first_item(t_begin, -1, -1);
  Item nxt = next_item(cur, cur.slot, -1);
  issue(cur, 0);
  cp_async_commit();
  issue(nxt, 1);
  cp_async_commit();
  Item iss = next_item(nxt, cur.slot, nxt.slot);
  int it = 0;
  while (true) {
    issue(iss, (it + 2) % kNumBuf);
    cp_async_commit();
    cp_async_wait<2>();
    __syncthreads();
    compute(cur, it % kNumBuf);
    if (cur.st == cur.nst - 1) emit(cur);
    __syncthreads();
    if (nxt.t < 0) break;
    cur = nxt;
    nxt = iss;
    iss = next_item(iss, cur.slot, nxt.slot);
    ++it;
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------- select and sort --

// 64-bit max / min written on 32-bit halves.
__device__ __forceinline__ unsigned long long u64_max(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}
__device__ __forceinline__ unsigned long long u64_min(unsigned long long a, unsigned long long b) {
  return a < b ? a : b;
}

// In-thread stages of the bitonic network for one size (strides 4, 2, 1):
// thread t holds elements base .. base + 7.  For size <= 8 the direction
// depends on the element, for larger sizes only on the thread.
__device__ __forceinline__ void bitonic_regs(unsigned long long (&v)[8], int base, int size) {
#pragma unroll
  for (int st = 4; st >= 1; st >>= 1) {
    if (st * 2 > size) continue;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if ((e & st) == 0) {
        const bool desc = ((base + e) & size) == 0;
        const unsigned long long a = v[e], b = v[e | st];
        const unsigned long long hi = u64_max(a, b), lo = u64_min(a, b);
        v[e] = desc ? hi : lo;
        v[e | st] = desc ? lo : hi;
      }
    }
  }
}

// Sorts s[0 .. m) descending (m a power of two, 256 <= m <= 8 blockDim.x).
// Threads t < m / 8 hold elements 8 t .. 8 t + 7 in registers; the bitonic
// network's exchanges run inside a thread (stride < 8), across lanes with
// shuffles (stride < 256) and through shared memory only for the few
// stages with stride >= 256.  Every thread of the block must call it.
__device__ void block_sort_desc(unsigned long long *s, int m) {
  constexpr int E = 8;
  const int t = threadIdx.x;
  const bool act = t < (m >> 3);
  const int base = t * E;
  unsigned long long v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] = act ? s[base + e] : 0ull;
  for (int size = 2; size <= m; size <<= 1) {
    // strides >= 8: the pair direction depends only on the thread
    for (int stride = size >> 1; stride >= E; stride >>= 1) {
      const bool keep_max = ((base & stride) == 0) == ((base & size) == 0);
      if (stride >= 32 * E) {
        __syncthreads();  // earlier readers of s are done
        if (act) {
#pragma unroll
          for (int e = 0; e < E; ++e) s[base + e] = v[e];
        }
        __syncthreads();
        if (act) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const unsigned long long o = s[(base + e) ^ stride];
            v[e] = keep_max ? u64_max(v[e], o) : u64_min(v[e], o);
          }
        }
      } else if (act) {  // whole warps are idle or active: m / 8 is a multiple of 32
        const int ls = stride / E;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const unsigned long long o = __shfl_xor_sync(0xffffffffu, v[e], ls);
          v[e] = keep_max ? u64_max(v[e], o) : u64_min(v[e], o);
        }
      }
    }
    if (act) bitonic_regs(v, base, size);
  }
  __syncthreads();
  if (act) {
#pragma unroll
    for (int e = 0; e < E; ++e) s[base + e] = v[e];
  }
  __syncthreads();
}

// Histogram select over float scores.  Scores are binned into kSelBins equal
// bins between lo and hi (bin = (score - lo) * scale, monotone in the score).
// block_hist_find returns the highest bin b such that at least `want` scores
// lie in bins >= b (0 if there are fewer), and the count above b in *above.
constexpr int kSelBins = 4096;

__device__ __forceinline__ int sel_bin(float v, float lo, float scale) {
  const int b = (int)((v - lo) * scale);
  return b >= kSelBins ? kSelBins - 1 : b;
}

__device__ int block_hist_find(const unsigned *hist, unsigned want, unsigned *s_wsum, int *s_bin,
                               unsigned *s_above) {
  // warp w sums bins [128 w, 128 w + 128) counted from the top
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  constexpr int kPer = kSelBins / 32;
  if (threadIdx.x == 0) {
    *s_bin = 0;
    *s_above = 0u;
  }
  for (int w = warp; w < 32; w += nw) {
    unsigned loc = 0;
#pragma unroll
    for (int q = 0; q < kPer / 32; ++q) loc += hist[kSelBins - 1 - (w * kPer + q * 32 + lane)];
    loc = __reduce_add_sync(0xffffffffu, loc);
    if (lane == 0) s_wsum[w] = loc;
  }
  __syncthreads();
  if (warp == 0) {
    const unsigned ws = s_wsum[lane];
    unsigned incl = ws;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    const unsigned excl = incl - ws;
    // the range (128 bins) holding the want-th score from the top
    const unsigned own = __ballot_sync(0xffffffffu, excl < want && want <= incl);
    if (own) {
      const int r = __ffs(own) - 1;
      unsigned run = __shfl_sync(0xffffffffu, excl, r);
      // lane l takes bins j = 128 r + 4 l .. 4 l + 3 (from the top)
      unsigned c4[kPer / 32], sum = 0;
#pragma unroll
      for (int q = 0; q < kPer / 32; ++q) {
        c4[q] = hist[kSelBins - 1 - (r * kPer + lane * (kPer / 32) + q)];
        sum += c4[q];
      }
      unsigned in2 = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned o = __shfl_up_sync(0xffffffffu, in2, off);
        if (lane >= off) in2 += o;
      }
      run += in2 - sum;
#pragma unroll
      for (int q = 0; q < kPer / 32; ++q) {
        if (run < want && want <= run + c4[q]) {
          *s_bin = kSelBins - 1 - (r * kPer + lane * (kPer / 32) + q);
          *s_above = run;
        }
        run += c4[q];
      }
    }
  }
  __syncthreads();
  return *s_bin;
}

// Block-wide min and max of (lo, hi) over all threads; every thread gets them.
__device__ __forceinline__ void block_minmax(float &lo, float &hi, float (*s_mm)[32]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
  if (lane == 0) {
    s_mm[0][warp] = lo;
    s_mm[1][warp] = hi;
  }
  __syncthreads();
  lo = s_mm[0][0];
  hi = s_mm[1][0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) {
    lo = fminf(lo, s_mm[0][w]);
    hi = fmaxf(hi, s_mm[1][w]);
  }
  __syncthreads();
}

// ------------------------------------------------------- threshold kernel --

// Warp 0 finds the digit bin holding the want-th largest among 256 bins
// (counted from the top) and the count above it.
__device__ __forceinline__ void find_bin_from_top(const unsigned *hist, unsigned want, int *s_digit,
                                                  unsigned *s_above) {
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < 32) {
    // lane l owns bins 255 - 8l ... 248 - 8l (top first)
    unsigned local[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      local[i] = hist[255 - 8 * lane - i];
      sum += local[i];
    }
    unsigned incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    const unsigned excl = incl - sum;
    if (excl < want && want <= incl) {
      unsigned run = excl;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (run < want && want <= run + local[i]) {
          *s_digit = 255 - 8 * lane - i;
          *s_above = run;
        }
        run += local[i];
      }
    }
  }
}

// Per head: a threshold that at least r of the sampled scores reach.  The
// sampled scores are binned between their min and max; the threshold is the
// smallest sampled score in the bins holding the r best, so it lies at or
// just below the r-th best.  No threshold (0 = keep every key) when fewer
// than r keys were sampled.  Up to kThrKeys keys a thread are held in
// registers (the common case); larger samples are read from memory.
constexpr int kThrKeys = 16;
__global__ void __launch_bounds__(1024) threshold_kernel(ScanParams p) {
  grid_dependency_wait();
  allow_dependent_launch();
  const int64_t h = blockIdx.x;
  const int s = (int)(h / p.h_q);
  const int64_t n = session_n(p, s);
  __shared__ unsigned hist[kSelBins];
  __shared__ unsigned s_wsum[32];
  __shared__ float s_mm[2][32];
  __shared__ int s_bin;
  __shared__ unsigned s_above;
  __shared__ unsigned s_valid;
  __shared__ unsigned s_minkey;
  if (!sampling_on(n, p.sample_rank, p.flags)) {
    if (threadIdx.x == 0) p.tau[h] = 0u;
    return;
  }
  int m = (int)(sampled_sectors(n) * 256);
  if (!in_bounds(m <= p.m_max, p.status)) m = (int)p.m_max;
  const uint32_t *keys = p.sample + h * p.m_max;
  const bool inreg = m <= kThrKeys * (int)blockDim.x;
  // element (j, e) of a thread: key 4 (j blockDim + tid) + e
  uint32_t kk[kThrKeys];
  if (inreg) {
#pragma unroll
    for (int j = 0; j < kThrKeys / 4; ++j) {
      const int b = 4 * (j * (int)blockDim.x + (int)threadIdx.x);
      uint4 u = make_uint4(0u, 0u, 0u, 0u);
      if (b < m) u = *reinterpret_cast<const uint4 *>(keys + b);  // m is a multiple of 256
      kk[4 * j] = u.x;
      kk[4 * j + 1] = u.y;
      kk[4 * j + 2] = u.z;
      kk[4 * j + 3] = u.w;
    }
  }
  for (int i = threadIdx.x; i < kSelBins; i += blockDim.x) hist[i] = 0u;
  if (threadIdx.x == 0) {
    s_valid = 0u;
    s_minkey = 0xffffffffu;
  }
  // range and count of the sampled scores (key 0 = no key sampled there)
  float lo = INFINITY, hi = -INFINITY;
  unsigned valid = 0;
  auto visit = [&](auto &&fn) {
    if (inreg) {
#pragma unroll
      for (int e = 0; e < kThrKeys; ++e)
        if (kk[e] != 0u) fn(kk[e]);
    } else {
      for (int i = threadIdx.x; i < m; i += blockDim.x) {
        const uint32_t x = keys[i];
        if (x != 0u) fn(x);
      }
    }
  };
  visit([&](uint32_t x) {
    const float v = key_float(x);
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
    ++valid;
  });
  valid = __reduce_add_sync(0xffffffffu, valid);
  if ((threadIdx.x & 31) == 0) atomicAdd(&s_valid, valid);
  block_minmax(lo, hi, s_mm);
  if (s_valid < (unsigned)p.sample_rank) {  // too few samples: keep every key
    if (threadIdx.x == 0) p.tau[h] = 0u;
    return;
  }
  const float scale = hi > lo ? (float)kSelBins / (hi - lo) : 0.0f;
  visit([&](uint32_t x) { atomicAdd(&hist[sel_bin(key_float(x), lo, scale)], 1u); });
  __syncthreads();
  const int bstar = block_hist_find(hist, (unsigned)p.sample_rank, s_wsum, &s_bin, &s_above);
  // smallest sampled key in bins >= bstar
  unsigned mk = 0xffffffffu;
  visit([&](uint32_t x) {
    if (sel_bin(key_float(x), lo, scale) >= bstar) mk = min(mk, x);
  });
  mk = __reduce_min_sync(0xffffffffu, mk);
  if ((threadIdx.x & 31) == 0) atomicMin(&s_minkey, mk);
  __syncthreads();
  if (threadIdx.x == 0) p.tau[h] = s_minkey;
}

// ---------------------------------------------------------- merge kernel --

// k-th largest (1-based) of cnt distinct 64-bit composites, k <= cnt.
__device__ unsigned long long block_kth(const unsigned long long *a, int64_t cnt, unsigned k,
                                        unsigned *hist, int *s_digit, unsigned *s_above) {
  unsigned long long prefix = 0ull, pmask = 0ull;
  unsigned want = k;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    if (threadIdx.x == 0) *s_digit = -1;
    __syncthreads();
    for (int64_t base = 0; base < cnt; base += blockDim.x) {
      const int64_t i = base + threadIdx.x;
      int digit = -1;
      if (i < cnt) {
        const unsigned long long v = a[i];
        if ((v & pmask) == prefix) digit = (int)((unsigned)(v >> shift) & 255u);
      }
      hist_add(hist, digit);
    }
    __syncthreads();
    find_bin_from_top(hist, want, s_digit, s_above);
    __syncthreads();
    prefix |= (unsigned long long)(*s_digit) << shift;
    pmask |= 255ull << shift;
    want -= *s_above;
    __syncthreads();
  }
  return prefix;
}

// Exact single-block answer for one head: stream all n keys, score each from
// its allocated prefixes (accumulated in fp64 from the exact products
// q_c s_c, rounded once to fp32), keep a candidate buffer above a running
// k-th best, compact it when it fills.  Under per-token-group statistics the
// keys are streamed group by group, each with its own (m, s).  Used when the
// sampled threshold fails.  Returns the number of buffered candidates
// (= min(k, n)).
__device__ int64_t fallback_head(const ScanParams &p, int s, int hl, unsigned long long *buf,
                                 unsigned long long *s_sort, unsigned *hist, int *s_digit,
                                 unsigned *s_above) {
  const fathom_session &se = session_of(p, s);
  const int d = p.d;
  const int g = hl / p.G;
  const int64_t n = session_n(p, s);
  const int64_t W = plane_words(n);
  __shared__ double s_qs[FATHOM_MAX_D];
  __shared__ uint8_t s_t[FATHOM_MAX_D];
  __shared__ double s_kc[32];
  __shared__ unsigned long long s_nbuf;
  __shared__ unsigned s_fill;
  for (int c = threadIdx.x; c < d; c += blockDim.x) s_t[c] = se.alloc[(int64_t)hl * d + c];
  if (threadIdx.x == 0) s_nbuf = 0;
  const uint32_t *gp = se.planes + (int64_t)g * d * 4 * W;
  unsigned long long theta = 0ull;
  const unsigned k = (unsigned)p.k;
  const int64_t tgk = p.token_group > 0 ? p.token_group : (n > 0 ? n : 1);  // keys per (m, s)
  int tg = 0;
  for (int64_t g0 = 0; g0 < n; g0 += tgk, ++tg) {
    __syncthreads();  // the previous group's s_qs and s_kc are no longer read
    const int64_t srow = ((int64_t)g * p.n_tgroups + tg) * d;
    double kc = 0.0;
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
      const int t = s_t[c];
      const float qv = load_q(se.q, p.q_bf16, (int64_t)hl * d + c);
      const float m = se.qmin[srow + c], sc = se.qscale[srow + c];
      s_qs[c] = (double)qv * (double)sc;  // exact
      const double cell = (double)(1 << (4 - t));
      kc += (double)qv * ((double)m + (double)sc * ((cell - 1.0) * 0.5));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kc += __shfl_xor_sync(0xffffffffu, kc, off);
    if ((threadIdx.x & 31) == 0) s_kc[threadIdx.x >> 5] = kc;
    __syncthreads();
    double ksum = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) ksum += s_kc[w];
    const double K = ksum;
    const int64_t g1 = min(n, g0 + tgk);
    for (int64_t base = g0; base < g1; base += blockDim.x) {
      const int64_t i = base + threadIdx.x;
      if (i < g1) {
        double acc = K;
        for (int c = 0; c < d; ++c) {
          const int t = s_t[c];
          if (t == 0) continue;
          uint32_t y = 0;
          for (int j = 0; j < t; ++j)
            y |= ((gp[((int64_t)c * 4 + j) * W + (i >> 5)] >> (i & 31)) & 1u) << (3 - j);
          acc = fma(s_qs[c], (double)y, acc);
        }
        const unsigned long long v = composite((float)acc, (uint32_t)i);
        if (v > theta) {
          const unsigned long long at = atomicAdd(&s_nbuf, 1ull);
          if (in_bounds((int64_t)at < p.cap, p.status)) buf[at] = v;
        }
      }
      __syncthreads();
      const int64_t nb = (int64_t)s_nbuf;
      if (nb > p.cap - (int64_t)blockDim.x) {
        theta = block_kth(buf, nb, k, hist, s_digit, s_above);
        if (threadIdx.x == 0) s_fill = 0;
        __syncthreads();
        for (int64_t j = threadIdx.x; j < nb; j += blockDim.x)
          if (buf[j] >= theta) {
            const unsigned at = atomicAdd(&s_fill, 1u);
            if (at < k) s_sort[at] = buf[j];
          }
        __syncthreads();
        for (int j = threadIdx.x; j < (int)k; j += blockDim.x) buf[j] = s_sort[j];
        if (threadIdx.x == 0) s_nbuf = k;
        __syncthreads();
        // the k kept are the best so far; a later key matters only above the
        // k-th of them, which is theta
      }
    }
  }
  __syncthreads();
  return (int64_t)s_nbuf;
}

// One block per head (kMergeThreads = 1024 threads).  Usually the
// candidates fit in registers (kMergeKeys a thread): they are binned by score
// (kSelBins equal bins between their min and max, monotone in the score) and
// the bin b holding the k-th best is found.  Candidates sit near the
// threshold, whose upper tail thins out fast, so a bin at or above b holds a
// handful of keys.  They are placed bin by bin from the top (a counting sort); then
// each candidate's place inside its bin is its rank there (the count of
// larger composites in the bin: descending composite = score desc, index
// asc).  The first k are the answer.  Crowded bins fall back to a register
// bitonic sort; more candidates than fit take an exact radix select.
constexpr int kMergeKeys = 8;
constexpr int kBinSortMax = 256;
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(ScanParams p, int kpow2,
                                                              int sort_cap) {
  grid_dependency_wait();
  allow_dependent_launch();
  // union planes of every (session, KV head), from the plan headers: the
  // block of each KV head's first query head adds its group's
  if (threadIdx.x == 0 && blockIdx.x % p.G == 0) {
    const unsigned char *plan =
        p.plans + (size_t)(blockIdx.x / p.G) * p.n_tgroups * p.plan_stride;  // token group 0's
    atomicAdd(&p.status->union_planes,
              (p.flags & FATHOM_FLAG_CUDA_CORES)
                  ? (unsigned)reinterpret_cast<const PlanHeader *>(plan)->union_planes
                  : (unsigned)*reinterpret_cast<const int *>(plan));  // the tc plan's P
  }
  // [sort_cap] placed candidates, then [sort_cap] ranked (sort_cap = 8 blockDim >= kpow2)
  extern __shared__ unsigned long long s_out[];
  unsigned long long *s_rank = s_out + sort_cap;
  __shared__ unsigned hist[kSelBins];
  __shared__ unsigned s_off[kSelBins];
  __shared__ unsigned s_wsum[32];
  __shared__ float s_mm[2][32];
  __shared__ int s_bin;
  __shared__ unsigned s_above;
  __shared__ unsigned s_fill;
  __shared__ int s_crowded;
  const int64_t h = blockIdx.x;
  const int s = (int)(h / p.h_q);
  const int hl = (int)(h - (int64_t)s * p.h_q);
  const fathom_session &se = session_of(p, s);
  const int64_t n = session_n(p, s);
  // a descriptor whose n lies outside [0, n_max] was scanned as empty
  if (hl == 0 && threadIdx.x == 0 && !session_n_valid(p, se.n))
    atomicAdd(&p.status->device_faults, 1u);
  const int k = p.k;
  unsigned long long *buf = p.cand + h * p.cap;
  int64_t cnt = p.counts[h];
  const uint32_t tauk = p.tau[h];
  const int64_t need = n < k ? n : k;
  const bool ok = cnt <= p.cap && (tauk == 0u || cnt >= need) &&
                  !(p.flags & FATHOM_FLAG_FORCE_FALLBACK);
  if (!ok) {
    cnt = fallback_head(p, s, hl, buf, s_out, hist, &s_bin, &s_above);
    if (threadIdx.x == 0) atomicAdd(&p.status->fallback_heads, 1u);
  }
  if (threadIdx.x == 0) {
    atomicMax(&p.status->max_candidates, (unsigned)(cnt < 0xffffffffll ? cnt : 0xffffffffll));
    s_crowded = 0;
  }
  const int take = (int)(cnt < k ? cnt : k);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthr = blockDim.x;
  int nsort = 0;  // > 0: sort s_out[0 .. nsort) with the bitonic network
  if (cnt <= k) {
    for (int i = tid; i < cnt; i += nthr) s_out[i] = buf[i];
    nsort = (int)cnt;
  } else if (cnt <= (int64_t)kMergeKeys * nthr) {
    // candidate j * blockDim + tid of this thread, 0 when absent
    unsigned long long c[kMergeKeys];
    float lo = INFINITY, hi = -INFINITY;
#pragma unroll
    for (int j = 0; j < kMergeKeys; ++j) {
      const int i = j * nthr + tid;
      c[j] = i < cnt ? buf[i] : 0ull;
    }
#pragma unroll
    for (int j = 0; j < kMergeKeys; ++j) {
      if (c[j] != 0ull) {
        const float v = key_float((uint32_t)(c[j] >> 32));
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
      }
    }
    for (int i = tid; i < kSelBins; i += nthr) hist[i] = 0u;
    block_minmax(lo, hi, s_mm);  // its barriers also order the clearing
    const float scale = hi > lo ? (float)kSelBins / (hi - lo) : 0.0f;
    int bin[kMergeKeys];
#pragma unroll
    for (int j = 0; j < kMergeKeys; ++j) {
      bin[j] = -1;
      if (c[j] != 0ull) {
        bin[j] = sel_bin(key_float((uint32_t)(c[j] >> 32)), lo, scale);
        atomicAdd(&hist[bin[j]], 1u);
      }
    }
    __syncthreads();
    int bstar = block_hist_find(hist, (unsigned)k, s_wsum, &s_bin, &s_above);
    // candidates below the k-th best's bin take no further part
#pragma unroll
    for (int j = 0; j < kMergeKeys; ++j)
      if (bin[j] < bstar) bin[j] = -1;
    // exclusive offsets of the bins in top order: thread t owns top-order
    // positions 4 t .. 4 t + 3 (bins kSelBins - 1 - 4 t - q)
    {
      unsigned cq[4], sum = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        cq[q] = hist[kSelBins - 1 - (4 * tid + q)];
        sum += cq[q];
      }
      unsigned incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (lane == 31) s_wsum[warp] = incl;
      __syncthreads();
      unsigned base = incl - sum;
      for (int w = 0; w < warp; ++w) base += s_wsum[w];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        s_off[kSelBins - 1 - (4 * tid + q)] = base;
        base += cq[q];
      }
    }
    __syncthreads();
    // counting-sort placement of the candidates of bins >= bstar
#pragma unroll
    for (int j = 0; j < kMergeKeys; ++j)
      if (bin[j] >= bstar) s_out[atomicAdd(&s_off[bin[j]], 1u)] = c[j];
    __syncthreads();
    // s_off[b] is now the end of bin b's run: rank each candidate in its run
#pragma unroll
    for (int j = 0; j < kMergeKeys; ++j) {
      if (bin[j] >= bstar) {
        const int e = (int)s_off[bin[j]], nb = (int)hist[bin[j]];
        const int b0 = e - nb;
        if (nb > kBinSortMax) {
          s_crowded = 1;
        } else if (b0 < k) {
          int r = 0;
          for (int i = b0; i < e; ++i) r += s_out[i] > c[j] ? 1 : 0;
          s_rank[b0 + r] = c[j];
        }
      }
    }
    __syncthreads();
    if (s_crowded) {
      nsort = (int)s_off[bstar];  // every candidate of bins >= bstar
    } else {
      for (int i = tid; i < take; i += nthr) s_out[i] = s_rank[i];
    }
  } else {
    // more candidates than the registers hold: exact radix select of the k-th
    const unsigned long long bar = block_kth(buf, cnt, (unsigned)k, hist, &s_bin, &s_above);
    if (tid == 0) s_fill = 0u;
    __syncthreads();
    for (int64_t i = tid; i < cnt; i += nthr) {
      const unsigned long long v = buf[i];
      if (v >= bar) {
        const unsigned at = atomicAdd(&s_fill, 1u);
        if (at < (unsigned)take) s_out[at] = v;
      }
    }
    nsort = take;
  }
  if (nsort > 0) {
    int mp = 256;
    while (mp < nsort) mp <<= 1;
    __syncthreads();
    for (int i = nsort + tid; i < mp; i += nthr) s_out[i] = 0ull;
    __syncthreads();
    block_sort_desc(s_out, mp);
  }
  __syncthreads();
  for (int r = tid; r < k; r += nthr) {
    int32_t idx = -1;
    float sc = -INFINITY;
    if (r < take) {
      const unsigned long long v = s_out[r];
      idx = (int32_t)(0xffffffffu - (uint32_t)(v & 0xffffffffull));
      sc = key_float((uint32_t)(v >> 32));
    }
    se.out_idx[(int64_t)hl * k + r] = idx;
    se.out_score[(int64_t)hl * k + r] = sc;
  }
}

// ------------------------------------------------------------- launchers --

// SM count of the current device, cached per device (a process may drive
// several).  Concurrent first calls may both query it and store the same
// value.
static std::atomic<int> g_num_sms[64];

static cudaError_t num_sms(int *out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64) {
    const int cached = g_num_sms[dev].load(std::memory_order_relaxed);
    if (cached > 0) {
      *out = cached;
      return cudaSuccess;
    }
  }
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64) g_num_sms[dev].store(sms, std::memory_order_relaxed);
  *out = sms;
  return cudaSuccess;
}

int scan_smem_bytes(int d, int S) {
  return kNumBuf * kStageBytes + kNumPlanSlots * plan_layout(d).bytes + 4 * (S + 1);
}

template <int G, int MODE>
static cudaError_t launch_scan_gm(const ScanParams &p, cudaStream_t stream) {
  const int smem = scan_smem_bytes(p.d, p.S);
  cudaError_t e = cudaFuncSetAttribute(scan_kernel<G, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, scan_kernel<G, MODE>, kScanThreads,
                                                    smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int sms = 0;
  e = num_sms(&sms);
  if (e != cudaSuccess) return e;
  scan_kernel<G, MODE><<<sms * per_sm, kScanThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int MODE>
static cudaError_t launch_scan_m(const ScanParams &p, cudaStream_t stream) {
  switch (p.G) {
    case 1: return launch_scan_gm<1, MODE>(p, stream);
    case 2: return launch_scan_gm<2, MODE>(p, stream);
    case 4: return launch_scan_gm<4, MODE>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_tc_plan(const ScanParams &p, cudaStream_t stream);
cudaError_t launch_tc_scan(const ScanParams &p, int mode, int sms, cudaStream_t stream);

cudaError_t launch_scan_pipeline(const ScanParams &p, bool any_sampling, cudaStream_t stream) {
  const int heads = p.S * p.h_q;
  int sms = 0;
  cudaError_t e = num_sms(&sms);
  if (e != cudaSuccess) return e;
  const bool tc = (p.flags & FATHOM_FLAG_CUDA_CORES) == 0;
  if (tc) {
    e = launch_tc_plan(p, stream);
  } else {
    e = launch_dependent(plan_kernel, dim3(p.S * p.h_kv), dim3(256), 0, stream, p);
  }
  if (e != cudaSuccess) return e;
  if (any_sampling) {
    e = tc ? launch_tc_scan(p, kModeSample, sms, stream) : launch_scan_m<kModeSample>(p, stream);
    if (e != cudaSuccess) return e;
    e = launch_dependent(threshold_kernel, dim3(heads), dim3(1024), 0, stream, p);
    if (e != cudaSuccess) return e;
  }
  if (p.prof_begin) {
    e = cudaEventRecord(p.prof_begin, stream);
    if (e != cudaSuccess) return e;
  }
  e = tc ? launch_tc_scan(p, kModeFilter, sms, stream) : launch_scan_m<kModeFilter>(p, stream);
  if (e != cudaSuccess) return e;
  if (p.prof_end) {
    e = cudaEventRecord(p.prof_end, stream);
    if (e != cudaSuccess) return e;
  }
  int kpow2 = 256;
  while (kpow2 < p.k) kpow2 <<= 1;
  // the k winners and the k-th best's histogram bin are sorted in registers:
  // up to 8 per thread
  const int sort_cap = 8 * kMergeThreads;
  const int msmem = 2 * sort_cap * 8;
  e = cudaFuncSetAttribute(merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem);
  if (e != cudaSuccess) return e;
  return launch_dependent(merge_kernel, dim3(heads), dim3(kMergeThreads), (size_t)msmem, stream, p,
                          kpow2, sort_cap);
}

}  // namespace fathom
