// Tensor-core form of the Fathom scan for sm_100a (tcgen05, kind::i8).
//
// The score of key i for query head h ("Fathom Makes KV-Cache Scans
// Query-Adaptive for Long-Context Decoding", method paragraphs 2-3; arXiv
// 2609.17652 abstract) is
//   s_h(i) = C_h + sum_{c: t_c > 0} q_c s_c y_{t_c}(i, c),
//   C_h    = sum_c q_c (m_c + s_c (2^(4-t_c) - 1) / 2),
// y_t = the top t bits of the 4-bit code, left-aligned (y_t = 2^(4-t) v_t).
// For the G query heads of one KV head this is a product of two matrices:
//   A [tokens x features], A = y_f(i) in 0..15 (a "feature" is one
//     (channel, prefix length) pair some head of the group reads),
//   B [features x (head, digit)], the weight q_c s_c of a head that reads
//     the feature, as a fixed-point integer W / Delta_h split into four
//     signed base-256 int8 digits (0 for the other heads).
// Integer products accumulate exactly in int32 on the tensor cores
// (tcgen05.mma kind::i8, M = 128 tokens, N = 16 = 4 heads x 4 digits,
// K = 32 features); the epilogue forms s_h = C_h + Delta_h sum_m 256^m acc_m.
//
// Layout (per block, 256 threads, 1024-token tiles):
//  * the union plane rows of a K-chunk are staged with 16-byte cp.async;
//  * every thread rebuilds the 4-bit prefix codes of its word (32 tokens)
//    as bytes in 8 registers and stores them MN-major into the A tile of
//    the chunk; one elected thread issues the 8 MMAs of the chunk and
//    commits them to an mbarrier that releases the A buffer;
//  * the accumulators of a tile (8 M-blocks x 16 columns) live in tensor
//    memory, double-buffered across tiles; after the last chunk of a tile
//    each warp reads its 32 lanes back (tcgen05.ld) and writes samples,
//    candidates or debug scores exactly like the CUDA-core form.
// Every wait on an mbarrier is bounded in time; a timeout records a device
// fault in the workspace status, releases tensor memory and ends the block.
#include "fathom_internal.cuh"

namespace fathom {

// ---------------------------------------------------------------- layout --
constexpr int kTcThreads = 256;
constexpr int kTcTileWords = 32;                      // 1024 tokens per tile
constexpr int kTcMBlocks = kTcTileWords * 32 / 128;   // 8 MMAs of M = 128 per K-chunk
constexpr int kTcKChunk = 32;                         // features per MMA (kind::i8 K)
constexpr int kTcMaxRows = 4 * kTcKChunk;             // plane rows a chunk can need
// A tile (one K-chunk): MN-major, no swizzle.  A core matrix is 16 tokens x
// 8 features (128 B, 16 B per feature row).  MN blocks are 144 B apart and
// K blocks 1152 B apart (the 16 B pads make the 16-byte stores of a warp
// fall on distinct banks); M-blocks are 4624 B apart.
constexpr int kTcSBO_A = 144;
constexpr int kTcLBO_A = 8 * kTcSBO_A;                 // 1152
constexpr int kTcMBlockBytes = 4 * kTcLBO_A + 16;     // 4624
constexpr int kTcABytes = kTcMBlocks * kTcMBlockBytes;  // 36992
// B tile (one K-chunk): K-major, no swizzle, 16 rows (head, digit) x 32
// features: 8-row blocks 128 B apart, 16-feature halves 256 B apart.
constexpr int kTcSBO_B = 128;
constexpr int kTcLBO_B = 256;
constexpr int kTcBBytes = 512;
constexpr int kTcStageBytes = kTcMaxRows * kTcTileWords * 4;  // 16 KiB
constexpr int kTcNumStage = 3;
constexpr int kTcNumPlanSlots = 3;
constexpr int kTcTmemCols = 2 * kTcMBlocks * 16;  // 256: two tiles of accumulators
constexpr int kTcSampleSectorsPerTile = kTcTileWords / kSectorWords;  // 4
// tcgen05 instruction descriptor: D s32, A u8 MN-major, B s8 K-major,
// M = 128, N = 16, dense.
constexpr uint32_t kTcIdesc = (2u << 4)       // D format s32
                              | (0u << 7)     // A format u8
                              | (1u << 10)    // B format s8
                              | (1u << 15)    // A MN-major
                              | (0u << 16)    // B K-major
                              | ((16u >> 3) << 17)   // N
                              | ((128u >> 4) << 24); // M

struct TcPlanHeader {
  int nent;
  int nchunk;
  int union_planes;
  int nrows;
  float K[4];      // C_h
  float delta[4];  // Delta_h (a power of two)
  float tau[4];    // candidate threshold, filled when a block loads the plan
  int pad[4];
};
static_assert(sizeof(TcPlanHeader) == 80, "header size");

struct TcPlanLayout {
  int maxch;
  int off_chunk_entry;  // uint16 [maxch + 1]
  int off_chunk_row;    // uint16 [maxch + 1]
  int off_rows;         // uint16 [4 d]: c * 4 + j of every staged row, by chunk
  int off_info;         // uint32 [d]: t* | nfeat << 3 | kpos0 << 6 | slot0 << 11
  int off_feat;         // uint32 [d]: feature f's prefix length in bits 3f .. 3f+2
  int off_b;            // int8 [maxch][512]
  int bytes;
};

__host__ __device__ inline TcPlanLayout tc_plan_layout(int d) {
  TcPlanLayout L;
  L.maxch = (4 * d) / (kTcKChunk - 3) + 2;
  int o = (int)sizeof(TcPlanHeader);
  L.off_chunk_entry = o;
  o = align16(o + 2 * (L.maxch + 1));
  L.off_chunk_row = o;
  o = align16(o + 2 * (L.maxch + 1));
  L.off_rows = o;
  o = align16(o + 2 * 4 * d);
  L.off_info = o;
  o = align16(o + 4 * d);
  L.off_feat = o;
  o = align16(o + 4 * d);
  L.off_b = o;
  o = align16(o + kTcBBytes * L.maxch);
  L.bytes = o;
  return L;
}

int tc_plan_bytes(int d) { return tc_plan_layout(d).bytes; }

int tc_smem_bytes(int d, int S) {
  return 2 * kTcABytes + kTcNumStage * kTcStageBytes + kTcNumPlanSlots * tc_plan_layout(d).bytes +
         4 * (S + 1) + 64;
}

// --------------------------------------------------------------- helpers --

__device__ __forceinline__ uint32_t tc_smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void tc_cp_async16(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(tc_smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ uint32_t tc_shift(uint32_t x, int s) {
  if (s > 0) return __umulhi(x, 1u << (32 - s));
  if (s < 0) return x * (1u << (-s));
  return x;
}

__device__ __forceinline__ uint64_t tc_smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3fffu) | ((uint64_t)((lbo >> 4) & 0x3fffu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3fffu) << 32) | (1ull << 46);  // version 1, no swizzle
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kTcIdesc), "r"(accumulate), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   mbar)
               : "memory");
}

// Waits for the completion of the mbarrier phase with the given parity, at
// most about two seconds.  Returns false on timeout.
__device__ __forceinline__ bool tc_wait(uint32_t mbar, uint32_t parity) {
  const long long t0 = clock64();
  while (true) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P;\n\t}\n"
        : "=r"(done)
        : "r"(mbar), "r"(parity)
        : "memory");
    if (done) return true;
    if (clock64() - t0 > (1ll << 32)) return false;
  }
}

__device__ __forceinline__ void tc_ld16(uint32_t taddr, int32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}

// int32 -> float for |v| < 2^22, exactly, without the conversion unit.
__device__ __forceinline__ float tc_i2f(int32_t v) {
  return __int_as_float(v + 0x4b400000) - 12582912.0f;
}

__device__ int tc_block_scan(int v, int *s_tmp) {
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

// ------------------------------------------------------------ plan kernel --

// One block of 256 threads per (session, KV head); thread c is channel c.
__global__ void __launch_bounds__(256) tc_plan_kernel(ScanParams p) {
  const int gid = blockIdx.x;
  const int s = gid / p.h_kv;
  const int g = gid - s * p.h_kv;
  const fathom_session &se = session_of(p, s);
  const int d = p.d, G = p.G;
  const int c = threadIdx.x;
  const TcPlanLayout L = tc_plan_layout(d);
  unsigned char *plan = p.plans + (size_t)gid * L.bytes;
  TcPlanHeader *hdr = reinterpret_cast<TcPlanHeader *>(plan);
  uint16_t *chunk_entry = reinterpret_cast<uint16_t *>(plan + L.off_chunk_entry);
  uint16_t *chunk_row = reinterpret_cast<uint16_t *>(plan + L.off_chunk_row);
  uint16_t *rows = reinterpret_cast<uint16_t *>(plan + L.off_rows);
  uint32_t *info = reinterpret_cast<uint32_t *>(plan + L.off_info);
  uint32_t *featw = reinterpret_cast<uint32_t *>(plan + L.off_feat);
  int8_t *bmat = reinterpret_cast<int8_t *>(plan + L.off_b);

  __shared__ int s_tmp[32];
  __shared__ double s_red[4][8];
  __shared__ double s_wmax[4];
  __shared__ uint8_t s_ts[FATHOM_MAX_D], s_nf[FATHOM_MAX_D];
  __shared__ uint8_t s_chunk[FATHOM_MAX_D], s_kpos[FATHOM_MAX_D], s_slot[FATHOM_MAX_D];
  __shared__ int s_nent, s_nchunk;

  // zero the B matrices (unused features and heads must contribute nothing)
  for (int i = threadIdx.x; i < kTcBBytes * L.maxch / 16; i += blockDim.x)
    reinterpret_cast<uint4 *>(bmat)[i] = make_uint4(0, 0, 0, 0);

  int t[4] = {0, 0, 0, 0};
  double w[4] = {0.0, 0.0, 0.0, 0.0};
  double kpart[4] = {0.0, 0.0, 0.0, 0.0};
  int tstar = 0, nfeat = 0;
  uint32_t ftf = 0;  // prefix length of feature f in bits 3f .. 3f+2
  if (c < d) {
    const double m = se.qmin[(int64_t)g * d + c];
    const double sc = se.qscale[(int64_t)g * d + c];
    for (int hh = 0; hh < G; ++hh) {
      const int64_t hq = (int64_t)(g * G + hh) * d + c;
      t[hh] = se.alloc[hq];
      const double qv = load_q(se.q, p.q_bf16, hq);
      tstar = max(tstar, t[hh]);
      w[hh] = t[hh] > 0 ? qv * sc : 0.0;
      const double cell = (double)(1 << (4 - t[hh]));
      kpart[hh] = qv * (m + sc * ((cell - 1.0) * 0.5));
    }
    for (int tf = 1; tf <= 4; ++tf) {
      bool used = false;
      for (int hh = 0; hh < G; ++hh) used |= t[hh] == tf;
      if (used) {
        ftf |= (uint32_t)tf << (3 * nfeat);
        ++nfeat;
      }
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < 4) s_wmax[threadIdx.x] = 0.0;
  __syncthreads();
  for (int hh = 0; hh < 4; ++hh) {
    double v = kpart[hh], a = fabs(w[hh]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      v += __shfl_xor_sync(0xffffffffu, v, off);
      a = fmax(a, __shfl_xor_sync(0xffffffffu, a, off));
    }
    if (lane == 0) {
      s_red[hh][warp] = v;
      // non-negative doubles order like their bit patterns
      atomicMax(reinterpret_cast<unsigned long long *>(&s_wmax[hh]),
                (unsigned long long)__double_as_longlong(a));
    }
  }
  __syncthreads();
  // entry order and the planes before each channel
  const int packed = (tstar > 0 ? 1 : 0) | (tstar << 12);
  const int incl = tc_block_scan(packed, s_tmp);
  const int e = (incl & 0xfff) - 1;
  if (tstar > 0) {
    s_ts[e] = (uint8_t)tstar;
    s_nf[e] = (uint8_t)nfeat;
  }
  if (threadIdx.x == blockDim.x - 1) s_nent = incl & 0xfff;
  __syncthreads();
  const int nent = s_nent;
  // pack whole entries into K-chunks of at most 32 features (serial, <= d entries)
  if (threadIdx.x == 0) {
    int ch = 0, kpos = 0, slot = 0, rowpos = 0;
    chunk_entry[0] = 0;
    chunk_row[0] = 0;
    for (int i = 0; i < nent; ++i) {
      if (kpos + s_nf[i] > kTcKChunk) {
        ++ch;
        chunk_entry[ch] = (uint16_t)i;
        chunk_row[ch] = (uint16_t)rowpos;
        kpos = 0;
        slot = 0;
      }
      s_chunk[i] = (uint8_t)ch;
      s_kpos[i] = (uint8_t)kpos;
      s_slot[i] = (uint8_t)slot;
      kpos += s_nf[i];
      slot += s_ts[i];
      rowpos += s_ts[i];
    }
    const int nchunk = nent > 0 ? ch + 1 : 0;
    chunk_entry[nchunk] = (uint16_t)nent;
    chunk_row[nchunk] = (uint16_t)rowpos;
    s_nchunk = nchunk;
    hdr->nent = nent;
    hdr->nchunk = nchunk;
    hdr->union_planes = rowpos;
    hdr->nrows = rowpos;
    for (int hh = 0; hh < 4; ++hh) {
      double sum = 0.0;
      for (int wv = 0; wv < 8; ++wv) sum += s_red[hh][wv];
      hdr->K[hh] = hh < G ? (float)sum : 0.0f;
      int ex = 0;
      frexp(s_wmax[hh], &ex);  // wmax < 2^ex
      hdr->delta[hh] = s_wmax[hh] > 0.0 ? (float)ldexp(1.0, ex - 30) : 1.0f;
      hdr->tau[hh] = -INFINITY;
    }
    atomicAdd(&p.status->union_planes, (uint32_t)rowpos);
  }
  __syncthreads();
  if (tstar > 0) {
    const int ch = s_chunk[e], kpos0 = s_kpos[e], slot0 = s_slot[e];
    info[e] = (uint32_t)tstar | ((uint32_t)nfeat << 3) | ((uint32_t)kpos0 << 6) |
              ((uint32_t)slot0 << 11);
    featw[e] = ftf;
    const int row0 = chunk_row[ch] + slot0;
    for (int j = 0; j < tstar; ++j) rows[row0 + j] = (uint16_t)(c * 4 + j);
    int8_t *bch = bmat + (size_t)ch * kTcBBytes;
    for (int f = 0; f < nfeat; ++f) {
      const int tf = (ftf >> (3 * f)) & 7;
      const int k = kpos0 + f;
      for (int hh = 0; hh < G; ++hh) {
        if (t[hh] != tf) continue;
        const double delta = (double)hdr->delta[hh];
        long long x = llrint(w[hh] / delta);
        for (int mdig = 0; mdig < 4; ++mdig) {
          const long long dg = ((x + 128) & 255) - 128;
          x = (x - dg) >> 8;
          const int n = 4 * hh + mdig;
          bch[(n >> 3) * kTcSBO_B + (k >> 4) * kTcLBO_B + (n & 7) * 16 + (k & 15)] = (int8_t)dg;
        }
      }
    }
  }
}

// ------------------------------------------------------------ scan kernel --

struct TcLoc {
  int s, g, ti;
  int64_t n, W;
  const uint32_t *planes;
};

template <int MODE>
__device__ __forceinline__ int64_t tc_tiles_per_group(int64_t n, const ScanParams &p) {
  if (MODE == kModeSample) {
    if (!sampling_on(n, p.sample_rank, p.flags)) return 0;
    return (sampled_sectors(n) + kTcSampleSectorsPerTile - 1) / kTcSampleSectorsPerTile;
  }
  return (plane_words(n) + kTcTileWords - 1) / kTcTileWords;
}

template <int MODE>
__device__ __forceinline__ TcLoc tc_locate(const ScanParams &p, const int *s_tprefix, int t) {
  int lo = 0, hi = p.S;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_tprefix[mid] <= t) lo = mid; else hi = mid;
  }
  TcLoc L;
  L.s = lo;
  const fathom_session &se = session_of(p, lo);
  L.n = se.n;
  L.W = plane_words(L.n);
  L.planes = se.planes;
  const int per = (int)tc_tiles_per_group<MODE>(L.n, p);
  const int r = t - s_tprefix[lo];
  L.g = r / per;
  L.ti = r - L.g * per;
  return L;
}

struct TcItem {
  int t;      // tile in the launch's tile space (-1 = none)
  int ch;     // K-chunk of the tile
  int slot;   // plan slot
  int nch;    // chunks of the tile
};

template <int G, int MODE>
__global__ void __launch_bounds__(kTcThreads, 1) tc_scan_kernel(ScanParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int d = p.d;
  const TcPlanLayout PL = tc_plan_layout(d);
  unsigned char *sA = smem;                                  // 2 x kTcABytes
  uint32_t *sStage = reinterpret_cast<uint32_t *>(smem + 2 * kTcABytes);
  unsigned char *sPlans = smem + 2 * kTcABytes + kTcNumStage * kTcStageBytes;
  int *s_tprefix = reinterpret_cast<int *>(sPlans + kTcNumPlanSlots * PL.bytes);
  __shared__ __align__(8) unsigned long long s_mbar[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_tmp[32];
  __shared__ int s_slot_gid[kTcNumPlanSlots];
  __shared__ int s_fault;

  // ---- tile space ----------------------------------------------------------
  for (int base = 0; base < p.S; base += kTcThreads) {
    const int s = base + tid;
    int v = 0;
    if (s < p.S) v = (int)(tc_tiles_per_group<MODE>(session_of(p, s).n, p) * p.h_kv);
    const int carry = base > 0 ? s_tprefix[base] : 0;
    __syncthreads();
    const int incl = tc_block_scan(v, s_tmp);
    if (s < p.S) s_tprefix[s + 1] = carry + incl;
    if (base == 0 && tid == 0) s_tprefix[0] = 0;
    __syncthreads();
  }
  const int total = s_tprefix[p.S];
  const int t_begin = (int)(((int64_t)blockIdx.x * total) / gridDim.x);
  const int t_end = (int)(((int64_t)(blockIdx.x + 1) * total) / gridDim.x);
  if (t_begin >= t_end) return;

  // ---- tensor memory and barriers -----------------------------------------
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     tc_smem_u32(&s_tmem)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(tc_smem_u32(&s_mbar[0])) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(tc_smem_u32(&s_mbar[1])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    s_fault = 0;
  }
  if (tid < kTcNumPlanSlots) s_slot_gid[tid] = -1;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  // ---- plans ---------------------------------------------------------------
  auto ensure_plan = [&](int gid, int busy0, int busy1) -> int {
    int slot = -1;
    for (int i = 0; i < kTcNumPlanSlots; ++i)
      if (s_slot_gid[i] == gid) slot = i;
    if (slot >= 0) return slot;
    for (int i = kTcNumPlanSlots - 1; i >= 0; --i)
      if (i != busy0 && i != busy1) slot = i;
    __syncthreads();
    const uint4 *src = reinterpret_cast<const uint4 *>(p.plans + (size_t)gid * PL.bytes);
    uint4 *dst = reinterpret_cast<uint4 *>(sPlans + slot * PL.bytes);
    for (int i = tid; i < PL.bytes / 16; i += kTcThreads) dst[i] = src[i];
    tc_fence_proxy_async();  // the B tiles are read by the tensor cores
    __syncthreads();
    if (tid < G) {
      TcPlanHeader *hdr = reinterpret_cast<TcPlanHeader *>(sPlans + slot * PL.bytes);
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
  auto first_item = [&](int t, int busy0, int busy1) -> TcItem {
    TcItem it;
    it.t = t;
    it.ch = 0;
    if (t >= t_end) {
      it.t = -1;
      it.slot = -1;
      it.nch = 0;
      return it;
    }
    const TcLoc L = tc_locate<MODE>(p, s_tprefix, t);
    it.slot = ensure_plan(L.s * p.h_kv + L.g, busy0, busy1);
    const int nch = reinterpret_cast<const TcPlanHeader *>(sPlans + it.slot * PL.bytes)->nchunk;
    it.nch = nch > 0 ? nch : 1;  // a head with no bits still needs its constant scores
    return it;
  };
  auto next_item = [&](const TcItem &a, int busy0, int busy1) -> TcItem {
    if (a.t < 0) return a;
    if (a.ch + 1 < a.nch) {
      TcItem b = a;
      b.ch += 1;
      return b;
    }
    return first_item(a.t + 1, busy0, busy1);
  };

  // ---- staged copies of a chunk's rows ------------------------------------
  auto issue = [&](const TcItem &it, int buf) {
    if (it.t < 0) return;
    const TcLoc L = tc_locate<MODE>(p, s_tprefix, it.t);
    const unsigned char *plan = sPlans + it.slot * PL.bytes;
    const TcPlanHeader *hdr = reinterpret_cast<const TcPlanHeader *>(plan);
    if (hdr->nchunk == 0) return;
    const uint16_t *chunk_row = reinterpret_cast<const uint16_t *>(plan + PL.off_chunk_row);
    const uint16_t *rows = reinterpret_cast<const uint16_t *>(plan + PL.off_rows);
    const int r0 = chunk_row[it.ch], nrows = chunk_row[it.ch + 1] - r0;
    uint32_t *dst_base = sStage + buf * (kTcStageBytes / 4);
    const uint32_t *gbase = L.planes + (int64_t)L.g * d * 4 * L.W;
    for (int id = tid; id < nrows * 8; id += kTcThreads) {
      const int slot = id >> 3, q = id & 7;
      const uint32_t *row = gbase + (int64_t)rows[r0 + slot] * L.W;
      int64_t gw;
      bool ok;
      if (MODE == kModeSample) {
        const int64_t sj = (int64_t)L.ti * kTcSampleSectorsPerTile + (q >> 1);
        gw = sj * kSampleStride * kSectorWords + (q & 1) * 4;
        ok = sj < sampled_sectors(L.n) && gw < L.W;
      } else {
        gw = (int64_t)L.ti * kTcTileWords + q * 4;
        ok = gw < L.W;
      }
      tc_cp_async16(dst_base + slot * kTcTileWords + q * 4,
                    ok ? (const void *)(row + gw) : (const void *)row, ok ? 16u : 0u);
    }
  };

  // ---- build the A tile of one chunk ---------------------------------------
  // Thread (warp w, lane l) owns word l of the tile and the chunk's entries
  // e = w, w + 8, ...  Register R[r], byte kk = the prefix code y (0..15) of
  // token 32 l + 8 kk + r; {R0..R3} and {R4..R7} are the 16-token MN rows
  // 2 (l % 4) and 2 (l % 4) + 1 of M-block l / 4.
  auto build = [&](const TcItem &it, int sbuf, int abuf) {
    const unsigned char *plan = sPlans + it.slot * PL.bytes;
    const TcPlanHeader *hdr = reinterpret_cast<const TcPlanHeader *>(plan);
    if (hdr->nchunk == 0) return;
    const uint16_t *chunk_entry = reinterpret_cast<const uint16_t *>(plan + PL.off_chunk_entry);
    const uint32_t *info = reinterpret_cast<const uint32_t *>(plan + PL.off_info);
    const uint32_t *featw = reinterpret_cast<const uint32_t *>(plan + PL.off_feat);
    const uint32_t *src_base = sStage + sbuf * (kTcStageBytes / 4) + lane;
    unsigned char *a_base = sA + abuf * kTcABytes + (lane >> 2) * kTcMBlockBytes +
                            (2 * (lane & 3)) * kTcSBO_A;
    const int e0 = chunk_entry[it.ch], e1 = chunk_entry[it.ch + 1];
    for (int e = e0 + warp; e < e1; e += kTcThreads / 32) {
      const uint32_t inf = info[e];
      const int tstar = inf & 7;
      const int nfeat = (inf >> 3) & 7;
      const int kpos0 = (inf >> 6) & 31;
      const int slot0 = (inf >> 11) & 127;
      const uint32_t *src = src_base + slot0 * kTcTileWords;
      uint32_t R[8];
      const uint32_t p0 = src[0];
#pragma unroll
      for (int r = 0; r < 8; ++r) R[r] = tc_shift(p0, r - 3) & 0x08080808u;
      if (tstar > 1) {
        const uint32_t p1 = src[kTcTileWords];
#pragma unroll
        for (int r = 0; r < 8; ++r) R[r] |= tc_shift(p1, r - 2) & 0x04040404u;
        if (tstar > 2) {
          const uint32_t p2 = src[2 * kTcTileWords];
#pragma unroll
          for (int r = 0; r < 8; ++r) R[r] |= tc_shift(p2, r - 1) & 0x02020202u;
          if (tstar > 3) {
            const uint32_t p3 = src[3 * kTcTileWords];
#pragma unroll
            for (int r = 0; r < 8; ++r) R[r] |= p3 >> r & 0x01010101u;
          }
        }
      }
      const uint32_t fw = featw[e];
      for (int f = 0; f < nfeat; ++f) {
        const int tf = (fw >> (3 * f)) & 7;
        // keep the top tf bits of every 4-bit code: bits 3 .. 4 - tf of each byte
        const uint32_t keep = (((1u << tf) - 1u) << (4 - tf)) * 0x01010101u;
        const int k = kpos0 + f;
        unsigned char *dst = a_base + (k >> 3) * kTcLBO_A + (k & 7) * 16;
        *reinterpret_cast<uint4 *>(dst) =
            make_uint4(R[0] & keep, R[1] & keep, R[2] & keep, R[3] & keep);
        *reinterpret_cast<uint4 *>(dst + kTcSBO_A) =
            make_uint4(R[4] & keep, R[5] & keep, R[6] & keep, R[7] & keep);
      }
    }
  };

  // ---- the tile's results ----------------------------------------------------
  // A tile's accumulators are read one item after its last chunk (so the
  // MMAs complete while the next chunk is being built); what the epilogue
  // needs from the plan is copied here first, since the plan slot may be
  // reused by then.
  struct Pending {
    int t, accbuf, has_mma, item;
    float K[G], D[G], tau[G];
  };
  auto make_pending = [&](const TcItem &it, int accbuf, int item) -> Pending {
    const TcPlanHeader *hdr = reinterpret_cast<const TcPlanHeader *>(sPlans + it.slot * PL.bytes);
    Pending pd;
    pd.t = it.t;
    pd.accbuf = accbuf;
    pd.has_mma = hdr->nchunk > 0;
    pd.item = item;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      pd.K[h] = hdr->K[h];
      pd.D[h] = hdr->delta[h];
      pd.tau[h] = hdr->tau[h];
    }
    return pd;
  };
  auto epilogue = [&](const Pending &pd) {
    const TcLoc L = tc_locate<MODE>(p, s_tprefix, pd.t);
    const int64_t head0 = (int64_t)L.s * p.h_q + L.g * G;
    const int quarter = warp & 3;
    // row 32 quarter + lane of M-block b is token 32 (4 b + quarter) + 8 kk + r
    const int kk = lane & 3, r = 4 * (lane >> 4) + ((lane >> 2) & 3);
#pragma unroll
    for (int j = 0; j < kTcMBlocks / 2; ++j) {
      const int b = 2 * j + (warp >> 2);
      float sc[G];
      if (pd.has_mma) {
        int32_t v[16];
        tc_ld16(tmem + ((uint32_t)(32 * quarter) << 16) +
                    (uint32_t)(pd.accbuf * kTcMBlocks * 16 + b * 16),
                v);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float sum = tc_i2f(v[4 * h + 3]);
          sum = fmaf(sum, 256.0f, tc_i2f(v[4 * h + 2]));
          sum = fmaf(sum, 256.0f, tc_i2f(v[4 * h + 1]));
          sum = fmaf(sum, 256.0f, tc_i2f(v[4 * h + 0]));
          sc[h] = fmaf(pd.D[h], sum, pd.K[h]);
        }
      } else {
#pragma unroll
        for (int h = 0; h < G; ++h) sc[h] = pd.K[h];
      }
      const int wl = 4 * b + quarter;   // word of the tile
      const int bit = 8 * kk + r;       // token bit within the word
      if (MODE == kModeSample) {
        const int64_t sj = (int64_t)L.ti * kTcSampleSectorsPerTile + (wl >> 3);
        if (sj < sampled_sectors(L.n)) {
          const int64_t tok = (sj * kSampleStride * kSectorWords + (wl & 7)) * 32 + bit;
          const int64_t sl = sj * 256 + (wl & 7) * 32 + bit;
#pragma unroll
          for (int h = 0; h < G; ++h)
            p.sample[(head0 + h) * p.m_max + sl] = tok < L.n ? float_key(sc[h]) : 0u;
        }
      } else {
        const int64_t tok = ((int64_t)L.ti * kTcTileWords + wl) * 32 + bit;
        const bool valid = tok < L.n;
        if (p.debug_scores && valid) {
#pragma unroll
          for (int h = 0; h < G; ++h) p.debug_scores[(head0 + h) * L.n + tok] = sc[h];
        }
        bool take[G], any = false;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          take[h] = valid && sc[h] >= pd.tau[h];
          any |= take[h];
        }
        if (__any_sync(0xffffffffu, any)) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const unsigned ballot = __ballot_sync(0xffffffffu, take[h]);
            if (ballot) {
              unsigned base = 0;
              if (lane == 0) base = atomicAdd(&p.counts[head0 + h], (unsigned)__popc(ballot));
              base = __shfl_sync(0xffffffffu, base, 0);
              if (take[h]) {
                const unsigned pos = base + __popc(ballot & ((1u << lane) - 1u));
                if ((int64_t)pos < p.cap)
                  p.cand[(head0 + h) * p.cap + pos] = composite(sc[h], (uint32_t)tok);
              }
            }
          }
        }
      }
    }
  };

  // ---- pipeline over (tile, chunk) items -----------------------------------
  const uint32_t mbar0 = tc_smem_u32(&s_mbar[0]);
  TcItem cur = first_item(t_begin, -1, -1);
  TcItem nxt = next_item(cur, cur.slot, -1);
  issue(cur, 0);
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  issue(nxt, 1);
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  TcItem iss = next_item(nxt, cur.slot, nxt.slot);
  int it = 0, tile_seq = 0;
  bool fault = false, pending = false;
  Pending pd;
  while (true) {
    issue(iss, (it + 2) % kTcNumStage);
    asm volatile("cp.async.commit_group;\n" ::: "memory");
    asm volatile("cp.async.wait_group 2;\n" ::: "memory");
    const int abuf = it & 1;
    // the MMAs that last read this A buffer (item it - 2) must have finished
    if (it >= 2 && !tc_wait(mbar0 + 8 * abuf, ((it - 2) >> 1) & 1)) s_fault = 1;
    __syncthreads();
    if (s_fault) {
      fault = true;
      break;
    }
    build(cur, it % kTcNumStage, abuf);
    tc_fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    const unsigned char *plan = sPlans + cur.slot * PL.bytes;
    const bool has_mma = reinterpret_cast<const TcPlanHeader *>(plan)->nchunk > 0;
    if (tid == 0) {
      tc_fence_after();
      if (has_mma) {
        const uint32_t a_addr = tc_smem_u32(sA + abuf * kTcABytes);
        const uint32_t b_addr = tc_smem_u32(plan + PL.off_b + cur.ch * kTcBBytes);
        const uint64_t bdesc = tc_smem_desc(b_addr, kTcLBO_B, kTcSBO_B);
#pragma unroll 1
        for (int mb = 0; mb < kTcMBlocks; ++mb) {
          const uint64_t adesc = tc_smem_desc(a_addr + mb * kTcMBlockBytes, kTcLBO_A, kTcSBO_A);
          tc_mma(tmem + (uint32_t)((tile_seq & 1) * kTcMBlocks * 16 + mb * 16), adesc, bdesc,
                 cur.ch > 0 ? 1u : 0u);
        }
      }
      tc_commit(mbar0 + 8 * abuf);  // also when empty: keeps the barrier phases in step
    }
    // results of the previous tile, whose MMAs ran while this chunk was built
    if (pending) {
      if (tc_wait(mbar0 + 8 * (pd.item & 1), (pd.item >> 1) & 1)) {
        tc_fence_after();
        epilogue(pd);
        tc_fence_before();
      } else {
        s_fault = 1;
      }
      pending = false;
    }
    if (cur.ch == cur.nch - 1) {
      pd = make_pending(cur, tile_seq & 1, it);
      pending = true;
      ++tile_seq;
    }
    __syncthreads();
    if (nxt.t < 0) break;
    cur = nxt;
    nxt = iss;
    iss = next_item(iss, cur.slot, nxt.slot);
    ++it;
  }
  if (pending && !fault) {
    if (tc_wait(mbar0 + 8 * (pd.item & 1), (pd.item >> 1) & 1)) {
      tc_fence_after();
      epilogue(pd);
    } else {
      s_fault = 1;
    }
  }
  __syncthreads();
  if (s_fault) fault = true;
  asm volatile("cp.async.wait_all;\n" ::: "memory");
  if (fault && tid == 0) atomicAdd(&p.status->device_faults, 1u);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                 "r"(kTcTmemCols)
                 : "memory");
  }
}

// ------------------------------------------------------------- launchers --

template <int G, int MODE>
static cudaError_t launch_tc_gm(const ScanParams &p, int sms, cudaStream_t stream) {
  const int smem = tc_smem_bytes(p.d, p.S);
  cudaError_t e = cudaFuncSetAttribute(tc_scan_kernel<G, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // one block per SM: each block holds 256 tensor-memory columns and more
  // than half of the shared memory
  tc_scan_kernel<G, MODE><<<sms, kTcThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_tc_plan(const ScanParams &p, cudaStream_t stream) {
  tc_plan_kernel<<<p.S * p.h_kv, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_tc_scan(const ScanParams &p, int mode, int sms, cudaStream_t stream) {
  if (mode == kModeSample) {
    switch (p.G) {
      case 1: return launch_tc_gm<1, kModeSample>(p, sms, stream);
      case 2: return launch_tc_gm<2, kModeSample>(p, sms, stream);
      case 4: return launch_tc_gm<4, kModeSample>(p, sms, stream);
    }
  } else {
    switch (p.G) {
      case 1: return launch_tc_gm<1, kModeFilter>(p, sms, stream);
      case 2: return launch_tc_gm<2, kModeFilter>(p, sms, stream);
      case 4: return launch_tc_gm<4, kModeFilter>(p, sms, stream);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace fathom
