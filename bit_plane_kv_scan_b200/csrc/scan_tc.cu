// Tensor-core form of the Fathom scan for sm_100a (tcgen05.mma kind::i8,
// A operand in tensor memory).
//
// The score of key i for query head h ("Fathom Makes KV-Cache Scans
// Query-Adaptive for Long-Context Decoding", method paragraphs 2-3; arXiv
// 2609.17652 abstract) is a sum over the bit planes the head reads:
//   s_h(i) = C_h + sum_{(c, j): j < t_hc} W_hcj b_cj(i),   W_hcj = q_hc s_c 2^(3 - j),
//   C_h    = sum_c q_hc (m_c + s_c (2^(4 - t_hc) - 1) / 2),
// b_cj(i) the bit of plane j of channel c for key i.  For the G query heads of
// one KV head this is one matrix product over the P union planes of the group:
//   A [keys x planes] = the plane bits,
//   B [planes x (head, digit)] = W_hcj / Delta_h as a 30-bit fixed-point
//     integer in four signed base-256 int8 digits (0 where the head does not
//     read the plane),
// accumulated exactly in int32 by the tensor cores; the epilogue forms
//   s_h = C_h + Delta_h sum_m 256^m acc_m.
//
// Layout (B200 design).  A tile is 1024 keys of one KV head: 32 plane words
// per plane.  Tensor-memory lane (quarter q, lane l) of M-block r (r < 8)
// stands for key 32 l + 8 q + r of the tile: word l, byte q, bit r.  Plane
// rows are taken four at a time, and byte q of the four rows' word l forms
//   T = [x0.byte q, x1.byte q, x2.byte q, x3.byte q];
// M-block r receives the 32-bit cell T & (0x01010101 << r): four int8 K
// elements, one per plane, each 0 or 2^r (undone by the epilogue's scale).
// Every key has its own row and B has N = 16 columns (head, digit).
//
// Work split (measured on B200: one thread issues a tcgen05.mma only every
// ~46 cycles, a tcgen05.commit reaches its mbarrier ~800 cycles after issue,
// and bulk copies of 128-byte row pieces are limited by their per-copy cost).
// The K-steps (32 union planes of one tile) of a run of tiles are taken two at
// a time as a chunk, so only a tile's last K-step can be part padding.
//  * Load warps 0-3: thread (plane group i, word quad m) loads four plane rows
//    of the chunk with 16-byte global loads (three chunks ahead in
//    registers; row addresses from a per-segment offset table), transposes
//    the bytes so that T = [x0.q, x1.q, x2.q, x3.q] for each lane quarter q,
//    and stores them in a four-stage shared-memory ring, where a build warp
//    reads its T values conflict-free.  One elected lane of load warp l also
//    issues the MMAs of M-blocks 2 l and 2 l + 1, five chunks behind its
//    loads: four issuers, every accumulator region always fed by the same
//    thread.
//  * Build warps 4-11 (lane quarter w % 4, group g = M-blocks 4 g .. 4 g + 3)
//    write the cells of their M-blocks for both K-steps to tensor memory (two
//    32-column stores) and signal them one chunk later, after reading the
//    next stage, so that the stores have that long to land.
//  * Epilogue warps 12-19 (lane quarter, half: four M-blocks each) read a
//    finished tile's accumulators back, score, and collect the keys above
//    the head's threshold in shared memory, flushing them to the candidate
//    buffer with one global atomic per flush.
// Stages, A buffers (two) and accumulators (two) are handed over with
// mbarriers.
// Accumulators are preset to the bits of 1.5 * 2^23, so that an accumulator
// read back as a float is 1.5 * 2^23 + acc exactly (|acc| <= 2^22).  When
// P > 256 the cells hold 0/1 instead of 0/2^r so that acc stays within 2^22.
// Every mbarrier wait is bounded in time; a timeout records a device fault in
// the workspace status.
#include "fathom_internal.cuh"

namespace fathom {

// ---------------------------------------------------------------- layout --
constexpr int kTcTileWords = 32;                        // 1024 keys per tile
constexpr int kTcChunkPlanes = 64;                      // plane rows per chunk
constexpr int kTcKStep = 32;                            // planes per MMA (K = 32 int8)
constexpr int kTcStageBytes = kTcChunkPlanes * kTcTileWords * 4;  // 8 KiB
constexpr int kTcLoadWarps = 4;                         // warps 0-3
constexpr int kTcBuildWarp0 = 4;                        // warps 4-11
constexpr int kTcBuildWarps = 8;
constexpr int kTcEpiWarp0 = 12;                         // warps 12-19
constexpr int kTcEpiWarps = 8;                          // two per lane quarter
constexpr int kTcThreads = (kTcLoadWarps + kTcBuildWarps + kTcEpiWarps) * 32;
constexpr int kTcStages = 4;                            // staged chunks in shared memory
constexpr int kTcRing = 3;                              // chunks a load thread holds in registers
constexpr int kTcMBlocks = 8;                           // one per bit position r
constexpr int kTcN = 16;                                // (head, digit) columns
constexpr int kTcAccCols = kTcMBlocks * kTcN;           // 128: one tile's accumulators
constexpr int kTcABufCols = kTcMBlocks * (kTcChunkPlanes / 4);  // 128: one chunk's cells
constexpr int kTcTmemCols = 512;                        // 2 x 128 accumulators + 2 x 128 A
constexpr int kTcAColBase = 2 * kTcAccCols;
constexpr int kTcSampleSectorsPerTile = kTcTileWords / kSectorWords;  // 4
constexpr int kTcCandBuf = 64;                          // candidates buffered per epilogue warp and head
// B for one K-step: 16 rows (head, digit) x 32 int8 K elements (planes),
// K-major, no swizzle.  Core matrices are 8 rows x 16 bytes; the two 8-row
// groups are 128 B apart (SBO), the two 16-byte K halves 256 B apart (LBO).
constexpr int kTcBChunkBytes = 512;  // per K-step of 32 planes
constexpr uint32_t kTcSBO = 128;
constexpr uint32_t kTcLBO = 256;
// Instruction descriptor: D s32, A u8 K-major (tensor memory), B s8
// K-major, N = 16, M = 128, dense.
constexpr uint32_t kTcIdesc = (2u << 4)                 // D format s32
                              | (0u << 7)               // A format u8
                              | (1u << 10)              // B format s8
                              | (0u << 15)              // A K-major
                              | (0u << 16)              // B K-major
                              | ((uint32_t)(kTcN >> 3) << 17)  // N
                              | ((128u >> 4) << 24);    // M
constexpr uint32_t kTcMagicBits = 0x4b400000u;  // 1.5 * 2^23
constexpr float kTcMagic = 12582912.0f;
// A plane count above which the cells hold 0/1 instead of 0/2^r, so that an
// accumulator stays within 2^22 (|digit| <= 128, 2^r <= 128).
constexpr int kTcSmallP = 256;

struct TcPlanHeader {
  int P;       // union planes of the group
  int nks;     // max(1, ceil(P / 32)): K-steps of 32 planes with a B block
  int pad0, pad1;
  float K[4];  // C_h
  float D[4];  // Delta_h (a power of two)
  float pad2[4];
};
static_assert(sizeof(TcPlanHeader) == 64, "header size");

struct TcPlanLayout {
  int off_rows;  // uint16 [4 d]: c * 4 + j of every union plane, channel-major
  int off_b;     // int8 [ceil(4 d / 32)][512]: B of every K-step
  int bytes;
};

__host__ __device__ inline TcPlanLayout tc_plan_layout(int d) {
  TcPlanLayout L;
  L.off_rows = (int)sizeof(TcPlanHeader);
  L.off_b = align16(L.off_rows + 2 * 4 * d);
  L.bytes = L.off_b + ((4 * d + kTcKStep - 1) / kTcKStep) * kTcBChunkBytes;
  return L;
}

int tc_plan_bytes(int d) { return tc_plan_layout(d).bytes; }

// Row offset table: one entry per union plane row, padded to whole K-steps.
__host__ __device__ inline int tc_off_bytes(int d) {
  return align16(4 * (((4 * d + kTcKStep - 1) / kTcKStep) * kTcKStep));
}

static int tc_smem_bytes(int d, int S) {
  int b = 128 + kTcStages * kTcStageBytes + tc_off_bytes(d) + tc_plan_layout(d).bytes +
          4 * (S + 1) + kTcEpiWarps * 4 * kTcCandBuf * 8;
  // more than half an SM's shared memory: one block per SM, so that the
  // block's 512 tensor-memory columns never wait for another block
  return b < 120 * 1024 ? 120 * 1024 : b;
}

// --------------------------------------------------------------- helpers --

__device__ __forceinline__ uint32_t tc_smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
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

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}\n" ::"r"(bar)
      : "memory");
}

// Waits for the completion of the phase of bar with the given parity, giving
// up after about a second (2^31 cycles).  Returns false on timeout.  Each
// try_wait may suspend the thread for a system-dependent time until the phase
// completes (an explicit suspend-time hint measured slower on B200).
// Non-blocking probe of the phase.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (clock64() - t0 > (1ll << 31)) return false;
  }
}

// Named barrier among the `count` threads of the build warps.
__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(kTcIdesc), "r"(1u)
      : "memory");
}

// One lane of the (converged) warp: the lowest.
__device__ __forceinline__ bool tc_elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n\t.reg .pred P;\n\t.reg .b32 R;\n\t"
      "elect.sync R|P, 0xffffffff;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}\n"
      : "=r"(pred));
  return pred != 0;
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
      : "memory");
}

__device__ __forceinline__ void tc_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};\n" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tc_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
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
  const TcPlanLayout L = tc_plan_layout(d);
  unsigned char *plan = p.plans + (size_t)gid * L.bytes;
  TcPlanHeader *hdr = reinterpret_cast<TcPlanHeader *>(plan);
  uint16_t *rows = reinterpret_cast<uint16_t *>(plan + L.off_rows);
  int8_t *bmat = reinterpret_cast<int8_t *>(plan + L.off_b);

  __shared__ int s_tmp[32];
  __shared__ double s_red[4][8];
  __shared__ unsigned long long s_wmax[4];
  __shared__ int s_P;

  int t[4] = {0, 0, 0, 0};
  double w[4] = {0.0, 0.0, 0.0, 0.0};      // q_c s_c of a head that reads channel c
  double kpart[4] = {0.0, 0.0, 0.0, 0.0};  // its share of C_h
  int tstar = 0;
  if (c < d) {
    const double m = se.qmin[(int64_t)g * d + c];
    const double sc = se.qscale[(int64_t)g * d + c];
    // fixed trip count, so that t, w and kpart stay in registers
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) {
      if (hh >= G) break;
      const int64_t hq = (int64_t)(g * G + hh) * d + c;
      t[hh] = se.alloc[hq];
      const double qv = load_q(se.q, p.q_bf16, hq);
      tstar = max(tstar, t[hh]);
      w[hh] = t[hh] > 0 ? qv * sc : 0.0;
      const double cell = (double)(1 << (4 - t[hh]));
      kpart[hh] = qv * (m + sc * ((cell - 1.0) * 0.5));
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < 4) s_wmax[threadIdx.x] = 0ull;
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
      atomicMax(&s_wmax[hh], (unsigned long long)__double_as_longlong(a));
    }
  }
  // the union planes of channel c are rows off .. off + t* - 1 of the plan
  const int incl = tc_block_scan(tstar, s_tmp);
  const int off = incl - tstar;
  if (threadIdx.x == blockDim.x - 1) s_P = incl;
  __syncthreads();
  const int P = s_P;
  const int nks = P > 0 ? (P + kTcKStep - 1) / kTcKStep : 1;
  // B of every used K-step starts at zero (padding planes and heads that do
  // not read a plane contribute nothing)
  for (int i = threadIdx.x; i < nks * kTcBChunkBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4 *>(bmat)[i] = make_uint4(0, 0, 0, 0);
  double delta[4], inv_delta[4];
#pragma unroll
  for (int hh = 0; hh < 4; ++hh) {
    // the largest plane weight is 8 max_c |q_c s_c|; W / Delta < 2^30
    const double wmax = 8.0 * __longlong_as_double((long long)s_wmax[hh]);
    int ex = 0;
    frexp(wmax, &ex);  // wmax < 2^ex
    delta[hh] = wmax > 0.0 ? ldexp(1.0, ex - 30) : 1.0;
    inv_delta[hh] = wmax > 0.0 ? ldexp(1.0, 30 - ex) : 1.0;  // exact: a power of two
  }
  if (threadIdx.x == 0) {
    hdr->P = P;
    hdr->nks = nks;
    hdr->pad0 = hdr->pad1 = 0;
    const int nw = (blockDim.x + 31) >> 5;
    for (int hh = 0; hh < 4; ++hh) {
      double sum = 0.0;
      for (int wv = 0; wv < nw; ++wv) sum += s_red[hh][wv];
      hdr->K[hh] = hh < G ? (float)sum : 0.0f;
      hdr->D[hh] = (float)delta[hh];
      hdr->pad2[hh] = 0.0f;
    }
  }
  __syncthreads();
  for (int j = 0; j < tstar; ++j) {
    const int pl = off + j;
    rows[pl] = (uint16_t)(c * 4 + j);
    int8_t *bk = bmat + (size_t)(pl / kTcKStep) * kTcBChunkBytes;
    const int k = pl % kTcKStep;
    const double pj = (double)(1 << (3 - j));  // 2^(3 - j), j <= 3
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) {
      if (hh >= G || j >= t[hh]) continue;
      // W / Delta scaled by powers of two only: exact, then rounded once
      long long x = __double2ll_rn(w[hh] * pj * inv_delta[hh]);
#pragma unroll
      for (int dg = 0; dg < 4; ++dg) {
        const long long v = dg < 3 ? ((x + 128) & 255) - 128 : x;
        x = (x - v) >> 8;
        const int n = hh * 4 + dg;
        bk[(n >> 3) * kTcSBO + (k >> 4) * kTcLBO + (n & 7) * 16 + (k & 15)] = (int8_t)v;
      }
    }
  }
}

// ------------------------------------------------------------ scan kernel --

template <int MODE>
__device__ __forceinline__ int64_t tc_tiles_per_group(int64_t n, const ScanParams &p) {
  if (MODE == kModeSample) {
    if (!sampling_on(n, p.sample_rank, p.flags)) return 0;
    return (sampled_sectors(n) + kTcSampleSectorsPerTile - 1) / kTcSampleSectorsPerTile;
  }
  return (plane_words(n) + kTcTileWords - 1) / kTcTileWords;
}

struct TcLoc {
  int s, g, ti, per;
  int64_t n, W;
  const uint32_t *planes;
};

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
  L.per = (int)tc_tiles_per_group<MODE>(L.n, p);
  const int r = t - s_tprefix[lo];
  L.g = r / L.per;
  L.ti = r - L.g * L.per;
  return L;
}

// A block whose tiles span two (session, KV head) groups drains its pipeline
// between them (measured: about 2.5 tiles of work).  The filtering pass
// splits the tiles over the blocks on a cost line on which every group is
// preceded by that overhead, so that a block that crosses a group boundary
// takes correspondingly fewer tiles.  Costs are in half tiles.
constexpr int kTcSwitchHalfTiles = 5;

// Cost position of global tile k: 2 k + sw (groups up to and including k's).
template <int MODE>
__device__ __forceinline__ int64_t tc_cost_pos(const ScanParams &p, const int *s_tprefix, int k,
                                               int64_t sw) {
  int lo = 0, hi = p.S;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_tprefix[mid] <= k) lo = mid; else hi = mid;
  }
  const int per = (int)tc_tiles_per_group<MODE>(session_of(p, lo).n, p);
  const int64_t group = (int64_t)lo * p.h_kv + (k - s_tprefix[lo]) / per;
  return 2 * (int64_t)k + sw * (group + 1);
}

// First tile of block b (b = nblocks gives the tile count): the first tile
// whose cost position is at or past b / nblocks of the cost line.
template <int MODE>
__device__ int tc_split_point(const ScanParams &p, const int *s_tprefix, int b, int nblocks) {
  const int total = s_tprefix[p.S];
  const int64_t sw = MODE == kModeFilter ? kTcSwitchHalfTiles : 0;
  const int64_t cost_total = 2 * (int64_t)total + sw * p.S * p.h_kv;
  const int64_t c = cost_total * b / nblocks;
  int lo = 0, hi = total;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (tc_cost_pos<MODE>(p, s_tprefix, mid, sw) < c) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Writes the n buffered candidates of one head to the candidate buffer: one
// global atomic reserves their places.  All lanes of the warp call it.  Out
// of line: it runs about once per 64 candidates, and the scoring loop keeps
// its registers and schedule.
__device__ __noinline__ void tc_flush(const ScanParams &p, int64_t head,
                                      const unsigned long long *buf, unsigned n) {
  const int lane = threadIdx.x & 31;
  __syncwarp();
  unsigned base = 0;
  if (lane == 0) base = atomicAdd(&p.counts[head], n);
  base = __shfl_sync(0xffffffffu, base, 0);
  unsigned long long *dst = p.cand + head * p.cap;
  for (unsigned i = lane; i < n; i += 32) {
    const int64_t pos = (int64_t)base + i;
    if (pos < p.cap) dst[pos] = buf[i];
  }
  __syncwarp();
}

// Appends this warp's candidates among keys tk, tk + 1 (bit 2 h + k of cm:
// key tk + k clears head h's threshold, score s[2 h + k]) to the warp's
// per-head buffers (fill[h] entries used), flushing a buffer before it
// overflows.  All lanes call it; out of line, since it is the rare path.
__device__ __noinline__ void tc_append(const ScanParams &p, int64_t head0, int G,
                                       unsigned long long *cbuf, unsigned *fill, uint32_t cm,
                                       int tk, float s0, float s1, float s2, float s3, float s4,
                                       float s5, float s6, float s7) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  const float sv[8] = {s0, s1, s2, s3, s4, s5, s6, s7};
  for (int h = 0; h < G; ++h) {
    const bool t0 = (cm >> (2 * h)) & 1u, t1 = (cm >> (2 * h + 1)) & 1u;
    const unsigned b0 = __ballot_sync(0xffffffffu, t0);
    const unsigned b1 = __ballot_sync(0xffffffffu, t1);
    if (!(b0 | b1)) continue;
    const unsigned nn = (unsigned)(__popc(b0) + __popc(b1));
    unsigned f = fill[h];
    unsigned long long *cb = cbuf + h * kTcCandBuf;
    if (f + nn > (unsigned)kTcCandBuf) {
      tc_flush(p, head0 + h, cb, f);
      f = 0u;
    }
    if (t0) cb[f + __popc(b0 & lt)] = composite(sv[2 * h], (uint32_t)tk);
    if (t1) cb[f + __popc(b0) + __popc(b1 & lt)] = composite(sv[2 * h + 1], (uint32_t)(tk + 1));
    __syncwarp();
    if (lane == 0) fill[h] = f + nn;
    __syncwarp();
  }
}

template <int G, int MODE>
__global__ void __launch_bounds__(kTcThreads, 1) tc_scan_kernel(ScanParams p) {
  // the prologue below (tile space, tensor memory, barriers) reads only the
  // call's inputs, so it overlaps the previous kernel; the plans, thresholds
  // and counters that kernel writes are read after grid_dependency_wait
  allow_dependent_launch();
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int d = p.d;
  const TcPlanLayout PL = tc_plan_layout(d);
  unsigned char *sStage = smem;
  uint32_t *sOff = reinterpret_cast<uint32_t *>(smem + kTcStages * kTcStageBytes);
  unsigned char *sPlan = smem + kTcStages * kTcStageBytes + tc_off_bytes(d);
  unsigned long long *sCand = reinterpret_cast<unsigned long long *>(sPlan + PL.bytes);
  int *s_tprefix = reinterpret_cast<int *>(sCand + kTcEpiWarps * 4 * kTcCandBuf);
  const TcPlanHeader *sHdr = reinterpret_cast<const TcPlanHeader *>(sPlan);
  const uint16_t *sRows = reinterpret_cast<const uint16_t *>(sPlan + PL.off_rows);
  __shared__ __align__(8) unsigned long long s_bar[2 * kTcStages + 12];
  __shared__ uint32_t s_tmem;
  __shared__ int s_tmp[32];
  __shared__ volatile int s_fault;
  __shared__ unsigned s_fill[kTcEpiWarps][4];  // candidates buffered per epilogue warp and head

  const uint32_t bar0 = tc_smem_u32(&s_bar[0]);
  auto stage_full = [=](int s) { return bar0 + 8u * (uint32_t)s; };
  auto stage_empty = [=](int s) { return bar0 + 8u * (uint32_t)(kTcStages + s); };
  auto a_empty = [=](int g, int b) { return bar0 + 8u * (uint32_t)(2 * kTcStages + 2 * g + b); };
  auto acc_full = [=](int b) { return bar0 + 8u * (uint32_t)(2 * kTcStages + 4 + b); };
  auto acc_empty = [=](int b) { return bar0 + 8u * (uint32_t)(2 * kTcStages + 6 + b); };
  auto a_full = [=](int g, int b) { return bar0 + 8u * (uint32_t)(2 * kTcStages + 8 + 2 * g + b); };
  // A wait that gives up records a fault; the caller carries on (never
  // leaving its warp's named barriers), so that the block still finishes.
  auto wait_or_fault = [&](uint32_t bar, uint32_t parity) {
    if (!s_fault && !mbar_wait(bar, parity)) s_fault = 1;
  };
  // one lane waits, the warp follows
  // every lane probes (one shared-memory word, so all see the same phase);
  // only a phase still open sends lane 0 into the bounded wait
  auto warp_wait = [&](uint32_t bar, uint32_t parity) {
    if (!__all_sync(0xffffffffu, mbar_test(bar, parity))) {
      if (lane == 0) wait_or_fault(bar, parity);
      __syncwarp();
    }
  };
  auto warp_arrive = [&](uint32_t bar) {
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
  };

  // ---- tile space: every (session, KV head) contributes its tiles --------
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
  if (tid < 2) s_tmp[tid] = tc_split_point<MODE>(p, s_tprefix, (int)blockIdx.x + tid, (int)gridDim.x);
  __syncthreads();
  const int t_begin = s_tmp[0];
  const int t_end = s_tmp[1];
  if (t_begin >= t_end) return;

  // ---- tensor memory, barriers, preset accumulators ----------------------
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     tc_smem_u32(&s_tmem)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(stage_full(s), kTcLoadWarps);    // every load warp
      mbar_init(stage_empty(s), kTcBuildWarps);  // every build warp
    }
    for (int i = 0; i < 2; ++i) {
      for (int g = 0; g < 2; ++g) {
        mbar_init(a_full(g, i), kTcBuildWarps / 2);   // the build warps of group g
        mbar_init(a_empty(g, i), kTcLoadWarps / 2);   // the MMA commits for group g
      }
      mbar_init(acc_full(i), kTcLoadWarps);         // every MMA issuer commits at a tile's end
      mbar_init(acc_empty(i), kTcEpiWarps);         // every epilogue warp
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    s_fault = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int quarter = warp & 3;
  const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
  uint32_t mg[8];  // the accumulator preset, stored eight columns at a time
#pragma unroll
  for (int i = 0; i < 8; ++i) mg[i] = kTcMagicBits;
  if (warp >= kTcEpiWarp0) {
    // epilogue warp (quarter, half eh) owns M-blocks 4 eh .. 4 eh + 3: columns 64 eh .. + 63
    const int eh = (warp - kTcEpiWarp0) >> 2;
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        tc_st8(tmem + lane_base + (uint32_t)(b * kTcAccCols + 64 * eh + 8 * i), mg);
    tc_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  grid_dependency_wait();

  // chunks and tiles since the start of the kernel
  uint32_t it = 0, tj = 0;

  // ---- segments: runs of tiles that share one (session, KV head) ---------
  int t = t_begin;
  while (t < t_end) {
    __syncthreads();
    if (s_fault) break;
    const TcLoc L0 = tc_locate<MODE>(p, s_tprefix, t);
    const int seg_end = min(t_end, t - L0.ti + L0.per);
    const int ntiles = seg_end - t;
    const int ti0 = L0.ti;
    {
      const int gid = L0.s * p.h_kv + L0.g;
      const unsigned char *gplan = p.plans + (size_t)gid * PL.bytes;
      const int nk = reinterpret_cast<const TcPlanHeader *>(gplan)->nks;
      const int used = PL.off_b + nk * kTcBChunkBytes;
      for (int i = tid; i < used / 16; i += kTcThreads)
        reinterpret_cast<uint4 *>(sPlan)[i] = reinterpret_cast<const uint4 *>(gplan)[i];
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // B is read by the MMAs
    }
    __syncthreads();
    const int P = sHdr->P;
    const int nks = sHdr->nks;
    const bool big = P > kTcSmallP;  // 0/1 cells instead of 0/2^r
    // word offset / 4 of every union row within the KV head's planes; the
    // padding rows of the last K-step repeat its first row (their B weights
    // are zero, and the repeated row is already on its way from memory)
    for (int r = tid; r < nks * kTcKStep; r += kTcThreads)
      sOff[r] = (uint32_t)((int64_t)sRows[r < P ? r : (r & ~(kTcKStep - 1))] * (L0.W >> 2));
    __syncthreads();
    const int64_t head0 = (int64_t)L0.s * p.h_q + L0.g * G;
    // The segment's K-steps (tile tl, plane block kidx), tile by tile, are
    // taken two at a time: chunk u holds K-steps 2 u and 2 u + 1, which may
    // belong to two tiles.  Only a tile's last K-step is ever partly padding.
    const int nksteps = ntiles * nks;
    const int nchunks = (nksteps + 1) / 2;

    if (warp < kTcLoadWarps) {
      // --------------------------------------------------------------- load --
      // Thread (group i, quad m) loads words 4 m .. 4 m + 3 of the tile from
      // the four plane rows 4 i .. 4 i + 3 of a chunk, and stores byte q of
      // the four rows' words as T = [x0.q, x1.q, x2.q, x3.q] at
      // stage[i][q][word]: a build warp of quarter q reads its T of plane
      // group i for word `lane` with one conflict-free load.
      const int m = tid & 7;
      const int grp = tid >> 3;  // 0 .. 15
      const uint32_t *gbase = L0.planes + (int64_t)L0.g * d * 4 * L0.W;
      const int64_t nsamp = MODE == kModeSample ? sampled_sectors(L0.n) : 0;
      // word offset of this thread's quad in tile ti, clamped into the row:
      // words past the data hold keys that the epilogue never reports
      const int64_t wmax = L0.W - 4;
      auto quad_word = [&](int ti) -> int64_t {
        int64_t gw;
        if (MODE == kModeSample) {
          const int64_t sj = (int64_t)ti * kTcSampleSectorsPerTile + (m >> 1);
          gw = sj * kSampleStride * kSectorWords + (m & 1) * 4;
          if (sj >= nsamp) gw = wmax;
        } else {
          gw = (int64_t)ti * kTcTileWords + m * 4;
        }
        return gw < wmax ? gw : wmax;
      };
      // this thread's K-step of a chunk is its half (grp >> 3); a cursor
      // (tile, kidx) walks the K-steps of that half, two K-steps per chunk
      const int half = grp >> 3;
      const int rgrp = 4 * (grp & 7);  // first of its four rows in the K-step
      auto cursor0 = [&](int &tl, int &kx) {
        tl = 0;
        kx = half;
        if (kx >= nks) { kx -= nks; ++tl; }
      };
      auto advance = [&](int &tl, int &kx) {
        kx += 2;
        while (kx >= nks) { kx -= nks; ++tl; }
      };
      int ltl, lk;  // next K-step to load
      cursor0(ltl, lk);
      auto load_next = [&](uint4 (&v)[4]) {
        if (ltl < ntiles) {
          const int64_t gw = quad_word(ti0 + ltl);
          const uint4 o = *reinterpret_cast<const uint4 *>(sOff + lk * kTcKStep + rgrp);
          v[0] = __ldcg(reinterpret_cast<const uint4 *>(gbase + (int64_t)o.x * 4 + gw));
          v[1] = __ldcg(reinterpret_cast<const uint4 *>(gbase + (int64_t)o.y * 4 + gw));
          v[2] = __ldcg(reinterpret_cast<const uint4 *>(gbase + (int64_t)o.z * 4 + gw));
          v[3] = __ldcg(reinterpret_cast<const uint4 *>(gbase + (int64_t)o.w * 4 + gw));
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) v[k] = make_uint4(0u, 0u, 0u, 0u);
        }
        advance(ltl, lk);
      };
      // MMA issue: lane 0 of load warp l feeds M-blocks 2 l and 2 l + 1 (build
      // group l / 2), NS + 1 chunks behind its loads: by the time it has
      // waited for stage u - NS to be read, the build warps have stored and
      // signalled chunk u - NS - 1.
      const int ig = warp >> 1;
      const uint64_t b_desc0 = tc_smem_desc(tc_smem_u32(sPlan + PL.off_b), kTcLBO, kTcSBO);
      int itl = 0, ik = 0;  // first K-step of the next chunk to issue
      auto issue = [&](int v) {
        const uint32_t ugv = it + (uint32_t)v;
        const int sbv = (int)(ugv & 1);
        // the chunk's two K-steps: (tile, block) and accumulator buffers,
        // all warp-uniform, worked out before the one elected lane issues
        const int tl0 = itl, kx0 = ik;
        const int tl1 = kx0 + 1 == nks ? tl0 + 1 : tl0;
        const int kx1 = kx0 + 1 == nks ? 0 : kx0 + 1;
        const bool two = 2 * v + 1 < nksteps;
        const uint32_t tt0 = tj + (uint32_t)tl0, tt1 = tj + (uint32_t)tl1;
        // a tile's first MMA needs its accumulators read out
        if (kx0 == 0 && tt0 >= 2) warp_wait(acc_empty((int)(tt0 & 1)), ((tt0 >> 1) - 1) & 1);
        if (two && kx1 == 0 && tt1 >= 2) warp_wait(acc_empty((int)(tt1 & 1)), ((tt1 >> 1) - 1) & 1);
        warp_wait(a_full(ig, sbv), (ugv >> 1) & 1);
        tc_fence_after();
        const uint32_t acl = tmem + (uint32_t)(kTcAColBase + sbv * kTcABufCols + 16 * warp);
        const uint32_t d0 = tmem + (uint32_t)((tt0 & 1) * kTcAccCols + 2 * kTcN * warp);
        const uint32_t d1 = tmem + (uint32_t)((tt1 & 1) * kTcAccCols + 2 * kTcN * warp);
        const uint64_t bd0 = b_desc0 + (uint64_t)(kx0 * (kTcBChunkBytes >> 4));
        const uint64_t bd1 = b_desc0 + (uint64_t)(kx1 * (kTcBChunkBytes >> 4));
        if (tc_elect_one()) {
          // M-blocks 2 l and 2 l + 1: A columns 8 r (+ 64 for the second K-step)
          tc_mma(d0, acl, bd0);
          tc_mma(d0 + kTcN, acl + 8u, bd0);
          if (kx0 == nks - 1) tc_commit(acc_full((int)(tt0 & 1)));
          if (two) {
            tc_mma(d1, acl + 64u, bd1);
            tc_mma(d1 + kTcN, acl + 72u, bd1);
            if (kx1 == nks - 1) tc_commit(acc_full((int)(tt1 & 1)));
          }
          tc_commit(a_empty(ig, sbv));
        }
        __syncwarp();
        ik += 2;
        while (ik >= nks) { ik -= nks; ++itl; }
      };
      uint4 ring[kTcRing][4];
#pragma unroll
      for (int j = 0; j < kTcRing; ++j) load_next(ring[j]);
      for (int u0 = 0; u0 < nchunks; u0 += kTcRing) {
#pragma unroll
        for (int jj = 0; jj < kTcRing; ++jj) {
          const int u = u0 + jj;
          if (u >= nchunks) break;
          const uint32_t ug = it + (uint32_t)u;
          const int s = (int)(ug % kTcStages);
          if (ug >= (uint32_t)kTcStages) warp_wait(stage_empty(s), ((ug / kTcStages) - 1) & 1);
          if (u > kTcStages) issue(u - kTcStages - 1);
          uint32_t *dst = reinterpret_cast<uint32_t *>(sStage + s * kTcStageBytes) + grp * 4 * kTcTileWords + 4 * m;
          uint32_t Tq[4][4];  // [quarter][word]
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const uint32_t x0 = (&ring[jj][0].x)[w], x1 = (&ring[jj][1].x)[w];
            const uint32_t x2 = (&ring[jj][2].x)[w], x3 = (&ring[jj][3].x)[w];
            const uint32_t a_lo = __byte_perm(x0, x1, 0x5140), a_hi = __byte_perm(x0, x1, 0x7362);
            const uint32_t b_lo = __byte_perm(x2, x3, 0x5140), b_hi = __byte_perm(x2, x3, 0x7362);
            Tq[0][w] = __byte_perm(a_lo, b_lo, 0x5410);
            Tq[1][w] = __byte_perm(a_lo, b_lo, 0x7632);
            Tq[2][w] = __byte_perm(a_hi, b_hi, 0x5410);
            Tq[3][w] = __byte_perm(a_hi, b_hi, 0x7632);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4 *>(dst + q * kTcTileWords) = make_uint4(Tq[q][0], Tq[q][1], Tq[q][2], Tq[q][3]);
          warp_arrive(stage_full(s));
          load_next(ring[jj]);
        }
      }
      for (int v = max(0, nchunks - kTcStages - 1); v < nchunks; ++v) issue(v);
    } else if (warp < kTcEpiWarp0) {
      // ------------------------------------------------------------ build --
      // Build warp (quarter q, group g) writes the cells of M-blocks
      // 4 g .. 4 g + 3 for its lane quarter, both K-steps of a chunk.  It
      // signals chunk u - 1 (its stores complete) after reading stage u, so
      // that the tensor memory stores have that long to land.
      const int g = (warp - kTcBuildWarp0) >> 2;
      auto signal = [&](int up) {
        tc_wait_st();
        tc_fence_before();
        warp_arrive(a_full(g, (int)((it + (uint32_t)up) & 1)));
      };
      for (int u = 0; u < nchunks; ++u) {
        const uint32_t ug = it + (uint32_t)u;
        const int s = (int)(ug % kTcStages);
        const int sb = (int)(ug & 1);
        warp_wait(stage_full(s), (ug / kTcStages) & 1);
        const uint32_t *src = reinterpret_cast<const uint32_t *>(sStage + s * kTcStageBytes) + quarter * kTcTileWords + lane;
        uint32_t T[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) T[i] = src[i * 4 * kTcTileWords];
        warp_arrive(stage_empty(s));
        if (u > 0) signal(u - 1);
        // chunk u's A buffer was last read by the MMAs of chunk u - 2
        if (ug >= 2) warp_wait(a_empty(g, sb), ((ug >> 1) - 1) & 1);
        const uint32_t acol = tmem + lane_base + (uint32_t)(kTcAColBase + sb * kTcABufCols + 32 * g);
        const int nk_here = 2 * u + 1 < nksteps ? 2 : 1;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          if (ks >= nk_here) break;
          uint32_t cell[32];
#pragma unroll
          for (int rr = 0; rr < 4; ++rr) {
            const int r = 4 * g + rr;
            if (!big) {
              const uint32_t msk = 0x01010101u << r;
#pragma unroll
              for (int i = 0; i < 8; ++i) cell[8 * rr + i] = T[8 * ks + i] & msk;
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i) cell[8 * rr + i] = (T[8 * ks + i] >> r) & 0x01010101u;
            }
          }
          tc_st32(acol + (uint32_t)(64 * ks), cell);
        }
      }
      signal(nchunks - 1);
    } else {
      // ---------------------------------------------------------- epilogue --
      // s = K + Delta 2^-r sum_m 256^m (f_m - M), f_m the accumulator of digit
      // m read as a float (the two low digits combined before M is removed)
      const int ew = warp - kTcEpiWarp0;
      const int eh = ew >> 2;  // M-blocks 4 eh .. 4 eh + 3
      unsigned long long *cbuf = sCand + (size_t)ew * 4 * kTcCandBuf;
      unsigned *fill = s_fill[ew];
      if (lane < 4) fill[lane] = 0u;
      __syncwarp();
      float Kh[G], Dh[G], tau[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        Kh[h] = sHdr->K[h];
        Dh[h] = sHdr->D[h];
        tau[h] = -INFINITY;
        if (MODE == kModeFilter) {
          const uint32_t key = p.tau[head0 + h];
          tau[h] = key == 0u ? -INFINITY : key_float(key);
        }
      }
      const int nsamp = MODE == kModeSample ? (int)sampled_sectors(L0.n) : 0;
      const int nkeys = (int)L0.n;
      for (int tl = 0; tl < ntiles; ++tl) {
        const uint32_t tt = tj + (uint32_t)tl;
        const int ti = ti0 + tl;
        const int ab = (int)(tt & 1);
        warp_wait(acc_full(ab), (tt >> 1) & 1);
        tc_fence_after();
        // key of (lane, quarter, r): 32 lane + 8 quarter + r of the tile
        int tok0, slot0 = 0;
        bool live = true;
        if (MODE == kModeSample) {
          const int sj = ti * kTcSampleSectorsPerTile + (lane >> 3);
          live = sj < nsamp;
          tok0 = (sj * kSampleStride * kSectorWords + (lane & 7)) * 32 + 8 * quarter;
          slot0 = sj * 256 + (lane & 7) * 32 + 8 * quarter;
        } else {
          tok0 = (ti * kTcTileWords + lane) * 32 + 8 * quarter;
        }
        const uint32_t abase = tmem + lane_base + (uint32_t)(ab * kTcAccCols);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          // M-blocks r = 2 rp, 2 rp + 1: keys tok0 + r
          const int rp = 2 * eh + rr;
          uint32_t v[32];
          tc_ld32(abase + (uint32_t)(32 * rp), v);
#pragma unroll
          for (int i = 0; i < 4; ++i) tc_st8(abase + (uint32_t)(32 * rp + 8 * i), mg);
          float sc[2][4];
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            const float scale = big ? 1.0f : __int_as_float((127 - (2 * rp + hr)) << 23);  // 2^-r
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              if (h < G) {
                const uint32_t *a = v + 16 * hr + 4 * h;
                const float hi = fmaf(__uint_as_float(a[3]) - kTcMagic, 256.0f,
                                      __uint_as_float(a[2]) - kTcMagic);
                const float lo = fmaf(__uint_as_float(a[1]), 256.0f,
                                      __uint_as_float(a[0]) - 257.0f * kTcMagic);
                sc[hr][h] = fmaf(fmaf(hi, 65536.0f, lo), Dh[h] * scale, Kh[h]);
              } else {
                sc[hr][h] = 0.0f;
              }
            }
          }
          const int tk = tok0 + 2 * rp;
          if (MODE == kModeSample) {
            if (live) {
#pragma unroll
              for (int h = 0; h < G; ++h) {
                uint32_t *dst = p.sample + (head0 + h) * p.m_max + slot0 + 2 * rp;
                dst[0] = tk < nkeys ? float_key(sc[0][h]) : 0u;
                dst[1] = tk + 1 < nkeys ? float_key(sc[1][h]) : 0u;
              }
            }
          } else {
            if (p.debug_scores) {
#pragma unroll
              for (int h = 0; h < G; ++h)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr)
                  if (tk + hr < nkeys)
                    p.debug_scores[(head0 + h) * (int64_t)nkeys + tk + hr] = sc[hr][h];
            }
            uint32_t cm = 0u;  // bit 2 h + k: key tk + k clears head h's threshold
#pragma unroll
            for (int h = 0; h < G; ++h) {
              cm |= (tk < nkeys && sc[0][h] >= tau[h] ? 1u : 0u) << (2 * h);
              cm |= (tk + 1 < nkeys && sc[1][h] >= tau[h] ? 1u : 0u) << (2 * h + 1);
            }
            if (__any_sync(0xffffffffu, cm != 0u))
              tc_append(p, head0, G, cbuf, fill, cm, tk, sc[0][0], sc[1][0], sc[0][1], sc[1][1],
                        sc[0][2], sc[1][2], sc[0][3], sc[1][3]);
          }
        }
        tc_wait_st();
        tc_fence_before();
        warp_arrive(acc_empty(ab));
      }
      if (MODE == kModeFilter) {
        for (int h = 0; h < G; ++h) {
          const unsigned f = fill[h];
          if (f) tc_flush(p, head0 + h, cbuf + h * kTcCandBuf, f);
        }
      }
    }
    it += (uint32_t)nchunks;
    tj += (uint32_t)ntiles;
    t = seg_end;
  }

  // ---- teardown ------------------------------------------------------------
  // The epilogue has seen every tile's accumulators, so every MMA is done;
  // wait for the arrivals of the last two chunks' commits before the
  // barriers and tensor memory go away.
  __syncthreads();
  if (tid == 0) {
    for (int back = 1; back <= 2; ++back) {
      if (it < (uint32_t)back) break;
      const uint32_t ug = it - (uint32_t)back;
      mbar_wait(a_empty(0, (int)(ug & 1)), (ug >> 1) & 1);
      mbar_wait(a_empty(1, (int)(ug & 1)), (ug >> 1) & 1);
    }
  }
  __syncthreads();
  if (s_fault && tid == 0) atomicAdd(&p.status->device_faults, 1u);
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
  return launch_dependent(tc_scan_kernel<G, MODE>, dim3(sms), dim3(kTcThreads), (size_t)smem, stream, p);
}

cudaError_t launch_tc_plan(const ScanParams &p, cudaStream_t stream) {
  return launch_dependent(tc_plan_kernel, dim3(p.S * p.h_kv), dim3(256), 0, stream, p);
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
