// Tensor-core form of the Fathom scan for sm_100a (tcgen05.mma kind::i8,
// A operand in tensor memory).
//
// The score of key i for query head h ("Fathom Makes KV-Cache Scans
// Query-Adaptive for Long-Context Decoding", method paragraphs 2-3; arXiv
// 2609.17652 abstract) is a sum over the bit planes the head reads:
//   s_h(i) = C_h + sum_{(c, j): j < t_hc} W_hcj b_cj(i),   W_hcj = q_hc s_c 2^(3 - j),
//   C_h    = sum_c q_hc (m_c + s_c (2^(4 - t_hc) - 1) / 2),
// b_cj(i) the bit of plane j of channel c for key i.  For the G query heads of
// one KV head this is one matrix product over the union planes of the group:
//   A [keys x planes] = the plane bits,
//   B [planes x (head, digit)] = W_hcj / Delta_h as a 30-bit fixed-point
//     integer in four signed base-256 int8 digits (0 where the head does not
//     read the plane),
// accumulated exactly in int32 by the tensor cores; the epilogue forms
//   s_h = C_h + Delta_h sum_m 256^m acc_m.
//
// Layout (B200 design).  A 1024-key tile of one KV head is 32 plane words per
// plane.  Tensor-memory lane (quarter q, lane l) of M-block (hr, e) stands for
// word l of the tile and bit position r = q + 4 hr of every byte of that word;
// the four bytes of its 32-bit column hold, for a pair of planes (p, p'), the
// bits of keys 8 kk + r for kk = 2e, 2e + 1:
//   cell = byte_perm(P_p, P_p', e ? 0x7632 : 0x5410) & (0x01010101 << r)
// (one permute per plane pair and one AND per cell, each byte 0 or 2^r).  The
// two keys in a cell are separated by B: its 32 columns are (kk', head, digit)
// and a column reads only the bytes of its kk'.  The 2^r of a lane is undone
// in the epilogue.
//
// Roles (10 warps): warp 8 stages 32 plane rows of a tile ("chunk") into
// shared memory with 16-byte cp.async copies; warps 0-7 turn a chunk into
// tensor-memory cells (warp w: lane quarter w % 4, half the chunk's planes)
// and, one tile later, read the tile's accumulators back, score and filter
// them; one thread of warp 9 issues the MMAs.  They hand chunks, A buffers
// and accumulators to each other through mbarriers; every wait is bounded in
// time and a timeout records a device fault in the workspace status.
// Accumulators are preset to the bits of 1.5 * 2^23, so that an accumulator
// read back as a float is 1.5 * 2^23 + acc exactly (|acc| <= 2^22).
#include "fathom_internal.cuh"

namespace fathom {

// ---------------------------------------------------------------- layout --
constexpr int kTcTileWords = 32;                        // 1024 keys per tile
constexpr int kTcChunkPlanes = 32;                      // plane rows per chunk
constexpr int kTcStageBytes = kTcChunkPlanes * kTcTileWords * 4;  // 4 KiB
constexpr int kTcNumStages = 16;                        // chunks staged ahead
constexpr int kTcNumABuf = 4;                           // A buffers in tensor memory
constexpr int kTcBuildWarps = 8;
constexpr int kTcProducerWarp = 8;
constexpr int kTcMmaWarp = 9;
constexpr int kTcThreads = 10 * 32;
constexpr int kTcAccCols = 4 * 32;                      // one tile: 4 M-blocks x N = 32
constexpr int kTcABufCols = 4 * 16;                     // one chunk: 4 M-blocks x 16 columns
constexpr int kTcTmemCols = 512;                        // 2 x 128 accumulators + 4 x 64 A
constexpr int kTcAColBase = 2 * kTcAccCols;
constexpr int kTcSampleSectorsPerTile = kTcTileWords / kSectorWords;  // 4
// B for one K-step (16 planes = 8 columns = 32 int8 K elements): 32 rows
// (kk', head, digit) x 32 bytes, K-major, no swizzle.  Core matrices are
// 8 rows x 16 bytes; 8-row groups are 128 B apart (SBO), the two 16-byte K
// halves 512 B apart (LBO).
constexpr int kTcKStepBytes = 1024;
constexpr uint32_t kTcSBO = 128;
constexpr uint32_t kTcLBO = 512;
// Instruction descriptor: D s32, A u8 K-major (tensor memory), B s8
// K-major, N = 32, M = 128, dense.
constexpr uint32_t kTcIdesc = (2u << 4)             // D format s32
                              | (0u << 7)           // A format u8
                              | (1u << 10)          // B format s8
                              | (0u << 15)          // A K-major
                              | (0u << 16)          // B K-major
                              | ((32u >> 3) << 17)  // N
                              | ((128u >> 4) << 24);  // M
constexpr uint32_t kTcMagicBits = 0x4b400000u;  // 1.5 * 2^23
constexpr float kTcMagic = 12582912.0f;
// A plane count above which the cells hold 0/1 instead of 0/2^r, so that an
// accumulator stays within 2^22 (|digit| <= 128, 2^r <= 128).
constexpr int kTcSmallP = 256;

struct TcPlanHeader {
  int P;       // union planes of the group
  int nchunk;  // ceil(P / 32)
  int pad0, pad1;
  float K[4];  // C_h
  float D[4];  // Delta_h (a power of two)
  float pad2[4];
};
static_assert(sizeof(TcPlanHeader) == 64, "header size");

struct TcPlanLayout {
  int off_rows;  // uint16 [4 d]: c * 4 + j of every union plane, channel-major
  int off_b;     // int8 [ceil(4 d / 16)][1024]
  int bytes;
};

__host__ __device__ inline TcPlanLayout tc_plan_layout(int d) {
  TcPlanLayout L;
  L.off_rows = (int)sizeof(TcPlanHeader);
  L.off_b = align16(L.off_rows + 2 * 4 * d);
  L.bytes = L.off_b + ((4 * d + 15) / 16) * kTcKStepBytes;
  return L;
}

int tc_plan_bytes(int d) { return tc_plan_layout(d).bytes; }

static int tc_smem_bytes(int d, int S) {
  int b = 128 + kTcNumStages * kTcStageBytes + tc_plan_layout(d).bytes + 4 * (S + 1);
  // more than half an SM's shared memory: one block per SM, so that the
  // block's 512 tensor-memory columns never wait for another block
  return b < 120 * 1024 ? 120 * 1024 : b;
}

// --------------------------------------------------------------- helpers --

__device__ __forceinline__ uint32_t tc_smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void tc_cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
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
// Arrives on bar once all of this thread's earlier cp.async copies are done.
__device__ __forceinline__ void mbar_arrive_cp_async(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}

// Waits for the completion of the phase of bar with the given parity, giving
// up after about a second (2^31 cycles).  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  if (done) return true;
  const long long t0 = clock64();
  while (true) {
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P;\n\t}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
    if (clock64() - t0 > (1ll << 31)) return false;
  }
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(kTcIdesc), "r"(1u)
      : "memory");
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

// Writes the value x into 32 consecutive columns of this warp's lanes.
__device__ __forceinline__ void tc_st32_fill(uint32_t taddr, uint32_t x) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, "
      "%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1};\n" ::"r"(
          taddr),
      "r"(x)
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
    for (int hh = 0; hh < G; ++hh) {
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
  const int nks = (P + 15) / 16;
  // B of every used K-step starts at zero (padding planes, heads that do not
  // read a plane, and the other key of every cell contribute nothing)
  for (int i = threadIdx.x; i < nks * kTcKStepBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4 *>(bmat)[i] = make_uint4(0, 0, 0, 0);
  double delta[4];
  for (int hh = 0; hh < 4; ++hh) {
    // the largest plane weight is 8 max_c |q_c s_c|; W / Delta < 2^30
    const double wmax = 8.0 * __longlong_as_double((long long)s_wmax[hh]);
    int ex = 0;
    frexp(wmax, &ex);  // wmax < 2^ex
    delta[hh] = wmax > 0.0 ? ldexp(1.0, ex - 30) : 1.0;
  }
  if (threadIdx.x == 0) {
    hdr->P = P;
    hdr->nchunk = (P + kTcChunkPlanes - 1) / kTcChunkPlanes;
    hdr->pad0 = hdr->pad1 = 0;
    const int nw = (blockDim.x + 31) >> 5;
    for (int hh = 0; hh < 4; ++hh) {
      double sum = 0.0;
      for (int wv = 0; wv < nw; ++wv) sum += s_red[hh][wv];
      hdr->K[hh] = hh < G ? (float)sum : 0.0f;
      hdr->D[hh] = (float)delta[hh];
      hdr->pad2[hh] = 0.0f;
    }
    atomicAdd(&p.status->union_planes, (uint32_t)P);
  }
  __syncthreads();
  for (int j = 0; j < tstar; ++j) {
    const int pl = off + j;
    rows[pl] = (uint16_t)(c * 4 + j);
    int8_t *bk = bmat + (size_t)(pl >> 4) * kTcKStepBytes;
    const int col = (pl & 15) >> 1, pp = pl & 1;
    for (int hh = 0; hh < G; ++hh) {
      if (j >= t[hh]) continue;
      long long x = llrint(ldexp(w[hh], 3 - j) / delta[hh]);
      for (int dg = 0; dg < 4; ++dg) {
        const long long v = dg < 3 ? ((x + 128) & 255) - 128 : x;
        x = (x - v) >> 8;
        for (int kq = 0; kq < 2; ++kq) {
          const int n = kq * 16 + hh * 4 + dg;
          const int k = 4 * col + 2 * pp + kq;
          bk[(n >> 3) * kTcSBO + (k >> 4) * kTcLBO + (n & 7) * 16 + (k & 15)] = (int8_t)v;
        }
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

template <int G, int MODE>
__global__ void __launch_bounds__(kTcThreads, 1) tc_scan_kernel(ScanParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int d = p.d;
  const TcPlanLayout PL = tc_plan_layout(d);
  unsigned char *sStage = smem;
  unsigned char *sPlan = smem + kTcNumStages * kTcStageBytes;
  const TcPlanHeader *sHdr = reinterpret_cast<const TcPlanHeader *>(sPlan);
  const uint16_t *sRows = reinterpret_cast<const uint16_t *>(sPlan + PL.off_rows);
  int *s_tprefix = reinterpret_cast<int *>(sPlan + PL.bytes);
  __shared__ __align__(8) unsigned long long s_bar[2 * kTcNumStages + 2 * kTcNumABuf + 4];
  __shared__ uint32_t s_tmem;
  __shared__ int s_tmp[32];
  __shared__ volatile int s_fault;

  const uint32_t bar0 = tc_smem_u32(&s_bar[0]);
  auto stage_full = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  auto stage_empty = [&](int i) { return bar0 + 8u * (uint32_t)(kTcNumStages + i); };
  auto a_full = [&](int i) { return bar0 + 8u * (uint32_t)(2 * kTcNumStages + i); };
  auto a_empty = [&](int i) { return bar0 + 8u * (uint32_t)(2 * kTcNumStages + kTcNumABuf + i); };
  auto acc_full = [&](int i) { return bar0 + 8u * (uint32_t)(2 * kTcNumStages + 2 * kTcNumABuf + i); };
  auto acc_empty = [&](int i) {
    return bar0 + 8u * (uint32_t)(2 * kTcNumStages + 2 * kTcNumABuf + 2 + i);
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
  const int total = s_tprefix[p.S];
  const int t_begin = (int)(((int64_t)blockIdx.x * total) / gridDim.x);
  const int t_end = (int)(((int64_t)(blockIdx.x + 1) * total) / gridDim.x);
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
    for (int i = 0; i < kTcNumStages; ++i) {
      mbar_init(stage_full(i), 32);             // every producer lane, after its copies
      mbar_init(stage_empty(i), kTcBuildWarps);
    }
    for (int i = 0; i < kTcNumABuf; ++i) {
      mbar_init(a_full(i), kTcBuildWarps);
      mbar_init(a_empty(i), 1);                 // tcgen05.commit
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full(i), 1);
      mbar_init(acc_empty(i), kTcBuildWarps);
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
  if (warp < kTcBuildWarps) {
    // warps q and q + 4 preset one half each of the two accumulator sets
    const int half = warp >> 2;
    for (int i = 0; i < 4; ++i)
      tc_st32_fill(tmem + lane_base + (uint32_t)(half * kTcAccCols + 32 * i), kTcMagicBits);
    tc_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // pipeline counters: chunk items and tiles since the start of the kernel,
  // and (MMA thread) the last item and tile whose completion was committed
  uint32_t it = 0, tj = 0;
  int last_item = -1, last_tile = -1;

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
      const int P = reinterpret_cast<const TcPlanHeader *>(gplan)->P;
      const int used = PL.off_b + ((P + 15) / 16) * kTcKStepBytes;
      for (int i = tid; i < used / 16; i += kTcThreads)
        reinterpret_cast<uint4 *>(sPlan)[i] = reinterpret_cast<const uint4 *>(gplan)[i];
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // B is read by the MMAs
    }
    __syncthreads();
    const int P = sHdr->P;
    const int nch = sHdr->nchunk > 0 ? sHdr->nchunk : 1;  // a plane-less group still has tiles
    const bool big = P > kTcSmallP;                        // 0/1 cells instead of 0/2^r
    const int64_t head0 = (int64_t)L0.s * p.h_q + L0.g * G;

    if (warp == kTcProducerWarp) {
      // ---------------------------------------------------------- producer --
      const uint32_t *gbase = L0.planes + (int64_t)L0.g * d * 4 * L0.W;
      const int64_t nsamp = MODE == kModeSample ? sampled_sectors(L0.n) : 0;
      uint32_t i = it;
      for (int j = 0; j < ntiles && !s_fault; ++j) {
        const int ti = ti0 + j;
        for (int c = 0; c < nch; ++c, ++i) {
          const int st = (int)(i % kTcNumStages);
          if (i >= (uint32_t)kTcNumStages &&
              !mbar_wait(stage_empty(st), ((i / kTcNumStages) - 1) & 1)) {
            s_fault = 1;
            break;
          }
          const int nrows = min(kTcChunkPlanes, P - c * kTcChunkPlanes);
          const uint32_t dst0 = tc_smem_u32(sStage + st * kTcStageBytes);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int id = lane + 32 * k;  // row id / 8, 16-byte piece id % 8
            const int row = id >> 3, piece = id & 7;
            if (row < nrows) {
              const uint32_t *src = gbase + (int64_t)sRows[c * kTcChunkPlanes + row] * L0.W;
              int64_t gw;
              bool ok;
              if (MODE == kModeSample) {
                const int64_t sj = (int64_t)ti * kTcSampleSectorsPerTile + (piece >> 1);
                gw = sj * kSampleStride * kSectorWords + (piece & 1) * 4;
                ok = sj < nsamp && gw < L0.W;
              } else {
                gw = (int64_t)ti * kTcTileWords + piece * 4;
                ok = gw < L0.W;
              }
              tc_cp_async16(dst0 + (uint32_t)(row * 128 + piece * 16),
                            ok ? (const void *)(src + gw) : (const void *)src, ok ? 16u : 0u);
            }
          }
          mbar_arrive_cp_async(stage_full(st));
        }
        if (s_fault) break;
      }
      asm volatile("cp.async.wait_all;\n" ::: "memory");
    } else if (warp == kTcMmaWarp) {
      // --------------------------------------------------------------- MMA --
      if (lane == 0) {
        const uint32_t b_addr = tc_smem_u32(sPlan + PL.off_b);
        uint32_t i = it, tt = tj;
        bool ok = true;
        for (int j = 0; j < ntiles && ok; ++j, ++tt) {
          const int ab = (int)(tt & 1);
          if (tt >= 2 && (s_fault || !mbar_wait(acc_empty(ab), ((tt >> 1) - 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dcol = tmem + (uint32_t)(ab * kTcAccCols);
          for (int c = 0; c < nch; ++c, ++i) {
            const int b = (int)(i % kTcNumABuf);
            if (s_fault || !mbar_wait(a_full(b), (i / kTcNumABuf) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t acol = tmem + (uint32_t)(kTcAColBase + b * kTcABufCols);
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
              if (c * kTcChunkPlanes + 16 * ks < P) {
                const uint64_t bdesc = tc_smem_desc(
                    b_addr + (uint32_t)((2 * c + ks) * kTcKStepBytes), kTcLBO, kTcSBO);
#pragma unroll
                for (int mb = 0; mb < 4; ++mb)
                  tc_mma(dcol + (uint32_t)(32 * mb), acol + (uint32_t)(16 * mb + 8 * ks), bdesc);
              }
            }
            tc_commit(a_empty(b));
            last_item = (int)i;
            if (c == nch - 1) {
              tc_commit(acc_full(ab));
              last_tile = (int)tt;
            }
          }
        }
        if (!ok) s_fault = 1;
      }
    } else {
      // ----------------------------------------------- build and epilogue --
      const int half = warp >> 2;  // which K-step of a chunk; which kk pair in the epilogue
      const uint32_t m0 = 0x01010101u << quarter;        // r = q
      const uint32_t m1 = 0x01010101u << (quarter + 4);  // r = q + 4
      float Kh[G], Dh[G][2], tau[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        Kh[h] = sHdr->K[h];
        Dh[h][0] = big ? sHdr->D[h] : ldexpf(sHdr->D[h], -quarter);
        Dh[h][1] = big ? sHdr->D[h] : ldexpf(sHdr->D[h], -(quarter + 4));
        tau[h] = -INFINITY;
        if (MODE == kModeFilter) {
          const uint32_t key = p.tau[head0 + h];
          tau[h] = key == 0u ? -INFINITY : key_float(key);
        }
      }
      const int64_t nsamp = MODE == kModeSample ? sampled_sectors(L0.n) : 0;

      auto epilogue = [&](int ti, uint32_t tt) -> bool {
        const int ab = (int)(tt & 1);
        if (s_fault || !mbar_wait(acc_full(ab), (tt >> 1) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const uint32_t taddr = tmem + lane_base + (uint32_t)(ab * kTcAccCols + 32 * (2 * hr + half));
          uint32_t v[32];
          tc_ld32(taddr, v);
          tc_st32_fill(taddr, kTcMagicBits);
          const int r = quarter + 4 * hr;
#pragma unroll
          for (int kq = 0; kq < 2; ++kq) {
            const int bit = 8 * (2 * half + kq) + r;  // key bit within the word
            float sc[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const uint32_t *a = v + 16 * kq + 4 * h;
              float x = __uint_as_float(a[3]) - kTcMagic;
              x = fmaf(x, 256.0f, __uint_as_float(a[2]) - kTcMagic);
              x = fmaf(x, 256.0f, __uint_as_float(a[1]) - kTcMagic);
              x = fmaf(x, 256.0f, __uint_as_float(a[0]) - kTcMagic);
              sc[h] = fmaf(x, Dh[h][hr], Kh[h]);
            }
            if (MODE == kModeSample) {
              const int64_t sj = (int64_t)ti * kTcSampleSectorsPerTile + (lane >> 3);
              if (sj < nsamp) {
                const int64_t tok = (sj * kSampleStride * kSectorWords + (lane & 7)) * 32 + bit;
                const int64_t sl = sj * 256 + (lane & 7) * 32 + bit;
#pragma unroll
                for (int h = 0; h < G; ++h)
                  p.sample[(head0 + h) * p.m_max + sl] = tok < L0.n ? float_key(sc[h]) : 0u;
              }
            } else {
              const int64_t tok = ((int64_t)ti * kTcTileWords + lane) * 32 + bit;
              const bool valid = tok < L0.n;
              if (p.debug_scores && valid) {
#pragma unroll
                for (int h = 0; h < G; ++h) p.debug_scores[(head0 + h) * L0.n + tok] = sc[h];
              }
              bool take[G], any = false;
#pragma unroll
              for (int h = 0; h < G; ++h) {
                take[h] = valid && sc[h] >= tau[h];
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
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty(ab));
        return true;
      };

      uint32_t i = it, tt = tj;
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j, ++tt) {
        const int ti = ti0 + j;
        for (int c = 0; c < nch; ++c, ++i) {
          const int st = (int)(i % kTcNumStages);
          const int b = (int)(i % kTcNumABuf);
          if (s_fault || !mbar_wait(stage_full(st), (i / kTcNumStages) & 1)) {
            ok = false;
            break;
          }
          if (i >= (uint32_t)kTcNumABuf &&
              (s_fault || !mbar_wait(a_empty(b), ((i / kTcNumABuf) - 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int p0 = c * kTcChunkPlanes + 16 * half;  // first plane of this warp's K-step
          if (p0 < P) {
            const uint32_t *srow =
                reinterpret_cast<const uint32_t *>(sStage + st * kTcStageBytes) + 16 * half * 32 + lane;
            uint32_t cell[4][8];
            if (!big) {
#pragma unroll
              for (int pr = 0; pr < 8; ++pr) {
                const uint32_t x0 = srow[(2 * pr) * 32];
                const uint32_t x1 = srow[(2 * pr + 1) * 32];
                const uint32_t c0 = __byte_perm(x0, x1, 0x5410);  // keys kk = 0, 1
                const uint32_t c1 = __byte_perm(x0, x1, 0x7632);  // keys kk = 2, 3
                cell[0][pr] = c0 & m0;
                cell[1][pr] = c1 & m0;
                cell[2][pr] = c0 & m1;
                cell[3][pr] = c1 & m1;
              }
            } else {
#pragma unroll
              for (int pr = 0; pr < 8; ++pr) {
                const uint32_t x0 = srow[(2 * pr) * 32];
                const uint32_t x1 = srow[(2 * pr + 1) * 32];
                const uint32_t c0 = __byte_perm(x0, x1, 0x5410);
                const uint32_t c1 = __byte_perm(x0, x1, 0x7632);
                cell[0][pr] = (c0 >> quarter) & 0x01010101u;
                cell[1][pr] = (c1 >> quarter) & 0x01010101u;
                cell[2][pr] = (c0 >> (quarter + 4)) & 0x01010101u;
                cell[3][pr] = (c1 >> (quarter + 4)) & 0x01010101u;
              }
            }
            const uint32_t acol = tmem + lane_base + (uint32_t)(kTcAColBase + b * kTcABufCols + 8 * half);
#pragma unroll
            for (int mb = 0; mb < 4; ++mb) tc_st8(acol + (uint32_t)(16 * mb), cell[mb]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(stage_empty(st));
          tc_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(a_full(b));
        }
        if (!ok) break;
        // the previous tile's MMAs ran while this tile was being built
        if (j > 0 && !epilogue(ti - 1, tt - 1)) ok = false;
      }
      if (ok && !epilogue(ti0 + ntiles - 1, tj + ntiles - 1)) ok = false;
      if (!ok) s_fault = 1;
    }
    it += (uint32_t)(ntiles * nch);
    tj += (uint32_t)ntiles;
    t = seg_end;
  }

  // ---- teardown ------------------------------------------------------------
  // every commit must have landed before the block's barriers and tensor
  // memory go away (on the normal path they have; after a fault, wait)
  if (warp == kTcMmaWarp && lane == 0) {
    if (last_item >= 0)
      mbar_wait(a_empty(last_item % kTcNumABuf), ((uint32_t)last_item / kTcNumABuf) & 1);
    if (last_tile >= 0) mbar_wait(acc_full(last_tile & 1), ((uint32_t)last_tile >> 1) & 1);
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
