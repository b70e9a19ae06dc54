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
//   B [planes x (head, digit)] = X_hp = W_hp / Delta_h rounded to an integer
//     (|X| < 2^30) in four signed base-256 int8 digits d_0..d_3 (0 where the
//     head does not read the plane),
// accumulated exactly in int32 by the tensor cores.  With a_m the
// accumulator of digit m, U = 256 a_3 + a_2 and L = 256 a_1 + a_0 are exact
// int32 values and
//   s_h = C_h + Delta_h 2^-e (65536 U + L)
// (e below).  The epilogue decides a key against the head's threshold on U
// alone, with a bound on |L| folded into an integer threshold per head, and
// forms the fp32 score only for the keys that pass.  Under per-token-group
// quantiser statistics m_c and s_c (so W, C_h and Delta_h) are those of the
// key's token group: each token group has its own plan, and a run of tiles is
// cut into segments at token-group boundaries.
//
// Layout (B200 design).  A tile is 1024 keys of one KV head: 32 plane words
// per plane row.  Tensor-memory lane 32 q + l (quarter q, lane l) of M-block
// r (r < 8) stands for key 32 l + 8 q + r of the tile: word l, byte q, bit r.
// Plane rows are taken four at a time; byte q of the four rows' word l forms
// T = [x0.byte q, x1.byte q, x2.byte q, x3.byte q] and M-block r of lane
// (q, l) receives the 32-bit cell T & (0x01010101 << r): four u8 K elements,
// one per plane, each 0 or 2^r (undone by the epilogue's scale 2^-r, e = r).
// When P > 256 the cells hold 0/1 instead (e = 0), so that the int32
// accumulators cannot overflow.
//
// Tensor memory (512 columns): two accumulator buffers of one tile each
// (8 M-blocks x N = 16 columns) and four A slots of one K-step each (8
// M-blocks x 8 columns: 32 planes of u8).
//
// Warp roles (one 672-thread CTA per SM, persistent over a contiguous run of
// tiles).  Each hand-over moves one K-step (4 KB of plane words, 1024 keys x
// 32 planes): the per-hand-over work of every role (waits, barrier and
// address arithmetic) is paid once per 4 KB.
//  * epilogue warps 0-7: warp (quarter q, half hh) reads M-blocks 4hh..4hh+3
//    of the lanes of quarter q of a finished tile (tcgen05.ld) and tests,
//    writes or samples those keys.  A key that may clear a head's threshold
//    is staged in the warp's own shared-memory region as its exact integer
//    parts (U, L, index); when a region might not hold another tile's keys,
//    and at the end of a run, the warp scores its staged keys in fp64, tests
//    them exactly and writes them to the workspace, one global atomic per
//    head reserving room for all of them (no barrier between epilogue warps);
//  * build warps 8-15: warp (quarter q, parity) turns the T values of the
//    K-steps of its parity into cells and stores them in the K-step's A slot
//    with tcgen05.st;
//  * load warps 16-19: warps 16 + 2w and 17 + 2w load the K-steps u = w
//    (mod 2).  Thread (plane quad i, word quad m) copies words 4m..4m+3 of
//    four plane rows with 16-byte cp.async copies (a row's 128 bytes come
//    from 8 threads) into its own slots of a raw ring in shared memory, seven
//    of its K-steps ahead, transposes the bytes into T and stores them in an
//    eight-stage ring, where a build warp reads its T values without bank
//    conflicts.  Four load warps keep about 56 KB of copies in flight per SM
//    while holding no plane words in registers;
//  * MMA warp 20: one elected thread issues the eight MMAs (M-blocks) and one
//    commit of every K-step (measured on B200: a thread issues an N = 16 MMA
//    about every 11 cycles, near the tensor pipe's rate for this shape), so
//    every accumulator is fed in order by that thread.
// Stages, A slots and accumulator buffers are handed over with mbarriers.
// Every wait is bounded in time; a timeout records a device fault in the
// workspace status, every role stops, and no further MMA is issued.
#include <limits.h>

#include <type_traits>

#include "fathom_internal.cuh"

namespace fathom {

// ---------------------------------------------------------------- layout --
constexpr int kTcTileWords = 32;   // 1024 keys per tile
constexpr int kTcKStep = 32;       // planes per MMA (K = 32 int8)
constexpr int kTcMBlocks = 8;      // one per bit position r of a code byte
constexpr int kTcN = 16;           // (head, digit) columns
constexpr int kTcAccCols = kTcMBlocks * kTcN;           // 128: one tile's accumulators
constexpr int kTcAccBufs = 2;
constexpr int kTcASlotCols = kTcMBlocks * (kTcKStep / 4);  // 64: one K-step's cells
constexpr int kTcASlots = 4;
constexpr int kTcAColBase = kTcAccBufs * kTcAccCols;    // 256
constexpr int kTcTmemCols = 512;
static_assert(kTcAColBase + kTcASlots * kTcASlotCols <= kTcTmemCols, "tensor memory budget");

constexpr int kTcEpiWarp0 = 0;                           // warps 0-7
constexpr int kTcEpiWarps = 8;
constexpr int kTcBuildWarp0 = kTcEpiWarp0 + kTcEpiWarps;  // warps 8-15
constexpr int kTcBuildPerQuarter = 2;
constexpr int kTcBuildWarps = 4 * kTcBuildPerQuarter;
constexpr int kTcLoadWarp0 = kTcBuildWarp0 + kTcBuildWarps;  // warps 16-19
constexpr int kTcLoadWarps = 4;
constexpr int kTcLoadPairs = kTcLoadWarps / 2;  // pair w loads the K-steps u = w (mod 2)
constexpr int kTcMmaWarp0 = kTcLoadWarp0 + kTcLoadWarps;  // warp 20
constexpr int kTcMmaWarps = 1;
constexpr int kTcWarps = kTcMmaWarp0 + kTcMmaWarps;
constexpr int kTcThreads = 32 * kTcWarps;                // 672
static_assert(kTcBuildWarp0 % 4 == 0 && kTcEpiWarp0 % 4 == 0,
              "a warp reaches the tensor-memory lanes of quarter warp % 4");

constexpr int kTcStages = 8;       // shared-memory ring of K-steps
// A stage holds T[plane quad i][quarter q][word w] (4 KB): the 16-byte stores
// of a load warp's quarter warp (one plane quad, eight word quads) and the
// word loads of a build warp both cover 32 consecutive words.
constexpr int kTcStageWords = 8 * 4 * kTcTileWords;
// K-steps each load thread keeps in flight: 16-byte cp.async copies into a
// ring of raw plane words in shared memory (its own four rows of each
// K-step, so the ring needs no barrier); the registers hold none of it.
constexpr int kTcRawDepth = 8;
constexpr int kTcRawWords = kTcKStep * kTcTileWords;  // one K-step: 32 rows x 32 words
// Candidates staged in shared memory per epilogue warp and head.  A warp
// adds at most 128 per head and tile (its 32 lanes x 4 M-blocks), so a region
// holding more than kTcWarpCap - 128 is flushed before the next tile.
constexpr int kTcWarpCap = 192;
constexpr int kTcSampleSectorsPerTile = kTcTileWords / kSectorWords;  // 4

// B for one K-step: 16 rows (head, digit) x 32 int8 K elements (planes),
// K-major, no swizzle.  Core matrices are 8 rows x 16 bytes; the two 8-row
// groups are 128 B apart (SBO), the two 16-byte K halves 256 B apart (LBO).
constexpr int kTcBStepBytes = 512;
constexpr uint32_t kTcSBO = 128;
constexpr uint32_t kTcLBO = 256;
// Instruction descriptor: D s32, A u8 K-major (tensor memory), B s8
// K-major, N = 16, M = 128, dense.
constexpr uint32_t kTcIdesc = (2u << 4)                        // D format s32
                              | (0u << 7)                      // A format u8
                              | (1u << 10)                     // B format s8
                              | (0u << 15)                     // A K-major
                              | (0u << 16)                     // B K-major
                              | ((uint32_t)(kTcN >> 3) << 17)  // N
                              | ((128u >> 4) << 24);           // M
// A plane count above which the cells hold 0/1 instead of 0/2^e.  With 0/2^e
// (e <= 7) and P <= 256, |a_m| <= 2^7 * 128 * 256 = 2^22, so U and L fit in
// int32; with 0/1 and P <= 1024, |a_m| <= 2^17.
constexpr int kTcSmallP = 256;

struct TcPlanHeader {
  int P;           // union planes of the group
  int nks;         // max(1, ceil(P / 32)): K-steps of 32 planes with a B block
  int big;         // P > kTcSmallP: cells hold 0/1
  int pad0;
  double K[4];     // C_h (fp64: a score is formed in fp64 and rounded once)
  float D[4];      // Delta_h (a power of two)
  float Wsum[4];   // sum over the planes head h reads of |W_hp|
  uint32_t Lsum[4];  // sum over those planes of |256 d_1 + d_0| (bounds |L| / 2^e)
};
static_assert(sizeof(TcPlanHeader) == 96, "header size");

struct TcPlanLayout {
  int off_rows;  // uint16 [4 d]: c * 4 + j of the union planes, channel-major (first P written)
  int off_b;     // int8 [ceil(4 d / 32)][512]: B of every K-step
  int bytes;
};

__host__ __device__ inline TcPlanLayout tc_plan_layout(int d) {
  TcPlanLayout L;
  L.off_rows = (int)sizeof(TcPlanHeader);
  L.off_b = (L.off_rows + 2 * 4 * d + 127) & ~127;
  L.bytes = L.off_b + ((4 * d + kTcKStep - 1) / kTcKStep) * kTcBStepBytes;
  return L;
}

int tc_plan_bytes(int d) { return tc_plan_layout(d).bytes; }

// Shared memory of the scan kernel, in bytes from the (128-byte aligned) base.
struct TcSmem {
  int stage, raw, plan, rows, cand, tprefix, bytes;
};
__host__ __device__ inline TcSmem tc_smem_layout(int d, int S) {
  TcSmem m;
  int o = 0;
  m.stage = o;
  o += kTcStages * kTcStageWords * 4;
  m.raw = o;
  o += kTcLoadPairs * kTcRawDepth * kTcRawWords * 4;
  m.plan = o;  // 128-byte aligned (B blocks are read by the MMAs)
  o += (tc_plan_layout(d).bytes + 127) & ~127;
  m.rows = o;  // uint32 row index of every union-plane slot
  o += 4 * 4 * d;
  m.cand = o;  // int4 {U, L, index, 0} per staged candidate, [warp][head][kTcWarpCap]
  o += kTcEpiWarps * 4 * kTcWarpCap * 16;
  m.tprefix = o;
  o += 4 * (S + 1);
  m.bytes = o;
  return m;
}

static int tc_smem_bytes(int d, int S) {
  const int b = tc_smem_layout(d, S).bytes + 128;  // + alignment slack
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
// Non-blocking probe of the phase with the given parity.
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
// try_wait may suspend the thread for a system-dependent time until the phase
// completes (an explicit suspend-time hint measured slower on B200: the
// woken warps resumed late).
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
// Waits for the phase, giving up after about a second (2^31 cycles).
// Returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (clock64() - t0 > (1ll << 31)) return false;
  }
}

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros.
__device__ __forceinline__ void tc_cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void tc_cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
// Waits until at most N of this thread's committed copy groups are pending.
template <int N>
__device__ __forceinline__ void tc_cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// D[tmem_d] (+)= A[tmem_a] x B[bdesc]; accumulate = 0 overwrites D.
__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(kTcIdesc), "r"(accumulate)
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

// Arrives once on the mbarrier when every tcgen05 operation this thread
// issued before has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
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

// 32 columns of this warp's 32 lanes; the caller waits (tc_wait_ld) before
// using them.
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
}
__device__ __forceinline__ void tc_wait_ld() {
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

// The fp32 score of a key from its exact integer parts; every path that
// reports, samples or filters a score forms it this way.  De = Delta_h 2^-e
// (a power of two).  65536 U + L (< 2^47) and its product with De are exact
// in fp64, so the score is C_h + Delta_h 2^-e V rounded once in fp64 and once
// to fp32: the fp32 cancellation of C_h against the plane sum never enters.
__device__ __forceinline__ float tc_score(int U, int L, float De, double K) {
  const double v = fma((double)U, 65536.0, (double)L);
  return (float)fma(v, (double)De, K);
}

// 2^-e as a float, 0 <= e <= 7.
__device__ __forceinline__ float tc_pow2_neg(int e) { return __int_as_float((127 - e) << 23); }

// ------------------------------------------------------------ plan kernel --

// One block of 256 threads per plan: (session, KV head, token group), the
// token group only under per-token-group statistics; thread c is channel c.
__global__ void __launch_bounds__(256) tc_plan_kernel(ScanParams p) {
  grid_dependency_wait();
  allow_dependent_launch();
  // clear the workspace's status, counters and thresholds (read by the
  // kernels after this one)
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.zero_words; i += gridDim.x * blockDim.x)
    p.zero[i] = 0u;
  const int pid = blockIdx.x;
  const int gid = pid / p.n_tgroups;  // (session, KV head)
  const int tg = pid - gid * p.n_tgroups;
  const int s = gid / p.h_kv;
  const int g = gid - s * p.h_kv;
  const fathom_session &se = session_of(p, s);
  const int d = p.d, G = p.G;
  const int c = threadIdx.x;
  const TcPlanLayout L = tc_plan_layout(d);
  unsigned char *plan = p.plans + (size_t)pid * L.bytes;
  const int64_t srow = ((int64_t)g * p.n_tgroups + tg) * d;  // this plan's (m, s) row
  TcPlanHeader *hdr = reinterpret_cast<TcPlanHeader *>(plan);
  uint16_t *rows = reinterpret_cast<uint16_t *>(plan + L.off_rows);
  int8_t *bmat = reinterpret_cast<int8_t *>(plan + L.off_b);

  __shared__ int s_tmp[32];
  __shared__ double s_red[4][8];
  __shared__ double s_wsum[4][8];
  __shared__ unsigned s_lsum[4][8];
  __shared__ unsigned long long s_wmax[4];
  __shared__ int s_P;

  int t[4] = {0, 0, 0, 0};
  double w[4] = {0.0, 0.0, 0.0, 0.0};      // q_c s_c of a head that reads channel c
  double kpart[4] = {0.0, 0.0, 0.0, 0.0};  // its share of C_h
  int tstar = 0;
  if (c < d) {
    const double m = se.qmin[srow + c];
    const double sc = se.qscale[srow + c];
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
#pragma unroll
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
  for (int i = threadIdx.x; i < nks * kTcBStepBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4 *>(bmat)[i] = make_uint4(0, 0, 0, 0);
  double delta[4], inv_delta[4];
#pragma unroll
  for (int hh = 0; hh < 4; ++hh) {
    // the largest plane weight is 8 max_c |q_c s_c|; |W| / Delta < 2^30
    const double wmax = 8.0 * __longlong_as_double((long long)s_wmax[hh]);
    int ex = 0;
    frexp(wmax, &ex);  // wmax < 2^ex
    delta[hh] = wmax > 0.0 ? ldexp(1.0, ex - 30) : 1.0;
    inv_delta[hh] = wmax > 0.0 ? ldexp(1.0, 30 - ex) : 1.0;  // exact: a power of two
  }
  __syncthreads();  // B zeroed before the digits are written
  double wsum[4] = {0.0, 0.0, 0.0, 0.0};
  unsigned lsum[4] = {0u, 0u, 0u, 0u};
  for (int j = 0; j < tstar; ++j) {
    const int pl = off + j;
    rows[pl] = (uint16_t)(c * 4 + j);
    int8_t *bk = bmat + (size_t)(pl / kTcKStep) * kTcBStepBytes;
    const int k = pl % kTcKStep;
    const double pj = (double)(1 << (3 - j));  // 2^(3 - j), j <= 3
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) {
      if (hh >= G || j >= t[hh]) continue;
      // W / Delta scaled by powers of two only: exact, then rounded once
      long long x = __double2ll_rn(w[hh] * pj * inv_delta[hh]);
      wsum[hh] += fabs(w[hh] * pj);
      int dig[4];
#pragma unroll
      for (int dg = 0; dg < 4; ++dg) {
        const long long v = dg < 3 ? ((x + 128) & 255) - 128 : x;
        x = (x - v) >> 8;
        dig[dg] = (int)v;
        const int n = hh * 4 + dg;
        bk[(n >> 3) * kTcSBO + (k >> 4) * kTcLBO + (n & 7) * 16 + (k & 15)] = (int8_t)v;
      }
      lsum[hh] += (unsigned)abs(256 * dig[1] + dig[0]);
    }
  }
#pragma unroll
  for (int hh = 0; hh < 4; ++hh) {
    double a = wsum[hh];
    unsigned b = lsum[hh];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      b += __shfl_xor_sync(0xffffffffu, b, o);
    }
    if (lane == 0) {
      s_wsum[hh][warp] = a;
      s_lsum[hh][warp] = b;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    hdr->P = P;
    hdr->nks = nks;
    hdr->big = P > kTcSmallP ? 1 : 0;
    hdr->pad0 = 0;
    const int nw = (blockDim.x + 31) >> 5;
    for (int hh = 0; hh < 4; ++hh) {
      double sum = 0.0, ws = 0.0;
      unsigned ls = 0u;
      for (int wv = 0; wv < nw; ++wv) {
        sum += s_red[hh][wv];
        ws += s_wsum[hh][wv];
        ls += s_lsum[hh][wv];
      }
      hdr->K[hh] = hh < G ? sum : 0.0;
      hdr->D[hh] = (float)delta[hh];
      hdr->Wsum[hh] = (float)ws;
      hdr->Lsum[hh] = ls;
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

// Tiles per token group under per-token-group statistics (0 without them).
// A filtering tile covers 1024 keys; a sample tile covers 65536 (it reads the
// first 256-key sector of four 64-sector strides), and a token group is a
// multiple of 65536 keys, so every tile lies in one token group.
template <int MODE>
__device__ __forceinline__ int tc_tiles_per_tgroup(const ScanParams &p) {
  if (p.token_group <= 0) return 0;
  const int64_t span = MODE == kModeSample
                           ? (int64_t)kTcSampleSectorsPerTile * kSampleStride * kSectorWords * 32
                           : (int64_t)kTcTileWords * 32;
  return (int)(p.token_group / span);
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
  L.n = session_n(p, lo);
  L.W = plane_words(L.n);
  L.planes = se.planes;
  L.per = (int)tc_tiles_per_group<MODE>(L.n, p);
  const int r = t - s_tprefix[lo];
  L.g = r / L.per;
  L.ti = r - L.g * L.per;
  return L;
}

// A block whose tiles span two plans ((session, KV head) groups, or token
// groups) drains its pipeline between them.  The cost line charges the drain
// at (session, KV head) boundaries only: token groups are 64 or more tiles
// long, so a run crosses at most one or two of them.  The filtering pass splits the tiles over the blocks on a
// cost line on which every group is preceded by that overhead, so that a
// block that crosses a group boundary takes correspondingly fewer tiles.
// Costs are in half tiles.
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
  const int per = (int)tc_tiles_per_group<MODE>(session_n(p, lo), p);
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

// The fp32 score and composite of a staged candidate; tau_h decides it.
__device__ __forceinline__ float tc_record_score(const TcPlanHeader *hdr, int h, int U, int L,
                                                 uint32_t tok) {
  const int e = hdr->big ? 0 : (int)(tok & 7u);  // key 32 l + 8 q + r of a tile: r = tok & 7
  return tc_score(U, L, hdr->D[h] * tc_pow2_neg(e), hdr->K[h]);
}

// DEBUG (filtering pass only): also write every score to p.debug_scores; a
// separate instance, so that the scan's hot loop carries none of it.
template <int G, int MODE, bool DEBUG>
__global__ void __launch_bounds__(kTcThreads, 1) tc_scan_kernel(ScanParams p) {
  // the prologue below (tile space, tensor memory, barriers) reads only the
  // call's inputs, so it overlaps the previous kernel; the plans, thresholds
  // and counters that kernel writes are read after grid_dependency_wait
  allow_dependent_launch();
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem =
      reinterpret_cast<unsigned char *>(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int d = p.d;
  const TcPlanLayout PL = tc_plan_layout(d);
  const TcSmem SM = tc_smem_layout(d, p.S);
  uint32_t *sStage = reinterpret_cast<uint32_t *>(smem + SM.stage);
  uint32_t *sRaw = reinterpret_cast<uint32_t *>(smem + SM.raw);
  unsigned char *sPlan = smem + SM.plan;
  uint32_t *sRow = reinterpret_cast<uint32_t *>(smem + SM.rows);
  int4 *sRec = reinterpret_cast<int4 *>(smem + SM.cand);
  int *s_tprefix = reinterpret_cast<int *>(smem + SM.tprefix);
  const TcPlanHeader *sHdr = reinterpret_cast<const TcPlanHeader *>(sPlan);
  const uint16_t *sRows16 = reinterpret_cast<const uint16_t *>(sPlan + PL.off_rows);

  constexpr int kBars = 2 * kTcStages + 2 * kTcASlots + 2 * kTcAccBufs + 1;
  __shared__ __align__(8) unsigned long long s_bar[kBars];
  __shared__ uint32_t s_tmem;
  __shared__ int s_tmp[32];
  __shared__ volatile int s_fault;
  __shared__ unsigned s_wcount[kTcEpiWarps][4];  // candidates staged per epilogue warp and head
  __shared__ float s_tau[4];
  // Integer thresholds of the run, [head][M-block]: a key whose fp32 score
  // reaches tau_h has U >= s_TU (the bound on |L| and on the score's rounding
  // folded in)
  __shared__ __align__(16) int s_TU[4][kTcMBlocks];

  const uint32_t bar0 = tc_smem_u32(&s_bar[0]);
  auto stage_full = [=](int s) { return bar0 + 8u * (uint32_t)s; };
  auto stage_empty = [=](int s) { return bar0 + 8u * (uint32_t)(kTcStages + s); };
  auto a_full = [=](int s) { return bar0 + 8u * (uint32_t)(2 * kTcStages + s); };
  auto a_empty = [=](int s) { return bar0 + 8u * (uint32_t)(2 * kTcStages + kTcASlots + s); };
  auto acc_full = [=](int b) {
    return bar0 + 8u * (uint32_t)(2 * kTcStages + 2 * kTcASlots + b);
  };
  auto acc_empty = [=](int b) {
    return bar0 + 8u * (uint32_t)(2 * kTcStages + 2 * kTcASlots + kTcAccBufs + b);
  };
  const uint32_t drain_bar = bar0 + 8u * (uint32_t)(kBars - 1);
  // A wait that gives up records a fault; every role then leaves its loops.
  // Every lane waits on the barrier itself (measured faster on B200 than one
  // lane waiting and broadcasting the outcome); the warp goes on only when
  // all of its lanes saw the phase complete.
  auto warp_wait = [&](uint32_t bar, uint32_t parity) -> bool {
    bool ok = mbar_try(bar, parity);
    if (!ok) {
      const long long t0 = clock64();
      while (!(ok = mbar_try(bar, parity))) {
        if (s_fault || clock64() - t0 > (1ll << 31)) break;
      }
    }
    if (!__all_sync(0xffffffffu, ok)) {
      s_fault = 1;
      return false;
    }
    return true;
  };
  auto warp_arrive = [&](uint32_t bar) {
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
  };

  // ---- tile space: every (session, KV head) contributes its tiles --------
  for (int base = 0; base < p.S; base += kTcThreads) {
    const int s = base + tid;
    int v = 0;
    if (s < p.S) v = (int)(tc_tiles_per_group<MODE>(session_n(p, s), p) * p.h_kv);
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

  // ---- tensor memory and barriers ----------------------------------------
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     tc_smem_u32(&s_tmem)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(stage_full(s), 2);   // the pair of load warps of the K-step
      mbar_init(stage_empty(s), 4);  // the four quarter build warps
    }
    for (int s = 0; s < kTcASlots; ++s) {
      mbar_init(a_full(s), 4);   // the four quarter build warps
      mbar_init(a_empty(s), 1);  // the MMA thread's commit
    }
    for (int b = 0; b < kTcAccBufs; ++b) {
      mbar_init(acc_full(b), 1);  // the MMA thread's commit at a tile's end
      mbar_init(acc_empty(b), kTcEpiWarps);  // every epilogue warp
    }
    mbar_init(drain_bar, kTcMmaWarps);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    s_fault = 0;
  }
  if (tid < 4 * kTcEpiWarps) (&s_wcount[0][0])[tid] = 0u;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int quarter = warp & 3;
  const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;

  grid_dependency_wait();

  // K-steps and tiles since the start of the kernel (every thread keeps the
  // same counts: they index the stages, slots, buffers and phases)
  uint32_t u0 = 0, tt0 = 0;

  // ---- segments: runs of tiles that share one plan -----------------------
  int t = t_begin;
  while (t < t_end) {
    __syncthreads();
    if (s_fault) break;
    const TcLoc L0 = tc_locate<MODE>(p, s_tprefix, t);
    // a segment is the run's tiles that share one plan (worked out by one
    // thread: measured faster than every thread doing it)
    if (tid == 0) {
      const int tpg = tc_tiles_per_tgroup<MODE>(p);
      const int tgx = tpg > 0 ? L0.ti / tpg : 0;
      const int plan_end = tpg > 0 ? min(L0.per, (tgx + 1) * tpg) : L0.per;
      s_tmp[2] = min(t_end, t - L0.ti + plan_end);
      s_tmp[3] = tgx;
    }
    __syncthreads();
    const int seg_end = s_tmp[2];
    const int tg = s_tmp[3];
    const int ntiles = seg_end - t;
    const int ti0 = L0.ti;
    const int gid = L0.s * p.h_kv + L0.g;
    {
      const unsigned char *gplan = p.plans + ((size_t)gid * p.n_tgroups + tg) * PL.bytes;
      const int nk = reinterpret_cast<const TcPlanHeader *>(gplan)->nks;
      const int used = PL.off_b + nk * kTcBStepBytes;
      for (int i = tid; i < used / 16; i += kTcThreads)
        reinterpret_cast<uint4 *>(sPlan)[i] = reinterpret_cast<const uint4 *>(gplan)[i];
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // B is read by the MMAs
      if (tid < G) {
        float tau = -INFINITY;
        if (MODE == kModeFilter) {
          const uint32_t key = p.tau[(int64_t)L0.s * p.h_q + L0.g * G + tid];
          tau = key == 0u ? -INFINITY : key_float(key);
        }
        s_tau[tid] = tau;
      }
    }
    __syncthreads();
    const int P = sHdr->P;
    const int nks = sHdr->nks;
    const bool big = sHdr->big != 0;
    // row (c * 4 + j < 4 d) of every union-plane slot; a padding slot of a
    // plane quad that holds real planes repeats the quad's first row (its B
    // weights are zero); quads past P are never loaded
    for (int r = tid; r < nks * kTcKStep; r += kTcThreads) {
      const int src = r < P ? r : (r & ~3);
      const uint32_t row = src < P ? (uint32_t)sRows16[src] : 0u;
      sRow[r] = row < (uint32_t)(4 * d) ? row : 0u;
    }
    if (tid < 32) {
      // s = K + D 2^-e (65536 U + L) >= tau with |L| <= 2^e Lsum needs
      // U >= ((tau - K - eps) 2^e / D - 2^e Lsum) / 65536, eps covering the
      // rounding of s; one less than its floor, to be safe
      const int h = tid >> 3, r = tid & 7;
      int tu = INT_MIN;
      if (MODE == kModeFilter && h < G && s_tau[h] != -INFINITY) {
        const double tau = s_tau[h], K = sHdr->K[h], D = sHdr->D[h];
        const double eps = ldexp(fabs(tau) + fabs(K) + (double)sHdr->Wsum[h], -20);
        const double sc = ldexp(1.0, big ? 0 : r);  // 2^e
        const double x = (tau - K - eps) * sc / D - (double)sHdr->Lsum[h] * sc;
        const double y = floor(x / 65536.0) - 1.0;
        tu = y < -2147483648.0 ? INT_MIN : (y > 2147483647.0 ? INT_MAX : (int)y);
      }
      s_TU[h][r] = tu;
    }
    __syncthreads();
    const int64_t head0 = (int64_t)L0.s * p.h_q + L0.g * G;
    const int nkst = ntiles * nks;  // K-steps of the run, tile by tile

    if (warp >= kTcLoadWarp0 && warp < kTcMmaWarp0) {
      // --------------------------------------------------------------- load --
      // Each pair of load warps loads every other K-step; thread (plane quad
      // qi, word quad m) copies words 4m..4m+3 of rows 4qi..4qi+3 into its
      // slots of the pair's raw ring, kTcRawDepth - 1 of its K-steps ahead,
      // then transposes them.
      const int t64 = (((warp - kTcLoadWarp0) & 1) << 5) | lane;
      const int qi = t64 >> 3;
      const int m = t64 & 7;
      const int wpar = (warp - kTcLoadWarp0) >> 1;  // this pair loads the K-steps u = wpar (mod 2)
      const int vfirst = (int)((uint32_t)(wpar + 2 - (int)(u0 & 1u)) & 1u);
      const uint32_t *gbase = L0.planes + (int64_t)L0.g * d * 4 * L0.W;
      const int64_t nsamp = MODE == kModeSample ? sampled_sectors(L0.n) : 0;
      const int64_t wlast = L0.W - 4;  // words past the data hold keys the epilogue drops
      auto quad_word = [&](int ti) -> int64_t {
        int64_t gw;
        if (MODE == kModeSample) {
          const int64_t sj = (int64_t)ti * kTcSampleSectorsPerTile + (m >> 1);
          gw = sj * kSampleStride * kSectorWords + (m & 1) * 4;
          if (sj >= nsamp) gw = wlast;
        } else {
          gw = (int64_t)ti * kTcTileWords + m * 4;
        }
        return gw < wlast ? gw : wlast;
      };
      // raw ring slot of this thread's row j for K-step v
      auto raw_at = [&](int v, int j) -> uint32_t * {
        return sRaw + ((v >> 1) % kTcRawDepth) * kTcRawWords + (4 * qi + j) * kTcTileWords + 4 * m +
               wpar * (kTcRawDepth * kTcRawWords);
      };
      int ltl = vfirst / nks, lk = vfirst - (vfirst / nks) * nks;  // cursor of the next K-step to copy
      auto copy_next = [&](int lv) {
        if (lv < nkst) {
          const int64_t gw = quad_word(ti0 + ltl);
          const uint4 o = *reinterpret_cast<const uint4 *>(sRow + lk * kTcKStep + 4 * qi);
          const bool real = kTcKStep * lk + 4 * qi < P &&
                            in_bounds(max(max(o.x, o.y), max(o.z, o.w)) < (uint32_t)(4 * d) &&
                                          gw >= 0 && gw + 4 <= L0.W,
                                      p.status);
          const uint32_t rows[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tc_cp_async16(tc_smem_u32(raw_at(lv, j)),
                          real ? (const void *)(gbase + (int64_t)rows[j] * L0.W + gw)
                               : (const void *)gbase,
                          real ? 16u : 0u);
          lk += 2;
          while (lk >= nks) { lk -= nks; ++ltl; }
        }
        tc_cp_async_commit();  // one group per K-step (empty past the end)
      };
#pragma unroll 1
      for (int j = 0; j < kTcRawDepth - 1; ++j) copy_next(vfirst + 2 * j);
      for (int v = vfirst; v < nkst; v += 2) {
        copy_next(v + 2 * (kTcRawDepth - 1));
        tc_cp_async_wait<kTcRawDepth - 1>();  // K-step v's copies have landed
        uint4 x[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) x[j] = *reinterpret_cast<const uint4 *>(raw_at(v, j));
        const uint32_t u = u0 + (uint32_t)v;
        const int s = (int)(u % kTcStages);
        if (u >= (uint32_t)kTcStages && !warp_wait(stage_empty(s), ((u / kTcStages) - 1) & 1))
          break;
        uint32_t *dst = sStage + s * kTcStageWords + qi * (4 * kTcTileWords) + 4 * m;
        uint32_t Tq[4][4];  // [quarter][word]
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const uint32_t x0 = (&x[0].x)[w], x1 = (&x[1].x)[w];
          const uint32_t x2 = (&x[2].x)[w], x3 = (&x[3].x)[w];
          const uint32_t a_lo = __byte_perm(x0, x1, 0x5140), a_hi = __byte_perm(x0, x1, 0x7362);
          const uint32_t b_lo = __byte_perm(x2, x3, 0x5140), b_hi = __byte_perm(x2, x3, 0x7362);
          Tq[0][w] = __byte_perm(a_lo, b_lo, 0x5410);
          Tq[1][w] = __byte_perm(a_lo, b_lo, 0x7632);
          Tq[2][w] = __byte_perm(a_hi, b_hi, 0x5410);
          Tq[3][w] = __byte_perm(a_hi, b_hi, 0x7632);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4 *>(dst + q * kTcTileWords) =
              make_uint4(Tq[q][0], Tq[q][1], Tq[q][2], Tq[q][3]);
        warp_arrive(stage_full(s));
      }
      tc_cp_async_wait<0>();  // no copy into the ring outlives the run
    } else if (warp >= kTcBuildWarp0 && warp < kTcLoadWarp0) {
      // ------------------------------------------------------------ build --
      // Warp (quarter q, parity) builds the K-steps u = parity (mod 2): the
      // cells of M-blocks 0-7 for its lanes, the 64 columns of the K-step's
      // slot, stored 32 columns (four M-blocks) at a time.
      const int par = (warp - kTcBuildWarp0) >> 2;
      // the cell form (0/2^r or 0/1) is fixed for the run: one loop each
      auto build_run = [&](auto big_c) {
        constexpr bool kBig = decltype(big_c)::value;
        for (int v = (int)((uint32_t)(par + kTcBuildPerQuarter - (int)(u0 % kTcBuildPerQuarter)) %
                           kTcBuildPerQuarter);
             v < nkst; v += kTcBuildPerQuarter) {
          const uint32_t u = u0 + (uint32_t)v;
          const int s = (int)(u % kTcStages);
          if (!warp_wait(stage_full(s), (u / kTcStages) & 1)) break;
          const uint32_t *src = sStage + s * kTcStageWords + quarter * kTcTileWords + lane;
          uint32_t T[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) T[i] = src[i * 4 * kTcTileWords];
          warp_arrive(stage_empty(s));
          const int slot = (int)(u % kTcASlots);
          // the slot was last read by the MMAs of K-step u - kTcASlots
          if (u >= (uint32_t)kTcASlots && !warp_wait(a_empty(slot), ((u / kTcASlots) - 1) & 1))
            break;
          const uint32_t acol = tmem + lane_base + (uint32_t)(kTcAColBase + slot * kTcASlotCols);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            uint32_t cell[32];
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
              const int r = 4 * hf + rr;
#pragma unroll
              for (int i = 0; i < 8; ++i)
                cell[8 * rr + i] = kBig ? (T[i] >> r) & 0x01010101u : T[i] & (0x01010101u << r);
            }
            tc_st32(acol + (uint32_t)(32 * hf), cell);
          }
          tc_wait_st();
          tc_fence_before();
          warp_arrive(a_full(slot));
        }
      };
      if (big)
        build_run(std::true_type());
      else
        build_run(std::false_type());
    } else if (warp < kTcEpiWarp0 + kTcEpiWarps) {
      // ---------------------------------------------------------- epilogue --
      // Warp (quarter q, half hh) holds, in lane l, keys 32 l + 8 q + r of
      // each tile for M-blocks r = 4 hh .. 4 hh + 3: accumulator columns
      // 16 r + 4 h + m, 64 columns read with two loads and one wait.
      const int hh = (warp - kTcEpiWarp0) >> 2;
      const int r0 = 4 * hh;
      const int nkeys = (int)L0.n;
      const int nsamp = MODE == kModeSample ? (int)sampled_sectors(L0.n) : 0;
      // this warp's staging: wRec[h][kTcWarpCap] records, wCnt[h] of them in use
      int4 *wRec = sRec + (warp - kTcEpiWarp0) * (4 * kTcWarpCap);
      unsigned *wCnt = s_wcount[warp - kTcEpiWarp0];
      // Flush of the staged keys of every head whose region holds more than
      // `above` of them: each is scored in fp64 and tested against tau_h
      // exactly (its composite, or 0, written back in place), then one global
      // atomic per head reserves the room of all its passing keys (the heads'
      // atomics in flight together), and the composites are written there.
      auto flush = [&](unsigned above) {
        const unsigned lt = (1u << lane) - 1u;
        unsigned kept = 0u;  // lane h: passing keys of head h
#pragma unroll 1
        for (int h = 0; h < G; ++h) {
          const unsigned nc = wCnt[h];
          if (nc <= above) continue;
          const float tau = s_tau[h];
          unsigned kh = 0u;
          for (unsigned i0 = 0; i0 < nc; i0 += 32) {
            const unsigned i = i0 + lane;
            bool keep = false;
            if (i < nc && in_bounds(i < (unsigned)kTcWarpCap, p.status)) {
              int4 *slot = &wRec[h * kTcWarpCap + i];
              const int4 rec = *slot;
              const float sc = tc_record_score(sHdr, h, rec.x, rec.y, (uint32_t)rec.z);
              keep = sc >= tau;
              *reinterpret_cast<unsigned long long *>(slot) =
                  keep ? composite(sc, (uint32_t)rec.z) : 0ull;
            }
            kh += (unsigned)__popc(__ballot_sync(0xffffffffu, keep));
          }
          if (lane == h) kept = kh;
        }
        unsigned base = 0u;
        if (lane < G && kept > 0u) base = atomicAdd(&p.counts[head0 + lane], kept);
        __syncwarp();
#pragma unroll 1
        for (int h = 0; h < G; ++h) {
          const unsigned nc = wCnt[h];
          if (nc <= above) continue;
          unsigned long long *dst = p.cand + (head0 + h) * p.cap;
          unsigned pos0 = __shfl_sync(0xffffffffu, base, h);
          for (unsigned i0 = 0; i0 < nc; i0 += 32) {
            const unsigned i = i0 + lane;
            unsigned long long cv = 0ull;
            if (i < nc && i < (unsigned)kTcWarpCap)
              cv = *reinterpret_cast<const unsigned long long *>(&wRec[h * kTcWarpCap + i]);
            const unsigned bal = __ballot_sync(0xffffffffu, cv != 0ull);
            if (cv != 0ull) {
              const int64_t pos = (int64_t)pos0 + __popc(bal & lt);
              if (pos < p.cap && in_bounds(head0 + h < (int64_t)p.S * p.h_q, p.status)) dst[pos] = cv;
            }
            pos0 += (unsigned)__popc(bal);
          }
        }
        __syncwarp();
        if (lane < G && wCnt[lane] > above) wCnt[lane] = 0u;
        __syncwarp();
      };
      for (int tl = 0; tl < ntiles; ++tl) {
        const uint32_t tt = tt0 + (uint32_t)tl;
        const int ab = (int)(tt % kTcAccBufs);
        if (!warp_wait(acc_full(ab), (tt / kTcAccBufs) & 1)) break;
        tc_fence_after();
        const uint32_t abase = tmem + lane_base + (uint32_t)(ab * kTcAccCols + 16 * r0);
        uint32_t a0[32], a1[32];
        tc_ld32(abase, a0);
        tc_ld32(abase + 32u, a1);
        tc_wait_ld();
        // column i of the warp's 64 (indexes are compile-time after unrolling)
        auto A = [&](int i) -> uint32_t { return i < 32 ? a0[i] : a1[i - 32]; };
        // every column this warp needs is in registers: the MMAs may refill it
        tc_fence_before();
        warp_arrive(acc_empty(ab));
        const int ti = ti0 + tl;
        if (MODE == kModeSample) {
          const int sj = ti * kTcSampleSectorsPerTile + (lane >> 3);
          const int wis = lane & 7;
          const int tok0 = (sj * kSampleStride * kSectorWords + wis) * 32 + 8 * quarter + r0;
          const int slot0 = sj * 256 + wis * 32 + 8 * quarter + r0;
          if (sj < nsamp &&
              in_bounds(slot0 + 4 <= p.m_max && head0 + G <= (int64_t)p.S * p.h_q, p.status)) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
              uint32_t kv[4];
#pragma unroll
              for (int rr = 0; rr < 4; ++rr) {
                const int c = 16 * rr + 4 * h;
                const int U = (int)(A(c + 3) << 8) + (int)A(c + 2);
                const int L = (int)(A(c + 1) << 8) + (int)A(c);
                const float De = sHdr->D[h] * tc_pow2_neg(big ? 0 : r0 + rr);
                kv[rr] = tok0 + rr < nkeys ? float_key(tc_score(U, L, De, sHdr->K[h])) : 0u;
              }
              *reinterpret_cast<uint4 *>(p.sample + (head0 + h) * p.m_max + slot0) =
                  make_uint4(kv[0], kv[1], kv[2], kv[3]);
            }
          }
        } else {
          const int tok0 = (ti * kTcTileWords + lane) * 32 + 8 * quarter + r0;
          if (DEBUG) {
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
              for (int rr = 0; rr < 4; ++rr) {
                const int c = 16 * rr + 4 * h;
                const int U = (int)(A(c + 3) << 8) + (int)A(c + 2);
                const int L = (int)(A(c + 1) << 8) + (int)A(c);
                const float De = sHdr->D[h] * tc_pow2_neg(big ? 0 : r0 + rr);
                if (tok0 + rr < nkeys)
                  p.debug_scores[(head0 + h) * (int64_t)nkeys + tok0 + rr] =
                      tc_score(U, L, De, sHdr->K[h]);
              }
          }
          // bit 4 h + rr: key tok0 + rr may clear head h's threshold
          uint32_t cm = 0u;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const int4 tu = *reinterpret_cast<const int4 *>(&s_TU[h][r0]);
            cm |= ((int)(a0[4 * h + 3] << 8) + (int)a0[4 * h + 2] >= tu.x ? 1u : 0u) << (4 * h);
            cm |= ((int)(a0[16 + 4 * h + 3] << 8) + (int)a0[16 + 4 * h + 2] >= tu.y ? 1u : 0u)
                  << (4 * h + 1);
            cm |= ((int)(a1[4 * h + 3] << 8) + (int)a1[4 * h + 2] >= tu.z ? 1u : 0u)
                  << (4 * h + 2);
            cm |= ((int)(a1[16 + 4 * h + 3] << 8) + (int)a1[16 + 4 * h + 2] >= tu.w ? 1u : 0u)
                  << (4 * h + 3);
          }
          // keys past n (only in a segment's last tile)
          if (tok0 + 3 >= nkeys) {
#pragma unroll
            for (int rr = 0; rr < 4; ++rr)
              if (tok0 + rr >= nkeys) cm &= ~(0x1111u << rr);
          }
          // stage each key that passed (rare: one in a few hundred) as its exact
          // parts in this warp's region
          if (__any_sync(0xffffffffu, cm != 0u)) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
#pragma unroll
              for (int rr = 0; rr < 4; ++rr) {
                if ((cm >> (4 * h + rr)) & 1u) {
                  const int c = 16 * rr + 4 * h;
                  const unsigned pos = atomicAdd(&wCnt[h], 1u);
                  if (in_bounds(pos < (unsigned)kTcWarpCap && tok0 + rr < nkeys, p.status))
                    wRec[h * kTcWarpCap + pos] =
                        make_int4((int)(A(c + 3) << 8) + (int)A(c + 2),
                                  (int)(A(c + 1) << 8) + (int)A(c), tok0 + rr, 0);
                }
              }
            }
            __syncwarp();
            // a region that might not hold another tile's keys is flushed now
            bool near_full = false;
#pragma unroll
            for (int h = 0; h < G; ++h) near_full |= wCnt[h] > (unsigned)(kTcWarpCap - 128);
            if (near_full) flush((unsigned)(kTcWarpCap - 128));
          }
        }
      }
      if (MODE == kModeFilter) {
        flush(0u);  // the run's remaining staged candidates
      }
    } else if (warp == kTcMmaWarp0) {
      // -------------------------------------------------------------- MMA --
      // One elected thread issues every MMA, in K-step order, so each
      // accumulator is fed in order.  M-block r of a K-step reads A columns
      // 8 r of the K-step's slot into columns 16 r of the tile's buffer; one
      // commit per K-step frees the slot.  (The whole warp runs the loop and
      // waits: measured faster on B200 than a loop in lane 0 alone.)
      const uint64_t b_desc0 = tc_smem_desc(tc_smem_u32(sPlan + PL.off_b), kTcLBO, kTcSBO);
      int tl = 0, kx = 0;
      for (int v = 0; v < nkst; ++v) {
        const uint32_t u = u0 + (uint32_t)v;
        const uint32_t tt = tt0 + (uint32_t)tl;
        const int ab = (int)(tt % kTcAccBufs);
        // a tile's first MMA needs its buffer read out by the epilogue
        if (kx == 0 && tt >= (uint32_t)kTcAccBufs &&
            !warp_wait(acc_empty(ab), ((tt / kTcAccBufs) - 1) & 1))
          break;
        const int slot = (int)(u % kTcASlots);
        if (!warp_wait(a_full(slot), (u / kTcASlots) & 1)) break;
        tc_fence_after();
        const uint32_t dcol = tmem + (uint32_t)(ab * kTcAccCols);
        const uint32_t acol = tmem + (uint32_t)(kTcAColBase + slot * kTcASlotCols);
        const uint64_t bd = b_desc0 + (uint64_t)(kx * (kTcBStepBytes >> 4));
        const uint32_t acc = kx > 0 ? 1u : 0u;
        if (tc_elect_one()) {
#pragma unroll
          for (int r = 0; r < kTcMBlocks; ++r)
            tc_mma(dcol + (uint32_t)(kTcN * r), acol + (uint32_t)(8 * r), bd, acc);
          tc_commit(a_empty(slot));
          if (kx == nks - 1) tc_commit(acc_full(ab));
        }
        __syncwarp();
        if (++kx == nks) {
          kx = 0;
          ++tl;
        }
      }
    }
    u0 += (uint32_t)nkst;
    tt0 += (uint32_t)ntiles;
    t = seg_end;
  }

  // ---- teardown ------------------------------------------------------------
  // Each MMA warp commits once more after its last MMA; when those commits
  // have arrived every MMA is complete.  Then the slots' last commits are
  // waited for, so that no arrival is pending when the barriers go away.
  __syncthreads();
  if (warp == kTcMmaWarp0) {
    if (tc_elect_one()) tc_commit(drain_bar);
    __syncwarp();
  }
  if (tid == 0) {
    if (!mbar_wait(drain_bar, 0)) s_fault = 1;
    if (!s_fault) {
      for (int back = 1; back <= kTcASlots; ++back) {
        if (u0 < (uint32_t)back) break;
        const uint32_t u = u0 - (uint32_t)back;
        if (!mbar_wait(a_empty((int)(u % kTcASlots)), (u / kTcASlots) & 1)) {
          s_fault = 1;
          break;
        }
      }
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

template <int G, int MODE, bool DEBUG>
static cudaError_t launch_tc_gm(const ScanParams &p, int sms, cudaStream_t stream) {
  const int smem = tc_smem_bytes(p.d, p.S);
  cudaError_t e = cudaFuncSetAttribute(tc_scan_kernel<G, MODE, DEBUG>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_dependent(tc_scan_kernel<G, MODE, DEBUG>, dim3(sms), dim3(kTcThreads), (size_t)smem,
                          stream, p);
}

cudaError_t launch_tc_plan(const ScanParams &p, cudaStream_t stream) {
  return launch_dependent(tc_plan_kernel, dim3(p.S * p.h_kv * p.n_tgroups), dim3(256), 0, stream,
                          p);
}

cudaError_t launch_tc_scan(const ScanParams &p, int mode, int sms, cudaStream_t stream) {
  if (mode == kModeSample) {
    switch (p.G) {
      case 1: return launch_tc_gm<1, kModeSample, false>(p, sms, stream);
      case 2: return launch_tc_gm<2, kModeSample, false>(p, sms, stream);
      case 4: return launch_tc_gm<4, kModeSample, false>(p, sms, stream);
    }
  } else if (p.debug_scores) {
    switch (p.G) {
      case 1: return launch_tc_gm<1, kModeFilter, true>(p, sms, stream);
      case 2: return launch_tc_gm<2, kModeFilter, true>(p, sms, stream);
      case 4: return launch_tc_gm<4, kModeFilter, true>(p, sms, stream);
    }
  } else {
    switch (p.G) {
      case 1: return launch_tc_gm<1, kModeFilter, false>(p, sms, stream);
      case 2: return launch_tc_gm<2, kModeFilter, false>(p, sms, stream);
      case 4: return launch_tc_gm<4, kModeFilter, false>(p, sms, stream);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace fathom
