// Per-query bit allocation by reverse water-filling (method paragraph 3 of
// "Fathom Makes KV-Cache Scans Query-Adaptive...": more bits go to the
// channels that matter more for the current query, in closed form; abstract
// of arXiv 2609.17652: "over the variance-weighted importance of its
// channels").
//
// Closed form: b_c = clip(log2(w_c / theta) / 2, 0, 4), sum_c b_c = B, with
// w_c = q_c^2 sigma_c^2.  Its exact integer form: each channel offers four
// slots (c, tau) worth w_c 4^-tau (the distortion one more bit removes);
// take the B most valuable, ties to the lower channel then lower tau.
// t_c = channel c's slots taken.
//
// One warp per query head.  The water level is found without any log2: the
// slot values are non-negative doubles, whose bit patterns order like the
// values, so the warp bisects the 64-bit pattern space for the largest
// level L with #{slots >= L} >= B (63 rounds of compare + warp-sum).  Slots
// above L are taken; slots equal to L are taken in (channel, tau) order
// until B is reached.  Every lane owns d/32 consecutive channels, so a warp
// prefix sum orders the ties by channel.  Bit-exact with any other exact
// evaluation of the same ordering: w_c is q*q times sigma*sigma in fp64
// (both squares exact), and the slot values are exact power-of-two scalings.
#include "fathom_internal.cuh"

namespace fathom {

template <int CPL>
__global__ void __launch_bounds__(128) allocate_kernel(const void *__restrict__ q, int q_bf16,
                                                       const float *__restrict__ sigma, int h_q,
                                                       int G, int budget,
                                                       uint8_t *__restrict__ alloc) {
  constexpr int d = CPL * 32;
  const int h = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (h >= h_q) return;
  const int g = h / G;

  unsigned long long key[CPL][4];
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const int c = lane * CPL + i;
    const double qv = (double)load_q(q, q_bf16, (int64_t)h * d + c);
    const double sv = (double)sigma[(int64_t)g * d + c];
    const double w = (qv * qv) * (sv * sv);
    key[i][0] = (unsigned long long)__double_as_longlong(w);
    key[i][1] = (unsigned long long)__double_as_longlong(w * 0.25);
    key[i][2] = (unsigned long long)__double_as_longlong(w * 0.0625);
    key[i][3] = (unsigned long long)__double_as_longlong(w * 0.015625);
  }

  int t[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) t[i] = 0;

  if (budget > 0) {
    // largest level L with #{slots >= L} >= budget
    unsigned long long lo = 0ull, hi = 0x7ff0000000000000ull;
    while (hi - lo > 1ull) {
      const unsigned long long mid = lo + ((hi - lo) >> 1);
      unsigned cnt = 0;
#pragma unroll
      for (int i = 0; i < CPL; ++i)
#pragma unroll
        for (int tau = 0; tau < 4; ++tau) cnt += key[i][tau] >= mid ? 1u : 0u;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= (unsigned)budget) lo = mid; else hi = mid;
    }
    unsigned gt = 0, ties = 0;
#pragma unroll
    for (int i = 0; i < CPL; ++i)
#pragma unroll
      for (int tau = 0; tau < 4; ++tau) {
        gt += key[i][tau] > lo ? 1u : 0u;
        ties += key[i][tau] == lo ? 1u : 0u;
      }
    const unsigned rem = (unsigned)budget - __reduce_add_sync(0xffffffffu, gt);
    // exclusive prefix of ties over lanes (lanes hold channels in order)
    unsigned incl = ties;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    unsigned seen = incl - ties;
#pragma unroll
    for (int i = 0; i < CPL; ++i)
#pragma unroll
      for (int tau = 0; tau < 4; ++tau) {
        if (key[i][tau] > lo) {
          t[i] += 1;
        } else if (key[i][tau] == lo) {
          if (seen < rem) t[i] += 1;
          seen += 1;
        }
      }
  }
#pragma unroll
  for (int i = 0; i < CPL; ++i) alloc[(int64_t)h * d + lane * CPL + i] = (uint8_t)t[i];
}

cudaError_t launch_allocate(const void *q, int q_bf16, const float *sigma, int h_q, int h_kv, int d,
                            int budget, uint8_t *alloc, cudaStream_t stream) {
  const int G = h_q / h_kv;
  const dim3 grid((unsigned)((h_q + 3) / 4));
  switch (d / 32) {
#define FATHOM_ALLOC_CASE(C)                                                              \
  case C:                                                                                 \
    allocate_kernel<C><<<grid, 128, 0, stream>>>(q, q_bf16, sigma, h_q, G, budget, alloc); \
    break;
    FATHOM_ALLOC_CASE(1)
    FATHOM_ALLOC_CASE(2)
    FATHOM_ALLOC_CASE(3)
    FATHOM_ALLOC_CASE(4)
    FATHOM_ALLOC_CASE(5)
    FATHOM_ALLOC_CASE(6)
    FATHOM_ALLOC_CASE(7)
    FATHOM_ALLOC_CASE(8)
#undef FATHOM_ALLOC_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace fathom
