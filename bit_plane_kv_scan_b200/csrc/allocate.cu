// Per-query bit allocation by reverse water-filling (method paragraph 3 of
// "Fathom Makes KV-Cache Scans Query-Adaptive...": more bits go to the
// channels that weigh most for the query at hand, in closed form; abstract
// of arXiv 2609.17652: the weights are the channels' variance-weighted
// importance).
//
// Closed form: b_c = clip(log2(w_c / theta) / 2, 0, 4), sum_c b_c = B, with
// w_c = q_c^2 sigma_c^2.  Its exact integer form: each channel offers four
// slots (c, tau) worth w_c 4^-tau (the distortion one more bit removes);
// take the B most valuable, ties to the lower channel then lower tau.
// t_c = channel c's slots taken.
//
// One block per query head, one thread per slot (slot s = 4 c + tau, so the
// thread order is the tie order).  The B-th most valuable slot value L is
// found by an exact radix select over the 64-bit patterns of the slot values
// (non-negative doubles order like their bit patterns): eight passes of an
// 8-bit digit histogram.  Slots above L are taken; slots equal to L are taken
// in slot order until B is reached (a block prefix count).  No log2 is
// needed, and the result is bit-exact with any exact evaluation of the same
// ordering: w_c is q*q times sigma*sigma in fp64 (both squares exact), and
// the slot values are exact power-of-two scalings.
#include "fathom_internal.cuh"

namespace fathom {

__global__ void __launch_bounds__(1024) allocate_kernel(const void *__restrict__ q, int q_bf16,
                                                        const float *__restrict__ sigma, int G,
                                                        int d, int budget,
                                                        uint8_t *__restrict__ alloc) {
  grid_dependency_wait();
  allow_dependent_launch();
  const int h = blockIdx.x;
  const int slot = threadIdx.x;  // 4 c + tau, slot < 4 d = blockDim.x
  const int c = slot >> 2, tau = slot & 3;
  const int lane = slot & 31, warp = slot >> 5;
  __shared__ unsigned hist[256];
  __shared__ unsigned s_warp[32];
  __shared__ int s_digit;
  __shared__ unsigned s_above;

  const double qv = (double)load_q(q, q_bf16, (int64_t)h * d + c);
  const double sv = (double)sigma[(int64_t)(h / G) * d + c];
  const double w = (qv * qv) * (sv * sv);
  const double scale[4] = {1.0, 0.25, 0.0625, 0.015625};
  const unsigned long long key = (unsigned long long)__double_as_longlong(w * scale[tau]);

  bool taken = false;
  if (budget > 0) {
    // radix select of the budget-th largest key, most significant digit first
    unsigned long long prefix = 0ull, pmask = 0ull;
    unsigned want = (unsigned)budget;
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0u;
      __syncthreads();
      if ((key & pmask) == prefix) atomicAdd(&hist[(unsigned)(key >> shift) & 255u], 1u);
      __syncthreads();
      if (warp == 0) {
        // lane l owns bins 255 - 8 l ... 248 - 8 l (largest first)
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
              s_digit = 255 - 8 * lane - i;
              s_above = run;
            }
            run += local[i];
          }
        }
      }
      __syncthreads();
      prefix |= (unsigned long long)s_digit << shift;
      pmask |= 255ull << shift;
      want -= s_above;
      __syncthreads();
    }
    // prefix = L; `want` slots equal to L are still to be taken, in slot order
    const bool eq = key == prefix;
    const unsigned ballot = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) s_warp[warp] = (unsigned)__popc(ballot);
    __syncthreads();
    unsigned before = (unsigned)__popc(ballot & ((1u << lane) - 1u));
    for (int i = 0; i < warp; ++i) before += s_warp[i];
    taken = key > prefix || (eq && before < want);
  }
  // t_c = the taken slots of channel c: lanes 4 c .. 4 c + 3 of a warp
  unsigned t = taken ? 1u : 0u;
  t += __shfl_xor_sync(0xffffffffu, t, 1);
  t += __shfl_xor_sync(0xffffffffu, t, 2);
  if (tau == 0) alloc[(int64_t)h * d + c] = (uint8_t)t;
}

cudaError_t launch_allocate(const void *q, int q_bf16, const float *sigma, int h_q, int h_kv, int d,
                            int budget, uint8_t *alloc, cudaStream_t stream) {
  const int G = h_q / h_kv;
  return launch_dependent(allocate_kernel, dim3(h_q), dim3(4 * d), 0, stream, q, q_bf16, sigma,
                          G, d, budget, alloc);
}

// Query-independent read of `budget` bits per key: every channel takes
// budget / d planes and channels c < budget % d one more.  This is the
// water-filling rule above with every channel equally important (its slot
// order takes all channels' first slots, lower channels first, then all
// second slots, ...), so every query head reads the same prefixes and a GQA
// group's union is one head's read.  One thread per (head, channel).
__global__ void __launch_bounds__(256) allocate_uniform_kernel(int n_entries, int d, int budget,
                                                               uint8_t *__restrict__ alloc) {
  grid_dependency_wait();
  allow_dependent_launch();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_entries) return;
  const int c = i % d;
  alloc[i] = (uint8_t)(budget / d + (c < budget % d ? 1 : 0));
}

cudaError_t launch_allocate_uniform(int h_q, int d, int budget, uint8_t *alloc,
                                    cudaStream_t stream) {
  const int n_entries = h_q * d;
  return launch_dependent(allocate_uniform_kernel, dim3((n_entries + 255) / 256), dim3(256), 0,
                          stream, n_entries, d, budget, alloc);
}

}  // namespace fathom
