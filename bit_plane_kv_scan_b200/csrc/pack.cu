// Bit-plane packer: 4-bit K codes (token-major nibbles) -> channel-major bit
// planes ("Fathom Makes KV-Cache Scans Query-Adaptive...", method paragraph
// 2: the 4-bit K cache is kept as channel-major bit planes; abstract: a
// channel's leading t planes are precisely its t-bit quantiser).
//
// One block turns 1024 tokens (32 plane words) of one KV head into every
// plane row of those words.  Thread (token group tg, code word cw) loads the
// 32-bit code word cw (channels 8 cw .. 8 cw + 7) of the 32 tokens of group
// tg, one coalesced 4-byte load each, and transposes that 32 x 32 bit matrix
// in registers (byte permutes for the 16- and 8-bit block swaps, masked
// shift-xor swaps below that).  Afterwards register i holds bit i of the
// code word for all 32 tokens: the plane word of (channel, plane) that bit i
// encodes.  The words are staged in shared memory and written out as
// 128-byte row segments.  Integer and bit-exact; each byte of the store is
// read and written once (HBM-bound).
#include <type_traits>

#include "fathom_internal.cuh"

namespace fathom {

// Swaps the off-diagonal halves of the 2 x 2 blocks of width J in the bit
// matrix rows a (upper) and b (lower): the bits of a at positions with bit J
// set trade places with the bits of b at positions J lower.
template <int J>
__device__ __forceinline__ void swap_blocks(uint32_t &a, uint32_t &b) {
  if (J == 16) {
    const uint32_t na = __byte_perm(a, b, 0x5410), nb = __byte_perm(a, b, 0x7632);
    a = na;
    b = nb;
  } else if (J == 8) {
    const uint32_t na = __byte_perm(a, b, 0x6240), nb = __byte_perm(a, b, 0x7351);
    a = na;
    b = nb;
  } else {
    constexpr uint32_t m = J == 4 ? 0x0F0F0F0Fu : J == 2 ? 0x33333333u : 0x55555555u;
    const uint32_t t = ((a >> J) ^ b) & m;
    b ^= t;
    a ^= t << J;
  }
}

template <int J>
__device__ __forceinline__ void transpose_stage(uint32_t (&x)[32]) {
#pragma unroll
  for (int t = 0; t < 32; ++t)
    if ((t & J) == 0) swap_blocks<J>(x[t], x[t + J]);
}

template <int D>
__global__ void __launch_bounds__(D * 4) pack_kernel(const uint8_t *__restrict__ codes, int64_t n,
                                                   uint32_t *__restrict__ planes, int64_t W) {
  constexpr int kWordsPerToken = D / 8;        // 32-bit code words (8 channels each)
  constexpr int kThreads = 32 * kWordsPerToken;
  constexpr int kRows = 4 * D;                 // plane rows c * 4 + j of one KV head
  // shared-memory column rotation per code word, so that the 32 lanes of a
  // warp store into 32 different banks
  constexpr int kRot = kWordsPerToken >= 32 ? 1 : 32 / kWordsPerToken;
  extern __shared__ uint32_t sm_words[];  // [kRows][32], row r rotated by kRot * (r / 32)
  const int g = blockIdx.y;
  const int tid = threadIdx.x;
  const int tg = tid / kWordsPerToken;
  const int cw = tid - tg * kWordsPerToken;
  const int64_t w0 = (int64_t)blockIdx.x * 32;
  const int64_t tok0 = (w0 + tg) * 32;
  const uint32_t *src = reinterpret_cast<const uint32_t *>(codes + (int64_t)g * n * (D / 2)) + cw;

  uint32_t x[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) {
    const int64_t tok = tok0 + t;
    x[t] = tok < n ? __ldg(src + tok * kWordsPerToken) : 0u;
  }
  transpose_stage<16>(x);
  transpose_stage<8>(x);
  transpose_stage<4>(x);
  transpose_stage<2>(x);
  transpose_stage<1>(x);

  // bit i of code word cw is bit i % 4 of nibble (i / 4) % 2 of byte i / 8:
  // channel 8 cw + 2 (i / 8) + (i / 4) % 2, plane 3 - i % 4
  const int col = (tg + kRot * cw) & 31;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int row = 32 * cw + 4 * (2 * (i >> 3) + ((i >> 2) & 1)) + 3 - (i & 3);
    sm_words[row * 32 + col] = x[i];
  }
  __syncthreads();

  const int lane = tid & 31;
  const int64_t w = w0 + lane;
  if (w < W) {
    uint32_t *dst = planes + (int64_t)g * kRows * W + w;
    for (int row = tid >> 5; row < kRows; row += kThreads / 32)
      dst[(int64_t)row * W] = sm_words[row * 32 + ((lane + kRot * (row >> 5)) & 31)];
  }
}

template <int D>
static cudaError_t launch_pack_d(const uint8_t *codes, int64_t n, int h_kv, uint32_t *planes,
                                 cudaStream_t stream) {
  const int64_t W = plane_words(n);
  const int smem = D * 4 * 32 * 4;
  // per launch: the opt-in belongs to the current device
  cudaError_t e = cudaFuncSetAttribute(pack_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((W + 31) / 32), (unsigned)h_kv);
  pack_kernel<D><<<grid, D * 4, smem, stream>>>(codes, n, planes, W);
  return cudaGetLastError();
}

// ------------------------------------------------------------- append --
// Decoding grows the cache one token at a time.  Appending m tokens' codes
// to a store of n tokens changes only the plane words that hold tokens
// n .. n + m - 1; a longer row (plane_words(n + m) > plane_words(n)) needs
// the old words copied into the new layout first.

// Out-of-place step: word w < W_in of every row comes from the old store,
// the rest of the new row is zero (padding, or about to receive new bits).
// Row lengths are multiples of 4 words, so with 16-byte aligned stores the
// copy moves whole 16-byte pieces (V = 4 words); else one word at a time.
template <int V>
__global__ void append_copy_kernel(const uint32_t *__restrict__ in, int64_t W_in,
                                   uint32_t *__restrict__ out, int64_t W_out, int64_t rows) {
  using Piece = typename std::conditional<V == 4, uint4, uint32_t>::type;
  const Piece *src = reinterpret_cast<const Piece *>(in);
  Piece *dst = reinterpret_cast<Piece *>(out);
  const int64_t q_in = W_in / V, q_out = W_out / V;
  const int64_t total = rows * q_out;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / q_out, w = i - r * q_out;
    Piece v{};  // zero past the old row
    if (w < q_in) v = src[r * q_in + w];
    dst[i] = v;
  }
}

// One thread per (KV head, channel, plane, word w) with w covering tokens
// n .. n + m - 1: OR in bit 3 - j of the new tokens' codes of channel c
// (the old store's bits past token n - 1 are zero).
__global__ void append_bits_kernel(const uint8_t *__restrict__ codes, int64_t n, int64_t m, int d,
                                   int h_kv, uint32_t *__restrict__ planes, int64_t W) {
  const int64_t w0 = n / 32, w1 = (n + m + 31) / 32;  // words [w0, w1) hold new tokens
  const int64_t nw = w1 - w0;
  const int64_t total = (int64_t)h_kv * d * 4 * nw;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / nw;  // (g, c, j)
    const int64_t w = w0 + (i - row * nw);
    const int j = (int)(row & 3);
    const int c = (int)((row >> 2) % d);
    const int64_t g = (row >> 2) / d;
    uint32_t word = 0u;
    for (int b = 0; b < 32; ++b) {
      const int64_t tok = 32 * w + b;
      if (tok < n || tok >= n + m) continue;
      const uint8_t byte = codes[(g * m + (tok - n)) * (d / 2) + c / 2];
      const uint32_t u = (c & 1) ? (uint32_t)(byte >> 4) : (uint32_t)(byte & 15u);
      word |= ((u >> (3 - j)) & 1u) << b;
    }
    planes[row * W + w] |= word;
  }
}

cudaError_t launch_append(const uint8_t *codes, int64_t n, int64_t m, int d, int h_kv,
                          const uint32_t *planes_in, uint32_t *planes_out, cudaStream_t stream) {
  const int64_t W_in = plane_words(n), W_out = plane_words(n + m);
  const int64_t rows = (int64_t)h_kv * d * 4;
  if (planes_out != planes_in && rows * W_out > 0) {
    const bool wide = ((uintptr_t)planes_in % 16 == 0) && ((uintptr_t)planes_out % 16 == 0) &&
                      W_in % 4 == 0 && W_out % 4 == 0;
    const int64_t total = rows * W_out / (wide ? 4 : 1);
    const int blocks = (int)((total + 255) / 256 < 148 * 16 ? (total + 255) / 256 : 148 * 16);
    if (wide)
      append_copy_kernel<4><<<blocks, 256, 0, stream>>>(planes_in, W_in, planes_out, W_out, rows);
    else
      append_copy_kernel<1><<<blocks, 256, 0, stream>>>(planes_in, W_in, planes_out, W_out, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (m == 0) return cudaSuccess;
  const int64_t nw = (n + m + 31) / 32 - n / 32;
  const int64_t total = rows * nw;
  const int blocks = (int)((total + 255) / 256 < 148 * 16 ? (total + 255) / 256 : 148 * 16);
  append_bits_kernel<<<blocks, 256, 0, stream>>>(codes, n, m, d, h_kv, planes_out, W_out);
  return cudaGetLastError();
}

cudaError_t launch_pack(const uint8_t *codes, int64_t n, int d, int h_kv, uint32_t *planes,
                        cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  switch (d) {
    case 32: return launch_pack_d<32>(codes, n, h_kv, planes, stream);
    case 64: return launch_pack_d<64>(codes, n, h_kv, planes, stream);
    case 96: return launch_pack_d<96>(codes, n, h_kv, planes, stream);
    case 128: return launch_pack_d<128>(codes, n, h_kv, planes, stream);
    case 160: return launch_pack_d<160>(codes, n, h_kv, planes, stream);
    case 192: return launch_pack_d<192>(codes, n, h_kv, planes, stream);
    case 224: return launch_pack_d<224>(codes, n, h_kv, planes, stream);
    case 256: return launch_pack_d<256>(codes, n, h_kv, planes, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fathom
