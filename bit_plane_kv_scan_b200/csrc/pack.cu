// Bit-plane packer: 4-bit K codes (token-major nibbles) -> channel-major bit
// planes ("Fathom Makes KV-Cache Scans Query-Adaptive...", method paragraph
// 2: the 4-bit K cache "is stored in channel-major bit planes"; abstract:
// "a prefix of t planes is exactly the channel's t-bit quantizer").
//
// One block turns 1024 tokens (32 plane words) of one KV head into every
// plane row of those words.  Warp w owns word w: lane b loads token 32w+b's
// d/2 code bytes with 16-byte loads, and one warp vote per (channel, plane)
// yields the plane word directly.  The words are staged in shared memory
// and written out as 128-byte row segments.  Integer and bit-exact; the
// transpose reads and writes each byte of the store once (HBM-bound).
#include "fathom_internal.cuh"

namespace fathom {

template <int D>
__global__ void __launch_bounds__(1024) pack_kernel(const uint8_t *__restrict__ codes, int64_t n,
                                                    uint32_t *__restrict__ planes, int64_t W) {
  extern __shared__ uint32_t sm_words[];  // [D * 4 rows][32 words]
  constexpr int kVec = D / 32;            // 16-byte vectors per token (D/2 bytes)
  const int g = blockIdx.y;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t w0 = (int64_t)blockIdx.x * 32;
  const int64_t tok = (w0 + warp) * 32 + lane;

  uint32_t v[kVec * 4];
  if (tok < n) {
    const uint4 *src = reinterpret_cast<const uint4 *>(codes + ((int64_t)g * n + tok) * (D / 2));
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      uint4 x = __ldg(src + i);
      v[4 * i + 0] = x.x;
      v[4 * i + 1] = x.y;
      v[4 * i + 2] = x.z;
      v[4 * i + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kVec * 4; ++i) v[i] = 0u;
  }

#pragma unroll
  for (int c = 0; c < D; ++c) {
    // channel c is nibble c % 8 of 32-bit word c / 8 (low nibble = even channel)
    const uint32_t u = (v[c >> 3] >> (4 * (c & 7))) & 15u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t word = __ballot_sync(0xffffffffu, (u >> (3 - j)) & 1u);
      if (lane == 0) sm_words[(c * 4 + j) * 32 + warp] = word;
    }
  }
  __syncthreads();

  for (int idx = threadIdx.x; idx < D * 4 * 32; idx += 1024) {
    const int row = idx >> 5;
    const int64_t w = w0 + (idx & 31);
    if (w < W) planes[((int64_t)g * D * 4 + row) * W + w] = sm_words[idx];
  }
}

template <int D>
static cudaError_t launch_pack_d(const uint8_t *codes, int64_t n, int h_kv, uint32_t *planes,
                                 cudaStream_t stream) {
  const int64_t W = plane_words(n);
  const int smem = D * 4 * 32 * 4;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(pack_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid((unsigned)((W + 31) / 32), (unsigned)h_kv);
  pack_kernel<D><<<grid, 1024, smem, stream>>>(codes, n, planes, W);
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
