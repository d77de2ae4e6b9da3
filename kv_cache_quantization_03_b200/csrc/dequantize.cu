// Dequantisation of cache pages to float32 (inspection and tests; not on the
// decode path).  Rotated domain: (a q + z) c per element; optionally rotated
// back with H/sqrt(d) (KVarN project page on open-radar, Key Features,
// "Variance-Normalized Quantization Pipeline": the stored tile is the
// rotated, normalised one).
#include <cuda_runtime.h>

#include "kvq_device.cuh"

namespace kvq {
namespace {

constexpr int kT = 16;  // rows per pass

template <int kD>
__device__ __forceinline__ uint32_t read_code(const uint8_t* codes, int bits, int T, int tok, int ch) {
  if (bits == 3) {
    const uint32_t lo = (codes[tok * (kD / 4) + ch / 4] >> (2 * (ch % 4))) & 3u;
    const uint32_t hi = (codes[T * (kD / 4) + tok * (kD / 8) + ch / 8] >> (ch % 8)) & 1u;
    return lo | (hi << 2);
  }
  const int bit = (tok * kD + ch) * bits;
  return (codes[bit >> 3] >> (bit & 7)) & ((1u << bits) - 1u);
}

template <int kD>
__global__ void __launch_bounds__(kD) dequantize_kernel(DequantParams p) {
  __shared__ float tile[kT][kD];
  const int ch = threadIdx.x;
  int64_t idx = blockIdx.x;
  const int head = (int)(idx % p.num_heads);
  idx /= p.num_heads;
  const int kind = (int)(idx % p.kinds);
  const int64_t pi = idx / p.kinds;
  const int page = p.pages[pi];
  if (page < 0 || page >= p.num_pages) {
    if (ch == 0) set_error(p.err, KVQ_DEVERR_BAD_PAGE);
    return;
  }
  const CacheArrays src = p.src[kind];
  const int T = p.tile_tokens;
  const size_t slot = ((size_t)p.layer * p.num_pages + page) * p.num_heads + head;
  const uint8_t* codes = src.codes + slot * ((size_t)T * kD * src.bits / 8);
  // a, z, c: float32 or IEEE half
  auto meta = [&](const void* base, size_t i) {
    return src.meta16 ? __half2float(static_cast<const __half*>(base)[i]) : static_cast<const float*>(base)[i];
  };
  // per-token groups: (a, z) per row and c per channel; per-channel key
  // groups: (s, m) of this thread's channel, no row scales
  const size_t tok0 = slot * T * 2;
  const float c = src.per_channel ? 1.f : meta(src.chan, slot * kD + ch);
  const float cs = src.per_channel ? meta(src.tok, slot * kD * 2 + 2 * ch) : 0.f;
  const float cm = src.per_channel ? meta(src.tok, slot * kD * 2 + 2 * ch + 1) : 0.f;
  float* out = p.out[kind] + (((size_t)pi * p.num_heads + head) * T) * kD;
  for (int r0 = 0; r0 < T; r0 += kT) {  // kT rows at a time
    for (int r = 0; r < kT; ++r)
      tile[r][ch] = src.per_channel
                        ? fmaf(cs, (float)read_code<kD>(codes, src.bits, T, r0 + r, ch), cm)
                        : fmaf(meta(src.tok, tok0 + 2 * (r0 + r)), (float)read_code<kD>(codes, src.bits, T, r0 + r, ch),
                               meta(src.tok, tok0 + 2 * (r0 + r) + 1)) * c;
    __syncthreads();
    if (p.unrotate) {  // H / sqrt(b) on each block of b = hblock channels
      for (int r = 0; r < kT; ++r) {
        for (int s = 1; s < p.hblock; s <<= 1) {
          const float x = tile[r][ch & ~s], y = tile[r][ch | s];
          __syncthreads();
          tile[r][ch] = (ch & s) ? (x - y) : (x + y);
          __syncthreads();
        }
        tile[r][ch] *= inv_sqrt_pow2(p.hblock);
      }
      __syncthreads();
    }
    for (int r = 0; r < kT; ++r) out[(r0 + r) * kD + ch] = tile[r][ch];
    __syncthreads();  // the tile is rewritten by the next rows
  }
}

}  // namespace

int launch_dequantize(const DequantParams& p, int head_dim, void* stream) {
  const int64_t blocks = p.n_pages * p.kinds * p.num_heads;
  if (blocks == 0) return cudaSuccess;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (head_dim == 128)
    dequantize_kernel<128><<<(unsigned)blocks, 128, 0, s>>>(p);
  else if (head_dim == 512)
    dequantize_kernel<512><<<(unsigned)blocks, 512, 0, s>>>(p);
  else
    return (int)cudaErrorInvalidValue;
  return (int)cudaGetLastError();
}

}  // namespace kvq
