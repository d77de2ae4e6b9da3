// Quantize-append for head_dim 128, 16-token tiles (sm_100a).
//
// Computes, per tile of 16 tokens x 128 channels of one (layer, kv-head,
// K-or-V), the KVarN pipeline (KVarN project page on open-radar, Key
// Features, "Variance-Normalized Quantization Pipeline"): Hadamard rotation
// along head_dim, Sinkhorn-like row/column second-moment normalisation,
// per-token asymmetric round-to-nearest, packing into the tile's cache page.
//
// One warp owns one tile.  Lane (g = lane/4, t = lane%4) ends up holding the
// rotated values of tokens {2t, 2t+1, 2t+8, 2t+9} and channels 16g..16g+15.
//
// Rotation: the Sylvester matrix factors over the 7 bits of the channel
// index, H_128 = (x) over bits of H_2.  Bits 3..6 are contracted with one
// 16x16 +-1 matrix on the tensor cores (mma.sync m16n8k16, exact products,
// fp32 accumulation; 16 MMAs per tile); bits 0..2 are three in-register
// butterfly stages on fp32 pairs.  The 1/sqrt(128) factor is not applied to
// the tile: the column factors c are invariant to a uniform scale of the
// tile, and a, z are scaled by it at the end.
//
// Normalisation: the rounds of "divide rows by their RMS, then columns by
// theirs" are carried out on the factors only.  With A = Z*Z,
//   r_i^2 = (1/d) sum_j A_ij / c_j^2      (row step; kept if the sum is 0)
//   c_j^2 = (1/T) sum_i A_ij / r_i^2      (column step; kept if the sum is 0)
// which is the same recursion as rescaling the tile each half-step, since
// Y = diag(r)^-1 Z diag(c)^-1 throughout.
//
// Quantisation: a row-wise affine map is invariant to a positive row factor,
// so codes come from Y' = Z / c directly, and a = r*s = s', z = r*m = m'
// (the step and minimum of the rows of Y').
#include <cuda_runtime.h>

#include "kvq_device.cuh"

namespace kvq {
namespace {

constexpr int kD = 128;
constexpr int kT = 16;
constexpr int kWarps = 8;
constexpr float kMagic = 12582912.0f;        // 1.5 * 2^23: adding it rounds to an integer (ties to even)
constexpr uint32_t kMagicBits = 0x4B400000u;
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1/sqrt(128)

// Channel bits carried by the MMA contraction index k = 2t + j0 + 8*j1
// (t = lane%4 of the B fragment): bits 3,4 <- t, bit 5 <- j0, bit 6 <- j1.
__device__ __forceinline__ int k_bits(int k) {
  return (((k >> 1) & 3) << 3) | ((k & 1) << 5) | (((k >> 3) & 1) << 6);
}
// Channel bits of the MMA output row m = g + 8*m3: bit 3 <- m3, bits 4..6 <- g.
__device__ __forceinline__ int m_bits(int m) { return ((m >> 3) << 3) | ((m & 7) << 4); }

template <bool F16>
__device__ __forceinline__ uint32_t sign_pair(int m, int k0) {
  const uint32_t one = F16 ? 0x3C00u : 0x3F80u, neg = F16 ? 0xBC00u : 0xBF80u;
  const uint32_t lo = (__popc(m_bits(m) & k_bits(k0)) & 1) ? neg : one;
  const uint32_t hi = (__popc(m_bits(m) & k_bits(k0 + 1)) & 1) ? neg : one;
  return lo | (hi << 16);
}

__device__ __forceinline__ uint32_t code_of(float t) {
  return __float_as_uint(t) - kMagicBits;
}

template <bool F16>
__global__ void __launch_bounds__(kWarps * 32) quantize_d128_kernel(QuantizeParams p) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  uint32_t afrag[4];
  afrag[0] = sign_pair<F16>(g, 2 * t);
  afrag[1] = sign_pair<F16>(g + 8, 2 * t);
  afrag[2] = sign_pair<F16>(g, 2 * t + 8);
  afrag[3] = sign_pair<F16>(g + 8, 2 * t + 8);
  const float zero4[4] = {0.f, 0.f, 0.f, 0.f};

  const int64_t ntt = p.n_tok / kT;
  const int64_t nwarps = (int64_t)gridDim.x * kWarps;
  for (int64_t tile = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); tile < p.total_tiles; tile += nwarps) {
    int64_t rem = tile;
    const int head = (int)(rem % p.num_heads);
    rem /= p.num_heads;
    const int64_t tt = rem % ntt;
    rem /= ntt;
    const int layer = (int)(rem % p.num_layers);
    const int kind = (int)(rem / p.num_layers);
    const int page = __ldg(p.dst_page + tt);
    if (page < 0 || page >= p.num_pages) {
      if (lane == 0) set_error(p.err, KVQ_DEVERR_BAD_PAGE);
      continue;
    }
    const CacheArrays dst = p.dst[kind];

    // ---- load: lane reads tokens g and g+8, channels 32l + 8t .. +7 (l = 0..3)
    const uint16_t* base = static_cast<const uint16_t*>(p.src[kind]) +
                           (((size_t)layer * p.n_tok + (size_t)tt * kT) * p.num_heads + head) * kD;
    const size_t row_stride = (size_t)p.num_heads * kD;
    uint32_t L[2][4][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint16_t* row = base + (size_t)(8 * h + g) * row_stride + 8 * t;
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        const uint4 v = ldg_nc_v4(row + 32 * l);
        L[h][l][0] = v.x;
        L[h][l][1] = v.y;
        L[h][l][2] = v.z;
        L[h][l][3] = v.w;
      }
    }

    // ---- rotation: MMA over channel bits 3..6, then butterflies over bits 0..2
    // P[h][m3][b] = values of tokens (8h+2t, 8h+2t+1) at channel 16g + 8*m3 + b
    f2 P[2][2][8];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const uint32_t sel = (b & 1) ? 0x7632u : 0x5410u;
        const uint32_t b0 = __byte_perm(L[h][0][b >> 1], L[h][1][b >> 1], sel);
        const uint32_t b1 = __byte_perm(L[h][2][b >> 1], L[h][3][b >> 1], sel);
        float d[4];
        mma16816<F16>(d, afrag, b0, b1, zero4);
        P[h][0][b] = f2{d[0], d[1]};
        P[h][1][b] = f2{d[2], d[3]};
      }
#pragma unroll
      for (int m3 = 0; m3 < 2; ++m3) {
#pragma unroll
        for (int s = 1; s < 8; s <<= 1) {
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            if (b & s) continue;
            const f2 x = P[h][m3][b], y = P[h][m3][b + s];
            P[h][m3][b] = add2(x, y);
            P[h][m3][b + s] = sub2(x, y);
          }
        }
      }
    }

    // ---- normalisation on the factors (A = Z^2 kept in registers)
    f2 A[2][2][8];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int m3 = 0; m3 < 2; ++m3)
#pragma unroll
        for (int b = 0; b < 8; ++b) A[h][m3][b] = mul2(P[h][m3][b], P[h][m3][b]);

    float w[16];   // 1 / c_j^2, j = 8*m3 + b
    float v[2][2]; // 1 / r_i^2 of tokens 8h + 2t + tp
    float C[16];   // last column sums
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = 1.f, C[j] = 0.f;
    v[0][0] = v[0][1] = v[1][0] = v[1][1] = 1.f;
    for (int it = 0; it < p.iters; ++it) {
      f2 R[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        R[h] = f2{0.f, 0.f};
#pragma unroll
        for (int m3 = 0; m3 < 2; ++m3)
#pragma unroll
          for (int b = 0; b < 8; ++b) R[h] = fma2(A[h][m3][b], splat2(w[8 * m3 + b]), R[h]);
      }
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          R[h].x += __shfl_xor_sync(0xffffffffu, R[h].x, off);
          R[h].y += __shfl_xor_sync(0xffffffffu, R[h].y, off);
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        v[h][0] = R[h].x > 0.f ? (float)kD / R[h].x : v[h][0];
        v[h][1] = R[h].y > 0.f ? (float)kD / R[h].y : v[h][1];
      }
#pragma unroll
      for (int m3 = 0; m3 < 2; ++m3)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          f2 acc = mul2(A[0][m3][b], f2{v[0][0], v[0][1]});
          acc = fma2(A[1][m3][b], f2{v[1][0], v[1][1]}, acc);
          C[8 * m3 + b] = acc.x + acc.y;
        }
#pragma unroll
      for (int off = 1; off < 4; off <<= 1)
#pragma unroll
        for (int j = 0; j < 16; ++j) C[j] += __shfl_xor_sync(0xffffffffu, C[j], off);
#pragma unroll
      for (int j = 0; j < 16; ++j) w[j] = C[j] > 0.f ? (float)kT / C[j] : w[j];
    }

    // ---- column factor c and Y' = Z / c
    float cf[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float c2 = C[j] > 0.f ? C[j] / (float)kT : 1.f;
      cf[j] = sqrtf(c2);
      const float ic = 1.f / cf[j];
#pragma unroll
      for (int h = 0; h < 2; ++h) P[h][j >> 3][j & 7] = mul2(P[h][j >> 3][j & 7], splat2(ic));
    }

    // ---- per-token min / max of Y'
    float mn[2][2], mx[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float a0 = P[h][0][0].x, b0 = P[h][0][0].x, a1 = P[h][0][0].y, b1 = P[h][0][0].y;
#pragma unroll
      for (int j = 1; j < 16; j += 2) {
        const f2 u = P[h][j >> 3][j & 7];
        const f2 u2 = (j + 1 < 16) ? P[h][(j + 1) >> 3][(j + 1) & 7] : u;
        a0 = min3(a0, u.x, u2.x);
        b0 = max3(b0, u.x, u2.x);
        a1 = min3(a1, u.y, u2.y);
        b1 = max3(b1, u.y, u2.y);
      }
      mn[h][0] = a0, mx[h][0] = b0, mn[h][1] = a1, mx[h][1] = b1;
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int tp = 0; tp < 2; ++tp) {
          mn[h][tp] = fminf(mn[h][tp], __shfl_xor_sync(0xffffffffu, mn[h][tp], off));
          mx[h][tp] = fmaxf(mx[h][tp], __shfl_xor_sync(0xffffffffu, mx[h][tp], off));
        }

    const int bits = dst.bits;
    const float qmax = (float)((1 << bits) - 1);
    const size_t slot = ((size_t)layer * p.num_pages + page) * p.num_heads + head;
    const int tile_bytes = kT * kD * bits / 8;
    uint8_t* codes = dst.codes + slot * tile_bytes;
    float inv_s[2][2], st[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int tp = 0; tp < 2; ++tp) {
        const float s = (mx[h][tp] - mn[h][tp]) / qmax;
        st[h][tp] = s;
        inv_s[h][tp] = s > 0.f ? 1.f / s : 0.f;
      }

    // ---- codes and packing, one token row at a time
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const f2 m2 = f2{mn[h][0], mn[h][1]}, is2 = f2{inv_s[h][0], inv_s[h][1]};
      uint32_t q[16][2];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const f2 tq = add2(mul2(sub2(P[h][j >> 3][j & 7], m2), is2), splat2(kMagic));
        q[j][0] = code_of(tq.x);
        q[j][1] = code_of(tq.y);
      }
#pragma unroll
      for (int tp = 0; tp < 2; ++tp) {
        const int tok = 8 * h + 2 * t + tp;
        if (bits == 4) {
          uint32_t lo = 0, hi = 0;
#pragma unroll
          for (int b = 0; b < 8; ++b) lo |= q[b][tp] << (4 * b), hi |= q[8 + b][tp] << (4 * b);
          *reinterpret_cast<uint2*>(codes + tok * 64 + 8 * g) = make_uint2(lo, hi);
        } else if (bits == 2) {
          uint32_t wd = 0;
#pragma unroll
          for (int j = 0; j < 16; ++j) wd |= q[j][tp] << (2 * j);
          *reinterpret_cast<uint32_t*>(codes + tok * 32 + 4 * g) = wd;
        } else if (bits == 8) {
          uint32_t wd[4] = {0, 0, 0, 0};
#pragma unroll
          for (int j = 0; j < 16; ++j) wd[j >> 2] |= q[j][tp] << (8 * (j & 3));
          *reinterpret_cast<uint4*>(codes + tok * 128 + 16 * g) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        } else {  // 3 bits: low-2-bit plane [T][32 B], then high-bit plane [T][16 B]
          uint32_t lo = 0, hi = 0;
#pragma unroll
          for (int j = 0; j < 16; ++j) lo |= (q[j][tp] & 3u) << (2 * j), hi |= (q[j][tp] >> 2) << j;
          *reinterpret_cast<uint32_t*>(codes + tok * 32 + 4 * g) = lo;
          *reinterpret_cast<uint16_t*>(codes + kT * 32 + tok * 16 + 2 * g) = (uint16_t)hi;
        }
      }
    }

    // ---- folded scales
    if (g == 0) {
      float* tokp = dst.tok + slot * (kT * 2);
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int tp = 0; tp < 2; ++tp) {
          const int tok = 8 * h + 2 * t + tp;
          *reinterpret_cast<float2*>(tokp + 2 * tok) =
              make_float2(st[h][tp] * kInvSqrtD, mn[h][tp] * kInvSqrtD);
        }
    }
    if (t == 0) {
      float4* cp = reinterpret_cast<float4*>(dst.chan + slot * kD + 16 * g);
#pragma unroll
      for (int k = 0; k < 4; ++k) cp[k] = make_float4(cf[4 * k], cf[4 * k + 1], cf[4 * k + 2], cf[4 * k + 3]);
    }
  }
}

}  // namespace

int launch_quantize_d128(const QuantizeParams& p, bool f16, void* stream) {
  if (p.total_tiles == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t need = (p.total_tiles + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)sms * 8;
  const int grid = (int)(need < cap ? need : cap);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (f16)
    quantize_d128_kernel<true><<<grid, kWarps * 32, 0, s>>>(p);
  else
    quantize_d128_kernel<false><<<grid, kWarps * 32, 0, s>>>(p);
  return (int)cudaGetLastError();
}

}  // namespace kvq
