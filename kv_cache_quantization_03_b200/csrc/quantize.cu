// Quantize-append for head_dim 128 (GQA; tiles of 16, 32, 64 or 128 tokens)
// and 512 (MLA latent; 16-token tiles) (sm_100a).
//
// Computes, per tile of T tokens x d channels of one (layer, kv-head,
// K-or-V), the KVarN pipeline (KVarN project page on open-radar, Key
// Features, "Variance-Normalized Quantization Pipeline"): Hadamard rotation
// along head_dim, Sinkhorn-like row/column second-moment normalisation,
// per-token asymmetric round-to-nearest, packing into the tile's cache page.
//
// One warp owns 16 tokens x one 128-channel block of a tile (head_dim 128,
// T = 16: the whole tile; 512: four warps share a tile across channels;
// T = 16 TW: TW warps share it across tokens, and their column sums are added
// through shared memory once per round).  Lane (g = lane/4, t = lane%4) ends up
// holding the rotated values of tokens {2t, 2t+1, 2t+8, 2t+9} and channels
// 16g..16g+15 of its block (register pairs hold the two tokens 8h + 2t,
// 8h + 2t + 1 of one channel).  For 512 channels, H_512 = H_4 (x) H_128: each
// warp applies H_128 to its block, then the four blocks are combined with the
// signs of H_4 through shared memory; row sums and row min/max are combined
// across the four warps the same way, column sums stay within a warp.
//
// Rotation: the Sylvester matrix factors over the 7 bits of the channel
// index, H_128 = (x) over bits of H_2.  Bits 3..6 are contracted with one
// 16x16 +-1 matrix on the tensor cores (mma.sync m16n8k16 with 8 tokens as
// N: exact products, fp32 accumulation, 16 MMAs per tile); bits 0..2 are
// three in-register butterfly stages on fp32 pairs.
// The 1/sqrt(128) factor is not applied to the tile: the column factors c
// are invariant to a uniform scale, and a, z are scaled by it at the end.
//
// Normalisation: the rounds of "divide rows by their RMS, then columns by
// theirs" are carried out on the factors only.  With A = Z*Z,
//   r_i^2 = (1/d) sum_j A_ij / c_j^2      (row step; kept if the sum is 0)
//   c_j^2 = (1/T) sum_i A_ij / r_i^2      (column step; kept if the sum is 0)
// which is the same recursion as rescaling the tile each half-step, since
// Y = diag(r)^-1 Z diag(c)^-1 throughout.  Row sums are reduced with
// shuffles (one lane per token computes its reciprocal); column sums go
// through the warp's shared memory (each lane owns four channels).
//
// Quantisation: a row-wise affine map is invariant to a positive row factor,
// so codes come from Y' = Z / c directly, and a = r*s = s', z = r*m = m'
// (the step and minimum of the rows of Y').
#include <cuda_runtime.h>

#include "kvq_device.cuh"

namespace kvq {
namespace {

constexpr int kBlk = 128;                  // channels per warp (one 128-channel block of a tile)
constexpr int kT = 16;                     // tokens per warp
constexpr int kWarps = 4;                  // warps per CTA, unless a tile needs more
// Warps per CTA: four, or one tile's TW token slices when that is more.
template <int TW>
constexpr int cta_warps() { return TW > kWarps ? TW : kWarps; }
constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }
template <int D, int TW>
constexpr int log2_dt() { return ilog2(D) - ilog2(kT * TW); }  // log2(d / T), may be <= 0
constexpr float kMagic = 12582912.0f;       // 1.5 * 2^23: adding it rounds to an integer (ties to even)

// Channel bits carried by the MMA contraction index k = 2t + j0 + 8*j1
// (t = lane%4 of the B fragment): bits 3,4 <- t, bit 5 <- j0, bit 6 <- j1.
__device__ __forceinline__ int k_bits(int k) {
  return (((k >> 1) & 3) << 3) | ((k & 1) << 5) | (((k >> 3) & 1) << 6);
}
// Channel bits of the MMA output row m = g + 8*m3: bit 3 <- m3, bits 4..6 <- g.
__device__ __forceinline__ int m_bits(int m) { return ((m >> 3) << 3) | ((m & 7) << 4); }

// Entry (m, k) of the 16x16 factor over channel bits 3..6: the product over
// those bits of H_2 entries, or, for bits at or above a block-diagonal
// rotation's block (mask `out`), of identity entries.
template <bool F16>
__device__ __forceinline__ uint32_t sign_entry(int m, int k, uint32_t out) {
  const uint32_t one = F16 ? 0x3C00u : 0x3F80u, neg = F16 ? 0xBC00u : 0xBF80u;
  const uint32_t mb = m_bits(m), kb = k_bits(k);
  if ((mb ^ kb) & out) return 0u;
  return (__popc(mb & kb & ~out) & 1) ? neg : one;
}
template <bool F16>
__device__ __forceinline__ uint32_t sign_pair(int m, int k0, uint32_t out) {
  return sign_entry<F16>(m, k0, out) | (sign_entry<F16>(m, k0 + 1, out) << 16);
}

// 1/x and 1/sqrt(x) from the hardware approximations plus one Newton step
// (about 1 ulp), for the few per-row / per-column factors of each tile.
__device__ __forceinline__ float rcp_nr(float x) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return fmaf(r, fmaf(-x, r, 1.f), r);
}
// 1/x from the hardware approximation alone (for the per-round factors).
__device__ __forceinline__ float rcp_fast(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
// 1 / x for a row or column sum x >= 0 of the normalisation rounds, finite
// for x = 0 (an all-zero row or column, whose factor multiplies only zeros).
// Tiles of one 16-token slice floor x at 2^-100 (one min); longer tiles
// select 0 for x = 0 (with the floor ptxas spills registers there).  The two
// agree for x = 0 in effect (a finite factor times zeros) and for every
// x >= 2^-100.
template <int TW>
__device__ __forceinline__ float rcp_sum(float x) {
  if constexpr (TW == 1) return rcp_fast(fmaxf(x, 0x1p-100f));
  else return x > 0.f ? rcp_fast(x) : 0.f;
}
// 1 / sqrt(x) of a pair: the approximation and one Newton step,
// y (1.5 - 0.5 x y y), in paired arithmetic.
__device__ __forceinline__ f2 rsqrt_nr2(f2 x) {
  f2 y;
  asm("rsqrt.approx.f32 %0, %1;" : "=f"(y.x) : "f"(x.x));
  asm("rsqrt.approx.f32 %0, %1;" : "=f"(y.y) : "f"(x.y));
  return mul2(y, fma2(mul2(mul2(splat2(-0.5f), x), y), y, splat2(1.5f)));
}

// Four per-lane values x[h][tp] of tokens 8h + 2t + tp (this lane's channels)
// reduced with `op` over the eight lanes g that share t; returns the value of
// the token this lane owns, 8 b2 + 2t + b1 (b1 = lane bit 3, b2 = lane bit 4).
template <typename Op>
__device__ __forceinline__ float reduce_tokens(const float (&x)[2][2], int b1, int b2, Op op) {
  const float k0 = op(b2 ? x[1][0] : x[0][0], __shfl_xor_sync(0xffffffffu, b2 ? x[0][0] : x[1][0], 16));
  const float k1 = op(b2 ? x[1][1] : x[0][1], __shfl_xor_sync(0xffffffffu, b2 ? x[0][1] : x[1][1], 16));
  const float r = op(b1 ? k1 : k0, __shfl_xor_sync(0xffffffffu, b1 ? k0 : k1, 8));
  return op(r, __shfl_xor_sync(0xffffffffu, r, 4));
}

// Squares paired along channels: A[h][tp][q] = channels 2q, 2q+1 (of 16g + ..)
// of token 8h + 2t + tp.
__device__ __forceinline__ void square_pairs(const f2 (&P)[2][2][8], f2 (&A)[2][2][8]) {
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const f2 x = P[h][q >> 2][2 * (q & 3)], y = P[h][q >> 2][2 * (q & 3) + 1];
      A[h][0][q] = make_float2(x.x * x.x, y.x * y.x);
      A[h][1][q] = make_float2(x.y * x.y, y.y * y.y);
    }
}

// Byte 0 of four words, in order: the code held by a magic-number float.
__device__ __forceinline__ uint32_t gather4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x4000u), 0x7610u);
}
// The words hold magic-number floats: bits 0..21 are the code, bits above
// them a constant whose low byte is 0.  So f0 + (f1 << 4) carries the two
// codes in its low byte: eight 4-bit codes -> one word, code i in bits
// 4i..4i+3.
__device__ __forceinline__ uint32_t pack_nibbles(const uint32_t* f) {
  return gather4(f[0] + (f[1] << 4), f[2] + (f[3] << 4), f[4] + (f[5] << 4), f[6] + (f[7] << 4));
}
// Sixteen 2-bit codes -> one word, code i in bits 2i..2i+1.
__device__ __forceinline__ uint32_t pack_crumbs(const uint32_t* f) {
  uint32_t b[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) b[k] = f[4 * k] + (f[4 * k + 1] << 2) + (f[4 * k + 2] << 4) + (f[4 * k + 3] << 6);
  return gather4(b[0], b[1], b[2], b[3]);
}

struct WarpScratch {
  float4 col[4][32];  // column partials: chunk k of lane (g, t) at [k][4g + (t ^ k)]
  float4 own[32];     // owned channels 16g + 4t .. +3
  float4 dup[2][32];  // owned 1/c twice each
};

// Quotient by a fixed divisor with a multiply-high (n < 2^31).
struct FastDiv {
  uint32_t d, m, s;
};
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) { return (__umulhi(n, f.m) + n) >> f.s; }

struct QuantLaunch {
  const uint16_t* src;   // [layer][n_tok][H][D]
  CacheArrays dst;
  int64_t n_tok;
  int num_layers, num_heads;
  int64_t num_pages;
  int iters;
  const int32_t* dst_page;
  uint32_t* err;
  uint32_t total;        // layers * (n_tok / T) * heads
  FastDiv div_h, div_ntt;
  const uint16_t* rope_src;  // MLA: [layer][n_tok][rope_dim] bf16, copied into rope_dst; else null
  uint16_t* rope_dst;        // [layer][page][T][rope_dim]
  int rope_dim;
  int hblock;                // Hadamard block (8 .. 128 channels; 512 for the MLA latent)
  float inv_sqrt_b;          // 1/sqrt(hblock)
  int after_k;               // 1: the V launch, enqueued as the programmatic dependent of the K launch
};

// Shared memory of one tile whose 512 channels are split over four warps.
struct TileShare {
  float row[2][4][kT];   // row partial sums, double-buffered by round parity
  float2 mm[4][kT];      // per block and token: (min, max)
  float cmax[4];         // per block: largest column factor
};

// Channel bits 0..6 of the 128-channel block: bits 3..6 on the tensor cores
// (16 MMAs), bits 0..2 as three butterfly stages on fp32 pairs (only the
// stages inside the rotation's block: none for block 1, no rotation).
template <bool F16, bool SMALL_BLOCKS>
__device__ __forceinline__ void hadamard128(const uint32_t (&L)[2][4][4], const uint32_t (&afrag)[4], f2 (&P)[2][2][8],
                                            int hblock) {
  const float zero4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const uint32_t sel = (b & 1) ? 0x7632u : 0x5410u;
      float d[4];
      mma16816<F16>(d, afrag, __byte_perm(L[h][0][b >> 1], L[h][1][b >> 1], sel),
                    __byte_perm(L[h][2][b >> 1], L[h][3][b >> 1], sel), zero4);
      P[h][0][b] = make_float2(d[0], d[1]);
      P[h][1][b] = make_float2(d[2], d[3]);
    }
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int m3 = 0; m3 < 2; ++m3)
#pragma unroll
      for (int s = 1; s < 8; s <<= 1)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          if ((b & s) || (SMALL_BLOCKS && s >= hblock)) continue;
          const f2 x = P[h][m3][b], y = P[h][m3][b + s];
          P[h][m3][b] = add2(x, y);
          P[h][m3][b + s] = sub2(x, y);
        }
}

// Raw 16 tokens x 128 channels (token slice wt of a tile of TW slices; at
// D = 512 channel block blk of the latent) staged per lane in shared memory
// by cp.async: slot [h * 4 + l][lane] holds tokens 8h + g, channels
// 128 blk + 8t + 32 l .. + 7, which read_staged puts in L[h][l].
template <int TW, int D>
__device__ __forceinline__ void stage_tile(uint4 (*dst)[32], const QuantLaunch& p, uint32_t tile, int wt, int blk, int g,
                                           int t, int lane, int32_t& page) {
  const uint32_t r1 = fdiv(tile, p.div_h), head = tile - r1 * p.div_h.d;
  const uint32_t layer = fdiv(r1, p.div_ntt), tt = r1 - layer * p.div_ntt.d;
  page = __ldg(p.dst_page + tt);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint16_t* row =
        p.src + (((size_t)layer * p.n_tok + (size_t)tt * (kT * TW) + kT * wt + 8 * h + g) * p.num_heads + head) * D +
        kBlk * blk + 8 * t;
#pragma unroll
    for (int l = 0; l < 4; ++l)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(&dst[h * 4 + l][lane])), "l"(row + 32 * l)
                   : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void read_staged(const uint4 (*src)[32], int lane, uint32_t (&L)[2][4][4]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 v = src[i][lane];
    L[i >> 2][i & 3][0] = v.x, L[i >> 2][i & 3][1] = v.y, L[i >> 2][i & 3][2] = v.z, L[i >> 2][i & 3][3] = v.w;
  }
}

template <int W>
__device__ __forceinline__ void tile_sync() {
  if constexpr (W > 1) __syncthreads();  // one tile per CTA when its blocks span warps
}
// The TW warps of one tile (tile slot `slot` of the CTA) meet at a named barrier.
template <int TW>
__device__ __forceinline__ void slice_sync(int slot) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + slot), "r"(TW * 32) : "memory");
}

// Raw-tile staging buffers of a CTA (dynamic shared memory): two tiles per warp.
template <int TW>
constexpr size_t stage_bytes() { return (size_t)cta_warps<TW>() * 2 * 8 * 32 * sizeof(uint4); }

// AXES = 1: the ablation instantiation (16-token tiles at head_dim 128):
// rotation blocks below 8 channels, and per-channel key groups when the
// stream asks for them; the standard instantiation (AXES = 0) carries
// neither.
template <bool F16, int BITS, int D, int TW, int AXES>
__global__ void __launch_bounds__(cta_warps<TW>() * 32, 16 / cta_warps<TW>())
    quantize_kernel(QuantLaunch p) {
  static_assert(TW == 1 || D == kBlk, "tiles longer than 16 tokens need head_dim 128");
  static_assert(AXES == 0 || (D == kBlk && TW == 1), "the ablation instantiation is for 16 x 128 tiles");
  // A launch enqueued as this grid's programmatic dependent may start now:
  // the call's V launch (independent of this K launch), or the decode of a
  // quantise-on-fill call, which waits for this grid before it reads a page
  // written here.
  asm volatile("griddepcontrol.launch_dependents;");
  constexpr int kCW = cta_warps<TW>();
  constexpr int W = D / kBlk;     // warps per tile along channels
  constexpr int kTile = kT * TW;  // tokens per tile
  constexpr int TPC = kCW / (W * TW);  // tiles per CTA
  // The rotated tile waits out the rounds in tensor memory (64 columns of the
  // warp's lane quarter).  The raw tiles are staged in shared memory by
  // cp.async (the next one while the current one is processed), which keeps
  // the kernel at 128 registers or fewer (four CTAs per SM).
  constexpr int kLogDT = log2_dt<D, TW>();
  constexpr int kTmemCols = 64 * (kCW / 4);  // 64 columns per warp, four lane quarters
  __shared__ WarpScratch scratch[kCW];
  __shared__ TileShare share[W > 1 ? 1 : 0 + 1];
  __shared__ float4 colw[TW > 1 ? TPC : 1][2][TW][32];  // column partials of the token slices, by round parity
  extern __shared__ uint4 dyn_smem[];
  uint4(*staged)[2][8][32] = reinterpret_cast<uint4(*)[2][8][32]>(dyn_smem);  // [kCW]
  __shared__ uint32_t tmem_slot;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int warp = threadIdx.x >> 5, blk = warp % W, wt = (warp / W) % TW, slot_id = warp / (W * TW);
  const int b1 = (lane >> 3) & 1, b2 = (lane >> 4) & 1;
  WarpScratch& sc = scratch[warp];
  TileShare& sh = share[0];
  uint32_t afrag[4];
  const uint32_t out_bits = D == kBlk ? 0x78u & ~(uint32_t)(p.hblock - 1) : 0u;  // channel bits 3..6 outside a block
  afrag[0] = sign_pair<F16>(g, 2 * t, out_bits);
  afrag[1] = sign_pair<F16>(g + 8, 2 * t, out_bits);
  afrag[2] = sign_pair<F16>(g, 2 * t + 8, out_bits);
  afrag[3] = sign_pair<F16>(g + 8, 2 * t + 8, out_bits);
  // 1/sqrt(block) (1/sqrt(d) for the full rotation)
  const float inv_sqrt_d = D == kBlk ? p.inv_sqrt_b : 0.044194173824159216f;
  const uint32_t stride = gridDim.x * TPC;
  uint32_t tile = blockIdx.x * TPC + slot_id;
  uint32_t tpark = 0;             // this warp's 64 TMEM columns
  {
    if (warp == 0) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                   "n"(kTmemCols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // a warp reaches the TMEM lanes 32 (warp % 4) .. +31 only
    tpark = tmem_slot + ((uint32_t)((warp & 3) * 32) << 16) + 64 * (warp >> 2);
  }
  // Packs and stores the codes of this lane's rows of the tile in `slot`:
  // tq_of(h, j) gives the magic-number-rounded codes of P[h][j >> 3][j & 7]
  // (tokens 8h + 2t, 8h + 2t + 1 at channel 16g + j of the warp's block).
  auto emit_codes = [&](size_t slot, auto&& tq_of) {
    uint8_t* codes = p.dst.codes + slot * (kTile * D * BITS / 8);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t q[2][16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const f2 tq = tq_of(h, j);
        q[0][j] = __float_as_uint(tq.x);
        q[1][j] = __float_as_uint(tq.y);
      }
#pragma unroll
      for (int tp = 0; tp < 2; ++tp) {
        const int tok = kT * wt + 8 * h + 2 * t + tp;  // row of the tile
        const uint32_t* f = q[tp];
        constexpr int row_bytes = D * BITS / 8, seg = kBlk * BITS / 8;
        if constexpr (BITS == 4) {
          *reinterpret_cast<uint2*>(codes + tok * row_bytes + seg * blk + 8 * g) =
              make_uint2(pack_nibbles(f), pack_nibbles(f + 8));
        } else if constexpr (BITS == 8) {
          *reinterpret_cast<uint4*>(codes + tok * row_bytes + seg * blk + 16 * g) =
              make_uint4(gather4(f[0], f[1], f[2], f[3]), gather4(f[4], f[5], f[6], f[7]),
                         gather4(f[8], f[9], f[10], f[11]), gather4(f[12], f[13], f[14], f[15]));
        } else if constexpr (BITS == 2) {
          *reinterpret_cast<uint32_t*>(codes + tok * row_bytes + seg * blk + 4 * g) = pack_crumbs(f);
        } else {  // 3 bits: low-2-bit plane [T][D/4 B], then high-bit plane [T][D/8 B]
          // Codes 4k..4k+3 gathered into the bytes of word x[k].  One
          // multiply moves the word's four low crumbs to its top byte (crumb
          // of byte j to bits 24 + 2j); one multiply moves the high bits of
          // two words (the second shifted up by 4) to the top byte (bit j of
          // the first word to 24 + j, of the second to 28 + j).  Below bit 24
          // the crumb products sum to less than 2^24 and the high-bit
          // products are disjoint bits, so nothing carries into the top
          // byte; byte permutes then collect the top bytes.
          uint32_t x[4], yl[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            x[k] = gather4(f[4 * k], f[4 * k + 1], f[4 * k + 2], f[4 * k + 3]);
            yl[k] = (x[k] & 0x03030303u) * 0x01041040u;
          }
          const uint32_t lo =
              __byte_perm(__byte_perm(yl[0], yl[1], 0x0073u), __byte_perm(yl[2], yl[3], 0x7300u), 0x7610u);
          const uint32_t y01 = ((x[0] & 0x04040404u) + ((x[1] & 0x04040404u) << 4)) * 0x00408102u;
          const uint32_t y23 = ((x[2] & 0x04040404u) + ((x[3] & 0x04040404u) << 4)) * 0x00408102u;
          const uint32_t hi = __byte_perm(y01, y23, 0x0073u);
          *reinterpret_cast<uint32_t*>(codes + tok * (D / 4) + (kBlk / 4) * blk + 4 * g) = lo;
          *reinterpret_cast<uint16_t*>(codes + kTile * (D / 4) + tok * (D / 8) + (kBlk / 8) * blk + 2 * g) =
              (uint16_t)hi;
        }
      }
    }
  };
  uint32_t L[2][4][4];
  int32_t page = 0;
  uint32_t rounds = 0;  // rounds done by this warp (parity of the column-partial buffer)
  if (tile < p.total) stage_tile<TW, D>(staged[warp][0], p, tile, wt, blk, g, t, lane, page);
  for (int buf = 0; tile < p.total; tile += stride, buf ^= 1) {
    f2 P[2][2][8];  // [h][m3][b]: tokens (8h+2t, 8h+2t+1) at channel 16g + 8m3 + b of the block
    const int32_t cur_page = page;
    asm volatile("cp.async.wait_group 0;" ::: "memory");  // this lane's copies of the current tile
    read_staged(staged[warp][buf], lane, L);
    if (tile + stride < p.total) stage_tile<TW, D>(staged[warp][buf ^ 1], p, tile + stride, wt, blk, g, t, lane, page);
    hadamard128<F16, AXES == 1>(L, afrag, P, D == kBlk ? p.hblock : kBlk);
    const uint32_t cur = tile;
    const uint32_t r1 = fdiv(cur, p.div_h), head = cur - r1 * p.div_h.d;
    const uint32_t layer = fdiv(r1, p.div_ntt), tt = r1 - layer * p.div_ntt.d;
    if (cur_page < 0 || cur_page >= p.num_pages) {  // same decision in every warp of the tile
      // page -1: the caller skips this tile (a sequence whose tail is not full)
      if (cur_page != -1 && lane == 0 && blk == 0 && wt == 0) set_error(p.err, KVQ_DEVERR_BAD_PAGE);
      continue;
    }
    const size_t slot = ((size_t)layer * p.num_pages + cur_page) * p.num_heads + head;
    if (p.rope_src && blk == 0) {  // MLA: the tile's rope rows go to the page unquantised
      const int rd = p.rope_dim;
      const uint16_t* rs = p.rope_src + ((size_t)layer * p.n_tok + (size_t)tt * kT) * rd;
      uint16_t* rdst = p.rope_dst + ((size_t)layer * p.num_pages + cur_page) * kT * rd;
      for (int i = lane * 8; i < kT * rd; i += 32 * 8)
        *reinterpret_cast<uint4*>(rdst + i) = *reinterpret_cast<const uint4*>(rs + i);
    }
    if constexpr (W > 1) {
      // Channel bits 7, 8: H_4 across the four blocks of the tile, one token
      // half at a time, through the tile warps' staging buffers of the
      // current tile (the raw tile is in registers by now, and the next
      // tile's copies go to the other buffer).
      const int w0 = warp - blk;  // the tile's first warp
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        f2(*own)[32] = reinterpret_cast<f2(*)[32]>(staged[warp][buf]);
#pragma unroll
        for (int i = 0; i < 16; ++i) own[i][lane] = P[h][i >> 3][i & 7];
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          f2 acc = reinterpret_cast<const f2(*)[32]>(staged[w0][buf])[i][lane];
#pragma unroll
          for (int k = 1; k < W; ++k) {
            const f2 y = reinterpret_cast<const f2(*)[32]>(staged[w0 + k][buf])[i][lane];
            acc = (__popc(blk & k) & 1) ? sub2(acc, y) : add2(acc, y);
          }
          P[h][i >> 3][i & 7] = acc;
        }
        __syncthreads();  // every warp has read this half before the next one is written
      }
    }
    if constexpr (AXES == 1 && BITS != 3) {
      if (p.dst.per_channel) {
        // Per-channel groups (the KIVI-style axes, no normalisation): channel
        // 16g + j is tokens {2t, 2t+1, 2t+8, 2t+9} of this lane and of the
        // lanes t' = t ^ 1, t ^ 2; its minimum and step go to the group
        // scales as (s, m) pairs, lane t writing channels 16g + 4t .. + 3.
        float cmn[16], cmx[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const f2 a = P[0][j >> 3][j & 7], b = P[1][j >> 3][j & 7];
          cmn[j] = fminf(fminf(a.x, a.y), fminf(b.x, b.y));
          cmx[j] = fmaxf(fmaxf(a.x, a.y), fmaxf(b.x, b.y));
        }
#pragma unroll
        for (int off = 1; off < 4; off <<= 1)
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            cmn[j] = fminf(cmn[j], __shfl_xor_sync(0xffffffffu, cmn[j], off));
            cmx[j] = fmaxf(cmx[j], __shfl_xor_sync(0xffffffffu, cmx[j], off));
          }
        constexpr float kQm = (float)((1 << BITS) - 1);
        float st[4], mt[4];  // the lane's four channels 16g + 4t + i
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = t == 0 ? cmn[i] : t == 1 ? cmn[4 + i] : t == 2 ? cmn[8 + i] : cmn[12 + i];
          const float hi = t == 0 ? cmx[i] : t == 1 ? cmx[4 + i] : t == 2 ? cmx[8 + i] : cmx[12 + i];
          st[i] = (hi - lo) / kQm * inv_sqrt_d;
          mt[i] = lo * inv_sqrt_d;
        }
        const size_t gi = slot * (D * 2) + 2 * (16 * g + 4 * t);
        if (p.dst.meta16) {
          const __half2 h0 = __floats2half2_rn(st[0], mt[0]), h1 = __floats2half2_rn(st[1], mt[1]);
          const __half2 h2 = __floats2half2_rn(st[2], mt[2]), h3 = __floats2half2_rn(st[3], mt[3]);
          *reinterpret_cast<uint4*>(static_cast<__half*>(p.dst.tok) + gi) =
              make_uint4(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1),
                         *reinterpret_cast<const uint32_t*>(&h2), *reinterpret_cast<const uint32_t*>(&h3));
        } else {
          float4* d4 = reinterpret_cast<float4*>(static_cast<float*>(p.dst.tok) + gi);
          d4[0] = make_float4(st[0], mt[0], st[1], mt[1]);
          d4[1] = make_float4(st[2], mt[2], st[3], mt[3]);
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {  // cmx becomes 1 / step
          const float sj = (cmx[j] - cmn[j]) / kQm;
          cmx[j] = sj > 0.f ? rcp_nr(sj) : 0.f;
        }
        emit_codes(slot, [&](int h, int j) {
          return fma2(sub2(P[h][j >> 3][j & 7], splat2(cmn[j])), splat2(cmx[j]), splat2(kMagic));
        });
        continue;  // (one warp per tile here: no tile barrier to meet)
      }
    }
    f2 A[2][2][8];
    square_pairs(P, A);
    // park the rotated tile in tensor memory until the factors are known
    auto park = [&]() {
      float v[32];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const f2 x = P[half][i >> 3][i & 7];
          v[2 * i] = x.x, v[2 * i + 1] = x.y;
        }
        tmem_st32(tpark + 32 * half, v);
      }
    };
    auto unpark = [&]() {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float v[32];
        tmem_ld32(tpark + 32 * half, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) P[half][i >> 3][i & 7] = make_float2(v[2 * i], v[2 * i + 1]);
      }
    };
    park();
    float w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = 1.f;
    // Row sums of A / c^2 (the row step), for the token this lane owns
    // (8 b2 + 2t + b1); at 512 channels the four blocks' sums are added through
    // shared memory (buffer `par`, alternating between rounds).
    auto row_sums = [&](int par) -> float {
      float R[2][2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int tp = 0; tp < 2; ++tp) {
          // one chain of paired FMAs (the ablation instance keeps two, which
          // spares it a register spill)
          if constexpr (AXES == 0) {
            f2 acc = mul2(A[h][tp][0], make_float2(w[0], w[1]));
#pragma unroll
            for (int q = 1; q < 8; ++q) acc = fma2(A[h][tp][q], make_float2(w[2 * q], w[2 * q + 1]), acc);
            R[h][tp] = acc.x + acc.y;
          } else {
            f2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 8; q += 2) {
              acc0 = fma2(A[h][tp][q], make_float2(w[2 * q], w[2 * q + 1]), acc0);
              acc1 = fma2(A[h][tp][q + 1], make_float2(w[2 * q + 2], w[2 * q + 3]), acc1);
            }
            const f2 s2 = add2(acc0, acc1);
            R[h][tp] = s2.x + s2.y;
          }
        }
      float rk = reduce_tokens(R, b1, b2, [](float a, float b) { return a + b; });
      if constexpr (W > 1) {
        const int tok = 8 * b2 + 2 * t + b1;
        if ((lane & 4) == 0) sh.row[par][blk][tok] = rk;
        __syncthreads();
        rk = sh.row[par][0][tok];
#pragma unroll
        for (int k = 1; k < W; ++k) rk += sh.row[par][k][tok];
      }
      return rk;
    };
    // Dynamic range.  The rounds run on fp32 squares of the rotated tile.  A
    // row whose sum of squares is zero or outside [2^-60, 2^60] (an input row
    // far from unit scale, or an all-zero row) is divided by a power of two
    // 2^e taken from its largest |value| before squaring.  That is exact, and
    // the method is invariant to it: the column factors only see A_ij / r_i^2,
    // and the codes only the row's affine map; a and z are multiplied back by
    // 2^e at the end.  An all-zero row keeps scale 1 and contributes nothing.
    float rsc_own = 1.f;  // 2^e of the owned token's row
    float rk = 0.f;
    if (p.iters > 0) {
      rk = row_sums(0);
      const bool odd = !(rk >= 0x1p-60f && rk <= 0x1p60f);
      if (__any_sync(0xffffffffu, odd)) {  // warp-uniform; at 512 channels tile-uniform too
        unpark();
        float mx[2][2];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int tp = 0; tp < 2; ++tp) {
            float m = 0.f;
#pragma unroll
            for (int b = 0; b < 16; ++b) {
              const f2 x = P[h][b >> 3][b & 7];
              m = fmaxf(m, fabsf(tp ? x.y : x.x));
            }
            mx[h][tp] = m;
          }
        float omx = reduce_tokens(mx, b1, b2, [](float a, float b) { return fmaxf(a, b); });
        if constexpr (W > 1) {
          const int tok = 8 * b2 + 2 * t + b1;
          if ((lane & 4) == 0) sh.mm[blk][tok] = make_float2(0.f, omx);
          __syncthreads();
#pragma unroll
          for (int k = 0; k < W; ++k) omx = fmaxf(omx, sh.mm[k][tok].y);
        }
        // exponent field E of the row max, kept in [1, 253]: scale 2^(127-E)
        // brings the max into [1, 2) (a subnormal max into (0, 1), a max of
        // 2^127 or more into [2, 4)); a zero row keeps scale 1
        const int e = min(max((int)(__float_as_uint(omx) >> 23), 1), 253);
        const float s_own = omx > 0.f ? __uint_as_float((uint32_t)(254 - e) << 23) : 1.f;
        rsc_own = omx > 0.f ? __uint_as_float((uint32_t)e << 23) : 1.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const f2 s2 = make_float2(__shfl_sync(0xffffffffu, s_own, (h << 4) | t),
                                    __shfl_sync(0xffffffffu, s_own, (h << 4) | 8 | t));
#pragma unroll
          for (int b = 0; b < 16; ++b) P[h][b >> 3][b & 7] = mul2(P[h][b >> 3][b & 7], s2);
        }
        square_pairs(P, A);
        park();
        rk = row_sums(0);
      }
    }
    // Per-round factors: v = (d/T) / R (row) and w = 1 / C (column) keep
    // w = 1 / c^2 of the textbook recursion exactly, so the final column sums
    // are c^2 itself.  A row or column whose sum is exactly 0 holds only
    // zeros; its factor multiplies nothing, so it only has to be finite
    // (rcp_sum; times d/T <= 32 it stays finite; its stored c is 1).  Every
    // nonzero row sum is at least 2^-60 (2^-46 after the prescale), so the
    // 2^-100 floor changes no other row.  A nonzero column sum below 2^-100
    // needs every entry of the column ~2^-50 below its row's largest in all
    // rows of the tile (rows whose inputs span ~2^50 and cancel their large
    // parts exactly in the same channels); such a column gets the factor of
    // a sum of 2^-100.
    constexpr float kDT = kLogDT >= 0 ? (float)(1 << kLogDT) : 1.f / (float)(1 << -kLogDT);
    float v_own = 1.f;
    float4 w_own = make_float4(1.f, 1.f, 1.f, 1.f);
    f2 c01 = make_float2(0.f, 0.f), c23 = make_float2(0.f, 0.f);
    // Column step of a round: the row factors from the row sums rk, then the
    // column sums c01, c23 of this lane's four channels.
    auto col_step = [&]() {
      v_own = rcp_sum<TW>(rk) * kDT;
      float v[2][2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int tp = 0; tp < 2; ++tp) v[h][tp] = __shfl_sync(0xffffffffu, v_own, (h << 4) | (tp << 3) | t);
      f2 C[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        C[q] = fma2(A[1][1][q], splat2(v[1][1]),
                    fma2(A[1][0][q], splat2(v[1][0]), fma2(A[0][1][q], splat2(v[0][1]), mul2(A[0][0][q], splat2(v[0][0])))));
#pragma unroll
      for (int k = 0; k < 4; ++k)
        sc.col[k][(lane & ~3) | (t ^ k)] = make_float4(C[2 * k].x, C[2 * k].y, C[2 * k + 1].x, C[2 * k + 1].y);
      __syncwarp();
      {
        const float4 x0 = sc.col[t][(lane & ~3) | t];
        c01 = make_float2(x0.x, x0.y), c23 = make_float2(x0.z, x0.w);
      }
#pragma unroll
      for (int i = 1; i < 4; ++i) {
        const float4 x = sc.col[t][(lane & ~3) | (i ^ t)];
        c01 = add2(c01, make_float2(x.x, x.y));
        c23 = add2(c23, make_float2(x.z, x.w));
      }
      if constexpr (TW > 1) {  // add the token slices' sums, in slice order (same result in every warp)
        float4(*cw)[32] = colw[slot_id][rounds & 1];
        cw[wt][lane] = make_float4(c01.x, c01.y, c23.x, c23.y);
        slice_sync<TW>(slot_id);
        float4 x = cw[0][lane];
        c01 = make_float2(x.x, x.y), c23 = make_float2(x.z, x.w);
#pragma unroll
        for (int k = 1; k < TW; ++k) {
          x = cw[k][lane];
          c01 = add2(c01, make_float2(x.x, x.y));
          c23 = add2(c23, make_float2(x.z, x.w));
        }
        ++rounds;
      }
    };
    // The column factors of the round just done, to the lanes that hold the
    // channels.  (The next round's column step passes a __syncwarp before
    // this buffer is written again.)
    auto w_step = [&]() {
      w_own.x = rcp_sum<TW>(c01.x);
      w_own.y = rcp_sum<TW>(c01.y);
      w_own.z = rcp_sum<TW>(c23.x);
      w_own.w = rcp_sum<TW>(c23.y);
      sc.own[lane] = w_own;
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 x = sc.own[(lane & ~3) | k];
        w[4 * k] = x.x, w[4 * k + 1] = x.y, w[4 * k + 2] = x.z, w[4 * k + 3] = x.w;
      }
    };
    // Round 0 takes the row sums from above; the last round's column sums
    // are c^2 itself, so its column factors are not formed.
    if (p.iters > 0) {
      col_step();
      for (int it = 1; it < p.iters; ++it) {
        w_step();
        rk = row_sums(it & 1);
        col_step();
      }
    }
    float cmax = 1.f;  // largest column factor of the tile
    float4 cv4;        // this lane's four column factors
    {
      const bool norm = p.iters > 0;
      const float ct[4] = {c01.x, c01.y, c23.x, c23.y};  // c^2 of the owned channels
      const f2 y01 = rsqrt_nr2(c01), y23 = rsqrt_nr2(c23);
      const f2 x01 = mul2(c01, y01), x23 = mul2(c23, y23);  // c = c^2 / c
      const float ys[4] = {y01.x, y01.y, y23.x, y23.y}, cs[4] = {x01.x, x01.y, x23.x, x23.y};
      float cv[4], ic[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool ok = norm && ct[i] > 0.f;
        ic[i] = ok ? ys[i] : 1.f;
        cv[i] = ok ? cs[i] : 1.f;
      }
      cmax = fmaxf(fmaxf(cv[0], cv[1]), fmaxf(cv[2], cv[3]));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, off));
      if constexpr (W > 1)
        if (lane == 0) sh.cmax[blk] = cmax;  // read after the tile's min/max exchange below
      cv4 = make_float4(cv[0], cv[1], cv[2], cv[3]);
      sc.dup[0][lane] = make_float4(ic[0], ic[0], ic[1], ic[1]);
      sc.dup[1][lane] = make_float4(ic[2], ic[2], ic[3], ic[3]);
      unpark();  // the rotated tile back from tensor memory
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float4 x = sc.dup[k & 1][(lane & ~3) | (k >> 1)];
        const int j = 2 * k;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          P[h][j >> 3][j & 7] = mul2(P[h][j >> 3][j & 7], make_float2(x.x, x.y));
          P[h][(j + 1) >> 3][(j + 1) & 7] = mul2(P[h][(j + 1) >> 3][(j + 1) & 7], make_float2(x.z, x.w));
        }
      }
      __syncwarp();
    }
    float mn[2][2], mx[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float a0 = P[h][0][0].x, c0 = a0, a1 = P[h][0][0].y, c1 = a1;
#pragma unroll
      for (int j = 1; j < 16; j += 2) {
        const f2 u = P[h][j >> 3][j & 7];
        const f2 u2 = (j + 1 < 16) ? P[h][(j + 1) >> 3][(j + 1) & 7] : u;
        a0 = min3(a0, u.x, u2.x), c0 = max3(c0, u.x, u2.x);
        a1 = min3(a1, u.y, u2.y), c1 = max3(c1, u.y, u2.y);
      }
      mn[h][0] = a0, mx[h][0] = c0, mn[h][1] = a1, mx[h][1] = c1;
    }
    float kmn0 = fminf(b2 ? mn[1][0] : mn[0][0], __shfl_xor_sync(0xffffffffu, b2 ? mn[0][0] : mn[1][0], 16));
    float kmn1 = fminf(b2 ? mn[1][1] : mn[0][1], __shfl_xor_sync(0xffffffffu, b2 ? mn[0][1] : mn[1][1], 16));
    float kmx0 = fmaxf(b2 ? mx[1][0] : mx[0][0], __shfl_xor_sync(0xffffffffu, b2 ? mx[0][0] : mx[1][0], 16));
    float kmx1 = fmaxf(b2 ? mx[1][1] : mx[0][1], __shfl_xor_sync(0xffffffffu, b2 ? mx[0][1] : mx[1][1], 16));
    float omn = fminf(b1 ? kmn1 : kmn0, __shfl_xor_sync(0xffffffffu, b1 ? kmn0 : kmn1, 8));
    float omx = fmaxf(b1 ? kmx1 : kmx0, __shfl_xor_sync(0xffffffffu, b1 ? kmx0 : kmx1, 8));
    omn = fminf(omn, __shfl_xor_sync(0xffffffffu, omn, 4));
    omx = fmaxf(omx, __shfl_xor_sync(0xffffffffu, omx, 4));
    if constexpr (W > 1) {
      const int tok = 8 * b2 + 2 * t + b1;
      if ((lane & 4) == 0) sh.mm[blk][tok] = make_float2(omn, omx);
      __syncthreads();
#pragma unroll
      for (int k = 0; k < W; ++k) {
        const float2 x = sh.mm[k][tok];
        omn = fminf(omn, x.x), omx = fmaxf(omx, x.y);
        cmax = fmaxf(cmax, sh.cmax[k]);
      }
    }
    // Stored balance: the power of two 2^kb with max c in (2^(kb-1), 2^kb]
    // moves from c into a and z (exact; the dequantised tile is unchanged).
    const uint32_t cbits = __float_as_uint(cmax);
    const int kb = (int)(cbits >> 23) - 127 + ((cbits & 0x7FFFFFu) != 0u);
    if (wt == 0) {
      const float cs = __uint_as_float((uint32_t)(127 - kb) << 23);
      const size_t ci = slot * D + kBlk * blk + 16 * g + 4 * t;
      if (p.dst.meta16) {  // half metadata: rounded to nearest from the float32 value
        const __half2 lo = __floats2half2_rn(cv4.x * cs, cv4.y * cs), hi = __floats2half2_rn(cv4.z * cs, cv4.w * cs);
        *reinterpret_cast<uint2*>(static_cast<__half*>(p.dst.chan) + ci) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
      } else {
        *reinterpret_cast<float4*>(static_cast<float*>(p.dst.chan) + ci) =
            make_float4(cv4.x * cs, cv4.y * cs, cv4.z * cs, cv4.w * cs);
      }
    }
    constexpr float kQmax = (float)((1 << BITS) - 1);
    const float s_own = (omx - omn) / kQmax;
    const float is_own = s_own > 0.f ? rcp_nr(s_own) : 0.f;
    // 1/sqrt(block) times the row's power of two times the balance 2^kb
    const float fold = inv_sqrt_d * rsc_own * __uint_as_float((uint32_t)(127 + kb) << 23);
    if ((lane & 4) == 0 && blk == 0) {
      const size_t ti = slot * (kTile * 2) + 2 * (kT * wt + 8 * b2 + 2 * t + b1);
      if (p.dst.meta16)
        *reinterpret_cast<__half2*>(static_cast<__half*>(p.dst.tok) + ti) = __floats2half2_rn(s_own * fold, omn * fold);
      else
        *reinterpret_cast<float2*>(static_cast<float*>(p.dst.tok) + ti) = make_float2(s_own * fold, omn * fold);
    }
    f2 m2h[2], is2h[2];  // row minimum and 1/step of the lane's tokens 8h + 2t, 8h + 2t + 1
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      m2h[h] = make_float2(__shfl_sync(0xffffffffu, omn, (h << 4) | t), __shfl_sync(0xffffffffu, omn, (h << 4) | 8 | t));
      is2h[h] = make_float2(__shfl_sync(0xffffffffu, is_own, (h << 4) | t),
                            __shfl_sync(0xffffffffu, is_own, (h << 4) | 8 | t));
    }
    // (y - m) / s rounded to the nearest integer (ties to even) by the single
    // rounding of the fused multiply-add into the magic number
    emit_codes(slot, [&](int h, int j) { return fma2(sub2(P[h][j >> 3][j & 7], m2h[h]), is2h[h], splat2(kMagic)); });
    tile_sync<W>();  // shared tile buffers are reused by the next tile
  }
  {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_slot), "n"(kTmemCols));
  }
  // Launched as the programmatic dependent of the call's K launch (the V
  // launch), the grid ends only after that one: later work on the stream
  // sees both complete.  In an ordinary launch this returns at once.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
}
FastDiv make_div(uint32_t d) {
  FastDiv f{d, 0, 0};
  uint32_t s = 0;
  while ((1ull << s) < d) ++s;
  f.s = s;
  f.m = (uint32_t)((((1ull << s) - d) << 32) / d + 1);
  return f;
}

template <bool F16, int BITS, int D, int TW, int AXES>
void launch_one(const QuantLaunch& q, int sms, cudaStream_t s) {
  constexpr int kCW = cta_warps<TW>(), tpc = kCW / ((D / kBlk) * TW);
  constexpr size_t dyn = stage_bytes<TW>();  // raw-tile staging
  const int64_t need = (q.total + tpc - 1) / tpc;
  const int64_t cap = (int64_t)sms * (16 / kCW);  // resident CTAs per SM
  const int grid = (int)(need < cap ? need : cap);
  auto kern = quantize_kernel<F16, BITS, D, TW, AXES>;
  // static + dynamic shared memory may pass 48 KB, which needs the opt-in
  if (dyn > 0) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
  if (q.after_k) {  // the V launch: independent of the K launch before it, so it may overlap that one's tail
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kCW * 32);
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kern, q);
  } else {
    kern<<<grid, kCW * 32, dyn, s>>>(q);
  }
}

template <bool F16, int D, int TW, int AXES = 0>
int launch_bits(const QuantLaunch& q, int bits, int sms, cudaStream_t s) {
  switch (bits) {
    case 2: launch_one<F16, 2, D, TW, AXES>(q, sms, s); break;
    case 3: launch_one<F16, 3, D, TW, AXES>(q, sms, s); break;
    case 4: launch_one<F16, 4, D, TW, AXES>(q, sms, s); break;
    case 8: launch_one<F16, 8, D, TW, AXES>(q, sms, s); break;
    default: return (int)cudaErrorInvalidValue;
  }
  return (int)cudaGetLastError();
}

template <bool F16>
int launch_shape(const QuantLaunch& q, int head_dim, int tile_tokens, int sms, cudaStream_t s) {
  const int bits = q.dst.bits;
  if (head_dim == 512 && tile_tokens == 16) return launch_bits<F16, 512, 1>(q, bits, sms, s);
  if (head_dim != 128) return (int)cudaErrorInvalidValue;
  switch (tile_tokens) {
    case 16:  // blocks below 8 channels or per-channel key groups: the ablation instantiation
      return (q.hblock < 8 || q.dst.per_channel) ? launch_bits<F16, 128, 1, 1>(q, bits, sms, s)
                                                 : launch_bits<F16, 128, 1>(q, bits, sms, s);
    case 32: return launch_bits<F16, 128, 2>(q, bits, sms, s);
    case 64: return launch_bits<F16, 128, 4>(q, bits, sms, s);
    case 128: return launch_bits<F16, 128, 8>(q, bits, sms, s);
    default: return (int)cudaErrorInvalidValue;
  }
}

}  // namespace

int launch_quantize(const QuantizeParams& p, bool f16, int head_dim, int tile_tokens, void* stream) {
  if (p.total_tiles == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const uint32_t per_kind = (uint32_t)(p.total_tiles / p.kinds);
  const uint32_t ntt = (uint32_t)(p.n_tok / tile_tokens);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int kind = 0; kind < p.kinds; ++kind) {
    QuantLaunch q;
    q.src = static_cast<const uint16_t*>(p.src[kind]);
    q.dst = p.dst[kind];
    q.n_tok = p.n_tok;
    q.num_layers = p.num_layers;
    q.num_heads = p.num_heads;
    q.num_pages = p.num_pages;
    q.iters = p.iters;
    q.dst_page = p.dst_page;
    q.err = p.err;
    q.total = per_kind;
    q.div_h = make_div((uint32_t)p.num_heads);
    q.div_ntt = make_div(ntt);
    q.rope_src = kind == 0 ? static_cast<const uint16_t*>(p.rope_src) : nullptr;
    q.rope_dst = static_cast<uint16_t*>(p.rope_dst);
    q.rope_dim = p.rope_dim;
    q.hblock = p.hblock;
    q.inv_sqrt_b = inv_sqrt_pow2(p.hblock);
    q.after_k = kind == 1;
    const int e = f16 ? launch_shape<true>(q, head_dim, tile_tokens, sms, s)
                      : launch_shape<false>(q, head_dim, tile_tokens, sms, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace kvq
