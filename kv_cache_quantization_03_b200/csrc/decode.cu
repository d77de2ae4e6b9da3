// Decode attention over the quantised cache, head_dim 128, pages of 16..128
// tokens, query groups of 1..8 heads per kv-head (sm_100a).
//
// Consumer of the KVarN cache (KVarN project page on open-radar, Key
// Features, "Variance-Normalized Quantization Pipeline" and "Throughput Above
// FP16": the cache is read in its quantised form).  The query is rotated with
// the same Sylvester H/sqrt(128) as the cache, so attention runs in the
// rotated domain on (a q + z) c with the scales folded in:
//   score(t, h) = scale * (a_t * sum_j u_hj q_tj + z_t * sum_j u_hj),
//                 u_h = rotate(q_h) * c_K             (per tile)
//   out_h      += c_V * (sum_t w_th qv_t + sum_t p_th z_t),  w_th = p_th a_t
// with an online softmax across tiles, then the output is rotated back.
//
// Work split: grid (splits, batch * kv_heads).  The unit of work is a tile of
// 16 tokens: a whole page, or one of the 16-token slices of a longer page
// (each slice reads its rows of codes and token scales and the page's channel
// scales).  Each CTA of 4 warps owns a contiguous range of one sequence's
// tiles; each warp takes every 4th tile and streams it through its own ring
// of shared-memory stages filled with 1-D bulk async copies (one mbarrier per
// stage, bounded waits).  Both
// contractions of a tile run as m16n8k16 f16 MMAs with fp32 accumulation:
// codes 0..255 are exact in f16; u and w are each carried as an f16 pair
// hi + lo (two MMAs into one fp32 accumulator), which keeps ~22 significant
// bits where a single f16 would cost up to 8e-3 of attention accuracy.
//   scores:  D[16 tokens x 8 heads]   = codes_K[16 x 128] * u^T[128 x 8]
//   values:  D[128 channels x 8 heads] = codes_V^T[128 x 16] * w[16 x 8]
// The per-channel c_V is applied to each tile's fresh MMA result before it
// joins the running output.  A second kernel merges the split partials,
// normalises and rotates back.
#include <cuda_runtime.h>

#include "kvq_device.cuh"

namespace kvq {
namespace {

constexpr int kD = 128;
constexpr int kT = 16;
constexpr int kDW = 4;      // warps per CTA
constexpr int kStages = 3;  // ring depth per warp
constexpr float kNegBig = -1e30f;

struct StageLayout {
  int kcb, vcb, off_kaz, off_kc, off_v, off_vaz, off_vc, bytes;
};

// One stage: the tile of nh adjacent kv-heads (their pages are contiguous in
// every cache array): K codes | K group scales | K c | V codes | V (a, z) |
// V c, with m bytes per scale (4: float32, 2: half).  Key group scales are
// (a, z) per token, or (s, m) per channel with per-channel keys (kpc), which
// have no c.
__host__ __device__ constexpr int kgroup_bytes(int m, int kpc) { return kpc ? kD * 2 * m : kT * 2 * m; }
__host__ __device__ constexpr StageLayout stage_layout(int bk, int bv, int nh, int m, int kpc) {
  return StageLayout{nh * kT * kD * bk / 8,
                     nh * kT * kD * bv / 8,
                     nh * (kT * kD * bk / 8),
                     nh * (kT * kD * bk / 8 + kgroup_bytes(m, kpc)),
                     nh * (kT * kD * bk / 8 + kgroup_bytes(m, kpc) + (kpc ? 0 : kD * m)),
                     nh * (kT * kD * bk / 8 + kgroup_bytes(m, kpc) + (kpc ? 0 : kD * m)) + nh * kT * kD * bv / 8,
                     nh * (kT * kD * bk / 8 + kgroup_bytes(m, kpc) + (kpc ? 0 : kD * m)) +
                         nh * (kT * kD * bv / 8 + kT * 2 * m),
                     nh * (kT * kD * (bk + bv) / 8 + kgroup_bytes(m, kpc) + (kpc ? 0 : kD * m) + kT * 2 * m + kD * m)};
}

// (a, z) of token i, and c of channels i .. i + 3, from a stage's metadata
// (M = 4: float32, 2: half).
template <int M>
__device__ __forceinline__ float2 ld_az(const uint8_t* base, int i) {
  if constexpr (M == 4) return reinterpret_cast<const float2*>(base)[i];
  else return __half22float2(reinterpret_cast<const __half2*>(base)[i]);
}
template <int M>
__device__ __forceinline__ float4 ld_c4(const uint8_t* base, int i) {
  if constexpr (M == 4) {
    return *reinterpret_cast<const float4*>(base + 4 * i);
  } else {
    const uint2 h = *reinterpret_cast<const uint2*>(base + 2 * i);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&h.y));
    return make_float4(a.x, a.y, b.x, b.y);
  }
}
// Ring depth per warp: 3 stages of one kv-head, 2 of a pair (four CTAs per SM).
__host__ __device__ constexpr int num_stages(int nh) { return nh == 2 ? 2 : kStages; }

// ---- code pairs -> f16x2 (exact small integers)
// A field of a 32-bit word masked in place in both halves and OR-ed into the
// exponent of 1024 reads as the f16 value 1024 + code * 2^shift; one HFMA2
// (scale 2^-shift, bias -1024 * 2^-shift) leaves the code.
template <int SHIFT>
__device__ __forceinline__ uint32_t h2_field(uint32_t word, uint32_t mask) {
  uint32_t v = (word & (mask << SHIFT)) | 0x64006400u;
  __half2 h = *reinterpret_cast<__half2*>(&v);
  if constexpr (SHIFT == 0) {
    h = __hsub2(h, __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400)));
  } else {
    constexpr float sc = 1.0f / (1 << SHIFT);
    const __half2 s2 = __float2half2_rn(sc), b2 = __float2half2_rn(-1024.0f * sc);
    h = __hfma2(h, s2, b2);
  }
  return *reinterpret_cast<uint32_t*>(&h);
}
// The same conversion for a word whose two fields (at bit `shift` of each
// half) are already masked and OR-ed into 0x6400 (shift constant after
// unrolling).
__device__ __forceinline__ uint32_t h2_scaled(uint32_t v, int shift) {
  __half2 h = *reinterpret_cast<__half2*>(&v);
  if (shift == 0) {
    h = __hsub2(h, __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400)));
  } else {
    const float sc = 1.0f / (float)(1 << shift);
    h = __hfma2(h, __float2half2_rn(sc), __float2half2_rn(-1024.0f * sc));
  }
  return *reinterpret_cast<uint32_t*>(&h);
}

// Four code pairs of one word of 4-bit codes: (nibble e, nibble e+4), e = 0..3.
__device__ __forceinline__ void nib_pairs(uint32_t w, uint32_t* out) {
  const uint32_t w8 = w >> 8;
  out[0] = h2_field<0>(w, 0x000F000Fu);
  out[1] = h2_field<4>(w, 0x000F000Fu);
  out[2] = h2_field<0>(w8, 0x000F000Fu);
  out[3] = h2_field<4>(w8, 0x000F000Fu);
}
// Eight code pairs of one word of 2-bit codes: (field e, field e+8), e = 0..7.
__device__ __forceinline__ void crumb_pairs(uint32_t w, uint32_t* out) {
  const uint32_t w8 = w >> 8;
  out[0] = h2_field<0>(w, 0x00030003u);
  out[1] = h2_field<2>(w, 0x00030003u);
  out[2] = h2_field<4>(w, 0x00030003u);
  out[3] = h2_field<6>(w, 0x00030003u);
  out[4] = h2_field<0>(w8, 0x00030003u);
  out[5] = h2_field<2>(w8, 0x00030003u);
  out[6] = h2_field<4>(w8, 0x00030003u);
  out[7] = h2_field<6>(w8, 0x00030003u);
}

// Key-side pairing: lane t covers channels 32t..32t+31 of a token row; pair
// pi (0..15) holds channels (chan(pi), chan(pi) + dist) relative to 32t.
template <int B>
__host__ __device__ constexpr int kdist() {
  return B == 4 ? 4 : (B == 8 ? 2 : 8);
}
template <int B>
__host__ __device__ constexpr int kchan(int pi) {
  return B == 4 ? 8 * (pi >> 2) + (pi & 3) : (B == 8 ? 4 * (pi >> 1) + (pi & 1) : 16 * (pi >> 3) + (pi & 7));
}

// Each lane t works on the 32 channels 32t..32t+31 in a "slot" order rotated
// by rot(t) channels: slot i is channel 32t + (i + rot(t)) % 32.  With the
// rotation the lanes t = 0..3 read the per-channel key scales from different
// shared-memory banks; codes, scales and the query use the same slot order.
template <int B>
__device__ __forceinline__ int rot_channels(int t) {
  return (B == 4 || B == 8) ? 8 * t : 16 * (t & 1);
}

// Pairs of one token row for the key MMA (16 pairs = 32 codes), slot order.
template <int B>
__device__ __forceinline__ void key_pairs(const uint8_t* codes, int row, int t, uint32_t (&pr)[16]) {
  if constexpr (B == 4) {  // slot word m = channel word (m + t) % 4
    const uint8_t* r = codes + row * 64 + 16 * t;
#pragma unroll
    for (int m = 0; m < 4; ++m) nib_pairs(*reinterpret_cast<const uint32_t*>(r + 4 * ((m + t) & 3)), pr + 4 * m);
  } else if constexpr (B == 2) {  // slot word m = channel word (m + t) % 2
    const uint8_t* r = codes + row * 32 + 8 * t;
    crumb_pairs(*reinterpret_cast<const uint32_t*>(r + 4 * (t & 1)), pr);
    crumb_pairs(*reinterpret_cast<const uint32_t*>(r + 4 * ((t + 1) & 1)), pr + 8);
  } else if constexpr (B == 8) {  // slot word m = channel word (m + 2t) % 8
    const uint8_t* r = codes + row * 128 + 32 * t;
    uint32_t ws[8];
#pragma unroll
    for (int m = 0; m < 8; m += 2) {
      const uint2 x = *reinterpret_cast<const uint2*>(r + 4 * ((m + 2 * t) & 7));
      ws[m] = x.x, ws[m + 1] = x.y;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      pr[2 * k] = h2_field<0>(ws[k], 0x00FF00FFu);
      pr[2 * k + 1] = h2_field<0>(ws[k] >> 8, 0x00FF00FFu);
    }
  } else {  // 3 bits: low plane [T][32 B] then high plane [T][16 B]; rotation by 16 (t & 1)
    const uint8_t* r = codes + row * 32 + 8 * t;
    const uint32_t w0 = *reinterpret_cast<const uint32_t*>(r + 4 * (t & 1));
    const uint32_t w1 = *reinterpret_cast<const uint32_t*>(r + 4 * ((t + 1) & 1));
    uint32_t hw = *reinterpret_cast<const uint32_t*>(codes + kT * 32 + row * 16 + 4 * t);
    hw = (t & 1) ? __funnelshift_r(hw, hw, 16) : hw;
    const uint32_t hs[2] = {__byte_perm(hw, 0u, 0x4140u), __byte_perm(hw, 0u, 0x4342u)};
    // Pair pi = channels (pi, pi + 8) of word pi >> 3: its low crumbs sit at
    // bit s = 2 (pi & 3) of each half (of the word, or of the word >> 8 for
    // pi & 4), its high bits at bit pi & 7 of each half of hs[pi >> 3].  The
    // high bits are moved next to the crumbs (bit s + 2), so one field of
    // 3-bit codes times 2^s goes through a single f16 conversion.
    const uint32_t w8[2] = {w0 >> 8, w1 >> 8};
#pragma unroll
    for (int pi = 0; pi < 16; ++pi) {
      const int s = 2 * (pi & 3), sh = s + 2 - (pi & 7);
      const uint32_t v = (pi & 4) ? w8[pi >> 3] : ((pi >> 3) ? w1 : w0);
      const uint32_t h = hs[pi >> 3];
      const uint32_t hb = sh >= 0 ? (h << sh) : (h >> -sh);
      const uint32_t f = (v & (0x00030003u << s)) | (hb & (0x00040004u << s)) | 0x64006400u;
      pr[pi] = h2_scaled(f, s);
    }
  }
}

// Value-side pairs: f16x2 of (token x, token y) at lane g's channel 16g + c.
template <int B>
__device__ __forceinline__ void value_pairs(const uint8_t* codes, int rx, int ry, int g, uint32_t (&pr)[16]) {
  if constexpr (B == 4) {
    const uint2 x = *reinterpret_cast<const uint2*>(codes + rx * 64 + 8 * g);
    const uint2 y = *reinterpret_cast<const uint2*>(codes + ry * 64 + 8 * g);
    const uint32_t xs[2] = {x.x, x.y}, ys[2] = {y.x, y.y};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // bytes 2(k&1), 2(k&1)+1 of both tokens: channels 4k..4k+3, x in the low half
      const uint32_t m = __byte_perm(xs[k >> 1], ys[k >> 1], (k & 1) ? 0x7632u : 0x5410u);
      const uint32_t m8 = m >> 8;
      pr[4 * k] = h2_field<0>(m, 0x000F000Fu);
      pr[4 * k + 1] = h2_field<4>(m, 0x000F000Fu);
      pr[4 * k + 2] = h2_field<0>(m8, 0x000F000Fu);
      pr[4 * k + 3] = h2_field<4>(m8, 0x000F000Fu);
    }
  } else if constexpr (B == 2) {
    const uint32_t x = *reinterpret_cast<const uint32_t*>(codes + rx * 32 + 4 * g);
    const uint32_t y = *reinterpret_cast<const uint32_t*>(codes + ry * 32 + 4 * g);
    crumb_pairs(__byte_perm(x, y, 0x5410u), pr);
    crumb_pairs(__byte_perm(x, y, 0x7632u), pr + 8);
  } else {  // 8 bits
    const uint4 x = *reinterpret_cast<const uint4*>(codes + rx * 128 + 16 * g);
    const uint4 y = *reinterpret_cast<const uint4*>(codes + ry * 128 + 16 * g);
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t m = __byte_perm(xs[k >> 1], ys[k >> 1], (k & 1) ? 0x7632u : 0x5410u);
      pr[2 * k] = h2_field<0>(m, 0x00FF00FFu);
      pr[2 * k + 1] = h2_field<0>(m >> 8, 0x00FF00FFu);
    }
  }
}

__device__ __forceinline__ float ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ float bf16_to_f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Waits until the grid this one was launched after as a programmatic
// dependent has completed and its writes are visible (returns at once in an
// ordinary launch).
__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// A device word that nothing ever sets: the testing hook's wait polls it
// until its time limit runs out.
__device__ uint32_t g_never_set = 0;

// Testing hook: lane 0 polls g_never_set for at most `ns` nanoseconds; true
// if the flag was seen set (never, by construction).
__device__ __forceinline__ bool wait_never_set(uint32_t ns) {
  uint64_t t0, t1;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (;;) {
    if (*reinterpret_cast<volatile uint32_t*>(&g_never_set)) return true;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
    if (t1 - t0 >= ns) return false;
  }
}

// NH = 1: one kv-head per CTA, its (up to 8) query heads on the MMA's 8
// columns.  NH = 2 (groups of at most 4 query heads): two adjacent kv-heads
// per CTA; head slot n (column n of the MMAs) is query head n % 4 of kv-head
// n / 4.  Lane (g, t) computes u for slot g and owns the score/output columns
// 2t, 2t+1, i.e. kv-head hs = t / 2.  The score MMAs run once per kv-head
// (each lane keeps the result of its own kv-head); for P V each kv-head's
// weights are masked to its own columns, so both MMAs add into one result.
// FILL: the instance for quantise-on-fill calls (p.fill_page set), launched as
// the programmatic dependent of the fill's quantize launch; the other
// instance carries none of its waits.
template <int BK, int BV, int NH, int M, int KPC, bool FILL>
__global__ void __launch_bounds__(kDW * 32, 4) decode_d128_kernel(DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  // the combine kernel (this grid's programmatic dependent) may start now: it
  // scores the unquantised tails, then waits for this grid's partials
  asm volatile("griddepcontrol.launch_dependents;");
  constexpr StageLayout SL = stage_layout(BK, BV, NH, M, KPC);
  constexpr int KG = kgroup_bytes(M, KPC);  // key group-scale bytes of one kv-head's tile
  constexpr int kStages = num_stages(NH);
  constexpr int KCB = SL.kcb / NH, VCB = SL.vcb / NH;  // code bytes of one kv-head's tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDW * kStages * SL.bytes);
  uint8_t* wsm = smem + warp * kStages * SL.bytes;
  uint64_t* wbar = bars + warp * kStages;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(&wbar[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  const int kvh_per_seq = p.num_kv_heads / NH;
  const int b = blockIdx.y / kvh_per_seq, kvh = (blockIdx.y % kvh_per_seq) * NH;  // first kv-head of the CTA
  const int split = blockIdx.x;
  int seq = p.seq_lens[b];
  if (seq < 0) {
    if (threadIdx.x == 0 && split == 0) set_error(p.err, KVQ_DEVERR_BAD_SEQ);
    seq = 0;
  }
  const int page_tokens = kT << p.sub_log2;
  int npages = seq / page_tokens;
  if ((seq % page_tokens) && threadIdx.x == 0 && split == 0) set_error(p.err, KVQ_DEVERR_PARTIAL_TILE);
  if (npages > p.max_pages) {
    if (threadIdx.x == 0 && split == 0) set_error(p.err, KVQ_DEVERR_BAD_SEQ);
    npages = p.max_pages;
  }
  const int ntiles = npages << p.sub_log2;  // 16-token tiles
  const int t0 = split * p.tiles_per_split;
  const int t1 = min(t0 + p.tiles_per_split, ntiles);
  const int my_n = (t1 > t0 + warp) ? (t1 - t0 - warp + kDW - 1) / kDW : 0;
  // the page id of each of this split's tiles, staged once in shared memory
  int32_t* spg = reinterpret_cast<int32_t*>(bars + kDW * kStages);
  // quantise-on-fill: the first of this split's tiles on the page the fill
  // writes for sequence b (INT_MAX: none); copies from there on wait for the
  // fill's grid
  __shared__ int fill_lo;
  int my_fill = INT_MAX;
  {
    const int32_t* btab = p.block_table + (size_t)b * p.max_pages;
    const int32_t fp = FILL ? p.fill_page[b] : -1;
    for (int i = threadIdx.x; i < t1 - t0; i += kDW * 32) {
      const int32_t pg = btab[(t0 + i) >> p.sub_log2];
      spg[i] = pg;
      if (FILL && fp >= 0 && pg == fp) my_fill = min(my_fill, i);
    }
  }
  if (FILL && threadIdx.x == 0) fill_lo = INT_MAX;
  __shared__ uint32_t tmem_slot;
  if (warp == 0) {  // 32 TMEM columns: each warp keeps its lanes' rotated query in its lane quarter
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 32;" ::"r"(smem_u32(&tmem_slot)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tq = tmem_slot + ((uint32_t)(warp * 32) << 16);
  if constexpr (FILL) {
    if (my_fill != INT_MAX) atomicMin(&fill_lo, my_fill);
    __syncthreads();
  }

  // ---- rotated, pre-scaled query of the CTA's 8 heads: lane (g, t) computes head
  // slot g, channels 32t..32t+31, puts them in its slot order (through this
  // warp's not-yet-used stage memory) and keeps them in tensor memory
  {
    float qr[32];
    const int hh = NH == 2 ? (g & 3) : g, hk = NH == 2 ? kvh + (g >> 2) : kvh;  // slot g: head hh of kv-head hk
    const bool live = hh < p.group;
    const uint16_t* qp = p.q + ((size_t)b * p.num_q_heads + (size_t)hk * p.group + (live ? hh : 0)) * kD + 32 * t;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 w = *reinterpret_cast<const uint4*>(qp + 8 * k);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qr[8 * k + 2 * e] = live ? bf16_to_f((uint16_t)(ws[e] & 0xFFFF)) : 0.f;
        qr[8 * k + 2 * e + 1] = live ? bf16_to_f((uint16_t)(ws[e] >> 16)) : 0.f;
      }
    }
    // H over channel bits 0..4 in registers, bits 5 and 6 across the lanes t;
    // a block-diagonal rotation (blocks of hblock channels) stops at its block
#pragma unroll
    for (int s = 1; s < 32; s <<= 1)
      if (s < p.hblock) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (!(i & s)) {
            const float x = qr[i], y = qr[i + s];
            qr[i] = x + y;
            qr[i + s] = x - y;
          }
      }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
      if (32 * off >= p.hblock) break;
      const bool upper = (t & off) != 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, qr[i], off);
        qr[i] = upper ? (o - qr[i]) : (qr[i] + o);
      }
    }
    const float f = p.scale_log2 * inv_sqrt_pow2(p.hblock);  // softmax scale * log2(e) / sqrt(block)
    float* scr = reinterpret_cast<float*>(wsm) + lane * 33;
#pragma unroll
    for (int i = 0; i < 32; ++i) scr[i] = qr[i] * f;
    __syncwarp();
    const int rot = rot_channels<BK>(t);
#pragma unroll
    for (int i = 0; i < 32; ++i) qr[i] = scr[(i + rot) & 31];
    __syncwarp();
    if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // before the stage refills
    tmem_st32(tq, qr);
  }

  // Testing hook (kvq_set_test_wait): a bounded wait on a flag that nothing
  // sets runs out before any copy is issued; the warp reports a timeout and
  // skips its tiles, so nothing is in flight when it leaves.
  int n_run = my_n;
  if (p.test_wait_ns) {
    const bool got = __shfl_sync(0xffffffffu, lane == 0 ? (int)wait_never_set(p.test_wait_ns) : 0, 0) != 0;
    if (!got) {
      n_run = 0;
      if (lane == 0) set_error(p.err, KVQ_DEVERR_TIMEOUT);
    }
  }

  // ---- producer: lane 0 fills stage (i % kStages) with local tile i
  auto issue = [&](int i) {
    if (lane != 0) return;
    uint64_t* bar = &wbar[i % kStages];
    uint8_t* st = wsm + (i % kStages) * SL.bytes;
    const int li = warp + i * kDW;
    const int page = spg[li];
    if (page < 0 || page >= p.num_pages) {
      set_error(p.err, KVQ_DEVERR_BAD_PAGE);
      mbar_arrive_expect_tx(bar, 0);
      return;
    }
    const size_t slot = ((size_t)p.layer * p.num_pages + page) * p.num_kv_heads + kvh;
    if (FILL && li >= fill_lo) wait_prior_grid();  // the fill's quantize grid writes this page
    mbar_arrive_expect_tx(bar, (uint32_t)SL.bytes);
    const uint8_t* ktok = static_cast<const uint8_t*>(p.k.tok);
    const uint8_t* kch = static_cast<const uint8_t*>(p.k.chan);
    const uint8_t* vtok = static_cast<const uint8_t*>(p.v.tok);
    const uint8_t* vch = static_cast<const uint8_t*>(p.v.chan);
    if (p.sub_log2 == 0) {  // 16-token pages: the nh kv-heads' pages are contiguous in every array
      bulk_g2s(st, p.k.codes + slot * KCB, SL.kcb, bar);
      bulk_g2s(st + SL.off_kaz, ktok + slot * KG, NH * KG, bar);
      if constexpr (!KPC) bulk_g2s(st + SL.off_kc, kch + slot * (kD * M), NH * kD * M, bar);
      bulk_g2s(st + SL.off_v, p.v.codes + slot * VCB, SL.vcb, bar);
      bulk_g2s(st + SL.off_vaz, vtok + slot * (kT * 2 * M), NH * kT * 2 * M, bar);
      bulk_g2s(st + SL.off_vc, vch + slot * (kD * M), NH * kD * M, bar);
      return;
    }
    // longer pages: slice `sub` of each kv-head's page, in the same stage layout
    // (per-channel keys come with 16-token pages only)
    const int spt = 1 << p.sub_log2, sub = (t0 + li) & (spt - 1);
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const size_t sh = slot + h;
      const uint8_t* kc = p.k.codes + sh * (size_t)(spt * KCB);
      if constexpr (BK == 3) {  // the slice's rows of the low-bit plane, then of the high-bit plane
        bulk_g2s(st + h * KCB, kc + sub * (kT * kD / 4), kT * kD / 4, bar);
        bulk_g2s(st + h * KCB + kT * kD / 4, kc + spt * (kT * kD / 4) + sub * (kT * kD / 8), kT * kD / 8, bar);
      } else {
        bulk_g2s(st + h * KCB, kc + sub * KCB, KCB, bar);
      }
      if constexpr (!KPC) {
        bulk_g2s(st + SL.off_kaz + h * (kT * 2 * M), ktok + (sh * spt + sub) * (kT * 2 * M), kT * 2 * M, bar);
        bulk_g2s(st + SL.off_kc + h * (kD * M), kch + sh * (kD * M), kD * M, bar);
      }
      static_assert(BV != 3, "3-bit values have two planes");
      bulk_g2s(st + SL.off_v + h * VCB, p.v.codes + (sh * spt + sub) * VCB, VCB, bar);
      bulk_g2s(st + SL.off_vaz + h * (kT * 2 * M), vtok + (sh * spt + sub) * (kT * 2 * M), kT * 2 * M, bar);
      bulk_g2s(st + SL.off_vc + h * (kD * M), vch + sh * (kD * M), kD * M, bar);
    }
  };
  const int pre = n_run < kStages ? n_run : kStages;
  for (int i = 0; i < pre; ++i) issue(i);
  int issued = pre;

  float mrun[2] = {kNegBig, kNegBig};  // running max of heads 2t, 2t+1 (log2 units)
  float lrun[2] = {0.f, 0.f};          // this lane's share of the running sums
  f2 O[8][2];                          // [m-block][row g / g+8] x heads (2t, 2t+1)
#pragma unroll
  for (int mb = 0; mb < 8; ++mb) O[mb][0] = O[mb][1] = make_float2(0.f, 0.f);
  const float zero4[4] = {0.f, 0.f, 0.f, 0.f};

  int stop = -1;  // local tile whose wait ran out
  for (int i = 0; i < n_run; ++i) {
    const bool ok = mbar_wait_bounded(&wbar[i % kStages], (uint32_t)(i / kStages) & 1u, kWaitLimit);
    if (!__all_sync(0xffffffffu, ok)) {
      stop = i;
      if (lane == 0) set_error(p.err, KVQ_DEVERR_TIMEOUT);
      break;
    }
    const int page = spg[warp + i * kDW];
    if (page >= 0 && page < p.num_pages) {
      const uint8_t* st = wsm + (i % kStages) * SL.bytes;
      const int hu = NH == 2 ? (g >> 2) : 0, hs = NH == 2 ? (t >> 1) : 0;  // kv-head of this lane's u / columns
      const uint8_t* kaz = st + SL.off_kaz + hs * KG;
      // per-token keys: c of kv-head hu; per-channel keys: its (s, m) pairs
      const uint8_t* kc = KPC ? st + SL.off_kaz + hu * KG : st + SL.off_kc + hu * (kD * M);
      const uint8_t* vaz = st + SL.off_vaz + hs * (2 * kT * M);
      const uint8_t* vc = st + SL.off_vc + hs * (kD * M);

      // u = q~ * c_K on this lane's 32 channels (slot order), and its sum
      float u[32];
      f2 su2 = make_float2(0.f, 0.f);
      {
        const int rq = rot_channels<BK>(t) >> 2;
        float qv[32];  // slot order
        tmem_ld32(tq, qv);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int kk = 4 * ((k + rq) & 7);
          const f2 q01 = make_float2(qv[4 * k], qv[4 * k + 1]), q23 = make_float2(qv[4 * k + 2], qv[4 * k + 3]);
          f2 a, d;
          if constexpr (KPC) {  // u = q~ s; su2 gathers beta = sum q~ m, which takes z's place
            const float2 p0 = ld_az<M>(kc, 32 * t + kk), p1 = ld_az<M>(kc, 32 * t + kk + 1);
            const float2 p2 = ld_az<M>(kc, 32 * t + kk + 2), p3 = ld_az<M>(kc, 32 * t + kk + 3);
            a = mul2(q01, make_float2(p0.x, p1.x));
            d = mul2(q23, make_float2(p2.x, p3.x));
            su2 = fma2(q01, make_float2(p0.y, p1.y), fma2(q23, make_float2(p2.y, p3.y), su2));
          } else {
            const float4 c4 = ld_c4<M>(kc, 32 * t + kk);
            a = mul2(q01, make_float2(c4.x, c4.y));
            d = mul2(q23, make_float2(c4.z, c4.w));
            su2 = add2(su2, add2(a, d));
          }
          u[4 * k] = a.x, u[4 * k + 1] = a.y, u[4 * k + 2] = d.x, u[4 * k + 3] = d.y;
        }
      }
      uint32_t ubh[16], ubl[16];  // u = hi + lo, both f16: ~22 significant bits
#pragma unroll
      for (int pi = 0; pi < 16; ++pi) {
        const int c0 = kchan<BK>(pi), c1 = c0 + kdist<BK>();
        split_f16x2(u[c0], u[c1], ubh[pi], ubl[pi]);
      }
      float su = su2.x + su2.y;
      su += __shfl_xor_sync(0xffffffffu, su, 1);
      su += __shfl_xor_sync(0xffffffffu, su, 2);
      const float su0 = __shfl_sync(0xffffffffu, su, 8 * t);       // head 2t
      const float su1 = __shfl_sync(0xffffffffu, su, 8 * t + 4);   // head 2t+1

      // scores: tokens g, g+8 x heads 2t, 2t+1 (each kv-head's codes against all
      // columns; a lane keeps its own kv-head's result)
      float S[4];
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        uint32_t kp0[16], kp1[16];
        key_pairs<BK>(st + h * KCB, g, t, kp0);
        key_pairs<BK>(st + h * KCB, g + 8, t, kp1);
        float Sh[4] = {0.f, 0.f, 0.f, 0.f}, Sl[4] = {0.f, 0.f, 0.f, 0.f};  // two independent MMA chains
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint32_t a[4] = {kp0[2 * s], kp1[2 * s], kp0[2 * s + 1], kp1[2 * s + 1]};
          mma16816<true>(Sh, a, ubh[2 * s], ubh[2 * s + 1], Sh);
          mma16816<true>(Sl, a, ubl[2 * s], ubl[2 * s + 1], Sl);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (h == 0 || hs == h) S[e] = Sh[e] + Sl[e];
      }
      // per-channel keys: score = S + beta (a = 1, and su0, su1 hold beta)
      const float2 az0 = KPC ? make_float2(1.f, 1.f) : ld_az<M>(kaz, g);
      const float2 az1 = KPC ? make_float2(1.f, 1.f) : ld_az<M>(kaz, g + 8);
      float sc[4];
      sc[0] = fmaf(az0.x, S[0], az0.y * su0);
      sc[1] = fmaf(az0.x, S[1], az0.y * su1);
      sc[2] = fmaf(az1.x, S[2], az1.y * su0);
      sc[3] = fmaf(az1.x, S[3], az1.y * su1);

      // online softmax (heads 2t, 2t+1; tokens spread over g)
      float tm0 = fmaxf(sc[0], sc[2]), tm1 = fmaxf(sc[1], sc[3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, off));
        tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, off));
      }
      const float mn0 = fmaxf(mrun[0], tm0), mn1 = fmaxf(mrun[1], tm1);
      const float al0 = ex2(mrun[0] - mn0), al1 = ex2(mrun[1] - mn1);
      mrun[0] = mn0, mrun[1] = mn1;
      const float p0 = ex2(sc[0] - mn0), p1 = ex2(sc[1] - mn1);
      const float p2 = ex2(sc[2] - mn0), p3 = ex2(sc[3] - mn1);
      lrun[0] = fmaf(lrun[0], al0, p0 + p2);
      lrun[1] = fmaf(lrun[1], al1, p1 + p3);

      // value weights w = p * a_V / max(a_V) (f16, transposed into B fragments)
      const float2 vz0 = ld_az<M>(vaz, g);
      const float2 vz1 = ld_az<M>(vaz, g + 8);
      float amax = fmaxf(vz0.x, vz1.x);
      float bz0 = fmaf(p0, vz0.y, p2 * vz1.y), bz1 = fmaf(p1, vz0.y, p3 * vz1.y);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        bz0 += __shfl_xor_sync(0xffffffffu, bz0, off);
        bz1 += __shfl_xor_sync(0xffffffffu, bz1, off);
      }
      const float ia = amax > 0.f ? 1.f / amax : 0.f;
      const float r0 = vz0.x * ia, r1 = vz1.x * ia;
      uint32_t wh0, wl0, wh1, wl1;  // w = hi + lo, both f16
      split_f16x2(p0 * r0, p1 * r0, wh0, wl0);
      split_f16x2(p2 * r1, p3 * r1, wh1, wl1);
      wh0 = movmatrix_trans(wh0), wl0 = movmatrix_trans(wl0);
      wh1 = movmatrix_trans(wh1), wl1 = movmatrix_trans(wl1);

      // values: channels 16g + [0,16) x heads 2t, 2t+1
      float cv[16];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 c4 = ld_c4<M>(vc, 16 * g + 4 * k);
        cv[4 * k] = c4.x, cv[4 * k + 1] = c4.y, cv[4 * k + 2] = c4.z, cv[4 * k + 3] = c4.w;
      }
      const f2 alpha = make_float2(al0, al1), bz = make_float2(bz0, bz1), am = splat2(amax);
      if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {  // a running max moved
#pragma unroll
        for (int mb = 0; mb < 8; ++mb) O[mb][0] = mul2(O[mb][0], alpha), O[mb][1] = mul2(O[mb][1], alpha);
      }
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        // B fragments of kv-head h: lane (g, t) holds column g, zero outside h's columns
        const bool mine = NH == 1 || (g >> 2) == h;
        const uint32_t bh0 = mine ? wh0 : 0u, bh1 = mine ? wh1 : 0u, bl0 = mine ? wl0 : 0u, bl1 = mine ? wl1 : 0u;
        const f2 bzh = (NH == 1 || hs == h) ? bz : make_float2(0.f, 0.f);
        uint32_t vp0[16], vp1[16];
        value_pairs<BV>(st + SL.off_v + h * VCB, 2 * t, 2 * t + 1, g, vp0);
        value_pairs<BV>(st + SL.off_v + h * VCB, 2 * t + 8, 2 * t + 9, g, vp1);
#pragma unroll
        for (int mb = 0; mb < 8; ++mb) {
          const uint32_t a[4] = {vp0[2 * mb], vp0[2 * mb + 1], vp1[2 * mb], vp1[2 * mb + 1]};
          float d[4];
          mma16816<true>(d, a, bh0, bh1, zero4);
          mma16816<true>(d, a, bl0, bl1, d);
          O[mb][0] = fma2(splat2(cv[2 * mb]), fma2(am, make_float2(d[0], d[1]), bzh), O[mb][0]);
          O[mb][1] = fma2(splat2(cv[2 * mb + 1]), fma2(am, make_float2(d[2], d[3]), bzh), O[mb][1]);
        }
      }
    }
    __syncwarp();
    if (issued < n_run) {
      // the stage's shared-memory reads by all lanes precede the async refill
      if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(issued++);
    }
  }
  if (stop >= 0) {
    // Drain: wait (bounded) for the copies this warp still has in flight.
    for (int i = stop + 1; i < issued; ++i)
      mbar_wait_bounded(&wbar[i % kStages], (uint32_t)(i / kStages) & 1u, kWaitLimit);
  }
  // after a fill, this grid ends only after the fill's quantize grid: work
  // later on the stream sees both complete
  if (FILL && threadIdx.x == 0) wait_prior_grid();

  // ---- merge the CTA's warps, write this split's partial
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    lrun[0] += __shfl_xor_sync(0xffffffffu, lrun[0], off);
    lrun[1] += __shfl_xor_sync(0xffffffffu, lrun[1], off);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();  // every warp is done with its stages and its tensor memory
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 32;" ::"r"(tmem_slot));
  float* mo = reinterpret_cast<float*>(smem);                  // [kDW][8 heads][128]
  float* ml = mo + kDW * 8 * kD;                               // [kDW][8][2]
#pragma unroll
  for (int mb = 0; mb < 8; ++mb)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int ch = 16 * g + 2 * mb + r;
      mo[(warp * 8 + 2 * t) * kD + ch] = O[mb][r].x;
      mo[(warp * 8 + 2 * t + 1) * kD + ch] = O[mb][r].y;
    }
  if (g == 0) {
    ml[(warp * 8 + 2 * t) * 2] = mrun[0], ml[(warp * 8 + 2 * t) * 2 + 1] = lrun[0];
    ml[(warp * 8 + 2 * t + 1) * 2] = mrun[1], ml[(warp * 8 + 2 * t + 1) * 2 + 1] = lrun[1];
  }
  __syncthreads();
  const int ch = threadIdx.x;  // kDW * 32 == 128 == kD
  for (int h = 0; h < 8; ++h) {  // head slot h: query head h % 4 of kv-head kvh + h / 4 when NH = 2
    const int hh = NH == 2 ? (h & 3) : h, hk = NH == 2 ? kvh + (h >> 2) : kvh;
    if (hh >= p.group) continue;
    const size_t pbase = (((size_t)b * p.num_kv_heads + hk) * p.splits + split) * 8 + hh;
    float mx = kNegBig;
#pragma unroll
    for (int w = 0; w < kDW; ++w) mx = fmaxf(mx, ml[(w * 8 + h) * 2]);
    float acc = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < kDW; ++w) {
      const float f = ex2(ml[(w * 8 + h) * 2] - mx);
      acc = fmaf(f, mo[(w * 8 + h) * kD + ch], acc);
      l = fmaf(f, ml[(w * 8 + h) * 2 + 1], l);
    }
    p.part_o[pbase * kD + ch] = acc;
    if (ch == 0) {
      p.part_ml[pbase * 2] = mx;
      p.part_ml[pbase * 2 + 1] = l;
    }
  }
}

// Merge the splits of one (sequence, kv-head) for up to four of its query
// heads, one warp each (blockIdx.y picks the group of four), rotate back and
// normalise.  Lane l holds channels 4l .. 4l+3: the rotation's channel bits
// 0 and 1 are in-register butterflies, bits 2..6 shuffles across the lanes.
// With a tail, its tokens join as one more partial: their scores q . k and
// their value sum are taken in the input basis (the rotation is orthogonal,
// so q~ . k~ = q . k), and the sum is added after the splits' sum is rotated
// back.  The kernel is launched as the decode grid's programmatic dependent:
// it scores the tail while that grid runs and waits for it before it reads
// the partials.
constexpr int kMaxTail = 128;
__global__ void __launch_bounds__(128) combine_d128_kernel(DecodeParams p) {
  const int pair = blockIdx.x;
  const int b = pair / p.num_kv_heads, kvh = pair % p.num_kv_heads;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * 4 + warp;  // query head of the kv-head's group
  if (h >= p.group) return;             // (the kernel has no block-wide barrier)
  int L = 0;
  if (p.k_tail) {
    L = p.tail_lens[b];
    if (L < 0 || L > p.tail_tokens || L > kMaxTail) {
      if (h == 0 && lane == 0) set_error(p.err, KVQ_DEVERR_BAD_SEQ);
      L = 0;
    }
  }
  float tm = kNegBig, tl = 0.f, tv[4] = {0.f, 0.f, 0.f, 0.f};  // tail: running max, sum, value sums
  if (L > 0) {
    auto elem = [&](uint16_t x) { return p.tail_f16 ? __half2float(__ushort_as_half(x)) : bf16_to_f(x); };
    const uint2 qw = *reinterpret_cast<const uint2*>(p.q + ((size_t)b * p.num_q_heads + (size_t)kvh * p.group + h) * kD +
                                                     4 * lane);
    const float q4[4] = {bf16_to_f((uint16_t)(qw.x & 0xFFFF)), bf16_to_f((uint16_t)(qw.x >> 16)),
                         bf16_to_f((uint16_t)(qw.y & 0xFFFF)), bf16_to_f((uint16_t)(qw.y >> 16))};
    const size_t row0 = ((size_t)p.layer * p.batch + b) * p.tail_tokens;
    // Eight tail tokens at a time: their rows are loaded together and their
    // eight dot products reduced side by side, so the load and shuffle
    // latencies are paid once per group.  Rows past L are not read (the
    // last valid row stands in) and take no weight.
    constexpr int kG = 8;
    for (int t0 = 0; t0 < L; t0 += kG) {
      uint2 kr[kG], vr[kG];
#pragma unroll
      for (int j = 0; j < kG; ++j) {
        const int t = min(t0 + j, L - 1);
        const size_t off = ((row0 + t) * p.num_kv_heads + kvh) * kD + 4 * lane;
        kr[j] = *reinterpret_cast<const uint2*>(p.k_tail + off);
        vr[j] = *reinterpret_cast<const uint2*>(p.v_tail + off);
      }
      float s[kG];
#pragma unroll
      for (int j = 0; j < kG; ++j) {
        float x = q4[0] * elem((uint16_t)(kr[j].x & 0xFFFF));
        x = fmaf(q4[1], elem((uint16_t)(kr[j].x >> 16)), x);
        x = fmaf(q4[2], elem((uint16_t)(kr[j].y & 0xFFFF)), x);
        s[j] = fmaf(q4[3], elem((uint16_t)(kr[j].y >> 16)), x);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int j = 0; j < kG; ++j) s[j] += __shfl_xor_sync(0xffffffffu, s[j], o);
      float cm = kNegBig;
#pragma unroll
      for (int j = 0; j < kG; ++j) {
        s[j] = t0 + j < L ? s[j] * p.scale_log2 : kNegBig;
        cm = fmaxf(cm, s[j]);
      }
      const float mn = fmaxf(tm, cm), al = ex2(tm - mn);
      tm = mn;
      tl *= al;
#pragma unroll
      for (int i = 0; i < 4; ++i) tv[i] *= al;
#pragma unroll
      for (int j = 0; j < kG; ++j) {
        const float e = t0 + j < L ? ex2(s[j] - mn) : 0.f;
        tl += e;
        tv[0] = fmaf(e, elem((uint16_t)(vr[j].x & 0xFFFF)), tv[0]);
        tv[1] = fmaf(e, elem((uint16_t)(vr[j].x >> 16)), tv[1]);
        tv[2] = fmaf(e, elem((uint16_t)(vr[j].y & 0xFFFF)), tv[2]);
        tv[3] = fmaf(e, elem((uint16_t)(vr[j].y >> 16)), tv[3]);
      }
    }
  }
  // the partials: written by the decode grid this one depends on
  wait_prior_grid();
  const float* pml = p.part_ml + ((size_t)pair * p.splits * 8 + h) * 2;       // split s at pml + 16 s
  const float* po = p.part_o + ((size_t)pair * p.splits * 8 + h) * kD + 4 * lane;  // split s at po + 8 kD s
  float mx = tm;
  for (int s = 0; s < p.splits; ++s) mx = fmaxf(mx, pml[16 * s]);
  float acc[4] = {0.f, 0.f, 0.f, 0.f}, l = 0.f;
  for (int s = 0; s < p.splits; ++s) {
    const float f = ex2(pml[16 * s] - mx);
    const float4 x = *reinterpret_cast<const float4*>(po + (size_t)8 * kD * s);
    acc[0] = fmaf(f, x.x, acc[0]), acc[1] = fmaf(f, x.y, acc[1]);
    acc[2] = fmaf(f, x.z, acc[2]), acc[3] = fmaf(f, x.w, acc[3]);
    l = fmaf(f, pml[16 * s + 1], l);
  }
  // H / sqrt(b) on each block of b = hblock channels
  if (p.hblock > 1) {
    const float a0 = acc[0] + acc[1], a1 = acc[0] - acc[1], a2 = acc[2] + acc[3], a3 = acc[2] - acc[3];
    acc[0] = a0, acc[1] = a1, acc[2] = a2, acc[3] = a3;
  }
  if (p.hblock > 2) {
    const float a0 = acc[0] + acc[2], a1 = acc[1] + acc[3], a2 = acc[0] - acc[2], a3 = acc[1] - acc[3];
    acc[0] = a0, acc[1] = a1, acc[2] = a2, acc[3] = a3;
  }
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    if (4 * off >= p.hblock) break;
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, acc[i], off);
      acc[i] = upper ? (o - acc[i]) : (acc[i] + o);
    }
  }
  const float sc = inv_sqrt_pow2(p.hblock);
  float o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] = acc[i] * sc;
  if (L > 0) {
    const float f = ex2(tm - mx);
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = fmaf(f, tv[i], o[i]);
    l = fmaf(f, tl, l);
  }
  const float il = l > 0.f ? 1.f / l : 0.f;
  *reinterpret_cast<float4*>(p.out + ((size_t)b * p.num_q_heads + (size_t)kvh * p.group + h) * kD + 4 * lane) =
      make_float4(o[0] * il, o[1] * il, o[2] * il, o[3] * il);
}

template <int BK, int BV, int NH, int M, int KPC, bool FILL>
int launch_fill(const DecodeParams& p, cudaStream_t s) {
  constexpr StageLayout SL = stage_layout(BK, BV, NH, M, KPC);
  constexpr int kStages = num_stages(NH);
  // stages, then one mbarrier per stage; the warp-merge buffer reuses the stage space
  static_assert(kDW * kStages * SL.bytes >= kDW * 8 * kD * 4 + kDW * 8 * 2 * 4, "merge buffer");
  const size_t smem = (size_t)kDW * kStages * SL.bytes + kDW * kStages * sizeof(uint64_t) +
                      ((size_t)p.tiles_per_split * sizeof(int32_t) + 15) / 16 * 16;
  auto kern = decode_d128_kernel<BK, BV, NH, M, KPC, FILL>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid(p.splits, p.batch * p.num_kv_heads / NH);
  if constexpr (FILL) {  // a programmatic dependent of the fill's quantize launch just before it
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kDW * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return (int)e;
  } else {
    kern<<<grid, kDW * 32, smem, s>>>(p);
  }
  {  // the combine: a programmatic dependent of the decode grid (its tail scoring overlaps that grid)
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(p.batch * p.num_kv_heads, (p.group + 3) / 4);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, combine_d128_kernel, p);
    if (e != cudaSuccess) return (int)e;
  }
  return (int)cudaGetLastError();
}
template <int BK, int BV, int NH, int M, int KPC>
int launch_bk_bv(const DecodeParams& p, cudaStream_t s) {
  return p.fill_page ? launch_fill<BK, BV, NH, M, KPC, true>(p, s) : launch_fill<BK, BV, NH, M, KPC, false>(p, s);
}

}  // namespace

int decode_kv_heads_per_cta(int group, int num_kv_heads) { return (group <= 4 && num_kv_heads % 2 == 0) ? 2 : 1; }

int launch_decode_d128(const DecodeParams& p, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int bk = p.k.bits, bv = p.v.bits;
  const bool pairs = decode_kv_heads_per_cta(p.group, p.num_kv_heads) == 2;
  if (p.k.per_channel) {  // the KIVI-style axes ablation: 2-, 4- and 8-bit codes (same widths for K and V)
#define KVQ_KPC(K)                                                                                            \
  if (bk == K && bv == K) {                                                                                   \
    if (p.k.meta16) return pairs ? launch_bk_bv<K, K, 2, 2, 1>(p, s) : launch_bk_bv<K, K, 1, 2, 1>(p, s); \
    return pairs ? launch_bk_bv<K, K, 2, 4, 1>(p, s) : launch_bk_bv<K, K, 1, 4, 1>(p, s);                 \
  }
    KVQ_KPC(2) KVQ_KPC(4) KVQ_KPC(8)
#undef KVQ_KPC
    return (int)cudaErrorInvalidValue;
  }
#define KVQ_CASE(K, V)                                                                              \
  if (bk == K && bv == V) {                                                                         \
    if (p.k.meta16) return pairs ? launch_bk_bv<K, V, 2, 2, 0>(p, s) : launch_bk_bv<K, V, 1, 2, 0>(p, s); \
    return pairs ? launch_bk_bv<K, V, 2, 4, 0>(p, s) : launch_bk_bv<K, V, 1, 4, 0>(p, s);                 \
  }
  KVQ_CASE(4, 4) KVQ_CASE(3, 4) KVQ_CASE(2, 4) KVQ_CASE(8, 4)
  KVQ_CASE(4, 2) KVQ_CASE(3, 2) KVQ_CASE(2, 2) KVQ_CASE(8, 2)
  KVQ_CASE(4, 8) KVQ_CASE(3, 8) KVQ_CASE(2, 8) KVQ_CASE(8, 8)
#undef KVQ_CASE
  return (int)cudaErrorInvalidValue;
}

}  // namespace kvq
