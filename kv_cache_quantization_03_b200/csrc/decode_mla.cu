// Decode attention over an MLA latent cache (sm_100a, tcgen05).
//
// KVarN project page (open-radar), Key Features, "MLA Model Support": the
// compressed latent of multi-head latent attention is quantised like a K/V
// tile.  One latent row c_t (512 channels, quantised, rotated domain) is both
// key and value; an unquantised bf16 rope key k_t (64 channels) adds to the
// score:  s_ht = scale * (rotate(q_h,lat) . c^_t + q_h,rope . k_t),
// o_h = rotate(sum_t softmax(s)_ht c^_t).
//
// All heads of a sequence (M = 128) share every tile, so both contractions
// run on the tensor cores with the tile dequantised once to f16 in shared
// memory: S = Q K^T (K = 576), out += P V.  128 x 512 fp32 output
// accumulators would fill all of an SM's tensor memory, so two CTAs share
// each (sequence, split): CTA r accumulates output channels [256r, 256r+256).
// Both compute the full scores and the same softmax, so no data moves
// between them.  The query's first 288 channels sit in tensor memory as the
// MMA's A operand, the other 288 in shared memory.
//
// Each CTA is a pipeline of three roles connected by mbarriers:
//   warp 21 (one thread)  bulk copies of the raw tiles into a ring of stages;
//   warp 20 (one thread)  the tcgen05 MMAs: S(c) into one of two TMEM score
//                         buffers, then O += P(c-1) V(c-1);
//   warps 4-19            dequantise a 32-token chunk, (a q + z) c in fp32,
//                         to f16 in the no-swizzle core-matrix operand layout
//                         (three buffers, two at 8 bits, so the dequantisation
//                         of chunk c+1 overlaps the MMAs of chunk c);
//   warps 0-3             one thread per head (a TMEM lane): online softmax
//                         with lazy rescaling of the TMEM output (only when
//                         the running max grows by more than 2^8), P in f16
//                         to tensor memory, where it is the A operand of P V.
// Every wait is bounded in time (1 s of global time); a wait that runs out
// raises KVQ_DEVERR_TIMEOUT and the remaining waits of that thread are
// skipped, so the kernel always terminates.
//
// mla_prep_q_kernel builds the rotated, pre-scaled f16 query of every
// sequence once: channels [0, 288) row-major (loaded into tensor memory by
// the softmax threads), channels [288, 576) in the shared-memory operand
// layout (one bulk copy).
#include <cuda_runtime.h>

#include "kvq_device.cuh"

namespace kvq {
namespace {

constexpr int kT = 16;
constexpr int kLat = 512, kRope = 64, kKf = kLat + kRope;  // 576: K extent of the scores
constexpr int kKT = 288;             // query channels [0, 288) in tensor memory
constexpr int kKS = kKf - kKT;       // query channels [288, 576) in shared memory
constexpr int kHalf = 256;           // output channels per CTA
constexpr int kH = 128;              // M: heads (rows beyond num_q_heads are zero)
constexpr int kChunk = 32;           // tokens per step (two tiles)
constexpr int kDqWarps = 16;
constexpr int kThreads = (4 + kDqWarps + 2) * 32;  // softmax 0-3, dequantisation 4-19, MMA 20, copies 21
constexpr int kMmaWarp = 4 + kDqWarps, kCopyWarp = kMmaWarp + 1;
constexpr float kNegBig = -1e30f;
// TMEM columns: O [0,256), S [256,320), Q [320,464), P [464,496)
constexpr uint32_t kTmemS = 256, kTmemQ = 320, kTmemP = 464;

// byte offsets in shared memory
constexpr int kSboQ = kKS / 8 * 128;         // 4608: next 8 rows of the shared query part
constexpr int kSboK = kKf / 8 * 128;         // 9216: next 8 rows of a dequantised chunk
constexpr int kQsBytes = kH * kKS * 2;       // 73728
constexpr int kQtBytes = kH * kKT * 2;       // 73728
constexpr int kKbBytes = kChunk * kKf * 2;   // 36864 per buffer
// prepared queries of one sequence: shared-memory part | tensor-memory part | per-head exponent (int)
constexpr int kQprepBytes = kQsBytes + kQtBytes + kH * 4;
constexpr int kOffQs = 0;
constexpr int kOffKb = kOffQs + kQsBytes;
__host__ __device__ constexpr int num_kb(int bits) { return bits == 8 ? 2 : 3; }  // dequantised chunk buffers
__host__ __device__ constexpr int st_offset(int bits) { return kOffKb + num_kb(bits) * kKbBytes; }
// a stage holds two tiles: codes | (a, z) | channel scales | rope; m bytes per
// a, z or c (4: float32, 2: half)
__host__ __device__ constexpr int tile_code_bytes(int bits) { return kT * kLat * bits / 8; }
__host__ __device__ constexpr int stage_bytes(int bits, int m) {
  return 2 * (tile_code_bytes(bits) + kT * 2 * m + kLat * m + kT * kRope * 2);
}
constexpr int kNS = 2;  // raw-tile stages
__host__ __device__ constexpr int bar_offset(int bits, int m) { return st_offset(bits) + kNS * stage_bytes(bits, m); }
// full[2] dq[3] sfull[2] pfull[2] pv[4] qf qt fin, the TMEM address, the operand
// exponents of the dequantised chunk buffers (int[4]), then the tile-validity bits
constexpr int kNumBars = kNS + 3 + 2 + 2 + 4 + 3;
__host__ __device__ constexpr int echunk_offset(int bits, int m) { return bar_offset(bits, m) + kNumBars * 8 + 8; }
__host__ __device__ constexpr int vmask_offset(int bits, int m) { return echunk_offset(bits, m) + 16; }
__host__ __device__ constexpr int smem_bytes(int bits, int m, int tiles_per_split) {
  return vmask_offset(bits, m) + ((tiles_per_split + 31) / 32) * 4;
}
static_assert(smem_bytes(4, 4, 8192) <= 232448 && smem_bytes(8, 4, 8192) <= 232448, "shared memory");

// (a, z) of a stage's token and c of eight channels (M = 4: float32, 2: half)
template <int M>
__device__ __forceinline__ float2 mla_az(const uint8_t* base) {
  if constexpr (M == 4) return *reinterpret_cast<const float2*>(base);
  else return __half22float2(*reinterpret_cast<const __half2*>(base));
}
template <int M>
__device__ __forceinline__ void mla_c8(const uint8_t* base, f2 (&cc)[4]) {
  if constexpr (M == 4) {
    const float4 c0 = reinterpret_cast<const float4*>(base)[0], c1 = reinterpret_cast<const float4*>(base)[1];
    cc[0] = make_float2(c0.x, c0.y), cc[1] = make_float2(c0.z, c0.w);
    cc[2] = make_float2(c1.x, c1.y), cc[3] = make_float2(c1.z, c1.w);
  } else {
    const uint4 h = *reinterpret_cast<const uint4*>(base);
    const uint32_t w[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) cc[e] = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
  }
}

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}
// No-swizzle core-matrix layout offset of element (row, k): 8 x 8 blocks of
// 16-bit elements (128 B, one row of 16 B per row), k-blocks 128 B apart,
// row-blocks `sbo` bytes apart.
__host__ __device__ __forceinline__ uint32_t cm_off(int row, int k, int sbo) {
  return (row >> 3) * sbo + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}
__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile("{.reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;}" ::"r"(
                   tmem_d),
               "l"(da), "l"(db), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive_local(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ float bf16f(uint32_t b) { return __uint_as_float(b << 16); }

// Eight consecutive codes (latent channels ch0 .. ch0 + 7) of tile row `tr`,
// as floats.  Layout of a tile's codes: row-major, lowest channel in the
// lowest bits; 3 bits as a plane of the low 2 bits of all rows followed by a
// plane of the high bits.
template <int BITS>
__device__ __forceinline__ void codes8(const uint8_t* codes, int tr, int ch0, float (&q)[8]) {
  uint32_t c[8];
  if constexpr (BITS == 4) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(codes + tr * 256 + ch0 / 2);
#pragma unroll
    for (int e = 0; e < 8; ++e) c[e] = (w >> (4 * e)) & 15u;
  } else if constexpr (BITS == 8) {
    const uint2 w = *reinterpret_cast<const uint2*>(codes + tr * 512 + ch0);
#pragma unroll
    for (int e = 0; e < 4; ++e) c[e] = (w.x >> (8 * e)) & 255u, c[e + 4] = (w.y >> (8 * e)) & 255u;
  } else if constexpr (BITS == 2) {
    const uint32_t w = *reinterpret_cast<const uint16_t*>(codes + tr * 128 + ch0 / 4);
#pragma unroll
    for (int e = 0; e < 8; ++e) c[e] = (w >> (2 * e)) & 3u;
  } else {  // 3 bits
    const uint32_t lo = *reinterpret_cast<const uint16_t*>(codes + tr * 128 + ch0 / 4);
    const uint32_t hi = codes[kT * 128 + tr * 64 + ch0 / 8];
#pragma unroll
    for (int e = 0; e < 8; ++e) c[e] = ((lo >> (2 * e)) & 3u) | (((hi >> e) & 1u) << 2);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) q[e] = __uint_as_float(0x4B000000u | c[e]) - 8388608.0f;  // exact small integers
}


__device__ __forceinline__ void umma_f16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc,
                                                uint32_t acc) {
  asm volatile("{.reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;}" ::"r"(
                   tmem_d),
               "r"(tmem_a), "l"(db), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]));
}

template <int BITS, int M>
__global__ void __launch_bounds__(kThreads, 1) decode_mla_kernel(MlaDecodeParams p) {
  constexpr int NS = kNS, NB = num_kb(BITS), SB = stage_bytes(BITS, M), CB = tile_code_bytes(BITS);
  constexpr int kOffSt = st_offset(BITS);
  constexpr int kStAz = 2 * CB, kStC = kStAz + 2 * kT * 2 * M, kStRope = kStC + 2 * kLat * M;
  extern __shared__ __align__(1024) uint8_t smem[];
  // the combine kernel (this grid's programmatic dependent) may start now: it
  // scores the unquantised tails, then waits for this grid's partials
  asm volatile("griddepcontrol.launch_dependents;");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x & 1, split = blockIdx.x >> 1, b = blockIdx.y;  // r: output half
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + bar_offset(BITS, M));
  uint64_t* dq = full + kNS;
  uint64_t* sfull = dq + 3;
  uint64_t* pfull = sfull + 2;
  uint64_t* pv = pfull + 2;
  uint64_t* qf = pv + 4;
  uint64_t* qt = qf + 1;
  uint64_t* fin = qt + 1;  // every MMA of the CTA has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint32_t* vmask = reinterpret_cast<uint32_t*>(smem + vmask_offset(BITS, M));
  int* echunk = reinterpret_cast<int*>(smem + echunk_offset(BITS, M));  // [NB]: operand exponent of each buffer
  const uint32_t s_base = smem_u32(smem);

  const int seq_raw = p.seq_lens[b];
  int ntiles = seq_raw < 0 ? 0 : seq_raw / kT;
  if (ntiles > p.max_pages) ntiles = p.max_pages;
  if (split == 0 && r == 0 && tid == 0) {
    if (seq_raw < 0 || seq_raw / kT > p.max_pages) set_error(p.err, KVQ_DEVERR_BAD_SEQ);
    if (seq_raw % kT) set_error(p.err, KVQ_DEVERR_PARTIAL_TILE);
  }
  const int t0 = split * p.tiles_per_split;
  const int t1 = min(t0 + p.tiles_per_split, ntiles);
  const int ntl = t1 > t0 ? t1 - t0 : 0;
  const int nchunks = (ntl + 1) / 2;
  const int32_t* btab = p.block_table + (size_t)b * p.max_pages + t0;
  const uint8_t* qprep = p.qprep + (size_t)b * kQprepBytes;

  // which tiles of the split have a valid page (bit lt of vmask)
  for (int i = tid; i < (ntl + 31) / 32; i += kThreads) vmask[i] = 0u;
  __syncthreads();
  for (int lt = tid; lt < ntl; lt += kThreads) {
    const int pg = btab[lt];
    if (pg >= 0 && pg < p.num_pages) atomicOr(&vmask[lt >> 5], 1u << (lt & 31));
    else if (r == 0) set_error(p.err, KVQ_DEVERR_BAD_PAGE);
  }
  auto tile_ok = [&](int lt) { return lt < ntl && ((vmask[lt >> 5] >> (lt & 31)) & 1u); };

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < NS; ++i) mbar_init(&full[i], 1);
#pragma unroll
    for (int i = 0; i < NB; ++i) mbar_init(&dq[i], kDqWarps * 32);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], kH);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) mbar_init(&pv[i], 1);
    mbar_init(qf, 1);
    mbar_init(qt, kH);
    mbar_init(fin, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == kCopyWarp) {
    // ---------------------------------------------------------------- bulk copies (one thread)
    if (lane == 0) {
      mbar_arrive_expect_tx(qf, kQsBytes);
      bulk_g2s(smem + kOffQs, qprep, kQsBytes, qf);
      // page ids of chunk c (two tiles); the loop loads them one chunk ahead
      auto pages_of = [&](int c, int (&pg)[2]) {
#pragma unroll
        for (int j = 0; j < 2; ++j) pg[j] = 2 * c + j < ntl ? btab[2 * c + j] : -1;
      };
      auto issue = [&](int c, const int (&pg)[2]) {  // raw chunk c into stage c % NS
        uint64_t* bar = &full[c % NS];
        uint8_t* st = smem + kOffSt + (c % NS) * SB;
        uint32_t bytes = 0;
#pragma unroll
        for (int j = 0; j < 2; ++j)
          if (tile_ok(2 * c + j)) bytes += CB + kT * 2 * M + kLat * M + kT * kRope * 2;
        mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (!tile_ok(2 * c + j)) continue;
          const size_t slot = (size_t)p.layer * p.num_pages + pg[j];
          bulk_g2s(st + j * CB, p.codes + slot * CB, CB, bar);
          bulk_g2s(st + kStAz + j * kT * 2 * M, static_cast<const uint8_t*>(p.tok) + slot * (kT * 2 * M), kT * 2 * M,
                   bar);
          bulk_g2s(st + kStC + j * kLat * M, static_cast<const uint8_t*>(p.chan) + slot * (kLat * M), kLat * M, bar);
          bulk_g2s(st + kStRope + j * kT * kRope * 2, p.rope + slot * kT * kRope, kT * kRope * 2, bar);
        }
      };
      const int pre = nchunks < NS ? nchunks : NS;
      for (int c = 0; c < pre; ++c) {
        int pg[2];
        pages_of(c, pg);
        issue(c, pg);
      }
      int pg_next[2];
      pages_of(NS, pg_next);
      for (int c = 0; c + NS < nchunks; ++c) {
        // chunk c is dequantised: its stage is free again
        ok &= mbar_wait_bounded(&dq[c % NB], (uint32_t)(c / NB) & 1u, ok ? kWaitLimit : 0u);
        proxy_fence();
        issue(c + NS, pg_next);
        pages_of(c + NS + 1, pg_next);  // in flight until the next chunk
      }
      // No bulk copy may still be writing when the CTA exits: every chunk is
      // issued (also after a timeout), and only the last NS can be in flight.
      // These waits take the full limit even after an earlier wait gave up.
      ok &= mbar_wait_bounded(qf, 0u, kWaitLimit);
      for (int c = nchunks > NS ? nchunks - NS : 0; c < nchunks; ++c)
        ok &= mbar_wait_bounded(&full[c % NS], (uint32_t)(c / NS) & 1u, kWaitLimit);
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA (one thread)
    if (lane == 0) {
      const uint32_t idesc_s = (1u << 4) | ((uint32_t)(kChunk >> 3) << 17) | ((uint32_t)(kH >> 4) << 24);
      const uint32_t idesc_pv = (1u << 4) | (1u << 16) | ((uint32_t)(kHalf >> 3) << 17) | ((uint32_t)(kH >> 4) << 24);
      const uint64_t dq0 = umma_desc(s_base + kOffQs, 128, kSboQ), dk0 = umma_desc(s_base + kOffKb, 128, kSboK);
      const uint64_t dv0 = umma_desc(s_base + kOffKb + r * (kHalf / 8) * 128, kSboK, 128);
      ok &= mbar_wait_bounded(qf, 0u, kWaitLimit);
      ok &= mbar_wait_bounded(qt, 0u, ok ? kWaitLimit : 0u);
      for (int c = 0; c <= nchunks; ++c) {
        if (c < nchunks) {
          ok &= mbar_wait_bounded(&dq[c % NB], (uint32_t)(c / NB) & 1u, ok ? kWaitLimit : 0u);
          tc_fence_after();
          // descriptors advance by 256 B (16 in the address field) per 16-channel step
          const uint64_t dk = dk0 + (uint64_t)((c % NB) * (kKbBytes >> 4));
          const uint32_t d = tmem + kTmemS + 32 * (c & 1);
#pragma unroll
          for (int s = 0; s < kKT / 16; ++s)  // query channels [0, 288) from tensor memory
            umma_f16_tmem_a(d, tmem + kTmemQ + 8 * s, dk + 16 * s, idesc_s, s > 0);
#pragma unroll
          for (int s = 0; s < kKS / 16; ++s)  // [288, 576) from shared memory
            umma_f16(d, dq0 + 16 * s, dk + (kKT / 8) * 8 + 16 * s, idesc_s, 1u);
          umma_commit(&sfull[c & 1]);
        }
        if (c >= 1) {
          const int x = c - 1;
          ok &= mbar_wait_bounded(&pfull[x & 1], (uint32_t)(x >> 1) & 1u, ok ? kWaitLimit : 0u);
          tc_fence_after();
          const uint64_t dv = dv0 + (uint64_t)((x % NB) * (kKbBytes >> 4));
#pragma unroll
          for (int s = 0; s < kChunk / 16; ++s)  // A = P(x) in tensor memory
            umma_f16_tmem_a(tmem, tmem + kTmemP + 16 * (x & 1) + 8 * s, dv + s * 2 * (kSboK >> 4), idesc_pv,
                            (x > 0 || s > 0) ? 1u : 0u);
          umma_commit(&pv[x & 3]);
        }
      }
      // every MMA issued above has completed before tensor memory is freed
      // (full limit, also after a timeout)
      umma_commit(fin);
      ok &= mbar_wait_bounded(fin, 0u, kWaitLimit);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- dequantisation
    // Warp dw covers tile j = dw / 8, latent channels 256 gh + 8 lane .. + 7
    // (gh = (dw / 4) % 2) of the tile rows 8 rh + ((lane + it + 4 hf) % 8),
    // it = 0..3 (rh = (dw / 2) % 2, hf = dw % 2): code loads and operand
    // stores are free of bank conflicts.  Warps 0..7 then convert 8 rope
    // channels of one row each, spread the same way.
    const int dw = warp - 4, j = dw >> 3, gh = (dw >> 2) & 1, rh = (dw >> 1) & 1, hf = dw & 1;
    const int ch0 = kHalf * gh + 8 * lane;
    const int ri = lane & 7, rP = (lane >> 3) + 4 * ((dw >> 2) & 1);
    const int rrow = 8 * (dw & 3) + ((ri + rP) & 7), rgrp = ri;  // rope (dw < 8): chunk row, 8-channel group
    for (int c = 0; c < nchunks; ++c) {
      ok &= mbar_wait_bounded(&full[c % NS], (uint32_t)(c / NS) & 1u, ok ? kWaitLimit : 0u);
      if (c >= NB)  // PV(c - NB) has read this operand buffer
        ok &= mbar_wait_bounded(&pv[(c - NB) & 3], (uint32_t)((c - NB) >> 2) & 1u, ok ? kWaitLimit : 0u);
      const uint8_t* st = smem + kOffSt + (c % NS) * SB;
      uint8_t* kb = smem + kOffKb + (c % NB) * kKbBytes;
      const bool valid = tile_ok(2 * c + j);
      // Operand scale of the chunk: the stored c is at most 1, so a row's
      // dequantised latent is bounded by max(|z|, |a (2^b - 1) + z|).  The
      // exact power of two 2^-e (e >= 0) that keeps the chunk's bound below
      // 2^14 multiplies the latent and the rope keys, so the f16 operands
      // cannot overflow; the softmax multiplies the chunk's scores by 2^e
      // and weighs its values by it.  Every warp computes e from lane l's
      // token (tile l / 16, row l % 16).
      int e_chunk;
      {
        const float2 az = mla_az<M>(st + kStAz + (lane >> 4) * kT * 2 * M + (lane & 15) * 2 * M);
        constexpr float kQm = (float)((1 << BITS) - 1);
        float bnd = tile_ok(2 * c + (lane >> 4)) ? fmaxf(fabsf(az.y), fabsf(fmaf(az.x, kQm, az.y))) : 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) bnd = fmaxf(bnd, __shfl_xor_sync(0xffffffffu, bnd, off));
        e_chunk = max(0, (int)(__float_as_uint(bnd) >> 23) - 140);  // bnd < 2^(E - 126): 2^-e bnd < 2^14
        if (dw == 0 && lane == 0) echunk[c % NB] = e_chunk;             // published by the dq arrive below
      }
      const float sE = __uint_as_float((uint32_t)(127 - e_chunk) << 23);
      f2 cc[4];
      mla_c8<M>(st + kStC + j * kLat * M + ch0 * M, cc);
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int tr = 8 * rh + ((lane + it + 4 * hf) & 7);
        float2 az = mla_az<M>(st + kStAz + j * kT * 2 * M + tr * 2 * M);
        az.x *= sE, az.y *= sE;
        float q[8];
        codes8<BITS>(st + j * CB, tr, ch0, q);
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const f2 v = mul2(fma2(splat2(az.x), make_float2(q[2 * e], q[2 * e + 1]), splat2(az.y)), cc[e]);
          pk[e] = valid ? pack_f16x2(v.x, v.y) : 0u;
        }
        *reinterpret_cast<uint4*>(kb + cm_off(16 * j + tr, ch0, kSboK)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      if (dw < 8) {
        const int jj = rrow >> 4;
        const bool v2 = tile_ok(2 * c + jj);
        const uint4 w4 = *reinterpret_cast<const uint4*>(st + kStRope + jj * kT * kRope * 2 + (rrow & 15) * kRope * 2 +
                                                         rgrp * 16);
        const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) pk[e] = v2 ? pack_f16x2(bf16f(w[e] & 0xFFFFu) * sE, bf16f(w[e] >> 16) * sE) : 0u;
        *reinterpret_cast<uint4*>(kb + cm_off(rrow, kLat + 8 * rgrp, kSboK)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      proxy_fence();
      mbar_arrive_local(&dq[c % NB]);
    }
  } else {
    // ---------------------------------------------------------------- softmax, one thread per head
    const int h = tid;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    {  // query channels [0, 288) of head h into tensor memory: f16 pairs, lane h
      const uint4* src = reinterpret_cast<const uint4*>(qprep + kQsBytes + (size_t)h * kKT * 2);
#pragma unroll 1
      for (int k = 0; k < kKT / 32; ++k) {
        uint32_t v[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 x = src[4 * k + i];
          v[4 * i] = x.x, v[4 * i + 1] = x.y, v[4 * i + 2] = x.z, v[4 * i + 3] = x.w;
        }
        tmem_st16(tmem + lane_base + kTmemQ + 16 * k, v);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive_local(qt);
    }
    // the head's query was prepared times 2^-eq (see mla_prep_q_kernel)
    const float s_q = __uint_as_float((uint32_t)(127 + reinterpret_cast<const int*>(qprep + kQsBytes + kQtBytes)[h])
                                      << 23);
    float m_run = kNegBig, l_run = 0.f;
    int e_ref = 0;  // the output accumulator holds sum p v 2^-e_ref (e_ref: largest chunk exponent so far)
    for (int x = 0; x < nchunks; ++x) {
      ok &= mbar_wait_bounded(&sfull[x & 1], (uint32_t)(x >> 1) & 1u, ok ? kWaitLimit : 0u);
      // the chunk's operand exponent (its dequantisation is complete: the scores are)
      ok &= mbar_wait_bounded(&dq[x % NB], (uint32_t)(x / NB) & 1u, ok ? kWaitLimit : 0u);
      const int ex = echunk[x % NB];
      tc_fence_after();
      float sc[32];
      tmem_ld32(tmem + lane_base + kTmemS + 32 * (x & 1), sc);
      const bool tv[2] = {tile_ok(2 * x), tile_ok(2 * x + 1)};
      // 2^ex 2^eq: the chunk's and the query's operand scales, undone
      const float s_up = __uint_as_float((uint32_t)(127 + ex) << 23) * s_q;
      float mx = kNegBig;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        sc[i] = tv[i >> 4] ? sc[i] * s_up : kNegBig;
        mx = fmaxf(mx, sc[i]);
      }
      // lazy rescale; the TMEM accesses are warp-wide, so the whole warp
      // joins (factor 1 where a head's max did not grow).  A chunk with a
      // larger operand exponent rescales the accumulator too (chunk-uniform).
      const bool grow = mx > m_run + 8.f;
      const float alpha = grow ? ex2f(m_run - mx) : 1.f;
      const bool egrow = ex > e_ref;
      const float alpha_o = egrow ? alpha * __uint_as_float((uint32_t)(127 + e_ref - ex) << 23) : alpha;
      if (egrow) e_ref = ex;
      if (__any_sync(0xffffffffu, (grow || egrow) && x > 0)) {
        ok &= mbar_wait_bounded(&pv[(x - 1) & 3], (uint32_t)((x - 1) >> 2) & 1u, ok ? kWaitLimit : 0u);
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < kHalf; c0 += 32) {
          float o[32];
          tmem_ld32(tmem + lane_base + c0, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha_o;
          tmem_st32(tmem + lane_base + c0, o);
        }
      }
      if (grow) {
        l_run *= alpha;
        m_run = mx;
      }
      if (x >= 2)  // PV(x - 2) has read P buffer x & 1
        ok &= mbar_wait_bounded(&pv[(x - 2) & 3], (uint32_t)((x - 2) >> 2) & 1u, ok ? kWaitLimit : 0u);
      uint32_t pk[16];
      float ls = 0.f;
      // weights of this chunk's (scaled) values: p 2^(ex - e_ref), ex <= e_ref
      const float wsc = ex - e_ref >= -126 ? __uint_as_float((uint32_t)(127 + ex - e_ref) << 23) : 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float p0 = tv[i >> 3] ? ex2f(sc[2 * i] - m_run) : 0.f;
        const float p1 = tv[i >> 3] ? ex2f(sc[2 * i + 1] - m_run) : 0.f;
        ls += p0 + p1;
        pk[i] = pack_f16x2(p0 * wsc, p1 * wsc);
      }
      l_run += ls;
      tmem_st16(tmem + lane_base + kTmemP + 16 * (x & 1), pk);
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive_local(&pfull[x & 1]);
    }
    // ---- epilogue: this split's partial output half, (max, sum) per head
    float* po = p.part_o + (((size_t)b * p.splits + split) * kH + h) * kLat + r * kHalf;
    if (nchunks > 0) {
      const int x = nchunks - 1;
      ok &= mbar_wait_bounded(&pv[x & 3], (uint32_t)(x >> 2) & 1u, ok ? kWaitLimit : 0u);
      tc_fence_after();
      const float s_out = __uint_as_float((uint32_t)(127 + e_ref) << 23);  // 2^e_ref
      for (int c0 = 0; c0 < kHalf; c0 += 32) {
        float o[32];
        tmem_ld32(tmem + lane_base + c0, o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= s_out;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float4*>(po + c0 + 4 * i) = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
      }
    } else {
      for (int c0 = 0; c0 < kHalf; c0 += 4) *reinterpret_cast<float4*>(po + c0) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (r == 0) {
      float* pm = p.part_ml + (((size_t)b * p.splits + split) * kH + h) * 2;
      pm[0] = m_run;
      pm[1] = l_run;
    }
  }
  if (!ok) set_error(p.err, KVQ_DEVERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
}

// Rotated, pre-scaled f16 queries of one sequence: element k of head h is
// (H_512 q_lat)[k] * scale * log2(e) / sqrt(512) for k < 512 and
// q_rope[k - 512] * scale * log2(e) after, both times 2^-eq_h; k in
// [0, 288) row-major, k in [288, 576) in the shared-memory operand layout,
// then eq_h (int) per head.  eq_h is the power of two that brings the
// head's largest element into [2^7, 2^8): queries of any magnitude keep
// f16's relative precision, and the softmax multiplies the head's scores by
// 2^eq_h.  One warp per head: lane l keeps latent elements 16l..16l+15;
// index bits 0..3 are butterflies in registers, bits 4..8 shuffles.
__global__ void __launch_bounds__(256) mla_prep_q_kernel(MlaDecodeParams p) {
  const int b = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* out_s = p.qprep + (size_t)b * kQprepBytes;
  uint8_t* out_t = out_s + kQsBytes;
  int* out_e = reinterpret_cast<int*>(out_t + kQtBytes);
  const float f0 = p.scale_log2 * 0.044194173824159216f;  // 1 / sqrt(512)
  for (int h = warp; h < kH; h += 8) {
    float v[16];
    const bool live = h < p.num_q_heads;
    const uint16_t* qh = p.q + ((size_t)b * p.num_q_heads + (live ? h : 0)) * kKf;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint4 x = *reinterpret_cast<const uint4*>(qh + 16 * lane + 8 * k);
      const uint32_t a[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[8 * k + 2 * e] = live ? bf16f(a[e] & 0xFFFFu) : 0.f;
        v[8 * k + 2 * e + 1] = live ? bf16f(a[e] >> 16) : 0.f;
      }
    }
#pragma unroll
    for (int s = 1; s < 16; s <<= 1)
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (!(i & s)) {
          const float x = v[i], y = v[i + s];
          v[i] = x + y;
          v[i + s] = x - y;
        }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, v[i], off);
        v[i] = upper ? (o - v[i]) : (v[i] + o);
      }
    }
    // the head's rope elements (lanes 0..7, eight each) and its exponent
    float rp[8];
    {
      const uint4 x = lane < kRope / 8 ? *reinterpret_cast<const uint4*>(qh + kLat + 8 * lane) : make_uint4(0, 0, 0, 0);
      const uint32_t a[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        rp[2 * e] = live ? bf16f(a[e] & 0xFFFFu) * p.scale_log2 : 0.f;
        rp[2 * e + 1] = live ? bf16f(a[e] >> 16) * p.scale_log2 : 0.f;
      }
    }
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fabsf(v[i] * f0));
#pragma unroll
    for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(rp[i]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    // mx in [2^(E-127), 2^(E-126)): eq = E - 134 puts it in [2^7, 2^8)
    const int eq = mx > 0.f ? min(max((int)(__float_as_uint(mx) >> 23) - 134, -126), 126) : 0;
    const float down = __uint_as_float((uint32_t)(127 - eq) << 23);  // 2^-eq, eq in [-126, 126]
    const float f = f0 * down;
    if (lane == 0) out_e[h] = eq;
    uint4 w[2];
#pragma unroll
    for (int k = 0; k < 2; ++k)
      w[k] = make_uint4(pack_f16x2(v[8 * k] * f, v[8 * k + 1] * f), pack_f16x2(v[8 * k + 2] * f, v[8 * k + 3] * f),
                        pack_f16x2(v[8 * k + 4] * f, v[8 * k + 5] * f), pack_f16x2(v[8 * k + 6] * f, v[8 * k + 7] * f));
    const int k0 = 16 * lane;
    if (k0 < kKT) {
      *reinterpret_cast<uint4*>(out_t + (size_t)(h * kKT + k0) * 2) = w[0];
      *reinterpret_cast<uint4*>(out_t + (size_t)(h * kKT + k0 + 8) * 2) = w[1];
    } else {
      *reinterpret_cast<uint4*>(out_s + cm_off(h, k0 - kKT, kSboQ)) = w[0];
      *reinterpret_cast<uint4*>(out_s + cm_off(h, k0 + 8 - kKT, kSboQ)) = w[1];
    }
    if (lane < kRope / 8) {
      uint32_t pk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) pk[e] = pack_f16x2(rp[2 * e] * down, rp[2 * e + 1] * down);
      *reinterpret_cast<uint4*>(out_s + cm_off(h, kLat - kKT + 8 * lane, kSboQ)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
}

// Merge the splits of one (sequence, head), rotate back with H_512,
// normalise: one warp per (sequence, head), four per CTA.  Lane l holds
// channels 16l .. 16l+15: the rotation's channel bits 0..3 are in-register
// butterflies, bits 4..8 shuffles across the lanes.  With a tail, its tokens
// join as one more partial: their scores q_lat . latent + q_rope . rope and
// their latent sum are taken in the input basis (the rotation is
// orthogonal), and the sum is added after the splits' sum has been rotated
// back.  Launched as the decode grid's programmatic dependent, it scores the
// tail while that grid runs and waits for it before it reads the partials.
constexpr int kMlaMaxTail = 16;
__device__ __forceinline__ void unpack8(uint4 w, bool f16, float* x) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if (f16) {
      const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&ws[e]));
      x[2 * e] = v.x, x[2 * e + 1] = v.y;
    } else {
      x[2 * e] = bf16f(ws[e] & 0xFFFFu), x[2 * e + 1] = bf16f(ws[e] >> 16);
    }
  }
}
__global__ void __launch_bounds__(128) combine_mla_kernel(MlaDecodeParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * 4 + warp;          // (sequence, head) of this warp
  if (gw >= p.batch * p.num_q_heads) return;     // (the kernel has no block-wide barrier)
  const int b = gw / p.num_q_heads, h = gw % p.num_q_heads;
  int L = 0;
  if (p.lat_tail) {
    L = p.tail_lens[b];
    if (L < 0 || L > p.tail_tokens || L > kMlaMaxTail) {
      if (h == 0 && lane == 0) set_error(p.err, KVQ_DEVERR_BAD_SEQ);
      L = 0;
    }
  }
  float tm = kNegBig, tl = 0.f, tv[16];  // tail: max, sum, value sums of this lane's channels
#pragma unroll
  for (int i = 0; i < 16; ++i) tv[i] = 0.f;
  if (L > 0) {
    const uint16_t* qh = p.q + ((size_t)b * p.num_q_heads + h) * kKf;
    float ql[16], x[16];
    unpack8(reinterpret_cast<const uint4*>(qh + 16 * lane)[0], false, ql);
    unpack8(reinterpret_cast<const uint4*>(qh + 16 * lane)[1], false, ql + 8);
    const uint32_t qrw = *reinterpret_cast<const uint32_t*>(qh + kLat + 2 * lane);
    const float qr0 = bf16f(qrw & 0xFFFFu), qr1 = bf16f(qrw >> 16);
    const size_t row0 = ((size_t)p.layer * p.batch + b) * p.tail_tokens;
    const bool f16 = p.tail_f16 != 0;
    auto lat_row = [&](int t, float* v) {
      const uint4* r = reinterpret_cast<const uint4*>(p.lat_tail + (row0 + t) * kLat + 16 * lane);
      unpack8(r[0], f16, v);
      unpack8(r[1], f16, v + 8);
    };
    float sc[kMlaMaxTail];
#pragma unroll
    for (int t = 0; t < kMlaMaxTail; ++t) {
      float a = 0.f;
      if (t < L) {
        lat_row(t, x);
#pragma unroll
        for (int i = 0; i < 16; ++i) a = fmaf(ql[i], x[i], a);
        const uint32_t rw = *reinterpret_cast<const uint32_t*>(p.rope_tail + (row0 + t) * kRope + 2 * lane);
        a = fmaf(qr0, bf16f(rw & 0xFFFFu), a);
        a = fmaf(qr1, bf16f(rw >> 16), a);
      }
      sc[t] = a;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int t = 0; t < kMlaMaxTail; ++t) sc[t] += __shfl_xor_sync(0xffffffffu, sc[t], off);
#pragma unroll
    for (int t = 0; t < kMlaMaxTail; ++t) {
      sc[t] = t < L ? sc[t] * p.scale_log2 : kNegBig;
      tm = fmaxf(tm, sc[t]);
    }
#pragma unroll
    for (int t = 0; t < kMlaMaxTail; ++t) {
      if (t < L) {
        const float e = ex2f(sc[t] - tm);
        tl += e;
        lat_row(t, x);
#pragma unroll
        for (int i = 0; i < 16; ++i) tv[i] = fmaf(e, x[i], tv[i]);
      }
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the decode grid's partials
  float mx = tm;
  for (int s = 0; s < p.splits; ++s) mx = fmaxf(mx, p.part_ml[(((size_t)b * p.splits + s) * kH + h) * 2]);
  float acc[16], l = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int s = 0; s < p.splits; ++s) {
    const size_t i = ((size_t)b * p.splits + s) * kH + h;
    const float f = ex2f(p.part_ml[i * 2] - mx);
    const float4* po = reinterpret_cast<const float4*>(p.part_o + i * kLat + 16 * lane);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 v = po[k];
      acc[4 * k] = fmaf(f, v.x, acc[4 * k]), acc[4 * k + 1] = fmaf(f, v.y, acc[4 * k + 1]);
      acc[4 * k + 2] = fmaf(f, v.z, acc[4 * k + 2]), acc[4 * k + 3] = fmaf(f, v.w, acc[4 * k + 3]);
    }
    l = fmaf(f, p.part_ml[i * 2 + 1], l);
  }
  // H_512: channel bits 0..3 within the lane, bits 4..8 across lanes 1, 2, 4, 8, 16
#pragma unroll
  for (int st = 1; st < 16; st <<= 1)
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (!(i & st)) {
        const float u = acc[i], v = acc[i + st];
        acc[i] = u + v;
        acc[i + st] = u - v;
      }
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, acc[i], off);
      acc[i] = upper ? (o - acc[i]) : (acc[i] + o);
    }
  }
  float o[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i] = acc[i] * 0.044194173824159216f;  // 1/sqrt(512)
  if (L > 0) {
    const float f = ex2f(tm - mx);
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = fmaf(f, tv[i], o[i]);
    l = fmaf(f, tl, l);
  }
  const float il = l > 0.f ? 1.f / l : 0.f;
  float4* out = reinterpret_cast<float4*>(p.out + ((size_t)b * p.num_q_heads + h) * kLat + 16 * lane);
#pragma unroll
  for (int k = 0; k < 4; ++k) out[k] = make_float4(o[4 * k] * il, o[4 * k + 1] * il, o[4 * k + 2] * il, o[4 * k + 3] * il);
}

template <int BITS, int M>
int launch_mla_bits(const MlaDecodeParams& p, cudaStream_t s) {
  const int smem = smem_bytes(BITS, M, p.tiles_per_split);
  cudaError_t e = cudaFuncSetAttribute(decode_mla_kernel<BITS, M>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * p.splits, p.batch, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  return (int)cudaLaunchKernelEx(&cfg, decode_mla_kernel<BITS, M>, p);
}

}  // namespace

size_t mla_qprep_bytes(int64_t batch) { return (size_t)batch * kQprepBytes; }

int launch_decode_mla(const MlaDecodeParams& p, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  mla_prep_q_kernel<<<p.batch, 256, 0, s>>>(p);
  int e = (int)cudaGetLastError();
  if (e != cudaSuccess) return e;
  const bool h = p.meta16 != 0;
  switch (p.bits) {
    case 2: e = h ? launch_mla_bits<2, 2>(p, s) : launch_mla_bits<2, 4>(p, s); break;
    case 3: e = h ? launch_mla_bits<3, 2>(p, s) : launch_mla_bits<3, 4>(p, s); break;
    case 4: e = h ? launch_mla_bits<4, 2>(p, s) : launch_mla_bits<4, 4>(p, s); break;
    default: e = h ? launch_mla_bits<8, 2>(p, s) : launch_mla_bits<8, 4>(p, s); break;
  }
  if (e != cudaSuccess) return e;
  {  // the combine: a programmatic dependent of the decode grid
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((p.batch * p.num_q_heads + 3) / 4);  // one warp per (sequence, head)
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = (int)cudaLaunchKernelEx(&cfg, combine_mla_kernel, p);
    if (e != cudaSuccess) return e;
  }
  return (int)cudaGetLastError();
}

}  // namespace kvq
