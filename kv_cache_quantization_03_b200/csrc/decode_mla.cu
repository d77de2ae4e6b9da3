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
// memory: scores = Q K^T, out += P V.  128 x 512 fp32 output accumulators
// would fill all of an SM's tensor memory, so a cluster of two CTAs shares
// each (sequence, split): CTA r owns latent channels [256r, 256r + 256) of
// the output and rope channels [32r, 32r + 32) of the score, computes the
// partial score over its 288 channels, and the two partial score blocks are
// exchanged through distributed shared memory.
//
// Each CTA is a pipeline of three roles connected by mbarriers:
//   warp 8 (one thread)  bulk copies of the raw tiles into a ring of stages,
//                        and the tcgen05 MMAs: S(c) = Q K(c)^T into one of
//                        two TMEM score buffers, then O += P(c-1) V(c-1);
//   warps 4-7            dequantise a 32-token chunk, (a q + z) c in fp32,
//                        to f16 in the no-swizzle core-matrix operand layout
//                        (three buffers, so they run up to two chunks ahead);
//   warps 0-3            one thread per head (a TMEM lane): load the partial
//                        score, send it to the peer CTA, add the peer's
//                        partial, online softmax with lazy rescaling of the
//                        TMEM output (only when the running max grows by
//                        more than 2^8), P in f16 to shared memory.
// The softmax of chunk c-1 overlaps the dequantisation of chunk c+1 and the
// score MMA of chunk c.  Every wait is bounded in time (1 s of global time);
// a wait that runs out raises KVQ_DEVERR_TIMEOUT and the remaining waits of
// that thread are skipped, so the kernel always terminates.
//
// The rotated, pre-scaled f16 query of every (sequence, latent half) is
// built once by mla_prep_q_kernel in exactly the shared-memory operand
// layout, and each CTA fetches its 72 KB with one bulk copy.
#include <cuda_runtime.h>

#include "kvq_device.cuh"

namespace kvq {
namespace {

constexpr int kT = 16;
constexpr int kLat = 512, kHalf = 256, kRope = 64, kRopeHalf = 32;
constexpr int kK = kHalf + kRopeHalf;  // 288: K extent of this CTA's score operands
constexpr int kH = 128;                // M: heads (rows beyond num_q_heads are zero)
constexpr int kChunk = 32;             // tokens per step (two tiles)
constexpr int kDqWarps = 4;
constexpr int kThreads = 9 * 32;       // softmax 0-3, dequantisation 4-7, copies + MMA 8
constexpr int kNB = 3;                 // dequantised chunk buffers
constexpr float kNegBig = -1e30f;

// byte offsets in shared memory
constexpr int kSbo = kK / 8 * 128;           // 4608: next 8 rows of a K-major operand
constexpr int kQsBytes = kH * kK * 2;        // 73728
constexpr int kKbBytes = kChunk * kK * 2;    // 18432 per buffer
constexpr int kPsBytes = kH * kChunk * 2;    // 8192 per buffer
constexpr int kSxBytes = kH * kChunk * 4;    // 16384 per buffer
constexpr int kOffQs = 0;
constexpr int kOffKb = kOffQs + kQsBytes;
constexpr int kOffPs = kOffKb + kNB * kKbBytes;
constexpr int kOffSx = kOffPs + 2 * kPsBytes;
constexpr int kOffSt = kOffSx + 2 * kSxBytes;
// a stage holds two tiles: codes | (a, z) | channel scales of this CTA's half | rope
__host__ __device__ constexpr int tile_code_bytes(int bits) { return kT * kLat * bits / 8; }
__host__ __device__ constexpr int stage_bytes(int bits) {
  return 2 * (tile_code_bytes(bits) + kT * 8 + kHalf * 4 + kT * kRope * 2);
}
__host__ __device__ constexpr int num_stages(int bits) { return bits == 8 ? 2 : 3; }
__host__ __device__ constexpr int bar_offset(int bits) { return kOffSt + num_stages(bits) * stage_bytes(bits); }
// full[3] dq[kNB] sfull[2] pfull[2] pv[4] sxf[2] sxe[2] qf[1], then the TMEM address
constexpr int kNumBars = 3 + kNB + 2 + 2 + 4 + 2 + 2 + 1;
__host__ __device__ constexpr int smem_bytes(int bits) { return bar_offset(bits) + kNumBars * 8 + 16; }
static_assert(smem_bytes(8) <= 232448 && smem_bytes(4) <= 232448, "shared memory");

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}
// K-major core-matrix layout offset of element (row, k), kSbo bytes per 8 rows
__host__ __device__ __forceinline__ uint32_t km_off(int row, int k) {
  return (row >> 3) * kSbo + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
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

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]),
      "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]),
      "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]),
      "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31]));
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t peer) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(peer));
  return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
// Arrive (count 1) on an mbarrier of the peer CTA; orders this thread's
// earlier shared-memory accesses of the cluster before it.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void mbar_arrive_local(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Bounded wait with cluster-scope acquire: for phases completed by the peer.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t limit) {
  const uint32_t a = smem_u32(bar);
  uint64_t t0 = 0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (;;) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
    uint64_t t1;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
    if (t1 - t0 >= limit) return false;
  }
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

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) decode_mla_kernel(MlaDecodeParams p) {
  constexpr int NS = num_stages(BITS), SB = stage_bytes(BITS), CB = tile_code_bytes(BITS);
  constexpr int kStAz = 2 * CB, kStC = kStAz + 2 * kT * 8, kStRope = kStC + 2 * kHalf * 4;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank(), peer = rank ^ 1u;  // latent half owned by this CTA
  const int split = blockIdx.x >> 1, b = blockIdx.y;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + bar_offset(BITS));
  uint64_t* dq = full + 3;
  uint64_t* sfull = dq + kNB;
  uint64_t* pfull = sfull + 2;
  uint64_t* pv = pfull + 2;
  uint64_t* sxf = pv + 4;
  uint64_t* sxe = sxf + 2;
  uint64_t* qf = sxe + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qf + 1);
  const uint32_t s_base = smem_u32(smem);

  const int seq_raw = p.seq_lens[b];
  int ntiles = seq_raw < 0 ? 0 : seq_raw / kT;
  if (ntiles > p.max_pages) ntiles = p.max_pages;
  if (split == 0 && rank == 0 && tid == 0) {
    if (seq_raw < 0 || seq_raw / kT > p.max_pages) set_error(p.err, KVQ_DEVERR_BAD_SEQ);
    if (seq_raw % kT) set_error(p.err, KVQ_DEVERR_PARTIAL_TILE);
  }
  const int t0 = split * p.tiles_per_split;
  const int t1 = min(t0 + p.tiles_per_split, ntiles);
  const int ntl = t1 > t0 ? t1 - t0 : 0;
  const int nchunks = (ntl + 1) / 2;
  const int32_t* btab = p.block_table + (size_t)b * p.max_pages + t0;
  auto tile_ok = [&](int lt) {
    if (lt >= ntl) return false;
    const int pg = __ldg(btab + lt);
    return pg >= 0 && pg < p.num_pages;
  };

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < NS; ++i) mbar_init(&full[i], 1);
#pragma unroll
    for (int i = 0; i < kNB; ++i) mbar_init(&dq[i], kDqWarps * 32);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], kH);
      mbar_init(&sxf[i], kH);
      mbar_init(&sxe[i], kH);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) mbar_init(&pv[i], 1);
    mbar_init(qf, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive
  const uint32_t tmem = *tmem_slot;  // columns [0, 256): output half; [256, 320): two score buffers
  bool ok = true;

  if (warp == 8) {
    // ---------------------------------------------------------------- copies + MMA (one thread)
    if (lane == 0) {
      mbar_arrive_expect_tx(qf, kQsBytes);
      bulk_g2s(smem + kOffQs, p.qprep + ((size_t)b * 2 + rank) * kQsBytes, kQsBytes, qf);
      auto issue = [&](int c) {  // raw chunk c into stage c % NS
        uint64_t* bar = &full[c % NS];
        uint8_t* st = smem + kOffSt + (c % NS) * SB;
        uint32_t bytes = 0;
#pragma unroll
        for (int j = 0; j < 2; ++j)
          if (tile_ok(2 * c + j)) bytes += CB + kT * 8 + kHalf * 4 + kT * kRope * 2;
        mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int lt = 2 * c + j;
          if (!tile_ok(lt)) {
            if (lt < ntl) set_error(p.err, KVQ_DEVERR_BAD_PAGE);
            continue;
          }
          const size_t slot = (size_t)p.layer * p.num_pages + __ldg(btab + lt);
          bulk_g2s(st + j * CB, p.codes + slot * CB, CB, bar);
          bulk_g2s(st + kStAz + j * kT * 8, p.tok + slot * kT * 2, kT * 8, bar);
          bulk_g2s(st + kStC + j * kHalf * 4, p.chan + slot * kLat + rank * kHalf, kHalf * 4, bar);
          bulk_g2s(st + kStRope + j * kT * kRope * 2, p.rope + slot * kT * kRope, kT * kRope * 2, bar);
        }
      };
      const int pre = nchunks < NS ? nchunks : NS;
      for (int c = 0; c < pre; ++c) issue(c);
      const uint32_t idesc_s = (1u << 4) | ((uint32_t)(kChunk >> 3) << 17) | ((uint32_t)(kH >> 4) << 24);
      const uint32_t idesc_pv = (1u << 4) | (1u << 16) | ((uint32_t)(kHalf >> 3) << 17) | ((uint32_t)(kH >> 4) << 24);
      const uint32_t qs = s_base + kOffQs;
      ok &= mbar_wait_bounded(qf, 0u, kWaitLimit);
      for (int c = 0; c <= nchunks; ++c) {
        if (c < nchunks) {
          // chunk c is dequantised; its raw stage is free again
          ok &= mbar_wait_bounded(&dq[c % kNB], (uint32_t)(c / kNB) & 1u, ok ? kWaitLimit : 0u);
          if (c + NS < nchunks) {
            proxy_fence();
            issue(c + NS);
          }
          tc_fence_after();
          const uint32_t kb = s_base + kOffKb + (c % kNB) * kKbBytes;
#pragma unroll 1
          for (int s = 0; s < kK / 16; ++s)
            umma_f16(tmem + kHalf + 32 * (c & 1), umma_desc(qs + s * 256, 128, kSbo), umma_desc(kb + s * 256, 128, kSbo),
                     idesc_s, s > 0);
          umma_commit(&sfull[c & 1]);
        }
        if (c >= 1) {
          const int x = c - 1;
          ok &= mbar_wait_bounded(&pfull[x & 1], (uint32_t)(x >> 1) & 1u, ok ? kWaitLimit : 0u);
          tc_fence_after();
          const uint32_t ps = s_base + kOffPs + (x & 1) * kPsBytes, kb = s_base + kOffKb + (x % kNB) * kKbBytes;
#pragma unroll
          for (int s = 0; s < kChunk / 16; ++s)
            umma_f16(tmem, umma_desc(ps + s * 256, 128, 512), umma_desc(kb + s * 2 * kSbo, kSbo, 128), idesc_pv,
                     (x > 0 || s > 0) ? 1u : 0u);
          umma_commit(&pv[x & 3]);
        }
      }
      // no bulk copy may still be writing when the CTA exits
      for (int c = nchunks > NS ? nchunks - NS : 0; c < nchunks; ++c)
        ok &= mbar_wait_bounded(&full[c % NS], (uint32_t)(c / NS) & 1u, ok ? kWaitLimit : 0u);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- dequantisation
    // Lane l converts latent channels 8l..8l+7 of this half for the chunk rows
    // 8 dw + ((l + it) & 7), it = 0..7 (both the code loads and the operand
    // stores are free of bank conflicts), then 8 rope channels of one row.
    const int dw = warp - 4, j = dw >> 1;
    for (int c = 0; c < nchunks; ++c) {
      ok &= mbar_wait_bounded(&full[c % NS], (uint32_t)(c / NS) & 1u, ok ? kWaitLimit : 0u);
      if (c >= kNB)  // PV(c - kNB) has read this operand buffer
        ok &= mbar_wait_bounded(&pv[(c - kNB) & 3], (uint32_t)((c - kNB) >> 2) & 1u, ok ? kWaitLimit : 0u);
      const uint8_t* st = smem + kOffSt + (c % NS) * SB;
      uint8_t* kb = smem + kOffKb + (c % kNB) * kKbBytes;
      const bool valid = tile_ok(2 * c + j);
      f2 cc[4];
      {
        const float4* cp = reinterpret_cast<const float4*>(st + kStC + j * kHalf * 4) + 2 * lane;
        const float4 c0 = cp[0], c1 = cp[1];
        cc[0] = make_float2(c0.x, c0.y), cc[1] = make_float2(c0.z, c0.w);
        cc[2] = make_float2(c1.x, c1.y), cc[3] = make_float2(c1.z, c1.w);
      }
#pragma unroll 2
      for (int it = 0; it < 8; ++it) {
        const int tr = 8 * (dw & 1) + ((lane + it) & 7);
        const float2 az = *reinterpret_cast<const float2*>(st + kStAz + j * kT * 8 + tr * 8);
        float q[8];
        codes8<BITS>(st + j * CB, tr, kHalf * (int)rank + 8 * lane, q);
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const f2 v = mul2(fma2(splat2(az.x), make_float2(q[2 * e], q[2 * e + 1]), splat2(az.y)), cc[e]);
          pk[e] = valid ? pack_f16x2(v.x, v.y) : 0u;
        }
        *reinterpret_cast<uint4*>(kb + km_off(16 * j + tr, 8 * lane)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      {
        const int row = 8 * dw + (lane & 7), grp = lane >> 3;
        const bool v2 = tile_ok(2 * c + (row >> 4));
        const uint4 r = *reinterpret_cast<const uint4*>(st + kStRope + (row >> 4) * kT * kRope * 2 +
                                                        (row & 15) * kRope * 2 + (kRopeHalf * rank + 8 * grp) * 2);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) pk[e] = v2 ? pack_f16x2(bf16f(w[e] & 0xFFFFu), bf16f(w[e] >> 16)) : 0u;
        *reinterpret_cast<uint4*>(kb + km_off(row, kHalf + 8 * grp)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      proxy_fence();
      mbar_arrive_local(&dq[c % kNB]);
    }
  } else {
    // ---------------------------------------------------------------- softmax, one thread per head
    const int h = tid;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t sx_peer = peer_addr(s_base + kOffSx, peer);
    const uint32_t sxf_peer = peer_addr(smem_u32(sxf), peer), sxe_peer = peer_addr(smem_u32(sxe), peer);
    float m_run = kNegBig, l_run = 0.f;
    float prev[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) prev[i] = 0.f;
    for (int c = 0; c <= nchunks; ++c) {
      float cur[32];
      if (c < nchunks) {
        // own partial score of chunk c -> row h of the peer's exchange buffer c & 1
        ok &= mbar_wait_bounded(&sfull[c & 1], (uint32_t)(c >> 1) & 1u, ok ? kWaitLimit : 0u);
        tc_fence_after();
        tmem_ld32(tmem + lane_base + kHalf + 32 * (c & 1), cur);
        if (c >= 2)  // the peer has read chunk c - 2 out of that buffer
          ok &= mbar_wait_cluster(&sxe[c & 1], (uint32_t)((c - 2) >> 1) & 1u, ok ? kWaitLimit : 0u);
        const uint32_t dst = sx_peer + (c & 1) * kSxBytes + h * 128;
#pragma unroll
        for (int i = 0; i < 8; ++i)  // 16-byte chunk i of the row at i ^ (h & 7): no bank conflicts
          st_cluster_v4(dst + 16 * (i ^ (h & 7)), cur[4 * i], cur[4 * i + 1], cur[4 * i + 2], cur[4 * i + 3]);
        mbar_arrive_remote(sxf_peer + 8 * (c & 1));
      }
      if (c >= 1) {
        const int x = c - 1;
        ok &= mbar_wait_cluster(&sxf[x & 1], (uint32_t)(x >> 1) & 1u, ok ? kWaitLimit : 0u);
        const float4* sx = reinterpret_cast<const float4*>(smem + kOffSx + (x & 1) * kSxBytes + h * 128);
        float sc[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 v = sx[i ^ (h & 7)];
          sc[4 * i] = prev[4 * i] + v.x, sc[4 * i + 1] = prev[4 * i + 1] + v.y;
          sc[4 * i + 2] = prev[4 * i + 2] + v.z, sc[4 * i + 3] = prev[4 * i + 3] + v.w;
        }
        mbar_arrive_remote(sxe_peer + 8 * (x & 1));
        const bool tv[2] = {tile_ok(2 * x), tile_ok(2 * x + 1)};
        float mx = kNegBig;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          sc[i] = tv[i >> 4] ? sc[i] : kNegBig;
          mx = fmaxf(mx, sc[i]);
        }
        // lazy rescale; the TMEM accesses are warp-wide, so the whole warp
        // joins (factor 1 where a head's max did not grow)
        const bool grow = mx > m_run + 8.f;
        const float alpha = grow ? ex2f(m_run - mx) : 1.f;
        if (__any_sync(0xffffffffu, grow && x > 0)) {
          ok &= mbar_wait_bounded(&pv[(x - 1) & 3], (uint32_t)((x - 1) >> 2) & 1u, ok ? kWaitLimit : 0u);
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < kHalf; c0 += 32) {
            float o[32];
            tmem_ld32(tmem + lane_base + c0, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
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
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = tv[i >> 3] ? ex2f(sc[2 * i] - m_run) : 0.f;
          const float p1 = tv[i >> 3] ? ex2f(sc[2 * i + 1] - m_run) : 0.f;
          ls += p0 + p1;
          pk[i] = pack_f16x2(p0, p1);
        }
        l_run += ls;
        uint8_t* ps = smem + kOffPs + (x & 1) * kPsBytes;
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8)
          *reinterpret_cast<uint4*>(ps + (h >> 3) * 512 + g8 * 128 + (h & 7) * 16) =
              make_uint4(pk[4 * g8], pk[4 * g8 + 1], pk[4 * g8 + 2], pk[4 * g8 + 3]);
        proxy_fence();
        tc_fence_before();
        mbar_arrive_local(&pfull[x & 1]);
      }
      if (c < nchunks) {
#pragma unroll
        for (int i = 0; i < 32; ++i) prev[i] = cur[i];
      }
    }
    // ---- epilogue: this split's partial output half, (max, sum) per head
    float* po = p.part_o + (((size_t)b * p.splits + split) * kH + h) * kLat + rank * kHalf;
    if (nchunks > 0) {
      const int x = nchunks - 1;
      ok &= mbar_wait_bounded(&pv[x & 3], (uint32_t)(x >> 2) & 1u, ok ? kWaitLimit : 0u);
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < kHalf; c0 += 32) {
        float o[32];
        tmem_ld32(tmem + lane_base + c0, o);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float4*>(po + c0 + 4 * i) = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
      }
    } else {
      for (int c0 = 0; c0 < kHalf; c0 += 4) *reinterpret_cast<float4*>(po + c0) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (rank == 0) {
      float* pm = p.part_ml + (((size_t)b * p.splits + split) * kH + h) * 2;
      pm[0] = m_run;
      pm[1] = l_run;
    }
  }
  if (!ok) set_error(p.err, KVQ_DEVERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no DSMEM traffic may target a CTA that has exited
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
}

// Rotated, pre-scaled f16 queries of one (sequence, latent half r), in the
// K-major core-matrix layout of the score operand: channels [0, 256) hold
// (H_512 q_lat)[256r + i] * scale * log2(e) / sqrt(512), which is
// H_256 (q[0:256] + (-1)^r q[256:512]) since H_512 = H_2 (x) H_256; channels
// [256, 288) hold rope channels [32r, 32r + 32) * scale * log2(e).
// One warp per head: lane l keeps elements 8l..8l+7; index bits 0..2 are
// butterflies in registers, bits 3..7 shuffles.
__global__ void __launch_bounds__(256) mla_prep_q_kernel(MlaDecodeParams p) {
  const int b = blockIdx.x, r = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* out = p.qprep + ((size_t)b * 2 + r) * kQsBytes;
  const float sgn = r ? -1.f : 1.f;
  const float f = p.scale_log2 * 0.044194173824159216f;  // 1 / sqrt(512)
  for (int h = warp; h < kH; h += 8) {
    float v[8];
    const bool live = h < p.num_q_heads;
    const uint16_t* qh = p.q + ((size_t)b * p.num_q_heads + (live ? h : 0)) * (kLat + kRope);
    {
      const uint4 lo = *reinterpret_cast<const uint4*>(qh + 8 * lane);
      const uint4 hi = *reinterpret_cast<const uint4*>(qh + kHalf + 8 * lane);
      const uint32_t a[4] = {lo.x, lo.y, lo.z, lo.w}, c[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = live ? bf16f(a[e] & 0xFFFFu) + sgn * bf16f(c[e] & 0xFFFFu) : 0.f;
        v[2 * e + 1] = live ? bf16f(a[e] >> 16) + sgn * bf16f(c[e] >> 16) : 0.f;
      }
    }
#pragma unroll
    for (int s = 1; s < 8; s <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (!(i & s)) {
          const float x = v[i], y = v[i + s];
          v[i] = x + y;
          v[i + s] = x - y;
        }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, v[i], off);
        v[i] = upper ? (o - v[i]) : (v[i] + o);
      }
    }
    *reinterpret_cast<uint4*>(out + km_off(h, 8 * lane)) =
        make_uint4(pack_f16x2(v[0] * f, v[1] * f), pack_f16x2(v[2] * f, v[3] * f), pack_f16x2(v[4] * f, v[5] * f),
                   pack_f16x2(v[6] * f, v[7] * f));
    if (lane < 4) {
      const uint4 w = *reinterpret_cast<const uint4*>(qh + kLat + kRopeHalf * r + 8 * lane);
      const uint32_t a[4] = {w.x, w.y, w.z, w.w};
      uint32_t pk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        pk[e] = live ? pack_f16x2(bf16f(a[e] & 0xFFFFu) * p.scale_log2, bf16f(a[e] >> 16) * p.scale_log2) : 0u;
      *reinterpret_cast<uint4*>(out + km_off(h, kHalf + 8 * lane)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
}

// Merge the splits of one (sequence, head), normalise, rotate back with H_512.
__global__ void __launch_bounds__(kLat) combine_mla_kernel(MlaDecodeParams p) {
  __shared__ float buf[kLat];
  const int b = blockIdx.x / p.num_q_heads, h = blockIdx.x % p.num_q_heads, j = threadIdx.x;
  float mx = kNegBig;
  for (int s = 0; s < p.splits; ++s) mx = fmaxf(mx, p.part_ml[(((size_t)b * p.splits + s) * kH + h) * 2]);
  float acc = 0.f, l = 0.f;
  for (int s = 0; s < p.splits; ++s) {
    const size_t i = ((size_t)b * p.splits + s) * kH + h;
    const float f = ex2f(p.part_ml[i * 2] - mx);
    acc = fmaf(f, p.part_o[i * kLat + j], acc);
    l = fmaf(f, p.part_ml[i * 2 + 1], l);
  }
  buf[j] = l > 0.f ? acc / l : 0.f;
  __syncthreads();
  for (int s = 1; s < kLat; s <<= 1) {
    const float x = buf[j & ~s], y = buf[j | s];
    __syncthreads();
    buf[j] = (j & s) ? (x - y) : (x + y);
    __syncthreads();
  }
  p.out[((size_t)b * p.num_q_heads + h) * kLat + j] = buf[j] * 0.044194173824159216f;
}

template <int BITS>
int launch_mla_bits(const MlaDecodeParams& p, cudaStream_t s) {
  const int smem = smem_bytes(BITS);
  cudaError_t e = cudaFuncSetAttribute(decode_mla_kernel<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * p.splits, p.batch, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&cfg, decode_mla_kernel<BITS>, p);
}

}  // namespace

size_t mla_qprep_bytes(int64_t batch) { return (size_t)batch * 2 * kQsBytes; }

int launch_decode_mla(const MlaDecodeParams& p, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  mla_prep_q_kernel<<<dim3(p.batch, 2, 1), 256, 0, s>>>(p);
  int e = (int)cudaGetLastError();
  if (e != cudaSuccess) return e;
  switch (p.bits) {
    case 2: e = launch_mla_bits<2>(p, s); break;
    case 3: e = launch_mla_bits<3>(p, s); break;
    case 4: e = launch_mla_bits<4>(p, s); break;
    default: e = launch_mla_bits<8>(p, s); break;
  }
  if (e != cudaSuccess) return e;
  combine_mla_kernel<<<p.batch * p.num_q_heads, kLat, 0, s>>>(p);
  return (int)cudaGetLastError();
}

}  // namespace kvq
