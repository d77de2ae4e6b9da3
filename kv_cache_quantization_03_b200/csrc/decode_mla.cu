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
// memory: scores = Q[128 x 576] K^T, out += P[128 x tokens] V[tokens x 512].
// 128 x 512 fp32 accumulators would fill all of the SM's tensor memory, so
// a cluster of two CTAs shares each (sequence, split): CTA r owns latent
// channels [256r, 256r + 256) of the output, computes the partial score over
// its channels (CTA 0 adds the rope part), and the two partial score blocks
// are exchanged through distributed shared memory.  Softmax runs one thread
// per head (a TMEM lane), with lazy rescaling of the output accumulator
// (only when the running max grows by more than 2^8).  Operands use the
// no-swizzle core-matrix layout (8 rows x 16 bytes per core matrix).
#include <cuda_runtime.h>

#include "kvq_device.cuh"

namespace kvq {
namespace {

constexpr int kT = 16;
constexpr int kLat = 512, kHalf = 256, kRope = 64;
constexpr int kKr = kHalf + kRope;     // K extent of the shared-memory operands (rope slot unused in CTA 1)
constexpr int kH = 128;                // M: heads (rows beyond num_q_heads are zero)
constexpr int kChunk = 32;             // tokens per step (two tiles)
constexpr int kThreads = 256;
constexpr float kNegBig = -1e30f;

// byte offsets in shared memory
constexpr int kSboK = kKr / 8 * 128;               // 5120: next 8 rows of a K-major operand
constexpr int kQsBytes = kH * kKr * 2;             // 81920
constexpr int kKbBytes = kChunk * kKr * 2;         // 20480 per buffer
constexpr int kPsBytes = kH * kChunk * 2;          // 8192
constexpr int kSxBytes = kH * kChunk * 4;          // 16384 per buffer
constexpr int kStageCodesMax = 2 * kT * kLat;      // 2 tiles at 8 bits
constexpr int kStageBytes = kStageCodesMax + 2 * kT * 8 + 2 * kHalf * 4 + 2 * kT * kRope * 2;  // 22784
constexpr int kOffQs = 0;
constexpr int kOffKb = kOffQs + kQsBytes;
constexpr int kOffPs = kOffKb + 2 * kKbBytes;
constexpr int kOffSx = kOffPs + kPsBytes;
constexpr int kOffSt = kOffSx + 2 * kSxBytes;
constexpr int kOffBar = kOffSt + 2 * kStageBytes;
constexpr int kOffPg = kOffBar + 64;
// within a stage: codes, (a, z), channel scales of this CTA's half, rope
constexpr int kStAz = kStageCodesMax, kStC = kStAz + 2 * kT * 8, kStRope = kStC + 2 * kHalf * 4;

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}
// K-major core-matrix layout offset of element (row, k) with kSboK bytes per 8 rows
__device__ __forceinline__ uint32_t km_off(int row, int k) {
  return (row >> 3) * kSboK + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
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
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Code of latent channel ch (0..511) of token row `row` of a tile, `bits` wide.
__device__ __forceinline__ uint32_t mla_code(const uint8_t* codes, int bits, int row, int ch) {
  if (bits == 3) {
    const uint32_t lo = (codes[row * (kLat / 4) + ch / 4] >> (2 * (ch % 4))) & 3u;
    const uint32_t hi = (codes[kT * (kLat / 4) + row * (kLat / 8) + ch / 8] >> (ch % 8)) & 1u;
    return lo | (hi << 2);
  }
  const int bit = (row * kLat + ch) * bits;
  return (codes[bit >> 3] >> (bit & 7)) & ((1u << bits) - 1u);
}

__global__ void __launch_bounds__(kThreads, 1) decode_mla_kernel(MlaDecodeParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t rank = cluster_rank();      // latent half owned by this CTA
  const int split = blockIdx.x >> 1, b = blockIdx.y;
  uint64_t* bar_stage = reinterpret_cast<uint64_t*>(smem + kOffBar);  // [2]
  uint64_t* bar_s = bar_stage + 2;
  uint64_t* bar_pv = bar_stage + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_stage + 4);
  int32_t* spg = reinterpret_cast<int32_t*>(smem + kOffPg);
  const uint32_t s_base = smem_u32(smem);

  int seq = p.seq_lens[b];
  if (seq < 0) seq = 0;
  int ntiles = seq / kT;
  if (ntiles > p.max_pages) ntiles = p.max_pages;
  if (split == 0 && rank == 0 && tid == 0) {
    if (p.seq_lens[b] < 0 || p.seq_lens[b] / kT > p.max_pages) set_error(p.err, KVQ_DEVERR_BAD_SEQ);
    if (p.seq_lens[b] % kT) set_error(p.err, KVQ_DEVERR_PARTIAL_TILE);
  }
  const int t0 = split * p.tiles_per_split;
  const int t1 = min(t0 + p.tiles_per_split, ntiles);
  const int ntl = t1 > t0 ? t1 - t0 : 0;
  const int nchunks = (ntl + 1) / 2;
  for (int i = tid; i < ntl; i += kThreads) spg[i] = p.block_table[(size_t)b * p.max_pages + t0 + i];
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bar_stage[i], 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;   // columns [0, 256): output half; [256, 288): scores

  // ---- producer: raw chunk c into stage c & 1 (thread 0)
  auto issue = [&](int c) {
    uint64_t* bar = &bar_stage[c & 1];
    uint8_t* st = smem + kOffSt + (c & 1) * kStageBytes;
    uint32_t bytes = 0;
    const int tile_code_bytes = kT * kLat * p.bits / 8;
    for (int j = 0; j < 2; ++j) {
      const int lt = 2 * c + j;
      if (lt >= ntl) break;
      const int page = spg[lt];
      if (page < 0 || page >= p.num_pages) continue;
      bytes += tile_code_bytes + kT * 8 + kHalf * 4 + (rank == 0 ? kT * kRope * 2 : 0);
    }
    mbar_arrive_expect_tx(bar, bytes);
    for (int j = 0; j < 2; ++j) {
      const int lt = 2 * c + j;
      if (lt >= ntl) break;
      const int page = spg[lt];
      if (page < 0 || page >= p.num_pages) {
        set_error(p.err, KVQ_DEVERR_BAD_PAGE);
        continue;
      }
      const size_t slot = (size_t)p.layer * p.num_pages + page;
      bulk_g2s(st + j * tile_code_bytes, p.codes + slot * tile_code_bytes, tile_code_bytes, bar);
      bulk_g2s(st + kStAz + j * kT * 8, p.tok + slot * kT * 2, kT * 8, bar);
      bulk_g2s(st + kStC + j * kHalf * 4, p.chan + slot * kLat + rank * kHalf, kHalf * 4, bar);
      if (rank == 0) bulk_g2s(st + kStRope + j * kT * kRope * 2, p.rope + slot * kT * kRope, kT * kRope * 2, bar);
    }
  };
  if (tid == 0) {
    if (nchunks > 0) issue(0);
    if (nchunks > 1) issue(1);
  }

  // ---- queries: rotated latent half and (CTA 0) rope, prescaled, f16, K-major in Qs.
  // Rotation of channels [256r, 256r + 256): H_512 = H_2 (x) H_256, so it is
  // H_256 (q[0:256] + (-1)^r q[256:512]) / sqrt(512).  Done 64 heads at a time
  // in fp32 scratch that overlays the not-yet-used operand buffers.
  {
    float* scr = reinterpret_cast<float*>(smem + kOffKb);   // [64][256] fp32 = 64 KB
    const float sgn = rank ? -1.f : 1.f;
    const float f = p.scale_log2 * 0.044194173824159216f;   // scale * log2(e) / sqrt(512)
    for (int hb = 0; hb < 2; ++hb) {
      for (int i = tid; i < 64 * kHalf; i += kThreads) {
        const int hl = i / kHalf, j = i % kHalf, h = hb * 64 + hl;
        float v = 0.f;
        if (h < p.num_q_heads) {
          const uint16_t* qh = p.q + ((size_t)b * p.num_q_heads + h) * (kLat + kRope);
          v = bf16f(qh[j]) + sgn * bf16f(qh[kHalf + j]);
        }
        scr[i] = v;
      }
      __syncthreads();
      for (int s = 1; s < kHalf; s <<= 1) {
        for (int i = tid; i < 64 * kHalf / 2; i += kThreads) {
          const int hl = i / (kHalf / 2), k = i % (kHalf / 2);
          const int lo = (k / s) * 2 * s + (k % s), hi = lo + s;
          const float x = scr[hl * kHalf + lo], y = scr[hl * kHalf + hi];
          scr[hl * kHalf + lo] = x + y;
          scr[hl * kHalf + hi] = x - y;
        }
        __syncthreads();
      }
      for (int i = tid; i < 64 * kHalf; i += kThreads) {
        const int hl = i / kHalf, j = i % kHalf;
        *reinterpret_cast<__half*>(smem + kOffQs + km_off(hb * 64 + hl, j)) = __float2half_rn(scr[i] * f);
      }
      __syncthreads();
    }
    for (int i = tid; i < kH * kRope; i += kThreads) {
      const int h = i / kRope, j = i % kRope;
      float v = 0.f;
      if (rank == 0 && h < p.num_q_heads)
        v = bf16f(p.q[((size_t)b * p.num_q_heads + h) * (kLat + kRope) + kLat + j]) * p.scale_log2;
      *reinterpret_cast<__half*>(smem + kOffQs + km_off(h, kHalf + j)) = __float2half_rn(v);
    }
  }

  // ---- main loop over 32-token chunks
  const uint32_t idesc_s = (1u << 4) | ((uint32_t)(kChunk >> 3) << 17) | ((uint32_t)(kH >> 4) << 24);
  const uint32_t idesc_pv = (1u << 4) | (1u << 16) | ((uint32_t)(kHalf >> 3) << 17) | ((uint32_t)(kH >> 4) << 24);
  const int ksteps_s = (rank == 0 ? kKr : kHalf) / 16;
  float m_run = kNegBig, l_run = 0.f;     // warps 0..3: head `tid`
  bool ok = true;
  const uint32_t peer = rank ^ 1u;
  for (int c = 0; c < nchunks; ++c) {
    // a. raw chunk arrived
    ok &= mbar_wait_bounded(&bar_stage[c & 1], (uint32_t)(c >> 1) & 1u, ok ? kWaitLimit : 0u);
    // b. dequantise into Kb[c & 1]: thread -> token tid / 8, 32 channels of this half
    {
      const uint8_t* st = smem + kOffSt + (c & 1) * kStageBytes;
      uint8_t* kb = smem + kOffKb + (c & 1) * kKbBytes;
      const int tl = tid >> 3, seg = tid & 7, j = tl >> 4, row = tl & 15;
      const int lt = 2 * c + j;
      const bool valid = lt < ntl && spg[lt] >= 0 && spg[lt] < p.num_pages;
      const int tile_code_bytes = kT * kLat * p.bits / 8;
      const float2 az = valid ? *reinterpret_cast<const float2*>(st + kStAz + j * kT * 8 + row * 8) : make_float2(0.f, 0.f);
      const float* cc = reinterpret_cast<const float*>(st + kStC + j * kHalf * 4) + 32 * seg;
      const uint8_t* codes = st + j * tile_code_bytes;
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v0 = 0.f, v1 = 0.f;
          if (valid) {
            const int k0 = 32 * seg + 8 * g8 + 2 * e;
            v0 = fmaf(az.x, (float)mla_code(codes, p.bits, row, kHalf * rank + k0), az.y) * cc[8 * g8 + 2 * e];
            v1 = fmaf(az.x, (float)mla_code(codes, p.bits, row, kHalf * rank + k0 + 1), az.y) * cc[8 * g8 + 2 * e + 1];
          }
          pk[e] = pack_f16x2(v0, v1);
        }
        *reinterpret_cast<uint4*>(kb + km_off(tl, 32 * seg + 8 * g8)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      if (rank == 0) {  // rope: 8 channels per thread
        const uint16_t* rp = reinterpret_cast<const uint16_t*>(st + kStRope + j * kT * kRope * 2) + row * kRope + 8 * seg;
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          pk[e] = valid ? pack_f16x2(bf16f(rp[2 * e]), bf16f(rp[2 * e + 1])) : 0u;
        *reinterpret_cast<uint4*>(kb + km_off(tl, kHalf + 8 * seg)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
    proxy_fence();
    __syncthreads();
    // c. refill the stage, issue the score MMAs
    if (tid == 0) {
      if (c + 2 < nchunks) issue(c + 2);
      tc_fence_after();
      const uint32_t qs = s_base + kOffQs, kb = s_base + kOffKb + (c & 1) * kKbBytes;
      for (int s = 0; s < ksteps_s; ++s)
        umma_f16(tmem + kHalf, umma_desc(qs + s * 256, 128, kSboK), umma_desc(kb + s * 256, 128, kSboK), idesc_s,
                 s > 0);
      umma_commit(bar_s);
    }
    // d. scores: own partial to the peer, full scores, online softmax, P
    float sc[32];
    if (warp < 4) {
      ok &= mbar_wait_bounded(bar_s, (uint32_t)c & 1u, ok ? kWaitLimit : 0u);
      tc_fence_after();
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + kHalf, sc);
      const uint32_t dst = peer_addr(s_base + kOffSx + (c & 1) * kSxBytes + tid * 128, peer);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        st_cluster_v4(dst + 16 * i, make_float4(sc[4 * i], sc[4 * i + 1], sc[4 * i + 2], sc[4 * i + 3]));
    }
    cluster_sync();
    if (warp < 4) {
      const float* sx = reinterpret_cast<const float*>(smem + kOffSx + (c & 1) * kSxBytes) + tid * 32;
      bool tv[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int lt = 2 * c + j;
        tv[j] = lt < ntl && spg[lt] >= 0 && spg[lt] < p.num_pages;
      }
      float mx = kNegBig;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        sc[i] = tv[i >> 4] ? sc[i] + sx[i] : kNegBig;
        mx = fmaxf(mx, sc[i]);
      }
      if (c > 0) ok &= mbar_wait_bounded(bar_pv, (uint32_t)(c - 1) & 1u, ok ? kWaitLimit : 0u);  // P and O are free
      tc_fence_after();
      // lazy rescale: a head whose max grew by more than 2^8 moves its running max;
      // the TMEM accesses are warp-wide, so the whole warp joins (factor 1 where unchanged)
      const bool grow = mx > m_run + 8.f;
      const float alpha = grow ? ex2f(m_run - mx) : 1.f;
      if (__any_sync(0xffffffffu, grow && c > 0)) {
        for (int c0 = 0; c0 < kHalf; c0 += 32) {
          float o[32];
          const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16) + c0;
          tmem_ld32(ta, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(ta, o);
        }
      }
      if (grow) {
        l_run *= alpha;
        m_run = mx;
      }
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
      uint8_t* ps = smem + kOffPs;
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8)
        *reinterpret_cast<uint4*>(ps + (tid >> 3) * 512 + g8 * 128 + (tid & 7) * 16) =
            make_uint4(pk[4 * g8], pk[4 * g8 + 1], pk[4 * g8 + 2], pk[4 * g8 + 3]);
      proxy_fence();
      tc_fence_before();
    }
    __syncthreads();
    // e. out += P V (V = the chunk's latent half, read as an MN-major operand)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ps = s_base + kOffPs, kb = s_base + kOffKb + (c & 1) * kKbBytes;
      for (int s = 0; s < kChunk / 16; ++s)
        umma_f16(tmem, umma_desc(ps + s * 256, 128, 512), umma_desc(kb + s * 2 * kSboK, kSboK, 128), idesc_pv,
                 (c > 0 || s > 0) ? 1u : 0u);
      umma_commit(bar_pv);
    }
  }

  // ---- epilogue: this split's partial output half, (max, sum) per head
  if (warp < 4) {
    float* po = p.part_o + (((size_t)b * p.splits + split) * kH + tid) * kLat + rank * kHalf;
    if (nchunks > 0) {
      ok &= mbar_wait_bounded(bar_pv, (uint32_t)(nchunks - 1) & 1u, ok ? kWaitLimit : 0u);
      tc_fence_after();
      for (int c0 = 0; c0 < kHalf; c0 += 32) {
        float o[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, o);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float4*>(po + c0 + 4 * i) = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
      }
    } else {
      for (int c0 = 0; c0 < kHalf; c0 += 4) *reinterpret_cast<float4*>(po + c0) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (rank == 0) {
      float* pm = p.part_ml + (((size_t)b * p.splits + split) * kH + tid) * 2;
      pm[0] = m_run;
      pm[1] = l_run;
    }
  }
  if (!ok && tid == 0) set_error(p.err, KVQ_DEVERR_TIMEOUT);
  tc_fence_before();
  cluster_sync();   // no DSMEM traffic may target a CTA that has exited
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
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

}  // namespace

int launch_decode_mla(const MlaDecodeParams& p, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int smem = kOffPg + ((p.tiles_per_split * 4 + 15) / 16) * 16;
  cudaFuncSetAttribute(decode_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
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
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_mla_kernel, p);
  if (e != cudaSuccess) return (int)e;
  combine_mla_kernel<<<p.batch * p.num_q_heads, kLat, 0, s>>>(p);
  return (int)cudaGetLastError();
}

}  // namespace kvq
