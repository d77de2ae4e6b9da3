// C ABI of the kvq library: argument validation, cache layout sizing,
// split-KV planning and kernel dispatch.  No allocation, no synchronisation
// (except kvq_read_error).  Declarations and the method's citations are in
// include/kvq.h.
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdio>
#include <cstring>

#include "kvq_internal.h"

using namespace kvq;

namespace {

// Testing hook (kvq_set_test_wait): 0 in normal use.
std::atomic<uint32_t> g_test_wait_ns{0};

constexpr int kDefaultSMs = 148;       // B200, when no device can be queried (host-only sizing)
constexpr int kDecodeCtasPerSm = 4;      // resident decode CTAs per SM (registers and shared memory)
constexpr int kDecodeWarps = 4;        // warps per decode CTA (tiles are dealt round robin)
constexpr int kMaxGroup = 8;

bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }

// SMs of the current device (the split plans size their grids by it); the
// B200's 148 when there is no device.  kvq_decode_workspace_bytes and the
// decode calls use the same count, so a workspace sized on a device fits
// the calls made on it.
int num_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();  // clear the error the failed query left behind
    return kDefaultSMs;
  }
  return sms;
}
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_bits(int b) { return b == 2 || b == 3 || b == 4 || b == 8; }

kvq_status check_config(const kvq_config* c) {
  if (!c) return KVQ_ERR_INVALID_ARG;
  if (!is_pow2(c->head_dim) || c->head_dim < 8 || c->head_dim > 1024) return KVQ_ERR_INVALID_ARG;
  if (c->num_kv_heads <= 0 || c->num_layers <= 0 || c->num_pages < 0) return KVQ_ERR_INVALID_ARG;
  if (!is_pow2(c->tile_tokens) || c->tile_tokens < 8) return KVQ_ERR_INVALID_ARG;
  if (c->sinkhorn_iters < 0 || c->sinkhorn_iters > 1000) return KVQ_ERR_INVALID_ARG;
  if (!valid_bits(c->bits_k)) return KVQ_ERR_INVALID_ARG;
  if (!c->mla && !valid_bits(c->bits_v)) return KVQ_ERR_INVALID_ARG;
  if (c->in_dtype != KVQ_F16 && c->in_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
  if (c->meta_f16 != 0 && c->meta_f16 != 1) return KVQ_ERR_INVALID_ARG;
  if (c->k_per_channel != 0 && c->k_per_channel != 1) return KVQ_ERR_INVALID_ARG;
  // per-channel key groups are the ablation without normalisation (a row factor
  // could not be folded into per-channel scales)
  if (c->k_per_channel && (c->mla || c->sinkhorn_iters != 0)) return KVQ_ERR_INVALID_ARG;
  if (c->mla) {
    if (c->num_kv_heads != 1 || c->rope_dim < 0 || (c->rope_dim % 8)) return KVQ_ERR_INVALID_ARG;
  }
  if (!is_pow2(c->hadamard_block) || c->hadamard_block > c->head_dim) return KVQ_ERR_INVALID_ARG;
  // block-diagonal rotations (blocks of 1 .. head_dim channels) for K/V caches; the MLA latent full width
  if (c->mla && c->hadamard_block != c->head_dim) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

// Shapes the kernels are built for: head_dim 128 K/V caches with tiles of
// 16, 32, 64 or 128 tokens; a 512-wide MLA latent with 16-token tiles.
kvq_status check_gpu_shape(const kvq_config* c) {
  if (c->head_dim != (c->mla ? 512 : 128)) return KVQ_ERR_UNSUPPORTED;
  // per-channel keys and rotation blocks below 8 channels: 16-token tiles
  if ((c->k_per_channel || c->hadamard_block < 8) && c->tile_tokens != 16) return KVQ_ERR_UNSUPPORTED;
  if (c->k_per_channel && c->bits_k == 3) return KVQ_ERR_UNSUPPORTED;
  if (c->mla ? c->tile_tokens != 16 : (c->tile_tokens < 16 || c->tile_tokens > 128)) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

// 16-token decode tiles per page, as a power of two.
int sub_log2(const kvq_config* c) {
  int s = 0;
  while ((16 << s) < c->tile_tokens) ++s;
  return s;
}

// Shapes the decode kernels are built for (MLA: 512-channel latent, 64 rope).
kvq_status check_decode_shape(const kvq_config* c) {
  if (c->mla && c->rope_dim != 64) return KVQ_ERR_UNSUPPORTED;
  return check_gpu_shape(c);
}

int64_t slots(const kvq_config* c) { return (int64_t)c->num_layers * c->num_pages * c->num_kv_heads; }

CacheArrays arrays(const kvq_cache_view* v, int which, int bits) {
  CacheArrays a;
  a.codes = static_cast<uint8_t*>(which == 0 ? v->k_codes : v->v_codes);
  a.tok = which == 0 ? v->k_tok_scale : v->v_tok_scale;
  a.chan = which == 0 ? v->k_chan_scale : v->v_chan_scale;
  a.bits = bits;
  a.meta16 = 0;
  a.per_channel = 0;
  return a;
}

kvq_status check_view(const kvq_config* c, const kvq_cache_view* v) {
  if (!v) return KVQ_ERR_INVALID_ARG;
  const void* need[4] = {v->k_codes, v->k_tok_scale, v->k_chan_scale, nullptr};
  for (int i = 0; i < 3; ++i)
    if ((!need[i] && !(i == 2 && c->k_per_channel)) || !aligned16(need[i])) return KVQ_ERR_INVALID_ARG;
  if (!c->mla) {
    const void* vv[3] = {v->v_codes, v->v_tok_scale, v->v_chan_scale};
    for (int i = 0; i < 3; ++i)
      if (!vv[i] || !aligned16(vv[i])) return KVQ_ERR_INVALID_ARG;
  } else if (c->rope_dim > 0 && (!v->rope || !aligned16(v->rope))) {
    return KVQ_ERR_INVALID_ARG;
  }
  return KVQ_OK;
}

struct DecodePlan {
  int splits;
  int tiles_per_split;
};

// Split the tiles of each (sequence, kv-head) over CTAs.  kDecodeCtasPerSm
// CTAs fit on an SM at once, so the split count minimises, in sixteenths of
// a tile's time, (waves) x (tiles per warp + a fixed cost of about six tiles
// for the prologue and the merge of the CTA's warps) plus one sixteenth per
// split for its share of the combine (the split partials it reads).  Measured
// on one B200 for short contexts, a warp's tile costs ~1.5 us and a split
// ~0.1 us of the combine; at full-GPU sizes the waves term decides.
DecodePlan decode_plan(int64_t pairs, int64_t max_tiles) {
  DecodePlan d{1, 0};
  if (pairs <= 0 || max_tiles <= 0) return d;
  const int64_t slots = (int64_t)kDecodeCtasPerSm * num_sms();
  const int64_t cap = (max_tiles + kDecodeWarps - 1) / kDecodeWarps;  // at least one tile per warp
  int64_t best = 1, best_cost = INT64_MAX;
  for (int64_t s = 1; s <= cap && s <= 256; ++s) {
    const int64_t per_warp = (max_tiles + s * kDecodeWarps - 1) / (s * kDecodeWarps);
    const int64_t waves = (pairs * s + slots - 1) / slots;
    const int64_t cost = waves * 16 * (per_warp + 6) + s;
    if (cost < best_cost) best_cost = cost, best = s;
  }
  int64_t tps = (max_tiles + best - 1) / best;
  tps = (tps + kDecodeWarps - 1) / kDecodeWarps * kDecodeWarps;
  d.tiles_per_split = (int)tps;
  d.splits = (int)((max_tiles + tps - 1) / tps);
  return d;
}

size_t decode_ws_bytes(int64_t pairs, const DecodePlan& d, int head_dim) {
  return (size_t)pairs * d.splits * kMaxGroup * ((size_t)head_dim + 2) * sizeof(float);
}

// MLA: one CTA pair per (sequence, split), one CTA per SM, so (SMs / 2)
// pairs run at once.  The split count minimises (waves) x (32-token chunks
// per split + a fixed cost of about four chunks for the query fetch, the
// output write and the combine); a split has an even number of tiles.
constexpr int kMlaHeads = 128;
DecodePlan decode_plan_mla(int64_t batch, int64_t max_tiles) {
  DecodePlan d{1, 2};
  if (batch <= 0 || max_tiles <= 0) return d;
  const int64_t slots = num_sms() / 2, chunks = (max_tiles + 1) / 2;
  int64_t best = 1, best_cost = INT64_MAX;
  for (int64_t s = 1; s <= chunks && s <= 64; ++s) {
    const int64_t per = (chunks + s - 1) / s, waves = (batch * s + slots - 1) / slots;
    const int64_t cost = waves * (per + 4);
    if (cost < best_cost) best_cost = cost, best = s;
  }
  const int64_t tps = 2 * ((chunks + best - 1) / best);
  d.tiles_per_split = (int)tps;
  d.splits = (int)((max_tiles + tps - 1) / tps);
  return d;
}

size_t decode_ws_bytes_mla(int64_t batch, const DecodePlan& d) {
  return (size_t)batch * d.splits * kMlaHeads * (512 + 2) * sizeof(float) + mla_qprep_bytes(batch);
}

kvq_status cuda_status(int e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

// Quantise n_tok rows of `layers` consecutive layers, the first being
// `layer0`, into the cache (arguments already validated).  The rows are
// [layers][n_tok][H][d] (MLA rope [layers][n_tok][rope_dim]); the kernel
// sees a cache whose first layer is layer0.
kvq_status quantize_rows(const kvq_config* c, const kvq_cache_view* cache, const void* k_rows, const void* v_rows,
                         const void* rope_rows, int64_t n_tok, const int32_t* dst_page, uint32_t* dev_error,
                         int layers, int layer0, void* stream) {
  const size_t slot0 = (size_t)layer0 * c->num_pages * c->num_kv_heads;  // slots before layer0
  const size_t msz = c->meta_f16 ? 2 : 4, T = c->tile_tokens, d = c->head_dim;
  QuantizeParams p{};
  p.src[0] = k_rows;
  p.src[1] = v_rows;
  for (int kind = 0; kind < 2; ++kind) {
    p.dst[kind] = arrays(cache, kind, kind == 0 ? c->bits_k : c->bits_v);
    p.dst[kind].meta16 = c->meta_f16;
    const bool pc = kind == 0 && c->k_per_channel;
    p.dst[kind].per_channel = pc;
    if (p.dst[kind].codes) p.dst[kind].codes += slot0 * (T * d * p.dst[kind].bits / 8);
    if (p.dst[kind].tok) p.dst[kind].tok = static_cast<uint8_t*>(p.dst[kind].tok) + slot0 * (pc ? d * 2 : T * 2) * msz;
    if (p.dst[kind].chan && !pc) p.dst[kind].chan = static_cast<uint8_t*>(p.dst[kind].chan) + slot0 * d * msz;
  }
  p.kinds = c->mla ? 1 : 2;
  p.n_tok = n_tok;
  p.num_layers = layers;
  p.num_heads = c->num_kv_heads;
  p.num_pages = c->num_pages;
  p.iters = c->sinkhorn_iters;
  p.dst_page = dst_page;
  p.err = dev_error;
  p.total_tiles = (int64_t)p.kinds * layers * (n_tok / c->tile_tokens) * c->num_kv_heads;
  if (p.total_tiles >= (int64_t)1 << 31) return KVQ_ERR_UNSUPPORTED;  // tile ids are 32-bit in the kernel
  p.rope_src = (c->mla && c->rope_dim > 0) ? rope_rows : nullptr;
  p.rope_dst = cache->rope ? static_cast<uint8_t*>(cache->rope) + (size_t)layer0 * c->num_pages * T * c->rope_dim * 2
                           : nullptr;
  p.rope_dim = c->rope_dim;
  p.hblock = c->hadamard_block;
  return cuda_status(launch_quantize(p, c->in_dtype == KVQ_F16, c->head_dim, c->tile_tokens, stream));
}

}  // namespace

extern "C" {

const char* kvq_version(void) { return "0.1.0"; }

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "KVQ_OK";
    case KVQ_ERR_INVALID_ARG: return "KVQ_ERR_INVALID_ARG";
    case KVQ_ERR_UNSUPPORTED: return "KVQ_ERR_UNSUPPORTED";
    case KVQ_ERR_WORKSPACE_TOO_SMALL: return "KVQ_ERR_WORKSPACE_TOO_SMALL";
    case KVQ_ERR_PARTIAL_TILE: return "KVQ_ERR_PARTIAL_TILE";
    case KVQ_ERR_BAD_PAGE: return "KVQ_ERR_BAD_PAGE";
    case KVQ_ERR_TIMEOUT: return "KVQ_ERR_TIMEOUT";
    case KVQ_ERR_CUDA: return "KVQ_ERR_CUDA";
  }
  return "KVQ_ERR_UNKNOWN";
}

kvq_status kvq_config_from_string(const char* name, kvq_config* inout) {
  if (!name || !inout) return KVQ_ERR_INVALID_ARG;
  int k = 0, v = 0, g = 0;
  char tail = 0;
  if (std::sscanf(name, "kvarn_k%dv%d_g%d%c", &k, &v, &g, &tail) != 3) return KVQ_ERR_INVALID_ARG;
  if (!valid_bits(k) || !valid_bits(v) || !is_pow2(g) || g < 8) return KVQ_ERR_INVALID_ARG;
  inout->bits_k = k;
  inout->bits_v = v;
  inout->tile_tokens = g;
  return KVQ_OK;
}

kvq_status kvq_cache_layout(const kvq_config* c, size_t bytes_out[7]) {
  if (!bytes_out) return KVQ_ERR_INVALID_ARG;
  const kvq_status st = check_config(c);
  if (st != KVQ_OK) return st;
  const size_t n = (size_t)slots(c), T = c->tile_tokens, d = c->head_dim;
  const size_t msz = c->meta_f16 ? 2 : 4;  // bytes of one a, z or c
  bytes_out[0] = n * T * d * c->bits_k / 8;
  bytes_out[1] = c->k_per_channel ? n * d * 2 * msz : n * T * 2 * msz;  // (s, m) per channel, or (a, z) per token
  bytes_out[2] = c->k_per_channel ? 0 : n * d * msz;
  const bool has_v = !c->mla;
  bytes_out[3] = has_v ? n * T * d * c->bits_v / 8 : 0;
  bytes_out[4] = has_v ? n * T * 2 * msz : 0;
  bytes_out[5] = has_v ? n * d * msz : 0;
  bytes_out[6] = c->mla ? (size_t)c->num_layers * c->num_pages * T * c->rope_dim * 2 : 0;
  return KVQ_OK;
}

kvq_status kvq_quantize_append(const kvq_config* c, const kvq_cache_view* cache, const void* k_new,
                               const void* v_new, const void* rope_new, int64_t n_tok,
                               const int32_t* dst_page, uint32_t* dev_error, void* stream) {
  kvq_status st = check_config(c);
  if (st != KVQ_OK) return st;
  if ((st = check_view(c, cache)) != KVQ_OK) return st;
  if (n_tok < 0) return KVQ_ERR_INVALID_ARG;
  if (n_tok % c->tile_tokens) return KVQ_ERR_PARTIAL_TILE;
  if (n_tok > 0 && (!k_new || !dst_page || (!c->mla && !v_new))) return KVQ_ERR_INVALID_ARG;
  if (c->mla && c->rope_dim > 0 && n_tok > 0 && !rope_new) return KVQ_ERR_INVALID_ARG;
  if ((k_new && !aligned16(k_new)) || (v_new && !aligned16(v_new))) return KVQ_ERR_INVALID_ARG;
  if ((st = check_gpu_shape(c)) != KVQ_OK) return st;
  if (n_tok == 0) return KVQ_OK;
  if (c->mla && c->rope_dim > 0 && !aligned16(rope_new)) return KVQ_ERR_INVALID_ARG;
  return quantize_rows(c, cache, k_new, v_new, rope_new, n_tok, dst_page, dev_error, c->num_layers, 0, stream);
}

kvq_status kvq_dequantize(const kvq_config* c, const kvq_cache_view* cache, int32_t layer,
                          const int32_t* pages, int64_t n_pages, int32_t unrotate, float* k_out,
                          float* v_out, uint32_t* dev_error, void* stream) {
  kvq_status st = check_config(c);
  if (st != KVQ_OK) return st;
  if ((st = check_view(c, cache)) != KVQ_OK) return st;
  if (layer < 0 || layer >= c->num_layers || n_pages < 0) return KVQ_ERR_INVALID_ARG;
  if (n_pages > 0 && (!pages || !k_out || (!c->mla && !v_out))) return KVQ_ERR_INVALID_ARG;
  if ((st = check_gpu_shape(c)) != KVQ_OK) return st;
  if (n_pages == 0) return KVQ_OK;
  DequantParams p{};
  p.src[0] = arrays(cache, 0, c->bits_k);
  p.src[1] = arrays(cache, 1, c->bits_v);
  p.src[0].meta16 = p.src[1].meta16 = c->meta_f16;
  p.src[0].per_channel = c->k_per_channel;
  p.kinds = c->mla ? 1 : 2;
  p.layer = layer;
  p.num_heads = c->num_kv_heads;
  p.num_pages = c->num_pages;
  p.pages = pages;
  p.n_pages = n_pages;
  p.unrotate = unrotate ? 1 : 0;
  p.tile_tokens = c->tile_tokens;
  p.hblock = c->hadamard_block;
  p.out[0] = k_out;
  p.out[1] = v_out;
  p.err = dev_error;
  return cuda_status(launch_dequantize(p, c->head_dim, stream));
}

kvq_status kvq_decode_workspace_bytes(const kvq_config* c, int32_t batch, int32_t num_q_heads,
                                      int32_t max_seq_len, size_t* bytes) {
  kvq_status st = check_config(c);
  if (st != KVQ_OK) return st;
  if (!bytes || batch < 0 || num_q_heads <= 0 || max_seq_len < 0) return KVQ_ERR_INVALID_ARG;
  const int64_t pairs = (int64_t)batch * c->num_kv_heads;
  const int64_t max_tiles = ((int64_t)max_seq_len + c->tile_tokens - 1) / c->tile_tokens;
  const int nh = decode_kv_heads_per_cta(num_q_heads / c->num_kv_heads, c->num_kv_heads);
  *bytes = c->mla ? decode_ws_bytes_mla(batch, decode_plan_mla(batch, max_tiles))
                  : decode_ws_bytes(pairs, decode_plan(pairs / nh, max_tiles << sub_log2(c)), c->head_dim);
  return KVQ_OK;
}

}  // extern "C"

namespace {

// Decode attention over the cache, plus the unquantised tails when k_tail is
// given (GQA caches only).
kvq_status decode(const kvq_config* c, const kvq_cache_view* cache, int32_t layer, const void* q,
                  const int32_t* block_table, int32_t max_pages_per_seq, const int32_t* seq_lens,
                  const void* k_tail, const void* v_tail, const int32_t* tail_lens, int32_t batch,
                  int32_t num_q_heads, float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                  uint32_t* dev_error, void* stream, const int32_t* fill_page = nullptr) {
  kvq_status st = check_config(c);
  if (st != KVQ_OK) return st;
  if ((st = check_view(c, cache)) != KVQ_OK) return st;
  if (layer < 0 || layer >= c->num_layers || batch < 0 || max_pages_per_seq < 0 || num_q_heads <= 0)
    return KVQ_ERR_INVALID_ARG;
  if (num_q_heads % c->num_kv_heads) return KVQ_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return KVQ_ERR_INVALID_ARG;
  if (batch > 0 && (!q || !seq_lens || !out || (max_pages_per_seq > 0 && !block_table)))
    return KVQ_ERR_INVALID_ARG;
  if ((q && !aligned16(q)) || (out && !aligned16(out))) return KVQ_ERR_INVALID_ARG;  // both moved in 16-byte units
  if ((st = check_decode_shape(c)) != KVQ_OK) return st;
  if (c->mla) {
    if (num_q_heads > kMlaHeads) return KVQ_ERR_UNSUPPORTED;
    if (batch == 0) return KVQ_OK;
    if (batch > 65535) return KVQ_ERR_UNSUPPORTED;
    const DecodePlan plan = decode_plan_mla(batch, max_pages_per_seq);
    const size_t need = decode_ws_bytes_mla(batch, plan);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
      return workspace_bytes < need ? KVQ_ERR_WORKSPACE_TOO_SMALL : KVQ_ERR_INVALID_ARG;
    MlaDecodeParams m{};
    m.codes = static_cast<const uint8_t*>(cache->k_codes);
    m.tok = cache->k_tok_scale;
    m.chan = cache->k_chan_scale;
    m.meta16 = c->meta_f16;
    m.rope = static_cast<const uint16_t*>(cache->rope);
    m.bits = c->bits_k;
    m.layer = layer;
    m.num_pages = c->num_pages;
    m.q = static_cast<const uint16_t*>(q);
    m.block_table = block_table;
    m.max_pages = max_pages_per_seq;
    m.seq_lens = seq_lens;
    m.batch = batch;
    m.num_q_heads = num_q_heads;
    m.scale_log2 = softmax_scale * 1.4426950408889634f;
    m.out = out;
    m.part_o = static_cast<float*>(workspace);
    m.part_ml = m.part_o + (size_t)batch * plan.splits * kMlaHeads * 512;
    m.splits = plan.splits;
    m.tiles_per_split = plan.tiles_per_split;
    m.qprep = reinterpret_cast<uint8_t*>(m.part_ml + (size_t)batch * plan.splits * kMlaHeads * 2);
    m.err = dev_error;
    m.lat_tail = static_cast<const uint16_t*>(k_tail);  // latent rows; v_tail holds the rope keys
    m.rope_tail = static_cast<const uint16_t*>(v_tail);
    m.tail_lens = tail_lens;
    m.tail_f16 = c->in_dtype == KVQ_F16;
    m.tail_tokens = c->tile_tokens;
    return cuda_status(launch_decode_mla(m, stream));
  }
  const int group = num_q_heads / c->num_kv_heads;
  if (group > kMaxGroup || c->bits_v == 3) return KVQ_ERR_UNSUPPORTED;
  if (batch == 0) return KVQ_OK;
  const int64_t pairs = (int64_t)batch * c->num_kv_heads;
  // one CTA covers decode_kv_heads_per_cta adjacent kv-heads of a sequence
  const DecodePlan plan = decode_plan(pairs / decode_kv_heads_per_cta(group, c->num_kv_heads),
                                      (int64_t)max_pages_per_seq << sub_log2(c));
  const size_t need = decode_ws_bytes(pairs, plan, c->head_dim);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return workspace_bytes < need ? KVQ_ERR_WORKSPACE_TOO_SMALL : KVQ_ERR_INVALID_ARG;
  if (pairs > 65535) return KVQ_ERR_UNSUPPORTED;
  DecodeParams p{};
  p.k = arrays(cache, 0, c->bits_k);
  p.v = arrays(cache, 1, c->bits_v);
  p.k.meta16 = p.v.meta16 = c->meta_f16;
  p.k.per_channel = c->k_per_channel;
  p.layer = layer;
  p.num_kv_heads = c->num_kv_heads;
  p.num_pages = c->num_pages;
  p.q = static_cast<const uint16_t*>(q);
  p.block_table = block_table;
  p.max_pages = max_pages_per_seq;
  p.seq_lens = seq_lens;
  p.batch = batch;
  p.num_q_heads = num_q_heads;
  p.group = group;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.out = out;
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = p.part_o + (size_t)pairs * plan.splits * kMaxGroup * c->head_dim;
  p.splits = plan.splits;
  p.tiles_per_split = plan.tiles_per_split;
  p.sub_log2 = sub_log2(c);
  p.err = dev_error;
  p.k_tail = static_cast<const uint16_t*>(k_tail);
  p.v_tail = static_cast<const uint16_t*>(v_tail);
  p.tail_lens = tail_lens;
  p.tail_f16 = c->in_dtype == KVQ_F16;
  p.tail_tokens = c->tile_tokens;
  p.hblock = c->hadamard_block;
  p.test_wait_ns = g_test_wait_ns.load(std::memory_order_relaxed);
  p.fill_page = fill_page;
  return cuda_status(launch_decode_d128(p, stream));
}

}  // namespace

extern "C" {

kvq_status kvq_decode_attention(const kvq_config* c, const kvq_cache_view* cache, int32_t layer,
                                const void* q, const int32_t* block_table, int32_t max_pages_per_seq,
                                const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                                float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                                uint32_t* dev_error, void* stream) {
  return decode(c, cache, layer, q, block_table, max_pages_per_seq, seq_lens, nullptr, nullptr, nullptr, batch,
                num_q_heads, softmax_scale, out, workspace, workspace_bytes, dev_error, stream);
}

kvq_status kvq_decode_attention_tail(const kvq_config* c, const kvq_cache_view* cache, int32_t layer,
                                     const void* q, const int32_t* block_table, int32_t max_pages_per_seq,
                                     const int32_t* seq_lens, const void* k_tail, const void* v_tail,
                                     const int32_t* tail_lens, int32_t batch, int32_t num_q_heads,
                                     float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                                     uint32_t* dev_error, void* stream) {
  if (batch > 0 && (!k_tail || !v_tail || !tail_lens)) return KVQ_ERR_INVALID_ARG;
  if ((k_tail && !aligned16(k_tail)) || (v_tail && !aligned16(v_tail))) return KVQ_ERR_INVALID_ARG;
  if (c && c->tile_tokens > 128) return KVQ_ERR_UNSUPPORTED;
  return decode(c, cache, layer, q, block_table, max_pages_per_seq, seq_lens, batch > 0 ? k_tail : nullptr,
                v_tail, tail_lens, batch, num_q_heads, softmax_scale, out, workspace, workspace_bytes, dev_error,
                stream);
}

void kvq_set_test_wait(uint32_t ns) { g_test_wait_ns.store(ns, std::memory_order_relaxed); }

kvq_status kvq_decode_attention_fill(const kvq_config* c, const kvq_cache_view* cache, int32_t layer,
                                     const void* q, const int32_t* block_table, int32_t max_pages_per_seq,
                                     const int32_t* seq_lens, const void* k_tail, const void* v_tail,
                                     const int32_t* tail_lens, const int32_t* fill_page, int32_t batch,
                                     int32_t num_q_heads, float softmax_scale, float* out, void* workspace,
                                     size_t workspace_bytes, uint32_t* dev_error, void* stream) {
  kvq_status st = check_config(c);
  if (st != KVQ_OK) return st;
  if ((st = check_view(c, cache)) != KVQ_OK) return st;
  if (layer < 0 || layer >= c->num_layers || batch < 0) return KVQ_ERR_INVALID_ARG;
  if (batch > 0 && (!k_tail || !v_tail || !tail_lens || !fill_page)) return KVQ_ERR_INVALID_ARG;
  if ((k_tail && !aligned16(k_tail)) || (v_tail && !aligned16(v_tail))) return KVQ_ERR_INVALID_ARG;
  if (c->tile_tokens > 128) return KVQ_ERR_UNSUPPORTED;
  if ((st = check_decode_shape(c)) != KVQ_OK) return st;
  if (batch == 0) return KVQ_OK;
  // the decode's own checks (shapes, workspace) before anything is launched
  size_t need = 0;
  if ((st = kvq_decode_workspace_bytes(c, batch, num_q_heads, max_pages_per_seq * c->tile_tokens, &need)) != KVQ_OK)
    return st;
  if (workspace_bytes < need) return KVQ_ERR_WORKSPACE_TOO_SMALL;
  // 1) this layer's full tails into their pages: the rows of every sequence
  //    (fill_page[b] = -1 skips b), as one append of batch * T tokens
  const size_t row_elems = (size_t)c->tile_tokens * c->num_kv_heads * c->head_dim;  // one sequence's tail
  const uint8_t* kl = static_cast<const uint8_t*>(k_tail) + (size_t)layer * batch * row_elems * 2;
  const uint8_t* vl = static_cast<const uint8_t*>(v_tail) +
                      (size_t)layer * batch * (c->mla ? (size_t)c->tile_tokens * c->rope_dim : row_elems) * 2;
  st = quantize_rows(c, cache, kl, c->mla ? nullptr : vl, c->mla ? vl : nullptr, (int64_t)batch * c->tile_tokens,
                     fill_page, dev_error, 1, layer, stream);
  if (st != KVQ_OK) return st;
  // 2) attention over the cache (now holding the filled pages) and the remaining tails
  // (GQA: the decode overlaps the fill's quantize launch and waits for it
  // only where it reads a filled page)
  return decode(c, cache, layer, q, block_table, max_pages_per_seq, seq_lens, k_tail, v_tail, tail_lens, batch,
                num_q_heads, softmax_scale, out, workspace, workspace_bytes, dev_error, stream, fill_page);
}

kvq_status kvq_read_error(uint32_t* dev_error, uint32_t* host_bits, void* stream) {
  if (!dev_error || !host_bits) return KVQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t bits = 0;
  if (cudaMemcpyAsync(&bits, dev_error, sizeof(bits), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return KVQ_ERR_CUDA;
  if (cudaMemsetAsync(dev_error, 0, sizeof(uint32_t), s) != cudaSuccess) return KVQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KVQ_ERR_CUDA;
  *host_bits = bits;
  return (bits & KVQ_DEVERR_TIMEOUT) ? KVQ_ERR_TIMEOUT : KVQ_OK;
}

}  // extern "C"
