// Internal launch parameters shared by the host entry points and kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/kvq.h"

namespace kvq {

// 1/sqrt(b) for a power of two b, correctly rounded: 2^(-k/2) for b = 2^k,
// k even, else sqrt(2) (rounded once) times the power of two 2^(-(k+1)/2).
inline __host__ __device__ float inv_sqrt_pow2(int b) {
  int k = 0;
  while ((1 << k) < b) ++k;
  float r = (k & 1) ? 1.41421356237309505f : 1.0f;
  for (int i = 0; i < (k + 1) / 2; ++i) r *= 0.5f;
  return r;
}

// Every spin-wait in a kernel gives up after this many nanoseconds (1 s of
// GPU global time) and raises KVQ_DEVERR_TIMEOUT.
constexpr uint32_t kWaitLimit = 1000000000u;

// One quantised stream (K, V or the MLA latent) of the cache.
struct CacheArrays {
  uint8_t* codes;    // [layer][page][head][T*d*bits/8]
  void* tok;         // [layer][page][head][T][2]  float32, or half when meta16
  void* chan;        // [layer][page][head][d]     float32, or half when meta16
  int bits;
  int meta16;        // 1: a, z, c stored as IEEE half
  int per_channel;   // 1: one (s, m) pair per channel in `tok` ([d][2]); no `chan`
};

struct QuantizeParams {
  const void* src[2];   // K, V inputs [layer][n_tok][H][d]
  CacheArrays dst[2];
  int kinds;            // 1 (MLA latent only) or 2 (K and V)
  int64_t n_tok;
  int num_layers;
  int num_heads;
  int64_t num_pages;
  int iters;
  const int32_t* dst_page;
  uint32_t* err;
  int64_t total_tiles;  // kinds * layers * (n_tok / T) * heads
  const void* rope_src; // MLA rope keys [layer][n_tok][rope_dim] bf16, or null
  void* rope_dst;       // cache rope array [layer][page][T][rope_dim]
  int rope_dim;
  int hblock;           // Hadamard block: channels per diagonal block (head_dim = full width)
};

struct DequantParams {
  CacheArrays src[2];
  int kinds;
  int layer;
  int num_heads;
  int64_t num_pages;
  const int32_t* pages;
  int64_t n_pages;
  int unrotate;
  int tile_tokens;      // T: rows per page (a multiple of 16)
  int hblock;           // Hadamard block
  float* out[2];
  uint32_t* err;
};

struct DecodeParams {
  CacheArrays k, v;
  int layer;
  int num_kv_heads;
  int64_t num_pages;
  const uint16_t* q;            // bf16 [B][Hq][d]
  const int32_t* block_table;   // [B][max_pages]
  int max_pages;
  const int32_t* seq_lens;      // [B]
  int batch;
  int num_q_heads;
  int group;                    // Hq / Hkv (1..8)
  float scale_log2;             // softmax_scale * log2(e)
  float* out;                   // [B][Hq][d]
  float* part_o;                // [B*Hkv][splits][8][d]  un-normalised partial outputs
  float* part_ml;               // [B*Hkv][splits][8][2]  (max, sum) in log2 units
  int splits;
  int tiles_per_split;          // in 16-token sub-tiles
  int sub_log2;                 // log2(16-token sub-tiles per page): 0 for 16-token pages, 3 for 128
  uint32_t* err;
  // unquantised tail of each sequence (the newest tokens short of a whole
  // page), merged by the combine kernel; k_tail == nullptr: no tail
  const uint16_t* k_tail;       // [layers][B][T][Hkv][d], fp16 or bf16
  const uint16_t* v_tail;
  const int32_t* tail_lens;     // [B], 0..T
  int tail_f16;                 // 1: fp16 rows, 0: bf16
  int tail_tokens;              // T
  int hblock;                   // Hadamard block: 8 .. 128 channels
  uint32_t test_wait_ns;        // testing only: > 0 makes every CTA first wait this long on a flag nothing sets
  // quantise-on-fill: [B], the page the preceding quantize launch of the same
  // call writes for sequence b (-1: none); the decode is then launched as its
  // programmatic dependent and waits for that grid only before it copies a
  // filled page (and once before it exits); nullptr: an ordinary launch
  const int32_t* fill_page;
};

struct MlaDecodeParams {
  const uint8_t* codes;         // latent codes [layer][page][T*512*bits/8]
  const void* tok;              // [layer][page][T][2]  float32, or half when meta16
  const void* chan;             // [layer][page][512]   float32, or half when meta16
  int meta16;
  const uint16_t* rope;         // bf16 [layer][page][T][64]
  int bits;
  int layer;
  int64_t num_pages;
  const uint16_t* q;            // bf16 [B][Hq][576]
  const int32_t* block_table;   // [B][max_pages]
  int max_pages;
  const int32_t* seq_lens;      // [B]
  int batch;
  int num_q_heads;              // <= 128
  float scale_log2;
  float* out;                   // [B][Hq][512]
  float* part_o;                // [B][splits][128][512]
  float* part_ml;               // [B][splits][128][2]
  int splits;
  int tiles_per_split;          // even
  uint8_t* qprep;               // [B][2][128 x 288 f16]: rotated queries in the score-operand layout
  uint32_t* err;
  // unquantised tail of each sequence, merged by the combine kernel;
  // lat_tail == nullptr: no tail
  const uint16_t* lat_tail;     // [layers][B][T][512], fp16 or bf16
  const uint16_t* rope_tail;    // [layers][B][T][64] bf16
  const int32_t* tail_lens;     // [B], 0..T
  int tail_f16;                 // 1: fp16 latent rows, 0: bf16
  int tail_tokens;              // T
};

// Launchers (defined in the .cu files); return a cudaError_t value.
int launch_quantize(const QuantizeParams& p, bool f16, int head_dim, int tile_tokens, void* stream);
int launch_dequantize(const DequantParams& p, int head_dim, void* stream);
int launch_decode_d128(const DecodeParams& p, void* stream);
// kv-heads one GQA decode CTA covers (2 for groups of at most 4 query heads)
int decode_kv_heads_per_cta(int group, int num_kv_heads);
int launch_decode_mla(const MlaDecodeParams& p, void* stream);
size_t mla_qprep_bytes(int64_t batch);  // workspace for the prepared MLA queries

}  // namespace kvq
