/*
 * kvq.h -- C ABI of a B200 (sm_100a) library for KVarN-style variance-
 * normalised KV-cache quantisation and decode attention over the quantised
 * cache.
 *
 * Method (what every call computes), as the KVarN pages state it:
 *   - KVarN project page (open-radar), Key Features, "Variance-Normalized
 *     Quantization Pipeline": each tile of the KV cache is rotated with a
 *     Hadamard transform to spread channel outliers, its variance is
 *     equalised by an iterative Sinkhorn-like normalisation, and it is then
 *     quantised with asymmetric round-to-nearest;
 *   - same page, "Calibration-Free Operation": the statistics are computed
 *     per tile on the fly;
 *   - same page, "4-bit Keys, 2-bit Values Preset": keys and values have
 *     their own bit widths and a tile is one cache block of the serving
 *     engine ("kvarn_k4v2_g128" = 4-bit K, 2-bit V, 128-token tiles);
 *   - same page, "MLA Model Support": the compressed latent of multi-head
 *     latent attention is quantised the same way;
 *   - KV-Cache tag page (baguaai.com), KVarN item: Hadamard rotation with
 *     dual-axis variance normalisation, round-to-nearest.
 *
 * Declared readings where the pages are silent (tile = T tokens x d
 * channels of one layer and kv-head; K and V quantised independently):
 *   Z = X H / sqrt(d)  (Sylvester H, full head_dim);
 *   n rounds of: divide each row by its root-mean-square, then each column
 *   by its root-mean-square (a zero RMS leaves its row/column alone); the
 *   factors accumulate in r (per token) and c (per channel);
 *   per token row of Y = Z / (r c): m = min, s = (max - min) / (2^b - 1),
 *   q = rint((Y - m) / s) (ties to even; s = 0 -> q = 0);
 *   stored: codes q, a = r*s and z = r*m (float32 per token), c (float32
 *   per channel).  Dequantised rotated value: (a q + z) c.
 *   Decode attention rotates the query by the same H/sqrt(d), attends in the
 *   rotated domain with the scales folded into the dot products, and rotates
 *   the output back.
 *
 * Ownership and threading: the caller allocates ALL device memory (the
 * cache arrays, inputs, outputs, the decode workspace and the device error
 * word).  The library never allocates, frees or synchronises, except
 * kvq_read_error, which synchronises the given stream.  Every call that
 * takes a stream only enqueues work on it (a cudaStream_t passed as void*;
 * NULL = the legacy default stream) and returns.  Calls are thread-safe,
 * and the work they enqueue can be captured into a CUDA graph.  Within a
 * call, a kernel may be enqueued as the programmatic dependent of the one
 * before it (CUDA's programmatic dependent launch); a call's last kernel
 * completes only after all of the call's kernels.  The library's kernels
 * also let a dependent start early: a kernel the caller enqueues right
 * after a call with programmatic stream serialisation must wait for its
 * prerequisite grid (cudaGridDependencySynchronize) before it reads the
 * call's results.
 *
 * Errors: every function returns kvq_status; nothing is thrown across the
 * ABI.  Host-detectable problems (null pointers, unsupported shapes or bit
 * widths, a workspace that is too small) are rejected before any launch.
 * Problems only the device can see (a page id outside [0, num_pages), a
 * sequence length that is not a multiple of the tile) set bits in the
 * caller's 32-bit device error word (KVQ_DEVERR_*); the affected tile is
 * skipped and nothing traps.  Read and clear it with kvq_read_error.
 *
 * Cache format (all arrays indexed [layer][page][kv_head][...], one page =
 * one tile of T tokens):
 *   codes:      T * d * bits / 8 bytes per (layer, page, head): token rows in
 *               order, each row's codes packed little-endian inside a byte,
 *               lowest channel in the lowest bits (2, 4 or 8 bits); 3-bit
 *               codes are a plane of all rows' low 2 bits (2-bit packing)
 *               followed by a plane of all rows' high bits (1-bit packing);
 *   tok_scale:  [T][2] = (a, z) per token;
 *   chan_scale: [d] = c per channel;
 *               both float32, or IEEE half when meta_f16 = 1; each tile's
 *               scales are balanced by a power of two so that max c lies in
 *               (1/2, 1] (the dequantised tile does not change);
 *   keys with k_per_channel = 1: k_tok_scale holds [d][2] = (s, m) per
 *               channel, the step and minimum of the channel's T rotated
 *               values, and k_chan_scale is unused (size 0, may be NULL);
 *               dequantised rotated value s q + m;
 *   rope (MLA): bf16 [layer][page][T][rope_dim], unquantised.
 *
 * Supported on the GPU: head_dim 128 (GQA) with tile_tokens 16, 32, 64 or
 * 128 (the shipped "4-bit Keys, 2-bit Values Preset" uses 128), or 512 (MLA
 * latent) with tile_tokens 16; bits_k in {2,3,4,8}, bits_v in {2,4,8}, query
 * group size 1..8 for GQA and 1..128 heads for MLA; inputs fp16 or bf16;
 * rotation blocks 1 (no rotation) .. head_dim for K/V caches; per-channel
 * keys with 2-, 4- or 8-bit codes at tile_tokens 16.
 * Other shapes return KVQ_ERR_UNSUPPORTED.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kvq_status {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,         /* null pointer, negative size, inconsistent config */
  KVQ_ERR_UNSUPPORTED = 2,         /* valid but not built: head_dim, bits, tile, group size */
  KVQ_ERR_WORKSPACE_TOO_SMALL = 3, /* decode workspace below kvq_decode_workspace_bytes */
  KVQ_ERR_PARTIAL_TILE = 4,        /* n_tok not a multiple of tile_tokens */
  KVQ_ERR_BAD_PAGE = 5,            /* reserved for host-side page checks */
  KVQ_ERR_TIMEOUT = 6,             /* a bounded device wait gave up (see KVQ_DEVERR_TIMEOUT) */
  KVQ_ERR_CUDA = 7                 /* a CUDA runtime call failed (launch or sync) */
} kvq_status;

/* Bits of the device error word. */
#define KVQ_DEVERR_BAD_PAGE 0x1u     /* page id < 0 or >= num_pages: tile skipped */
#define KVQ_DEVERR_PARTIAL_TILE 0x2u /* seq_len % tile_tokens != 0: tail ignored */
#define KVQ_DEVERR_TIMEOUT 0x4u      /* an mbarrier wait ran out of iterations */
#define KVQ_DEVERR_BAD_SEQ 0x8u      /* seq_len < 0 or needs more pages than the block table row */

typedef enum kvq_dtype { KVQ_F16 = 0, KVQ_BF16 = 1, KVQ_F32 = 2 } kvq_dtype;

/* One cache (all layers share it).  Fill it yourself or with
 * kvq_config_from_string. */
typedef struct kvq_config {
  int32_t head_dim;       /* d: 128 (GQA) or 512 (MLA latent); power of two */
  int32_t num_kv_heads;   /* H_kv (1 for MLA) */
  int32_t tile_tokens;    /* T == page size in tokens (16; 32, 64, 128 at head_dim 128) */
  int32_t bits_k;         /* key (MLA: latent) code width: 2, 3, 4 or 8 */
  int32_t bits_v;         /* value code width: 2, 4 or 8; ignored when mla */
  int32_t sinkhorn_iters; /* n >= 0 normalisation rounds (0 = rotation + RTN only) */
  int32_t hadamard_block; /* channels per block of the rotation: head_dim = the full
                           * Sylvester rotation; 1..head_dim/2 (K/V caches only) = a
                           * block-diagonal rotation of consecutive channels (the
                           * SAW-INT4 entry on the Hugging Face paper listing);
                           * 1 = no rotation */
  int32_t mla;            /* 1: one latent per token is key and value; no V arrays */
  int32_t rope_dim;       /* MLA: width of the unquantised bf16 rope key (64) */
  int32_t num_layers;     /* layers in the pool */
  int64_t num_pages;      /* pages per layer in the pool */
  kvq_dtype in_dtype;     /* dtype of the new K/V rows: KVQ_F16 or KVQ_BF16 */
  int32_t meta_f16;       /* metadata format of a, z and c: 0 = float32 (a
                           * zero-filled config gets it), 1 = IEEE half
                           * (the compact layout: same codes, scales rounded
                           * to 11 significant bits; rows must stay within the
                           * half range, |a|, |z| < 65504) */
  int32_t k_per_channel;  /* key quantisation axis: 0 = per token (KVarN; a
                           * zero-filled config gets it), 1 = per channel
                           * (the KIVI-style axes ablation: each channel's T
                           * tokens are one RTN group; needs sinkhorn_iters = 0;
                           * head_dim 128, tile_tokens 16).  Values stay per token */
} kvq_config;

/* Caller-owned device arrays of one cache; byte sizes from kvq_cache_layout
 * (in this order: k_codes, k_tok_scale, k_chan_scale, v_codes, v_tok_scale,
 * v_chan_scale, rope).  Unused arrays (V when mla, rope when not) may be
 * NULL.  Every pointer must be 16-byte aligned. */
typedef struct kvq_cache_view {
  void* k_codes;
  void* k_tok_scale;
  void* k_chan_scale;
  void* v_codes;
  void* v_tok_scale;
  void* v_chan_scale;
  void* rope;
} kvq_cache_view;

/* Parse a KVarN preset name "kvarn_k<K>v<V>_g<T>" (KVarN project page,
 * "Native vLLM Integration" and "4-bit Keys, 2-bit Values Preset") into
 * bits_k, bits_v and tile_tokens of *inout; the other fields are left as
 * they are.  KVQ_ERR_INVALID_ARG if the string does not parse. */
kvq_status kvq_config_from_string(const char* name, kvq_config* inout);

/* Byte sizes of the seven cache arrays for *cfg (0 for unused arrays).
 * Host only. */
kvq_status kvq_cache_layout(const kvq_config* cfg, size_t bytes_out[7]);

/* Quantise n_tok new tokens of every layer into the paged cache (the
 * whole pipeline: rotation, dual-axis normalisation, asymmetric RTN,
 * packing).
 *   k_new, v_new: device, in_dtype [num_layers][n_tok][num_kv_heads][head_dim]
 *                 (MLA: k_new is the latent [num_layers][n_tok][1][d];
 *                 v_new is ignored and may be NULL);
 *   rope_new:     MLA only, device bf16 [num_layers][n_tok][rope_dim],
 *                 copied into the rope array; NULL otherwise;
 *   n_tok:        tokens per layer, a multiple of tile_tokens
 *                 (else KVQ_ERR_PARTIAL_TILE);
 *   dst_page:     device int32 [n_tok / tile_tokens]: the page that receives
 *                 tokens [i*T, (i+1)*T) of every layer and kv-head; -1
 *                 skips that tile (no error: quantise-on-fill passes a
 *                 whole tail buffer and skips the tails that are not full);
 *                 any other id outside [0, num_pages) sets
 *                 KVQ_DEVERR_BAD_PAGE and that tile is not written;
 *   dev_error:    device uint32 error word (bits are OR-ed in).
 * Pages must be distinct within one call. */
kvq_status kvq_quantize_append(const kvq_config* cfg, const kvq_cache_view* cache,
                               const void* k_new, const void* v_new, const void* rope_new,
                               int64_t n_tok, const int32_t* dst_page, uint32_t* dev_error,
                               void* stream);

/* Dequantise n_pages pages of one layer to float32 (inspection and tests).
 *   pages:  device int32 [n_pages]; out-of-range ids set KVQ_DEVERR_BAD_PAGE
 *           and their output is left untouched;
 *   unrotate: 0 = rotated domain (a q + z) c; 1 = rotated back to the
 *           input basis;
 *   k_out, v_out: device float32 [n_pages][num_kv_heads][T][head_dim]
 *           (v_out ignored when mla). */
kvq_status kvq_dequantize(const kvq_config* cfg, const kvq_cache_view* cache, int32_t layer,
                          const int32_t* pages, int64_t n_pages, int32_t unrotate,
                          float* k_out, float* v_out, uint32_t* dev_error, void* stream);

/* Bytes of device workspace kvq_decode_attention needs for this shape
 * (split-KV partial results).  Host only. */
kvq_status kvq_decode_workspace_bytes(const kvq_config* cfg, int32_t batch,
                                      int32_t num_q_heads, int32_t max_seq_len,
                                      size_t* bytes);

/* One decode step of attention over the quantised cache of one layer.
 *   q:           device bf16 [batch][num_q_heads][head_dim (+ rope_dim if mla)],
 *                un-rotated;
 *   block_table: device int32 [batch][max_pages_per_seq], pages in token order;
 *   seq_lens:    device int32 [batch], multiples of tile_tokens (a remainder
 *                sets KVQ_DEVERR_PARTIAL_TILE and is ignored);
 *   num_q_heads: a multiple of num_kv_heads; q head h reads kv-head
 *                h / (num_q_heads / num_kv_heads);
 *   softmax_scale: multiplies q.k (1/sqrt(128) for GQA, 1/sqrt(576) for MLA);
 *   out:         device float32 [batch][num_q_heads][head_dim], un-rotated,
 *                16-byte aligned; a sequence of length 0 gets zeros;
 *   workspace:   device scratch of at least kvq_decode_workspace_bytes(...,
 *                max_seq_len >= every seq_len) bytes, 256-byte aligned; its
 *                contents need no initialisation and are overwritten. */
kvq_status kvq_decode_attention(const kvq_config* cfg, const kvq_cache_view* cache, int32_t layer,
                                const void* q, const int32_t* block_table,
                                int32_t max_pages_per_seq, const int32_t* seq_lens,
                                int32_t batch, int32_t num_q_heads, float softmax_scale,
                                float* out, void* workspace, size_t workspace_bytes,
                                uint32_t* dev_error, void* stream);

/* kvq_decode_attention for sequences whose newest tokens do not fill a page
 * yet.  The KVarN pages are silent on partial tiles; here the last
 * tail_lens[b] < T tokens of sequence b stay unquantised in a tail buffer
 * and attention runs over its cached tokens and its tail together (a tail
 * token is scored with q . k and weighted by its value row as is; the
 * result is the softmax over all of the sequence's keys).
 *   k_tail, v_tail: device, 16-byte aligned, [num_layers][batch]
 *                [tile_tokens][num_kv_heads][head_dim] in in_dtype: rows 0 ..
 *                tail_lens[b] - 1 of sequence b are its tail in this layer;
 *                the same layout as kvq_quantize_append's input with
 *                n_tok = batch * tile_tokens, so full tails are quantised in
 *                one append call (dst_page[b] = -1 skips the others).
 *                MLA caches: k_tail holds the latent rows [num_layers]
 *                [batch][tile_tokens][head_dim] in in_dtype and v_tail the
 *                rope keys [num_layers][batch][tile_tokens][rope_dim] bf16;
 *   tail_lens:   device int32 [batch], 0 .. tile_tokens (a value outside
 *                sets KVQ_DEVERR_BAD_SEQ and the tail is ignored);
 * the other arguments and the workspace are those of kvq_decode_attention.
 * Tiles longer than 128 tokens return KVQ_ERR_UNSUPPORTED. */
kvq_status kvq_decode_attention_tail(const kvq_config* cfg, const kvq_cache_view* cache, int32_t layer,
                                     const void* q, const int32_t* block_table,
                                     int32_t max_pages_per_seq, const int32_t* seq_lens,
                                     const void* k_tail, const void* v_tail, const int32_t* tail_lens,
                                     int32_t batch, int32_t num_q_heads, float softmax_scale,
                                     float* out, void* workspace, size_t workspace_bytes,
                                     uint32_t* dev_error, void* stream);

/* One decode step with quantise-on-fill: for every sequence b with
 * fill_page[b] >= 0, the full tail of this layer (all tile_tokens rows of
 * k_tail / v_tail for b) is first quantised into page fill_page[b] of this
 * layer, exactly as kvq_quantize_append would; then attention runs over the
 * cached pages and the remaining tails as in kvq_decode_attention_tail.
 * Both steps are enqueued on `stream` in that order by this one call.  For
 * K/V caches the attention kernel is enqueued as the programmatic dependent
 * of the fill's quantize launch, so the two overlap: a CTA waits for the
 * fill only before it reads a page of fill_page (the call's result is the
 * same as with the steps run one after the other, and the call completes
 * after both).
 * (The pages are silent on tokens short of a tile; this is the serving
 * reading of the unquantised tail: a tail is quantised when it fills.)
 *   fill_page:   device int32 [batch]: the page that receives b's full tail,
 *                or -1 (no fill); pages must be distinct and outside what
 *                other calls are reading, and in this call fill_page[b]
 *                appears in no block-table row but b's;
 * the caller describes the state after the fill: block_table row b already
 * ends with fill_page[b], seq_lens[b] counts it, and tail_lens[b] = 0 for a
 * filled sequence (its tail buffer rows are read by the fill only).  The
 * other arguments are those of kvq_decode_attention_tail. */
kvq_status kvq_decode_attention_fill(const kvq_config* cfg, const kvq_cache_view* cache, int32_t layer,
                                     const void* q, const int32_t* block_table,
                                     int32_t max_pages_per_seq, const int32_t* seq_lens,
                                     const void* k_tail, const void* v_tail, const int32_t* tail_lens,
                                     const int32_t* fill_page, int32_t batch, int32_t num_q_heads,
                                     float softmax_scale, float* out, void* workspace,
                                     size_t workspace_bytes, uint32_t* dev_error, void* stream);

/* kvq_decode_attention for callers that cannot allocate device memory when
 * they decode (a plug-in whose host process owns all device allocations and
 * has no scratch hook, or a deployment that forbids allocation after
 * start-up).  The KVarN pages have no counterpart; this is a deployment
 * variant of the call above with the same arguments except the workspace.
 *
 * The split-KV partial results live in one fixed 8 MiB array of this
 * library (every GPU that loads the library holds it until the process
 * exits); nothing is allocated.  Shapes that need more than 8 MiB (see
 * kvq_decode_workspace_bytes with max_seq_len = max_pages_per_seq *
 * tile_tokens) return KVQ_ERR_WORKSPACE_TOO_SMALL before any launch.
 * The first call on a device looks up the array's address on that device
 * and keeps it, so make that first call before any stream capture.  A
 * device reset (cudaDeviceReset) invalidates the kept address: do not call
 * this entry point again after one.  A call that fails with KVQ_ERR_CUDA
 * drops the kept address, and the next call looks it up again.  Sizes are
 * checked after every other argument: KVQ_ERR_WORKSPACE_TOO_SMALL means the
 * call was otherwise valid.  All calls share the
 * array and it keeps the last call's contents (nothing in it needs to start
 * at zero): calls that overlap on the GPU, on any streams of the process,
 * race and give wrong results; serialise them. */
kvq_status kvq_decode_attention_noalloc(const kvq_config* cfg, const kvq_cache_view* cache,
                                        int32_t layer, const void* q, const int32_t* block_table,
                                        int32_t max_pages_per_seq, const int32_t* seq_lens,
                                        int32_t batch, int32_t num_q_heads, float softmax_scale,
                                        float* out, uint32_t* dev_error, void* stream);

/* Testing hook for the failure path of the bounded device waits (the pages
 * have no counterpart).  With ns > 0, every CTA of each later GQA decode
 * call (kvq_decode_attention and its variants) first waits, for at most ns
 * nanoseconds of GPU time, on a device flag that nothing ever sets.  The
 * wait runs out before the CTA issues any copy: the CTA sets
 * KVQ_DEVERR_TIMEOUT, skips its tiles and returns, so the call ends with
 * zeros in place of the attention output and kvq_read_error reports
 * KVQ_ERR_TIMEOUT.  ns = 0 (the default) turns the hook off.  Process-wide;
 * affects only calls made after it. */
void kvq_set_test_wait(uint32_t ns);

/* Synchronise `stream`, copy the device error word to *host_bits and reset
 * it to 0.  KVQ_ERR_TIMEOUT if the TIMEOUT bit was set, else KVQ_OK (other
 * bits are only reported in *host_bits). */
kvq_status kvq_read_error(uint32_t* dev_error, uint32_t* host_bits, void* stream);

/* Static, human-readable name of a status. */
const char* kvq_status_string(kvq_status status);

/* Library version as "major.minor.patch". */
const char* kvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
