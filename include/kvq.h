/*
 * kvq.h -- C ABI of libkvq: decode attention over a KV cache whose precision
 * pair (key bits, value bits) is set per layer by an offline-searched layer map.
 *
 * The method is KVTuner ("KVTuner: Sensitivity-Aware Layer-wise Mixed Precision
 * KV Cache Quantization", arXiv 2502.04420). The pages this library follows:
 *   [facts]  llms-explorer.com, "Mixed-precision KV-cache quantization
 *            per-layer sensitivity" -- facts list (per-layer pairs applied at
 *            inference with no online decision; keys per-channel asymmetric,
 *            values per-token asymmetric; 3.25-bit / 4.0-bit maps).
 *   [abs]    mlsanity.com, arXiv 2502.04420 abstract (layer-wise precision pairs,
 *            offline-searched configurations used during online inference).
 *   [qa]     machinoai.in Q&A on mixed BF16/FP8 KV, section 2 (byte accounting,
 *            sensitive layers kept in BF16).
 *   [rebut]  paperhub.cn OpenReview rebuttal: "Computational cost" (only newly
 *            generated tokens are quantized online), "Baseline Implementation"
 *            (FlashAttention-style decode kernels over int8 / mixed K-V
 *            precision), "New GQA efficiency results" (GQA), and the per-layer
 *            K4V8 facts for layers 0, 1, 2, 31 of Llama-3.1-8B-Instruct.
 *
 * Fixed by this library where the pages are silent: key groups of 32 tokens
 * (one fp16 scale and zero per channel per group), one fp16 scale and zero per
 * value token, and a bf16 window holding the most recent (T mod 32) tokens that
 * are not yet quantized.
 *
 * Conventions for every call:
 *  - Device pointers are plain CUDA device addresses (e.g. a torch tensor's
 *    data_ptr()); `stream` is a cudaStream_t passed as void* (NULL = legacy
 *    default stream). Calls only enqueue work: none synchronises the device
 *    except kvq_export_layer and kvq_sync.
 *  - The caller owns Q, K, V, out and the stream. The library owns the cache
 *    metadata and, unless a device pool is passed to kvq_cache_create, the
 *    device memory of the cache.
 *  - Errors are returned as kvq_status; no exception crosses the ABI. Invalid
 *    arguments and capacity overflow are detected on the host before any launch
 *    and leave the cache unchanged. kvq_last_error() gives a message for the
 *    last failing call on the calling thread.
 *  - Sequence lengths are mirrored on the host; no call reads them back.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct kvq_cache kvq_cache;

/* Key quantization mode of a layer ([rebut] section 4 "Per-channel vs.
 * per-token quantization"; [facts]: per-channel asymmetric keys beat per-token
 * asymmetric keys on channel-outlier keys, and the Pareto-optimal pairs differ
 * between the two modes). */
typedef enum {
  KVQ_KEY_PER_CHANNEL = 0, /* one scale/zero per key channel over each 32-token group (KIVI-like) */
  KVQ_KEY_PER_TOKEN = 1    /* one scale/zero per key token over head_dim (per-token-asym) */
} kvq_key_mode;

/* Element format of a layer's pages. */
typedef enum {
  KVQ_FMT_INT = 0, /* asymmetric integer codes with fp16 scale/zero in every page */
  KVQ_FMT_FP8 = 1  /* fp8 e4m3 elements, x / s_h rounded to nearest even and saturated
                      at 448, with per-KV-head fp32 key and value scales s_h
                      ([facts]: vLLM FP8 KV cache with per-attention-head scales;
                      [qa] section 2: BF16 and FP8 layers); k_bits = v_bits = 8 */
} kvq_format;

/* One layer's precision pair: k_bits, v_bits in {2, 4, 8}, or {16, 16} for a
 * layer kept in bf16 ([qa] section 2: sensitive layers stay BF16; [facts]:
 * vLLM-style skip layers). Mixed bf16/int pairs are rejected. key_mode is a
 * kvq_key_mode and format a kvq_format; both must be 0 for a bf16 layer, and
 * an fp8 layer is (8, 8, KVQ_KEY_PER_CHANNEL, KVQ_FMT_FP8). A zero-initialised
 * pair field means per-channel integer keys. */
typedef struct {
  uint8_t k_bits;
  uint8_t v_bits;
  uint8_t key_mode;
  uint8_t format;
} kvq_pair;

typedef enum {
  KVQ_OK = 0,
  KVQ_EINVAL = 1,    /* bad argument: null/misaligned pointer, bad layer, bad pair, bad shape */
  KVQ_ECAPACITY = 2, /* append would exceed max_tokens or max_batch */
  KVQ_ENOMEM = 3,    /* device allocation failed or the given pool is too small */
  KVQ_ECUDA = 4      /* a CUDA call failed (message in kvq_last_error) */
} kvq_status;

typedef enum {
  KVQ_BF16 = 0, /* bfloat16 */
  KVQ_F32 = 1   /* float32; rounded to bf16 (round-to-nearest-even) on entry */
} kvq_dtype;

/*
 * Storage format (per layer, per sequence b, per KV head h).
 * Tokens [0, 32*floor(T/32)) live in full 32-token pages; the remaining
 * W = T mod 32 tokens live in a bf16 window [2][32][head_dim] (keys, values;
 * row = slot = token mod 32). A page is 16-byte aligned and holds
 *   quantized pair: [K codes 4*D*k_bits B][V codes 4*D*v_bits B]
 *                   [K scale D x fp16][K zero D x fp16][V scale 32 x fp16][V zero 32 x fp16]
 *   per-token keys: [K codes][V codes][K scale 32 x fp16][K zero 32 x fp16][V scale][V zero]
 *                   (key scales and zeros in token order, like the values')
 *   fp8 layer:      [K e4m3 32*D B][V e4m3 32*D B] (8-bit tile layout, scales per KV head
 *                   held by the cache, see kvq_set_fp8_scales)
 *   bf16 layer:     [K 64*D B][V 64*D B]
 * Code blocks are stored as 16x16 tiles f = 2*dt + tt (dt: 16-channel tile,
 * tt: 16-token tile) laid out so that lane l = 4g + t of a warp reads its eight
 * elements of every tile as contiguous 16-byte vectors: element e = 2p + j of
 * tile f sits at row g + 8*(p & 1), column 2t + j + 8*(p >> 1), rows being
 * tokens for keys and channels for values. Lane word w of lane l lives at byte
 * ((w/4)*32 + l)*16 + (w%4)*4; 8-bit tiles take two words (element e in byte e),
 * 4-bit tiles one word (nibble (e>>1) + 4*(e&1)), two 2-bit tiles share a word
 * (slot 4u + (e>>1) + 8*(e&1) for tile 2w+u), bf16 tiles four words (half e).
 * Key scale/zero entry i (per-channel keys) holds channel 16*dt + 2t + (j&1) +
 * 8*(j>>1) with t = i/(D/4), dt = (i%(D/4))/4, j = i%4.
 */

/* Bytes of one 32-token page of `pair` at head_dim D (0 if invalid). */
int64_t kvq_page_bytes(kvq_pair pair, int head_dim);

/* Equivalent bitwidth of a layer map: the mean over layers of
 * (k_bits + v_bits)/2, bf16 layers counting 16 ([facts], [abs]: 3.25-bit and
 * 4.0-bit maps). Scales and zero points are not counted. Returns -1.0 on an
 * invalid map. Host only, pure. */
double kvq_equiv_bits(const kvq_pair* layer_map, int n_layers);

/* Device bytes kvq_cache_create needs for these dimensions (0 if invalid).
 * Use it to size a caller-owned pool. */
size_t kvq_cache_pool_bytes(const kvq_pair* layer_map, int n_layers, int n_q_heads, int n_kv_heads,
                            int head_dim, int max_batch, int64_t max_tokens);

/* Create a cache for `n_layers` layers with the given per-layer pairs
 * ([facts]: the per-layer configuration is searched offline and applied at
 * inference with no online decision). n_q_heads must be a multiple of
 * n_kv_heads with n_q_heads/n_kv_heads in [1, 8] (GQA, [rebut] "New GQA
 * efficiency results"); head_dim in {64, 128}; max_batch in [1, 1024];
 * max_tokens >= 1 per sequence.
 * device_pool/pool_bytes: a caller-owned, 256-byte-aligned device buffer of at
 * least kvq_cache_pool_bytes(...) bytes, or NULL/0 for the library to allocate
 * with cudaMalloc. Uses the current CUDA device. The new cache holds empty
 * sequences. On error *out is set to NULL. */
kvq_status kvq_cache_create(const kvq_pair* layer_map, int n_layers, int n_q_heads, int n_kv_heads,
                            int head_dim, int max_batch, int64_t max_tokens, void* device_pool,
                            size_t pool_bytes, kvq_cache** out);

/* Release the cache (synchronises the device first). NULL is a no-op. */
void kvq_cache_destroy(kvq_cache* cache);

/* Empty every sequence of every layer and zero the error reports (enqueued on
 * `stream`). */
kvq_status kvq_cache_reset(kvq_cache* cache, void* stream);

/* Append n_new[b] tokens to sequence b of `layer`, for b < batch ([rebut]
 * "Computational cost": only the newly generated keys and values are quantized
 * online, with the layer's calibrated pair).
 *   K, V: device, [sum(n_new), n_kv_heads, head_dim] in `dtype`, sequences packed
 *         in order b = 0..batch-1, 16-byte aligned.
 *   n_new: host array [batch], each >= 0.
 * Tokens enter the bf16 window; every time a sequence's window reaches 32
 * tokens they are quantized as one group -- keys per channel over the 32
 * tokens (per token over head_dim in a KVQ_KEY_PER_TOKEN layer), values per
 * token over head_dim ([facts]: per-channel asymmetric keys, per-token
 * asymmetric values) -- bit-packed into the next page, and the window
 * is emptied. The stored result does not depend on how tokens are split across
 * calls. Quantizer: z = fp16 round-down(min), s = fp16 round-up((max - z)/qmax),
 * code = clamp(rint((x - z) * (1/s)), 0, 2^bits - 1); all fp32 steps are single
 * IEEE operations; z is clamped to >= -65504 and s to <= 65504; s = 0 gives
 * all-zero codes. Inputs must be finite.
 * Errors: KVQ_EINVAL (bad layer, batch, pointer, dtype), KVQ_ECAPACITY (some
 * sequence would pass max_tokens); the cache is unchanged on error. */
kvq_status kvq_append(kvq_cache* cache, int layer, const void* K, const void* V, kvq_dtype dtype,
                      const int32_t* n_new, int batch, void* stream);

/* Decode attention of `layer` for sequences b < batch ([rebut] "Baseline
 * Implementation": FlashAttention-style decoding over the quantized cache):
 *   out[b, hq, :] = sum_t softmax_t(q . k_t / sqrt(D)) v_t over every token
 *   appended so far, keys/values dequantized as code*s + z (window tokens
 *   exact bf16), q head hq reading KV head hq / (n_q_heads/n_kv_heads).
 *   Q:   device bf16 [batch, n_q_heads, head_dim], 16-byte aligned.
 *   out: device fp32 [batch, n_q_heads, head_dim], 16-byte aligned.
 * An empty sequence gives zeros. One kernel launch: either the CTAs of a
 * persistent grid share each (sequence, KV head) segment's pages and the last
 * CTA of a split segment merges the partial softmax states, or, for short
 * sequences (see kvq_set_decode_mode), one warp attends each segment whole.
 * Launched on a stream that is not being captured, the call passes the
 * sequence lengths to the kernel (no device-side scan), and, unless the last
 * launch this cache made on `stream` wrote `layer` (kvq_append,
 * kvq_decode_step, kvq_cache_reset), the kernel may start copying pages below
 * those lengths before the preceding kernel on the stream has finished
 * (programmatic dependent launch). So a kernel of the caller's own that writes
 * this cache's pages (a caller-owned pool) must not be the one launched right
 * before this call on the same stream; record an event or launch anything else
 * in between.
 * Errors: KVQ_EINVAL. */
kvq_status kvq_decode_attn(kvq_cache* cache, int layer, const void* Q, int batch, float* out,
                           void* stream);

/* One decode step of `layer`: append one new token to every sequence b < batch,
 * then attend over all tokens including it -- the same result as
 * kvq_append(n_new = 1 for each b) followed by kvq_decode_attn, with the same
 * pages, window, lengths and error report afterwards.
 *   K, V: device bf16 [batch, n_kv_heads, head_dim], the new token of each
 *         sequence, 16-byte aligned.
 *   Q, out: as for kvq_decode_attn.
 * ONE kernel launch, in either work split of kvq_decode_attn: the warp that
 * owns segment (b, h)'s tail unit first writes its new token into the window
 * or, when the token completes a 32-token group, quantizes and packs that group
 * into the next page (the append kernel's quantizer and packing, bit for bit)
 * and attends it from there; the other warps stream the older pages meanwhile.
 * The KVTuner pages warn that per-layer dispatch overhead can erase the savings
 * of a small KV cache. With KVQ_DECODE_KERNEL=simt (the CUDA-core check kernel)
 * it runs kvq_append and kvq_decode_attn. The same early page copies as
 * kvq_decode_attn apply. Inside a captured CUDA graph the kernel reads and
 * advances the device lengths, and a sequence already at max_tokens is left
 * unchanged with the cache's error flag raised (see kvq_refresh_lengths).
 * Errors: KVQ_EINVAL, KVQ_ECAPACITY (some sequence is full; nothing changes). */
kvq_status kvq_decode_step(kvq_cache* cache, int layer, const void* K, const void* V, const void* Q, int batch,
                           float* out, void* stream);

/* kvq_decode_attn for callers that cannot allocate device memory. The KVTuner
 * pages have no counterpart of this call; it exists for programs whose device
 * memory belongs to someone else (a serving engine that reserves all of HBM for
 * its own arena, a plug-in inside another runtime, a latency-critical loop that
 * must not call cudaMalloc/cudaFree). Such callers cannot use kvq_cache_create,
 * which allocates, so they keep one layer in their own buffers, in the storage
 * format described above:
 *   pages:   device, [batch][n_kv_heads][max_pages] pages of
 *            kvq_page_bytes(pair, head_dim) bytes, 16-byte aligned;
 *   window:  device, bf16 [batch][n_kv_heads][2][32][head_dim] (keys, values);
 *   seq_len: device int32 [batch]: tokens of each sequence; every entry must be
 *            in [0, max_seq_len] (entries beyond it read outside `pages`);
 *   max_seq_len: host bound on seq_len, with max_seq_len/32 <= max_pages;
 *   Q, out:  as for kvq_decode_attn.
 * The result is that of kvq_decode_attn on the same state, up to rounding
 * order. This call allocates nothing: its split-K scratch is a fixed 16 MiB
 * static device array that every GPU loading the library holds until the
 * process exits. The first call on a device looks up that array's address
 * (cudaGetSymbolAddress), so make the first call on each device before any
 * stream capture. Every call shares the array and clears the part that must
 * start at zero; calls whose kernels overlap on the GPU race on it, so
 * serialise them. The scratch holds one 4-byte merge counter per
 * (sequence, KV head) and split-K records of (n_q_heads / n_kv_heads) *
 * (head_dim + 2) * 4 bytes; KVQ_ECAPACITY when the counters leave no room for
 * two records in 16 MiB; KVQ_EINVAL for bad arguments (including more than
 * 2^31 units of work: batch * n_kv_heads * (max_seq_len/32 + 33)). Nothing is
 * launched on error. A call whose kernel gave up waiting for a page copy (its
 * output is then wrong) raises an error word in the same array; read it with
 * kvq_noalloc_check. */
kvq_status kvq_decode_attn_noalloc(kvq_pair pair, int head_dim, int n_q_heads, int n_kv_heads,
                                   const void* pages, int64_t max_pages, const void* window,
                                   const int32_t* seq_len, int64_t max_seq_len, const void* Q,
                                   int batch, float* out, void* stream);

/* Status of the kvq_decode_attn_noalloc calls made on the current device since
 * the last check: waits for the device, then returns KVQ_ECUDA (and clears the
 * word) if one of them gave up waiting for a page copy, KVQ_OK otherwise.
 * Allocates nothing. Like kvq_decode_attn_noalloc, it has no counterpart on the
 * KVTuner pages. */
kvq_status kvq_noalloc_check(void);

/* Per-layer quantization error report ([rebut] Table 3 and the layer-wise
 * error figures: quantization error is tracked layer by layer). Sums over every
 * element that a page flush of `layer` has quantized since creation or the last
 * reset, in fp64: (k - k_hat)^2, k^2, (v - v_hat)^2, v^2, with k, v the bf16
 * inputs and k_hat, v_hat their dequantized values; `elements` counts the
 * quantized key (= value) elements. Window tokens and bf16 layers add nothing.
 * The relative errors are k_sq_err / k_sq and v_sq_err / v_sq. */
typedef struct {
  double k_sq_err, k_sq, v_sq_err, v_sq;
  int64_t elements;
} kvq_error_stats;

/* Read `layer`'s report (synchronises the device). */
kvq_status kvq_layer_error(const kvq_cache* cache, int layer, kvq_error_stats* out);

/* Set the per-KV-head fp32 scales of an fp8 layer (host arrays of n_kv_heads
 * values, each finite and > 0; every head defaults to 1.0). Stored elements are
 * e4m3(x / scale) and read back as e4m3 * scale. The layer must be empty (no
 * token appended to any sequence since creation or the last reset), so every
 * stored element uses the same scales. Synchronous. Errors: KVQ_EINVAL (not an
 * fp8 layer, non-empty layer, bad scale), KVQ_ECUDA. */
kvq_status kvq_set_fp8_scales(kvq_cache* cache, int layer, const float* k_scale, const float* v_scale);

/* Pages per split-K CTA for kvq_decode_attn: 0 = automatic (default). Changing
 * it changes only the rounding order of the result. */
kvq_status kvq_set_split_pages(kvq_cache* cache, int pages_per_split);

/* Work split of kvq_decode_attn's tensor-core kernel when the query group has
 * at most 4 heads (n_q_heads / n_kv_heads <= 4): either each warp attends whole
 * (sequence, KV head) segments on its own and writes their outputs (no split
 * records, no merge), or the CTAs of a persistent grid share each segment's
 * pages. The first wins when sequences are short and segments many (batch 64 x
 * 160 tokens: 10 vs 19 us per layer on B200), the second otherwise.
 *   -1 (default): automatic -- the split a cost model fitted on B200 predicts
 *       faster (warp split about 5 + 1.0 us per page of the longest sequence;
 *       shared split about 11.5 + 0.01 us per segment + 0.15 us per page per SM);
 *    0: always the shared split;
 *    n > 0: the warp split whenever no sequence holds more than n full pages.
 * The warp split also needs every segment to fit the resident warps, else the
 * shared split runs. The choice is taken at launch from the host's view of the
 * lengths, so a CUDA graph keeps the split it was captured with (both are
 * correct at any length). It changes only the rounding order of the result.
 * Errors: KVQ_EINVAL (null cache, value < -1). */
kvq_status kvq_set_decode_mode(kvq_cache* cache, int max_pages_per_warp);

/* Tokens currently held by sequence `seq` of `layer` (host mirror), -1 if invalid. */
int64_t kvq_seq_len(const kvq_cache* cache, int layer, int seq);

/* Bytes the decode attention of `layer` reads for sequences b < batch at their
 * current lengths: packed codes, plus (include_metadata != 0) fp16 scales/zeros
 * and the bf16 window. -1 if invalid. */
int64_t kvq_bytes(const kvq_cache* cache, int layer, int batch, int include_metadata);

/* Size of kvq_export_layer's output for sequences b < batch, -1 if invalid. */
int64_t kvq_export_bytes(const kvq_cache* cache, int layer, int batch);

/* Copy `layer`'s stored state to host memory (synchronises the device): for
 * b < batch, for each KV head: the full pages (raw, format above), then the
 * window keys [W][D] bf16, then the window values [W][D] bf16. `bytes` must be
 * at least kvq_export_bytes(cache, layer, batch). */
kvq_status kvq_export_layer(const kvq_cache* cache, int layer, int batch, void* host_dst,
                            size_t bytes);

/* Wait for the cache's work and report any asynchronous CUDA error, or
 * KVQ_ECAPACITY if a one-token append launched from a replayed CUDA graph met a
 * full sequence (that sequence was left unchanged). */
kvq_status kvq_sync(kvq_cache* cache);

/* CUDA graphs. A decode step -- kvq_append with one token for every sequence,
 * then kvq_decode_attn -- can be captured on a stream and replayed: those two
 * calls enqueue kernels only (no host synchronisation, no host-to-device copy),
 * and the kernels read the sequence lengths on the device. Replays do not run
 * host code, so the host's mirror of the lengths (kvq_seq_len, kvq_bytes,
 * kvq_export_layer, capacity checks) lags until this call copies the device
 * lengths back (synchronises the device). Multi-token appends copy a plan from
 * the host and must not be captured. */
kvq_status kvq_refresh_lengths(kvq_cache* cache);

/* Number of kernels the library has launched on this cache so far. */
int64_t kvq_launch_count(const kvq_cache* cache);

/* Message describing the last failing call on this thread ("" if none). */
const char* kvq_last_error(void);

/* Name of a status code. */
const char* kvq_status_string(kvq_status status);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
