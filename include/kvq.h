/* kvq.h — C ABI of libkvq: asymmetric low-bit KV cache quantization and decode attention that
 * reads the packed cache directly, for NVIDIA B200 (sm_100a).
 *
 * The method (passages on the source pages):
 *   - keys are quantized per channel, values per token ("KIVI partitioning": The Asymmetric
 *     Key-Value Cache Compression framework page, Method; KVQuant review, Method and Key idea;
 *     KV cache quantization wiki page, verification notes on the KIVI full text);
 *   - keys form groups of G tokens along the sequence and values groups of G channels within a
 *     token; each group has its own min/max scale and zero-point, codes are 2 or 4 bits,
 *     round to nearest (KVQuant review, Problem and Comparison: uniform INT grids);
 *   - the newest tokens stay in FP16 (framework page, In practice) and a full group leaves that
 *     window and is appended to the quantized part along the token axis (wiki page, KIVI
 *     grouped/residual split);
 *   - an optional 128-point Walsh-Hadamard rotation is applied to keys and, identically, to the
 *     query (framework page, Method and In practice; Dual-QK abstract on the thelatestinai listing);
 *   - decode attention is bandwidth-bound because every step reads the whole cache (NOVA-KV
 *     abstract on the thelatestinai listing), so it reads the packed codes without expanding them
 *     in memory (KVQuant review, Method: custom kernels on the compressed cache).
 *
 * Conventions shared by every entry point:
 *   - Ownership: the caller allocates and frees every buffer; the library allocates nothing on the
 *     device or host and keeps no global mutable state. All device work is enqueued on the caller's
 *     stream (`cuda_stream` is a cudaStream_t; NULL means the legacy default stream) and runs
 *     asynchronously; the host-side length mirror is updated before the call returns.
 *   - Errors: every entry point returns a kvq_status and never aborts. Arguments are validated on
 *     the host before anything is launched; on an error nothing is enqueued and the cache is left
 *     unchanged. A failed launch is reported as KVQ_ERR_CUDA (the CUDA error is left for the caller
 *     to inspect with cudaGetLastError).
 *   - Inputs must be finite fp16 values (NaN / Inf are not checked on the device).
 *   - Only head_dim == 128 is supported.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = -1, /* null pointer, bad size, misaligned pointer, inconsistent config */
  KVQ_ERR_UNSUPPORTED = -2, /* a configuration the library does not implement (e.g. head_dim != 128) */
  KVQ_ERR_CAPACITY = -3,    /* a sequence would exceed config.capacity tokens */
  KVQ_ERR_WORKSPACE = -4,   /* workspace missing or smaller than kvq_decode_workspace_bytes */
  KVQ_ERR_CUDA = -5,        /* a kernel launch or copy failed */
  KVQ_ERR_TIMEOUT = -6      /* kvq_decode_status: a decode kernel gave up a bounded wait (outputs NaN) */
} kvq_status;

/* Packed layouts (see kvq_cache below): "tile v1" feeds warp-level mma fragments, "rows v2" feeds
 * the tcgen05 tensor cores and the pre-RoPE decode (one token's key codes / one channel's value codes
 * per row). */
#define KVQ_LAYOUT_TILE_V1 1
#define KVQ_LAYOUT_ROWS_V2 2

/* Problem definition. Requirements checked by every entry point:
 *   batch >= 1; num_kv_heads >= 1; num_q_heads a multiple of num_kv_heads with
 *   num_q_heads / num_kv_heads in {1, 2, 3, 4}; head_dim == 128;
 *   key_bits, value_bits in {2, 4};
 *   group_size G in {16, 32, 64, 128} (a multiple of the 16-token tile and a divisor of 128);
 *   residual R >= 0 (tokens kept in FP16 beyond the last full group; 0 <= R <= 4096);
 *   hadamard in {0, 1}; layout KVQ_LAYOUT_TILE_V1 or KVQ_LAYOUT_ROWS_V2; sink in {0, 1};
 *   rope_theta finite and >= 0; rope_theta > 0 needs hadamard = 0 (KVQ_ERR_INVALID_ARG) and layout
 *   KVQ_LAYOUT_ROWS_V2 (KVQ_ERR_UNSUPPORTED); outliers in {0, 1}, outliers = 1 needs layout
 *   KVQ_LAYOUT_TILE_V1 and rope_theta = 0 (KVQ_ERR_UNSUPPORTED);
 *   capacity >= 0, a multiple of G (maximum tokens per sequence); with layout ROWS_V2 also a
 *   multiple of 128 (value rows come in whole 128-token blocks);
 *   page_tokens 0 (contiguous) or a positive multiple of 128 that divides capacity, with
 *   num_pages >= 1; paging needs layout KVQ_LAYOUT_TILE_V1 and rope_theta = 0 (KVQ_ERR_UNSUPPORTED). */
typedef struct {
  int32_t batch;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t key_bits;
  int32_t value_bits;
  int32_t group_size;
  int32_t residual;
  int32_t hadamard;
  int32_t layout;
  int32_t sink;  /* 1: the first token of every sequence stays in fp16 (see below) */
  float rope_theta; /* > 0: keys are cached before RoPE and decode rotates them (see below); 0: off */
  int32_t outliers; /* 1: each quantized token's largest key / value entry stays fp16 (see below) */
  int32_t page_tokens; /* > 0: paged storage, pages of this many tokens (see below); 0: contiguous */
  int32_t num_pages;   /* pages in the pool (paged storage only) */
  int64_t capacity;
} kvq_config;

/* The packed cache: eight caller-owned device buffers plus the sequence lengths.
 * A "unit" is one (sequence b, KV head h); unit index u = b * num_kv_heads + h. Sizes per unit:
 *   k_codes  u32 [capacity/16][64*key_bits]     tile v1: key codes, one 16-token tile per row
 *            u32 [capacity][4*key_bits]         rows v2: one row of codes per token
 *   v_codes  u32 [capacity/16][64*value_bits]   tile v1: value codes, same tiling
 *            u32 [ceil(capacity/128)][128][4*value_bits]  rows v2: per 128-token block, one row per channel
 *   k_scale  fp16 [capacity/G][128]             per key group and channel (tile v1: permuted channel
 *                                               order as below; rows v2: natural order)
 *   k_zero   fp16 [capacity/G][128]             same; the zero-point is the group minimum
 *   v_scale  fp16 [capacity][128/G]             per token and channel group
 *   v_zero   fp16 [capacity][128/G]             same
 *   k_res    fp16 [R+G+sink][128]               FP16 ring of the newest keys (rotated if hadamard);
 *                                               with sink = 1, row R+G holds the first token's key
 *   v_res    fp16 [R+G+sink][128]               same for values
 * Every buffer must be 16-byte aligned. kvq_cache_buffer_bytes gives the total sizes.
 *
 * Quantized length of a sequence of T tokens: Q = G * floor(max(T - R, 0) / G). Tokens [0, Q) are
 * quantized, tokens [Q, T) live in the ring at slot t mod (R + G).
 *
 * Attention sink (sink = 1; the KVQuant review, Method, keeps the first token in fp16): token 0's key
 * and value are also kept in fp16 in ring row R+G, written by the prefill or by the append that adds
 * token 0. Key group 0's min/max leave token 0 out, token 0's codes and value scale / zero are 0, and
 * decode reads token 0 only from its fp16 row.
 *
 * Pre-RoPE keys (rope_theta > 0; the KVQuant review, Method and Key idea, quantizes keys before RoPE
 * and applies RoPE after dequantization): the cache holds the keys as passed to prefill and append,
 * without RoPE. Decode rotates every key at its absolute position t (0-based) after dequantization,
 * or from its fp16 row: channel pairs (i, i + 64), i < 64, by the angle t * rope_theta^(-i/64),
 * k'[i] = k[i] cos - k[i+64] sin, k'[i+64] = k[i] sin + k[i+64] cos. The query is used as given
 * (already rotated at its own position by the caller). The decode workspace then also holds the
 * angle tables, built at the start of every call.
 *
 * Dense-and-sparse outliers (outliers = 1; the KVQuant review, Method, keeps about 1% of the entries
 * in an fp16 sparse store with per-vector thresholds): per quantized token and tensor, the entry of
 * largest magnitude (ties: the lowest channel) is kept exactly. k_out / v_out hold one u32 per token
 * and unit: bits 0..15 the channel (0xffff: none, e.g. the sink token), bits 16..31 the fp16 value.
 * That entry stays out of its key group's (per channel) or value group's (per token) min / max and
 * is coded 0; dequantization puts the fp16 value back. A key channel whose entries in a group are all
 * outliers gets scale and zero 0. Sizes: kvq_outlier_buffer_bytes.
 *
 * Paged storage (page_tokens = P > 0; the KVQuant review, Limitations, Future work and Sparks, names
 * blocked allocation as the fix for copying earlier tokens' data on every update): the quantized part
 * of a unit is cut into logical pages of P tokens. Logical page j of unit u lives in pool page
 * page_table[u][j] (int32 [units][capacity / P]). k_codes, v_codes, k_scale, k_zero, v_scale, v_zero,
 * k_out and v_out then hold num_pages pages instead of one slot per unit: each page holds what the
 * per-unit layout above holds for P tokens (read "P" for "capacity"), at the in-page token t mod P;
 * k_res and v_res stay per unit. The library reads the entries of the pages that hold quantized
 * tokens, j < ceil(Q / P), and rejects (KVQ_ERR_INVALID_ARG) such an entry outside [0, num_pages);
 * other entries may hold anything (e.g. -1, not yet handed out). Distinct (unit, page) pairs must get
 * distinct pool pages, and an entry must not change while its page holds tokens.
 * page_table_host is the caller's table in host memory; page_table_dev is its device mirror (caller-
 * allocated, same shape), written by the library on the stream: the whole table is copied on every
 * prefill and on every append in which some unit's quantized part enters a new page. That copy is an
 * asynchronous host-to-device copy: if page_table_host is pinned, the caller must not change it
 * until the stream has passed the call (from pageable memory the copy is staged before the call
 * returns).
 *
 * Tile v1: tile row k of a unit holds tokens 16k..16k+15. Within a tile, "lane" L (0..31) owns
 * words (w / 4) * 128 + 4L + (w % 4) for w in [0, 2*bits). Word w holds 16/bits code pairs; pair j
 * has its first code at bits [bits*j, bits*j + bits) and its second at bits [16 + bits*j, ...).
 * With pair slot p = w * (16/bits) + j, m = p / 4, u = p % 2, hh = (p / 2) % 2, L = 4r + qd and
 * e in {0, 1} naming the first / second code of the pair:
 *   keys:   token 16k + r + 8u,          channel 16m + 2qd + 8hh + e
 *   values: token 16k + 2qd + 8hh + e,   channel 16m + r + 8u
 * Key scale/zero entry of channel c = 16m + 2qd + 8hh + e sits at index 32qd + 4m + 2hh + e.
 * (This order lets the decode kernel feed 16-byte loads straight into tensor-core fragments.)
 *
 * Rows v2 (P = 16/bits code pairs per u32 word; pair k of a word has its first code at bits
 * [bits*k, bits*k + bits) and its second at bits [16 + bits*k, ...)):
 *   keys:   token t's row holds channel pair j = c/2 in word j/P as pair j%P (channel 2j first);
 *   values: token t lies in block t/128 at i = t%128; channel c's row of that block holds token
 *           pair j = i/2 in word j/P as pair j%P (token 2j first).
 *
 * seq_len_host: int64 [batch] in host memory, read and updated by the library on the calling thread.
 *               The library never queues a copy from it: lengths reach the device as kernel
 *               arguments, so the array may be pageable or pinned and is free to change as soon
 *               as a call returns.
 * seq_len_dev:  int64 [batch] in device memory, the device mirror, written by kernels on the stream
 *               (prefill, and each append for the new lengths).
 */
typedef struct {
  void* k_codes;
  void* v_codes;
  void* k_scale;
  void* k_zero;
  void* v_scale;
  void* v_zero;
  void* k_res;
  void* v_res;
  int64_t* seq_len_host;
  int64_t* seq_len_dev;
  void* k_out;  /* outliers = 1 only: u32 [capacity] per unit, see below (NULL otherwise) */
  void* v_out;
  int32_t* page_table_host; /* page_tokens > 0 only: int32 [units][capacity / page_tokens], see above */
  int32_t* page_table_dev;  /* its device mirror, written by the library */
} kvq_cache;

enum {
  KVQ_BUF_K_CODES = 0,
  KVQ_BUF_V_CODES = 1,
  KVQ_BUF_K_SCALE = 2,
  KVQ_BUF_K_ZERO = 3,
  KVQ_BUF_V_SCALE = 4,
  KVQ_BUF_V_ZERO = 5,
  KVQ_BUF_K_RES = 6,
  KVQ_BUF_V_RES = 7,
  KVQ_NUM_BUFFERS = 8
};

/* Byte size of each of the eight cache buffers for `cfg` (all units, or the whole pool of num_pages
 * pages for the first six with paged storage), in kvq_cache field order.
 * Returns KVQ_ERR_INVALID_ARG / KVQ_ERR_UNSUPPORTED for a bad config or null pointers. */
kvq_status kvq_cache_buffer_bytes(const kvq_config* cfg, size_t out_bytes[KVQ_NUM_BUFFERS]);

/* Byte size of the two outlier buffers (k_out, v_out) for `cfg`: units * capacity * 4 each (paged:
 * num_pages * page_tokens * 4) when outliers = 1, else 0. */
kvq_status kvq_outlier_buffer_bytes(const kvq_config* cfg, size_t out_bytes[2]);

/* Prefill: quantize whole prompts at once (KVQuant review, Limitations and Sparks: a prefill-side
 * kernel that compresses many keys and values in one pass).
 * k, v: device fp16, element (b, t, h, d) at b*stride_b + t*stride_t + h*stride_h + d (strides in
 * elements, d contiguous, the same strides for k and v; rows must be 16-byte aligned, i.e. the
 * pointers 16-byte aligned and every stride a multiple of 8). seq_lens: host int64 [batch], each in
 * [0, capacity]. Replaces the state of every sequence: T_b := seq_lens[b]; tokens [0, Q_b) are
 * quantized (keys rotated first when hadamard is set) and [Q_b, T_b) copied to the ring.
 * Errors: KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CAPACITY (a length above capacity),
 * KVQ_ERR_CUDA. */
kvq_status kvq_quantize_prefill(const kvq_config* cfg, kvq_cache* cache, const void* k, const void* v,
                                int64_t stride_b, int64_t stride_t, int64_t stride_h, const int64_t* seq_lens,
                                void* cuda_stream);

/* Streaming append (wiki page, KIVI notes: new tokens join the FP16 window, and a window that has
 * grown a whole group past R is quantized and appended along the token axis).
 * k_new, v_new: device fp16 [batch][num_kv_heads][128], 16-byte aligned. Appends exactly one token
 * to every sequence (T_b += 1) and flushes group Q_b / G of every sequence whose T_b - R reached
 * Q_b + G. Errors: KVQ_ERR_CAPACITY if any T_b + 1 > capacity (nothing is changed), plus the
 * generic ones. */
kvq_status kvq_append_token(const kvq_config* cfg, kvq_cache* cache, const void* k_new, const void* v_new,
                            void* cuda_stream);

/* Bytes of device workspace kvq_decode_attention needs for `cfg` (an upper bound that holds for
 * every set of sequence lengths up to capacity). */
kvq_status kvq_decode_workspace_bytes(const kvq_config* cfg, size_t* bytes);

/* Decode attention of one query token per sequence over everything cached (NOVA-KV abstract:
 * decoding reads the whole cache each step; wiki page, KIVI notes: the grouped and the FP16
 * residual parts both enter the scores).
 * q: device fp16 [batch][num_q_heads][128]; out: device fp16 [batch][num_q_heads][128]
 * (16-byte aligned). Query head h attends to KV head h / (num_q_heads / num_kv_heads) over all
 * T_b tokens: out = softmax(sm_scale * q~ . K^) V^ with K^, V^ the dequantized cache
 * (code * scale + zero; FP16 residual as stored; with sink = 1 token 0 from its fp16 row; with
 * rope_theta > 0 every key turned at its position as described above) and q~ = H q / sqrt(128)
 * when hadamard is set. A sequence with T_b == 0 gets a zero output. The caller appends the current
 * token first.
 * workspace: device, 256-byte aligned, at least kvq_decode_workspace_bytes(cfg) bytes; it is
 * scratch for split partials and may be reused after the stream passes this call.
 * Errors: KVQ_ERR_WORKSPACE, KVQ_ERR_INVALID_ARG (non-finite or non-positive sm_scale, nulls,
 * misalignment), KVQ_ERR_CUDA. */
kvq_status kvq_decode_attention(const kvq_config* cfg, const kvq_cache* cache, const void* q, void* out, float sm_scale,
                                void* workspace, size_t workspace_bytes, void* cuda_stream);

/* Decode attention without a caller-provided workspace. The source pages have no counterpart to
 * this entry point; it serves callers that cannot allocate device memory, such as a plugin inside a
 * host framework that owns every device allocation through its own pool, or a serving loop whose
 * policy forbids allocation after start-up.
 * Same arguments, results and errors as kvq_decode_attention, except that the split partials live
 * in a fixed device array inside the library: KVQ_STATIC_SCRATCH_BYTES (16 MiB) per GPU that loads
 * the library, held until the process exits. It allocates nothing (no cudaMalloc, no allocating
 * library routine).
 *   - Returns KVQ_ERR_WORKSPACE if kvq_decode_workspace_bytes(cfg) exceeds KVQ_STATIC_SCRATCH_BYTES.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *     that device current; make that first call before any stream capture.
 *   - Every call shares the one array per device: calls whose GPU work overlaps (e.g. on two
 *     streams) race on it; the caller must serialise them. No scratch content needs to start at
 *     zero. */
#define KVQ_STATIC_SCRATCH_BYTES (16u << 20)
kvq_status kvq_decode_attention_noalloc(const kvq_config* cfg, const kvq_cache* cache, const void* q, void* out,
                                        float sm_scale, void* cuda_stream);

/* Outcome of the last decode call that used `workspace` for `cfg`. The source pages have no
 * counterpart to this entry point; it reports a failure that the asynchronous decode call itself
 * cannot. The rows-v2 (tcgen05) decode kernel waits on its own copies and tensor-core products with
 * bounded waits (about 2 s); a CTA that gives up writes NaN partials instead of hanging, and the
 * split combine then records, per (sequence, query head), whether its output came out NaN that way.
 * Every decode call rewrites those records (they sit at the end of the workspace, within
 * kvq_decode_workspace_bytes), so nothing needs clearing. With KVQ_TEST_STALL_TC=1 in the process
 * environment, the rows-v2 decode (no RoPE) issues no quantized step and waits on a barrier that
 * nothing completes, so that it gives up on purpose: a test hook for this path, off by default.
 * This call copies the records to the host on `cuda_stream` and synchronises that stream: call it
 * on the stream of the decode (or after it), before the workspace is reused.
 * Returns KVQ_OK, KVQ_ERR_TIMEOUT if some output of that decode is NaN from a give-up, or
 * KVQ_ERR_INVALID_ARG / KVQ_ERR_UNSUPPORTED / KVQ_ERR_CUDA. */
kvq_status kvq_decode_status(const kvq_config* cfg, const void* workspace, void* cuda_stream);

/* Static description of a status code. */
const char* kvq_status_string(kvq_status status);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
