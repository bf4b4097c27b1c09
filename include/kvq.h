/*
 * kvq.h -- C ABI of libkvq: attention over a block-quantized KV cache
 * (Q8_0 keys, Q4_0 values) at long context, for NVIDIA B200 (sm_100a).
 *
 * Sources (web pages on quantized KV at long context):
 *  "OSCAR2 KV Cache benchmark" (molayo1419.me), Compression Ratios table:
 *      q8_0 costs 136 bytes per 128 elements (34-byte blocks of 32).
 *  "Adaptive KV streaming lands on ROCm: Qwen3.8-27B at full 262k context ..."
 *      (richland.au), "What shipped" and "Why it matters": the full KV history
 *      stays in host RAM and a bounded working set is streamed to the GPU and
 *      reused across layers; Q8_0 K + Q4_0 V costs 26,624 B/token for 16
 *      attention layers of 4 KV heads x 256.
 *  "Qwen 27B (IQ4_XS, Q8/Q4 KV) ... 262k context" (molayo1419.me), list of
 *      improvements, "Online Log-Sum-Exp prefill & pipelined prefetch":
 *      chunked prefill over streamed pages with online LSE accumulation, and
 *      layer L+1's transfer overlapped with layer L's compute; speculative-
 *      decoding paragraph: paged decode attention extended to the verify batch.
 *  "Context window and KV cache" (localaiforum.com), "GQA" section: a few KV
 *      heads are shared by many query heads; "levers" section: llama.cpp
 *      quantizes the KV cache (q8_0 halves it, q4_0 quarters it).
 *
 * Conventions for every entry point
 *  - The caller owns all memory.  Device buffers are passed as plain device
 *    pointers; the library allocates no device memory.  kvq_layer structs and
 *    arrays of them are read from HOST memory during the call only.
 *  - Calls are asynchronous on the given stream (a cudaStream_t passed as
 *    void*, NULL = the legacy default stream) and never synchronise, except
 *    kvq_check.  Results are valid once the stream reaches that point.
 *  - Arguments are validated before anything is launched.  On error nothing
 *    is launched, the status says why and kvq_last_error() gives a
 *    thread-local message.  A launch failure returns KVQ_ERR_CUDA.
 *  - No call aborts, exits or traps.  Every device-side wait is bounded; a
 *    wait that runs out records KVQ_ERR_TIMEOUT in a device status word that
 *    kvq_check() reads and clears.
 *  - fp16 values are passed as uint16_t bit patterns (IEEE binary16).
 *
 * Block formats (llama.cpp-style; the pages give sizes, these are the
 * readings of the bit layout):
 *  Q8_0, 34 B per 32 elements: fp16 d (little-endian) then int8 q[32];
 *        x^ = d * q.  Quantized in fp32 without FMA: d = amax/127,
 *        id = d ? 1/d : 0, q = roundf(x*id) (ties away from zero).
 *  Q4_0, 18 B per 32 elements: fp16 d then 16 bytes; byte j holds element
 *        j in the low nibble and element j+16 in the high nibble; x^ = d*(u-8).
 *        m = the signed first element of largest |x|, d = m/-8,
 *        id = d ? 1/d : 0, u = min(15, trunc(x*id + 8.5)).
 *  OSCAR2, 36 B per 128 elements (the INT2 format of the OSCAR2 page's
 *        Compression Ratios table, 2.25 bits per element, with an fp16
 *        zero-point): fp16 d, fp16 m, then 32 bytes; byte j holds the 2-bit
 *        codes u of elements j, j+32, j+64, j+96 in bits 0-1, 2-3, 4-5, 6-7;
 *        x^ = d*u + m.  mn = min x, mx = max x, d = (mx - mn)/3,
 *        id = d ? 1/d : 0, u = min(3, trunc((x - mn)*id + 0.5)); m = fp16(mn).
 *        A tensor in this format needs head_dim a multiple of 128, and its
 *        values must lie inside the fp16 range (m is stored as fp16).  The
 *        page's Hadamard rotation is baked into a model's weights before any
 *        row reaches the cache; no call rotates.
 *  Only fp16(d) is stored; the quantizer divides by the fp32 d.
 *
 * Cache layout of one layer (head-major, fixed):
 *  K: [n_kv_heads][capacity][head_dim/32] Q8_0 blocks
 *     -> one head-row of a token is head_dim/32*34 bytes (272 B at 256)
 *  V: [n_kv_heads][capacity][head_dim/32] Q4_0 blocks
 *     -> one head-row is head_dim/32*18 bytes (144 B at 256)
 *  That is the pages' configuration (kvq_layer k_type = v_type = 0).  Either
 *  tensor may instead use another format (KVQ_TYPE_Q8_0 / KVQ_TYPE_Q4_0, the
 *  q8_0 and q4_0 choices of the KV-cache guide's levers section, or
 *  KVQ_TYPE_OSCAR2); its head-rows are then head_dim / (elements per block)
 *  blocks of that format (36*head_dim/128 bytes for OSCAR2).
 *  Head-rows of consecutive tokens of a head are contiguous, so a run of
 *  tokens is one contiguous byte range.  Both base pointers must be 16-byte
 *  aligned and capacity a multiple of 8: then every head starts on a 16-byte
 *  boundary (8 head-rows are 272*(head_dim/32), 144*(head_dim/32) or
 *  288*(head_dim/128) bytes),
 *  and so does every run of tokens that starts at a multiple of 8.
 *  head_dim is a multiple of 32 (of 128 where a tensor is OSCAR2), at most 512.
 *
 * Attention (the plainest reading): query head g reads KV head
 * g / (n_q_heads / n_kv_heads); s_j = scale * sum_i q_i k^_ij;
 * o = sum_j exp(s_j - m) v^_j / l, lse = m + ln l (natural log), m the max
 * over the complete visible scores, l = sum_j exp(s_j - m).  An empty key
 * set gives o = 0 and lse = -inf.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kvq_status {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size or shape              */
    KVQ_ERR_ALIGNMENT = 2,    /* a pointer is not aligned as documented        */
    KVQ_ERR_UNSUPPORTED = 3,  /* valid but not implemented (e.g. head_dim)     */
    KVQ_ERR_CUDA = 4,         /* a CUDA runtime call or a launch failed        */
    KVQ_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out            */
    KVQ_ERR_COPY = 6,         /* a host<->device copy could not be enqueued    */
    KVQ_ERR_WORKSPACE = 7     /* workspace missing or smaller than required    */
} kvq_status;

/* A cudaStream_t, passed as an opaque pointer so that this header needs no
 * CUDA header.  NULL is the legacy default stream. */
typedef void *kvq_stream;

/* One attention layer of the cache.  All layers passed to one call must have
 * the same n_kv_heads and head_dim. */
/* Block format of a cache tensor.  KVQ_TYPE_DEFAULT is Q8_0 for K and Q4_0
 * for V.  All layers passed to one call must use the same formats.  Every call
 * accepts every combination; the tensor-core kernels are built for the
 * default pair (decode and prefill run the other pairs on their general,
 * CUDA-core kernels). */
typedef enum kvq_type {
    KVQ_TYPE_DEFAULT = 0,
    KVQ_TYPE_Q8_0 = 1,   /* 34 B per 32 elements */
    KVQ_TYPE_Q4_0 = 2,   /* 18 B per 32 elements */
    KVQ_TYPE_OSCAR2 = 3  /* 36 B per 128 elements (INT2, fp16 zero-point) */
} kvq_type;

typedef struct kvq_layer {
    void *k;             /* K blocks, layout above (device memory, or pinned
                            host memory for kvq_stream_decode's host_layers) */
    void *v;             /* V blocks, layout above                           */
    int64_t capacity;    /* tokens per head the two arrays hold              */
    int32_t n_kv_heads;  /* KV heads (4 in the pages' hybrid model)          */
    int32_t head_dim;    /* elements per head-row, a multiple of 32 (128 for
                            an OSCAR2 tensor), <= 512                        */
    int32_t k_type;      /* kvq_type of K (0: Q8_0)                          */
    int32_t v_type;      /* kvq_type of V (0: Q4_0)                          */
} kvq_layer;

/* Largest number of layers one call accepts (layer tables travel as kernel
 * parameters). */
#define KVQ_MAX_LAYERS 64
/* Largest decode batch (query tokens per layer per call): the verify batch. */
#define KVQ_MAX_DECODE_T 4

/* ---------------------------------------------------------------------- */
/* Quantize-on-append                                                      */
/* ---------------------------------------------------------------------- */

/* Quantize n fp32 values to Q8_0 blocks.
 * Source: Compression Ratios table of the OSCAR2 page (34 B per 32 elements);
 * the levers section of the KV-cache guide (q8_0 KV).
 *  x      device, fp32[n], 4-byte aligned
 *  blocks device, n/32 blocks of 34 bytes, written in order, 2-byte aligned
 *  n      multiple of 32, >= 0 (0 launches nothing)
 * Errors: INVALID_ARG (null pointer with n > 0, n % 32 != 0, n < 0),
 *         ALIGNMENT (x not 4-byte or blocks not 2-byte aligned), CUDA. */
kvq_status kvq_quantize_q8_0(const float *x, void *blocks, int64_t n, kvq_stream stream);

/* Quantize n fp32 values to Q4_0 blocks (18 B per 32 elements).
 * Source: 26,624 B/token in "Why it matters" of the ROCm streaming page
 * implies 18 B per 32 V elements; the KV-cache guide's levers (q4_0 KV).
 * Arguments and errors as kvq_quantize_q8_0. */
kvq_status kvq_quantize_q4_0(const float *x, void *blocks, int64_t n, kvq_stream stream);

/* Quantize n fp32 values to OSCAR2 blocks (36 B per 128 elements).
 * Source: Compression Ratios table of the OSCAR2 page (oscar2: 36 B per 128
 * elements, 2.25 bits, INT2 with fp16 zero-point metadata); the bit layout
 * and the rule are this library's reading (block formats above).
 *  x      device, fp32[n], 4-byte aligned, values inside the fp16 range
 *  blocks device, n/128 blocks of 36 bytes, written in order, 4-byte aligned
 *  n      multiple of 128, >= 0 (0 launches nothing)
 * Errors: INVALID_ARG (null pointer with n > 0, n % 128 != 0, n < 0),
 *         ALIGNMENT (x or blocks not 4-byte aligned), CUDA. */
kvq_status kvq_quantize_oscar2(const float *x, void *blocks, int64_t n, kvq_stream stream);

/* Quantize-on-append of new K/V rows into rows [pos, pos+n_tok) of every KV
 * head of n_layers layers (K -> Q8_0, V -> Q4_0, or the layers' k_type /
 * v_type).
 * Source: the KV-cache guide's levers section (the KV cache is stored
 * quantized); the Q8_0 K / Q4_0 V cache of the RX 9070 XT page.
 *  layers  host array of n_layers kvq_layer (device caches)
 *  k_new   device fp32 [n_layers][n_tok][n_kv_heads][head_dim], 16-B aligned
 *  v_new   device fp32, same shape
 *  pos     first row written; pos + n_tok <= capacity of every layer
 * Errors: INVALID_ARG (nulls, n_layers outside [1, KVQ_MAX_LAYERS], n_tok < 1,
 *         pos < 0, pos + n_tok > capacity, layers that differ in heads/dim,
 *         capacity % 8 != 0, an unknown block type), ALIGNMENT, UNSUPPORTED
 *         (head_dim not a multiple of 32, or of 128 for an OSCAR2 tensor, or
 *         > 512), CUDA.  Every call that takes layers checks them the same way. */
kvq_status kvq_append(const kvq_layer *layers, int n_layers, const float *k_new,
                      const float *v_new, int64_t pos, int n_tok, kvq_stream stream);

/* ---------------------------------------------------------------------- */
/* Split-KV GQA decode attention                                           */
/* ---------------------------------------------------------------------- */

/* Decode attention of T query tokens per layer (T = 1 decode, T <= 4 a
 * speculative verify batch) over the first n_kv keys of each layer, split
 * into chunks of `chunk` keys; returns every chunk's partial (out, lse).
 * Query token t sees keys j <= n_kv - T + t (n_kv counts the T new rows,
 * which must already be appended).  Dequantization happens in registers;
 * each chunk keeps an online softmax whose max covers complete scores.
 * Source: speculative-decoding paragraph of the RX 9070 XT page (paged decode
 * attention extended to the verify batch); "Known Issues Fixed" of the
 * OSCAR2 page (max over the full KQ scores); GQA section of the KV-cache guide.
 *  layers    host array of n_layers kvq_layer (device caches)
 *  q         device fp16 bits [n_layers][T][n_q_heads][head_dim], 16-B aligned
 *  n_q_heads multiple of n_kv_heads; n_q_heads/n_kv_heads * T <= 32
 *  n_kv      keys per layer, T <= n_kv <= capacity
 *  chunk     keys per chunk, a positive multiple of 64
 *  scale     softmax scale applied to q.k (1/16 for head_dim 256)
 *  out_part  device fp32 [n_layers][T][n_q_heads][n_chunks][head_dim], 16-B
 *            aligned, n_chunks = ceil(n_kv / chunk); fully masked chunks get 0
 *  lse_part  device fp32 [n_layers][T][n_q_heads][n_chunks]; -inf if masked
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED (T > KVQ_MAX_DECODE_T, group
 *         too large), CUDA. */
kvq_status kvq_decode_attn(const kvq_layer *layers, int n_layers, const uint16_t *q,
                           int n_q_heads, int T, int64_t n_kv, int chunk, float scale,
                           float *out_part, float *lse_part, kvq_stream stream);

/* kvq_decode_attn over one contiguous shard of a context, for a
 * context-parallel split (each GPU holds keys [key0, key0 + n_keys) of an
 * n_kv-key context and decodes only those; the shards' results are then
 * combined by the LSE merge, e.g. kvq_merge_lse followed by an all-gather and
 * kvq_merge_lse_parts).  The layers hold the shard's keys at their rows
 * [0, n_keys); query token t sees the global keys j <= n_kv - T + t, i.e. the
 * shard rows j' <= n_kv - T + t - key0 (a row that sees none of the shard gets
 * out = 0, lse = -inf).  Chunks split the shard: n_chunks = ceil(n_keys /
 * chunk).  With key0 = 0 and n_keys = n_kv this is kvq_decode_attn.
 * Source: as kvq_decode_attn; the split is this library's extension (the
 * merge that combines the shards is the one the pages use across pages).
 *  n_keys    keys in the shard, 1 <= n_keys <= capacity
 *  key0      global index of the shard's first key, 0 <= key0 <= n_kv - n_keys
 *  n_kv      keys in the whole context (including the T new rows), >= T
 *  other arguments as kvq_decode_attn, with n_chunks from n_keys
 * Errors: those of kvq_decode_attn; INVALID_ARG for a shard outside the
 *         context. */
kvq_status kvq_decode_attn_shard(const kvq_layer *layers, int n_layers, const uint16_t *q,
                                 int n_q_heads, int T, int64_t n_keys, int64_t key0,
                                 int64_t n_kv, int chunk, float scale, float *out_part,
                                 float *lse_part, kvq_stream stream);

/* ---------------------------------------------------------------------- */
/* LSE merge                                                               */
/* ---------------------------------------------------------------------- */

/* Merge per-chunk partials: lse = M + ln sum_c exp(lse_c - M) with
 * M = max_c lse_c, out = sum_c exp(lse_c - lse) out_c; partials with
 * lse_c = -inf are skipped; if every partial is -inf, out = 0, lse = -inf.
 * Source: "Online Log-Sum-Exp prefill & pipelined prefetch" of the RX 9070 XT
 * page (partials over pages combined through their log-sum-exp).
 *  out_part device fp32 [rows][n_chunks][head_dim], 16-B aligned
 *  lse_part device fp32 [rows][n_chunks]
 *  out      device fp32 [rows][head_dim]; lse device fp32 [rows]
 * Errors: INVALID_ARG (nulls, rows < 0, n_chunks < 1, head_dim % 4),
 *         ALIGNMENT, CUDA. */
kvq_status kvq_merge_lse(const float *out_part, const float *lse_part, int64_t rows,
                         int n_chunks, int head_dim, float *out, float *lse,
                         kvq_stream stream);

/* The same merge over partials stored part-major, as an all-gather of
 * per-rank merged rows lays them out: part p of row r at
 * out_parts[(p * rows + r) * head_dim ...] and lse_parts[p * rows + r].  The
 * order of operations is that of kvq_merge_lse (parts in increasing p).
 *  out_parts device fp32 [n_parts][rows][head_dim], 16-B aligned
 *  lse_parts device fp32 [n_parts][rows]
 *  out       device fp32 [rows][head_dim]; lse device fp32 [rows]
 * Errors: INVALID_ARG (nulls, rows < 0, n_parts < 1, head_dim % 4),
 *         ALIGNMENT, CUDA. */
kvq_status kvq_merge_lse_parts(const float *out_parts, const float *lse_parts, int n_parts,
                               int64_t rows, int head_dim, float *out, float *lse,
                               kvq_stream stream);

/* ---------------------------------------------------------------------- */
/* Fused decode step                                                       */
/* ---------------------------------------------------------------------- */

/* One decode step of all layers:
 *   kvq_append(layers, k_new, v_new, pos = n_kv - T, T), then
 *   kvq_decode_attn(...), then kvq_merge_lse(...)
 * issued as those three launches, back to back on `stream`, with the same
 * results (cache bytes, out_part, lse_part, out, lse).  All arguments are
 * checked before the first launch.  A single launch that appends in the
 * decode kernel and merges in the last CTA of each head was built and
 * measured: it saved two launches of a few microseconds on a step of
 * milliseconds and cost more inside the decode kernel than that, so the step
 * is three launches (capture them in a CUDA graph to drop the launch gaps).
 *  k_new, v_new  device fp32 [n_layers][T][n_kv_heads][head_dim], 16-B aligned
 *  n_kv          keys after the append (the new rows are [n_kv - T, n_kv))
 *  q, out_part, lse_part, out, lse, chunk, scale: as kvq_decode_attn and
 *                kvq_merge_lse (rows = n_layers * T * n_q_heads)
 *  workspace, ws_bytes  reserved: not read; may be NULL / 0
 *                (kvq_workspace_bytes(KVQ_OP_DECODE_STEP, ...) is 0)
 * Errors: those of kvq_append, kvq_decode_attn and kvq_merge_lse. */
kvq_status kvq_decode_step(const kvq_layer *layers, int n_layers, const float *k_new,
                           const float *v_new, const uint16_t *q, int n_q_heads, int T,
                           int64_t n_kv, int chunk, float scale, float *out_part,
                           float *lse_part, float *out, float *lse, void *workspace,
                           size_t ws_bytes, kvq_stream stream);

/* kvq_decode_step with the step's inputs and results in host memory: copies
 * q_host, k_host and v_host into the device buffers q, k_new and v_new, runs
 * the step (append, decode, merge), and copies out and lse back into out_host
 * and lse_host -- five cudaMemcpyAsync and three launches, in that order on
 * `stream`.  The host results are valid once the stream reaches the end of the
 * call (kvq_check or a stream synchronisation).  Host buffers should be
 * pinned: pageable memory makes the copies synchronous.
 *  k_host, v_host  host fp32 [n_layers][T][n_kv_heads][head_dim]
 *  q_host          host fp16 bits [n_layers][T][n_q_heads][head_dim]
 *  out_host        host fp32 [n_layers][T][n_q_heads][head_dim]
 *  lse_host        host fp32 [n_layers][T][n_q_heads]
 *  k_new, v_new, q device buffers of those sizes (the copies' targets)
 *  the rest        as kvq_decode_step (the workspace is not needed)
 * Errors: INVALID_ARG (a NULL host buffer), those of kvq_decode_step (all
 *         checked before the first copy), COPY (a copy could not be enqueued;
 *         the copies and launches before it stay enqueued). */
kvq_status kvq_decode_step_host(const kvq_layer *layers, int n_layers, const float *k_host,
                                const float *v_host, const uint16_t *q_host, float *out_host,
                                float *lse_host, float *k_new, float *v_new, uint16_t *q,
                                int n_q_heads, int T, int64_t n_kv, int chunk, float scale,
                                float *out_part, float *lse_part, float *out, float *lse,
                                kvq_stream stream);

/* ---------------------------------------------------------------------- */
/* Chunked prefill                                                         */
/* ---------------------------------------------------------------------- */

/* Prefill attention of T new query tokens per layer over n_cached + T keys
 * (the T new rows must already be appended at rows [n_cached, n_cached+T));
 * token t sees keys j <= n_cached + t.  Keys are processed in tiles with an
 * online LSE merge carried across pages of keys inside the kernel.  Rows that
 * see at least 16,384 keys run on the tensor cores (tcgen05): K tiles are
 * dequantized on chip to an exact two-part f16 sum (so the logits carry only
 * fp32 rounding), V tiles and P to f16 (one rounding each), fp32
 * accumulation in tensor memory; the V and P rounding errors average over the
 * visible keys (measured max-abs error 2.2e-4 at 16,384 keys and 8.8e-5 at
 * 262,144 on N(0,1) K/V with x8 outlier channels).  Rows that see fewer keys
 * run an exact fp32 kernel on the CUDA cores.
 * The tensor-core path needs head_dim 256; other head_dims take the exact
 * kernel.
 * Source: "Online Log-Sum-Exp prefill & pipelined prefetch" of the RX 9070 XT
 * page (chunked prefill over streamed pages with online LSE accumulation).
 *  q         device fp16 bits [n_layers][T][n_q_heads][head_dim], 16-B aligned
 *  n_cached  keys before the new rows; n_cached + T <= capacity
 *  page      keys per page, a positive multiple of 128 (the online merge makes
 *            the result independent of it)
 *  out, lse  device fp32 [n_layers][T][n_q_heads][head_dim] and [...][n_q_heads]
 *  page_out, page_lse  optional (both NULL or both set), device fp32
 *            [n_layers][T][n_q_heads][n_pages][head_dim] (16-B aligned) and
 *            [n_layers][T][n_q_heads][n_pages], n_pages = ceil((n_cached + T) /
 *            page): the partial of page p (keys [p page, (p + 1) page) that the
 *            row sees) as out = sum_j p_j v^_j / l and lse = m + ln l, out = 0 and
 *            lse = -inf where the row sees no key of the page.  out and lse are
 *            then the LSE merge of the pages (the kvq_merge_lse kernel, launched
 *            by this call after the prefill kernels).
 *  workspace optional, device, 256-B aligned.  NULL: each CTA of the
 *            tensor-core path dequantizes the key tiles it reads.  Otherwise
 *            the call expands the key tiles of each (layer, KV head) pair once
 *            into a "slab" of the workspace (f16 K^hi, K^lo, V^: 1,536 B per
 *            key at head_dim 256; one slab = kvq_prefill_workspace_bytes(1, 1,
 *            head_dim, n_cached + T)), which the tensor-core kernel then copies
 *            in without dequantizing (every row tile of a pair reads the same
 *            keys).  ws_bytes must hold at least one slab.  With a slab for
 *            every pair (kvq_prefill_workspace_bytes(n_layers, n_kv_heads,
 *            head_dim, n_cached + T)) one expansion and one attention launch
 *            cover the call; with fewer, the pairs go in chunks of
 *            floor(slabs / 2) through the two halves of the workspace,
 *            alternating between `stream` and a second stream of the library
 *            (forked from and joined back into `stream` with events, so the
 *            call stays stream-ordered and can be captured in a CUDA graph);
 *            with one slab, one pair at a time on `stream`.  All sizes give
 *            the same results bit for bit.  Ignored when the tensor-core path
 *            does not run.  Owned by the caller; not used after the call's
 *            work completes.
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED (group size > 32),
 *         WORKSPACE (a workspace smaller than one slab), CUDA. */
kvq_status kvq_prefill_attn(const kvq_layer *layers, int n_layers, const uint16_t *q,
                            int n_q_heads, int T, int64_t n_cached, int page, float scale,
                            float *out, float *lse, float *page_out, float *page_lse,
                            void *workspace, size_t ws_bytes, kvq_stream stream);

/* ---------------------------------------------------------------------- */
/* Layer-pipelined host streaming                                          */
/* ---------------------------------------------------------------------- */

/* Decode attention with the cache in pinned host memory, except for layers
 * kept resident on the device.  Each layer of host_layers is either streamed
 * (its k and v are PINNED host memory) or resident (both are device memory of
 * the current device).  The i-th streamed layer's K and V rows [0, n_kv) of
 * every head are copied with cudaMemcpyAsync on `copy` into device slot i % 2
 * while the layers before it compute on `compute`; then decode + merge of the
 * layer run on `compute` from the slot.  A resident layer is decode + merge in
 * place.  Layers are computed in order.  Events order the two streams: the
 * copy into a slot waits until the compute that last read it is done.
 * Results equal kvq_decode_attn + kvq_merge_lse on a resident cache bit for
 * bit (same kernels, same data).
 * Source: "Online Log-Sum-Exp prefill & pipelined prefetch" of the RX 9070 XT
 * page (layer L+1's transfer overlapped with layer L's compute); "What
 * shipped" of the ROCm streaming page (the whole KV history in host RAM, a
 * bounded GPU working set reused across layers, sized to the device memory
 * left over: the adaptive part; kvq_resident_layers gives how many layers fit).
 *  host_layers  host array of n_layers kvq_layer: pinned host memory
 *               (cudaHostAlloc / cudaHostRegister) or device memory, per layer
 *  dev_slots    host array of 2 kvq_layer (device memory), capacity >= n_kv,
 *               same heads/dim as host_layers; may be NULL if no layer is
 *               streamed
 *  q            device fp16 bits [n_layers][T][n_q_heads][head_dim]
 *  out_part, lse_part  device scratch for ONE layer's partials:
 *               [T][n_q_heads][n_chunks][head_dim] and [T][n_q_heads][n_chunks]
 *  out, lse     device fp32 [n_layers][T][n_q_heads][head_dim], [...][n_q_heads]
 *  compute, copy  two different streams
 * The call enqueues everything and returns; `compute` is complete when all
 * layers are.  Errors: those of kvq_decode_attn, plus COPY when a copy cannot
 * be enqueued (nothing further is enqueued; work already enqueued completes). */
kvq_status kvq_stream_decode(const kvq_layer *host_layers, int n_layers,
                             const kvq_layer *dev_slots, const uint16_t *q, int n_q_heads,
                             int T, int64_t n_kv, int chunk, float scale, float *out_part,
                             float *lse_part, float *out, float *lse, kvq_stream compute,
                             kvq_stream copy);

/* Adaptive residency: how many of n_layers layers (each n_kv_heads x capacity
 * K and V head-rows at head_dim, in block formats k_type / v_type, 0 for the
 * defaults) can stay resident in budget_bytes of device
 * memory while the rest stream through kvq_stream_decode's two slots of one
 * layer each.  n_layers if everything fits (no slots are needed then);
 * otherwise the largest R <= n_layers - 1 with (R + 2) layers <= budget; -1 if
 * not even the two slots fit, or for an invalid shape.  Host arithmetic only.
 * Source: "What shipped" / "Why it matters" of the ROCm streaming page (a
 * bounded working set streamed from host RAM when the cache does not fit). */
int kvq_resident_layers(size_t budget_bytes, int n_layers, int64_t capacity, int n_kv_heads,
                        int head_dim, int k_type, int v_type);

/* ---------------------------------------------------------------------- */
/* Decode + merge without caller-provided scratch                          */
/* ---------------------------------------------------------------------- */

/* Size of the library's own device array for chunk partials (8 MiB). */
#define KVQ_STATIC_SCRATCH_BYTES (8u << 20)

/* kvq_decode_attn followed by kvq_merge_lse, for callers that cannot allocate
 * device memory for the chunk partials -- for example a plug-in inside a host
 * program that owns all device memory and passes only inputs and outputs, or
 * a step loop where a cudaMalloc (which may synchronise the device or fail
 * under memory pressure) is not allowed.  The pages have no counterpart: this
 * entry point exists for such callers only.
 * The partials live in one 8 MiB array inside the library (a __device__
 * object that every GPU which loads the library keeps until the process
 * exits); the call itself allocates nothing.  Its first call on a device looks
 * the array's address up (cudaGetSymbolAddress) with that device current; make
 * that first call before capturing any stream.  All calls share the array and
 * it keeps the last call's contents: the decode rewrites every partial it
 * reads, so nothing needs clearing, but calls whose work overlaps on the GPU
 * (on different streams, or different threads) race on it -- order them.
 *  layers, q, n_q_heads, T, n_kv, chunk, scale  as kvq_decode_attn
 *  out   device fp32 [n_layers][T][n_q_heads][head_dim], 16-B aligned
 *  lse   device fp32 [n_layers][T][n_q_heads]
 * Limit: n_layers * T * n_q_heads * ceil(n_kv / chunk) * (head_dim + 1) * 4
 * bytes (rounded up) must fit in KVQ_STATIC_SCRATCH_BYTES -- e.g. one layer of
 * the 262,144-key verify batch, or 16 layers at 65,536 keys with chunk 4,096.
 * Errors: those of kvq_decode_attn and kvq_merge_lse; UNSUPPORTED when the
 * partials exceed the array. */
kvq_status kvq_decode_merged_static(const kvq_layer *layers, int n_layers, const uint16_t *q,
                                    int n_q_heads, int T, int64_t n_kv, int chunk, float scale,
                                    float *out, float *lse, kvq_stream stream);

/* ---------------------------------------------------------------------- */
/* Housekeeping                                                            */
/* ---------------------------------------------------------------------- */

/* Bytes of the optional kvq_prefill_attn workspace that holds a slab for every
 * (layer, KV head) pair, for n_keys = n_cached + T keys: n_layers * n_kv_heads *
 * ceil(n_keys / 32) * 49,152 at head_dim 256 (n_layers = n_kv_heads = 1 gives
 * one slab, the smallest usable workspace); 0 when the shape has no
 * tensor-core path (head_dim != 256). */
size_t kvq_prefill_workspace_bytes(int n_layers, int n_kv_heads, int head_dim, int64_t n_keys);

#define KVQ_OP_DECODE 1
#define KVQ_OP_PREFILL 2
#define KVQ_OP_DECODE_STEP 3

/* Bytes of device workspace an operation requires (0 if none).
 * KVQ_OP_DECODE: always 0.  KVQ_OP_PREFILL: always 0 -- its workspace is
 * optional and its size depends on the key count, see
 * kvq_prefill_workspace_bytes.  KVQ_OP_DECODE_STEP: always 0.
 * Returns (size_t)-1 for an unknown op. */
size_t kvq_workspace_bytes(int op, int n_layers, int n_q_heads, int n_kv_heads, int T,
                           int head_dim);

/* Synchronise `stream`, then read and clear the device status word of the
 * current device.  KVQ_OK, KVQ_ERR_TIMEOUT (a bounded wait ran out in some
 * kernel since the last check) or KVQ_ERR_CUDA (an asynchronous CUDA error). */
kvq_status kvq_check(kvq_stream stream);

/* Static description of a status code (never NULL). */
const char *kvq_status_string(kvq_status status);

/* Thread-local detail of the last error returned on this thread ("" if none). */
const char *kvq_last_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int kvq_version(void);

/* ---------------------------------------------------------------------- */
/* Test hooks                                                              */
/* ---------------------------------------------------------------------- */

/* Process-wide switches for the library's own tests (all off by default; no
 * production caller sets them).  Each call reads them once (atomic loads); the
 * library reads no environment variables.
 *  decode_general     1: decode runs on the general kernel (kernel comparisons)
 *  decode_timeout     1: every decode launch waits on a barrier that nothing
 *                     completes, so its bounded wait runs out (about a second)
 *                     and kvq_check reports KVQ_ERR_TIMEOUT
 *  prefill_timeout    1: the same for the tensor-core prefill launches (the
 *                     tile expansion and the attention kernel)
 *  stream_fail_layer  >= 0: kvq_stream_decode fails the host-to-device copy of
 *                     this layer (a host-side injected fault); -1: off */
typedef struct kvq_test_hooks {
    int32_t decode_general;
    int32_t decode_timeout;
    int32_t prefill_timeout;
    int32_t stream_fail_layer;
} kvq_test_hooks;

/* Set the test hooks; NULL turns them all off.  Always KVQ_OK. */
kvq_status kvq_test_set_hooks(const kvq_test_hooks *hooks);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
