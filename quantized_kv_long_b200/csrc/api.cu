// api.cu -- the extern "C" entry points of libkvq (declared in kvq.h):
// argument validation, error reporting and dispatch to the kernels.
//
// Every entry point validates all of its arguments before it launches
// anything; on an error it returns the status and leaves a thread-local
// message for kvq_last_error().  Nothing here synchronises except kvq_check.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cmath>

#include "common.cuh"

namespace kvq {

// Status word written by kernels whose bounded waits run out.  Host code
// reaches it through the address cudaGetSymbolAddress reports for the
// current device (cached per device).
static __device__ unsigned int g_status_word;

static thread_local char t_err[512];

kvq_status set_error(kvq_status s, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_err, sizeof(t_err), fmt, ap);
    va_end(ap);
    return s;
}

kvq_status check_launch(const char *what)
{
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return set_error(KVQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return KVQ_OK;
}

kvq_status status_word(unsigned int **out)
{
    // one entry per device; two threads that look the address up at the same time
    // store the same value
    static std::atomic<unsigned int *> cache[MAX_DEVICES];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES)
        return set_error(KVQ_ERR_CUDA, "no current CUDA device");
    unsigned int *w = cache[dev].load(std::memory_order_acquire);
    if (!w) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_status_word);
        if (e != cudaSuccess)
            return set_error(KVQ_ERR_CUDA, "status word: %s", cudaGetErrorString(e));
        w = static_cast<unsigned int *>(p);
        cache[dev].store(w, std::memory_order_release);
    }
    *out = w;
    return KVQ_OK;
}

TestHooks &test_hooks()
{
    static TestHooks h;
    return h;
}

// ---- validation helpers ---------------------------------------------------

static kvq_status check_layers(const kvq_layer *layers, int n_layers, const char *fn)
{
    if (!layers)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: layers is NULL", fn);
    if (n_layers < 1 || n_layers > KVQ_MAX_LAYERS)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: n_layers=%d outside [1, %d]", fn, n_layers,
                         KVQ_MAX_LAYERS);
    const int H = layers[0].n_kv_heads, D = layers[0].head_dim;
    if (H < 1)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: n_kv_heads=%d", fn, H);
    if (D < QK || D % QK != 0)
        return set_error(KVQ_ERR_UNSUPPORTED, "%s: head_dim=%d is not a positive multiple of 32",
                         fn, D);
    if (D > 512)
        return set_error(KVQ_ERR_UNSUPPORTED, "%s: head_dim=%d > 512", fn, D);
    for (int l = 0; l < n_layers; ++l) {
        const kvq_layer &L = layers[l];
        for (const int t : {L.k_type, L.v_type})
            if (!known_type(t))
                return set_error(KVQ_ERR_INVALID_ARG, "%s: layer %d has block type %d", fn, l, t);
        if (k_type_of(L) != k_type_of(layers[0]) || v_type_of(L) != v_type_of(layers[0]))
            return set_error(KVQ_ERR_INVALID_ARG, "%s: layer %d differs in block formats", fn, l);
        if (!L.k || !L.v)
            return set_error(KVQ_ERR_INVALID_ARG, "%s: layer %d has a NULL cache pointer", fn, l);
        if (L.n_kv_heads != H || L.head_dim != D)
            return set_error(KVQ_ERR_INVALID_ARG, "%s: layer %d differs in heads/head_dim", fn, l);
        if (L.capacity < 1 || L.capacity % 8 != 0)
            return set_error(KVQ_ERR_INVALID_ARG, "%s: layer %d capacity=%lld not a positive "
                             "multiple of 8", fn, l, (long long)L.capacity);
        if (!aligned(L.k, 16) || !aligned(L.v, 16))
            return set_error(KVQ_ERR_ALIGNMENT, "%s: layer %d cache not 16-byte aligned", fn, l);
    }
    for (const int t : {k_type_of(layers[0]), v_type_of(layers[0])})
        if (D % block_elems(t) != 0)
            return set_error(KVQ_ERR_UNSUPPORTED, "%s: head_dim=%d is not a multiple of the "
                             "%d-element OSCAR2 block", fn, D, block_elems(t));
    return KVQ_OK;
}

template <typename P>
static kvq_status need(const P *p, uintptr_t align, const char *name, const char *fn)
{
    if (!p)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: %s is NULL", fn, name);
    if (!aligned(p, align))
        return set_error(KVQ_ERR_ALIGNMENT, "%s: %s not %d-byte aligned", fn, name, (int)align);
    return KVQ_OK;
}

#define KVQ_TRY(expr)                      \
    do {                                   \
        const kvq_status _s = (expr);      \
        if (_s != KVQ_OK)                  \
            return _s;                     \
    } while (0)

static void fill_table(const kvq_layer *layers, int n, LayerTable &t)
{
    for (int l = 0; l < KVQ_MAX_LAYERS; ++l) {
        t.k[l] = l < n ? static_cast<const uint8_t *>(layers[l].k) : nullptr;
        t.v[l] = l < n ? static_cast<const uint8_t *>(layers[l].v) : nullptr;
        t.cap[l] = l < n ? layers[l].capacity : 0;
    }
}

// Shared by kvq_decode_attn and kvq_stream_decode.
kvq_status validate_decode(const kvq_layer *layers, int n_layers, const uint16_t *q,
                           int n_q_heads, int T, int64_t n_kv, int chunk, float scale,
                           const float *out_part, const float *lse_part, const char *fn,
                           int64_t min_keys)
{
    KVQ_TRY(check_layers(layers, n_layers, fn));
    KVQ_TRY(need(q, 16, "q", fn));
    KVQ_TRY(need(out_part, 16, "out_part", fn));
    KVQ_TRY(need(lse_part, 4, "lse_part", fn));
    const int H = layers[0].n_kv_heads;
    if (n_q_heads < 1 || n_q_heads % H != 0)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: n_q_heads=%d not a multiple of n_kv_heads=%d",
                         fn, n_q_heads, H);
    if (T < 1)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: T=%d < 1", fn, T);
    if (T > KVQ_MAX_DECODE_T)
        return set_error(KVQ_ERR_UNSUPPORTED, "%s: T=%d > %d", fn, T, KVQ_MAX_DECODE_T);
    if ((n_q_heads / H) * T > 32)
        return set_error(KVQ_ERR_UNSUPPORTED, "%s: group*T=%d > 32 rows", fn,
                         (n_q_heads / H) * T);
    if (chunk < 64 || chunk % 64 != 0)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: chunk=%d not a positive multiple of 64", fn,
                         chunk);
    if (min_keys < 0)
        min_keys = T;
    if (n_kv < min_keys)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: n_kv=%lld < %lld", fn, (long long)n_kv,
                         (long long)min_keys);
    for (int l = 0; l < n_layers; ++l)
        if (n_kv > layers[l].capacity)
            return set_error(KVQ_ERR_INVALID_ARG, "%s: n_kv=%lld > capacity of layer %d", fn,
                             (long long)n_kv, l);
    if (!std::isfinite(scale))
        return set_error(KVQ_ERR_INVALID_ARG, "%s: scale is not finite", fn);
    if ((n_kv + chunk - 1) / chunk > (1ll << 30))
        return set_error(KVQ_ERR_INVALID_ARG, "%s: too many chunks", fn);
    return KVQ_OK;
}

static kvq_status fill_decode(const kvq_layer *layers, int n_layers, const uint16_t *q,
                              int n_q_heads, int T, int64_t n_kv, int chunk, float scale,
                              float *out_part, float *lse_part, DecodeArgs &a)
{
    a = DecodeArgs{};
    fill_table(layers, n_layers, a.layers);
    a.n_layers = n_layers;
    a.n_kv_heads = layers[0].n_kv_heads;
    a.head_dim = layers[0].head_dim;
    a.n_q_heads = n_q_heads;
    a.T = T;
    a.k_type = k_type_of(layers[0]);
    a.v_type = v_type_of(layers[0]);
    a.n_kv = n_kv;
    a.chunk = chunk;
    a.scale = scale;
    a.q = reinterpret_cast<const __half *>(q);
    a.out_part = out_part;
    a.lse_part = lse_part;
    a.vis_last = n_kv - T;
    KVQ_TRY(status_word(&a.status));
    // test hooks (kvq_test_set_hooks): the general kernel, a forced wait timeout
    a.force_simple = test_hooks().decode_general.load(std::memory_order_relaxed);
    a.test_timeout = test_hooks().decode_timeout.load(std::memory_order_relaxed);
    return KVQ_OK;
}

// Shared by kvq_decode_attn, kvq_stream_decode and kvq_decode_merged_static.
kvq_status enqueue_decode(const kvq_layer *layers, int n_layers, const uint16_t *q,
                          int n_q_heads, int T, int64_t n_kv, int chunk, float scale,
                          float *out_part, float *lse_part, cudaStream_t s)
{
    DecodeArgs a;
    KVQ_TRY(fill_decode(layers, n_layers, q, n_q_heads, T, n_kv, chunk, scale, out_part,
                        lse_part, a));
    if (!launch_decode(a, s))
        return set_error(KVQ_ERR_UNSUPPORTED, "kvq_decode_attn: no kernel for this shape");
    return check_launch("kvq_decode_attn");
}

kvq_status validate_merge(const float *out_part, const float *lse_part, int64_t rows,
                          int n_chunks, int head_dim, const float *out, const float *lse,
                          const char *fn)
{
    KVQ_TRY(need(out_part, 16, "out_part", fn));
    KVQ_TRY(need(lse_part, 4, "lse_part", fn));
    KVQ_TRY(need(out, 16, "out", fn));
    KVQ_TRY(need(lse, 4, "lse", fn));
    if (rows < 0 || rows >= (1ll << 31))
        return set_error(KVQ_ERR_INVALID_ARG, "%s: rows=%lld", fn, (long long)rows);
    if (n_chunks < 1)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: n_chunks=%d < 1", fn, n_chunks);
    if (head_dim < 4 || head_dim % 4 != 0)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: head_dim=%d not a positive multiple of 4", fn,
                         head_dim);
    return KVQ_OK;
}

}  // namespace kvq

using namespace kvq;

extern "C" {

kvq_status kvq_quantize_q8_0(const float *x, void *blocks, int64_t n, kvq_stream stream)
{
    const char *fn = "kvq_quantize_q8_0";
    if (n < 0 || n % QK != 0)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: n=%lld not a non-negative multiple of 32", fn,
                         (long long)n);
    if (n == 0)
        return KVQ_OK;
    KVQ_TRY(need(x, 4, "x", fn));
    KVQ_TRY(need(static_cast<const uint8_t *>(blocks), 2, "blocks", fn));
    launch_quantize_q8_0(x, static_cast<uint8_t *>(blocks), n, as_stream(stream));
    return check_launch(fn);
}

kvq_status kvq_quantize_q4_0(const float *x, void *blocks, int64_t n, kvq_stream stream)
{
    const char *fn = "kvq_quantize_q4_0";
    if (n < 0 || n % QK != 0)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: n=%lld not a non-negative multiple of 32", fn,
                         (long long)n);
    if (n == 0)
        return KVQ_OK;
    KVQ_TRY(need(x, 4, "x", fn));
    KVQ_TRY(need(static_cast<const uint8_t *>(blocks), 2, "blocks", fn));
    launch_quantize_q4_0(x, static_cast<uint8_t *>(blocks), n, as_stream(stream));
    return check_launch(fn);
}

kvq_status kvq_quantize_oscar2(const float *x, void *blocks, int64_t n, kvq_stream stream)
{
    const char *fn = "kvq_quantize_oscar2";
    if (n < 0 || n % QK_OSCAR2 != 0)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: n=%lld not a non-negative multiple of 128",
                         fn, (long long)n);
    if (n == 0)
        return KVQ_OK;
    KVQ_TRY(need(x, 4, "x", fn));
    KVQ_TRY(need(static_cast<const uint8_t *>(blocks), 4, "blocks", fn));
    launch_quantize_oscar2(x, static_cast<uint8_t *>(blocks), n, as_stream(stream));
    return check_launch(fn);
}

kvq_status kvq_append(const kvq_layer *layers, int n_layers, const float *k_new,
                      const float *v_new, int64_t pos, int n_tok, kvq_stream stream)
{
    const char *fn = "kvq_append";
    KVQ_TRY(check_layers(layers, n_layers, fn));
    KVQ_TRY(need(k_new, 16, "k_new", fn));
    KVQ_TRY(need(v_new, 16, "v_new", fn));
    if (n_tok < 1)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: n_tok=%d < 1", fn, n_tok);
    if (pos < 0)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: pos=%lld < 0", fn, (long long)pos);
    for (int l = 0; l < n_layers; ++l)
        if (pos + n_tok > layers[l].capacity)
            return set_error(KVQ_ERR_INVALID_ARG, "%s: rows [%lld, %lld) exceed capacity of "
                             "layer %d", fn, (long long)pos, (long long)(pos + n_tok), l);
    const int H = layers[0].n_kv_heads, D = layers[0].head_dim;
    if ((int64_t)n_layers * n_tok * H >= (1ll << 31))
        return set_error(KVQ_ERR_INVALID_ARG, "%s: too many rows in one call", fn);
    if (2 * (D / QK) * 32 > 1024)
        return set_error(KVQ_ERR_UNSUPPORTED, "%s: head_dim=%d", fn, D);
    MutLayerTable t;
    for (int l = 0; l < KVQ_MAX_LAYERS; ++l) {
        t.k[l] = l < n_layers ? static_cast<uint8_t *>(layers[l].k) : nullptr;
        t.v[l] = l < n_layers ? static_cast<uint8_t *>(layers[l].v) : nullptr;
        t.cap[l] = l < n_layers ? layers[l].capacity : 0;
    }
    launch_append(t, n_layers, H, D, k_type_of(layers[0]), v_type_of(layers[0]), k_new, v_new,
                  pos, n_tok, as_stream(stream));
    return check_launch(fn);
}

kvq_status kvq_decode_attn(const kvq_layer *layers, int n_layers, const uint16_t *q,
                           int n_q_heads, int T, int64_t n_kv, int chunk, float scale,
                           float *out_part, float *lse_part, kvq_stream stream)
{
    KVQ_TRY(validate_decode(layers, n_layers, q, n_q_heads, T, n_kv, chunk, scale, out_part,
                            lse_part, "kvq_decode_attn"));
    return enqueue_decode(layers, n_layers, q, n_q_heads, T, n_kv, chunk, scale, out_part,
                          lse_part, as_stream(stream));
}

kvq_status kvq_decode_attn_shard(const kvq_layer *layers, int n_layers, const uint16_t *q,
                                 int n_q_heads, int T, int64_t n_keys, int64_t key0,
                                 int64_t n_kv, int chunk, float scale, float *out_part,
                                 float *lse_part, kvq_stream stream)
{
    const char *fn = "kvq_decode_attn_shard";
    KVQ_TRY(validate_decode(layers, n_layers, q, n_q_heads, T, n_keys, chunk, scale, out_part,
                            lse_part, fn, 1));
    if (key0 < 0 || n_kv < T || key0 > n_kv - n_keys)
        return set_error(KVQ_ERR_INVALID_ARG,
                         "%s: keys [%lld, %lld) not inside a context of n_kv=%lld >= T=%d", fn,
                         (long long)key0, (long long)(key0 + n_keys), (long long)n_kv, T);
    DecodeArgs a;
    KVQ_TRY(fill_decode(layers, n_layers, q, n_q_heads, T, n_keys, chunk, scale, out_part,
                        lse_part, a));
    a.vis_last = n_kv - T - key0;  // token t sees global keys <= n_kv - T + t
    if (!launch_decode(a, as_stream(stream)))
        return set_error(KVQ_ERR_UNSUPPORTED, "%s: no kernel for this shape", fn);
    return check_launch(fn);
}

kvq_status kvq_merge_lse(const float *out_part, const float *lse_part, int64_t rows,
                         int n_chunks, int head_dim, float *out, float *lse, kvq_stream stream)
{
    const char *fn = "kvq_merge_lse";
    KVQ_TRY(validate_merge(out_part, lse_part, rows, n_chunks, head_dim, out, lse, fn));
    launch_merge_lse(out_part, lse_part, rows, n_chunks, head_dim, out, lse, as_stream(stream));
    return check_launch(fn);
}

kvq_status kvq_merge_lse_parts(const float *out_parts, const float *lse_parts, int n_parts,
                               int64_t rows, int head_dim, float *out, float *lse,
                               kvq_stream stream)
{
    const char *fn = "kvq_merge_lse_parts";
    KVQ_TRY(validate_merge(out_parts, lse_parts, rows, n_parts, head_dim, out, lse, fn));
    launch_merge_lse_parts(out_parts, lse_parts, n_parts, rows, head_dim, out, lse,
                           as_stream(stream));
    return check_launch(fn);
}

kvq_status kvq_decode_step(const kvq_layer *layers, int n_layers, const float *k_new,
                           const float *v_new, const uint16_t *q, int n_q_heads, int T,
                           int64_t n_kv, int chunk, float scale, float *out_part,
                           float *lse_part, float *out, float *lse, void *workspace,
                           size_t ws_bytes, kvq_stream stream)
{
    (void)workspace;  // reserved: the step needs none
    (void)ws_bytes;
    const char *fn = "kvq_decode_step";
    KVQ_TRY(validate_decode(layers, n_layers, q, n_q_heads, T, n_kv, chunk, scale, out_part,
                            lse_part, fn));
    KVQ_TRY(need(k_new, 16, "k_new", fn));
    KVQ_TRY(need(v_new, 16, "v_new", fn));
    const int D = layers[0].head_dim;
    const int64_t rows = (int64_t)n_layers * T * n_q_heads;
    const int n_chunks = (int)((n_kv + chunk - 1) / chunk);
    KVQ_TRY(validate_merge(out_part, lse_part, rows, n_chunks, D, out, lse, fn));
    DecodeArgs a;
    KVQ_TRY(fill_decode(layers, n_layers, q, n_q_heads, T, n_kv, chunk, scale, out_part,
                        lse_part, a));
    const cudaStream_t s = as_stream(stream);
    KVQ_TRY(kvq_append(layers, n_layers, k_new, v_new, n_kv - T, T, stream));
    if (!launch_decode(a, s))
        return set_error(KVQ_ERR_UNSUPPORTED, "%s: no kernel for this shape", fn);
    KVQ_TRY(check_launch(fn));
    launch_merge_lse(out_part, lse_part, rows, n_chunks, D, out, lse, s);
    return check_launch(fn);
}

kvq_status kvq_decode_step_host(const kvq_layer *layers, int n_layers, const float *k_host,
                                const float *v_host, const uint16_t *q_host, float *out_host,
                                float *lse_host, float *k_new, float *v_new, uint16_t *q,
                                int n_q_heads, int T, int64_t n_kv, int chunk, float scale,
                                float *out_part, float *lse_part, float *out, float *lse,
                                kvq_stream stream)
{
    const char *fn = "kvq_decode_step_host";
    if (!k_host || !v_host || !q_host || !out_host || !lse_host)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: a host buffer is NULL", fn);
    // the device-side arguments are those of kvq_decode_step: check them all before
    // the first copy
    KVQ_TRY(validate_decode(layers, n_layers, q, n_q_heads, T, n_kv, chunk, scale, out_part,
                            lse_part, fn));
    KVQ_TRY(need(k_new, 16, "k_new", fn));
    KVQ_TRY(need(v_new, 16, "v_new", fn));
    const int H = layers[0].n_kv_heads, D = layers[0].head_dim;
    const int64_t rows = (int64_t)n_layers * T * n_q_heads;
    const int n_chunks = (int)((n_kv + chunk - 1) / chunk);
    KVQ_TRY(validate_merge(out_part, lse_part, rows, n_chunks, D, out, lse, fn));
    const cudaStream_t s = as_stream(stream);
    const size_t kv_bytes = (size_t)n_layers * T * H * D * sizeof(float);
    const struct {
        void *dst;
        const void *src;
        size_t bytes;
        const char *what;
    } in[3] = {{q, q_host, (size_t)rows * D * sizeof(uint16_t), "q"},
               {k_new, k_host, kv_bytes, "k"},
               {v_new, v_host, kv_bytes, "v"}};
    for (const auto &c : in)
        if (cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return set_error(KVQ_ERR_COPY, "%s: host-to-device copy of %s: %s", fn, c.what,
                             cudaGetErrorString(cudaGetLastError()));
    KVQ_TRY(kvq_decode_step(layers, n_layers, k_new, v_new, q, n_q_heads, T, n_kv, chunk, scale,
                            out_part, lse_part, out, lse, nullptr, 0, stream));
    if (cudaMemcpyAsync(out_host, out, (size_t)rows * D * sizeof(float), cudaMemcpyDeviceToHost,
                        s) != cudaSuccess ||
        cudaMemcpyAsync(lse_host, lse, (size_t)rows * sizeof(float), cudaMemcpyDeviceToHost,
                        s) != cudaSuccess)
        return set_error(KVQ_ERR_COPY, "%s: device-to-host copy of the results: %s", fn,
                         cudaGetErrorString(cudaGetLastError()));
    return KVQ_OK;
}

kvq_status kvq_prefill_attn(const kvq_layer *layers, int n_layers, const uint16_t *q,
                            int n_q_heads, int T, int64_t n_cached, int page, float scale,
                            float *out, float *lse, float *page_out, float *page_lse,
                            void *workspace, size_t ws_bytes, kvq_stream stream)
{
    const char *fn = "kvq_prefill_attn";
    KVQ_TRY(check_layers(layers, n_layers, fn));
    KVQ_TRY(need(q, 16, "q", fn));
    KVQ_TRY(need(out, 16, "out", fn));
    KVQ_TRY(need(lse, 4, "lse", fn));
    if ((page_out == nullptr) != (page_lse == nullptr))
        return set_error(KVQ_ERR_INVALID_ARG, "%s: page_out and page_lse must both be set or "
                         "both be NULL", fn);
    if (page_out) {
        KVQ_TRY(need(page_out, 16, "page_out", fn));
        KVQ_TRY(need(page_lse, 4, "page_lse", fn));
    }
    const int H = layers[0].n_kv_heads, D = layers[0].head_dim;
    if (n_q_heads < 1 || n_q_heads % H != 0)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: n_q_heads=%d not a multiple of n_kv_heads=%d",
                         fn, n_q_heads, H);
    if (T < 1)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: T=%d < 1", fn, T);
    if (n_cached < 0)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: n_cached < 0", fn);
    if (page < 128 || page % 128 != 0)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: page=%d not a positive multiple of 128", fn,
                         page);
    for (int l = 0; l < n_layers; ++l)
        if (n_cached + T > layers[l].capacity)
            return set_error(KVQ_ERR_INVALID_ARG, "%s: n_cached + T exceeds capacity of layer %d",
                             fn, l);
    if (!std::isfinite(scale))
        return set_error(KVQ_ERR_INVALID_ARG, "%s: scale is not finite", fn);
    if (!prefill_supported(n_q_heads, H, D))
        return set_error(KVQ_ERR_UNSUPPORTED, "%s: head_dim=%d, group=%d not supported", fn, D,
                         n_q_heads / H);
    const size_t ws = prefill_workspace_bytes(n_layers, n_q_heads, H, T, D);
    if (ws > 0 && (workspace == nullptr || ws_bytes < ws))
        return set_error(KVQ_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn,
                         ws, workspace ? ws_bytes : (size_t)0);
    if (ws > 0 && !aligned(workspace, 256))
        return set_error(KVQ_ERR_ALIGNMENT, "%s: workspace not 256-byte aligned", fn);
    PrefillArgs a;
    fill_table(layers, n_layers, a.layers);
    a.n_layers = n_layers;
    a.n_kv_heads = H;
    a.head_dim = D;
    a.n_q_heads = n_q_heads;
    a.T = T;
    a.n_cached = n_cached;
    a.page = page;
    a.scale = scale;
    a.q = reinterpret_cast<const __half *>(q);
    a.out = out;
    a.lse = lse;
    a.page_out = page_out;
    a.page_lse = page_lse;
    a.k_type = k_type_of(layers[0]);
    a.v_type = v_type_of(layers[0]);
    // optional workspace: the f16 key tiles of the tensor-core path, expanded once
    a.workspace = nullptr;
    a.ws_bytes = 0;
    const size_t slab = prefill_slab_bytes(D, n_cached + T);
    if (workspace != nullptr && slab > 0) {
        if (ws_bytes < slab)
            return set_error(KVQ_ERR_WORKSPACE,
                             "%s: workspace of %zu bytes given, one (layer, KV head) of expanded "
                             "key tiles needs %zu; pass NULL to dequantize in place",
                             fn, ws_bytes, slab);
        if (!aligned(workspace, 256))
            return set_error(KVQ_ERR_ALIGNMENT, "%s: workspace not 256-byte aligned", fn);
        a.workspace = workspace;
        a.ws_bytes = ws_bytes;
    }
    KVQ_TRY(status_word(&a.status));
    a.test_timeout = test_hooks().prefill_timeout.load(std::memory_order_relaxed);
    if (!launch_prefill(a, as_stream(stream)))
        return set_error(KVQ_ERR_CUDA, "%s: setting up the second stream of the chunked "
                         "expansion failed", fn);
    KVQ_TRY(check_launch(fn));
    if (page_out) {
        // the kernels wrote the per-page partials; out and lse are their merge
        const int64_t rows = (int64_t)n_layers * T * n_q_heads;
        const int n_pages = (int)((n_cached + T + page - 1) / page);
        launch_merge_lse(page_out, page_lse, rows, n_pages, D, out, lse, as_stream(stream));
        KVQ_TRY(check_launch(fn));
    }
    return KVQ_OK;
}

size_t kvq_prefill_workspace_bytes(int n_layers, int n_kv_heads, int head_dim, int64_t n_keys)
{
    return prefill_expand_bytes(n_layers, n_kv_heads, head_dim, n_keys);
}

size_t kvq_workspace_bytes(int op, int n_layers, int n_q_heads, int n_kv_heads, int T,
                           int head_dim)
{
    if (op == KVQ_OP_DECODE)
        return 0;
    if (op == KVQ_OP_DECODE_STEP)
        return 0;
    if (op == KVQ_OP_PREFILL)
        return 0;  // required: none (the optional workspace: kvq_prefill_workspace_bytes)
    return (size_t)-1;
}

kvq_status kvq_check(kvq_stream stream)
{
    cudaError_t e = cudaStreamSynchronize(as_stream(stream));
    if (e != cudaSuccess)
        return set_error(KVQ_ERR_CUDA, "kvq_check: %s", cudaGetErrorString(e));
    unsigned int *w = nullptr;
    KVQ_TRY(status_word(&w));
    unsigned int v = 0;
    e = cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess)
        return set_error(KVQ_ERR_CUDA, "kvq_check: %s", cudaGetErrorString(e));
    if (v != 0) {
        const unsigned int zero = 0;
        cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice);
        if (v & STATUS_TIMEOUT)
            return set_error(KVQ_ERR_TIMEOUT, "kvq_check: a bounded device wait ran out");
    }
    return KVQ_OK;
}

const char *kvq_status_string(kvq_status s)
{
    switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_ALIGNMENT: return "misaligned pointer";
    case KVQ_ERR_UNSUPPORTED: return "unsupported shape";
    case KVQ_ERR_CUDA: return "CUDA error";
    case KVQ_ERR_TIMEOUT: return "device wait timed out";
    case KVQ_ERR_COPY: return "copy could not be enqueued";
    case KVQ_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

const char *kvq_last_error(void) { return t_err; }

int kvq_version(void) { return 100; }

kvq_status kvq_test_set_hooks(const kvq_test_hooks *hooks)
{
    TestHooks &h = test_hooks();
    h.decode_general.store(hooks ? hooks->decode_general : 0);
    h.decode_timeout.store(hooks ? hooks->decode_timeout : 0);
    h.prefill_timeout.store(hooks ? hooks->prefill_timeout : 0);
    h.stream_fail_layer.store(hooks ? hooks->stream_fail_layer : -1);
    return KVQ_OK;
}

}  // extern "C"
