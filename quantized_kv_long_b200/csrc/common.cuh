// common.cuh -- shared definitions of the CUDA library (not of the oracle).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <type_traits>

#include "kvq.h"

namespace kvq {

constexpr int QK = 32;           // elements per Q8_0 / Q4_0 block
constexpr int Q8_0_BYTES = 34;   // fp16 d + 32 x int8
constexpr int Q4_0_BYTES = 18;   // fp16 d + 16 bytes of nibbles
constexpr int QK_OSCAR2 = 128;   // elements per OSCAR2 block
constexpr int OSCAR2_BYTES = 36; // fp16 d + fp16 m + 32 bytes of 2-bit codes

// Block formats (kvq_type resolved: KVQ_TYPE_DEFAULT becomes Q8_0 for K, Q4_0 for V).
__host__ __device__ constexpr int block_elems(int type) { return type == KVQ_TYPE_OSCAR2 ? QK_OSCAR2 : QK; }
__host__ __device__ constexpr int block_bytes(int type)
{
    return type == KVQ_TYPE_Q8_0 ? Q8_0_BYTES : type == KVQ_TYPE_Q4_0 ? Q4_0_BYTES : OSCAR2_BYTES;
}
__host__ __device__ inline int64_t row_bytes(int type, int head_dim)
{
    return (int64_t)(head_dim / block_elems(type)) * block_bytes(type);
}

// Every block decodes as x^ = d * code + m.  Integer code of element i of a block:
// int8 q (Q8_0); nibble - 8 (Q4_0: byte i holds element i in the low nibble and
// element i + 16 in the high); the 2-bit u (OSCAR2: byte 4 + j holds elements j,
// j + 32, j + 64, j + 96 in bits 0-1, 2-3, 4-5, 6-7).
template <int TYPE>
__device__ __forceinline__ int block_int(const uint8_t *blk, int i)
{
    if (TYPE == KVQ_TYPE_Q8_0)
        return (int)(int8_t)blk[2 + i];
    if (TYPE == KVQ_TYPE_OSCAR2)
        return (blk[4 + (i & 31)] >> (2 * (i >> 5))) & 3;
    const uint8_t byte = blk[2 + (i & 15)];
    return (i < 16 ? (byte & 15) : (byte >> 4)) - 8;
}

// The block's fp16 scale d (first two bytes, little-endian) as fp32.
__device__ __forceinline__ float block_d(const uint8_t *blk)
{
    return __half2float(__ushort_as_half((unsigned short)(blk[0] | (blk[1] << 8))));
}

// The block's offset m as fp32: the fp16 zero-point in bytes 2-3 of an OSCAR2
// block, 0 for the symmetric formats.
template <int TYPE>
__device__ __forceinline__ float block_m(const uint8_t *blk)
{
    if (TYPE != KVQ_TYPE_OSCAR2)
        return 0.0f;
    return __half2float(__ushort_as_half((unsigned short)(blk[2] | (blk[3] << 8))));
}

// Calls f(K, V) with K, V = std::integral_constant<int, format> for the resolved
// formats kt, vt, so that a launcher can instantiate a kernel per format pair;
// returns f's result, or false for an unknown format.
template <typename F>
bool launch_for_types(int kt, int vt, F &&f)
{
    using Q8 = std::integral_constant<int, KVQ_TYPE_Q8_0>;
    using Q4 = std::integral_constant<int, KVQ_TYPE_Q4_0>;
    using O2 = std::integral_constant<int, KVQ_TYPE_OSCAR2>;
    auto with_v = [&](auto k) -> bool {
        switch (vt) {
        case KVQ_TYPE_Q8_0: return f(k, Q8{});
        case KVQ_TYPE_Q4_0: return f(k, Q4{});
        case KVQ_TYPE_OSCAR2: return f(k, O2{});
        default: return false;
        }
    };
    switch (kt) {
    case KVQ_TYPE_Q8_0: return with_v(Q8{});
    case KVQ_TYPE_Q4_0: return with_v(Q4{});
    case KVQ_TYPE_OSCAR2: return with_v(O2{});
    default: return false;
    }
}

// Whether a block type is one of the formats (resolved or KVQ_TYPE_DEFAULT).
inline bool known_type(int t)
{
    return t == KVQ_TYPE_DEFAULT || t == KVQ_TYPE_Q8_0 || t == KVQ_TYPE_Q4_0 ||
           t == KVQ_TYPE_OSCAR2;
}
inline int k_type_of(const kvq_layer &l) { return l.k_type ? l.k_type : KVQ_TYPE_Q8_0; }
inline int v_type_of(const kvq_layer &l) { return l.v_type ? l.v_type : KVQ_TYPE_Q4_0; }

// Layer table passed by value as a kernel parameter.
struct LayerTable {
    const uint8_t *k[KVQ_MAX_LAYERS];
    const uint8_t *v[KVQ_MAX_LAYERS];
    int64_t cap[KVQ_MAX_LAYERS];
};

struct MutLayerTable {
    uint8_t *k[KVQ_MAX_LAYERS];
    uint8_t *v[KVQ_MAX_LAYERS];
    int64_t cap[KVQ_MAX_LAYERS];
};

// Device status word: bit flags set by kernels whose bounded waits ran out.
// Kernels receive its address as a parameter (see status_word()).
constexpr unsigned STATUS_TIMEOUT = 1u;

__device__ __forceinline__ void report_timeout(unsigned int *status)
{
    atomicOr(status, STATUS_TIMEOUT);
}

// Bounded spin limit for any device-side wait (iterations of a try_wait loop).
constexpr long long SPIN_LIMIT = 1ll << 26;

// ---- test hooks (host): set only through kvq_test_set_hooks -------------------
struct TestHooks {
    std::atomic<int> decode_general{0}, decode_timeout{0}, prefill_timeout{0},
        stream_fail_layer{-1};
};
TestHooks &test_hooks();

// ---- error plumbing (host) ------------------------------------------------
kvq_status set_error(kvq_status s, const char *fmt, ...);
kvq_status check_launch(const char *what);
kvq_status status_word(unsigned int **out);  // address of the current device's word

// Dynamic shared memory limit of a kernel: raises it on the current device to at
// least `bytes`, remembering the largest value set per device in `done` (one
// array per kernel); safe to call from several host threads.
constexpr int MAX_DEVICES = 64;
inline bool ensure_smem(const void *kernel, std::atomic<int> (&done)[MAX_DEVICES], int bytes)
{
    if (bytes <= 48 * 1024)
        return true;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES)
        return false;
    if (done[dev].load(std::memory_order_acquire) >= bytes)
        return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
        return false;
    int seen = done[dev].load(std::memory_order_relaxed);
    while (seen < bytes && !done[dev].compare_exchange_weak(seen, bytes, std::memory_order_release))
    {
    }
    return true;
}

inline bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }
inline cudaStream_t as_stream(kvq_stream s) { return reinterpret_cast<cudaStream_t>(s); }

// ---- launchers (host, internal) -------------------------------------------
void launch_quantize_q8_0(const float *x, uint8_t *blocks, int64_t n, cudaStream_t s);
void launch_quantize_q4_0(const float *x, uint8_t *blocks, int64_t n, cudaStream_t s);
void launch_quantize_oscar2(const float *x, uint8_t *blocks, int64_t n, cudaStream_t s);
void launch_append(const MutLayerTable &t, int n_layers, int n_kv_heads, int head_dim,
                   int k_type, int v_type, const float *k_new, const float *v_new, int64_t pos,
                   int n_tok, cudaStream_t s);
void launch_merge_lse(const float *out_part, const float *lse_part, int64_t rows, int n_chunks,
                      int head_dim, float *out, float *lse, cudaStream_t s);
void launch_merge_lse_parts(const float *out_parts, const float *lse_parts, int n_parts,
                            int64_t rows, int head_dim, float *out, float *lse, cudaStream_t s);

struct DecodeArgs {
    LayerTable layers;
    int n_layers, n_kv_heads, head_dim, n_q_heads, T;
    int k_type, v_type;  // resolved block formats (KVQ_TYPE_Q8_0 / _Q4_0 / _OSCAR2)
    int64_t n_kv;
    // causal visibility: the row of token t sees the keys (rows of the layers) j <=
    // vis_last + t; n_kv - T for a whole context, less for a shard of one
    int64_t vis_last;
    int chunk;
    float scale;
    const __half *q;
    float *out_part, *lse_part;
    unsigned int *status;  // device status word (bounded waits that ran out)
    int force_simple;      // host test hook: use the general kernel
    int test_timeout;      // host test hook: make the first wait run out
};
// Returns false (and launches nothing) if no kernel supports the shape.
bool launch_decode(const DecodeArgs &a, cudaStream_t s);

// Argument checks and the decode launch shared by the C ABI's decode entry points
// (api.cu).  validate_decode: n_kv must be at least min_keys (T when negative).
kvq_status validate_decode(const kvq_layer *layers, int n_layers, const uint16_t *q,
                           int n_q_heads, int T, int64_t n_kv, int chunk, float scale,
                           const float *out_part, const float *lse_part, const char *fn,
                           int64_t min_keys = -1);
kvq_status enqueue_decode(const kvq_layer *layers, int n_layers, const uint16_t *q,
                          int n_q_heads, int T, int64_t n_kv, int chunk, float scale,
                          float *out_part, float *lse_part, cudaStream_t s);
kvq_status validate_merge(const float *out_part, const float *lse_part, int64_t rows,
                          int n_chunks, int head_dim, const float *out, const float *lse,
                          const char *fn);
// True for the shapes of the persistent tensor-core kernel.
bool decode_tc_supported(const DecodeArgs &a);

struct PrefillArgs {
    LayerTable layers;
    int n_layers, n_kv_heads, head_dim, n_q_heads, T;
    int64_t n_cached;
    int page;
    float scale;
    const __half *q;
    float *out, *lse, *page_out, *page_lse;
    void *workspace;
    size_t ws_bytes;
    unsigned int *status;
    int test_timeout;  // test hook: one bounded wait of each tensor-core launch runs out
    int pair0;         // first (layer, KV head) pair, layer * n_kv_heads + head, of a launch
    int k_type, v_type;  // block formats (KVQ_TYPE_Q8_0 / _Q4_0 / _OSCAR2)
};
size_t prefill_workspace_bytes(int n_layers, int n_q_heads, int n_kv_heads, int T, int head_dim);
// Optional workspace of the tensor-core path: the f16 key tiles expanded once per
// call (0 if the shape has no such path).  n_keys = n_cached + T.
size_t prefill_expand_bytes(int n_layers, int n_kv_heads, int head_dim, int64_t n_keys);
// One (layer, KV head) pair's expanded key tiles: the smallest usable workspace.
size_t prefill_slab_bytes(int head_dim, int64_t n_keys);
bool prefill_supported(int n_q_heads, int n_kv_heads, int head_dim);
// false: a stream or event for the chunked expansion could not be set up.
bool launch_prefill(const PrefillArgs &a, cudaStream_t s);

}  // namespace kvq
