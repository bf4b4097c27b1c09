// quant.cu -- quantize-on-append: fp32 rows -> Q8_0 (K) and Q4_0 (V) blocks, or
// either tensor in any of the block formats.
//
// One warp quantizes one block: lane i holds element i of a 32-element block
// (elements i + 32 k of a 128-element OSCAR2 block), the block extremes come
// from warp shuffles, and every arithmetic step is an explicitly
// rounded fp32 operation (__fdiv_rn, __fmul_rn, __fadd_rn) so that no
// multiply-add is contracted and the blocks are bit-identical to any other
// IEEE implementation of the same definition.
//
// Definitions (llama.cpp-style blocks; sizes from the "Compression Ratios"
// table of the OSCAR2 KV-cache benchmark page and the 26,624 B/token of "Why
// it matters" on the ROCm KV-streaming page; the rules are the plainest
// reading of "d = amax/127, int8 round-to-nearest" and "d = max/-8, nibbles
// q+8 clamped to 0..15"):
//   Q8_0: d = amax/127; id = d ? 1/d : 0; q = roundf(x*id)  (ties away from 0)
//   Q4_0: m = signed first max-|x| element (+0 if the block is all zeros);
//         d = m/-8; id = d ? 1/d : 0; u = min(15, trunc(x*id + 8.5));
//         byte j = u_j | u_{j+16} << 4
//   OSCAR2 (36 B per 128 elements, "OSCAR2 KV Cache benchmark", Compression
//   Ratios table; rule and layout are this library's reading):
//         mn, mx = block min / max; d = (mx - mn)/3; id = d ? 1/d : 0;
//         u = min(3, trunc((x - mn)*id + 0.5)); fp16(mn) stored after fp16(d);
//         byte 4 + j = u_j | u_{j+32} << 2 | u_{j+64} << 4 | u_{j+96} << 6
//   fp16(d) stored first, little-endian.
#include "common.cuh"
#include "quant.cuh"

namespace kvq {

// One warp quantizes the block that starts at `src` into `dst` (lane = threadIdx % 32).
template <int TYPE>
__device__ __forceinline__ void warp_quant(const float *src, uint8_t *dst, int lane)
{
    if (TYPE == KVQ_TYPE_OSCAR2) {
        const float x[4] = {src[lane], src[lane + 32], src[lane + 64], src[lane + 96]};
        warp_quant_oscar2(x, dst, lane);
    } else if (TYPE == KVQ_TYPE_Q8_0) {
        warp_quant_q8_0(src[lane], dst, lane);
    } else {
        warp_quant_q4_0(src[lane], dst, lane);
    }
}

template <int TYPE>
__global__ void quantize_kernel(const float *__restrict__ x, uint8_t *__restrict__ blocks,
                                int64_t n_blocks)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t b = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); b < n_blocks;
         b += warps)
        warp_quant<TYPE>(x + b * block_elems(TYPE), blocks + b * block_bytes(TYPE), lane);
}

static int quant_grid(int64_t n_blocks)
{
    const int64_t per_cta = 8;  // 256 threads
    int64_t g = (n_blocks + per_cta - 1) / per_cta;
    const int64_t cap = 148 * 16;
    return (int)(g < cap ? (g > 0 ? g : 1) : cap);
}

void launch_quantize_q8_0(const float *x, uint8_t *blocks, int64_t n, cudaStream_t s)
{
    const int64_t nb = n / QK;
    quantize_kernel<KVQ_TYPE_Q8_0><<<quant_grid(nb), 256, 0, s>>>(x, blocks, nb);
}

void launch_quantize_q4_0(const float *x, uint8_t *blocks, int64_t n, cudaStream_t s)
{
    const int64_t nb = n / QK;
    quantize_kernel<KVQ_TYPE_Q4_0><<<quant_grid(nb), 256, 0, s>>>(x, blocks, nb);
}

void launch_quantize_oscar2(const float *x, uint8_t *blocks, int64_t n, cudaStream_t s)
{
    const int64_t nb = n / QK_OSCAR2;
    quantize_kernel<KVQ_TYPE_OSCAR2><<<quant_grid(nb), 256, 0, s>>>(x, blocks, nb);
}

// Append: one CTA per (layer, token, kv head); warps [0, nb) quantize the K
// blocks of the head-row, warps [nb, 2 nb) the V blocks (nb = head_dim / 32),
// each tensor in its block format (an OSCAR2 tensor has head_dim / 128 blocks:
// its warps b >= head_dim / 128 have none).
__global__ void append_kernel(MutLayerTable t, int n_kv_heads, int head_dim, int k_type,
                              int v_type, const float *__restrict__ k_new,
                              const float *__restrict__ v_new, int64_t pos, int n_tok)
{
    const int h = blockIdx.x % n_kv_heads;
    const int tok = (blockIdx.x / n_kv_heads) % n_tok;
    const int layer = blockIdx.x / (n_kv_heads * n_tok);
    const int nb = head_dim / QK;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool is_v = w >= nb;
    const int b = is_v ? w - nb : w;
    const int type = is_v ? v_type : k_type;  // uniform across the warp
    if (b * block_elems(type) >= head_dim)
        return;  // a warp without a block (OSCAR2), uniform across the warp
    const size_t src = (((size_t)layer * n_tok + tok) * n_kv_heads + h) * head_dim +
                       (size_t)b * block_elems(type);
    const int64_t row = (int64_t)h * t.cap[layer] + pos + tok;
    uint8_t *dst = (is_v ? t.v[layer] : t.k[layer]) + row * row_bytes(type, head_dim) +
                   (int64_t)b * block_bytes(type);
    const float *x = (is_v ? v_new : k_new) + src;
    if (type == KVQ_TYPE_Q8_0)
        warp_quant<KVQ_TYPE_Q8_0>(x, dst, lane);
    else if (type == KVQ_TYPE_Q4_0)
        warp_quant<KVQ_TYPE_Q4_0>(x, dst, lane);
    else
        warp_quant<KVQ_TYPE_OSCAR2>(x, dst, lane);
}

void launch_append(const MutLayerTable &t, int n_layers, int n_kv_heads, int head_dim,
                   int k_type, int v_type, const float *k_new, const float *v_new, int64_t pos,
                   int n_tok, cudaStream_t s)
{
    const int64_t ctas = (int64_t)n_layers * n_tok * n_kv_heads;
    const int threads = 2 * (head_dim / QK) * 32;
    // grid.x is at most 2^31-1; n_tok is an int and n_layers <= 64, heads small
    append_kernel<<<(unsigned)ctas, threads, 0, s>>>(t, n_kv_heads, head_dim, k_type, v_type,
                                                     k_new, v_new, pos, n_tok);
}

}  // namespace kvq
