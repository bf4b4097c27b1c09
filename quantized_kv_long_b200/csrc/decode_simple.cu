// decode_simple.cu -- the general split-KV decode attention: any head_dim
// (a multiple of 32, at most 512), up to 32 rows (GQA group x tokens) per KV
// head, every pair of block formats.
//
// The general path of kvq_decode_attn: it serves the shapes and formats the
// persistent tensor-core kernel (decode_tmem.cu) does not cover.  One CTA of
// 256 threads per (chunk, KV head, layer); the chunk's keys in tiles of 32:
//  0. the tile's K and V head-rows are dequantized once into shared memory as
//     fp32, x^ = d * code + m per element (m = 0 but for OSCAR2 blocks); K rows
//     with a pitch of head_dim + 4 floats, so that the 8 lanes of a
//     quarter-warp that read 16-byte words of 8 different keys hit 8 disjoint
//     groups of banks;
//  1. scores: warp w owns rows w, w + 8, w + 16, w + 24 and lane jj the key
//     j0 + jj; s = scale * q . k^, each K word loaded once for all of the
//     warp's rows and the q words read as broadcasts;
//  2. in the same warp, the online softmax of each row over the tile (max and
//     sum by shuffles): p to shared memory and the row's rescale factor;
//  3. P V: thread (slot, i4) owns head dims 4 i4 .. 4 i4 + 3 of the rows
//     slot, slot + NS, ... (NS = 256 / (head_dim / 4) row slots) and keeps
//     their accumulators in registers; each V word is loaded once for all of
//     its rows and p is read as a broadcast.
// Only fp32 rounding separates it from the exact result.
//
// Semantics (speculative-decoding paragraph of the RX 9070 XT KV-streaming
// page: paged decode attention over the verify batch; "Known Issues Fixed" of
// the OSCAR2 page: the max covers complete scores; GQA section of the KV-cache
// guide): row r = t*G + g is query head h*G + g of token t and sees keys
// j <= vis_last + t (n_kv - T + t for a whole context) of chunk c = keys
// [c*chunk, (c+1)*chunk).
#include "common.cuh"

namespace kvq {

constexpr int GEN_THREADS = 256;
constexpr int GEN_TILE = 32;      // keys per tile (a chunk is a multiple of 64 keys)
constexpr int GEN_ROWS = 32;      // rows per KV head the kernel holds
constexpr int GEN_ITEMS = 16;     // P V rows per thread: 32 rows over >= 2 row slots

// Dequantizes keys [j0, j0 + GEN_TILE) of a head's rows (`base`, `rb` bytes per
// head-row) in block format TYPE into dst[jj * pitch + i] as fp32; keys at or
// past c1 become zeros (their weights are 0, and 0 * 0 stays 0 in P V).
template <int TYPE>
__device__ __forceinline__ void dequant_tile(const uint8_t *base, int64_t rb, int64_t j0,
                                             int64_t c1, int D, float *dst, int pitch)
{
    constexpr int E = block_elems(TYPE), BB = block_bytes(TYPE);
    const int D4 = D / 4;
    for (int g = threadIdx.x; g < GEN_TILE * D4; g += GEN_THREADS) {
        const int jj = g / D4, i = (g - jj * D4) * 4;
        float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (j0 + jj < c1) {
            const uint8_t *blk = base + (j0 + jj) * rb + (i / E) * BB;
            const int ii = i % E;  // the 4 elements share a block (E is a multiple of 4)
            const float d = block_d(blk), m = block_m<TYPE>(blk);
            v.x = d * (float)block_int<TYPE>(blk, ii) + m;
            v.y = d * (float)block_int<TYPE>(blk, ii + 1) + m;
            v.z = d * (float)block_int<TYPE>(blk, ii + 2) + m;
            v.w = d * (float)block_int<TYPE>(blk, ii + 3) + m;
        }
        *reinterpret_cast<float4 *>(dst + jj * pitch + i) = v;
    }
}

__device__ __forceinline__ void dequant_tile_any(int type, const uint8_t *base, int64_t rb,
                                                 int64_t j0, int64_t c1, int D, float *dst,
                                                 int pitch)
{
    if (type == KVQ_TYPE_Q8_0)
        dequant_tile<KVQ_TYPE_Q8_0>(base, rb, j0, c1, D, dst, pitch);
    else if (type == KVQ_TYPE_Q4_0)
        dequant_tile<KVQ_TYPE_Q4_0>(base, rb, j0, c1, D, dst, pitch);
    else
        dequant_tile<KVQ_TYPE_OSCAR2>(base, rb, j0, c1, D, dst, pitch);
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void fma4(float4 &acc, float a, const float4 &b)
{
    acc.x = fmaf(a, b.x, acc.x);
    acc.y = fmaf(a, b.y, acc.y);
    acc.z = fmaf(a, b.z, acc.z);
    acc.w = fmaf(a, b.w, acc.w);
}

__global__ void __launch_bounds__(GEN_THREADS) decode_simple_kernel(const DecodeArgs a)
{
    extern __shared__ __align__(16) float sm[];
    const int G = a.n_q_heads / a.n_kv_heads;
    const int R = G * a.T;  // <= GEN_ROWS (validated)
    const int D = a.head_dim, D4 = D / 4, KP = D + 4;
    float *q_s = sm;                      // [R][D]
    float *kt = q_s + R * D;              // [GEN_TILE][KP]
    float *vt = kt + GEN_TILE * KP;       // [GEN_TILE][D]
    float *p_s = vt + GEN_TILE * D;       // [R][GEN_TILE]
    float *al_s = p_s + R * GEN_TILE;     // [GEN_ROWS]
    float *m_s = al_s + GEN_ROWS;         // [GEN_ROWS]
    float *l_s = m_s + GEN_ROWS;          // [GEN_ROWS]

    const int c = blockIdx.x, h = blockIdx.y, layer = blockIdx.z;
    const int n_chunks = (int)((a.n_kv + a.chunk - 1) / a.chunk);
    const int64_t c0 = (int64_t)c * a.chunk;
    const int64_t c1 = c0 + a.chunk < a.n_kv ? c0 + a.chunk : a.n_kv;
    const int64_t krow = row_bytes(a.k_type, D), vrow = row_bytes(a.v_type, D);
    const uint8_t *kb = a.layers.k[layer] + (int64_t)h * a.layers.cap[layer] * krow;
    const uint8_t *vb = a.layers.v[layer] + (int64_t)h * a.layers.cap[layer] * vrow;

    for (int p = threadIdx.x; p < R * D; p += GEN_THREADS) {
        const int r = p / D, i = p - r * D;
        const int t = r / G, g = r - t * G;
        q_s[p] = __half2float(a.q[(((int64_t)layer * a.T + t) * a.n_q_heads + h * G + g) * D + i]);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // steps 1-2: rows warp + 8 k of this warp; m and l are the same in every lane
    float m_r[4], l_r[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        m_r[k] = -INFINITY;
        l_r[k] = 0.0f;
    }
    // step 3: row slot `slot`, head dims 4 i4 .. 4 i4 + 3
    const int NS = GEN_THREADS / D4;
    const int slot = threadIdx.x / D4, i4 = threadIdx.x - slot * D4;
    const bool pv = slot < NS;
    float4 o[GEN_ITEMS];
#pragma unroll
    for (int it = 0; it < GEN_ITEMS; ++it)
        o[it] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);

    for (int64_t j0 = c0; j0 < c1; j0 += GEN_TILE) {
        __syncthreads();  // q_s written; the previous tile's P V is done with kt, vt, p_s
        dequant_tile_any(a.k_type, kb, krow, j0, c1, D, kt, KP);
        dequant_tile_any(a.v_type, vb, vrow, j0, c1, D, vt, D);
        __syncthreads();
        // ---- 1. scores of key j0 + lane for the warp's rows
        float s[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        {
            const float4 *kr = reinterpret_cast<const float4 *>(kt + lane * KP);
            const float4 *qr = reinterpret_cast<const float4 *>(q_s);
            for (int x = 0; x < D4; ++x) {
                const float4 k4 = kr[x];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int r = warp + 8 * k;
                    if (r >= R)
                        break;  // uniform across the warp
                    const float4 q4 = qr[r * D4 + x];
                    s[k] = fmaf(q4.x, k4.x, s[k]);
                    s[k] = fmaf(q4.y, k4.y, s[k]);
                    s[k] = fmaf(q4.z, k4.z, s[k]);
                    s[k] = fmaf(q4.w, k4.w, s[k]);
                }
            }
        }
        // ---- 2. online softmax of each row over the tile
        const int64_t j = j0 + lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int r = warp + 8 * k;
            if (r >= R)
                break;
            const int t = r / G;
            const float sc = (j < c1 && j <= a.vis_last + t) ? a.scale * s[k] : -INFINITY;
            const float m_new = fmaxf(m_r[k], warp_max(sc));
            float alpha = 1.0f, pw = 0.0f;
            if (m_new != -INFINITY) {
                alpha = (m_r[k] == -INFINITY) ? 0.0f : expf(m_r[k] - m_new);
                pw = (sc == -INFINITY) ? 0.0f : expf(sc - m_new);
            }
            l_r[k] = l_r[k] * alpha + warp_sum(pw);
            m_r[k] = m_new;
            p_s[r * GEN_TILE + lane] = pw;
            if (lane == 0)
                al_s[r] = alpha;
        }
        __syncthreads();
        // ---- 3. rescale, then O += P V over the tile
        if (pv) {
#pragma unroll
            for (int it = 0; it < GEN_ITEMS; ++it) {
                const int r = slot + NS * it;
                if (r >= R)
                    break;
                const float al = al_s[r];
                o[it].x *= al;
                o[it].y *= al;
                o[it].z *= al;
                o[it].w *= al;
            }
            const float4 *vr = reinterpret_cast<const float4 *>(vt) + i4;
            for (int jj = 0; jj < GEN_TILE; ++jj) {
                const float4 v4 = vr[jj * D4];
#pragma unroll
                for (int it = 0; it < GEN_ITEMS; ++it) {
                    const int r = slot + NS * it;
                    if (r >= R)
                        break;
                    fma4(o[it], p_s[r * GEN_TILE + jj], v4);
                }
            }
        }
    }
    // ---- the chunk partial of every row
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int r = warp + 8 * k;
        if (r < R && lane == 0) {
            m_s[r] = m_r[k];
            l_s[r] = l_r[k];
        }
    }
    __syncthreads();
    if (!pv)
        return;
#pragma unroll
    for (int it = 0; it < GEN_ITEMS; ++it) {
        const int r = slot + NS * it;
        if (r >= R)
            break;
        const int t = r / G, g = r - t * G;
        const int64_t row = ((int64_t)layer * a.T + t) * a.n_q_heads + h * G + g;
        const float l = l_s[r];
        float4 res = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (l > 0.0f)
            res = make_float4(o[it].x / l, o[it].y / l, o[it].z / l, o[it].w / l);
        *reinterpret_cast<float4 *>(a.out_part + (row * n_chunks + c) * D + 4 * i4) = res;
        if (i4 == 0)
            a.lse_part[row * n_chunks + c] = (l > 0.0f) ? m_s[r] + logf(l) : -INFINITY;
    }
}

size_t decode_simple_smem(int R, int D)
{
    return sizeof(float) * ((size_t)R * D + (size_t)GEN_TILE * (D + 4) + (size_t)GEN_TILE * D +
                            (size_t)R * GEN_TILE + 3 * (size_t)GEN_ROWS);
}

bool launch_decode_simple(const DecodeArgs &a, cudaStream_t s)
{
    const int G = a.n_q_heads / a.n_kv_heads;
    const int R = G * a.T;
    if (R > GEN_ROWS || a.head_dim % 32 != 0 || a.head_dim > 512 ||
        a.head_dim % block_elems(a.k_type) != 0 || a.head_dim % block_elems(a.v_type) != 0)
        return false;
    if (!known_type(a.k_type) || !known_type(a.v_type) || a.k_type == KVQ_TYPE_DEFAULT ||
        a.v_type == KVQ_TYPE_DEFAULT)
        return false;
    const size_t smem = decode_simple_smem(R, a.head_dim);
    static std::atomic<int> smem_set[MAX_DEVICES];
    if (!ensure_smem(reinterpret_cast<const void *>(decode_simple_kernel), smem_set, (int)smem))
        return false;
    const int n_chunks = (int)((a.n_kv + a.chunk - 1) / a.chunk);
    dim3 grid(n_chunks, a.n_kv_heads, a.n_layers);
    decode_simple_kernel<<<grid, GEN_THREADS, smem, s>>>(a);
    return true;
}

}  // namespace kvq
