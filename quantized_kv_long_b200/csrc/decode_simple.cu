// decode_simple.cu -- straightforward split-KV decode attention, any shape.
//
// The general path of kvq_decode_attn: one CTA per (chunk, kv head, layer),
// every row of the GQA group (G query heads x T tokens) handled together,
// keys processed in tiles of 64 with an online softmax.  K and V are read
// from global memory and dequantized in registers; the per-block K scale is
// applied to each block's fp32 partial dot product, so only fp32 rounding
// separates it from the exact result.  It serves the shapes and formats the
// persistent tensor-core kernel (decode_tmem.cu) does not cover.
//
// Semantics (speculative-decoding paragraph of the RX 9070 XT KV-streaming
// page: paged decode attention over the verify batch; "Known Issues Fixed" of
// the OSCAR2 page: the max covers complete scores; GQA section of the KV-cache
// guide): row r = t*G + g is query head h*G + g of token t and sees keys
// j <= vis_last + t (n_kv - T + t for a whole context) of chunk c = keys
// [c*chunk, (c+1)*chunk).
//
// K and V may each be in any block format (template parameters KT, VT:
// KVQ_TYPE_Q8_0, KVQ_TYPE_Q4_0 or KVQ_TYPE_OSCAR2, whose zero-point m enters
// the score as m * sum(q) per block); the pages' configuration is Q8_0 K / Q4_0 V.
#include "common.cuh"

namespace kvq {

constexpr int SIMPLE_THREADS = 256;
constexpr int SIMPLE_TILE = 64;

template <int KT, int VT>
__global__ void __launch_bounds__(SIMPLE_THREADS)
decode_simple_kernel(DecodeArgs a)
{
    extern __shared__ float sm[];
    const int G = a.n_q_heads / a.n_kv_heads;
    const int R = G * a.T;
    const int D = a.head_dim;
    constexpr int KE = block_elems(KT), VE = block_elems(VT);  // elements per block
    const int nb = D / KE;
    float *q_s = sm;                       // [R][D]
    float *acc = q_s + R * D;              // [R][D]
    float *p_s = acc + R * D;              // [R][TILE]
    float *m_s = p_s + R * SIMPLE_TILE;    // [R]
    float *l_s = m_s + R;                  // [R]
    float *al_s = l_s + R;                 // [R]

    const int c = blockIdx.x, h = blockIdx.y, layer = blockIdx.z;
    const int n_chunks = (int)((a.n_kv + a.chunk - 1) / a.chunk);
    const int64_t c0 = (int64_t)c * a.chunk;
    const int64_t c1 = c0 + a.chunk < a.n_kv ? c0 + a.chunk : a.n_kv;
    const int64_t krow = row_bytes(KT, D), vrow = row_bytes(VT, D);
    const uint8_t *kb = a.layers.k[layer] + (int64_t)h * a.layers.cap[layer] * krow;
    const uint8_t *vb = a.layers.v[layer] + (int64_t)h * a.layers.cap[layer] * vrow;

    for (int p = threadIdx.x; p < R * D; p += blockDim.x) {
        const int r = p / D, i = p % D;
        const int t = r / G, g = r % G;
        q_s[p] = __half2float(a.q[(((int64_t)layer * a.T + t) * a.n_q_heads + h * G + g) * D + i]);
        acc[p] = 0.0f;
    }
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
        m_s[r] = -INFINITY;
        l_s[r] = 0.0f;
    }
    __syncthreads();

    for (int64_t j0 = c0; j0 < c1; j0 += SIMPLE_TILE) {
        // 1. complete scores of the tile
        for (int p = threadIdx.x; p < R * SIMPLE_TILE; p += blockDim.x) {
            const int r = p / SIMPLE_TILE, jj = p % SIMPLE_TILE;
            const int64_t j = j0 + jj;
            const int t = r / G;
            float s = -INFINITY;
            if (j < c1 && j <= a.vis_last + t) {
                const uint8_t *kr = kb + j * krow;
                const float *qr = q_s + r * D;
                float tot = 0.0f;
                for (int b = 0; b < nb; ++b) {
                    const uint8_t *blk = kr + b * block_bytes(KT);
                    float part = 0.0f, qsum = 0.0f;
                    for (int i = 0; i < KE; ++i) {
                        part += qr[b * KE + i] * (float)block_int<KT>(blk, i);
                        if (KT == KVQ_TYPE_OSCAR2)
                            qsum += qr[b * KE + i];
                    }
                    tot += block_d(blk) * part;
                    if (KT == KVQ_TYPE_OSCAR2)  // q . (d u + m) = d (q . u) + m sum(q)
                        tot += block_m<KT>(blk) * qsum;
                }
                s = a.scale * tot;
            }
            p_s[p] = s;
        }
        __syncthreads();
        // 2. online softmax update per row
        for (int r = threadIdx.x; r < R; r += blockDim.x) {
            float mt = -INFINITY;
            for (int jj = 0; jj < SIMPLE_TILE; ++jj)
                mt = fmaxf(mt, p_s[r * SIMPLE_TILE + jj]);
            const float m_old = m_s[r];
            const float m_new = fmaxf(m_old, mt);
            float alpha = 1.0f, sum = 0.0f;
            if (m_new != -INFINITY) {
                alpha = (m_old == -INFINITY) ? 0.0f : expf(m_old - m_new);
                for (int jj = 0; jj < SIMPLE_TILE; ++jj) {
                    const float s = p_s[r * SIMPLE_TILE + jj];
                    const float pw = (s == -INFINITY) ? 0.0f : expf(s - m_new);
                    p_s[r * SIMPLE_TILE + jj] = pw;
                    sum += pw;
                }
            } else {
                for (int jj = 0; jj < SIMPLE_TILE; ++jj)
                    p_s[r * SIMPLE_TILE + jj] = 0.0f;
            }
            l_s[r] = l_s[r] * alpha + sum;
            m_s[r] = m_new;
            al_s[r] = alpha;
        }
        __syncthreads();
        // 3. rescale and accumulate the weighted V rows
        for (int p = threadIdx.x; p < R * D; p += blockDim.x) {
            const int r = p / D, i = p % D;
            const int b = i / VE, ii = i % VE;
            float o = acc[p] * al_s[r];
            for (int jj = 0; jj < SIMPLE_TILE; ++jj) {
                const float pw = p_s[r * SIMPLE_TILE + jj];
                if (pw == 0.0f)
                    continue;
                const uint8_t *blk = vb + (j0 + jj) * vrow + b * block_bytes(VT);
                o += pw * (block_d(blk) * (float)block_int<VT>(blk, ii) + block_m<VT>(blk));
            }
            acc[p] = o;
        }
        __syncthreads();
    }
    // 4. normalise and write the chunk partial
    for (int p = threadIdx.x; p < R * D; p += blockDim.x) {
        const int r = p / D, i = p % D;
        const int t = r / G, g = r % G;
        const int64_t row = ((int64_t)layer * a.T + t) * a.n_q_heads + h * G + g;
        const float l = l_s[r];
        a.out_part[(row * n_chunks + c) * D + i] = (l > 0.0f) ? acc[p] / l : 0.0f;
        if (i == 0)
            a.lse_part[row * n_chunks + c] = (l > 0.0f) ? m_s[r] + logf(l) : -INFINITY;
    }
}

size_t decode_simple_smem(int R, int D)
{
    return sizeof(float) * ((size_t)2 * R * D + (size_t)R * SIMPLE_TILE + 3 * (size_t)R);
}

template <int KT, int VT>
static bool launch_simple_typed(const DecodeArgs &a, size_t smem, cudaStream_t s)
{
    static std::atomic<int> smem_set[MAX_DEVICES];
    if (!ensure_smem(reinterpret_cast<const void *>(decode_simple_kernel<KT, VT>), smem_set,
                     (int)smem))
        return false;
    const int n_chunks = (int)((a.n_kv + a.chunk - 1) / a.chunk);
    dim3 grid(n_chunks, a.n_kv_heads, a.n_layers);
    decode_simple_kernel<KT, VT><<<grid, SIMPLE_THREADS, smem, s>>>(a);
    return true;
}

bool launch_decode_simple(const DecodeArgs &a, cudaStream_t s)
{
    const int G = a.n_q_heads / a.n_kv_heads;
    const int R = G * a.T;
    const size_t smem = decode_simple_smem(R, a.head_dim);
    if (smem > 227 * 1024)
        return false;
    return launch_for_types(a.k_type, a.v_type, [&](auto kt, auto vt) {
        return launch_simple_typed<decltype(kt)::value, decltype(vt)::value>(a, smem, s);
    });
}

}  // namespace kvq
