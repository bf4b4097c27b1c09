// merge.cu -- LSE merge of per-chunk attention partials.
//
// For one row with partials (o_c, lse_c), c < C:
//   M = max_c lse_c;  lse = M + ln sum_c exp(lse_c - M);  o = sum_c exp(lse_c - lse) o_c
// Partials with lse_c = -inf (fully masked chunks) carry weight 0; a row whose
// partials are all -inf gets o = 0, lse = -inf.  This is the log-sum-exp
// combination that the "Online Log-Sum-Exp prefill" item of the RX 9070 XT
// KV-streaming page accumulates across pages.
//
// One CTA per row.  The weights exp(lse_c - lse) are computed once into
// shared memory; then each thread owns 4 consecutive output elements and
// streams the C partial rows with 16-byte loads (coalesced across the CTA).
// The kernel is HBM-bound: it reads C * head_dim * 4 + C * 4 bytes per row
// and writes head_dim * 4 + 4.
#include "common.cuh"

namespace kvq {

constexpr int MERGE_THREADS = 64;
constexpr int MERGE_MAX_SMEM_CHUNKS = 8192;

__device__ __forceinline__ float block_max(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0)
        red[w] = v;
    __syncthreads();
    v = red[0];
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i)
        v = fmaxf(v, red[i]);
    return v;
}

__device__ __forceinline__ float block_sum(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0)
        red[w] = v;
    __syncthreads();
    v = red[0];
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i)
        v += red[i];
    return v;
}

__global__ void __launch_bounds__(MERGE_THREADS)
merge_lse_kernel(const float *__restrict__ out_part, const float *__restrict__ lse_part,
                 int n_chunks, int head_dim, float *__restrict__ out, float *__restrict__ lse)
{
    extern __shared__ float w_s[];  // [min(n_chunks, MERGE_MAX_SMEM_CHUNKS)]
    __shared__ float red[MERGE_THREADS / 32];
    const int64_t row = blockIdx.x;
    const float *lp = lse_part + row * n_chunks;

    float m = -INFINITY;
    for (int c = threadIdx.x; c < n_chunks; c += blockDim.x)
        m = fmaxf(m, lp[c]);
    m = block_max(m, red);

    float *o = out + row * head_dim;
    if (m == -INFINITY) {
        for (int i = threadIdx.x; i < head_dim; i += blockDim.x)
            o[i] = 0.0f;
        if (threadIdx.x == 0)
            lse[row] = -INFINITY;
        return;
    }
    float s = 0.0f;
    for (int c = threadIdx.x; c < n_chunks; c += blockDim.x) {
        const float l = lp[c];
        if (l != -INFINITY)
            s += expf(l - m);
    }
    s = block_sum(s, red);
    const float L = m + logf(s);
    const bool in_smem = n_chunks <= MERGE_MAX_SMEM_CHUNKS;
    if (in_smem) {
        for (int c = threadIdx.x; c < n_chunks; c += blockDim.x) {
            const float l = lp[c];
            w_s[c] = (l == -INFINITY) ? 0.0f : expf(l - L);
        }
        __syncthreads();
    }
    const float *op = out_part + row * (int64_t)n_chunks * head_dim;
    for (int i = threadIdx.x * 4; i < head_dim; i += blockDim.x * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c = 0; c < n_chunks; ++c) {
            float w;
            if (in_smem) {
                w = w_s[c];
            } else {
                const float l = lp[c];
                w = (l == -INFINITY) ? 0.0f : expf(l - L);
            }
            if (w == 0.0f)
                continue;
            const float4 v = *reinterpret_cast<const float4 *>(op + (int64_t)c * head_dim + i);
            acc.x += w * v.x;
            acc.y += w * v.y;
            acc.z += w * v.z;
            acc.w += w * v.w;
        }
        *reinterpret_cast<float4 *>(o + i) = acc;
    }
    if (threadIdx.x == 0)
        lse[row] = L;
}

void launch_merge_lse(const float *out_part, const float *lse_part, int64_t rows, int n_chunks,
                      int head_dim, float *out, float *lse, cudaStream_t s)
{
    if (rows == 0)
        return;
    const int smem_chunks = n_chunks <= MERGE_MAX_SMEM_CHUNKS ? n_chunks : 0;
    merge_lse_kernel<<<(unsigned)rows, MERGE_THREADS, smem_chunks * sizeof(float), s>>>(
        out_part, lse_part, n_chunks, head_dim, out, lse);
}

}  // namespace kvq
