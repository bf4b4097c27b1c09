// merge.cu -- LSE merge of per-chunk attention partials (the definition and
// the fixed order of operations are in merge.cuh).
//
// One 64-thread CTA per row.  The weights exp(lse_c - lse) are computed once
// into shared memory (up to MERGE_MAX_SMEM_CHUNKS chunks; beyond that they are
// recomputed per element); each thread owns 4 consecutive output elements and
// streams the C partial rows with 16-byte loads (coalesced across the CTA).
// The kernel is HBM-bound: it reads C * head_dim * 4 + C * 4 bytes per row
// and writes head_dim * 4 + 4.
#include "common.cuh"
#include "merge.cuh"

namespace kvq {

constexpr int MERGE_MAX_SMEM_CHUNKS = 8192;

__global__ void __launch_bounds__(MERGE_GROUP)
merge_lse_kernel(const float *__restrict__ out_part, const float *__restrict__ lse_part,
                 int n_chunks, int head_dim, float *__restrict__ out, float *__restrict__ lse)
{
    extern __shared__ float w_s[];  // [n_chunks] when n_chunks <= MERGE_MAX_SMEM_CHUNKS
    __shared__ float red[MERGE_GROUP / 32];
    const int64_t row = blockIdx.x;
    merge_row<false>(out_part + row * (int64_t)n_chunks * head_dim, lse_part + row * n_chunks,
                     n_chunks, head_dim, out + row * head_dim, lse + row,
                     n_chunks <= MERGE_MAX_SMEM_CHUNKS ? w_s : nullptr, red, (int)threadIdx.x,
                     [] { __syncthreads(); });
}

void launch_merge_lse(const float *out_part, const float *lse_part, int64_t rows, int n_chunks,
                      int head_dim, float *out, float *lse, cudaStream_t s)
{
    if (rows == 0)
        return;
    const int smem_chunks = n_chunks <= MERGE_MAX_SMEM_CHUNKS ? n_chunks : 0;
    merge_lse_kernel<<<(unsigned)rows, MERGE_GROUP, smem_chunks * sizeof(float), s>>>(
        out_part, lse_part, n_chunks, head_dim, out, lse);
}

}  // namespace kvq
