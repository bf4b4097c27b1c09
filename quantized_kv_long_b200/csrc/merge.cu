// merge.cu -- LSE merge of attention partials (the definition and the fixed
// order of operations are in merge.cuh): per-chunk partials of one call
// ([rows][n_chunks][head_dim]) or per-part results gathered from several
// calls, e.g. the ranks of a context-parallel split ([n_parts][rows][head_dim]).
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

// Row r's partial c: out_part[r * row_stride + c * part_stride + 0..head_dim) and
// lse_part[r * lrow_stride + c * lpart_stride].
__global__ void __launch_bounds__(MERGE_GROUP)
merge_lse_kernel(const float *__restrict__ out_part, const float *__restrict__ lse_part,
                 int64_t row_stride, int64_t part_stride, int64_t lrow_stride,
                 int64_t lpart_stride, int n_chunks, int head_dim, float *__restrict__ out,
                 float *__restrict__ lse)
{
    extern __shared__ float w_s[];  // [n_chunks] when n_chunks <= MERGE_MAX_SMEM_CHUNKS
    __shared__ float red[MERGE_GROUP / 32];
    const int64_t row = blockIdx.x;
    merge_row(out_part + row * row_stride, part_stride, lse_part + row * lrow_stride,
                     lpart_stride, n_chunks, head_dim, out + row * head_dim, lse + row,
                     n_chunks <= MERGE_MAX_SMEM_CHUNKS ? w_s : nullptr, red, (int)threadIdx.x,
                     [] { __syncthreads(); });
}

namespace {

void launch_strided(const float *out_part, const float *lse_part, int64_t rows, int n_chunks,
                    int head_dim, int64_t row_stride, int64_t part_stride, int64_t lrow_stride,
                    int64_t lpart_stride, float *out, float *lse, cudaStream_t s)
{
    if (rows == 0)
        return;
    const int smem_chunks = n_chunks <= MERGE_MAX_SMEM_CHUNKS ? n_chunks : 0;
    merge_lse_kernel<<<(unsigned)rows, MERGE_GROUP, smem_chunks * sizeof(float), s>>>(
        out_part, lse_part, row_stride, part_stride, lrow_stride, lpart_stride, n_chunks,
        head_dim, out, lse);
}

}  // namespace

void launch_merge_lse(const float *out_part, const float *lse_part, int64_t rows, int n_chunks,
                      int head_dim, float *out, float *lse, cudaStream_t s)
{
    // [rows][n_chunks][head_dim] and [rows][n_chunks]
    launch_strided(out_part, lse_part, rows, n_chunks, head_dim, (int64_t)n_chunks * head_dim,
                   head_dim, n_chunks, 1, out, lse, s);
}

void launch_merge_lse_parts(const float *out_parts, const float *lse_parts, int n_parts,
                            int64_t rows, int head_dim, float *out, float *lse, cudaStream_t s)
{
    // [n_parts][rows][head_dim] and [n_parts][rows]
    launch_strided(out_parts, lse_parts, rows, n_parts, head_dim, head_dim,
                   rows * (int64_t)head_dim, 1, rows, out, lse, s);
}

}  // namespace kvq
