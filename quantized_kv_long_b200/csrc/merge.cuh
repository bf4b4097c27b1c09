// merge.cuh -- LSE merge of one row's chunk partials by a group of 64 threads.
//
// For one row with partials (o_c, lse_c), c < C:
//   M = max_c lse_c;  lse = M + ln sum_c exp(lse_c - M);  o = sum_c exp(lse_c - lse) o_c
// Partials with lse_c = -inf (fully masked chunks) carry weight 0; a row whose
// partials are all -inf gets o = 0, lse = -inf.  This is the log-sum-exp
// combination that the "Online Log-Sum-Exp prefill" item of the RX 9070 XT
// KV-streaming page accumulates across pages.
//
// The order of every floating-point operation is fixed by the 64-thread group
// (strided partial sums, a warp shuffle tree, then the two warp results added
// in order) and by explicit fused multiply-adds, so a row's result does not
// depend on the launch shape or on where its partials are stored.
#pragma once

#include "common.cuh"

namespace kvq {

constexpr int MERGE_GROUP = 64;

template <class Sync>
__device__ __forceinline__ float group_max(float v, float *red, int t, Sync sync)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    sync();
    if ((t & 31) == 0)
        red[t >> 5] = v;
    sync();
    return fmaxf(red[0], red[1]);
}

template <class Sync>
__device__ __forceinline__ float group_sum(float v, float *red, int t, Sync sync)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    sync();
    if ((t & 31) == 0)
        red[t >> 5] = v;
    sync();
    return red[0] + red[1];
}

// Merge row partials op[c * op_stride + 0..head_dim) and lp[c * lp_stride]
// (c < n_chunks) into o[0..head_dim) and *lse_out.  t = thread index in the group (0..63);
// red = 2 floats of shared memory private to the group; w_s = n_chunks floats
// of shared memory private to the group, or nullptr (the weights are then
// recomputed per element, with the same arithmetic).
// head_dim % 4 == 0; op, op_stride * 4 bytes and o 16-byte aligned.
template <class Sync>
__device__ __forceinline__ void merge_row(const float *op, int64_t op_stride, const float *lp,
                                          int64_t lp_stride, int n_chunks, int head_dim, float *o,
                                          float *lse_out, float *w_s, float *red, int t, Sync sync)
{
    auto ld = [](const float *p) -> float { return *p; };
    float m = -INFINITY;
    for (int c = t; c < n_chunks; c += MERGE_GROUP)
        m = fmaxf(m, ld(lp + c * lp_stride));
    m = group_max(m, red, t, sync);
    if (m == -INFINITY) {
        for (int i = t; i < head_dim; i += MERGE_GROUP)
            o[i] = 0.0f;
        if (t == 0)
            *lse_out = -INFINITY;
        sync();  // red is reused by the group's next row
        return;
    }
    float s = 0.0f;
    for (int c = t; c < n_chunks; c += MERGE_GROUP) {
        const float l = ld(lp + c * lp_stride);
        if (l != -INFINITY)
            s += expf(l - m);
    }
    s = group_sum(s, red, t, sync);
    const float L = m + logf(s);
    if (w_s) {
        for (int c = t; c < n_chunks; c += MERGE_GROUP) {
            const float l = ld(lp + c * lp_stride);
            w_s[c] = (l == -INFINITY) ? 0.0f : expf(l - L);
        }
        sync();
    }
    // acc = sum over c in increasing order of w_c * o_c (chunks of weight 0 skipped); the
    // loads of MERGE_BATCH chunks are issued before their multiply-adds, which keep the order
    constexpr int MERGE_BATCH = 16;
    for (int i = t * 4; i < head_dim; i += MERGE_GROUP * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c0 = 0; c0 < n_chunks; c0 += MERGE_BATCH) {
            float w[MERGE_BATCH];
            float4 v[MERGE_BATCH];
#pragma unroll
            for (int k = 0; k < MERGE_BATCH; ++k) {
                const int c = c0 + k;
                w[k] = 0.0f;
                if (c < n_chunks) {
                    if (w_s) {
                        w[k] = w_s[c];
                    } else {
                        const float l = ld(lp + c * lp_stride);
                        w[k] = (l == -INFINITY) ? 0.0f : expf(l - L);
                    }
                }
                if (w[k] != 0.0f) {
                    const float4 *src =
                        reinterpret_cast<const float4 *>(op + (int64_t)c * op_stride + i);
                    v[k] = *src;
                }
            }
#pragma unroll
            for (int k = 0; k < MERGE_BATCH; ++k) {
                if (w[k] == 0.0f)
                    continue;
                acc.x = __fmaf_rn(w[k], v[k].x, acc.x);
                acc.y = __fmaf_rn(w[k], v[k].y, acc.y);
                acc.z = __fmaf_rn(w[k], v[k].z, acc.z);
                acc.w = __fmaf_rn(w[k], v[k].w, acc.w);
            }
        }
        *reinterpret_cast<float4 *>(o + i) = acc;
    }
    if (t == 0)
        *lse_out = L;
    sync();  // w_s and red are reused by the group's next row
}

}  // namespace kvq
