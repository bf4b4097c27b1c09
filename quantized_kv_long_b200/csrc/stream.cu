// stream.cu -- layer-pipelined host streaming of the KV cache.
//
// The whole cache stays in pinned host memory; two device slots (each one
// layer's worth of K and V) form a double-buffered working set that is reused
// across layers.  Layer L's rows are copied into slot L % 2 on the copy stream
// while the compute stream runs decode attention + LSE merge of layer L-1 on
// the other slot.  This is the prefetch scheme of the "Online Log-Sum-Exp
// prefill & pipelined prefetch" item on the RX 9070 XT KV-streaming page
// (layer L+1's transfer overlaps layer L's compute) with the bounded,
// reused working set of "What shipped" on the ROCm KV-streaming page.
//
// Ordering, per layer L with slot s = L % 2:
//   copy:    wait freed[s] (compute of layer L-2 is done with slot s)
//            memcpy2D K rows [0, n_kv) of every head, then V rows
//            record ready[s]
//   compute: wait ready[s]; decode; merge into out[L]; record freed[s]
// Before the first copy the copy stream also waits for all work already
// enqueued on the compute stream, so a previous call's reads of the slots
// finish before they are overwritten.
//
// Test hook (host side, no device fault): if the environment variable
// KVQ_TEST_FAIL_COPY_LAYER is set to L, enqueueing layer L's copy is treated
// as failed: the call returns KVQ_ERR_COPY with nothing further enqueued.
#include <stdlib.h>

#include "common.cuh"

namespace kvq {
kvq_status validate_decode(const kvq_layer *layers, int n_layers, const uint16_t *q,
                           int n_q_heads, int T, int64_t n_kv, int chunk, float scale,
                           const float *out_part, const float *lse_part, const char *fn);
kvq_status enqueue_decode(const kvq_layer *layers, int n_layers, const uint16_t *q,
                          int n_q_heads, int T, int64_t n_kv, int chunk, float scale,
                          float *out_part, float *lse_part, cudaStream_t s);
kvq_status validate_merge(const float *out_part, const float *lse_part, int64_t rows,
                          int n_chunks, int head_dim, const float *out, const float *lse,
                          const char *fn);

namespace {

struct Events {
    cudaEvent_t ev[5] = {};
    int made = 0;
    ~Events()
    {
        for (int i = 0; i < made; ++i)
            cudaEventDestroy(ev[i]);  // released once the device passes them
    }
    bool make()
    {
        for (; made < 5; ++made)
            if (cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming) != cudaSuccess)
                return false;
        return true;
    }
};

bool is_pinned_host(const void *p)
{
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeHost;
}

int fail_copy_layer()
{
    const char *e = getenv("KVQ_TEST_FAIL_COPY_LAYER");
    return e ? atoi(e) : -1;
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" kvq_status kvq_stream_decode(const kvq_layer *host_layers, int n_layers,
                                        const kvq_layer *dev_slots, const uint16_t *q,
                                        int n_q_heads, int T, int64_t n_kv, int chunk,
                                        float scale, float *out_part, float *lse_part,
                                        float *out, float *lse, kvq_stream compute,
                                        kvq_stream copy)
{
    const char *fn = "kvq_stream_decode";
    kvq_status st = validate_decode(host_layers, n_layers, q, n_q_heads, T, n_kv, chunk, scale,
                                    out_part, lse_part, fn);
    if (st != KVQ_OK)
        return st;
    if (!dev_slots)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: dev_slots is NULL", fn);
    st = validate_decode(dev_slots, 2, q, n_q_heads, T, n_kv, chunk, scale, out_part, lse_part,
                         fn);
    if (st != KVQ_OK)
        return st;
    const int H = host_layers[0].n_kv_heads, D = host_layers[0].head_dim;
    if (dev_slots[0].n_kv_heads != H || dev_slots[0].head_dim != D)
        return set_error(KVQ_ERR_INVALID_ARG, "%s: slots and host layers differ in shape", fn);
    const int G = n_q_heads / H;
    const int64_t rows = (int64_t)T * n_q_heads;
    const int n_chunks = (int)((n_kv + chunk - 1) / chunk);
    st = validate_merge(out_part, lse_part, rows, n_chunks, D, out, lse, fn);
    if (st != KVQ_OK)
        return st;
    for (int l = 0; l < n_layers; ++l)
        if (!is_pinned_host(host_layers[l].k) || !is_pinned_host(host_layers[l].v))
            return set_error(KVQ_ERR_INVALID_ARG, "%s: host layer %d is not pinned host memory",
                             fn, l);
    (void)G;

    cudaStream_t cs = as_stream(compute), ps = as_stream(copy);
    Events E;
    if (!E.make())
        return set_error(KVQ_ERR_CUDA, "%s: cudaEventCreate failed", fn);
    cudaEvent_t start = E.ev[0], *ready = &E.ev[1], *freed = &E.ev[3];
    if (cudaEventRecord(start, cs) != cudaSuccess || cudaStreamWaitEvent(ps, start, 0) != cudaSuccess)
        return set_error(KVQ_ERR_CUDA, "%s: event ordering failed", fn);

    const int64_t kr = k_row_bytes(D), vr = v_row_bytes(D);
    const int fail_at = fail_copy_layer();
    for (int L = 0; L < n_layers; ++L) {
        const int s = L & 1;
        const kvq_layer &hl = host_layers[L];
        const kvq_layer &sl = dev_slots[s];
        if (L >= 2 && cudaStreamWaitEvent(ps, freed[s], 0) != cudaSuccess)
            return set_error(KVQ_ERR_CUDA, "%s: event wait failed", fn);
        if (L == fail_at)
            return set_error(KVQ_ERR_COPY, "%s: copy of layer %d failed (test hook)", fn, L);
        cudaError_t e = cudaMemcpy2DAsync(sl.k, (size_t)(sl.capacity * kr), hl.k,
                                          (size_t)(hl.capacity * kr), (size_t)(n_kv * kr), H,
                                          cudaMemcpyHostToDevice, ps);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(sl.v, (size_t)(sl.capacity * vr), hl.v,
                                  (size_t)(hl.capacity * vr), (size_t)(n_kv * vr), H,
                                  cudaMemcpyHostToDevice, ps);
        if (e != cudaSuccess)
            return set_error(KVQ_ERR_COPY, "%s: copy of layer %d: %s", fn, L,
                             cudaGetErrorString(e));
        if (cudaEventRecord(ready[s], ps) != cudaSuccess ||
            cudaStreamWaitEvent(cs, ready[s], 0) != cudaSuccess)
            return set_error(KVQ_ERR_CUDA, "%s: event ordering failed", fn);
        const uint16_t *ql = q + (size_t)L * rows * D;
        st = enqueue_decode(&sl, 1, ql, n_q_heads, T, n_kv, chunk, scale, out_part, lse_part, cs);
        if (st != KVQ_OK)
            return st;
        launch_merge_lse(out_part, lse_part, rows, n_chunks, D, out + (size_t)L * rows * D,
                         lse + (size_t)L * rows, cs);
        st = check_launch(fn);
        if (st != KVQ_OK)
            return st;
        if (cudaEventRecord(freed[s], cs) != cudaSuccess)
            return set_error(KVQ_ERR_CUDA, "%s: event record failed", fn);
    }
    return KVQ_OK;
}
