// stream.cu -- layer-pipelined host streaming of the KV cache, with a
// resident set of layers.
//
// Each layer's cache is either resident (device memory: computed in place)
// or streamed (pinned host memory).  Two device slots (each one layer's worth
// of K and V) form a double-buffered working set reused by the streamed
// layers: the i-th streamed layer's rows are copied into slot i % 2 on the
// copy stream while the compute stream runs decode attention + LSE merge of
// the layers before it.  This is the prefetch scheme of the "Online
// Log-Sum-Exp prefill & pipelined prefetch" item on the RX 9070 XT
// KV-streaming page (layer L+1's transfer overlaps layer L's compute) with
// the bounded, reused working set of "What shipped" on the ROCm KV-streaming
// page; which layers stay resident is the caller's choice for a device-memory
// budget (kvq_resident_layers gives the count that fits next to the slots).
//
// Ordering, per streamed layer L, the i-th streamed one, slot s = i % 2:
//   copy:    wait freed[s] (compute of streamed layer i-2 is done with slot s)
//            memcpy2D K rows [0, n_kv) of every head, then V rows
//            record ready[s]
//   compute: wait ready[s]; decode; merge into out[L]; record freed[s]
// A resident layer is decode + merge on the compute stream, in layer order.
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

// Where a layer's cache lives: 1 = pinned host, 2 = device memory of the current
// device, 0 = anything else (pageable host memory, another device, unknown).
int placement(const void *p)
{
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    if (at.type == cudaMemoryTypeHost)
        return 1;
    int dev = -1;
    if (at.type == cudaMemoryTypeDevice && cudaGetDevice(&dev) == cudaSuccess &&
        at.device == dev)
        return 2;
    return 0;
}

int fail_copy_layer()
{
    return test_hooks().stream_fail_layer.load(std::memory_order_relaxed);
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
    const int H = host_layers[0].n_kv_heads, D = host_layers[0].head_dim;
    const int64_t rows = (int64_t)T * n_q_heads;
    const int n_chunks = (int)((n_kv + chunk - 1) / chunk);
    st = validate_merge(out_part, lse_part, rows, n_chunks, D, out, lse, fn);
    if (st != KVQ_OK)
        return st;
    bool resident[KVQ_MAX_LAYERS];
    int n_streamed = 0;
    for (int l = 0; l < n_layers; ++l) {
        const int pk = placement(host_layers[l].k), pv = placement(host_layers[l].v);
        if (pk == 0 || pv == 0 || pk != pv)
            return set_error(KVQ_ERR_INVALID_ARG,
                             "%s: layer %d: K and V must both be pinned host memory or both "
                             "device memory of the current device",
                             fn, l);
        resident[l] = pk == 2;
        n_streamed += !resident[l];
    }
    if (n_streamed > 0) {
        if (!dev_slots)
            return set_error(KVQ_ERR_INVALID_ARG, "%s: dev_slots is NULL", fn);
        st = validate_decode(dev_slots, 2, q, n_q_heads, T, n_kv, chunk, scale, out_part,
                             lse_part, fn);
        if (st != KVQ_OK)
            return st;
        if (dev_slots[0].n_kv_heads != H || dev_slots[0].head_dim != D ||
            k_type_of(dev_slots[0]) != k_type_of(host_layers[0]) ||
            v_type_of(dev_slots[0]) != v_type_of(host_layers[0]))
            return set_error(KVQ_ERR_INVALID_ARG,
                             "%s: slots and host layers differ in shape or block formats", fn);
        for (int s = 0; s < 2; ++s)
            if (placement(dev_slots[s].k) != 2 || placement(dev_slots[s].v) != 2)
                return set_error(KVQ_ERR_INVALID_ARG,
                                 "%s: slot %d is not device memory of the current device", fn, s);
    }

    cudaStream_t cs = as_stream(compute), ps = as_stream(copy);
    Events E;
    if (!E.make())
        return set_error(KVQ_ERR_CUDA, "%s: cudaEventCreate failed", fn);
    cudaEvent_t start = E.ev[0], *ready = &E.ev[1], *freed = &E.ev[3];
    if (cudaEventRecord(start, cs) != cudaSuccess || cudaStreamWaitEvent(ps, start, 0) != cudaSuccess)
        return set_error(KVQ_ERR_CUDA, "%s: event ordering failed", fn);

    const int64_t kr = row_bytes(k_type_of(host_layers[0]), D);
    const int64_t vr = row_bytes(v_type_of(host_layers[0]), D);
    const int fail_at = fail_copy_layer();
    int i_streamed = 0;  // streamed layers enqueued so far
    for (int L = 0; L < n_layers; ++L) {
        const kvq_layer &hl = host_layers[L];
        const uint16_t *ql = q + (size_t)L * rows * D;
        if (resident[L]) {
            st = enqueue_decode(&hl, 1, ql, n_q_heads, T, n_kv, chunk, scale, out_part, lse_part,
                                cs);
            if (st != KVQ_OK)
                return st;
            launch_merge_lse(out_part, lse_part, rows, n_chunks, D, out + (size_t)L * rows * D,
                             lse + (size_t)L * rows, cs);
            st = check_launch(fn);
            if (st != KVQ_OK)
                return st;
            continue;
        }
        const int s = i_streamed & 1;
        const kvq_layer &sl = dev_slots[s];
        if (i_streamed >= 2 && cudaStreamWaitEvent(ps, freed[s], 0) != cudaSuccess)
            return set_error(KVQ_ERR_CUDA, "%s: event wait failed", fn);
        ++i_streamed;
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

extern "C" int kvq_resident_layers(size_t budget_bytes, int n_layers, int64_t capacity,
                                   int n_kv_heads, int head_dim, int k_type, int v_type)
{
    if (n_layers < 1 || capacity < 1 || n_kv_heads < 1 || head_dim < QK || head_dim % QK != 0)
        return -1;
    for (const int t : {k_type, v_type})
        if (!known_type(t))
            return -1;
    const int kt = k_type ? k_type : KVQ_TYPE_Q8_0, vt = v_type ? v_type : KVQ_TYPE_Q4_0;
    if (head_dim % block_elems(kt) != 0 || head_dim % block_elems(vt) != 0)
        return -1;
    const double layer = (double)n_kv_heads * (double)capacity *
                         (double)(row_bytes(kt, head_dim) + row_bytes(vt, head_dim));
    const double budget = (double)budget_bytes;
    if (layer * n_layers <= budget)
        return n_layers;  // everything resident: no slots needed
    if (2.0 * layer > budget)
        return -1;  // not even the two streaming slots fit
    const double r = (budget - 2.0 * layer) / layer;
    return r >= n_layers - 1 ? n_layers - 1 : (int)r;
}
