// noalloc.cu -- decode attention + LSE merge for callers that cannot allocate.
//
// kvq_decode_attn followed by kvq_merge_lse needs the chunk partials
// (out_part, lse_part) in device memory that the caller provides.  Some callers
// have no way to provide it: a plug-in that runs inside a host program which
// owns every byte of device memory and hands out only the input and output
// tensors, or a latency-critical loop where a cudaMalloc (which may
// synchronise the device and may fail under memory pressure) is not allowed
// between steps.  kvq_decode_merged_static serves them: the partials live in a
// fixed array in the library itself, so the call needs only its inputs and
// its outputs.
//
// The array is a file-scope __device__ object of KVQ_STATIC_SCRATCH_BYTES
// (8 MiB): every GPU on which the library is loaded keeps those 8 MiB until
// the process exits.  Host code never uses the array's name as an address:
// the device address comes from cudaGetSymbolAddress, taken per device (with
// that device current) on the first call made on it and kept in an atomic, so
// that host threads calling at the same time may each look it up but never
// race on the stored value.
#include <atomic>

#include "common.cuh"

namespace kvq {

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[KVQ_STATIC_SCRATCH_BYTES];

std::atomic<unsigned char *> g_scratch_addr[MAX_DEVICES];

// Device address of this device's scratch array (looked up once per device).
kvq_status scratch_address(unsigned char **out, const char *fn)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return set_error(KVQ_ERR_CUDA, "%s: cudaGetDevice: %s", fn, cudaGetErrorString(e));
    if (dev < 0 || dev >= MAX_DEVICES)
        return set_error(KVQ_ERR_UNSUPPORTED, "%s: device %d beyond %d", fn, dev, MAX_DEVICES);
    unsigned char *addr = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!addr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess || p == nullptr)
            return set_error(KVQ_ERR_CUDA, "%s: cudaGetSymbolAddress: %s", fn,
                             cudaGetErrorString(e));
        addr = static_cast<unsigned char *>(p);
        g_scratch_addr[dev].store(addr, std::memory_order_release);
    }
    *out = addr;
    return KVQ_OK;
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" kvq_status kvq_decode_merged_static(const kvq_layer *layers, int n_layers,
                                               const uint16_t *q, int n_q_heads, int T,
                                               int64_t n_kv, int chunk, float scale, float *out,
                                               float *lse, kvq_stream stream)
{
    const char *fn = "kvq_decode_merged_static";
    unsigned char *base = nullptr;
    kvq_status st = scratch_address(&base, fn);
    if (st != KVQ_OK)
        return st;
    // every argument is checked before any size is derived from it; the partial
    // pointers given here are the array's start (the real lse_part offset follows)
    st = validate_decode(layers, n_layers, q, n_q_heads, T, n_kv, chunk, scale,
                         reinterpret_cast<float *>(base), reinterpret_cast<float *>(base), fn);
    if (st != KVQ_OK)
        return st;
    // validated: 1 <= n_layers <= KVQ_MAX_LAYERS, n_kv <= capacity, at most 2^30
    // chunks and head_dim <= 512, so a row's partials take below 2^42 bytes and the
    // row count test below keeps every product in range
    const int D = layers[0].head_dim;
    const int64_t rows = (int64_t)n_layers * T * n_q_heads;
    const int64_t n_chunks = (n_kv + chunk - 1) / chunk;
    const int64_t row_bytes = n_chunks * ((int64_t)D * 4 + 4);
    // partials: out_part [rows][n_chunks][D] then lse_part [rows][n_chunks], 256-B aligned
    const int64_t fits = rows <= (int64_t)KVQ_STATIC_SCRATCH_BYTES / row_bytes;
    const int64_t part_bytes = fits ? ((rows * n_chunks * D * 4 + 255) / 256) * 256 : 0;
    const int64_t need = fits ? part_bytes + rows * n_chunks * 4 : 0;
    if (!fits || need > (int64_t)KVQ_STATIC_SCRATCH_BYTES)
        return set_error(KVQ_ERR_UNSUPPORTED,
                         "%s: %lld rows x %lld chunks of partials exceed the %lld-byte static "
                         "scratch (fewer layers or larger chunks per call)",
                         fn, (long long)rows, (long long)n_chunks,
                         (long long)KVQ_STATIC_SCRATCH_BYTES);
    float *out_part = reinterpret_cast<float *>(base);
    float *lse_part = reinterpret_cast<float *>(base + part_bytes);
    st = validate_merge(out_part, lse_part, rows, (int)n_chunks, D, out, lse, fn);
    if (st != KVQ_OK)
        return st;
    // the decode writes every chunk partial (fully masked ones as 0 and -inf), so
    // nothing in the array needs clearing between calls
    st = enqueue_decode(layers, n_layers, q, n_q_heads, T, n_kv, chunk, scale, out_part, lse_part,
                        as_stream(stream));
    if (st != KVQ_OK)
        return st;
    launch_merge_lse(out_part, lse_part, rows, (int)n_chunks, D, out, lse, as_stream(stream));
    return check_launch(fn);
}
