// decode.cu -- which kernel runs a split-KV decode.
//
// Both kernels compute the same chunk partials (speculative-decoding
// paragraph of the RX 9070 XT KV-streaming page: paged decode attention over
// a verify batch; GQA section of the KV-cache guide):
//  * decode_tmem.cu -- head_dim 256, up to 24 query rows per KV head, Q8_0 K
//    with Q4_0 V: the persistent tcgen05 kernel;
//  * decode_simple.cu -- every other supported shape and block format.
#include "common.cuh"

namespace kvq {

bool launch_decode_simple(const DecodeArgs &a, cudaStream_t s);
bool launch_decode_tmem(const DecodeArgs &a, cudaStream_t s);

bool decode_tc_supported(const DecodeArgs &a)
{
    const int rows = (a.n_q_heads / a.n_kv_heads) * a.T;
    return a.head_dim == 256 && rows <= 24 && a.k_type == KVQ_TYPE_Q8_0 &&
           a.v_type == KVQ_TYPE_Q4_0;
}

bool launch_decode(const DecodeArgs &a, cudaStream_t s)
{
    if (!a.force_simple && decode_tc_supported(a))
        return launch_decode_tmem(a, s);
    return launch_decode_simple(a, s);
}

}  // namespace kvq
