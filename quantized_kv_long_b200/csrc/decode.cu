// decode.cu -- dispatch of split-KV decode attention.
#include "common.cuh"

namespace kvq {

bool launch_decode_simple(const DecodeArgs &a, cudaStream_t s);

bool launch_decode(const DecodeArgs &a, cudaStream_t s)
{
    return launch_decode_simple(a, s);
}

}  // namespace kvq
