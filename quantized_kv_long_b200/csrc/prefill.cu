// prefill.cu -- chunked prefill attention (not yet built: reports unsupported).
#include "common.cuh"

namespace kvq {

size_t prefill_workspace_bytes(int, int, int, int, int) { return 0; }

bool prefill_supported(int, int, int) { return false; }

void launch_prefill(const PrefillArgs &, cudaStream_t) {}

}  // namespace kvq
