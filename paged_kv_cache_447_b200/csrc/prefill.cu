// prefill.cu -- paged causal prefill attention (placeholder until the tcgen05 kernel lands).
#include "common.cuh"
#include "internal.h"

namespace pkv {
cudaError_t launch_paged_prefill(const PrefillArgs &, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace pkv
