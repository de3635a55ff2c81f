// Tensor-core (tcgen05) chunked prefill for bf16 q/k/v, d_k = d_v = 128, chunk 64.
#include "kda_internal.h"

namespace kda {

bool prefill_tc_supported(const PrefillArgs &) { return false; }

cudaError_t launch_prefill_tc(const PrefillArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kda
