// Chunked-prefill attention against the paged cache (tcgen05 tensor-core path).
#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {

cudaError_t launch_prefill(const PrefillLaunch &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace pa
