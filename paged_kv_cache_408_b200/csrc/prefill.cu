// prefill.cu -- causal chunked-prefill attention over a paged prefix (sm_100a).
#include "common.cuh"
#include "kernels.h"

namespace pa {

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t st) {
    (void)a;
    (void)st;
    return cudaErrorNotSupported;
}

}  // namespace pa
