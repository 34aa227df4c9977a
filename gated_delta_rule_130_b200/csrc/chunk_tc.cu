// Fused tcgen05 chunkwise forward (not yet enabled: every size takes the
// CUDA-core path).
#include "kernels.h"

namespace gdn {

bool tc_supported(int, int, int, int, int, int, bool) { return false; }

cudaError_t launch_chunk_tc(const void *, const void *, const void *, const float *,
                            const float *, const float *, void *, float *, int, int, int, int,
                            int, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace gdn
