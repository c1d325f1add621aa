// k_tc_chunk_state.cu -- tcgen05 ssd_chunk_state (bf16, P == 64).
#include "common.cuh"
#include "kernels.h"

namespace ssd {

bool tc_chunk_state_supported(const Dims &) { return false; }

cudaError_t launch_chunk_state_tc(const Dims &, const void *, const void *, const float *,
                                  float *, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace ssd
