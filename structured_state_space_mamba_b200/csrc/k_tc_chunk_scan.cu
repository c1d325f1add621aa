// k_tc_chunk_scan.cu -- tcgen05 ssd_chunk_scan (bf16, P == 64).
#include "common.cuh"
#include "kernels.h"

namespace ssd {

bool tc_chunk_scan_supported(const Dims &) { return false; }

cudaError_t launch_chunk_scan_tc(const Dims &, const void *, const float *, const void *,
                                 const void *, const float *, const float *, const void *,
                                 void *, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace ssd
