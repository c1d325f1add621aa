// tma_host.h -- host-side creation of TMA tensor maps.
//
// cuTensorMapEncodeTiled is a driver API function; it is looked up once per
// process through cudaGetDriverEntryPoint so that libssd.so carries no link
// dependency on the driver library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// Encode a tiled bf16 tensor map of rank 2..5.
//   dims[i]          extent of dimension i (dimension 0 is contiguous)
//   stride_bytes[i]  byte stride of dimension i+1 (i = 0 .. rank-2), multiple of 16
//   box[i]           box extent per dimension (<= 256; box[0] * 2 bytes <= swizzle span)
//   swizzle_bytes    0 (none), 32, 64 or 128
// Returns false if the driver entry point is unavailable or encoding fails.
bool make_tmap_bf16(CUtensorMap *out, int rank, const void *base, const uint64_t *dims,
                    const uint64_t *stride_bytes, const uint32_t *box, int swizzle_bytes);

// Make sure a kernel's dynamic shared memory limit on the current device is at
// least `bytes` (the attribute is set only when it must grow; otherwise this
// is a lookup).  Returns false on failure.
bool smem_attr_once(const void *kernel, int bytes);

// Number of SMs of the current device (cached per device).
int device_sm_count();

}  // namespace ssd
