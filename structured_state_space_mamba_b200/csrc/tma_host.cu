// tma_host.cu -- see tma_host.h.
#include <cudaTypedefs.h>

#include <mutex>
#include <map>
#include <utility>

#include "tma_host.h"

namespace ssd {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_once;

void resolve() {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    else
        cudaGetLastError();
}

}  // namespace

bool make_tmap_bf16(CUtensorMap *out, int rank, const void *base, const uint64_t *dims,
                    const uint64_t *stride_bytes, const uint32_t *box, int swizzle_bytes) {
    std::call_once(g_once, resolve);
    if (!g_encode || rank < 2 || rank > 5) return false;
    CUtensorMapSwizzle swz;
    switch (swizzle_bytes) {
        case 0: swz = CU_TENSOR_MAP_SWIZZLE_NONE; break;
        case 32: swz = CU_TENSOR_MAP_SWIZZLE_32B; break;
        case 64: swz = CU_TENSOR_MAP_SWIZZLE_64B; break;
        case 128: swz = CU_TENSOR_MAP_SWIZZLE_128B; break;
        default: return false;
    }
    cuuint64_t gdim[5], gstride[4];
    cuuint32_t bdim[5], estride[5];
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        bdim[i] = box[i];
        estride[i] = 1;
        if (i + 1 < rank) gstride[i] = stride_bytes[i];
    }
    CUresult r = g_encode(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cuuint32_t(rank),
                          const_cast<void *>(base), gdim, gstride, bdim, estride,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool smem_attr_once(const void *kernel, int bytes) {
    static std::mutex mu;
    static std::map<std::pair<int, const void *>, int> done;  // largest limit set so far
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(dev, kernel);
    auto it = done.find(key);
    if (it != done.end() && it->second >= bytes) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    done[key] = bytes;
    return true;
}

int device_sm_count() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 148;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        cache[dev] = n;
    }
    return cache[dev];
}

}  // namespace ssd
