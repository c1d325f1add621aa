// tc_scan_common.cuh -- shared-memory operand helpers of the tensor-core chunk
// scan kernels.
#pragma once

#include "tc_common.cuh"

namespace ssd {
namespace tc {

// Bytes per row of a K-major operand slab: 64-column (128-byte) slabs for
// N >= 64, one narrower slab otherwise.
__host__ __device__ constexpr int row_bytes(int n) { return n >= 64 ? 128 : n * 2; }
__host__ __device__ constexpr uint32_t kmajor_swz(int n) { return n >= 64 ? kSw128 : (n == 32 ? kSw64 : kSw32); }
__host__ __device__ constexpr uint32_t up1k(uint32_t v) { return (v + 1023u) & ~1023u; }
__host__ __device__ constexpr uint32_t umax(uint32_t a, uint32_t b) { return a > b ? a : b; }

// K-major operand descriptor for K step k of a tile split into 64-column slabs
// of `rows` rows (N >= 64) or a single slab of narrower rows (N = 16, 32).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int k, int rows, int n) {
    if (n >= 64) return smem_desc(base + (k >> 2) * rows * 128 + (k & 3) * 32, 16, 1024, kSw128);
    return smem_desc(base + k * 32, 16, 8 * row_bytes(n), kmajor_swz(n));
}

// Scale every bf16 of `n16` 16-byte chunks starting at `p` by f(chunk index);
// thread i handles chunks i, i + nthr, ...  Four chunks (and their factors)
// are loaded before any is stored: the stores may alias the loads, so a fused
// loop would run at shared-memory latency.
template <typename F>
__device__ __forceinline__ void scale_chunks(uint8_t *p, int n16, int i, int nthr, F f) {
    uint4 *q = reinterpret_cast<uint4 *>(p);
    for (int k0 = i; k0 < n16; k0 += 4 * nthr) {
        uint4 v[4];
        float sc[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = k0 + j * nthr;
            if (k < n16) {
                v[j] = q[k];
                sc[j] = f(k);
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = k0 + j * nthr;
            if (k < n16) {
                uint4 o;
                o.x = pack_bf16x2(bf16lo(v[j].x) * sc[j], bf16hi(v[j].x) * sc[j]);
                o.y = pack_bf16x2(bf16lo(v[j].y) * sc[j], bf16hi(v[j].y) * sc[j]);
                o.z = pack_bf16x2(bf16lo(v[j].z) * sc[j], bf16hi(v[j].z) * sc[j]);
                o.w = pack_bf16x2(bf16lo(v[j].w) * sc[j], bf16hi(v[j].w) * sc[j]);
                q[k] = o;
            }
        }
    }
}

}  // namespace tc
}  // namespace ssd
