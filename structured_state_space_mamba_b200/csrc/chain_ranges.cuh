// chain_ranges.cuh -- how the single-pass kernels split the (chain, chunk) work
// items over CTAs.  A chain is the chunk sequence of one (batch, head pair),
// chain-major: item i = chain * nc + chunk.  CTA k of G takes the items
// [k I / G, (k + 1) I / G) (I items).  Every kernel that must agree on where a
// CTA's range begins and ends (the single pass, the pass that computes the
// states entering the ranges, and the pass that combines them) uses this one
// definition.
#pragma once

#include <cstdint>

namespace ssd {

struct ChainRange {
    int cf, cfc;  // first chain, and its first chunk
    int cl, clc;  // last chain, and its end chunk (exclusive)
};

// First item of CTA k of G.
__host__ __device__ inline long long chain_range_begin(long long items, int k, int G) {
    return items * k / G;
}

__host__ __device__ inline ChainRange chain_range(long long chains, int nc, int k, int G) {
    const long long items = chains * nc;
    const long long i0 = chain_range_begin(items, k, G), i1 = chain_range_begin(items, k + 1, G);
    ChainRange r;
    r.cf = int(i0 / nc);
    r.cfc = int(i0 % nc);
    r.cl = int((i1 - 1) / nc);
    r.clc = int((i1 - 1) % nc) + 1;
    return r;
}

}  // namespace ssd
