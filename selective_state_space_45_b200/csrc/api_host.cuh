// api_host.cuh -- host-side argument helpers shared by the C ABI translation units.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/ssm.h"

namespace ssm_host {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool valid_dtype(int t) { return t == SSM_F32 || t == SSM_BF16; }

inline int status_of(cudaError_t e) { return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA; }

inline size_t dtype_size(int t) { return t == SSM_F32 ? 4 : 2; }

// Do the byte ranges [p, p + pb) and [q, q + qb) share a byte?
inline bool overlaps(const void *p, size_t pb, const void *q, size_t qb) {
    if (!p || !q || pb == 0 || qb == 0) return false;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
    return a < b + qb && b < a + pb;
}

}  // namespace ssm_host
