// common.cuh -- small device helpers shared by the scan and decode kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ int tid_x() { return static_cast<int>(threadIdx.x); }

// Hardware base-2 exponential (the SFU's ex2), flush-to-zero.  Used for the per-(t, n)
// decay exp(Delta * a) = 2^(Delta * a * log2 e), with a * log2 e folded in once per state.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Hardware reciprocal (SFU); rcp(+inf) = 0, which the SiLU gate relies on for z -> -inf.
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log1p(u) for u in [0, 1], as u * p(u) with p a degree-7 polynomial fitted to log1p(u)/u
// (least squares at Chebyshev nodes, relative weighting).  Evaluated in fp32 Horner form
// its relative error is below 3.3e-7 on the whole interval.
__device__ __forceinline__ float log1p_unit(float u) {
    float p = -0.008336497470736504f;
    p = fmaf(p, u, 0.04337085038423538f);
    p = fmaf(p, u, -0.10667790472507477f);
    p = fmaf(p, u, 0.1767549365758896f);
    p = fmaf(p, u, -0.2447046935558319f);
    p = fmaf(p, u, 0.3327118754386902f);
    p = fmaf(p, u, -0.49997127056121826f);
    p = fmaf(p, u, 0.9999997615814209f);
    return u * p;
}

// softplus(v) = log(1 + e^v), in the overflow-free form max(v, 0) + log1p(e^-|v|):
// one SFU exponential, the logarithm on the FMA pipe.
__device__ __forceinline__ float softplus_f(float v) {
    return fmaxf(v, 0.f) + log1p_unit(ex2_approx(-fabsf(v) * kLog2e));
}

// expm1(v) for |v| < 0.1 from its Taylor series through v^5 (truncation below 1.4e-8
// relative): near 0, exp(v) - 1 computed from exp(v) would lose the leading digits.
__device__ __forceinline__ float expm1_small(float v) {
    float p = 1.f / 120.f;
    p = fmaf(p, v, 1.f / 24.f);
    p = fmaf(p, v, 1.f / 6.f);
    p = fmaf(p, v, 0.5f);
    p = fmaf(p, v, 1.f);
    return v * p;
}

// SiLU(z) = z * sigmoid(z) = z / (1 + e^-z).
__device__ __forceinline__ float silu_f(float z) {
    return z * rcp_approx(1.f + ex2_approx(-z * kLog2e));
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// 16-byte asynchronous global -> shared copy (bypasses L1), grouped with commit/wait.
__device__ __forceinline__ void cp_async_16(void *smem_dst, const void *gmem_src) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Sum of per-lane partials over the G lanes that share one channel (G consecutive lanes),
// "transposed": on entry each lane holds partial sums p[0..G) for G consecutive
// timesteps; on exit lane r of the group holds the full sum for timestep r.  Costs
// G-1 shuffles per G timesteps instead of G*log2(G) for G separate butterflies.
template <int G> struct GroupReduceScatter;

template <> struct GroupReduceScatter<1> {
    __device__ __forceinline__ static float run(const float *p, int) { return p[0]; }
};

template <> struct GroupReduceScatter<2> {
    __device__ __forceinline__ static float run(const float *p, int r) {
        const float send = (r & 1) ? p[0] : p[1];
        const float keep = (r & 1) ? p[1] : p[0];
        return keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
};

template <> struct GroupReduceScatter<4> {
    __device__ __forceinline__ static float run(const float *p, int r) {
        const bool hi = (r & 2) != 0;
        const float s0 = hi ? p[0] : p[2], s1 = hi ? p[1] : p[3];
        const float k0 = hi ? p[2] : p[0], k1 = hi ? p[3] : p[1];
        const float q0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 2);
        const float q1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 2);
        const bool lo = (r & 1) != 0;
        const float send = lo ? q0 : q1;
        const float keep = lo ? q1 : q0;
        return keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
};

}  // namespace ssm
