// common.cuh -- small device helpers shared by the scan, decode and convolution kernels.
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

// Packed FP32 pairs (sm_100: one instruction does two FP32 FMAs / sums / products, each
// rounded as fmaf / a plain sum or product would be).  Used where independent values pair up.
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 ex2_pair(float2 v) { return f2(ex2_approx(v.x), ex2_approx(v.y)); }

// A constant shaped like v, and one Horner step p * u + c, on a value or on a pair of
// values (c the same for both halves).
__device__ __forceinline__ float splat(float, float c) { return c; }
__device__ __forceinline__ float2 splat(float2, float c) { return f2(c, c); }
__device__ __forceinline__ float horner(float p, float u, float c) { return fmaf(p, u, c); }
__device__ __forceinline__ float2 horner(float2 p, float2 u, float c) { return ffma2(p, u, f2(c, c)); }

// log1p(u) for u in [0, 1] is u * p(u), p a degree-7 polynomial fitted to log1p(u)/u (least
// squares at Chebyshev nodes, relative weighting).  Evaluated in fp32 Horner form u * p(u)
// has a relative error below 3.3e-7 on the whole interval.  log1p_poly gives p(u), for one
// value or a pair (each half rounded exactly as the single value is).
template <typename V> __device__ __forceinline__ V log1p_poly(V u) {
    V p = splat(u, -0.008336497470736504f);
    p = horner(p, u, 0.04337085038423538f);
    p = horner(p, u, -0.10667790472507477f);
    p = horner(p, u, 0.1767549365758896f);
    p = horner(p, u, -0.2447046935558319f);
    p = horner(p, u, 0.3327118754386902f);
    p = horner(p, u, -0.49997127056121826f);
    p = horner(p, u, 0.9999997615814209f);
    return p;
}

// softplus(v) = log(1 + e^v), in the overflow-free form max(v, 0) + log1p(e^-|v|): one SFU
// exponential, the logarithm on the FMA pipe, its last product fused with the sum.
__device__ __forceinline__ float softplus_f(float v) {
    const float u = ex2_approx(-fabsf(v) * kLog2e);
    return fmaf(u, log1p_poly(u), fmaxf(v, 0.f));
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

// softplus_f and silu_f on two values at once: the same operations in the same order on
// each half, the FP32 ones as packed pairs, so the results are bit-identical to the scalar
// functions'.
__device__ __forceinline__ float2 softplus_pair(float2 v) {
    const float2 u = f2(ex2_approx(-fabsf(v.x) * kLog2e), ex2_approx(-fabsf(v.y) * kLog2e));
    return ffma2(u, log1p_poly(u), f2(fmaxf(v.x, 0.f), fmaxf(v.y, 0.f)));
}
__device__ __forceinline__ float2 silu_pair(float2 z) {
    const float2 e = ex2_pair(fmul2(z, f2(-kLog2e, -kLog2e)));
    const float2 d = fadd2(f2(1.f, 1.f), e);
    return fmul2(z, f2(rcp_approx(d.x), rcp_approx(d.y)));
}

// A pair of bf16 values packed in 32 bits (first in the low half) as an fp32 pair: bf16 ->
// fp32 is a 16-bit shift (exact).
__device__ __forceinline__ float2 bf16x2_to_f2(unsigned w) {
    return f2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
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

// 8 consecutive values of a staged row as fp32 (16-byte aligned source).
template <typename T> __device__ __forceinline__ void load8(const T *src, float (&v)[8]);
template <> __device__ __forceinline__ void load8<float>(const float *src, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4 *>(src);
    const float4 b = *reinterpret_cast<const float4 *>(src + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <> __device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *src, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(src);
    const unsigned w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {            // bf16 -> fp32 is a 16-bit left shift
        v[2 * k] = __uint_as_float(w[k] << 16);
        v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
}

// 8 fp32 values stored as 8 values of T (16-byte aligned destination).
template <typename T> __device__ __forceinline__ void store8(T *dst, const float (&v)[8]);
template <> __device__ __forceinline__ void store8<float>(float *dst, const float (&v)[8]) {
    *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4 *>(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
template <> __device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16 *dst, const float (&v)[8]) {
    unsigned w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
        w[k] = *reinterpret_cast<const unsigned *>(&p);
    }
    *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Store n (4 or 8) consecutive outputs with the widest aligned vectors: n * sizeof(T)
// bytes, so the destination must be aligned to that (16 bytes, or 8 for 4 bf16).
template <int n> __device__ __forceinline__ void store_run(float *p, const float *v) {
#pragma unroll
    for (int k = 0; k < n; k += 4)
        *reinterpret_cast<float4 *>(p + k) = make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
}
__device__ __forceinline__ unsigned pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const unsigned *>(&h);
}
template <int n> __device__ __forceinline__ void store_run(__nv_bfloat16 *p, const float *v) {
    if constexpr (n == 4) {
        *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    } else {
#pragma unroll
        for (int k = 0; k < n; k += 8)
            *reinterpret_cast<uint4 *>(p + k) =
                make_uint4(pack_bf16x2(v[k], v[k + 1]), pack_bf16x2(v[k + 2], v[k + 3]),
                           pack_bf16x2(v[k + 4], v[k + 5]), pack_bf16x2(v[k + 6], v[k + 7]));
    }
}

// n = 4 or 8 consecutive values of a staged row as fp32 / stored from fp32 (the source or
// destination aligned to n * sizeof(T) bytes).
template <int n, typename T> __device__ __forceinline__ void loadn(const T *src, float (&v)[n]) {
    if constexpr (n == 8) {
        load8<T>(src, v);
    } else if constexpr (sizeof(T) == 4) {
        const float4 a = *reinterpret_cast<const float4 *>(src);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else {
        const uint2 u = *reinterpret_cast<const uint2 *>(src);
        v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xffff0000u);
        v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xffff0000u);
    }
}
template <int n, typename T> __device__ __forceinline__ void storen(T *dst, const float (&v)[n]) {
    if constexpr (n == 8) store8<T>(dst, v);
    else store_run<4>(dst, v);
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

}  // namespace ssm
