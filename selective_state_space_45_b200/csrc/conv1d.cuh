// conv1d.cuh -- the causal depthwise convolution (+ bias, + SiLU) that filters each channel
// over its last K inputs before the selective scan, and its one-token decode form.
//
// Definition (learnllm "Module 19: State Space Models & Mamba", section "The Causal
// Convolution"; xmarva "Lesson 10", section 4 "The Mamba block"): each channel d has its
// own K taps w[d][0..K); output t reads x[t-K+1..t], tap i on x[t-K+1+i], with the K-1
// positions before the sequence taken from a carried history (zeros by default, the left
// pad), then SiLU.  The decode form (xmarva section 7) keeps the last K-1 inputs per
// channel as a window, oldest first.
//
// Both kernels are HBM-bound (K FMAs and one SiLU per element against 2-8 bytes moved).
#pragma once

#include "common.cuh"

namespace ssm {

struct ConvArgs {
    const void *x;         // [batch][dim][seqlen], Tin
    const float *w;        // [dim][K]
    const float *bias;     // [dim] or null
    const float *hist;     // [batch][dim][K-1] or null (zeros)
    void *u;               // [batch][dim][seqlen], Tout
    float *hist_out;       // [batch][dim][K-1] or null
    long long rows;        // batch * dim
    int dim;
    long long seqlen;
    int K;
    int silu;
};

template <typename T> struct Vec16;  // one 16-byte vector of T
template <> struct Vec16<float> {
    static constexpr int kN = 4;
    __device__ __forceinline__ static void load(const float *p, float *v) {
        const float4 q = __ldg(reinterpret_cast<const float4 *>(p));
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int kN = 8;
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float *v) {
        const uint4 q = __ldg(reinterpret_cast<const uint4 *>(p));
        const unsigned w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w4[i] << 16);
            v[2 * i + 1] = __uint_as_float(w4[i] & 0xffff0000u);
        }
    }
};

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

// Vector path: rows whose length is a multiple of one 16-byte vector and 16-byte aligned
// tensors.  Thread g owns chunk c = g mod nchunk of row g / nchunk: CH = 2 vectors of
// consecutive tokens (the last chunk of a row may hold one).  The K-1 inputs before the
// chunk come from lane - 1 by shuffle (it owns chunk c-1 of the same row), from the carried
// history when c = 0, and from global memory for lane 0.  All lanes of a warp run the
// loop together so that the shuffles see every lane.
template <typename Tin, typename Tout, int K>
__global__ void __launch_bounds__(256)
causal_conv1d_vec_kernel(ConvArgs a, long long nchunk, long long total) {
    constexpr int V = Vec16<Tin>::kN;
    constexpr int CH = 2 * V;
    constexpr int H = K - 1;
    const Tin *__restrict__ x = static_cast<const Tin *>(a.x);
    Tout *__restrict__ u = static_cast<Tout *>(a.u);
    const int lane = threadIdx.x & 31;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
         g - lane < total; g += stride) {
        const bool active = g < total;
        const long long row = active ? g / nchunk : 0;
        const long long c = active ? g - row * nchunk : 0;
        const long long t0 = c * CH;
        const long long base = row * a.seqlen + t0;
        const bool second = active && t0 + V < a.seqlen;
        // xe[0..H) = inputs t0-H .. t0-1, xe[H..H+CH) = this chunk
        float xe[H + CH];
#pragma unroll
        for (int i = 0; i < H + CH; ++i) xe[i] = 0.f;
        if (active) Vec16<Tin>::load(x + base, xe + H);
        if (second) Vec16<Tin>::load(x + base + V, xe + H + V);
        // the previous chunk is always full, so its last H values are xe[CH..CH+H) of lane - 1
#pragma unroll
        for (int j = 0; j < H; ++j) xe[j] = __shfl_up_sync(0xffffffffu, xe[CH + j], 1);
        if (active && c == 0) {
            const float *hp = a.hist ? a.hist + row * H : nullptr;
#pragma unroll
            for (int j = 0; j < H; ++j) xe[j] = hp ? __ldg(hp + j) : 0.f;
        } else if (active && lane == 0) {
#pragma unroll
            for (int j = 0; j < H; ++j) xe[j] = to_f32<Tin>(x[base - H + j]);
        }
        if (!active) continue;
        const int d = static_cast<int>(row % a.dim);
        float w[K];
#pragma unroll
        for (int i = 0; i < K; ++i) w[i] = __ldg(a.w + static_cast<long long>(d) * K + i);
        const float b0 = a.bias ? __ldg(a.bias + d) : 0.f;
        float o[CH];
#pragma unroll
        for (int t = 0; t < CH; ++t) {
            float acc = b0;
#pragma unroll
            for (int i = 0; i < K; ++i) acc = fmaf(w[i], xe[t + i], acc);
            o[t] = a.silu ? silu_f(acc) : acc;
        }
        store_run<V>(u + base, o);
        if (second) store_run<V>(u + base + V, o + V);
        if (a.hist_out && H > 0 && t0 + CH >= a.seqlen) {
            // the row's last chunk: the window a decode step continues from
            // its last H inputs end the chunk's one or two vectors (V >= H)
#pragma unroll
            for (int j = 0; j < H; ++j) a.hist_out[row * H + j] = second ? xe[CH + j] : xe[V + j];
        }
    }
}

// General path: any width 1 <= K <= kMaxConvWidth, any row length, any alignment.  One
// thread per output element, each reading its K inputs (neighbours share them through L1).
constexpr int kMaxConvWidth = 8;

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) causal_conv1d_any_kernel(ConvArgs a) {
    const Tin *__restrict__ x = static_cast<const Tin *>(a.x);
    Tout *__restrict__ u = static_cast<Tout *>(a.u);
    const int K = a.K, H = K - 1;
    const long long total = a.rows * a.seqlen;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += stride) {
        const long long row = e / a.seqlen;
        const long long t = e - row * a.seqlen;
        const int d = static_cast<int>(row % a.dim);
        const float *hp = a.hist ? a.hist + row * H : nullptr;
        float acc = a.bias ? __ldg(a.bias + d) : 0.f;
        for (int i = 0; i < K; ++i) {
            const long long s = t - H + i;  // position of tap i's input; < 0 is the history
            const float xv = s >= 0 ? to_f32<Tin>(x[row * a.seqlen + s])
                                    : (hp ? __ldg(hp + H + s) : 0.f);
            acc = fmaf(__ldg(a.w + static_cast<long long>(d) * K + i), xv, acc);
        }
        u[e] = from_f32<Tout>(a.silu ? silu_f(acc) : acc);
        if (a.hist_out && t == a.seqlen - 1) {
            for (int j = 0; j < H; ++j) {
                const long long s = a.seqlen - H + j;
                a.hist_out[row * H + j] = s >= 0 ? to_f32<Tin>(x[row * a.seqlen + s])
                                                 : (hp ? __ldg(hp + H + s) : 0.f);
            }
        }
    }
}

// Decode: one token per (batch, channel) row.  window[row][0..K-1) holds the previous K-1
// inputs, oldest first; the output reads them and the new input, then the window drops its
// oldest entry and appends the new input, in place.  One thread per row, all loads before
// the stores.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256)
conv1d_step_kernel(float *__restrict__ window, const Tin *__restrict__ x,
                   const float *__restrict__ w, const float *__restrict__ bias, Tout *__restrict__ u,
                   long long rows, int dim, int K, int silu) {
    const long long row = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (row >= rows) return;
    const int H = K - 1;
    const int d = static_cast<int>(row % dim);
    float win[kMaxConvWidth];
#pragma unroll
    for (int j = 0; j < kMaxConvWidth - 1; ++j)
        win[j] = j < H ? window[row * H + j] : 0.f;
    const float xv = to_f32<Tin>(x[row]);
    const float *wd = w + static_cast<long long>(d) * K;
    float acc = bias ? __ldg(bias + d) : 0.f;
#pragma unroll
    for (int i = 0; i < kMaxConvWidth - 1; ++i)
        if (i < H) acc = fmaf(__ldg(wd + i), win[i], acc);
    acc = fmaf(__ldg(wd + H), xv, acc);
    u[row] = from_f32<Tout>(silu ? silu_f(acc) : acc);
#pragma unroll
    for (int j = 0; j < kMaxConvWidth - 1; ++j)
        if (j < H) window[row * H + j] = j + 1 < H ? win[j + 1] : xv;
}

}  // namespace ssm
