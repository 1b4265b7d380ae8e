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

// One 16-byte vector of T: kN elements, loaded raw (Raw) and widened to fp32 (unpack).
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int kN = 4;
    using Raw = float4;
    __device__ __forceinline__ static void unpack(const float4 &q, float *v) {
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int kN = 8;
    using Raw = uint4;
    __device__ __forceinline__ static void unpack(const uint4 &q, float *v) {
        const unsigned w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {   // bf16 -> fp32 is exact: the bits move up 16 places
            v[2 * i] = __uint_as_float(w4[i] << 16);
            v[2 * i + 1] = __uint_as_float(w4[i] & 0xffff0000u);
        }
    }
};

// Vector path: rows whose length is a multiple of one 16-byte vector (V elements), widths
// 1..4 (K-1 <= V).  Each warp owns a span of 32*U consecutive vectors of one row, laid out
// as a copy kernel lays them out: vector v0 + 32k + lane goes to lane `lane`, load k, so
// every load and store instruction of the warp covers 512 contiguous bytes.  The K-1
// inputs in front of a vector are the tail of the vector before it: lane - 1's vector of
// the same load, lane 31's vector of the previous load (for lane 0), and for the span's
// first vector the row itself (span > 0) or the carried window (span 0).  All U loads are
// issued before any arithmetic.
// 6 resident blocks of 256 threads per SM (a 40-register budget); fp32 inputs with bf16
// outputs need a few more registers to pack, and take 5.
template <typename Tin, typename Tout, int K, int U>
__global__ void __launch_bounds__(256, (sizeof(Tin) == 4 && sizeof(Tout) == 2) ? 5 : 6)
causal_conv1d_vec_kernel(ConvArgs a, long long nvr, long long spans_per_row, long long total_spans) {
    constexpr int V = Vec16<Tin>::kN;
    constexpr int H = K - 1;
    static_assert(H <= V, "the window must fit in one vector");
    using R = typename Vec16<Tin>::Raw;
    const int lane = threadIdx.x & 31;
    const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (gw >= total_spans) return;   // the whole warp: the shuffles below see all lanes
    const long long row = gw / spans_per_row;
    const long long v0 = (gw - row * spans_per_row) * (32 * U);
    const Tin *__restrict__ xr = static_cast<const Tin *>(a.x) + row * a.seqlen;
    Tout *__restrict__ ur = static_cast<Tout *>(a.u) + row * a.seqlen;
    R raw[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
        const long long p = v0 + 32 * k + lane;
        if (p < nvr) raw[k] = __ldg(reinterpret_cast<const R *>(xr + p * V));
        else raw[k] = R{};
    }
    const int d = static_cast<int>(row % a.dim);
    float w[K];
#pragma unroll
    for (int i = 0; i < K; ++i) w[i] = __ldg(a.w + static_cast<long long>(d) * K + i);
    const float b0 = a.bias ? __ldg(a.bias + d) : 0.f;
    float halo0[H > 0 ? H : 1];      // inputs before the span (lane 0 only)
#pragma unroll
    for (int j = 0; j < H; ++j) halo0[j] = 0.f;
    if (lane == 0) {
        if (v0 > 0) {
#pragma unroll
            for (int j = 0; j < H; ++j) halo0[j] = to_f32<Tin>(xr[v0 * V - H + j]);
        } else if (a.hist) {
#pragma unroll
            for (int j = 0; j < H; ++j) halo0[j] = __ldg(a.hist + row * H + j);
        }
    }
    float tail[H > 0 ? H : 1];       // the last H inputs of this lane's previous vector
#pragma unroll
    for (int j = 0; j < H; ++j) tail[j] = 0.f;
#pragma unroll
    for (int k = 0; k < U; ++k) {
        const long long p = v0 + 32 * k + lane;
        float xe[H + V];             // xe[0..H) the inputs before the vector, then the vector
        Vec16<Tin>::unpack(raw[k], xe + H);
#pragma unroll
        for (int j = 0; j < H; ++j) {
            const float up = __shfl_up_sync(0xffffffffu, xe[V + j], 1);
            const float wrap = __shfl_sync(0xffffffffu, tail[j], 31);
            xe[j] = lane > 0 ? up : (k > 0 ? wrap : halo0[j]);
            tail[j] = xe[V + j];
        }
        if (p < nvr) {
            float o[V];
#pragma unroll
            for (int t = 0; t < V; t += 2) {  // outputs in pairs, the gate on packed FP32
                float2 acc = f2(b0, b0);
#pragma unroll
                for (int i = 0; i < K; ++i) {
                    acc.x = fmaf(w[i], xe[t + i], acc.x);
                    acc.y = fmaf(w[i], xe[t + 1 + i], acc.y);
                }
                if (a.silu) acc = silu_pair(acc);
                o[t] = acc.x;
                o[t + 1] = acc.y;
            }
            store_run<V>(ur + p * V, o);
            if (a.hist_out && p == nvr - 1) {   // the row's last vector: the window to continue from
#pragma unroll
                for (int j = 0; j < H; ++j) a.hist_out[row * H + j] = xe[V + j];
            }
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
