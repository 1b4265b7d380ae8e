// state_step.cuh -- one decode token of the selective SSM, state updated in place.
//
// Per sequence b and channel d with the fp32 state h[b,d,0..N):
//   h_n <- exp(Delta * A[d,n]) h_n + Delta * B[b,n] * x,   y = (C[b,:] . h + D[d] x) SiLU(z)
// Source: "Beyond attention with Mamba, state space models and hybrids" (xmarva lesson 10),
// section 7 "Generation with a state of fixed size" (the recurrence for one position on a
// carried state); the step Delta arrives already positive.
//
// The step is bound by HBM: the fp32 state is read and written once (128 B per channel at
// N = 16) against a few bytes of token inputs.  G = NP / 4 consecutive lanes share a
// channel, each moving 16 contiguous bytes of its state, so one warp streams 8 whole
// channels (512 contiguous bytes) per access at N = 16.
#pragma once

#include "common.cuh"

namespace ssm {

struct StepArgs {
    float *state;
    const void *x;
    const void *delta;
    const float *A;
    const void *B;
    const void *C;
    const float *D;
    const void *z;
    void *y;
    int batch, dim, dstate;
};

template <int NP, typename Tin, typename Tout, bool VEC4>
__global__ void __launch_bounds__(256) state_step_kernel(const StepArgs p) {
    constexpr int G = NP / 4;
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long nchan = (long long)p.batch * p.dim;
    const long long chl = gid / G;
    const int r = int(gid - chl * G);
    const bool active = chl < nchan;
    const long long ch = active ? chl : 0;   // inactive lanes still join the shuffles
    const int N = p.dstate;
    const int b = int(ch / p.dim);
    const int d = int(ch - (long long)b * p.dim);

    const float dl = to_f32(static_cast<const Tin *>(p.delta)[ch]);
    const float xv = to_f32(static_cast<const Tin *>(p.x)[ch]);
    const float dx = dl * xv;
    const Tin *Bb = static_cast<const Tin *>(p.B) + (size_t)b * N;
    const Tin *Cb = static_cast<const Tin *>(p.C) + (size_t)b * N;
    float *hp = p.state + (size_t)ch * N;
    const float *Ap = p.A + (size_t)d * N;
    const int n0 = 4 * r;

    float h[4], a4[4], bb[4], cc[4];
    if constexpr (VEC4) {   // N % 4 == 0: whole 16-byte quads
        const bool q = active && n0 < N;
        float4 hv = q ? *reinterpret_cast<const float4 *>(hp + n0) : make_float4(0.f, 0.f, 0.f, 0.f);
        float4 av = q ? __ldg(reinterpret_cast<const float4 *>(Ap + n0)) : make_float4(0.f, 0.f, 0.f, 0.f);
        h[0] = hv.x; h[1] = hv.y; h[2] = hv.z; h[3] = hv.w;
        a4[0] = av.x; a4[1] = av.y; a4[2] = av.z; a4[3] = av.w;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            bb[s] = q ? to_f32(Bb[n0 + s]) : 0.f;
            cc[s] = q ? to_f32(Cb[n0 + s]) : 0.f;
        }
    } else {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const bool q = active && n0 + s < N;
            h[s] = q ? hp[n0 + s] : 0.f;
            a4[s] = q ? Ap[n0 + s] : 0.f;
            bb[s] = q ? to_f32(Bb[n0 + s]) : 0.f;
            cc[s] = q ? to_f32(Cb[n0 + s]) : 0.f;
        }
    }

    float acc = 0.f;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        h[s] = fmaf(ex2_approx(dl * a4[s] * kLog2e), h[s], dx * bb[s]);
        acc = fmaf(cc[s], h[s], acc);
    }

    if constexpr (VEC4) {
        if (active && n0 < N)
            *reinterpret_cast<float4 *>(hp + n0) = make_float4(h[0], h[1], h[2], h[3]);
    } else {
#pragma unroll
        for (int s = 0; s < 4; ++s)
            if (active && n0 + s < N) hp[n0 + s] = h[s];
    }

#pragma unroll
    for (int off = G / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);

    if (active && r == 0) {
        float yv = fmaf(p.D != nullptr ? p.D[d] : 0.f, xv, acc);
        if (p.z != nullptr) yv *= silu_f(to_f32(static_cast<const Tin *>(p.z)[ch]));
        static_cast<Tout *>(p.y)[ch] = from_f32<Tout>(yv);
    }
}

}  // namespace ssm
