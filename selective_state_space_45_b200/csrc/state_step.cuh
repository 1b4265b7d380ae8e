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
    int ntok;             // tokens per call (state_steps_kernel): x, delta, z, y are
                          // [ntok][batch][dim], B, C [ntok][batch][dstate]
};

// 4 consecutive input values (8 or 16 bytes, aligned) as fp32.
template <typename T> __device__ __forceinline__ void load4_nc(const T *src, float (&v)[4]);
template <> __device__ __forceinline__ void load4_nc<float>(const float *src, float (&v)[4]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(src));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <> __device__ __forceinline__ void load4_nc<__nv_bfloat16>(const __nv_bfloat16 *src, float (&v)[4]) {
    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(src));
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xffff0000u);
}

// One thread = J channel-quads (4 states each).  Quad j of a thread is global quad
// gq = (blockIdx.x * J + j) * blockDim.x + threadIdx.x, so each of the J accesses of a
// warp covers 32 consecutive quads (512 contiguous bytes of state at N = 16).  Every load
// of all J quads is issued before the first store (the state is written in place, so a
// store could otherwise hold back the next quad's loads), keeping J * 16 bytes of state
// in flight per thread.
template <int NP, typename Tin, typename Tout, bool VEC4, int J>
__global__ void __launch_bounds__(256) state_step_kernel(const StepArgs p) {
    constexpr int G = NP / 4;
    const long long nquad = (long long)p.batch * p.dim * G;
    const int N = p.dstate;
    long long chs[J];
    int rs[J], ds[J];
    bool act[J];
    float h[J][4], a4[J][4], bb[J][4], cc[J][4], dl[J], xv[J], zv[J], Dv[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const long long g = ((long long)blockIdx.x * J + j) * blockDim.x + threadIdx.x;
        act[j] = g < nquad;
        const long long q = act[j] ? g : 0;          // inactive lanes still join the shuffles
        const long long ch = q / G;
        const int r = int(q - ch * G);
        const int b = int(ch / p.dim);
        const int d = int(ch - (long long)b * p.dim);
        chs[j] = ch; rs[j] = r; ds[j] = d;
        const int n0 = 4 * r;
        const float *hp = p.state + (size_t)ch * N + n0;
        const float *Ap = p.A + (size_t)d * N + n0;
        const Tin *Bb = static_cast<const Tin *>(p.B) + (size_t)b * N + n0;
        const Tin *Cb = static_cast<const Tin *>(p.C) + (size_t)b * N + n0;
        if constexpr (VEC4) {   // N % 4 == 0: whole 16-byte quads
            if (act[j] && n0 < N) {
                const float4 hv = *reinterpret_cast<const float4 *>(hp);
                const float4 av = __ldg(reinterpret_cast<const float4 *>(Ap));
                h[j][0] = hv.x; h[j][1] = hv.y; h[j][2] = hv.z; h[j][3] = hv.w;
                a4[j][0] = av.x; a4[j][1] = av.y; a4[j][2] = av.z; a4[j][3] = av.w;
                load4_nc<Tin>(Bb, bb[j]);
                load4_nc<Tin>(Cb, cc[j]);
            } else {
#pragma unroll
                for (int s = 0; s < 4; ++s) h[j][s] = a4[j][s] = bb[j][s] = cc[j][s] = 0.f;
            }
        } else {
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const bool ok = act[j] && n0 + s < N;
                h[j][s] = ok ? hp[s] : 0.f;
                a4[j][s] = ok ? Ap[s] : 0.f;
                bb[j][s] = ok ? to_f32(Bb[s]) : 0.f;
                cc[j][s] = ok ? to_f32(Cb[s]) : 0.f;
            }
        }
        dl[j] = to_f32(static_cast<const Tin *>(p.delta)[ch]);
        xv[j] = to_f32(static_cast<const Tin *>(p.x)[ch]);
        zv[j] = p.z != nullptr ? to_f32(static_cast<const Tin *>(p.z)[ch]) : 0.f;
        Dv[j] = p.D != nullptr ? p.D[d] : 0.f;
    }
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const float dx = dl[j] * xv[j];
        float acc = 0.f;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            h[j][s] = fmaf(ex2_approx(dl[j] * a4[j][s] * kLog2e), h[j][s], dx * bb[j][s]);
            acc = fmaf(cc[j][s], h[j][s], acc);
        }
        const int n0 = 4 * rs[j];
        float *hp = p.state + (size_t)chs[j] * N + n0;
        if constexpr (VEC4) {
            if (act[j] && n0 < N)
                *reinterpret_cast<float4 *>(hp) = make_float4(h[j][0], h[j][1], h[j][2], h[j][3]);
        } else {
#pragma unroll
            for (int s = 0; s < 4; ++s)
                if (act[j] && n0 + s < N) hp[s] = h[j][s];
        }
#pragma unroll
        for (int off = G / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (act[j] && rs[j] == 0) {
            float yv = fmaf(Dv[j], xv[j], acc);
            if (p.z != nullptr) yv *= silu_f(zv[j]);
            static_cast<Tout *>(p.y)[chs[j]] = from_f32<Tout>(yv);
        }
    }
}

// Several decode tokens per call (speculative or chunked decoding): the state of a
// channel-quad is loaded once, carried through the ntok tokens in registers and stored
// once, so the state traffic is that of one step whatever ntok is.  The token inputs of a
// round of up to kStepsRound tokens are first staged in shared memory by the whole block,
// every load independent of the others, so no thread waits on one token's loads before
// issuing the next token's.  Per token the arithmetic is the one-step kernel's, in the
// same order: ntok chained one-token calls give bit-identical results.
constexpr int kStepsRound = 8;

// Shared memory of one block of state_steps_kernel: per round token, x, delta, z of the
// block's channels and B, C of the sequences they belong to (nb of them).
__host__ __device__ constexpr size_t steps_smem_bytes(int ch_per_block, int nb, int N) {
    return size_t(kStepsRound) * (3 * size_t(ch_per_block) + 2 * size_t(nb) * N) * sizeof(float);
}

template <int NP, typename Tin, typename Tout, bool VEC4>
__global__ void __launch_bounds__(256) state_steps_kernel(const StepArgs p, int nb_max) {
    constexpr int G = NP / 4;
    constexpr int CPB = 256 / G;                     // channels per block
    extern __shared__ __align__(16) float sm[];
    const long long nquad = (long long)p.batch * p.dim * G;
    const long long chans = (long long)p.batch * p.dim;
    const int N = p.dstate;
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const bool act = g < nquad;
    const long long q = act ? g : 0;          // inactive lanes still join the shuffles
    const long long ch = q / G;
    const int r = int(q - ch * G);
    const int b = int(ch / p.dim);
    const int d = int(ch - (long long)b * p.dim);
    const int n0 = 4 * r;
    // the block's channels ch0 .. ch0+CPB-1 and the sequences b_lo .. they belong to
    const long long ch0 = (long long)blockIdx.x * CPB;
    const int b_lo = int(ch0 / p.dim);
    // this thread's channel within the block and its sequence among the staged ones
    // (0 for the idle threads past the last channel, which read but never use them)
    const int cl = act ? int(ch - ch0) : 0;
    const int bsel = act ? b - b_lo : 0;
    float *sx = sm;                           // [round][CPB]
    float *sd = sx + kStepsRound * CPB;
    float *sz = sd + kStepsRound * CPB;
    float *sb = sz + kStepsRound * CPB;       // [round][nb_max][N]
    float *sc = sb + (size_t)kStepsRound * nb_max * N;

    float *hp = p.state + (size_t)ch * N + n0;
    const float *Ap = p.A + (size_t)d * N + n0;
    float h[4], a4[4];
    if constexpr (VEC4) {
        if (act && n0 < N) {
            const float4 hv = *reinterpret_cast<const float4 *>(hp);
            const float4 av = __ldg(reinterpret_cast<const float4 *>(Ap));
            h[0] = hv.x; h[1] = hv.y; h[2] = hv.z; h[3] = hv.w;
            a4[0] = av.x; a4[1] = av.y; a4[2] = av.z; a4[3] = av.w;
        } else {
#pragma unroll
            for (int s = 0; s < 4; ++s) h[s] = a4[s] = 0.f;
        }
    } else {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const bool ok = act && n0 + s < N;
            h[s] = ok ? hp[s] : 0.f;
            a4[s] = ok ? Ap[s] : 0.f;
        }
    }
    const float Dv = p.D != nullptr ? p.D[d] : 0.f;
    const Tin *gx = static_cast<const Tin *>(p.x);
    const Tin *gd = static_cast<const Tin *>(p.delta);
    const Tin *gz = static_cast<const Tin *>(p.z);
    const Tin *gB = static_cast<const Tin *>(p.B);
    const Tin *gC = static_cast<const Tin *>(p.C);
    for (int t0 = 0; t0 < p.ntok; t0 += kStepsRound) {
        const int nt = min(kStepsRound, p.ntok - t0);
        __syncthreads();                      // the previous round's reads are done
        for (int i = threadIdx.x; i < nt * CPB; i += blockDim.x) {
            const int tt = i / CPB, c = i % CPB;
            const long long cg = ch0 + c;
            const bool ok = cg < chans;
            const size_t idx = (size_t)(t0 + tt) * chans + (ok ? cg : 0);
            sx[tt * CPB + c] = ok ? to_f32(gx[idx]) : 0.f;
            sd[tt * CPB + c] = ok ? to_f32(gd[idx]) : 0.f;
            sz[tt * CPB + c] = (ok && gz != nullptr) ? to_f32(gz[idx]) : 0.f;
        }
        for (int i = threadIdx.x; i < nt * nb_max * N; i += blockDim.x) {
            const int tt = i / (nb_max * N), rem = i % (nb_max * N);
            const int bb = b_lo + rem / N, n = rem % N;
            const bool ok = bb < p.batch;
            const size_t idx = ((size_t)(t0 + tt) * p.batch + (ok ? bb : 0)) * N + n;
            sb[(size_t)tt * nb_max * N + rem] = ok ? to_f32(gB[idx]) : 0.f;
            sc[(size_t)tt * nb_max * N + rem] = ok ? to_f32(gC[idx]) : 0.f;
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const float dl = sd[tt * CPB + cl];
            const float xv = sx[tt * CPB + cl];
            const float zv = sz[tt * CPB + cl];
            const float *bq = sb + ((size_t)tt * nb_max + bsel) * N + n0;
            const float *cq = sc + ((size_t)tt * nb_max + bsel) * N + n0;
            float bb[4], cc[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const bool ok = act && n0 + s < N;
                bb[s] = ok ? bq[s] : 0.f;
                cc[s] = ok ? cq[s] : 0.f;
            }
            const float dx = dl * xv;
            float acc = 0.f;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                h[s] = fmaf(ex2_approx(dl * a4[s] * kLog2e), h[s], dx * bb[s]);
                acc = fmaf(cc[s], h[s], acc);
            }
#pragma unroll
            for (int off = G / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (act && r == 0) {
                float yv = fmaf(Dv, xv, acc);
                if (p.z != nullptr) yv *= silu_f(zv);
                static_cast<Tout *>(p.y)[(size_t)(t0 + tt) * chans + ch] = from_f32<Tout>(yv);
            }
        }
    }
    if constexpr (VEC4) {
        if (act && n0 < N) *reinterpret_cast<float4 *>(hp) = make_float4(h[0], h[1], h[2], h[3]);
    } else {
#pragma unroll
        for (int s = 0; s < 4; ++s)
            if (act && n0 + s < N) hp[s] = h[s];
    }
}

}  // namespace ssm
