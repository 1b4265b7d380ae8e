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

// One token on a quad of 4 states of one channel, as packed FP32 pairs (0,1), (2,3):
// h_n <- 2^(Delta A2_n) h_n + (Delta x) B_n with A2 = A log2(e), and the quad's share of
// the readout, (C_0 h_0 + C_2 h_2) + (C_1 h_1 + C_3 h_3).  Both decode kernels update and
// read out every quad through this one function, so they agree bit for bit.
__device__ __forceinline__ float quad_step(float (&h)[4], const float (&A2)[4], float dl, float dx,
                                           const float (&b)[4], const float (&c)[4]) {
    const float2 dl2 = f2(dl, dl), dx2 = f2(dx, dx);
    float2 acc = f2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float2 a = ex2_pair(fmul2(dl2, f2(A2[2 * k], A2[2 * k + 1])));
        const float2 hk = ffma2(a, f2(h[2 * k], h[2 * k + 1]), fmul2(dx2, f2(b[2 * k], b[2 * k + 1])));
        h[2 * k] = hk.x; h[2 * k + 1] = hk.y;
        acc = ffma2(f2(c[2 * k], c[2 * k + 1]), hk, acc);
    }
    return acc.x + acc.y;
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
    float h[J][4], a4[J][4], bb[J][4], cc[J][4], dl[J], xv[J], zv[J], Dv[J];   // a4: A log2(e)
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
                a4[j][0] = av.x * kLog2e; a4[j][1] = av.y * kLog2e;
                a4[j][2] = av.z * kLog2e; a4[j][3] = av.w * kLog2e;
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
                a4[j][s] = ok ? Ap[s] * kLog2e : 0.f;
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
        float acc = quad_step(h[j], a4[j], dl[j], dl[j] * xv[j], bb[j], cc[j]);
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

// Several decode tokens per call (ssm_state_step_multi: speculative or chunked decoding),
// one channel per thread with all of its states in registers: the state is read once,
// carried through the ntok tokens in registers and written once, so the state traffic is
// that of one step whatever ntok is.
//
// A block holds kStepThreads consecutive channels and walks the sequences b = slice,
// slice + slices, ... (blockIdx.x = slice * dblocks + channel block), so A and D stay in
// registers for all of them, and while the current sequence is computed the next one's
// state row streams into a shared ring (cp.async) and its first tokens into registers, so
// loads stay in flight through the whole kernel instead of only at its start.  Per round of up to kStepsRound tokens the
// block stages the sequence's B and C rows in shared memory (padded to NP with zeros),
// read back as 16-byte broadcasts.
//
// Per token the arithmetic is the one-token kernel's, in the same order: each quad of 4
// states is updated and read out as one thread of state_step_kernel does, and the quad
// shares are summed in the order the xor-butterfly over the G lanes of a channel gives
// lane 0.  ntok chained one-token calls therefore give bit-identical states and outputs.
constexpr int kStepThreads = 128;
constexpr int kStepsRound = 4;

// The readout of a channel from its G = NP / 4 quad shares, in the xor-butterfly order
// (offsets G/2, ..., 1) as seen by lane 0.
template <int G> __device__ __forceinline__ float quad_sum(const float (&s)[G]) {
    if constexpr (G == 1) return s[0];
    else if constexpr (G == 2) return s[0] + s[1];
    else return (s[0] + s[2]) + (s[1] + s[3]);
}

#ifndef SSM_STEPS_MINB
#define SSM_STEPS_MINB 5     // resident blocks per SM the registers target
#endif
template <int NP, typename Tin, typename Tout, bool VEC4>
__global__ void __launch_bounds__(kStepThreads, SSM_STEPS_MINB) state_steps_kernel(const StepArgs p, int dblocks) {
    constexpr int G = NP / 4, R = kStepsRound;
    static_assert(2 * R * NP <= kStepThreads, "one thread per staged B/C value");
    __shared__ __align__(16) float sbc[2][R][NP];
    const int cb = int(blockIdx.x % unsigned(dblocks));
    const int slice = int(blockIdx.x / unsigned(dblocks));
    const int slices = int(gridDim.x / unsigned(dblocks));
    const int d = cb * kStepThreads + int(threadIdx.x);
    const bool act = d < p.dim;
    const int N = p.dstate, ntok = p.ntok;
    const size_t chans = size_t(p.batch) * p.dim;
    const Tin *gx = static_cast<const Tin *>(p.x);
    const Tin *gd = static_cast<const Tin *>(p.delta);
    const Tin *gz = static_cast<const Tin *>(p.z);
    const Tin *gB = static_cast<const Tin *>(p.B);
    const Tin *gC = static_cast<const Tin *>(p.C);
    Tout *gy = static_cast<Tout *>(p.y);

    // A log2(e) (and D) of this channel, for every sequence of the block
    const float *As = p.A + size_t(act ? d : 0) * N;
    float a[G][4];
    if constexpr (VEC4) {
#pragma unroll
        for (int q = 0; q < G; ++q) {
            float4 av = make_float4(0.f, 0.f, 0.f, 0.f);
            if (act && 4 * q < N) av = __ldg(reinterpret_cast<const float4 *>(As + 4 * q));
            a[q][0] = av.x * kLog2e; a[q][1] = av.y * kLog2e; a[q][2] = av.z * kLog2e; a[q][3] = av.w * kLog2e;
        }
    } else {
#pragma unroll
        for (int n = 0; n < NP; ++n) a[n / 4][n % 4] = (act && n < N) ? As[n] * kLog2e : 0.f;
    }
    const float Dv = (p.D != nullptr && act) ? p.D[d] : 0.f;

    auto state_row = [&](int b) { return p.state + (size_t(b) * p.dim + (act ? d : 0)) * N; };
    auto load_state = [&](int b, float (&hv)[G][4]) {
        const float *hs = state_row(b);
        if constexpr (VEC4) {
#pragma unroll
            for (int q = 0; q < G; ++q) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (act && 4 * q < N) v = *reinterpret_cast<const float4 *>(hs + 4 * q);
                hv[q][0] = v.x; hv[q][1] = v.y; hv[q][2] = v.z; hv[q][3] = v.w;
            }
        } else {
#pragma unroll
            for (int n = 0; n < NP; ++n) hv[n / 4][n % 4] = (act && n < N) ? hs[n] : 0.f;
        }
    };
    // the round's token inputs of sequence b (raw, converted when used)
    auto load_tokens = [&](int b, int t0, Tin (&xr)[R], Tin (&dr)[R], Tin (&zr)[R]) {
        const size_t ch = size_t(b) * p.dim + (act ? d : 0);
#pragma unroll
        for (int tt = 0; tt < R; ++tt) {
            const bool ok = act && t0 + tt < ntok;
            const size_t idx = size_t(t0 + tt) * chans + ch;
            xr[tt] = ok ? gx[idx] : Tin(0.f);
            dr[tt] = ok ? gd[idx] : Tin(0.f);
            zr[tt] = (ok && gz != nullptr) ? gz[idx] : Tin(0.f);
        }
    };
    // this thread's staged B/C value of the round (threads 0 .. 2 R NP - 1)
    auto load_bc = [&](int b, int t0) {
        const int i = threadIdx.x;
        const int which = i / (R * NP);
        const int tt = (i / NP) % R, n = i % NP;
        float v = 0.f;
        if (i < 2 * R * NP && t0 + tt < ntok && n < N)
            v = to_f32((which ? gC : gB)[(size_t(t0 + tt) * p.batch + b) * N + n]);
        return v;
    };

    // whole quads (N % 4 == 0): the next sequence's state row goes into a 2-slot shared
    // ring with cp.async, each thread copying and reading back only its own row, so the
    // prefetch holds no registers (5 blocks per SM fit); otherwise into registers
    constexpr bool RING = VEC4;
    constexpr int RPL = 8 / G;
    __shared__ __align__(16) float4 sring[RING ? 2 : 1][kStepThreads * G];
    const int tid = int(threadIdx.x);
    auto slot = [&](int q) { return tid * G + (q ^ ((tid / RPL) & (G - 1))); };
    auto ring_issue = [&](long long bq, int st) {
        if constexpr (RING) {
            if (act && bq < p.batch) {
                const float *hs = state_row(int(bq));
#pragma unroll
                for (int q = 0; q < G; ++q)
                    if (4 * q < N) cp_async_16(&sring[st][slot(q)], hs + 4 * q);
            }
            cp_async_commit();
        }
    };

    // the first sequence's state and first round, then one sequence ahead
    float hn[RING ? 1 : G][4];
    Tin xn[R], dn[R], zn[R];
    float bcn = 0.f;
    ring_issue(slice, 0);
    if (slice < p.batch) {
        if constexpr (!RING) load_state(slice, *reinterpret_cast<float (*)[G][4]>(&hn[0][0]));
        load_tokens(slice, 0, xn, dn, zn);
        bcn = load_bc(slice, 0);
    }
    int it = 0;
    for (int b = slice; b < p.batch; b += slices, ++it) {
        float h[G][4];
        if constexpr (RING) {
            ring_issue((long long)b + slices, (it + 1) & 1);
            cp_async_wait<1>();                          // this sequence's row has landed
#pragma unroll
            for (int q = 0; q < G; ++q) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (act && 4 * q < N) v = sring[it & 1][slot(q)];
                h[q][0] = v.x; h[q][1] = v.y; h[q][2] = v.z; h[q][3] = v.w;
            }
        } else {
            const float (&hp)[G][4] = *reinterpret_cast<const float (*)[G][4]>(&hn[0][0]);
#pragma unroll
            for (int n = 0; n < NP; ++n) h[n / 4][n % 4] = hp[n / 4][n % 4];
        }
        Tin xq[R], dq[R], zq[R];
#pragma unroll
        for (int tt = 0; tt < R; ++tt) { xq[tt] = xn[tt]; dq[tt] = dn[tt]; zq[tt] = zn[tt]; }
        float bcv = bcn;
        if ((long long)b + slices < p.batch) {
            if constexpr (!RING) load_state(b + slices, *reinterpret_cast<float (*)[G][4]>(&hn[0][0]));
            load_tokens(b + slices, 0, xn, dn, zn);
            bcn = load_bc(b + slices, 0);
        }
        const size_t ch = size_t(b) * p.dim + (act ? d : 0);
        for (int t0 = 0; t0 < ntok; t0 += R) {
            const int nt = min(R, ntok - t0);
            if (t0 > 0) {
                load_tokens(b, t0, xq, dq, zq);
                bcv = load_bc(b, t0);
            }
            __syncthreads();                      // the previous round's reads are done
            if (threadIdx.x < 2 * R * NP) (&sbc[0][0][0])[threadIdx.x] = bcv;
            __syncthreads();
#pragma unroll
            for (int tt = 0; tt < R; ++tt) {
                if (tt >= nt) break;
                const float dl = to_f32(dq[tt]), xv = to_f32(xq[tt]);
                const float dx = dl * xv;
                float sq[G];
#pragma unroll
                for (int q = 0; q < G; ++q) {
                    const float4 bq = *reinterpret_cast<const float4 *>(&sbc[0][tt][4 * q]);
                    const float4 cq = *reinterpret_cast<const float4 *>(&sbc[1][tt][4 * q]);
                    const float bb[4] = {bq.x, bq.y, bq.z, bq.w};
                    const float cc[4] = {cq.x, cq.y, cq.z, cq.w};
                    sq[q] = quad_step(h[q], a[q], dl, dx, bb, cc);
                }
                float yv = fmaf(Dv, xv, quad_sum<G>(sq));
                if (gz != nullptr) yv *= silu_f(to_f32(zq[tt]));
                if (act) gy[size_t(t0 + tt) * chans + ch] = from_f32<Tout>(yv);
            }
        }
        float *hs = state_row(b);
        if constexpr (VEC4) {
#pragma unroll
            for (int q = 0; q < G; ++q)
                if (act && 4 * q < N)
                    *reinterpret_cast<float4 *>(hs + 4 * q) = make_float4(h[q][0], h[q][1], h[q][2], h[q][3]);
        } else {
#pragma unroll
            for (int n = 0; n < NP; ++n)
                if (act && n < N) hs[n] = h[n / 4][n % 4];
        }
    }
    if constexpr (RING) cp_async_wait<0>();
}

}  // namespace ssm
