// scan_bwd.cuh -- backward of the selective scan (S6, Euler gain) for sm_100a.
//
// Gradients of  loss = sum dy * y + sum dfinal * h_last  with respect to x, delta, z, A,
// B, C, D, delta_bias and the start state, by reverse-mode differentiation of the
// recurrence (forward: scan_fwd.cuh).  With mu the adjoint flowing into h_t from later
// tokens, going t = L-1 .. 0:
//     dypre_t  = dy_t * SiLU(z_t);   dz_t = dy_t * ypre_t * SiLU'(z_t)
//     lambda_n = dypre_t C_t[n] + mu_n                      (adjoint of h_t[n])
//     dC_t[n] += dypre_t h_t[n];     dB_t[n] += lambda_n Delta_t x_t
//     dx_t     = dypre_t D + sum_n lambda_n Delta_t B_t[n]
//     dDelta_t = sum_n lambda_n (B_t[n] x_t + h_{t-1}[n] Abar_t[n] A[n])
//     dA[n]   += lambda_n h_{t-1}[n] Abar_t[n] Delta_t;     mu_n = Abar_t[n] lambda_n
// and ddelta_t = dDelta_t * sigmoid(delta_t + bias) under softplus.
// Source: the states are recomputed in the backward pass rather than stored, as Mamba's own
// kernel does ("Beyond attention with Mamba, state space models and hybrids", xmarva
// lesson 10, section 6); the recurrence is the one of sections 3-4 of that lesson.
//
// Layout of the work (one CTA = 32 channels x 16 states of one sequence, 4 warps, one
// channel per lane and one state quad per warp, as in the forward kernel):
//   phase F   the forward recurrence over the whole sequence, keeping only the state
//             before every 4th token (a global scratch array);
//   phase R   16-token tiles in reverse.  Per tile: per (t, d) the step Delta and
//             dypre = dy * SiLU(z); then sub-chunks of 4 tokens, last first: the states
//             of the sub-chunk recomputed from its checkpoint (with the readout, for dz),
//             then walked backwards carrying mu; the dB / dC terms of the 32 channels are
//             summed through a per-warp shared transpose and written as per-CTA partial
//             sums; finally per (t, d) the quads' dx, dDelta and readout partials summed,
//             the softplus slope and dz, 16-byte row stores.
//   Partial sums over channel groups (dB, dC) and over sequences (dA, dD, dbias) are
//   added up by reduce_partials_kernel in a fixed order: the gradients are deterministic.
#pragma once

#include "common.cuh"

// Build-time tuning: independent partial sums in the column reduction of the dB / dC
// transpose, and how many 4-token sub-chunks the reverse loop unrolls.
#ifndef SSM_BWD_COLSUM_ACC
#define SSM_BWD_COLSUM_ACC 4
#endif
#ifndef SSM_BWD_UNROLL_J
#define SSM_BWD_UNROLL_J 1
#endif

namespace ssm {

constexpr int kBwdUnrollJ = SSM_BWD_UNROLL_J;

// sigmoid(v) = 1 / (1 + e^-v) with the SFU exponential and reciprocal (0 for v -> -inf).
__device__ __forceinline__ float sigmoid_f(float v) {
    return rcp_approx(1.f + ex2_approx(-v * kLog2e));
}

struct BwdArgs {
    const void *x;
    const void *delta;
    const float *delta_bias;
    const float *A;
    const void *B;
    const void *C;
    const float *D;
    const void *z;
    const float *h0;      // [batch][dim][dstate] or null (zero start)
    const void *dy;       // [batch][dim][L], gradient dtype
    const float *dfinal;  // [batch][dim][dstate] or null
    void *dx;
    void *ddelta;
    void *dz;             // written when given (z must be given too)
    float *dh0;           // [batch][dim][dstate] or null
    float *ck;            // [ctas][ntiles*T/4][4][32] float4: state before every 4th token
    float *part_bc;       // [2][ctas][L][16]: per-CTA channel sums of the dB and dC terms
    float *part_a;        // [batch][dim][16]: per-sequence dA
    float *part_dd;       // [2][batch][dim]: per-sequence dD and ddelta_bias
    int batch, dim, seqlen, dstate;
    int softplus;
    int groups_per_seq;
    int ntiles;
};

template <typename Tin_, typename Tg_, bool VEC_>
struct BwdCfg {
    using Tin = Tin_;
    using Tg = Tg_;
    static constexpr int NP = 16, Q = 4, CH = 32, T = 16, NSTAGE = 2, NT = 128;
    static constexpr bool VEC = VEC_;
    static constexpr int EIN = 16 / sizeof(Tin);
    static constexpr int EG = 16 / sizeof(Tg);
    static constexpr int RAW_ROW = T + EIN;     // staged rows: 16 B past a multiple of 16 B
    static constexpr int G_ROW = T + EG;
    static constexpr int P_ROW = T + 4;         // per-quad partial rows (floats)
    static constexpr int X_ROW = 36;            // transpose rows: conflict-free both ways
    static constexpr bool BCPACK = sizeof(Tin) == 2;   // B, C staged as bf16 quads
    static_assert(!BCPACK || T * Q <= NT, "one thread per packed (token, quad)");
    static constexpr int TW = 4;                // tokens per (t, d) task
    static constexpr int NTW = T / TW;          // task chunks per row
    static constexpr int NTASK = CH * NTW;      // (channel, token chunk) tasks per tile
    static_assert(NTASK <= NT, "at most one task per thread");

    static constexpr size_t al(size_t v) { return (v + 15) & ~size_t(15); }
    static constexpr size_t RAW_ARR = al(size_t(CH) * RAW_ROW * sizeof(Tin));
    static constexpr size_t G_ARR = al(size_t(CH) * G_ROW * sizeof(Tg));
    static constexpr size_t RAW_BC = al(size_t(T) * NP * sizeof(Tin));
    static constexpr size_t STAGE_BYTES = 3 * RAW_ARR + G_ARR + 2 * RAW_BC;
    static constexpr size_t OFF_RAW = 0;
    static constexpr size_t OFF_PREP = OFF_RAW + NSTAGE * STAGE_BYTES;   // float4 [T][CH]
    static constexpr size_t OFF_BF = OFF_PREP + al(size_t(T) * CH * sizeof(float4));
    static constexpr size_t OFF_CF = OFF_BF + al(size_t(T) * NP * sizeof(float));
    static constexpr size_t PART_ARR = al(size_t(Q) * CH * P_ROW * sizeof(float));
    static constexpr size_t OFF_PART = OFF_CF + al(size_t(T) * NP * sizeof(float));
    static constexpr size_t OFF_XP = OFF_PART + 3 * PART_ARR;
    static constexpr size_t SMEM_BYTES = OFF_XP + al(size_t(Q) * 32 * X_ROW * sizeof(float));
    // the staged dx / ddelta / dz rows reuse the partial arrays once they are summed
    static_assert(3 * CH * G_ROW * sizeof(Tg) <= 3 * PART_ARR, "output staging must fit");
};

// Views of one ring stage: x, delta, z rows [CH][RAW_ROW], dy rows [CH][G_ROW], B, C [T][N].
template <class Cfg> struct BwdStage {
    typename Cfg::Tin *xs, *ds, *zs, *bs, *cs;
    typename Cfg::Tg *gs;
    __device__ __forceinline__ BwdStage(unsigned char *smem, int s) {
        unsigned char *base = smem + Cfg::OFF_RAW + size_t(s) * Cfg::STAGE_BYTES;
        xs = reinterpret_cast<typename Cfg::Tin *>(base);
        ds = reinterpret_cast<typename Cfg::Tin *>(base + Cfg::RAW_ARR);
        zs = reinterpret_cast<typename Cfg::Tin *>(base + 2 * Cfg::RAW_ARR);
        gs = reinterpret_cast<typename Cfg::Tg *>(base + 3 * Cfg::RAW_ARR);
        bs = reinterpret_cast<typename Cfg::Tin *>(base + 3 * Cfg::RAW_ARR + Cfg::G_ARR);
        cs = reinterpret_cast<typename Cfg::Tin *>(base + 3 * Cfg::RAW_ARR + Cfg::G_ARR + Cfg::RAW_BC);
    }
};

// Stage tile [t0, t0 + T): x, delta and B always; z, dy and C when `full` (phase R).
// VEC: 16-byte cp.async chunks, each wholly inside or outside [0, L) (L is a multiple of
// both chunk widths); else guarded scalar copies.
template <class Cfg>
__device__ __forceinline__ void bwd_load_tile(const BwdArgs &p, unsigned char *smem, int st, int t0,
                                              size_t row0, size_t bc0, int nch, bool full) {
    using Tin = typename Cfg::Tin;
    using Tg = typename Cfg::Tg;
    constexpr int CH = Cfg::CH, T = Cfg::T, NT = Cfg::NT, EIN = Cfg::EIN, EG = Cfg::EG, NP = Cfg::NP;
    BwdStage<Cfg> s(smem, st);
    const int L = p.seqlen, N = p.dstate;
    const Tin *gx = static_cast<const Tin *>(p.x) + row0;
    const Tin *gd = static_cast<const Tin *>(p.delta) + row0;
    const Tin *gz = p.z ? static_cast<const Tin *>(p.z) + row0 : gx;
    const Tg *gg = static_cast<const Tg *>(p.dy) + row0;
    const int narr = full ? (p.z ? 3 : 2) : 2;
    const int nbc = full ? 2 : 1;
    const Tin *gb = static_cast<const Tin *>(p.B) + bc0 + size_t(t0) * N;
    const Tin *gc = static_cast<const Tin *>(p.C) + bc0 + size_t(t0) * N;
    if constexpr (Cfg::VEC) {
        constexpr int CPR = T / EIN;
        constexpr int ROWC = 3 * CH * CPR;
#pragma unroll
        for (int k = 0; k < (ROWC + NT - 1) / NT; ++k) {
            const int i = tid_x() + k * NT;
            const int a = i / (CH * CPR);
            const int rem = i % (CH * CPR);
            const int cc = rem / CPR, qq = rem % CPR;
            if (i < ROWC && a < narr && cc < nch && t0 + qq * EIN < L) {
                const Tin *src = (a == 0 ? gx : a == 1 ? gd : gz) + size_t(cc) * L + t0 + qq * EIN;
                Tin *dst = (a == 0 ? s.xs : a == 1 ? s.ds : s.zs) + cc * Cfg::RAW_ROW + qq * EIN;
                cp_async_16(dst, src);
            }
        }
        if (full) {
            constexpr int CPRG = T / EG;
#pragma unroll
            for (int k = 0; k < (CH * CPRG + NT - 1) / NT; ++k) {
                const int i = tid_x() + k * NT;
                const int cc = i / CPRG, qq = i % CPRG;
                if (i < CH * CPRG && cc < nch && t0 + qq * EG < L)
                    cp_async_16(s.gs + cc * Cfg::G_ROW + qq * EG, gg + size_t(cc) * L + t0 + qq * EG);
            }
        }
        if (N == NP) {
            constexpr int BCC = T * NP / EIN;
#pragma unroll
            for (int k = 0; k < (2 * BCC + NT - 1) / NT; ++k) {
                const int i = tid_x() + k * NT;
                const int which = i / BCC, qq = i % BCC;
                if (i < 2 * BCC && which < nbc && t0 + (qq * EIN) / NP < L)
                    cp_async_16((which ? s.cs : s.bs) + qq * EIN, (which ? gc : gb) + qq * EIN);
            }
        } else {
            const int valid_t = min(T, L - t0);
            const int bc_chunks = (valid_t * N * int(sizeof(Tin))) / 16;
            for (int i = tid_x(); i < nbc * bc_chunks; i += NT) {
                const int which = i >= bc_chunks;
                const int qq = i - which * bc_chunks;
                cp_async_16((which ? s.cs : s.bs) + qq * EIN, (which ? gc : gb) + qq * EIN);
            }
        }
    } else {
        constexpr int NEL = 3 * CH * T;
#pragma unroll 4
        for (int k = 0; k < (NEL + NT - 1) / NT; ++k) {
            const int i = tid_x() + k * NT;
            const int a = i / (CH * T);
            const int rem = i % (CH * T);
            const int cc = rem / T, tt = rem % T;
            if (i < NEL && a < narr && cc < nch && t0 + tt < L) {
                const Tin *src = (a == 0 ? gx : a == 1 ? gd : gz) + size_t(cc) * L + t0 + tt;
                Tin *dst = (a == 0 ? s.xs : a == 1 ? s.ds : s.zs) + cc * Cfg::RAW_ROW + tt;
                *dst = *src;
            }
        }
        if (full) {
            for (int i = tid_x(); i < CH * T; i += NT) {
                const int cc = i / T, tt = i % T;
                if (cc < nch && t0 + tt < L) s.gs[cc * Cfg::G_ROW + tt] = gg[size_t(cc) * L + t0 + tt];
            }
        }
        const int nel = min(T, L - t0) * N;
        for (int i = tid_x(); i < nbc * nel; i += NT) {
            const int which = i >= nel;
            const int qq = i - which * nel;
            (which ? s.cs : s.bs)[qq] = (which ? gc : gb)[qq];
        }
    }
}


// Per-(t, d) task of this thread: channel cc, tokens TW*tk .. TW*tk+TW-1 of the tile.  Writes
// prep[t][cc] = (Delta_t, x_t, dypre_t, 0) with dypre = dy * SiLU(z) (dy alone without a
// gate) when `full`, else (Delta_t, x_t, 0, 0).  Tokens past L and channels past dim become
// no-op tokens (Delta = 0, x = 0, dypre = 0: the state passes through, no gradient arises).
template <class Cfg>
__device__ __forceinline__ void bwd_prep(const BwdArgs &p, const BwdStage<Cfg> &sv, float4 *prep,
                                         int cc, int tk, bool cvalid, float bias, int t0, bool full) {
    using Tin = typename Cfg::Tin;
    using Tg = typename Cfg::Tg;
    constexpr int CH = Cfg::CH;
    constexpr int TW = Cfg::TW;
    float dr[TW], xr[TW], gr[TW], zr[TW];
    loadn<TW, Tin>(sv.ds + cc * Cfg::RAW_ROW + TW * tk, dr);
    loadn<TW, Tin>(sv.xs + cc * Cfg::RAW_ROW + TW * tk, xr);
    if (full) {
        loadn<TW, Tg>(sv.gs + cc * Cfg::G_ROW + TW * tk, gr);
        if (p.z != nullptr) loadn<TW, Tin>(sv.zs + cc * Cfg::RAW_ROW + TW * tk, zr);
    }
#pragma unroll
    for (int u = 0; u < TW; ++u) {
        float dl = dr[u] + bias;
        if (p.softplus) dl = softplus_f(dl);
        const bool ok = cvalid && t0 + TW * tk + u < p.seqlen;
        float dyp = 0.f;
        if (full) dyp = p.z != nullptr ? gr[u] * (zr[u] * sigmoid_f(zr[u])) : gr[u];
        prep[(TW * tk + u) * CH + cc] = make_float4(ok ? dl : 0.f, ok ? xr[u] : 0.f, ok ? dyp : 0.f, 0.f);
    }
}

// B (and C when `both`) of the tile, zero past dstate and past L: for bf16 inputs as bf16
// quads (8 bytes per (token, state quad): the recurrence reads them as 8-byte broadcasts,
// half the shared-memory wavefronts of fp32 quads, and widens them in registers), else
// widened to fp32 [T][NP].
template <class Cfg>
__device__ __forceinline__ void bwd_widen_bc(const BwdArgs &p, const BwdStage<Cfg> &sv, float *Bf,
                                             float *Cf, int t0, bool both) {
    constexpr int T = Cfg::T, NP = Cfg::NP, NT = Cfg::NT, Q = Cfg::Q;
    const int L = p.seqlen, N = p.dstate;
    if constexpr (Cfg::BCPACK) {
        const unsigned short *rb = reinterpret_cast<const unsigned short *>(sv.bs);
        const unsigned short *rc = reinterpret_cast<const unsigned short *>(sv.cs);
        const int i = tid_x();
        if (i < T * Q) {
            const int tt = i / Q, qq = i % Q;
            uint2 b2 = make_uint2(0u, 0u), c2 = make_uint2(0u, 0u);
            if (N == NP && t0 + tt < L) {            // dense rows: 8-byte reads
                b2 = *reinterpret_cast<const uint2 *>(rb + tt * NP + 4 * qq);
                if (both) c2 = *reinterpret_cast<const uint2 *>(rc + tt * NP + 4 * qq);
            } else {
                unsigned bw[4], cw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int n = 4 * qq + e;
                    const bool ok = n < N && t0 + tt < L;
                    bw[e] = ok ? rb[tt * N + n] : 0u;
                    cw[e] = (ok && both) ? rc[tt * N + n] : 0u;
                }
                b2 = make_uint2(bw[0] | (bw[1] << 16), bw[2] | (bw[3] << 16));
                c2 = make_uint2(cw[0] | (cw[1] << 16), cw[2] | (cw[3] << 16));
            }
            reinterpret_cast<uint2 *>(Bf)[i] = b2;
            if (both) reinterpret_cast<uint2 *>(Cf)[i] = c2;
        }
    } else {
#pragma unroll
        for (int k = 0; k < (T * NP + NT - 1) / NT; ++k) {
            const int i = tid_x() + k * NT;
            if (i < T * NP) {
                const int tt = i / NP, n = i % NP;
                const bool ok = n < N && t0 + tt < L;
                Bf[i] = ok ? to_f32(sv.bs[tt * N + n]) : 0.f;
                if (both) Cf[i] = ok ? to_f32(sv.cs[tt * N + n]) : 0.f;
            }
        }
    }
}

// The B (or C) quad q of token t from the tile's staging as fp32 pairs (0,1), (2,3).
template <class Cfg>
__device__ __forceinline__ void bwd_quad(const float *Xf, int t, int q, float2 (&v)[2]) {
    if constexpr (Cfg::BCPACK) {
        const uint2 w = reinterpret_cast<const uint2 *>(Xf)[t * Cfg::Q + q];
        v[0] = bf16x2_to_f2(w.x);
        v[1] = bf16x2_to_f2(w.y);
    } else {
        const float4 x4 = *reinterpret_cast<const float4 *>(Xf + t * Cfg::NP + 4 * q);
        v[0] = f2(x4.x, x4.y);
        v[1] = f2(x4.z, x4.w);
    }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::NT, 3) scan_bwd_kernel(const BwdArgs p) {
    using Tin = typename Cfg::Tin;
    using Tg = typename Cfg::Tg;
    constexpr int NP = Cfg::NP, Q = Cfg::Q, CH = Cfg::CH, T = Cfg::T, NT = Cfg::NT;
    extern __shared__ __align__(16) unsigned char smem[];

    const int tid = threadIdx.x;
    const int q = tid >> 5, lane = tid & 31, c = lane;
    const int cta = blockIdx.x;
    const int ctas = gridDim.x;
    const int b = cta / p.groups_per_seq;
    const int d0 = (cta - b * p.groups_per_seq) * CH;
    const int L = p.seqlen, N = p.dstate, dim = p.dim, ntiles = p.ntiles;
    const int nch = min(CH, dim - d0);
    const bool dvalid = c < nch;

    float4 *prep = reinterpret_cast<float4 *>(smem + Cfg::OFF_PREP);
    float *Bf = reinterpret_cast<float *>(smem + Cfg::OFF_BF);
    float *Cf = reinterpret_cast<float *>(smem + Cfg::OFF_CF);
    float *part0 = reinterpret_cast<float *>(smem + Cfg::OFF_PART);
    float *part1 = part0 + Cfg::PART_ARR / sizeof(float);
    float *xp = reinterpret_cast<float *>(smem + Cfg::OFF_XP) + q * 32 * Cfg::X_ROW;

    // this lane's 4 states as two pairs (0,1), (2,3) for the packed FP32 instructions
    float2 Af[2], A2[2];
    {
        float av[4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int n = 4 * q + s;
            av[s] = (dvalid && n < N) ? p.A[size_t(d0 + c) * N + n] : 0.f;
        }
        Af[0] = f2(av[0], av[1]);
        Af[1] = f2(av[2], av[3]);
        A2[0] = fmul2(Af[0], f2(kLog2e, kLog2e));
        A2[1] = fmul2(Af[1], f2(kLog2e, kLog2e));
    }
    // this thread's (t, d) task, if it has one: channel cc, token chunk tk of every tile
    constexpr int TW = Cfg::TW;
    const bool has_task = tid < Cfg::NTASK;
    const int cc = tid % CH, tk = has_task ? tid / CH : 0;
    const bool cvalid = has_task && cc < nch;
    const float tbias = (p.delta_bias != nullptr && cvalid) ? p.delta_bias[d0 + cc] : 0.f;
    const float tD = (p.D != nullptr && cvalid) ? p.D[d0 + cc] : 0.f;

    const size_t row0 = (size_t(b) * dim + d0) * size_t(L);
    const size_t bc0 = size_t(b) * L * size_t(N);
    const size_t chrow = size_t(b) * dim + d0 + c;
    // checkpoint k of this CTA (the state before token 4k) for this lane: float4 at ck(k)
    float4 *ckb = reinterpret_cast<float4 *>(p.ck) + (size_t(cta) * ntiles * (T / 4) * Q + q) * 32 + lane;
    auto ck = [&](int k) { return ckb + size_t(k) * Q * 32; };

    // ---------------- phase F: forward, keeping the state before every 4th token ----------------
    float2 h[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
    if (p.h0 != nullptr && dvalid) {
        float hv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < 4; ++s)
            if (4 * q + s < N) hv[s] = p.h0[chrow * N + 4 * q + s];
        h[0] = f2(hv[0], hv[1]);
        h[1] = f2(hv[2], hv[3]);
    }
    bwd_load_tile<Cfg>(p, smem, 0, 0, row0, bc0, nch, false);
    cp_async_commit();
    for (int tile = 0; tile < ntiles; ++tile) {
        const int t0 = tile * T;
        cp_async_wait<0>();
        __syncthreads();
        if (tile + 1 < ntiles) bwd_load_tile<Cfg>(p, smem, (tile + 1) & 1, t0 + T, row0, bc0, nch, false);
        cp_async_commit();
        const BwdStage<Cfg> sv(smem, tile & 1);
        if (has_task) bwd_prep<Cfg>(p, sv, prep, cc, tk, cvalid, tbias, t0, false);
        bwd_widen_bc<Cfg>(p, sv, Bf, Cf, t0, false);
        __syncthreads();
#pragma unroll
        for (int t = 0; t < T; ++t) {
            if (t % 4 == 0) *ck(tile * (T / 4) + t / 4) = make_float4(h[0].x, h[0].y, h[1].x, h[1].y);
            const float4 pv = prep[t * CH + c];
            float2 bb[2];
            bwd_quad<Cfg>(Bf, t, q, bb);
            const float2 dl2 = f2(pv.x, pv.x);
            const float dx = pv.x * pv.y;
            const float2 dx2 = f2(dx, dx);
#pragma unroll
            for (int k = 0; k < 2; ++k)
                h[k] = ffma2(ex2_pair(fmul2(dl2, A2[k])), h[k], fmul2(dx2, bb[k]));
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---------------- phase R: tiles in reverse ----------------
    float2 mu[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
    if (p.dfinal != nullptr && dvalid) {
        float mv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < 4; ++s)
            if (4 * q + s < N) mv[s] = p.dfinal[chrow * N + 4 * q + s];
        mu[0] = f2(mv[0], mv[1]);
        mu[1] = f2(mv[2], mv[3]);
    }
    float2 dA_acc[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
    float dD_acc = 0.f, db_acc = 0.f;          // this thread's task channel, over its chunks
    float *part2 = part1 + Cfg::PART_ARR / sizeof(float);
    float *dxp = part0 + (q * CH + c) * Cfg::P_ROW;    // per-quad partials of this lane:
    float *ddp = part1 + (q * CH + c) * Cfg::P_ROW;    //   sum_n lambda B, the dDelta terms,
    float *ypp = part2 + (q * CH + c) * Cfg::P_ROW;    //   and the readout sum_n C h
    float *xrow = xp + lane * Cfg::X_ROW;
    const size_t bc_stride = size_t(ctas) * L * NP;    // dB block -> dC block of part_bc
    float *pbc = p.part_bc + size_t(cta) * L * NP;
    // checkpoints are read two sub-chunks ahead of their use (they come from HBM)
    const int nck = ntiles * (T / 4);
    float4 ck1 = *ck(nck - 1);
    float4 ck2 = nck >= 2 ? *ck(nck - 2) : make_float4(0.f, 0.f, 0.f, 0.f);
    int knext = nck - 3;

    bwd_load_tile<Cfg>(p, smem, 0, (ntiles - 1) * T, row0, bc0, nch, true);
    cp_async_commit();
    for (int r = 0; r < ntiles; ++r) {
        const int tile = ntiles - 1 - r;
        const int t0 = tile * T;
        cp_async_wait<0>();
        __syncthreads();
        if (tile > 0) bwd_load_tile<Cfg>(p, smem, (r + 1) & 1, t0 - T, row0, bc0, nch, true);
        cp_async_commit();
        const BwdStage<Cfg> sv(smem, r & 1);
        if (has_task) bwd_prep<Cfg>(p, sv, prep, cc, tk, cvalid, tbias, t0, true);
        bwd_widen_bc<Cfg>(p, sv, Bf, Cf, t0, true);
        __syncthreads();

        // sub-chunks of 4 tokens, last first: recompute their states from the checkpoint,
        // keep the readout, then walk them backwards carrying mu
#pragma unroll kBwdUnrollJ
        for (int j = T / 4 - 1; j >= 0; --j) {
            const float4 hv = ck1;
            ck1 = ck2;
            if (knext >= 0) ck2 = *ck(knext);
            --knext;
            float2 hs[5][2], a[4][2];
            float dl[4], xv[4], dyp[4], yo[4];
            hs[0][0] = f2(hv.x, hv.y);
            hs[0][1] = f2(hv.z, hv.w);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int t = 4 * j + u;
                const float4 pv = prep[t * CH + c];
                dl[u] = pv.x; xv[u] = pv.y; dyp[u] = pv.z;
                float2 bb[2], cb[2];
                bwd_quad<Cfg>(Bf, t, q, bb);
                bwd_quad<Cfg>(Cf, t, q, cb);
                const float2 dl2 = f2(dl[u], dl[u]);
                const float dx = dl[u] * xv[u];
                const float2 dx2 = f2(dx, dx);
                float2 acc = f2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    a[u][k] = ex2_pair(fmul2(dl2, A2[k]));
                    hs[u + 1][k] = ffma2(a[u][k], hs[u][k], fmul2(dx2, bb[k]));
                    acc = ffma2(cb[k], hs[u + 1][k], acc);
                }
                yo[u] = acc.x + acc.y;
            }
            *reinterpret_cast<float4 *>(ypp + 4 * j) = make_float4(yo[0], yo[1], yo[2], yo[3]);
            float dxo[4], ddo[4];
#pragma unroll
            for (int u = 3; u >= 0; --u) {
                const int t = 4 * j + u;
                float2 bb[2], cb[2];
                bwd_quad<Cfg>(Bf, t, q, bb);
                bwd_quad<Cfg>(Cf, t, q, cb);
                const float dlx = dl[u] * xv[u];
                const float2 dyp2 = f2(dyp[u], dyp[u]), dlx2 = f2(dlx, dlx), dl2 = f2(dl[u], dl[u]);
                // sum_n lambda B_n gives both dx (times Delta) and, times x, the B part of
                // dDelta; the decay part of dDelta and dA share lambda h_{t-1} Abar
                float2 lb = f2(0.f, 0.f), s2 = f2(0.f, 0.f), vb[2], vc[2];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float2 lam = ffma2(dyp2, cb[k], mu[k]);
                    const float2 lha = fmul2(lam, fmul2(hs[u][k], a[u][k]));
                    vb[k] = fmul2(lam, dlx2);                    // dB terms
                    vc[k] = fmul2(dyp2, hs[u + 1][k]);           // dC terms
                    lb = ffma2(lam, bb[k], lb);
                    s2 = ffma2(lha, Af[k], s2);
                    dA_acc[k] = ffma2(lha, dl2, dA_acc[k]);
                    mu[k] = fmul2(a[u][k], lam);
                }
                const float lbs = lb.x + lb.y;
                dxo[u] = lbs * dl[u];
                ddo[u] = fmaf(lbs, xv[u], s2.x + s2.y);
                *reinterpret_cast<float4 *>(xrow + 8 * u) = make_float4(vb[0].x, vb[0].y, vb[1].x, vb[1].y);
                *reinterpret_cast<float4 *>(xrow + 8 * u + 4) = make_float4(vc[0].x, vc[0].y, vc[1].x, vc[1].y);
            }
            *reinterpret_cast<float4 *>(dxp + 4 * j) = make_float4(dxo[0], dxo[1], dxo[2], dxo[3]);
            *reinterpret_cast<float4 *>(ddp + 4 * j) = make_float4(ddo[0], ddo[1], ddo[2], ddo[3]);
            __syncwarp();
            // column `lane` of the warp's transpose: value (token u, B or C, state s) summed
            // over the 32 channels
            float part[SSM_BWD_COLSUM_ACC];
#pragma unroll
            for (int k = 0; k < SSM_BWD_COLSUM_ACC; ++k) part[k] = 0.f;
#pragma unroll
            for (int rr = 0; rr < 32; ++rr) part[rr % SSM_BWD_COLSUM_ACC] += xp[rr * Cfg::X_ROW + lane];
            float sum = part[0];
#pragma unroll
            for (int k = 1; k < SSM_BWD_COLSUM_ACC; ++k) sum += part[k];
            __syncwarp();
            const int u = lane >> 3, which = (lane >> 2) & 1, st = lane & 3;
            const int tok = t0 + 4 * j + u;
            if (tok < L && 4 * q + st < N)
                pbc[which * bc_stride + size_t(tok) * NP + 4 * q + st] = sum;
        }
        __syncthreads();

        // per (t, d): the quads' partials summed; dx with the skip, dDelta through the
        // softplus slope, dz from the pre-gate output
        {
            float dxs[TW], dds[TW], yps[TW], dzv[TW];
#pragma unroll
            for (int u = 0; u < TW; ++u) { dxs[u] = 0.f; dds[u] = 0.f; yps[u] = 0.f; }
#pragma unroll
            for (int qq = 0; qq < Q; ++qq) {
                const float *s0 = part0 + (qq * CH + cc) * Cfg::P_ROW + TW * tk;
                const float *s1 = part1 + (qq * CH + cc) * Cfg::P_ROW + TW * tk;
                const float *s2 = part2 + (qq * CH + cc) * Cfg::P_ROW + TW * tk;
                float v0[TW], v1[TW], v2[TW];
                loadn<TW, float>(s0, v0);
                loadn<TW, float>(s1, v1);
                loadn<TW, float>(s2, v2);
#pragma unroll
                for (int u = 0; u < TW; ++u) { dxs[u] += v0[u]; dds[u] += v1[u]; yps[u] += v2[u]; }
            }
            float xr[TW], dr[TW], gr[TW], zr[TW];
            loadn<TW, Tin>(sv.xs + cc * Cfg::RAW_ROW + TW * tk, xr);
            loadn<TW, Tin>(sv.ds + cc * Cfg::RAW_ROW + TW * tk, dr);
            loadn<TW, Tg>(sv.gs + cc * Cfg::G_ROW + TW * tk, gr);
            if (p.z != nullptr) loadn<TW, Tin>(sv.zs + cc * Cfg::RAW_ROW + TW * tk, zr);
#pragma unroll
            for (int u = 0; u < TW; ++u) {
                const float dyp = prep[(TW * tk + u) * CH + cc].z;
                const bool ok = cvalid && t0 + TW * tk + u < L;
                dxs[u] = fmaf(dyp, tD, dxs[u]);
                if (p.softplus) dds[u] *= sigmoid_f(dr[u] + tbias);
                dds[u] = ok ? dds[u] : 0.f;          // no-op tokens carry no step gradient
                dzv[u] = 0.f;
                if (p.z != nullptr) {
                    const float ypre = fmaf(tD, xr[u], yps[u]);
                    const float sg = sigmoid_f(zr[u]);
                    dzv[u] = ok ? gr[u] * ypre * sg * fmaf(zr[u], 1.f - sg, 1.f) : 0.f;
                }
                dD_acc = fmaf(dyp, ok ? xr[u] : 0.f, dD_acc);
                db_acc += dds[u];
            }
            __syncthreads();                         // the partials are read: reuse as staging
            if (has_task) {
                Tg *ox = reinterpret_cast<Tg *>(part0);
                Tg *od = ox + CH * Cfg::G_ROW;
                Tg *oz = od + CH * Cfg::G_ROW;
                storen<TW, Tg>(ox + cc * Cfg::G_ROW + TW * tk, dxs);
                storen<TW, Tg>(od + cc * Cfg::G_ROW + TW * tk, dds);
                if (p.z != nullptr) storen<TW, Tg>(oz + cc * Cfg::G_ROW + TW * tk, dzv);
            }
        }
        __syncthreads();

        // dx, ddelta, dz rows of the tile back to global memory (coalesced)
        {
            const Tg *ox = reinterpret_cast<const Tg *>(part0);
            const int narr = p.dz != nullptr ? 3 : 2;
            if constexpr (Cfg::VEC) {
                constexpr int CPR = T / Cfg::EG;
#pragma unroll
                for (int k = 0; k < (3 * CH * CPR + NT - 1) / NT; ++k) {
                    const int i = tid + k * NT;
                    const int a = i / (CH * CPR);
                    const int rem = i % (CH * CPR);
                    const int ch = rem / CPR, qq = rem % CPR;
                    const int tg = t0 + qq * Cfg::EG;
                    if (i < 3 * CH * CPR && a < narr && ch < nch && tg < L) {
                        Tg *dst = static_cast<Tg *>(a == 0 ? p.dx : a == 1 ? p.ddelta : p.dz) + row0 +
                                  size_t(ch) * L + tg;
                        *reinterpret_cast<uint4 *>(dst) =
                            *reinterpret_cast<const uint4 *>(ox + (a * CH + ch) * Cfg::G_ROW + qq * Cfg::EG);
                    }
                }
            } else {
                for (int i = tid; i < narr * CH * T; i += NT) {
                    const int a = i / (CH * T);
                    const int rem = i % (CH * T);
                    const int ch = rem / T, tt = rem % T;
                    if (ch < nch && t0 + tt < L) {
                        Tg *dst = static_cast<Tg *>(a == 0 ? p.dx : a == 1 ? p.ddelta : p.dz) + row0 +
                                  size_t(ch) * L + t0 + tt;
                        *dst = ox[(a * CH + ch) * Cfg::G_ROW + tt];
                    }
                }
            }
        }
    }
    cp_async_wait<0>();

    // per-sequence partials: dA of this lane's states; dD and ddelta_bias of the channels
    if (dvalid) {
        *reinterpret_cast<float4 *>(p.part_a + chrow * NP + 4 * q) =
            make_float4(dA_acc[0].x, dA_acc[0].y, dA_acc[1].x, dA_acc[1].y);
        if (p.dh0 != nullptr) {
            const float mv[4] = {mu[0].x, mu[0].y, mu[1].x, mu[1].y};
#pragma unroll
            for (int s = 0; s < 4; ++s)
                if (4 * q + s < N) p.dh0[chrow * N + 4 * q + s] = mv[s];
        }
    }
    __syncthreads();
    float *red = reinterpret_cast<float *>(prep);   // [2][NTW][CH]
    if (has_task) {
        red[tk * CH + cc] = dD_acc;
        red[(Cfg::NTW + tk) * CH + cc] = db_acc;
    }
    __syncthreads();
    if (tid < nch) {
        float sd = 0.f, sb = 0.f;
#pragma unroll
        for (int k = 0; k < Cfg::NTW; ++k) {
            sd += red[k * CH + tid];
            sb += red[(Cfg::NTW + k) * CH + tid];
        }
        const size_t bd = size_t(b) * dim + d0 + tid;
        p.part_dd[bd] = sd;
        p.part_dd[size_t(p.batch) * dim + bd] = sb;
    }
}

// The same sum when every row is whole (NPin == Nout, a multiple of 4): four consecutive
// outputs per thread with 16-byte loads, eight loads in flight, summed in k order in two
// interleaved halves (even k, odd k) that are added at the end -- a fixed order, so the
// result is deterministic.
template <typename To>
__global__ void __launch_bounds__(256)
reduce_partials_vec4_kernel(const float *__restrict__ in, To *__restrict__ out, long long outer,
                            int K, long long R4) {
    const long long total = outer * R4;               // float4 groups of the output
    for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long i = e / R4, r = e - i * R4;
        const float4 *src = reinterpret_cast<const float4 *>(in) + (i * K) * R4 + r;
        float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
        int k = 0;
        for (; k + 8 <= K; k += 8) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __ldg(src + static_cast<long long>(k + u) * R4);
#pragma unroll
            for (int u = 0; u < 8; u += 2) {
                a0.x += v[u].x; a0.y += v[u].y; a0.z += v[u].z; a0.w += v[u].w;
                a1.x += v[u + 1].x; a1.y += v[u + 1].y; a1.z += v[u + 1].z; a1.w += v[u + 1].w;
            }
        }
        for (; k < K; ++k) {
            const float4 v = __ldg(src + static_cast<long long>(k) * R4);
            if (k & 1) { a1.x += v.x; a1.y += v.y; a1.z += v.z; a1.w += v.w; }
            else       { a0.x += v.x; a0.y += v.y; a0.z += v.z; a0.w += v.w; }
        }
        const float o[4] = {a0.x + a1.x, a0.y + a1.y, a0.z + a1.z, a0.w + a1.w};
        store_run<4>(out + 4 * e, o);
    }
}

// out[(i*R + r)*Nout + n] = sum_{k<K} in[((i*K + k)*R + r)*NPin + n] for n < Nout, summed
// in k order (deterministic).  One thread per output element.
template <typename To>
__global__ void __launch_bounds__(256)
reduce_partials_kernel(const float *__restrict__ in, To *__restrict__ out, long long outer, int K,
                       long long R, int NPin, int Nout) {
    const long long total = outer * R * Nout;
    for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long n = e % Nout;
        const long long ir = e / Nout;                 // i * R + r
        const long long i = ir / R, r = ir - i * R;
        const float *src = in + ((i * K) * R + r) * NPin + n;
        float acc = 0.f;
        for (int k = 0; k < K; ++k) acc += src[static_cast<long long>(k) * R * NPin];
        out[e] = from_f32<To>(acc);
    }
}


}  // namespace ssm
