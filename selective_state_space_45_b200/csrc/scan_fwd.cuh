// scan_fwd.cuh -- the selective scan (S6) forward kernel for sm_100a.
//
// What one launch computes (per sequence b, channel d, state n, token t):
//   Delta = softplus(delta + bias[d]) (optional), Abar = exp(Delta * A[d,n]),
//   h_n <- Abar * h_n + Delta * B[b,t,n] * x,  y = (C[b,t,:] . h + D[d] x) * SiLU(z).
// Sources: "Module 19: State-Space Models (Mamba)" (learnllm), "The Math: The
// State-Space Recurrence" (ZOH decay, Euler gain) and "The Parallel Scan" (the affine
// composition used for the in-tile stitch); "Beyond attention with Mamba, state space
// models and hybrids" (xmarva lesson 10), sections 3-4 (selective Delta, B, C; the skip
// and the gate) and 6 (the scan whose N-expanded states never go to main memory).
//
// Work decomposition
//   * A CTA owns CH channels of one sequence for the whole length L and walks L in tiles
//     of T = K * TS tokens.  The state never leaves registers/shared memory; the only
//     HBM traffic is x, delta, z, B, C in and y, final_state out.
//   * G = NP / 4 consecutive lanes share one channel, each lane owning 4 of its NP
//     (padded) states, so one 16-byte shared load gives a lane its B (or C) values.
//   * K warps split each tile in time (sub-chunk j = tokens [j*TS, (j+1)*TS)).  Every
//     sub-chunk scans from a zero state and records its running decay product P_t and
//     local state; the K aggregates (P_end, h_end) are composed in shared memory with
//     (a2, b2) o (a1, b1) = (a2 a1, a2 b1 + b2), and each sub-chunk corrects
//     h_t = h_loc,t + P_t * h_in before the readout.  No exponential is recomputed.
//     K = 1 skips the stitch and keeps the carried state in registers.
//   * Per-(token, channel) work -- the softplus step, Delta * x, the skip and the SiLU
//     gate -- is done once per (t, d), spread over all threads, never once per state.
//   * Inputs are staged through a cp.async ring of NSTAGE tiles (16-byte copies) when
//     every row is 16-byte aligned (VEC); otherwise by guarded scalar loads.
//   * y is staged in shared memory and written back as 16-byte rows.
#pragma once

#include "common.cuh"

namespace ssm {

struct ScanArgs {
    const void *x;
    const void *delta;
    const float *delta_bias;
    const float *A;
    const void *B;
    const void *C;
    const float *D;
    const void *z;
    void *y;
    float *final_state;
    int batch, dim, seqlen, dstate;
    int softplus;
    int groups_per_seq;  // ceil(dim / CH)
};

template <int NP_, int K_, int TS_, int CG_, int NSTAGE_, typename Tin_, typename Tout_, bool VEC_,
          int MINB_ = 1>
struct ScanCfg {
    using Tin = Tin_;
    using Tout = Tout_;
    static constexpr int NP = NP_;            // padded state width: 4, 8 or 16
    static constexpr int K = K_;              // sub-chunks (warps) per tile, per channel group
    static constexpr int TS = TS_;            // tokens per sub-chunk
    static constexpr int CG = CG_;            // channel groups (of CPW channels) per CTA
    static constexpr int NSTAGE = NSTAGE_;    // cp.async ring depth (tiles)
    static constexpr bool VEC = VEC_;
    static constexpr int MINB = MINB_;        // resident CTAs per SM the register budget targets
    static constexpr int G = NP / 4;          // lanes per channel
    static constexpr int CPW = 32 / G;        // channels per warp
    static constexpr int CH = CG * CPW;       // channels per CTA
    static constexpr int T = K * TS;          // tokens per tile
    static constexpr int NWARP = CG * K;
    static constexpr int NTHREADS = NWARP * 32;
    static constexpr int EIN = 16 / sizeof(Tin);    // elements per 16-byte chunk
    static constexpr int EOUT = 16 / sizeof(Tout);
    static constexpr int RAW_ROW = T + EIN;         // padded rows keep rows 16B-aligned and
    static constexpr int Y_ROW = T + EOUT;          // spread channels over banks
    static constexpr int PREP_ROW = T + 1;          // float2 elements
    static_assert(TS % G == 0, "sub-chunk must be a multiple of the lane group");
    static_assert(K > 1, "the stitched kernel splits every tile over several warps");
    static_assert((T * sizeof(Tin)) % 16 == 0 && (T * sizeof(Tout)) % 16 == 0, "tile rows");

    // shared-memory layout (byte offsets, 16-byte aligned pieces)
    static constexpr size_t al(size_t v) { return (v + 15) & ~size_t(15); }
    static constexpr size_t RAW_ARR = al(size_t(CH) * RAW_ROW * sizeof(Tin));
    static constexpr size_t RAW_BC = al(size_t(T) * NP * sizeof(Tin));
    static constexpr size_t STAGE_BYTES = 3 * RAW_ARR + 2 * RAW_BC;
    static constexpr size_t OFF_RAW = 0;
    static constexpr size_t OFF_PREP = OFF_RAW + NSTAGE * STAGE_BYTES;
    static constexpr size_t OFF_BF = OFF_PREP + al(size_t(CH) * PREP_ROW * sizeof(float2));
    static constexpr size_t OFF_CF = OFF_BF + al(size_t(T) * NP * sizeof(float));
    static constexpr size_t OFF_Y = OFF_CF + al(size_t(T) * NP * sizeof(float));
    static constexpr size_t OFF_BIAS = OFF_Y + al(size_t(CH) * Y_ROW * sizeof(Tout));
    static constexpr size_t OFF_AGG = OFF_BIAS + al(size_t(CH) * sizeof(float));
    static constexpr size_t AGG_BYTES = (K > 1) ? al(size_t(2) * K * CH * NP * sizeof(float)) : 0;
    static constexpr size_t OFF_CARRY = OFF_AGG + AGG_BYTES;
    static constexpr size_t CARRY_BYTES = (K > 1) ? al(size_t(2) * CH * NP * sizeof(float)) : 0;
    static constexpr size_t SMEM_BYTES = OFF_CARRY + CARRY_BYTES;
};

// Views of one ring stage.
template <class Cfg> struct Stage {
    typename Cfg::Tin *xs, *ds, *zs, *bs, *cs;
    __device__ __forceinline__ Stage(unsigned char *smem, int s) {
        unsigned char *base = smem + Cfg::OFF_RAW + size_t(s) * Cfg::STAGE_BYTES;
        xs = reinterpret_cast<typename Cfg::Tin *>(base);
        ds = reinterpret_cast<typename Cfg::Tin *>(base + Cfg::RAW_ARR);
        zs = reinterpret_cast<typename Cfg::Tin *>(base + 2 * Cfg::RAW_ARR);
        bs = reinterpret_cast<typename Cfg::Tin *>(base + 3 * Cfg::RAW_ARR);
        cs = reinterpret_cast<typename Cfg::Tin *>(base + 3 * Cfg::RAW_ARR + Cfg::RAW_BC);
    }
};

// Stage tile [t0, t0 + T) of x, delta, z (nch channel rows) and of B, C into ring stage st.
// VEC path: 16-byte cp.async chunks; every chunk is either wholly inside [0, L) or
// wholly outside, because L is a multiple of the chunk width.  Scalar path: guarded
// loads, complete when the function returns.
template <class Cfg>
__device__ __forceinline__ void load_tile(const ScanArgs &p, unsigned char *smem, int st, int t0,
                                          size_t row0, size_t bc0, int nch) {
    using Tin = typename Cfg::Tin;
    Stage<Cfg> s(smem, st);
    const int L = p.seqlen, N = p.dstate;
    const Tin *gx = static_cast<const Tin *>(p.x) + row0;
    const Tin *gd = static_cast<const Tin *>(p.delta) + row0;
    const Tin *gz = p.z ? static_cast<const Tin *>(p.z) + row0 : nullptr;
    const int narr = p.z ? 3 : 2;
    if constexpr (Cfg::VEC) {
        constexpr int CPR = Cfg::T / Cfg::EIN;  // chunks per row
        const int nrow_chunks = narr * nch * CPR;
        for (int i = threadIdx.x; i < nrow_chunks; i += Cfg::NTHREADS) {
            const int a = i / (nch * CPR);
            const int rem = i - a * nch * CPR;
            const int cc = rem / CPR;
            const int q = rem - cc * CPR;
            const int tg = t0 + q * Cfg::EIN;
            if (tg < L) {
                const Tin *src = (a == 0 ? gx : a == 1 ? gd : gz) + size_t(cc) * L + tg;
                Tin *dst = (a == 0 ? s.xs : a == 1 ? s.ds : s.zs) + cc * Cfg::RAW_ROW + q * Cfg::EIN;
                cp_async_16(dst, src);
            }
        }
        const int valid_t = min(Cfg::T, L - t0);
        const int bc_chunks = (valid_t * N * int(sizeof(Tin))) / 16;
        const Tin *gb = static_cast<const Tin *>(p.B) + bc0 + size_t(t0) * N;
        const Tin *gc = static_cast<const Tin *>(p.C) + bc0 + size_t(t0) * N;
        for (int i = threadIdx.x; i < 2 * bc_chunks; i += Cfg::NTHREADS) {
            const int which = i >= bc_chunks;
            const int q = i - which * bc_chunks;
            cp_async_16((which ? s.cs : s.bs) + q * Cfg::EIN, (which ? gc : gb) + q * Cfg::EIN);
        }
    } else {
        const int nel = narr * nch * Cfg::T;
        for (int i = threadIdx.x; i < nel; i += Cfg::NTHREADS) {
            const int a = i / (nch * Cfg::T);
            const int rem = i - a * nch * Cfg::T;
            const int cc = rem / Cfg::T;
            const int tt = rem - cc * Cfg::T;
            const int tg = t0 + tt;
            if (tg < L) {
                const Tin *src = (a == 0 ? gx : a == 1 ? gd : gz) + size_t(cc) * L + tg;
                Tin *dst = (a == 0 ? s.xs : a == 1 ? s.ds : s.zs) + cc * Cfg::RAW_ROW + tt;
                *dst = *src;
            }
        }
        const int valid_t = min(Cfg::T, L - t0);
        const int nbc = valid_t * N;
        const Tin *gb = static_cast<const Tin *>(p.B) + bc0 + size_t(t0) * N;
        const Tin *gc = static_cast<const Tin *>(p.C) + bc0 + size_t(t0) * N;
        for (int i = threadIdx.x; i < 2 * nbc; i += Cfg::NTHREADS) {
            const int which = i >= nbc;
            const int q = i - which * nbc;
            (which ? s.cs : s.bs)[q] = (which ? gc : gb)[q];
        }
    }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::NTHREADS, Cfg::MINB)
scan_fwd_kernel(const ScanArgs p) {
    using Tin = typename Cfg::Tin;
    using Tout = typename Cfg::Tout;
    constexpr int NP = Cfg::NP, K = Cfg::K, TS = Cfg::TS, T = Cfg::T, G = Cfg::G;
    constexpr int CPW = Cfg::CPW, CH = Cfg::CH, NT = Cfg::NTHREADS;
    extern __shared__ __align__(16) unsigned char smem[];

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int cg = warp / K;          // channel group of this warp
    const int j = warp - cg * K;      // time sub-chunk of this warp
    const int ci = lane / G;          // channel within the warp
    const int r = lane - ci * G;      // state quad within the channel
    const int c = cg * CPW + ci;      // channel within the CTA
    const int b = blockIdx.x / p.groups_per_seq;
    const int d0 = (blockIdx.x - b * p.groups_per_seq) * CH;
    const int d = d0 + c;
    const int L = p.seqlen, N = p.dstate, dim = p.dim;
    const int nch = min(CH, dim - d0);
    const bool dvalid = c < nch;

    float2 *prep = reinterpret_cast<float2 *>(smem + Cfg::OFF_PREP);
    float *Bf = reinterpret_cast<float *>(smem + Cfg::OFF_BF);
    float *Cf = reinterpret_cast<float *>(smem + Cfg::OFF_CF);
    Tout *ys = reinterpret_cast<Tout *>(smem + Cfg::OFF_Y);
    float *bias_s = reinterpret_cast<float *>(smem + Cfg::OFF_BIAS);
    float *aggP = reinterpret_cast<float *>(smem + Cfg::OFF_AGG);
    float *aggH = aggP + K * CH * NP;
    float *carry = reinterpret_cast<float *>(smem + Cfg::OFF_CARRY);

    // per-lane constants: A * log2(e) for the 4 owned states, the skip weight
    float A2[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const int n = 4 * r + s;
        A2[s] = (dvalid && n < N) ? p.A[size_t(d) * N + n] * kLog2e : 0.f;
    }
    const float Dd = (p.D != nullptr && dvalid) ? p.D[d] : 0.f;
    for (int i = tid; i < CH; i += NT)
        bias_s[i] = (p.delta_bias != nullptr && i < nch) ? p.delta_bias[d0 + i] : 0.f;
    if constexpr (K > 1) {
        for (int i = tid; i < CH * NP; i += NT) carry[i] = 0.f;
    }

    const size_t row0 = (size_t(b) * dim + d0) * size_t(L);
    const size_t bc0 = size_t(b) * L * size_t(N);
    const int ntiles = (L + T - 1) / T;

    // prologue: fill NSTAGE - 1 ring stages
#pragma unroll
    for (int s = 0; s < Cfg::NSTAGE - 1; ++s) {
        if (s < ntiles) load_tile<Cfg>(p, smem, s, s * T, row0, bc0, nch);
        cp_async_commit();
    }

    float h[4] = {0.f, 0.f, 0.f, 0.f};       // carry after the last tile (kept by warp K-1)
    int cur = 0;                               // carry double-buffer index (K > 1)

    for (int tile = 0; tile < ntiles; ++tile) {
        const int st = tile % Cfg::NSTAGE;
        const int t0 = tile * T;
        cp_async_wait<Cfg::NSTAGE - 2>();
        __syncthreads();
        {   // refill the stage freed by the previous tile
            const int nt = tile + Cfg::NSTAGE - 1;
            if (nt < ntiles) load_tile<Cfg>(p, smem, nt % Cfg::NSTAGE, nt * T, row0, bc0, nch);
            cp_async_commit();
        }
        Stage<Cfg> sv(smem, st);

        // ---- per-(t, d) step and per-(t, n) B, C widening, once per tile ----
        for (int i = tid; i < CH * T; i += NT) {
            const int cc = i / T, tt = i - (i / T) * T;
            float2 v = make_float2(0.f, 0.f);   // tokens past L / channels past dim: no-op step
            if (cc < nch && t0 + tt < L) {
                float dl = to_f32(sv.ds[cc * Cfg::RAW_ROW + tt]) + bias_s[cc];
                if (p.softplus) dl = softplus_f(dl);
                v = make_float2(dl, dl * to_f32(sv.xs[cc * Cfg::RAW_ROW + tt]));
            }
            prep[cc * Cfg::PREP_ROW + tt] = v;
        }
        for (int i = tid; i < T * NP; i += NT) {
            const int tt = i / NP, n = i - (i / NP) * NP;
            const bool ok = n < N && t0 + tt < L;
            Bf[i] = ok ? to_f32(sv.bs[tt * N + n]) : 0.f;
            Cf[i] = ok ? to_f32(sv.cs[tt * N + n]) : 0.f;
        }
        __syncthreads();

        // ---- scan of this warp's sub-chunk ----
        // yout[m]: the channel's full readout for token j*TS + m*G + r, once summed
        // over the G lanes of the channel.
        float yout[TS / G];
        const float2 *prow = prep + c * Cfg::PREP_ROW + j * TS;
        {
            float hl[TS][4], Pl[TS][4];
            float hs[4] = {0.f, 0.f, 0.f, 0.f}, P[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
            for (int i = 0; i < TS; ++i) {
                const int tt = j * TS + i;
                const float2 dd = prow[i];
                const float4 bq = *reinterpret_cast<const float4 *>(Bf + tt * NP + 4 * r);
                const float bb[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const float a = ex2_approx(dd.x * A2[s]);
                    hs[s] = fmaf(a, hs[s], dd.y * bb[s]);
                    P[s] *= a;
                    hl[i][s] = hs[s];
                    Pl[i][s] = P[s];
                }
            }
            float *myP = aggP + (j * CH + c) * NP + 4 * r;
            float *myH = aggH + (j * CH + c) * NP + 4 * r;
            *reinterpret_cast<float4 *>(myP) = make_float4(P[0], P[1], P[2], P[3]);
            *reinterpret_cast<float4 *>(myH) = make_float4(hs[0], hs[1], hs[2], hs[3]);
            __syncthreads();
            // state entering this sub-chunk: carry composed with sub-chunks 0 .. j-1
            float hin[4];
            {
                const float4 cv = *reinterpret_cast<const float4 *>(carry + (cur * CH + c) * NP + 4 * r);
                hin[0] = cv.x; hin[1] = cv.y; hin[2] = cv.z; hin[3] = cv.w;
            }
            for (int jj = 0; jj < j; ++jj) {
                const float4 pv = *reinterpret_cast<const float4 *>(aggP + (jj * CH + c) * NP + 4 * r);
                const float4 hv = *reinterpret_cast<const float4 *>(aggH + (jj * CH + c) * NP + 4 * r);
                hin[0] = fmaf(pv.x, hin[0], hv.x);
                hin[1] = fmaf(pv.y, hin[1], hv.y);
                hin[2] = fmaf(pv.z, hin[2], hv.z);
                hin[3] = fmaf(pv.w, hin[3], hv.w);
            }
            if (j == K - 1) {
#pragma unroll
                for (int s = 0; s < 4; ++s) h[s] = fmaf(P[s], hin[s], hs[s]);
                *reinterpret_cast<float4 *>(carry + ((cur ^ 1) * CH + c) * NP + 4 * r) =
                    make_float4(h[0], h[1], h[2], h[3]);
            }
            cur ^= 1;
            float yp[TS];
#pragma unroll
            for (int i = 0; i < TS; ++i) {
                const int tt = j * TS + i;
                const float4 cq = *reinterpret_cast<const float4 *>(Cf + tt * NP + 4 * r);
                const float cc4[4] = {cq.x, cq.y, cq.z, cq.w};
                float acc = 0.f;
#pragma unroll
                for (int s = 0; s < 4; ++s) acc = fmaf(cc4[s], fmaf(Pl[i][s], hin[s], hl[i][s]), acc);
                yp[i] = acc;
            }
#pragma unroll
            for (int m = 0; m < TS / G; ++m) yout[m] = GroupReduceScatter<G>::run(yp + m * G, r);
        }

        // ---- skip, gate; stage y ----
#pragma unroll
        for (int m = 0; m < TS / G; ++m) {
            const float ysum = yout[m];
            const int tt = j * TS + m * G + r;
            const float xv = to_f32(sv.xs[c * Cfg::RAW_ROW + tt]);
            float yv = fmaf(Dd, xv, ysum);
            if (p.z != nullptr) yv *= silu_f(to_f32(sv.zs[c * Cfg::RAW_ROW + tt]));
            ys[c * Cfg::Y_ROW + tt] = from_f32<Tout>(yv);
        }
        __syncthreads();

        // ---- write y rows back ----
        Tout *gy = static_cast<Tout *>(p.y) + row0;
        if constexpr (Cfg::VEC) {
            constexpr int CPR = T / Cfg::EOUT;
            for (int i = tid; i < nch * CPR; i += NT) {
                const int cc = i / CPR, q = i - (i / CPR) * CPR;
                const int tg = t0 + q * Cfg::EOUT;
                if (tg < L)
                    *reinterpret_cast<uint4 *>(gy + size_t(cc) * L + tg) =
                        *reinterpret_cast<const uint4 *>(ys + cc * Cfg::Y_ROW + q * Cfg::EOUT);
            }
        } else {
            for (int i = tid; i < nch * T; i += NT) {
                const int cc = i / T, tt = i - (i / T) * T;
                if (t0 + tt < L) gy[size_t(cc) * L + t0 + tt] = ys[cc * Cfg::Y_ROW + tt];
            }
        }
    }
    cp_async_wait<0>();

    // ---- final state: held by the last sub-chunk's warp ----
    if (p.final_state != nullptr && dvalid && j == K - 1) {
        float *fs = p.final_state + (size_t(b) * dim + d) * N;
#pragma unroll
        for (int s = 0; s < 4; ++s)
            if (4 * r + s < N) fs[4 * r + s] = h[s];
    }
}

}  // namespace ssm
