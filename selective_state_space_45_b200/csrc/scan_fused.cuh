// scan_fused.cuh -- selective scan forward, one channel per lane, phases interleaved.
//
// Same computation as scan_fwd.cuh (sources there).  One CTA owns 32 channels of one
// sequence for the whole length L and walks it in T-token tiles; warp q holds states
// 4q..4q+3 of the 32 channels (one channel per lane) in registers from the first token to
// the last.  B_t and C_t of a state quad are warp-uniform: one broadcast load each.
//
// While scanning tile i, warp q also does its quarter (tokens 4q..4q+3 of a tile) of
//   * the step of tile i+1:  Delta = softplus(delta + bias), Delta * x     (prep), and
//   * the output of tile i-1: sum of the four quads' partial readouts, + D x, * SiLU(z),
// with the three instruction streams mixed in one loop body, so the SFU-heavy recurrence
// and the FMA-heavy per-(t, d) work overlap inside every warp.  One CTA barrier per tile
// publishes prep(i+1), B/C(i+1), the partial readouts of tile i and y(i-1).  y of tile i-2
// is written to global memory with 16-byte coalesced stores at the start of tile i.
//
// x, delta, z, B, C are staged by a cp.async ring of 5 tiles (tile i-1 is still read by the
// epilogue, i+1 by the prep, i+2 has landed, i+3 is in flight).
#pragma once

#include "common.cuh"
#include "scan_fwd.cuh"   // ScanArgs, Stage
#include "scan_lanes.cuh" // load8 / store8
#include "scan_ws.cuh"    // load4s / store4s

namespace ssm {

template <int NP_, int T_, typename Tin_, typename Tout_, bool VEC_, int MINB_>
struct FusedCfg {
    using Tin = Tin_;
    using Tout = Tout_;
    static constexpr int NP = NP_;
    static constexpr int Q = NP / 4;             // warps = state quads
    static constexpr int CH = 32;                // channels per CTA, one per lane
    static constexpr int T = T_;                 // tokens per tile
    static constexpr int TQ = T / Q;             // tokens of a tile in one warp's slice
    static constexpr int NSTAGE = 5;
    static constexpr bool VEC = VEC_;
    static constexpr int MINB = MINB_;
    static constexpr int NTHREADS = 32 * Q;
    static constexpr int EIN = 16 / sizeof(Tin);
    static constexpr int EOUT = 16 / sizeof(Tout);
    static constexpr int RAW_ROW = T + EIN;      // row stride 16 B past a multiple of 16 B
    static constexpr int Y_ROW = T + EOUT;
    static constexpr int YP_ROW = T + 4;         // floats
    static_assert(T % 4 == 0 && T % Q == 0 && TQ % 4 == 0, "tile / slice shape");
    static_assert(T * sizeof(Tin) % 16 == 0 && T * sizeof(Tout) % 16 == 0, "16-byte rows");

    static constexpr size_t al(size_t v) { return (v + 127) & ~size_t(127); }
    static constexpr size_t RAW_ARR = al(size_t(CH) * RAW_ROW * sizeof(Tin));
    static constexpr size_t RAW_BC = al(size_t(T) * NP * sizeof(Tin));
    static constexpr size_t STAGE_BYTES = 3 * RAW_ARR + 2 * RAW_BC;
    static constexpr size_t OFF_RAW = 0;
    static constexpr size_t PREP_BYTES = al(size_t(T / 2) * CH * sizeof(float4));
    static constexpr size_t BC_BYTES = al(size_t(T) * NP * sizeof(float));
    static constexpr size_t YP_BYTES = al(size_t(Q) * CH * YP_ROW * sizeof(float));
    static constexpr size_t Y_BYTES = al(size_t(CH) * Y_ROW * sizeof(Tout));
    static constexpr size_t OFF_PREP = OFF_RAW + NSTAGE * STAGE_BYTES;   // x2
    static constexpr size_t OFF_BF = OFF_PREP + 2 * PREP_BYTES;          // x2
    static constexpr size_t OFF_CF = OFF_BF + 2 * BC_BYTES;              // x2
    static constexpr size_t OFF_YP = OFF_CF + 2 * BC_BYTES;              // x2
    static constexpr size_t OFF_Y = OFF_YP + 2 * YP_BYTES;               // x2
    static constexpr size_t SMEM_BYTES = OFF_Y + 2 * Y_BYTES;
    static constexpr int NHELP_T = NTHREADS;     // loader thread count (all threads load)
};

template <class Cfg>
__global__ void __launch_bounds__(Cfg::NTHREADS, Cfg::MINB)
scan_fused_kernel(const ScanArgs p) {
    using Tin = typename Cfg::Tin;
    using Tout = typename Cfg::Tout;
    constexpr int NP = Cfg::NP, Q = Cfg::Q, CH = Cfg::CH, T = Cfg::T, TQ = Cfg::TQ;
    constexpr int NT = Cfg::NTHREADS, NS = Cfg::NSTAGE;
    constexpr int NG = T / 4;            // scan groups of 4 tokens per tile
    constexpr int SPG = TQ / NG;         // slice tokens handled per scan group
    extern __shared__ __align__(16) unsigned char smem[];

    const int tid = threadIdx.x;
    const int q = tid >> 5, c = tid & 31;          // warp = state quad, lane = channel
    const int b = blockIdx.x / p.groups_per_seq;
    const int d0 = (blockIdx.x - b * p.groups_per_seq) * CH;
    const int L = p.seqlen, N = p.dstate, dim = p.dim;
    const int nch = min(CH, dim - d0);
    const bool cvalid = c < nch;
    const size_t row0 = (size_t(b) * dim + d0) * size_t(L);
    const size_t bc0 = size_t(b) * L * size_t(N);
    const int ntiles = (L + T - 1) / T;
    const int s0 = q * TQ;                          // first token of this warp's slice

    auto prep_buf = [&](int i) { return reinterpret_cast<float4 *>(smem + Cfg::OFF_PREP + (i & 1) * Cfg::PREP_BYTES); };
    auto bf_buf = [&](int i) { return reinterpret_cast<float *>(smem + Cfg::OFF_BF + (i & 1) * Cfg::BC_BYTES); };
    auto cf_buf = [&](int i) { return reinterpret_cast<float *>(smem + Cfg::OFF_CF + (i & 1) * Cfg::BC_BYTES); };
    auto yp_buf = [&](int i) { return reinterpret_cast<float *>(smem + Cfg::OFF_YP + (i & 1) * Cfg::YP_BYTES); };
    auto y_buf = [&](int i) { return reinterpret_cast<Tout *>(smem + Cfg::OFF_Y + (i & 1) * Cfg::Y_BYTES); };

    float A2[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const int n = 4 * q + s;
        A2[s] = (cvalid && n < N) ? p.A[size_t(d0 + c) * N + n] * kLog2e : 0.f;
    }
    const float bias = (p.delta_bias != nullptr && cvalid) ? p.delta_bias[d0 + c] : 0.f;
    const float Dd = (p.D != nullptr && cvalid) ? p.D[d0 + c] : 0.f;
    const bool hasz = p.z != nullptr;

    // prep (Delta, Delta*x) of this warp's slice of tile `it`, from its staged raw data
    auto prep_slice = [&](int it, float (&dr)[TQ], float (&xr)[TQ]) {
        Stage<Cfg> sv(smem, it % NS);
#pragma unroll
        for (int k = 0; k < TQ / 4; ++k) {
            float a4[4], x4[4];
            load4s<Tin>(sv.ds + c * Cfg::RAW_ROW + s0 + 4 * k, a4);
            load4s<Tin>(sv.xs + c * Cfg::RAW_ROW + s0 + 4 * k, x4);
#pragma unroll
            for (int u = 0; u < 4; ++u) { dr[4 * k + u] = a4[u] + bias; xr[4 * k + u] = x4[u]; }
        }
    };
    auto prep_finish = [&](float v, float x, int tg) {   // -> (Delta, Delta*x), zero past L / dim
        const float dl = p.softplus ? softplus_f(v) : v;
        const bool ok = cvalid && tg < L;
        return make_float2(ok ? dl : 0.f, ok ? dl * x : 0.f);
    };
    auto prep_store = [&](int it, const float2 (&pv)[TQ]) {
        float4 *pp = prep_buf(it);
#pragma unroll
        for (int k = 0; k < TQ / 2; ++k)
            pp[((s0 >> 1) + k) * CH + c] = make_float4(pv[2 * k].x, pv[2 * k].y, pv[2 * k + 1].x, pv[2 * k + 1].y);
    };
    auto widen_bc = [&](int it) {          // B, C of tile `it` to fp32, zero past dstate / L
        Stage<Cfg> sv(smem, it % NS);
        float *Bf = bf_buf(it);
        float *Cf = cf_buf(it);
        const int t0 = it * T;
        if (N == NP && t0 + T <= L) {
            constexpr int NV = T * NP / 8;
#pragma unroll
            for (int k = 0; k < (2 * NV + NT - 1) / NT; ++k) {
                const int i = tid + k * NT;
                if (i < 2 * NV) {
                    const int which = i / NV, v = i % NV;
                    float f[8];
                    load8<Tin>((which ? sv.cs : sv.bs) + 8 * v, f);
                    store8<float>((which ? Cf : Bf) + 8 * v, f);
                }
            }
        } else {
            for (int i = tid; i < T * NP; i += NT) {
                const int tt = i / NP, n = i % NP;
                const bool ok = n < N && t0 + tt < L;
                Bf[i] = ok ? to_f32(sv.bs[tt * N + n]) : 0.f;
                Cf[i] = ok ? to_f32(sv.cs[tt * N + n]) : 0.f;
            }
        }
    };
    auto copy_out = [&](int it) {          // y of tile `it`: staged rows -> global, 16 B stores
        const Tout *ys = y_buf(it);
        Tout *gy = static_cast<Tout *>(p.y) + row0;
        const int t0 = it * T;
        if constexpr (Cfg::VEC) {
            constexpr int CPR = T / Cfg::EOUT;
#pragma unroll
            for (int k = 0; k < (CH * CPR + NT - 1) / NT; ++k) {
                const int i = tid + k * NT;
                const int cc = i / CPR, qq = i % CPR;
                const int tg = t0 + qq * Cfg::EOUT;
                if (i < CH * CPR && cc < nch && tg < L)
                    *reinterpret_cast<uint4 *>(gy + size_t(cc) * L + tg) =
                        *reinterpret_cast<const uint4 *>(ys + cc * Cfg::Y_ROW + qq * Cfg::EOUT);
            }
        } else {
            for (int i = tid; i < nch * T; i += NT) {
                const int cc = i / T, tt = i % T;
                if (t0 + tt < L) gy[size_t(cc) * L + t0 + tt] = ys[cc * Cfg::Y_ROW + tt];
            }
        }
    };

    // ---- prologue: stage tiles 0..2, prep and widen tile 0 ----
#pragma unroll
    for (int s = 0; s < 3; ++s) {
        if (s < ntiles) ws_load_tile<Cfg>(p, smem, s, s * T, row0, bc0, nch, tid);
        cp_async_commit();
    }
    cp_async_wait<2>();
    __syncthreads();
    if (ntiles > 0) {
        float dr[TQ], xr[TQ];
        float2 pv[TQ];
        prep_slice(0, dr, xr);
#pragma unroll
        for (int u = 0; u < TQ; ++u) pv[u] = prep_finish(dr[u], xr[u], s0 + u);
        prep_store(0, pv);
        widen_bc(0);
    }
    cp_async_wait<1>();
    __syncthreads();

    float h[4] = {0.f, 0.f, 0.f, 0.f};

    for (int i = 0; i <= ntiles + 1; ++i) {
        const bool do_scan = i < ntiles;
        const bool do_prep = i + 1 < ntiles;
        const bool do_epi = i >= 1 && i <= ntiles;
        if (i >= 2) copy_out(i - 2);
        // stage tile i+3 into the slot tile i-2 left (its epilogue ran in tile i-1)
        if (i + 3 < ntiles) ws_load_tile<Cfg>(p, smem, (i + 3) % NS, (i + 3) * T, row0, bc0, nch, tid);
        cp_async_commit();

        // inputs of this warp's slices: prep of tile i+1, output of tile i-1
        float dr[TQ], xr[TQ];
        float ysum[TQ], xe[TQ], ze[TQ];
        if (do_prep) prep_slice(i + 1, dr, xr);
        if (do_epi) {
            Stage<Cfg> sv(smem, (i - 1) % NS);
            const float *yp = yp_buf(i - 1);
#pragma unroll
            for (int k = 0; k < TQ / 4; ++k) {
                float4 acc = *reinterpret_cast<const float4 *>(yp + c * Cfg::YP_ROW + s0 + 4 * k);
#pragma unroll
                for (int qq = 1; qq < Q; ++qq) {
                    const float4 v = *reinterpret_cast<const float4 *>(yp + (qq * CH + c) * Cfg::YP_ROW + s0 + 4 * k);
                    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
                }
                ysum[4 * k] = acc.x; ysum[4 * k + 1] = acc.y; ysum[4 * k + 2] = acc.z; ysum[4 * k + 3] = acc.w;
                float x4[4], z4[4];
                load4s<Tin>(sv.xs + c * Cfg::RAW_ROW + s0 + 4 * k, x4);
                if (hasz) load4s<Tin>(sv.zs + c * Cfg::RAW_ROW + s0 + 4 * k, z4);
#pragma unroll
                for (int u = 0; u < 4; ++u) { xe[4 * k + u] = x4[u]; ze[4 * k + u] = hasz ? z4[u] : 0.f; }
            }
        }

        float2 pv[TQ];
        float yo[TQ];
        if (do_scan) {
            const float4 *pp = prep_buf(i) + c;
            const float *Bf = bf_buf(i);
            const float *Cf = cf_buf(i);
            float *ypr = yp_buf(i) + (q * CH + c) * Cfg::YP_ROW;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                const float4 d01 = pp[(2 * g) * CH];
                const float4 d23 = pp[(2 * g + 1) * CH];
                const float dl[4] = {d01.x, d01.z, d23.x, d23.z};
                const float dx[4] = {d01.y, d01.w, d23.y, d23.w};
                float a[4][4], w[4][4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 bq = *reinterpret_cast<const float4 *>(Bf + (4 * g + u) * NP + 4 * q);
                    const float bb[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        a[u][s] = ex2_approx(dl[u] * A2[s]);
                        w[u][s] = dx[u] * bb[s];
                    }
                }
                // interleaved per-(t, d) work of the slices
#pragma unroll
                for (int v = 0; v < SPG; ++v) {
                    const int u = g * SPG + v;
                    if (do_prep) pv[u] = prep_finish(dr[u], xr[u], (i + 1) * T + s0 + u);
                    if (do_epi) {
                        float y = fmaf(Dd, xe[u], ysum[u]);
                        if (hasz) y *= silu_f(ze[u]);
                        yo[u] = y;
                    }
                }
                float out[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 cq = *reinterpret_cast<const float4 *>(Cf + (4 * g + u) * NP + 4 * q);
                    const float cc4[4] = {cq.x, cq.y, cq.z, cq.w};
                    float acc = 0.f;
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        h[s] = fmaf(a[u][s], h[s], w[u][s]);
                        acc = fmaf(cc4[s], h[s], acc);
                    }
                    out[u] = acc;
                }
                *reinterpret_cast<float4 *>(ypr + 4 * g) = make_float4(out[0], out[1], out[2], out[3]);
            }
        } else {
#pragma unroll
            for (int u = 0; u < TQ; ++u) {
                if (do_prep) pv[u] = prep_finish(dr[u], xr[u], (i + 1) * T + s0 + u);
                if (do_epi) {
                    float y = fmaf(Dd, xe[u], ysum[u]);
                    if (hasz) y *= silu_f(ze[u]);
                    yo[u] = y;
                }
            }
        }
        if (do_prep) {
            prep_store(i + 1, pv);
            widen_bc(i + 1);
        }
        if (do_epi) {
            Tout *ys = y_buf(i - 1) + c * Cfg::Y_ROW + s0;
#pragma unroll
            for (int k = 0; k < TQ / 4; ++k) {
                const float y4[4] = {yo[4 * k], yo[4 * k + 1], yo[4 * k + 2], yo[4 * k + 3]};
                store4s<Tout>(ys + 4 * k, y4);
            }
        }
        cp_async_wait<1>();     // tile i+2 has landed (i+3 may be in flight)
        __syncthreads();
    }
    cp_async_wait<0>();

    if (p.final_state != nullptr && cvalid) {
        float *fs = p.final_state + (size_t(b) * dim + d0 + c) * N;
#pragma unroll
        for (int s = 0; s < 4; ++s)
            if (4 * q + s < N) fs[4 * q + s] = h[s];
    }
}

}  // namespace ssm
