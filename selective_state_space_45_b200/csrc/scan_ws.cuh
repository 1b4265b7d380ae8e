// scan_ws.cuh -- selective scan forward, warp-specialised (many-channel inputs).
//
// Same computation as scan_fwd.cuh (sources there).  One CTA owns 32 channels of one
// sequence for the whole length L; the state is carried in registers from the first
// token to the last.  Two kinds of warps share the CTA:
//
//   scan warps (Q = NP/4 of them): warp q holds states 4q..4q+3 of the 32 channels, one
//     channel per lane, and does nothing but the recurrence and its readout:
//       a = 2^(Delta*A*log2 e) (SFU), h = a*h + (Delta*x)*B, part = sum_s C*h.
//     B_t and C_t of a state quad are warp-uniform: one broadcast shared load each.
//   helper warps (NH of them): stage x, delta, z, B, C with cp.async, compute the
//     softplus step and Delta*x once per (t, d) for tile i+1, widen B and C to fp32,
//     and finish tile i-1 (sum of the quads' partial readouts, skip D*x, SiLU gate,
//     conversion, coalesced store of y) while the scan warps work on tile i.
//
// Hand-off between the two groups uses double-buffered shared tiles and named hardware
// barriers (bar.arrive by the producing group, bar.sync by the consuming group):
//   PREP_FULL[b]  helpers -> scans   prep/B/C of a tile in buffer b are ready
//   PREP_EMPTY[b] scans -> helpers   the scans are done reading buffer b
//   YP_FULL[b]    scans -> helpers   partial readouts of a tile in buffer b are ready
//   YP_EMPTY[b]   helpers -> scans   the helpers are done reading buffer b
// Every arrive is matched by exactly one sync of the same barrier; arrivals that no later
// tile would consume are skipped, so no barrier is left half-arrived at exit.
#pragma once

#include "common.cuh"
#include "scan_fwd.cuh"   // ScanArgs

namespace ssm {

__device__ __forceinline__ void bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void bar_arrive(int id, int nthreads) {
    asm volatile("bar.arrive %0, %1;\n" ::"r"(id), "r"(nthreads) : "memory");
}

// 4 consecutive values of a staged row (8-byte aligned for bf16, 16 for fp32) as fp32.
template <typename T> __device__ __forceinline__ void load4s(const T *src, float (&v)[4]);
template <> __device__ __forceinline__ void load4s<float>(const float *src, float (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4 *>(src);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <> __device__ __forceinline__ void load4s<__nv_bfloat16>(const __nv_bfloat16 *src, float (&v)[4]) {
    const uint2 u = *reinterpret_cast<const uint2 *>(src);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xffff0000u);
}
template <typename T> __device__ __forceinline__ void store4s(T *dst, const float (&v)[4]);
template <> __device__ __forceinline__ void store4s<float>(float *dst, const float (&v)[4]) {
    *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
}
template <> __device__ __forceinline__ void store4s<__nv_bfloat16>(__nv_bfloat16 *dst, const float (&v)[4]) {
    const __nv_bfloat162 p0 = __floats2bfloat162_rn(v[0], v[1]);
    const __nv_bfloat162 p1 = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2 *>(dst) =
        make_uint2(*reinterpret_cast<const unsigned *>(&p0), *reinterpret_cast<const unsigned *>(&p1));
}

template <int NP_, int NH_, int T_, typename Tin_, typename Tout_, bool VEC_, int MINB_>
struct WsCfg {
    using Tin = Tin_;
    using Tout = Tout_;
    static constexpr int NP = NP_;            // padded state width (multiple of 4)
    static constexpr int Q = NP / 4;          // scan warps
    static constexpr int NH = NH_;            // helper warps
    static constexpr int CH = 32;             // channels per CTA (one per lane)
    static constexpr int T = T_;              // tokens per tile
    static constexpr int NSTAGE = 3;          // raw staging ring (tiles)
    static constexpr bool VEC = VEC_;
    static constexpr int MINB = MINB_;
    static constexpr int NSCAN_T = 32 * Q;    // scan threads
    static constexpr int NHELP_T = 32 * NH;   // helper threads
    static constexpr int NTHREADS = NSCAN_T + NHELP_T;
    static constexpr int ALL_T = NTHREADS;
    static constexpr int EIN = 16 / sizeof(Tin);
    static constexpr int EOUT = 16 / sizeof(Tout);
    static constexpr int TT = 4;                       // tokens per helper task
    static constexpr int NTASK = CH * (T / TT);        // helper tasks per tile
    static constexpr int TASKS_PER_THREAD = NTASK / NHELP_T;
    static constexpr int RAW_ROW = T + EIN;            // row stride: 16 B past a multiple of 16
    static constexpr int Y_ROW = T + EOUT;
    static constexpr int YP_ROW = T + 4;               // floats
    static_assert(T % 8 == 0 && T % TT == 0, "tile shape");
    static_assert(NTASK % NHELP_T == 0 && TASKS_PER_THREAD >= 1, "helper tasks must divide evenly");

    static constexpr size_t al(size_t v) { return (v + 127) & ~size_t(127); }
    static constexpr size_t RAW_ARR = al(size_t(CH) * RAW_ROW * sizeof(Tin));
    static constexpr size_t RAW_BC = al(size_t(T) * NP * sizeof(Tin));
    static constexpr size_t STAGE_BYTES = 3 * RAW_ARR + 2 * RAW_BC;
    static constexpr size_t OFF_RAW = 0;
    static constexpr size_t PREP_BYTES = al(size_t(T / 2) * CH * sizeof(float4));
    static constexpr size_t BC_BYTES = al(size_t(T) * NP * sizeof(float));
    static constexpr size_t YP_BYTES = al(size_t(Q) * CH * YP_ROW * sizeof(float));
    static constexpr size_t OFF_PREP = OFF_RAW + NSTAGE * STAGE_BYTES;      // x2 buffers
    static constexpr size_t OFF_BF = OFF_PREP + 2 * PREP_BYTES;             // x2
    static constexpr size_t OFF_CF = OFF_BF + 2 * BC_BYTES;                 // x2
    static constexpr size_t OFF_YP = OFF_CF + 2 * BC_BYTES;                 // x2
    static constexpr size_t OFF_Y = OFF_YP + 2 * YP_BYTES;
    static constexpr size_t SMEM_BYTES = OFF_Y + al(size_t(CH) * Y_ROW * sizeof(Tout));

    // named barrier ids (0 is __syncthreads)
    static constexpr int BAR_HELP = 1;
    static constexpr int BAR_PREP_FULL = 2;    // + buffer
    static constexpr int BAR_PREP_EMPTY = 4;   // + buffer
    static constexpr int BAR_YP_FULL = 6;      // + buffer
    static constexpr int BAR_YP_EMPTY = 8;     // + buffer
};

// Helpers stage tile [t0, t0 + T) into ring stage st (ht: helper thread index).  VEC:
// 16-byte cp.async chunks, each wholly inside or outside [0, L) (L is a multiple of the
// chunk width); otherwise guarded scalar loads.
template <class Cfg>
__device__ __forceinline__ void ws_load_tile(const ScanArgs &p, unsigned char *smem, int st, int t0,
                                             size_t row0, size_t bc0, int nch, int ht) {
    using Tin = typename Cfg::Tin;
    constexpr int CH = Cfg::CH, T = Cfg::T, NH = Cfg::NHELP_T, EIN = Cfg::EIN, NP = Cfg::NP;
    Stage<Cfg> s(smem, st);
    const int L = p.seqlen, N = p.dstate;
    const Tin *gx = static_cast<const Tin *>(p.x) + row0;
    const Tin *gd = static_cast<const Tin *>(p.delta) + row0;
    const Tin *gz = p.z ? static_cast<const Tin *>(p.z) + row0 : gx;
    const int narr = p.z ? 3 : 2;
    const Tin *gb = static_cast<const Tin *>(p.B) + bc0 + size_t(t0) * N;
    const Tin *gc = static_cast<const Tin *>(p.C) + bc0 + size_t(t0) * N;
    if constexpr (Cfg::VEC) {
        constexpr int CPR = T / EIN;
        constexpr int ROWC = 3 * CH * CPR;
#pragma unroll
        for (int k = 0; k < (ROWC + NH - 1) / NH; ++k) {
            const int i = ht + k * NH;
            const int a = i / (CH * CPR);
            const int rem = i % (CH * CPR);
            const int cc = rem / CPR, q = rem % CPR;
            if (i < ROWC && a < narr && cc < nch && t0 + q * EIN < L) {
                const Tin *src = (a == 0 ? gx : a == 1 ? gd : gz) + size_t(cc) * L + t0 + q * EIN;
                Tin *dst = (a == 0 ? s.xs : a == 1 ? s.ds : s.zs) + cc * Cfg::RAW_ROW + q * EIN;
                cp_async_16(dst, src);
            }
        }
        if (N == NP) {
            constexpr int BCC = T * NP / EIN;          // 16-byte chunks per array
#pragma unroll
            for (int k = 0; k < (2 * BCC + NH - 1) / NH; ++k) {
                const int i = ht + k * NH;
                const int which = i / BCC, q = i % BCC;
                if (i < 2 * BCC && t0 + (q * EIN) / NP < L)
                    cp_async_16((which ? s.cs : s.bs) + q * EIN, (which ? gc : gb) + q * EIN);
            }
        } else {
            const int valid_t = min(T, L - t0);
            const int bc_chunks = (valid_t * N * int(sizeof(Tin))) / 16;
            for (int i = ht; i < 2 * bc_chunks; i += NH) {
                const int which = i >= bc_chunks;
                const int q = i - which * bc_chunks;
                cp_async_16((which ? s.cs : s.bs) + q * EIN, (which ? gc : gb) + q * EIN);
            }
        }
    } else {
        constexpr int NEL = 3 * CH * T;
#pragma unroll 4
        for (int k = 0; k < (NEL + NH - 1) / NH; ++k) {
            const int i = ht + k * NH;
            const int a = i / (CH * T);
            const int rem = i % (CH * T);
            const int cc = rem / T, tt = rem % T;
            if (i < NEL && a < narr && cc < nch && t0 + tt < L) {
                const Tin *src = (a == 0 ? gx : a == 1 ? gd : gz) + size_t(cc) * L + t0 + tt;
                Tin *dst = (a == 0 ? s.xs : a == 1 ? s.ds : s.zs) + cc * Cfg::RAW_ROW + tt;
                *dst = *src;
            }
        }
        const int nbc = min(T, L - t0) * N;
        for (int i = ht; i < 2 * nbc; i += NH) {
            const int which = i >= nbc;
            const int q = i - which * nbc;
            (which ? s.cs : s.bs)[q] = (which ? gc : gb)[q];
        }
    }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::NTHREADS, Cfg::MINB)
scan_ws_kernel(const ScanArgs p) {
    using Tin = typename Cfg::Tin;
    using Tout = typename Cfg::Tout;
    constexpr int NP = Cfg::NP, Q = Cfg::Q, CH = Cfg::CH, T = Cfg::T, ALL = Cfg::ALL_T;
    constexpr int NHT = Cfg::NHELP_T, TT = Cfg::TT;
    extern __shared__ __align__(16) unsigned char smem[];

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x / p.groups_per_seq;
    const int d0 = (blockIdx.x - b * p.groups_per_seq) * CH;
    const int L = p.seqlen, N = p.dstate, dim = p.dim;
    const int nch = min(CH, dim - d0);
    const size_t row0 = (size_t(b) * dim + d0) * size_t(L);
    const size_t bc0 = size_t(b) * L * size_t(N);
    const int ntiles = (L + T - 1) / T;

    auto prep_buf = [&](int buf) {
        return reinterpret_cast<float4 *>(smem + Cfg::OFF_PREP + buf * Cfg::PREP_BYTES);
    };
    auto bf_buf = [&](int buf) { return reinterpret_cast<float *>(smem + Cfg::OFF_BF + buf * Cfg::BC_BYTES); };
    auto cf_buf = [&](int buf) { return reinterpret_cast<float *>(smem + Cfg::OFF_CF + buf * Cfg::BC_BYTES); };
    auto yp_buf = [&](int buf) { return reinterpret_cast<float *>(smem + Cfg::OFF_YP + buf * Cfg::YP_BYTES); };

    if (warp < Q) {
        // ================= scan warp: states 4q..4q+3 of channel `lane` =================
        const int q = warp, c = lane;
        const bool dvalid = c < nch;
        float A2[4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int n = 4 * q + s;
            A2[s] = (dvalid && n < N) ? p.A[size_t(d0 + c) * N + n] * kLog2e : 0.f;
        }
        float h[4] = {0.f, 0.f, 0.f, 0.f};
        for (int tile = 0; tile < ntiles; ++tile) {
            const int buf = tile & 1;
            bar_sync(Cfg::BAR_PREP_FULL + buf, ALL);
            if (tile >= 2) bar_sync(Cfg::BAR_YP_EMPTY + buf, ALL);
            const float4 *pp = prep_buf(buf) + c;
            const float *Bf = bf_buf(buf);
            const float *Cf = cf_buf(buf);
            float *ypr = yp_buf(buf) + (q * CH + c) * Cfg::YP_ROW;
#pragma unroll
            for (int g = 0; g < T / 4; ++g) {
                const float4 d01 = pp[(2 * g) * CH];      // (Delta, Delta*x) of tokens 4g, 4g+1
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
            __threadfence_block();
            if (tile + 2 < ntiles) bar_arrive(Cfg::BAR_PREP_EMPTY + buf, ALL);
            bar_arrive(Cfg::BAR_YP_FULL + buf, ALL);
        }
        if (p.final_state != nullptr && dvalid) {
            float *fs = p.final_state + (size_t(b) * dim + d0 + c) * N;
#pragma unroll
            for (int s = 0; s < 4; ++s)
                if (4 * q + s < N) fs[4 * q + s] = h[s];
        }
        return;
    }

    // ================= helper warps =================
    const int ht = tid - Cfg::NSCAN_T;
    float tbias[Cfg::TASKS_PER_THREAD], tD[Cfg::TASKS_PER_THREAD];
#pragma unroll
    for (int k = 0; k < Cfg::TASKS_PER_THREAD; ++k) {
        const int cc = (ht + k * NHT) % CH;
        tbias[k] = (p.delta_bias != nullptr && cc < nch) ? p.delta_bias[d0 + cc] : 0.f;
        tD[k] = (p.D != nullptr && cc < nch) ? p.D[d0 + cc] : 0.f;
    }
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        if (s < ntiles) ws_load_tile<Cfg>(p, smem, s, s * T, row0, bc0, nch, ht);
        cp_async_commit();
    }
    Tout *ys = reinterpret_cast<Tout *>(smem + Cfg::OFF_Y);
    Tout *gy = static_cast<Tout *>(p.y) + row0;

    for (int tile = 0; tile <= ntiles; ++tile) {
        if (tile < ntiles) {
            // ---- prep of this tile into buffer tile & 1 ----
            const int buf = tile & 1;
            const int t0 = tile * T;
            if (tile >= 2) bar_sync(Cfg::BAR_PREP_EMPTY + buf, ALL);
            cp_async_wait<1>();
            bar_sync(Cfg::BAR_HELP, NHT);
            Stage<Cfg> sv(smem, tile % Cfg::NSTAGE);
            float4 *prep = prep_buf(buf);
#pragma unroll
            for (int k = 0; k < Cfg::TASKS_PER_THREAD; ++k) {
                const int task = ht + k * NHT;
                const int cc = task % CH, t4 = task / CH;
                float dr[4], xr[4];
                load4s<Tin>(sv.ds + cc * Cfg::RAW_ROW + TT * t4, dr);
                load4s<Tin>(sv.xs + cc * Cfg::RAW_ROW + TT * t4, xr);
                float o[8];
                const bool full = cc < nch && t0 + TT * t4 + TT <= L;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float dl = dr[u] + tbias[k];
                    if (p.softplus) dl = softplus_f(dl);
                    const bool ok = full || (cc < nch && t0 + TT * t4 + u < L);   // else a no-op token
                    o[2 * u] = ok ? dl : 0.f;
                    o[2 * u + 1] = ok ? dl * xr[u] : 0.f;
                }
                prep[(2 * t4) * CH + cc] = make_float4(o[0], o[1], o[2], o[3]);
                prep[(2 * t4 + 1) * CH + cc] = make_float4(o[4], o[5], o[6], o[7]);
            }
            float *Bf = bf_buf(buf);
            float *Cf = cf_buf(buf);
            if (N == NP && t0 + T <= L) {
                constexpr int NV = T * NP / 8;
#pragma unroll
                for (int k = 0; k < (2 * NV + NHT - 1) / NHT; ++k) {
                    const int i = ht + k * NHT;
                    if (i < 2 * NV) {
                        const int which = i / NV, v = i % NV;
                        float f[8];
                        load8<Tin>((which ? sv.cs : sv.bs) + 8 * v, f);
                        store8<float>((which ? Cf : Bf) + 8 * v, f);
                    }
                }
            } else {
                for (int i = ht; i < T * NP; i += NHT) {
                    const int tt = i / NP, n = i % NP;
                    const bool ok = n < N && t0 + tt < L;
                    Bf[i] = ok ? to_f32(sv.bs[tt * N + n]) : 0.f;
                    Cf[i] = ok ? to_f32(sv.cs[tt * N + n]) : 0.f;
                }
            }
            __threadfence_block();
            bar_arrive(Cfg::BAR_PREP_FULL + buf, ALL);
        }
        if (tile >= 1) {
            // ---- finish the previous tile: sum quads, skip, gate, convert, store ----
            const int pt = tile - 1, pb = pt & 1;
            const int t0 = pt * T;
            bar_sync(Cfg::BAR_YP_FULL + pb, ALL);
            Stage<Cfg> sv(smem, pt % Cfg::NSTAGE);
            const float *yp = yp_buf(pb);
#pragma unroll
            for (int k = 0; k < Cfg::TASKS_PER_THREAD; ++k) {
                const int task = ht + k * NHT;
                const int cc = task % CH, t4 = task / CH;
                float acc[4];
                {
                    const float4 v = *reinterpret_cast<const float4 *>(yp + cc * Cfg::YP_ROW + TT * t4);
                    acc[0] = v.x; acc[1] = v.y; acc[2] = v.z; acc[3] = v.w;
                }
#pragma unroll
                for (int qq = 1; qq < Q; ++qq) {
                    const float4 v = *reinterpret_cast<const float4 *>(yp + (qq * CH + cc) * Cfg::YP_ROW + TT * t4);
                    acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
                }
                float xr[4];
                load4s<Tin>(sv.xs + cc * Cfg::RAW_ROW + TT * t4, xr);
#pragma unroll
                for (int u = 0; u < 4; ++u) acc[u] = fmaf(tD[k], xr[u], acc[u]);
                if (p.z != nullptr) {
                    float zr[4];
                    load4s<Tin>(sv.zs + cc * Cfg::RAW_ROW + TT * t4, zr);
#pragma unroll
                    for (int u = 0; u < 4; ++u) acc[u] *= silu_f(zr[u]);
                }
                store4s<Tout>(ys + cc * Cfg::Y_ROW + TT * t4, acc);
            }
            bar_sync(Cfg::BAR_HELP, NHT);                // ys complete, stage pt%3 fully read
            if (pt + 2 < ntiles) bar_arrive(Cfg::BAR_YP_EMPTY + pb, ALL);
            if constexpr (Cfg::VEC) {
                constexpr int CPR = T / Cfg::EOUT;
#pragma unroll
                for (int k = 0; k < (CH * CPR + NHT - 1) / NHT; ++k) {
                    const int i = ht + k * NHT;
                    const int cc = i / CPR, qq = i % CPR;
                    const int tg = t0 + qq * Cfg::EOUT;
                    if (i < CH * CPR && cc < nch && tg < L)
                        *reinterpret_cast<uint4 *>(gy + size_t(cc) * L + tg) =
                            *reinterpret_cast<const uint4 *>(ys + cc * Cfg::Y_ROW + qq * Cfg::EOUT);
                }
            } else {
                for (int i = ht; i < nch * T; i += NHT) {
                    const int cc = i / T, tt = i % T;
                    if (t0 + tt < L) gy[size_t(cc) * L + t0 + tt] = ys[cc * Cfg::Y_ROW + tt];
                }
            }
        }
        if (tile < ntiles) {
            // refill the stage whose tile (tile - 1) was just finished
            if (tile + 2 < ntiles)
                ws_load_tile<Cfg>(p, smem, (tile + 2) % Cfg::NSTAGE, (tile + 2) * T, row0, bc0, nch, ht);
            cp_async_commit();
        }
    }
    cp_async_wait<0>();
}

}  // namespace ssm
