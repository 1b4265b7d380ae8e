// scan_fwd.cuh -- the selective scan (S6) forward kernel for sm_100a.
//
// What it computes, per sequence b, channel d, state n and token t:
//   Delta = softplus(delta[b,d,t] + bias[d])            (bias and softplus optional)
//   h_n  <- exp(Delta * A[d,n]) * h_n + Delta * B[b,t,n] * x[b,d,t]
//   y     = (sum_n C[b,t,n] * h_n + D[d] * x[b,d,t]) * SiLU(z[b,d,t])
// Sources: zero-order-hold decay and its Euler input gain ("Module 19: State-Space Models
// (Mamba)", learnllm, "The Math: The State-Space Recurrence"); input-dependent Delta, B, C,
// the softplus step, the skip and the gate ("Beyond attention with Mamba, state space
// models and hybrids", xmarva lesson 10, sections 3 and 4); the N-expanded states never
// reach main memory (same lesson, section 6); composing affine steps
// (a2, b2) o (a1, b1) = (a2 a1, a2 b1 + b2) ("Module 19", "The Parallel Scan").
//
// Layout of the work
//   * A CTA owns CH = 32*CG channels of one sequence and walks a token range in T-token
//     tiles.  Warp (cg, q) holds states 4q..4q+3 of the 32 channels of channel group cg,
//     one channel per lane, in registers for the whole range.  B_t and C_t of a state quad
//     are the same for every lane: one broadcast shared load each per token.  The quads
//     of a channel live in different warps; their readouts are summed once per (t, d)
//     after the tile through a shared buffer, not by shuffles inside the recurrence.
//   * Per (t, d) work -- the softplus step before the scan (prep), the skip, gate and
//     output conversion after it (epilogue) -- is done once per (t, d) by tasks of 8
//     tokens of one channel with 16-byte, bank-conflict-free shared accesses, on packed
//     FP32 pairs.  Each warp forms Delta*x itself from the staged x, and reads B_t and
//     C_t as fp32 quads widened once per tile.
//   * The decays and writes of the next 4 tokens are computed before the recurrence of
//     the current 4, so SFU work overlaps the FFMA chain.
//   * x, delta, z, B, C are staged by a cp.async ring of NSTAGE tiles (16-byte copies)
//     when every row is 16-byte aligned, else by guarded scalar loads; y leaves as 16-byte
//     stores of 8 tokens straight from the epilogue's registers.
//
// Long sequences with few channels are split into segments scanned by different CTAs.
// The scan is linear in its carry, so a segment's end state from a zero start is
//     h_end[n] = sum_t exp(A_n R_t) * Delta_t B_t[n] x_t,   R_t = sum of the steps after t
// and only the tokens whose decay exp(A_n R_t) is not yet 0 in fp32 enter it:
//   tail    every segment but the last sums h_end over its last tokens, walking back from
//           its end until every state's decay has flushed to 0, and records its step sum S
//           (or +inf once the decay over the whole segment is certain to be 0)
//           (scan_tail_kernel);
//   fold    the end states are folded in order into each segment's true carry
//           h <- exp(A*S) h + h_end, from the start state (scan_fold_kernel);
//   scan    every segment is scanned once from its true carry, writing y, the last one
//           also the final state (scan_fwd_kernel with SEG).
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
    int zoh;              // host side: exact zero-order-hold gain requested
    int groups_per_seq;   // ceil(dim / CH)
    // segmented scan (long sequences): nseg segments of seg_len tokens
    int nseg;
    int seg_len;          // tokens per segment, a multiple of the tile
    float *seg_h;         // [batch*dim][nseg][NP] tail sums h_end, carries after the fold
    float *seg_s;         // [batch*dim][nseg] step sums of the segments (+inf: decay is 0)
    const float *h0;      // [batch][dim][dstate] start state, or null for zero
};

template <int NP_, int CG_, int T_, int NSTAGE_, typename Tin_, typename Tout_, bool VEC_, int MINB_>
struct ScanCfg {
    using Tin = Tin_;
    using Tout = Tout_;
    static constexpr int NP = NP_;          // padded state width (4, 8 or 16)
    static constexpr int Q = NP / 4;        // state quads = warps per channel group
    static constexpr int CG = CG_;          // channel groups of 32 per CTA
    static constexpr int CH = 32 * CG;      // channels per CTA
    static constexpr int T = T_;            // tokens per tile
    static constexpr int NSTAGE = NSTAGE_;
    static constexpr bool VEC = VEC_;
    static constexpr int MINB = MINB_;
    static constexpr int NWARP = Q * CG;
    static constexpr int NTHREADS = 32 * NWARP;
    static constexpr int EIN = 16 / sizeof(Tin);
    static constexpr int T8 = T / 8;                  // 8-token chunks per tile row
    static constexpr int NTASK = CH * T8;             // per-(t, d) tasks per tile
    static constexpr int TASKS_PER_THREAD = (NTASK + NTHREADS - 1) / NTHREADS;
    // staged x, delta, z rows: CPR 16-byte chunks per channel, RPL rows to a 128-byte line;
    // chunk j of row cc sits in slot j XOR ((cc / RPL) mod CPR), so 16-byte reads of one
    // chunk column across 8 consecutive channels hit distinct banks without padding
    static constexpr int CPR = T / EIN;
    static constexpr int RPL = CPR >= 8 ? 1 : 8 / CPR;
    static_assert((CPR & (CPR - 1)) == 0 && T % 8 == 0, "staged rows: a power of two of 16-byte chunks");
    static constexpr int RAW_ROW = T;
    __host__ __device__ static constexpr int raw_at(int cc, int t) {
        return cc * RAW_ROW + (((t / EIN) ^ ((cc / RPL) & (CPR - 1))) * EIN) + t % EIN;
    }
    static constexpr int YP_SLOTS = T / 4;            // float4 slots of a partial-sum row
    static_assert(T % 8 == 0, "tile must hold whole 8-token chunks");
    static_assert(NTASK % NTHREADS == 0, "tasks must divide evenly");

    static constexpr size_t al(size_t v) { return (v + 15) & ~size_t(15); }
    static constexpr size_t RAW_ARR = al(size_t(CH) * RAW_ROW * sizeof(Tin));
    static constexpr size_t RAW_BC = al(size_t(T) * NP * sizeof(Tin));
    static constexpr size_t STAGE_BYTES = 3 * RAW_ARR + 2 * RAW_BC;
    static constexpr size_t OFF_RAW = 0;
    // prep: Delta as fp32 rows [CH][T], 4-token slot g of channel c's row stored at
    // g XOR (c mod 8) as the partial rows are; the recurrence takes x from the staged rows
    static constexpr size_t OFF_PREP = OFF_RAW + NSTAGE * STAGE_BYTES;
    // B, C of the tile widened to fp32 rows [T][NP] once per tile, so that the recurrence
    // reads each state quad as one 16-byte broadcast (two shared-memory wavefronts for a
    // warp) and spends no instruction on widening
    static constexpr size_t BF_BYTES = al(size_t(T) * NP * sizeof(float));
    static constexpr size_t CF_BYTES = al(size_t(T) * NP * sizeof(float));
    static constexpr size_t OFF_BF = OFF_PREP + al(size_t(CH) * T * sizeof(float));
    static constexpr size_t OFF_CF = OFF_BF + BF_BYTES;
    // quad partial sums of the readout [Q][CH][T], slot g of a row stored at g XOR (channel
    // mod 8): the recurrence's 16-byte writes (lanes over channels) and the epilogue's reads
    // are conflict free without padding
    static constexpr size_t OFF_YP = OFF_CF + CF_BYTES;
    static constexpr size_t SMEM_BYTES = OFF_YP + al(size_t(Q) * CH * T * sizeof(float));
    static_assert(YP_SLOTS == 8, "the XOR swizzle of the partial rows assumes 8 slots");
};

// Views of one ring stage: x, delta, z as [CH][T] in swizzled 16-byte chunks (raw_at); B, C
// as [T][N] contiguous.
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

// Tokens 8 t8 .. 8 t8 + 7 of channel cc of a staged x, delta or z array, as fp32.
template <class Cfg>
__device__ __forceinline__ void stage_row8(const typename Cfg::Tin *arr, int cc, int t8, float (&v)[8]) {
    using Tin = typename Cfg::Tin;
    if constexpr (Cfg::EIN == 8) {
        load8<Tin>(arr + Cfg::raw_at(cc, 8 * t8), v);
    } else {
        float lo[4], hi[4];
        loadn<4, Tin>(arr + Cfg::raw_at(cc, 8 * t8), lo);
        loadn<4, Tin>(arr + Cfg::raw_at(cc, 8 * t8 + 4), hi);
#pragma unroll
        for (int u = 0; u < 4; ++u) { v[u] = lo[u]; v[4 + u] = hi[u]; }
    }
}

// Stage tile [t0, t0 + T) of x, delta, z (rows of nch channels) and of B, C into ring stage
// st, with every index split by compile-time divisors; thread `me` of the NT staging
// threads.  VEC: 16-byte cp.async chunks, each wholly inside or wholly outside [0, L)
// because L is a multiple of the chunk width.
template <class Cfg, int NT = Cfg::NTHREADS>
__device__ __forceinline__ void load_tile(const ScanArgs &p, unsigned char *smem, int st, int t0,
                                          size_t row0, size_t bc0, int nch, int me = tid_x()) {
    using Tin = typename Cfg::Tin;
    constexpr int CH = Cfg::CH, T = Cfg::T, EIN = Cfg::EIN, NP = Cfg::NP;
    Stage<Cfg> s(smem, st);
    const int L = p.seqlen, N = p.dstate;
    const Tin *gx = static_cast<const Tin *>(p.x) + row0;
    const Tin *gd = static_cast<const Tin *>(p.delta) + row0;
    const Tin *gz = p.z ? static_cast<const Tin *>(p.z) + row0 : gx;
    const int narr = p.z ? 3 : 2;
    const Tin *gb = static_cast<const Tin *>(p.B) + bc0 + size_t(t0) * N;
    const Tin *gc = static_cast<const Tin *>(p.C) + bc0 + size_t(t0) * N;
    if constexpr (Cfg::VEC) {
        constexpr int CPR = T / EIN;                 // 16-byte chunks per row
        constexpr int ROWC = 3 * CH * CPR;
#pragma unroll
        for (int k = 0; k < (ROWC + NT - 1) / NT; ++k) {
            const int i = me + k * NT;
            const int a = i / (CH * CPR);
            const int rem = i % (CH * CPR);
            const int cc = rem / CPR, q = rem % CPR;
            if (i < ROWC && a < narr && cc < nch && t0 + q * EIN < L) {
                const Tin *src = (a == 0 ? gx : a == 1 ? gd : gz) + size_t(cc) * L + t0 + q * EIN;
                Tin *dst = (a == 0 ? s.xs : a == 1 ? s.ds : s.zs) + Cfg::raw_at(cc, q * EIN);
                cp_async_16(dst, src);
            }
        }
        if (N == NP) {                               // dense B, C rows: T * NP values each
            constexpr int BCC = T * NP / EIN;        // chunks per array
#pragma unroll
            for (int k = 0; k < (2 * BCC + NT - 1) / NT; ++k) {
                const int i = me + k * NT;
                const int which = i / BCC, q = i % BCC;
                if (i < 2 * BCC && t0 + (q * EIN) / NP < L)   // first token of the chunk
                    cp_async_16((which ? s.cs : s.bs) + q * EIN, (which ? gc : gb) + q * EIN);
            }
        } else {
            const int valid_t = min(T, L - t0);
            const int bc_chunks = (valid_t * N * int(sizeof(Tin))) / 16;
            for (int i = me; i < 2 * bc_chunks; i += NT) {
                const int which = i >= bc_chunks;
                const int q = i - which * bc_chunks;
                cp_async_16((which ? s.cs : s.bs) + q * EIN, (which ? gc : gb) + q * EIN);
            }
        }
    } else {
        constexpr int NEL = 3 * CH * T;
#pragma unroll 4
        for (int k = 0; k < (NEL + NT - 1) / NT; ++k) {
            const int i = me + k * NT;
            const int a = i / (CH * T);
            const int rem = i % (CH * T);
            const int cc = rem / T, tt = rem % T;
            if (i < NEL && a < narr && cc < nch && t0 + tt < L) {
                const Tin *src = (a == 0 ? gx : a == 1 ? gd : gz) + size_t(cc) * L + t0 + tt;
                Tin *dst = (a == 0 ? s.xs : a == 1 ? s.ds : s.zs) + Cfg::raw_at(cc, tt);
                *dst = *src;
            }
        }
        const int nbc = min(T, L - t0) * N;
        for (int i = me; i < 2 * nbc; i += NT) {
            const int which = i >= nbc;
            const int q = i - which * nbc;
            (which ? s.cs : s.bs)[q] = (which ? gc : gb)[q];
        }
    }
}


// SEG: one segment of the segmented scan, from the folded carry into it (else the whole
// sequence from the start state).  ZOH: exact zero-order-hold
// input gain (exp(Delta a) - 1) / a * B instead of the Euler gain Delta * B.
template <class Cfg, bool SEG, bool ZOH>
__global__ void __launch_bounds__(Cfg::NTHREADS, Cfg::MINB)
scan_fwd_kernel(const ScanArgs p) {
    using Tin = typename Cfg::Tin;
    using Tout = typename Cfg::Tout;
    constexpr int NP = Cfg::NP, Q = Cfg::Q, CH = Cfg::CH, T = Cfg::T, NT = Cfg::NTHREADS;
    extern __shared__ __align__(16) unsigned char smem[];

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int cg = warp / Q;            // channel group of this warp
    const int q = warp - cg * Q;        // state quad of this warp
    const int c = cg * 32 + lane;       // channel within the CTA
    // CTA -> (sequence, channel group[, segment])
    int bg = blockIdx.x, seg = 0;
    if constexpr (SEG) {
        seg = bg % p.nseg;
        bg /= p.nseg;
    }
    const int b = bg / p.groups_per_seq;
    const int d0 = (bg - b * p.groups_per_seq) * CH;
    const int L = p.seqlen, N = p.dstate, dim = p.dim;
    const int nch = min(CH, dim - d0);
    const bool dvalid = c < nch;

    float4 *prep = reinterpret_cast<float4 *>(smem + Cfg::OFF_PREP);
    float *Bf = reinterpret_cast<float *>(smem + Cfg::OFF_BF);
    float *Cf = reinterpret_cast<float *>(smem + Cfg::OFF_CF);
    float *yp = reinterpret_cast<float *>(smem + Cfg::OFF_YP);

    // this lane's 4 states: A * log2(e)
    float A2[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const int n = 4 * q + s;
        A2[s] = (dvalid && n < N) ? p.A[size_t(d0 + c) * N + n] * kLog2e : 0.f;
    }
    // exact ZOH: 1 / a per state (0 where a = 0, whose gain is the limit Delta)
    float invA[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (ZOH) {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const float a = A2[s] * (1.f / kLog2e);
            invA[s] = a != 0.f ? 1.f / a : 0.f;
        }
    }
    // per chunk task: its channel is the same in every tile, so bias and D live in registers
    float tbias[Cfg::TASKS_PER_THREAD], tD[Cfg::TASKS_PER_THREAD];
#pragma unroll
    for (int k = 0; k < Cfg::TASKS_PER_THREAD; ++k) {
        const int cc = (tid + k * NT) % CH;
        tbias[k] = (p.delta_bias != nullptr && cc < nch) ? p.delta_bias[d0 + cc] : 0.f;
        tD[k] = (p.D != nullptr && cc < nch) ? p.D[d0 + cc] : 0.f;
    }

    const size_t row0 = (size_t(b) * dim + d0) * size_t(L);
    const size_t bc0 = size_t(b) * L * size_t(N);
    const size_t chrow = size_t(b) * dim + d0 + c;      // this lane's (sequence, channel) row
    const int tbeg = SEG ? seg * p.seg_len : 0;         // token range of this CTA
    const int tend = SEG ? min(L, tbeg + p.seg_len) : L;
    const int ntiles = (tend - tbeg + T - 1) / T;

#pragma unroll
    for (int s = 0; s < Cfg::NSTAGE - 1; ++s) {
        if (s < ntiles) load_tile<Cfg>(p, smem, s, tbeg + s * T, row0, bc0, nch);
        cp_async_commit();
    }

    float h[4] = {0.f, 0.f, 0.f, 0.f};
    if (SEG) {                              // the folded carry into the segment
        if (dvalid) {
            const float4 hv = *reinterpret_cast<const float4 *>(p.seg_h + (chrow * p.nseg + seg) * NP + 4 * q);
            h[0] = hv.x; h[1] = hv.y; h[2] = hv.z; h[3] = hv.w;
        }
    } else if (p.h0 != nullptr && dvalid) {
#pragma unroll
        for (int s = 0; s < 4; ++s)
            if (4 * q + s < N) h[s] = p.h0[chrow * N + 4 * q + s];
    }

    // the state in the recurrence: pairs (0,1), (2,3) for the packed FP32 instructions
    float2 hp[2] = {f2(h[0], h[1]), f2(h[2], h[3])};
    const float2 A2p[2] = {f2(A2[0], A2[1]), f2(A2[2], A2[3])};
    for (int tile = 0; tile < ntiles; ++tile) {
        const int st = tile % Cfg::NSTAGE;
        const int t0 = tbeg + tile * T;
        cp_async_wait<Cfg::NSTAGE - 2>();
        __syncthreads();
        {
            const int nt = tile + Cfg::NSTAGE - 1;
            if (nt < ntiles) load_tile<Cfg>(p, smem, nt % Cfg::NSTAGE, tbeg + nt * T, row0, bc0, nch);
            cp_async_commit();
        }
        Stage<Cfg> sv(smem, st);

        // ---- prep: Delta once per (t, d); task = (channel, 8-token chunk), lanes run over
        //      channels so the 16-byte row reads and writes are conflict free.  No-op tokens
        //      (past L or past dim) get Delta = 0 and a staged x of 0, so that they leave the
        //      state as it is.
#pragma unroll
        for (int k = 0; k < Cfg::TASKS_PER_THREAD; ++k) {
            const int task = tid + k * NT;
            const int cc = task % CH, t8 = task / CH;
            float dr[8];
            stage_row8<Cfg>(sv.ds, cc, t8, dr);
            const float bias = tbias[k];
            float o[8];
            if (cc < nch && t0 + 8 * t8 + 8 <= L) {          // whole chunk inside the data
#pragma unroll
                for (int u = 0; u < 8; u += 2) {                // tokens in pairs, packed FP32
                    float2 dl = fadd2(f2(dr[u], dr[u + 1]), f2(bias, bias));
                    if (p.softplus) dl = softplus_pair(dl);
                    o[u] = dl.x;
                    o[u + 1] = dl.y;
                }
            } else {
                const bool cok = cc < nch;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    float dl = dr[u] + bias;
                    if (p.softplus) dl = softplus_f(dl);
                    const bool ok = cok && (t0 + 8 * t8 + u < L);
                    o[u] = ok ? dl : 0.f;
                    if (!ok) sv.xs[Cfg::raw_at(cc, 8 * t8 + u)] = Tin(0.f);
                }
            }
            float4 *prow = prep + cc * Cfg::YP_SLOTS;
            prow[(2 * t8) ^ (cc & 7)] = make_float4(o[0], o[1], o[2], o[3]);
            prow[(2 * t8 + 1) ^ (cc & 7)] = make_float4(o[4], o[5], o[6], o[7]);
        }
        // B, C of the tile for the recurrence as fp32 rows, zero past dstate / past L
        if constexpr (sizeof(Tin) == 2) {
            // bf16: one (token, state quad) per item, both quads read as 8-byte words and
            // stored as 16-byte fp32 quads by consecutive lanes (conflict free)
            constexpr int QD = NP / 4;
            const unsigned short *rb = reinterpret_cast<const unsigned short *>(sv.bs);
            const unsigned short *rc = reinterpret_cast<const unsigned short *>(sv.cs);
#pragma unroll
            for (int k = 0; k < (T * QD + NT - 1) / NT; ++k) {
                const int i = tid + k * NT;
                if (i < T * QD) {
                    const int tt = i / QD, qq = i % QD;
                    uint4 v;
                    if (N == NP && t0 + tt < L) {            // dense rows: two 8-byte reads
                        const uint2 b2 = *reinterpret_cast<const uint2 *>(rb + tt * NP + 4 * qq);
                        const uint2 c2 = *reinterpret_cast<const uint2 *>(rc + tt * NP + 4 * qq);
                        v = make_uint4(b2.x, b2.y, c2.x, c2.y);
                    } else {
                        unsigned bw[4], cw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int n = 4 * qq + e;
                            const bool ok = n < N && t0 + tt < L;
                            bw[e] = ok ? rb[tt * N + n] : 0u;
                            cw[e] = ok ? rc[tt * N + n] : 0u;
                        }
                        v = make_uint4(bw[0] | (bw[1] << 16), bw[2] | (bw[3] << 16),
                                       cw[0] | (cw[1] << 16), cw[2] | (cw[3] << 16));
                    }
                    reinterpret_cast<float4 *>(Bf)[i] =
                        make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                                    __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
                    reinterpret_cast<float4 *>(Cf)[i] =
                        make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xffff0000u),
                                    __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xffff0000u));
                }
            }
        } else if (N == NP && t0 + T <= L) {                // dense rows: 8 values at a time
            constexpr int NV = T * NP / 8;
#pragma unroll
            for (int k = 0; k < (2 * NV + NT - 1) / NT; ++k) {
                const int i = tid + k * NT;
                if (i < 2 * NV) {
                    const int which = i >= NV;
                    const int v = i - which * NV;
                    float f[8];
                    load8<Tin>((which ? sv.cs : sv.bs) + 8 * v, f);
                    store8<float>((which ? Cf : Bf) + 8 * v, f);
                }
            }
        } else {
#pragma unroll
            for (int k = 0; k < (T * NP + NT - 1) / NT; ++k) {
                const int i = tid + k * NT;
                if (i < T * NP) {
                    const int tt = i / NP, n = i % NP;
                    const bool ok = n < N && t0 + tt < L;
                    Bf[i] = ok ? to_f32(sv.bs[tt * N + n]) : 0.f;
                    Cf[i] = ok ? to_f32(sv.cs[tt * N + n]) : 0.f;
                }
            }
        }
        __syncthreads();

        // ---- the recurrence: 4 states of one channel per lane, carried across tiles ----
        {
            const float4 *pp = prep + c * Cfg::YP_SLOTS;
            uint4 xq = make_uint4(0u, 0u, 0u, 0u);     // staged x chunk of the current token pair
            float4 *ypr = reinterpret_cast<float4 *>(yp) + (q * CH + c) * Cfg::YP_SLOTS;
            // the B or C quad of token t (fp32 rows) as pairs (0,1), (2,3)
            auto quad = [&](const float *X, int t, float2 (&v)[2]) {
                const float4 x4 = *reinterpret_cast<const float4 *>(X + t * NP + 4 * q);
                v[0] = f2(x4.x, x4.y);
                v[1] = f2(x4.z, x4.w);
            };
            // decays a = exp(Delta*A) and writes w = Delta*x*B of the 4 tokens of group g, as
            // state pairs (0,1), (2,3) for the packed FP32 instructions
            auto decay_write = [&](int g, float2 (&a)[4][2], float2 (&w)[4][2]) {
                const float4 d4 = pp[g ^ (c & 7)];     // Delta of tokens 4g .. 4g+3
                const float dl[4] = {d4.x, d4.y, d4.z, d4.w};
                float xv[4];                           // x of the same tokens (staged rows)
                if constexpr (Cfg::EIN == 8) {         // a 16-byte chunk serves two groups
                    if ((g & 1) == 0) xq = *reinterpret_cast<const uint4 *>(sv.xs + Cfg::raw_at(c, 4 * g));
                    const unsigned lo = (g & 1) ? xq.z : xq.x, hi = (g & 1) ? xq.w : xq.y;
                    xv[0] = __uint_as_float(lo << 16); xv[1] = __uint_as_float(lo & 0xffff0000u);
                    xv[2] = __uint_as_float(hi << 16); xv[3] = __uint_as_float(hi & 0xffff0000u);
                } else {
                    loadn<4, Tin>(sv.xs + Cfg::raw_at(c, 4 * g), xv);
                }
                float dx[4];                           // Delta*x (or x for the exact gain)
#pragma unroll
                for (int u = 0; u < 4; ++u) dx[u] = ZOH ? xv[u] : dl[u] * xv[u];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float2 bb[2];
                    quad(Bf, 4 * g + u, bb);
                    const float2 dl2 = f2(dl[u], dl[u]);
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        a[u][k] = ex2_pair(fmul2(dl2, A2p[k]));
                        if constexpr (ZOH) {   // dx holds x here; gain = expm1(Delta a) / a
                            float gw[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int s = 2 * k + e;
                                const float av = e ? a[u][k].y : a[u][k].x;
                                const float v = dl[u] * A2[s] * (1.f / kLog2e);
                                const float em1 = fabsf(v) < 0.1f ? expm1_small(v) : av - 1.f;
                                const float gain = invA[s] != 0.f ? em1 * invA[s] : dl[u];
                                gw[e] = gain * dx[u] * (e ? bb[k].y : bb[k].x);
                            }
                            w[u][k] = f2(gw[0], gw[1]);
                        } else {
                            w[u][k] = fmul2(f2(dx[u], dx[u]), bb[k]);
                        }
                    }
                }
            };
            auto recur_read = [&](int g, const float2 (&a)[4][2], const float2 (&w)[4][2]) {
                float out[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float2 cc2[2];
                    quad(Cf, 4 * g + u, cc2);
                    float2 acc = f2(0.f, 0.f);
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        hp[k] = ffma2(a[u][k], hp[k], w[u][k]);
                        acc = ffma2(cc2[k], hp[k], acc);
                    }
                    out[u] = acc.x + acc.y;
                }
                ypr[g ^ (c & 7)] = make_float4(out[0], out[1], out[2], out[3]);
            };
            // decays and writes of the next 4 tokens are computed before the recurrence
            // of the current 4, so the SFU work overlaps the FFMA chain
            float2 a0[4][2], w0[4][2];
            decay_write(0, a0, w0);
#pragma unroll
            for (int g = 0; g < T / 4; ++g) {
                float2 a1[4][2], w1[4][2];
                if (g + 1 < T / 4) decay_write(g + 1, a1, w1);
                recur_read(g, a0, w0);
                if (g + 1 < T / 4) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
#pragma unroll
                        for (int k = 0; k < 2; ++k) { a0[u][k] = a1[u][k]; w0[u][k] = w1[u][k]; }
                    }
                }
            }
        }
        __syncthreads();

        // ---- epilogue: sum the quads, skip, gate, convert; 16-byte stores of y ----
        Tout *gy = static_cast<Tout *>(p.y) + row0;
#pragma unroll
        for (int k = 0; k < Cfg::TASKS_PER_THREAD; ++k) {
            const int task = tid + k * NT;
            const int cc = task % CH, t8 = task / CH;
            // tokens in pairs, packed FP32: the quads' partials summed in order, the skip,
            // the gate
            float2 acc2[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
            for (int qq = 0; qq < Q; ++qq) {
                const float4 *row = reinterpret_cast<const float4 *>(yp) + (qq * CH + cc) * Cfg::YP_SLOTS;
                const float4 a0 = row[(2 * t8) ^ (cc & 7)];
                const float4 a1 = row[(2 * t8 + 1) ^ (cc & 7)];
                acc2[0] = fadd2(acc2[0], f2(a0.x, a0.y)); acc2[1] = fadd2(acc2[1], f2(a0.z, a0.w));
                acc2[2] = fadd2(acc2[2], f2(a1.x, a1.y)); acc2[3] = fadd2(acc2[3], f2(a1.z, a1.w));
            }
            float xr[8];
            stage_row8<Cfg>(sv.xs, cc, t8, xr);
            const float Dd = tD[k];
#pragma unroll
            for (int j = 0; j < 4; ++j) acc2[j] = ffma2(f2(Dd, Dd), f2(xr[2 * j], xr[2 * j + 1]), acc2[j]);
            if (p.z != nullptr) {
                float zr[8];
                stage_row8<Cfg>(sv.zs, cc, t8, zr);
#pragma unroll
                for (int j = 0; j < 4; ++j) acc2[j] = fmul2(acc2[j], silu_pair(f2(zr[2 * j], zr[2 * j + 1])));
            }
            float acc[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) { acc[2 * j] = acc2[j].x; acc[2 * j + 1] = acc2[j].y; }
            const int tg = t0 + 8 * t8;
            if (cc < nch) {
                if (Cfg::VEC && tg + 8 <= L) {
                    store_run<8>(gy + size_t(cc) * L + tg, acc);
                } else {
                    for (int u = 0; u < 8; ++u)
                        if (tg + u < L) gy[size_t(cc) * L + tg + u] = from_f32<Tout>(acc[u]);
                }
            }
        }
        // the next tile's first barrier orders these reads before the partials and the
        // stage are written again
    }
    cp_async_wait<0>();
    h[0] = hp[0].x; h[1] = hp[0].y; h[2] = hp[1].x; h[3] = hp[1].y;

    if ((!SEG || seg == p.nseg - 1) && p.final_state != nullptr && dvalid) {
        float *fs = p.final_state + chrow * N;
#pragma unroll
        for (int s = 0; s < 4; ++s)
            if (4 * q + s < N) fs[4 * q + s] = h[s];
    }
}

// ---------------------------------------------------------------------------------------
// Tail and fold passes of the segmented scan.

// scan_tail_kernel: one CTA per (sequence, channel, segment but the last).  The CTA walks
// back from the segment's end in windows of kTailWarps x 32 lanes x kTailTok tokens; lane l
// of warp w takes kTailTok consecutive tokens of the w-th run of the window, so its steps
// and inputs arrive in single vector loads.  R_t (the steps after t) comes from a serial
// suffix sum over the lane's tokens, a shuffle suffix scan over the lanes and a shared scan
// over the warps.  exp(A_n R_t) is ex2 with subnormal results flushed to 0, so a state whose
// log2 decay A_n log2(e) R_t stays below -127 over a warp's run adds exactly 0 there and is
// skipped (states go in pairs; a spent state computed beside a live one adds exactly 0).
// With the softplus step every step is positive and R only grows going back: a state n
// with A_n < 0 is spent for R > -127 / (A_n log2 e), tested once per run against the R
// after the run, and the walk stops at the first window that starts with every state
// spent; the segment's step sum S is then recorded as +inf (its decay is 0 for every
// state).  Without the softplus a step can be negative, so each run is tested on its own
// range of R and the walk covers the whole segment.  Lane sums are reduced in a fixed order.
#ifndef SSM_TAIL_WARPS
#define SSM_TAIL_WARPS 8      // warps per CTA
#endif
#ifndef SSM_TAIL_MINB
#define SSM_TAIL_MINB 3       // resident CTAs per SM the registers target
#endif
constexpr int kTailWarps = SSM_TAIL_WARPS;
constexpr int kTailTok = 4;           // consecutive tokens per lane and window
constexpr float kSpentLog2 = -127.f;  // log2 decay below which ex2 flushes to 0

// kTailTok consecutive values from src (vector load when `vec`: 4 values, 8- or 16-byte
// aligned) as fp32; zeros when !ok.
template <typename Tin>
__device__ __forceinline__ void load_run4(const Tin *src, bool vec, bool ok, float (&v)[4]) {
    if (!ok) {
        v[0] = v[1] = v[2] = v[3] = 0.f;
    } else if (vec) {
        loadn<4, Tin>(src, v);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = to_f32(src[i]);
    }
}

template <int NP, typename Tin, bool ZOH>
__global__ void __launch_bounds__(32 * kTailWarps, SSM_TAIL_MINB)
scan_tail_kernel(const ScanArgs p) {
    constexpr int NQ = NP / 2;                          // state pairs
    constexpr int EC = int(16 / sizeof(Tin));           // values per 16-byte chunk
    __shared__ float wsum[2][kTailWarps];
    __shared__ float hred[kTailWarps][NP];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per = p.nseg - 1;
    const int seg = int(blockIdx.x % unsigned(per));
    const long long row = blockIdx.x / unsigned(per);     // b * dim + d
    const int d = int(row % p.dim);
    const int b = int(row / p.dim);
    const int L = p.seqlen, N = p.dstate;
    const int tbeg = seg * p.seg_len;                   // a multiple of 32, as is tend:
    const int tend = tbeg + p.seg_len;                  // segments before the last are whole
    const bool vec = (L % 4) == 0;                      // 4-token runs aligned in every row

    float2 A2p[NQ];
    float Rdead[NQ];      // (softplus) the pair is spent once R exceeds this
#pragma unroll
    for (int k = 0; k < NQ; ++k) {
        float a[2], r = -INFINITY;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int n = 2 * k + e;
            a[e] = n < N ? p.A[size_t(d) * N + n] * kLog2e : 0.f;
            if (n < N) r = fmaxf(r, a[e] < 0.f ? kSpentLog2 / a[e] : INFINITY);
        }
        A2p[k] = f2(a[0], a[1]);
        Rdead[k] = r;
    }
    // pairs not yet spent over a run whose R lies in [lo, hi] (any sign of the steps)
    auto live_range = [&](float lo, float hi) {
        unsigned m = 0;
#pragma unroll
        for (int k = 0; k < NQ; ++k) {
            const float ex = A2p[k].x * (A2p[k].x < 0.f ? lo : hi);   // the largest log2 decay
            const float ey = A2p[k].y * (A2p[k].y < 0.f ? lo : hi);
            if ((2 * k < N && !(ex < kSpentLog2)) || (2 * k + 1 < N && !(ey < kSpentLog2)))
                m |= 1u << k;
        }
        return m;
    };
    // (softplus) pairs not yet spent at step sum lo, R >= lo
    auto live_from = [&](float lo) {
        unsigned m = 0;
#pragma unroll
        for (int k = 0; k < NQ; ++k)
            if (!(lo > Rdead[k])) m |= 1u << k;
        return m;
    };

    const float bias = p.delta_bias != nullptr ? p.delta_bias[d] : 0.f;
    const size_t row0 = size_t(row) * L;
    const Tin *gd = static_cast<const Tin *>(p.delta) + row0;
    const Tin *gx = static_cast<const Tin *>(p.x) + row0;
    const Tin *gb = static_cast<const Tin *>(p.B) + size_t(b) * L * N;

    const bool grows = p.softplus != 0;
    constexpr int WT = 32 * kTailTok;                  // tokens per warp and window
    constexpr int WIN = kTailWarps * WT;
    float2 acc[NQ];
#pragma unroll
    for (int k = 0; k < NQ; ++k) acc[k] = f2(0.f, 0.f);
    float R = 0.f;                                     // steps after the window
    bool spent = false;
    int par = 0;
    // this lane's raw steps in the window ending at w1, loaded one window ahead
    float draw[kTailTok];
    auto load_steps = [&](int w1) {
        const int t0 = w1 - WIN + warp * WT + kTailTok * lane;
        load_run4<Tin>(gd + (t0 >= tbeg ? t0 : tbeg), vec, t0 >= tbeg, draw);
    };
    load_steps(tend);
    for (int w1 = tend; w1 > tbeg; w1 -= WIN, par ^= 1) {
        if (grows && live_from(R) == 0u) { spent = true; break; }   // the same R in every thread
        const int t0 = w1 - WIN + warp * WT + kTailTok * lane;   // this lane's first token
        const bool ok = t0 >= tbeg;                    // all kTailTok tokens or none
        float dl[kTailTok];
#pragma unroll
        for (int i = 0; i < kTailTok; ++i) {
            float v = draw[i] + bias;
            if (p.softplus) v = softplus_f(v);
            dl[i] = ok ? v : 0.f;
        }
        if (w1 - WIN > tbeg) load_steps(w1 - WIN);
        float xv[kTailTok];
        load_run4<Tin>(gx + (ok ? t0 : tbeg), vec, ok, xv);
        // steps after each of this lane's tokens, within the lane, then across the lanes
        float sl[kTailTok];
        sl[kTailTok - 1] = 0.f;
#pragma unroll
        for (int i = kTailTok - 2; i >= 0; --i) sl[i] = sl[i + 1] + dl[i + 1];
        float incl = sl[0] + dl[0];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_down_sync(0xffffffffu, incl, o);
            if (lane + o < 32) incl += u;
        }
        float excl = __shfl_down_sync(0xffffffffu, incl, 1);
        if (lane == 31) excl = 0.f;
        const float tot = __shfl_sync(0xffffffffu, incl, 0);
        if (lane == 0) wsum[par][warp] = tot;
        __syncthreads();
        float Rw = R;                                  // steps after this warp's run
#pragma unroll
        for (int k = kTailWarps - 1; k >= 0; --k) {
            const float v = wsum[par][k];
            if (k > warp) Rw += v;
            R += v;
        }
        const float Rl = Rw + excl;                    // steps after this lane's last token
        unsigned m;
        if (grows) {
            m = live_from(Rw);
        } else {
            float lo = Rl, hi = Rl;
#pragma unroll
            for (int i = 0; i < kTailTok; ++i) { lo = fminf(lo, Rl + sl[i]); hi = fmaxf(hi, Rl + sl[i]); }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
                hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
            }
            m = live_range(lo, hi);
        }
        if (m == 0u || w1 - WIN + warp * WT + WT <= tbeg) continue;   // uniform over the warp

        // B rows of this lane's tokens, raw, then the live pairs
#pragma unroll
        for (int i = 0; i < kTailTok; ++i) {
            const int t = t0 + i;
            float bf[NP];
            if (ok && N == NP) {                       // dense rows: 16-byte (or 8-byte) loads
                const Tin *br = gb + size_t(t) * NP;
                if constexpr (NP >= EC) {
#pragma unroll
                    for (int c = 0; c < NP; c += EC) {
                        float v[EC];
                        loadn<EC, Tin>(br + c, v);
#pragma unroll
                        for (int e = 0; e < EC; ++e) bf[c + e] = v[e];
                    }
                } else {
                    loadn<NP, Tin>(br, bf);
                }
            } else {
#pragma unroll
                for (int n = 0; n < NP; ++n) bf[n] = (ok && n < N) ? to_f32(gb[size_t(t) * N + n]) : 0.f;
            }
            const float Rt = Rl + sl[i];
            const float2 Rt2 = f2(Rt, Rt);
            const float dx = ZOH ? xv[i] : dl[i] * xv[i];
            const float2 dx2 = f2(dx, dx);
#pragma unroll
            for (int k = 0; k < NQ; ++k) {
                if (!((m >> k) & 1u)) continue;
                float2 w = fmul2(dx2, f2(bf[2 * k], bf[2 * k + 1]));
                if constexpr (ZOH) {   // gain expm1(Delta a) / a, Delta where a = 0
                    float g[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float a2 = e ? A2p[k].y : A2p[k].x;
                        const float a = a2 * (1.f / kLog2e);
                        const float v = dl[i] * a;
                        const float em1 = fabsf(v) < 0.1f ? expm1_small(v) : ex2_approx(dl[i] * a2) - 1.f;
                        g[e] = a != 0.f ? em1 / a : dl[i];
                    }
                    w = fmul2(w, f2(g[0], g[1]));
                }
                acc[k] = ffma2(ex2_pair(fmul2(A2p[k], Rt2)), w, acc[k]);
            }
        }
    }
    // h_end: lanes (butterfly), then warps in order
#pragma unroll
    for (int k = 0; k < NQ; ++k) {
        float vx = acc[k].x, vy = acc[k].y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            vx += __shfl_xor_sync(0xffffffffu, vx, o);
            vy += __shfl_xor_sync(0xffffffffu, vy, o);
        }
        if (lane == 0) { hred[warp][2 * k] = vx; hred[warp][2 * k + 1] = vy; }
    }
    __syncthreads();
    if (threadIdx.x < NP) {
        float h = 0.f;
#pragma unroll
        for (int k = 0; k < kTailWarps; ++k) h += hred[k][threadIdx.x];
        p.seg_h[(size_t(row) * p.nseg + seg) * NP + threadIdx.x] = h;
    }
    if (threadIdx.x == 0) p.seg_s[size_t(row) * p.nseg + seg] = spent ? __int_as_float(0x7f800000) : R;
}

// scan_fold_kernel: one thread per (sequence, channel, padded state).  Walks the segments
// in order from the start state, replacing each tail sum h_end_j by the carry into segment
// j and stepping h <- exp(A S_j) h + h_end_j (S_j = +inf: decay 0).  The last segment's
// slot only receives its carry.
template <int NP>
__global__ void scan_fold_kernel(const ScanArgs p) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long rows = (long long)p.batch * p.dim;
    if (i >= rows * NP) return;
    const long long row = i / NP;
    const int n = int(i - row * NP);
    const int d = int(row % p.dim);
    const int N = p.dstate;
    const float A2 = n < N ? p.A[size_t(d) * N + n] * kLog2e : 0.f;
    float h = (p.h0 != nullptr && n < N) ? p.h0[size_t(row) * N + n] : 0.f;
    for (int j = 0; j < p.nseg; ++j) {
        float *hj = p.seg_h + (size_t(row) * p.nseg + j) * NP + n;
        if (j == p.nseg - 1) { *hj = h; break; }
        const float hend = *hj;
        const float sj = p.seg_s[size_t(row) * p.nseg + j];
        *hj = h;
        const float decay = isinf(sj) ? 0.f : ex2_approx(A2 * sj);
        h = fmaf(decay, h, hend);
    }
}

}  // namespace ssm
