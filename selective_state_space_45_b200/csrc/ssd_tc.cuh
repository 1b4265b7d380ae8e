// ssd_tc.cuh -- Mamba-2's state-space dual (SSD) forward on the sm_100 tensor cores
// (tcgen05 MMAs with accumulators in tensor memory, TMA tile loads).
//
// What it computes (per sequence b and head h, a P x N state S, one decay per head):
//     S <- exp(a_t) S + x_t B_t^T,     y_t = S C_t
// with x already times the step and a = step * A ("Beyond attention with Mamba, state
// space models and hybrids", xmarva lesson 10, section 8 "Mamba-2: the same model as
// attention").  By chunks of Q = 128 tokens, with cum_l = a_0 + ... + a_l inside the chunk
// and S the state entering it:
//     y_l  = sum_{s<=l} (C_l . B_s) exp(cum_l - cum_s) x_s  +  exp(cum_l) (C_l S^T)
//     S'   = exp(cum_{Q-1}) S + sum_s exp(cum_{Q-1} - cum_s) B_s x_s^T      (kept as [N][P])
// -- attention with the decay as its mask inside the chunk, the recurrence between chunks.
//
// Layout of the work: one CTA per (sequence, head) walks its chunks in order; the state
// never leaves the chip (fp32 in registers, a bf16 copy in shared memory as an MMA
// operand), so the only HBM traffic is x, a, B, C in and y out.  Per chunk:
//   TMA      x [Q][P], B and C [Q][N] (64-state column blocks), double-buffered;
//   MMA 1    G = C B^T            (M = Q, N = Q, K = N; both K-major)
//   MMA 2    Yc = C S^T           (K = N; S^T from the [N][P] copy, MN-major)
//   MMA 3    D = B^T (w o x)      (M = N, K = Q; B^T MN-major, w o x MN-major), w_s = e^{cum_end - cum_s}
//   MMA 4    Yi = Mask(G) x       (K = Q; masked scores K-major, x MN-major)
// and, on the CUDA cores: the cumulative decays, w o x, the masked scores (bf16),
// S' = e^{tot} S + D and y = Yi + e^{cum} Yc.  The CTA has NWG groups of 4 warps: warp w
// serves tensor-memory lanes 32 (w % 4) .. +31 -- row l of G, Yi, Yc and row n of D -- and
// column slice w / 4 of each of those rows.  One thread issues the MMAs; tcgen05.commit
// signals mbarriers.  The next chunk's MMA 1 + 2 are issued before this chunk's outputs are
// formed (two Yc accumulators alternate), so they overlap.
#pragma once

#include "common.cuh"
#include "tc_common.cuh"

namespace ssm {

struct SsdTcArgs {
    const float *a;           // [batch][L][heads]
    void *y;                  // [batch][L][heads][P], Tout
    const float *h0;          // [batch][heads][P][N] or null
    float *hN;                // [batch][heads][P][N] or null
    unsigned *timeouts;       // incremented when a wait gives up (never in normal operation)
    int batch, seqlen, heads;
};

template <int P_, int N_, typename Tout_, int NWG_ = 2>
struct SsdTcCfg {
    using Tout = Tout_;
    static constexpr int P = P_, N = N_, Q = 128, NWG = NWG_, NT = 128 * NWG_;
    static constexpr int PS = P / NWG, QS = Q / NWG;   // columns per warp slice (of P, of Q)
    static constexpr int XROW = P * 2;                 // bytes per row of x, w o x, S (64 or 128)
    static constexpr uint32_t XLAYOUT = XROW == 128 ? kLayoutSw128 : kLayoutSw64;
    static constexpr int NB = N / 64;                  // 64-state column blocks of B, C
    static_assert(P == 32 || P == 64, "head width 32 or 64");
    static_assert(N == 64 || N == 128, "state width 64 or 128");
    static_assert(PS % 16 == 0 && QS % 32 == 0, "slices of whole 16-column tensor-memory loads");
    // shared memory (every tile 1024-byte aligned)
    static constexpr uint32_t X_BYTES = Q * XROW;            // [Q][P]
    static constexpr uint32_t BC_BLOCK = Q * 128;            // [Q][64] bf16
    static constexpr uint32_t BC_BYTES = NB * BC_BLOCK;
    static constexpr uint32_t STAGE = X_BYTES + 2 * BC_BYTES;
    static constexpr uint32_t OFF_STAGE = 0;                 // [2] x, B, C
    static constexpr uint32_t OFF_M = OFF_STAGE + 2 * STAGE; // masked scores [Q][Q] K-major, 2 blocks
    static constexpr uint32_t OFF_WX = OFF_M + 2 * BC_BLOCK; // w o x [Q][P]
    static constexpr uint32_t OFF_S = OFF_WX + X_BYTES;      // S bf16 [128][P] (rows >= N zero)
    static constexpr uint32_t OFF_ZERO = OFF_S + 128 * XROW; // a zero [Q][64] block (N = 64)
    static constexpr uint32_t OFF_CUM = OFF_ZERO + (N == 64 ? BC_BLOCK : 0);
    static constexpr uint32_t OFF_BAR = OFF_CUM + 4 * (Q + 8);
    static constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;   // + alignment slack
    // tensor memory columns: G, two Yc buffers (chunk c's is read while chunk c+1's is
    // computed), Yi, D
    static constexpr uint32_t TM_G = 0, TM_YC = 128, TM_YI = TM_YC + 2 * P, TM_D = TM_YI + P;
    static constexpr uint32_t TM_COLS = (TM_D + P) <= 256 ? 256 : 512;
    static constexpr uint32_t TX_BYTES = X_BYTES + 2 * BC_BYTES;
};

// SM cycles an mbarrier wait may take before the kernel gives up (about a second)
constexpr long long kSsdWaitCycles = 2000000000LL;

// `W` consecutive fp32 columns (16 or 32) of this thread's tensor-memory lane, as raw bits;
// valid after tmem_wait_ld()
template <int W>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t *v) {
    if constexpr (W == 32) {
        tmem_ld32_async(taddr, *reinterpret_cast<uint32_t (*)[32]>(v));
    } else {
        static_assert(W == 16, "16 or 32 columns");
        tmem_ld16_async(taddr, *reinterpret_cast<uint32_t (*)[16]>(v));
    }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::NT, 1)
ssd_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
              const __grid_constant__ CUtensorMap tm_c, const SsdTcArgs p) {
    using Tout = typename Cfg::Tout;
    constexpr int P = Cfg::P, N = Cfg::N, Q = Cfg::Q, NB = Cfg::NB, XROW = Cfg::XROW;
    constexpr int PS = Cfg::PS, QS = Cfg::QS;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *cum = reinterpret_cast<float *>(smem + Cfg::OFF_CUM);           // [Q] + warp totals
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);   // tma[2], mma[3]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 6);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = 32 * (warp & 3) + lane;      // tensor-memory lane = row of the products
    const int slice = warp >> 2;                 // column slice of this warp
    const int bh = blockIdx.x;
    const int b = bh / p.heads, h = bh - b * p.heads;
    const int L = p.seqlen, H = p.heads;
    const int nchunk = (L + Q - 1) / Q;

    if (tid == 0) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&tm_c);
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, Cfg::TM_COLS);
    // zero the S copy (rows >= N stay zero) and the zero block
    for (int i = tid; i < (128 * XROW) / 16; i += Cfg::NT)
        reinterpret_cast<uint4 *>(smem + Cfg::OFF_S)[i] = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (N == 64)
        for (int i = tid; i < int(Cfg::BC_BLOCK / 16); i += Cfg::NT)
            reinterpret_cast<uint4 *>(smem + Cfg::OFF_ZERO)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;   // this warp's tensor-memory lanes

    auto issue_loads = [&](int c) {
        const int st = c & 1;
        unsigned char *sb = smem + Cfg::OFF_STAGE + st * Cfg::STAGE;
        mbar_arrive_expect_tx(&bars[st], Cfg::TX_BYTES);
        tma_load_4d(sb, &tm_x, &bars[st], 0, h, c * Q, b);
#pragma unroll
        for (int k = 0; k < NB; ++k) {
            tma_load_4d(sb + Cfg::X_BYTES + k * Cfg::BC_BLOCK, &tm_b, &bars[st], 64 * k, h, c * Q, b);
            tma_load_4d(sb + Cfg::X_BYTES + Cfg::BC_BYTES + k * Cfg::BC_BLOCK, &tm_c, &bars[st], 64 * k, h,
                        c * Q, b);
        }
    };
    if (tid == 0) {
        issue_loads(0);
        if (nchunk > 1) issue_loads(1);
    }

    // the state: thread (row n < N, slice g) holds S[p][n] for the p of its slice
    float S[PS];
    const size_t sbase = size_t(bh) * P * N;
    const int p0 = slice * PS;
#pragma unroll
    for (int q = 0; q < PS; ++q)
        S[q] = (p.h0 != nullptr && row < N) ? p.h0[sbase + size_t(p0 + q) * N + row] : 0.f;
    auto write_state = [&]() {      // bf16 copy of S as rows n of P values (MN-major operand)
        if (row < N) {
#pragma unroll
            for (int j = 0; j < PS / 8; ++j) {
                uint4 v;
                v.x = pack_bf16x2(S[8 * j + 0], S[8 * j + 1]);
                v.y = pack_bf16x2(S[8 * j + 2], S[8 * j + 3]);
                v.z = pack_bf16x2(S[8 * j + 4], S[8 * j + 5]);
                v.w = pack_bf16x2(S[8 * j + 6], S[8 * j + 7]);
                *reinterpret_cast<uint4 *>(smem + Cfg::OFF_S + swz<XROW>(row, 2 * p0 + 16 * j)) = v;
            }
        }
    };
    write_state();
    fence_async_smem();

    constexpr uint32_t ID_G = idesc_bf16(128, Q, false, false);
    constexpr uint32_t ID_YC = idesc_bf16(128, P, false, true);
    constexpr uint32_t ID_D = idesc_bf16(128, P, true, true);
    constexpr uint32_t ID_YI = idesc_bf16(128, P, false, true);
    const uint32_t s_m = smem_addr(smem + Cfg::OFF_M), s_wx = smem_addr(smem + Cfg::OFF_WX);
    const uint32_t s_s = smem_addr(smem + Cfg::OFF_S), s_zero = smem_addr(smem + Cfg::OFF_ZERO);
    // MN-major operand with rows of XROW bytes: K-step of 16 rows
    constexpr uint32_t MN_SBO = 8 * XROW, MN_KSTEP = 16 * XROW;
    // every thread waits, then the block agrees: on a time-out all threads leave the loop
    auto wait_all = [&](uint64_t *bar, uint32_t parity) {
        const bool mine = mbar_wait(bar, parity, kSsdWaitCycles);
        return __syncthreads_and(mine) != 0;
    };
    auto stage_of = [&](int c) { return smem + Cfg::OFF_STAGE + (c & 1) * Cfg::STAGE; };
    // MMA 1 + 2 of chunk c: G = C B^T, Yc = C S^T (S: the state entering chunk c)
    auto issue_scores = [&](int c) {
        unsigned char *sb = stage_of(c);
        const uint32_t s_b = smem_addr(sb + Cfg::X_BYTES), s_c = smem_addr(sb + Cfg::X_BYTES + Cfg::BC_BYTES);
        const uint32_t yc = tmem + Cfg::TM_YC + (c & 1) * P;
        tc_fence_after_sync();
#pragma unroll
        for (int k = 0; k < N / 16; ++k) {
            const uint32_t koff = (k >> 2) * Cfg::BC_BLOCK + (k & 3) * 32;
            const uint64_t ad = smem_desc(s_c + koff, 16, 1024, kLayoutSw128);
            umma_bf16(tmem + Cfg::TM_G, ad, smem_desc(s_b + koff, 16, 1024, kLayoutSw128), ID_G, k > 0);
            umma_bf16(yc, ad, smem_desc(s_s + k * MN_KSTEP, 8192, MN_SBO, Cfg::XLAYOUT), ID_YC, k > 0);
        }
        umma_commit(&bars[2]);
    };
    auto load_a = [&](int c) {
        const int t = c * Q + row;
        return (slice == 0 && c < nchunk && t < L) ? p.a[(size_t(b) * L + t) * H + h] : 0.f;
    };
    bool ok = wait_all(&bars[0], 0u);
    if (ok && tid == 0) issue_scores(0);
    float a_next = load_a(0);
    int c = 0;
    for (; ok && c < nchunk; ++c) {
        const int t0 = c * Q, t = t0 + row;
        const uint32_t par = uint32_t(c & 1);
        unsigned char *sb = stage_of(c);
        const uint32_t s_x = smem_addr(sb), s_b = smem_addr(sb + Cfg::X_BYTES);

        // the chunk's decays: inclusive cumulative sum over the chunk (zero past L), by the
        // first warp group; everyone reads them from shared memory
        float cs = a_next;
        a_next = load_a(c + 1);
        if (slice == 0) {
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = __shfl_up_sync(0xffffffffu, cs, o);
                if (lane >= o) cs += u;
            }
            if (lane == 31) cum[Q + warp] = cs;
        }
        __syncthreads();
        if (slice == 0) {
            for (int w = 0; w < warp; ++w) cs += cum[Q + w];
            cum[row] = cs;
        }
        const float tot = cum[Q] + cum[Q + 1] + cum[Q + 2] + cum[Q + 3];
        __syncthreads();
        cs = cum[row];

        // w o x: row s of x times w_s = e^{tot - cum_s}, this warp's slice of P
        {
            const float w = ex2_approx((tot - cs) * kLog2e);
#pragma unroll
            for (int j = 0; j < PS / 8; ++j) {
                const uint32_t off = swz<XROW>(row, 2 * p0 + 16 * j);
                const uint4 v = *reinterpret_cast<const uint4 *>(sb + off);
                const unsigned vv[4] = {v.x, v.y, v.z, v.w};
                unsigned o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    o[e] = pack_bf16x2(__uint_as_float(vv[e] << 16) * w, __uint_as_float(vv[e] & 0xffff0000u) * w);
                *reinterpret_cast<uint4 *>(smem + Cfg::OFF_WX + off) = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
        fence_async_smem();
        __syncthreads();
        // MMA 3: D = B^T (w o x), rows n (B^T MN-major: 64-state blocks LBO apart)
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t lbo = N == 128 ? Cfg::BC_BLOCK : (s_zero - s_b);
#pragma unroll
            for (int k = 0; k < Q / 16; ++k)
                umma_bf16(tmem + Cfg::TM_D, smem_desc(s_b + k * 2048, lbo, 1024, kLayoutSw128),
                          smem_desc(s_wx + k * MN_KSTEP, 8192, MN_SBO, Cfg::XLAYOUT), ID_D, k > 0);
            umma_commit(&bars[3]);
        }
        // masked scores from G (row l): e^{cum_l - cum_s} for s <= l, 0 above; this warp's
        // slice of the columns s
        if (!(ok = wait_all(&bars[2], par))) break;
        tc_fence_after_sync();
        {
            const int rmax = 32 * (warp & 3) + 31;     // last row of this warp
            uint32_t graw[QS / 32][32];
#pragma unroll
            for (int jb = 0; jb < QS / 32; ++jb) {
                const int s0b = slice * QS + 32 * jb;
                if (s0b <= rmax) tmem_ld32_async(tmem + lane_base + Cfg::TM_G + s0b, graw[jb]);
            }
            tmem_wait_ld();
#pragma unroll
            for (int jb = 0; jb < QS / 32; ++jb) {
                const int s0b = slice * QS + 32 * jb;
                if (s0b > rmax) {                       // wholly above this warp's rows: zeros
#pragma unroll
                    for (int j8 = 0; j8 < 4; ++j8) {
                        const int s0 = s0b + 8 * j8;
                        *reinterpret_cast<uint4 *>(smem + Cfg::OFF_M + (s0 >> 6) * Cfg::BC_BLOCK +
                                                   swz<128>(row, 2 * (s0 & 63))) = make_uint4(0u, 0u, 0u, 0u);
                    }
                    continue;
                }
                float g[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) g[e] = __uint_as_float(graw[jb][e]);
#pragma unroll
                for (int j8 = 0; j8 < 4; ++j8) {
                    float m[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int s = s0b + 8 * j8 + e;
                        const float dec = ex2_approx((cs - cum[s]) * kLog2e);
                        m[e] = s <= row ? g[8 * j8 + e] * dec : 0.f;
                    }
                    const int s0 = s0b + 8 * j8;
                    uint4 v;
                    v.x = pack_bf16x2(m[0], m[1]); v.y = pack_bf16x2(m[2], m[3]);
                    v.z = pack_bf16x2(m[4], m[5]); v.w = pack_bf16x2(m[6], m[7]);
                    *reinterpret_cast<uint4 *>(smem + Cfg::OFF_M + (s0 >> 6) * Cfg::BC_BLOCK +
                                               swz<128>(row, 2 * (s0 & 63))) = v;
                }
            }
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        // MMA 4: Yi = Mask x
        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int k = 0; k < Q / 16; ++k) {
                const uint32_t koff = (k >> 2) * Cfg::BC_BLOCK + (k & 3) * 32;
                umma_bf16(tmem + Cfg::TM_YI, smem_desc(s_m + koff, 16, 1024, kLayoutSw128),
                          smem_desc(s_x + k * MN_KSTEP, 8192, MN_SBO, Cfg::XLAYOUT), ID_YI, k > 0);
            }
            umma_commit(&bars[4]);
        }
        // the state: S' = e^{tot} S + D (row n, this warp's slice of P); MMA 2 has read the
        // old copy
        if (!(ok = wait_all(&bars[3], par))) break;
        tc_fence_after_sync();
        {
            const float dtot = ex2_approx(tot * kLog2e);
            uint32_t d[PS];
#pragma unroll
            for (int j = 0; j < PS; j += (PS >= 32 ? 32 : 16))
                tmem_ld_cols<(PS >= 32 ? 32 : 16)>(tmem + lane_base + Cfg::TM_D + p0 + j, d + j);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < PS; ++e) S[e] = fmaf(dtot, S[e], __uint_as_float(d[e]));
            write_state();
        }
        fence_async_smem();
        // the next chunk's scores and state readout run while this chunk's outputs are formed
        if (c + 1 < nchunk) {
            if (!(ok = wait_all(&bars[(c + 1) & 1], uint32_t(((c + 1) >> 1) & 1)))) break;
            if (tid == 0) issue_scores(c + 1);
        }
        // y = Yi + e^{cum_l} Yc, row l, this warp's slice of P
        if (!(ok = wait_all(&bars[4], par))) break;
        tc_fence_after_sync();
        {
            const float el = ex2_approx(cs * kLog2e);
            Tout *yrow = static_cast<Tout *>(p.y) + ((size_t(b) * L + t) * H + h) * P + p0;
            const uint32_t yc = Cfg::TM_YC + (c & 1) * P + p0;
            uint32_t yir[PS], ycr[PS];
#pragma unroll
            for (int j = 0; j < PS; j += (PS >= 32 ? 32 : 16)) {
                tmem_ld_cols<(PS >= 32 ? 32 : 16)>(tmem + lane_base + Cfg::TM_YI + p0 + j, yir + j);
                tmem_ld_cols<(PS >= 32 ? 32 : 16)>(tmem + lane_base + yc + j, ycr + j);
            }
            tmem_wait_ld();
            float yi[PS];
#pragma unroll
            for (int e = 0; e < PS; ++e) yi[e] = fmaf(el, __uint_as_float(ycr[e]), __uint_as_float(yir[e]));
            if (t < L) {
#pragma unroll
                for (int e = 0; e < PS; e += 8) store_run<8>(yrow + e, yi + e);
            }
        }
        tc_fence_before_sync();
        __syncthreads();
        // every product reading this chunk's stage is done: load chunk c + 2 into it
        if (tid == 0 && c + 2 < nchunk) issue_loads(c + 2);
    }
    if (ok) {
        if (p.hN != nullptr && row < N) {
#pragma unroll
            for (int q = 0; q < PS; ++q) p.hN[sbase + size_t(p0 + q) * N + row] = S[q];
        }
    } else {
        // a wait gave up: report it, then let whatever this CTA still has in flight (the
        // loads of the next chunks, the MMAs of this one and the next) finish, each wait bounded
        if (tid == 0) {
            if (p.timeouts != nullptr) atomicAdd(p.timeouts, 1u);
            for (int k = 0; k < 3; ++k)
                if (c + k < nchunk) mbar_wait(&bars[(c + k) & 1], uint32_t(((c + k) >> 1) & 1), kSsdWaitCycles);
            for (int k = 2; k < 5; ++k) mbar_wait(&bars[k], uint32_t(c & 1), kSsdWaitCycles);
            mbar_wait(&bars[2], uint32_t((c + 1) & 1), kSsdWaitCycles);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, Cfg::TM_COLS);
}

}  // namespace ssm
