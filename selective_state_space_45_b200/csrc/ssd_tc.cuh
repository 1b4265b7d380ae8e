// ssd_tc.cuh -- Mamba-2's state-space dual (SSD) forward on the sm_100 tensor cores,
// laid out so that two CTAs share an SM.
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
// One CTA of 4 warps per (sequence, head) walks its chunks in order, the state on the chip
// (fp32 in registers, a bf16 copy in shared memory as an MMA operand); HBM sees only x, a,
// B, C in and y (and the final state) out.  Thread i owns tensor-memory lane i: row l of
// the scores and outputs, row n of the state.  Per chunk:
//   TMA      x [Q][P], B and C [Q][N] (64-state column blocks) into one buffer set
//   MMA 1    G  = C B^T                (tensor-memory columns 0 .. Q-1)
//   MMA 2    Yc = C S^T                (columns Q .. Q+P-1)
//   CUDA     masked scores M = G o e^{cum_l - cum_s} (s <= l) written as bf16 over C, whose
//            products are done -- below the diagonal block as a running product of e^{a_s}
//            from one exponential per 32 columns; B's rows scaled in place by
//            w_s = e^{cum_end - cum_s}
//   MMA 3    D  = (w o B)^T x          (columns 0 .. P-1: G has been read)
//   MMA 4    Yi = M x                  (columns Q+P .. Q+2P-1)
//   CUDA     the next chunk's loads go out once MMA 4 is done (its tiles were sent
//            towards L2 when this chunk's MMA 1 was issued); S' = e^{cum_end} S + D; the
//            next chunk's cumulative decays; once its tiles land, its MMA 1 (D has been
//            read, so G's columns are free) runs while this chunk's y = Yi + e^{cum_l} Yc
//            is written; its MMA 2 follows once Yc has been read
// So a CTA holds one buffer set (~98 KB of shared memory at P = 64, N = 128) and 256
// tensor-memory columns: two CTAs fit on an SM, and one CTA's loads and barriers overlap
// the other's products and row-wise work.  Every mbarrier wait is bounded; a CTA whose
// wait gives up leaves its loop, lets its copies and products in flight finish (each wait
// bounded), frees its tensor memory and counts the event.
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

template <int P_, int N_, typename Tout_>
struct SsdTcCfg {
    using Tout = Tout_;
    static constexpr int P = P_, N = N_, Q = 128, NT = 128;
    static constexpr int XROW = P * 2;                 // bytes per row of x and S (64 or 128)
    static constexpr uint32_t XLAYOUT = XROW == 128 ? kLayoutSw128 : kLayoutSw64;
    static constexpr int NB = N / 64;                  // 64-state column blocks of B, C
    static_assert(P == 32 || P == 64, "head width 32 or 64");
    static_assert(N == 64 || N == 128, "state width 64 or 128");
    // shared memory, every tile 1024-byte aligned
    static constexpr uint32_t X_BYTES = Q * XROW;            // x [Q][P]
    static constexpr uint32_t BC_BLOCK = Q * 128;            // [Q][64] bf16
    static constexpr uint32_t OFF_X = 0;
    static constexpr uint32_t OFF_B = OFF_X + X_BYTES;       // B [Q][N], later w o B
    static constexpr uint32_t OFF_CM = OFF_B + NB * BC_BLOCK; // C [Q][N], later M [Q][Q] (2 blocks)
    static constexpr uint32_t OFF_S = OFF_CM + 2 * BC_BLOCK;  // S bf16 [128][P] (rows >= N zero)
    static constexpr uint32_t OFF_ZERO = OFF_S + 128 * XROW;  // a zero [Q][64] block (N = 64)
    static constexpr uint32_t OFF_CUM = OFF_ZERO + (N == 64 ? BC_BLOCK : 0);   // cum [Q], totals
    static constexpr uint32_t OFF_EA = OFF_CUM + 4 * (Q + 8);                   // e^{a} [Q]
    static constexpr uint32_t OFF_EAI = OFF_EA + 4 * Q;                         // e^{-a} [Q]
    static constexpr uint32_t OFF_BAR = OFF_EAI + 4 * Q;
    static constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;   // + alignment slack
    static constexpr uint32_t TX_BYTES = X_BYTES + 2 * NB * BC_BLOCK;
    // tensor memory columns: G (then D), Yc, Yi
    static constexpr uint32_t TM_G = 0, TM_YC = Q, TM_YI = Q + P;
    static constexpr uint32_t TM_COLS = 256;
    static_assert(TM_YI + P <= TM_COLS, "tensor-memory columns");
    static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");
};

// SM cycles an mbarrier wait may take before the kernel gives up (about a second)
constexpr long long kSsdWaitCycles = 2000000000LL;

// `W` (16 or 32) consecutive fp32 columns of this thread's tensor-memory lane, as raw
// bits; valid after tmem_wait_ld()
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
__global__ void __launch_bounds__(Cfg::NT, 2)
ssd_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
           const __grid_constant__ CUtensorMap tm_c, const SsdTcArgs p) {
    using Tout = typename Cfg::Tout;
    constexpr int P = Cfg::P, N = Cfg::N, Q = Cfg::Q, NB = Cfg::NB, XROW = Cfg::XROW;
    constexpr int PW = P >= 32 ? 32 : 16;          // columns per tensor-memory load of a P row
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *cum = reinterpret_cast<float *>(smem + Cfg::OFF_CUM);           // [Q] + warp totals
    float *ea = reinterpret_cast<float *>(smem + Cfg::OFF_EA);             // e^{a_s} [Q]
    float *eai = reinterpret_cast<float *>(smem + Cfg::OFF_EAI);           // e^{-a_s} [Q]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *bar_tma = bars + 0, *bar_g = bars + 1, *bar_d = bars + 2, *bar_yi = bars + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = tid;                          // tensor-memory lane = row of the products
    const int bh = blockIdx.x;
    const int b = bh / p.heads, h = bh - b * p.heads;
    const int L = p.seqlen, H = p.heads;
    const int nchunk = (L + Q - 1) / Q;

    if (tid == 0) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&tm_c);
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
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
    const uint32_t lane_base = uint32_t(warp * 32) << 16;   // this warp's tensor-memory lanes

    // phases of each barrier issued (counted by thread 0, which issues) and waited for
    // (counted by every thread), for the drain after a time-out
    int n_tma = 0, n_g = 0, n_d = 0, n_yi = 0;
    auto issue_loads = [&](int c) {
        mbar_arrive_expect_tx(bar_tma, Cfg::TX_BYTES);
        tma_load_4d(smem + Cfg::OFF_X, &tm_x, bar_tma, 0, h, c * Q, b);
#pragma unroll
        for (int k = 0; k < NB; ++k) {
            tma_load_4d(smem + Cfg::OFF_B + k * Cfg::BC_BLOCK, &tm_b, bar_tma, 64 * k, h, c * Q, b);
            tma_load_4d(smem + Cfg::OFF_CM + k * Cfg::BC_BLOCK, &tm_c, bar_tma, 64 * k, h, c * Q, b);
        }
        ++n_tma;
    };
    if (tid == 0) issue_loads(0);

    // the state: thread n < N holds S[p][n] for every p
    float S[P];
    const size_t sbase = size_t(bh) * P * N;
#pragma unroll
    for (int q = 0; q < P; ++q)
        S[q] = (p.h0 != nullptr && row < N) ? p.h0[sbase + size_t(q) * N + row] : 0.f;
    auto write_state = [&]() {      // bf16 copy of S as rows n of P values (MN-major operand)
        if (row < N) {
#pragma unroll
            for (int j = 0; j < P / 8; ++j) {
                uint4 v;
                v.x = pack_bf16x2(S[8 * j + 0], S[8 * j + 1]);
                v.y = pack_bf16x2(S[8 * j + 2], S[8 * j + 3]);
                v.z = pack_bf16x2(S[8 * j + 4], S[8 * j + 5]);
                v.w = pack_bf16x2(S[8 * j + 6], S[8 * j + 7]);
                *reinterpret_cast<uint4 *>(smem + Cfg::OFF_S + swz<XROW>(row, 16 * j)) = v;
            }
        }
    };
    write_state();
    fence_async_smem();
    __syncthreads();

    constexpr uint32_t ID_G = idesc_bf16(128, Q, false, false);
    constexpr uint32_t ID_YC = idesc_bf16(128, P, false, true);
    constexpr uint32_t ID_D = idesc_bf16(128, P, true, true);
    constexpr uint32_t ID_YI = idesc_bf16(128, P, false, true);
    const uint32_t s_x = smem_addr(smem + Cfg::OFF_X), s_b = smem_addr(smem + Cfg::OFF_B);
    const uint32_t s_cm = smem_addr(smem + Cfg::OFF_CM), s_s = smem_addr(smem + Cfg::OFF_S);
    const uint32_t s_zero = smem_addr(smem + Cfg::OFF_ZERO);
    // MN-major operand with rows of XROW bytes: K-step of 16 rows
    constexpr uint32_t MN_SBO = 8 * XROW, MN_KSTEP = 16 * XROW;
    // the tiles never move, so every descriptor is a base plus a byte offset / 16 in its
    // 14-bit start-address field (shared addresses stay below 2^18, so nothing carries out)
    const uint64_t dsc_cm = smem_desc(s_cm, 16, 1024, kLayoutSw128);     // C, later M: K-major
    const uint64_t dsc_b = smem_desc(s_b, 16, 1024, kLayoutSw128);       // B: K-major
    const uint64_t dsc_s = smem_desc(s_s, 8192, MN_SBO, Cfg::XLAYOUT);   // S^T: MN-major
    const uint64_t dsc_x = smem_desc(s_x, 8192, MN_SBO, Cfg::XLAYOUT);   // x: MN-major
    const uint64_t dsc_bt = smem_desc(s_b, N == 128 ? Cfg::BC_BLOCK : (s_zero - s_b), 1024, kLayoutSw128);
    auto at = [](uint64_t d, uint32_t bytes) { return d + uint64_t(bytes >> 4); };
    // every thread waits, then the block agrees: on a time-out all threads leave the loop
    // (and the phase is not counted as done, so the drain waits for it again)
    auto wait_all = [&](uint64_t *bar, int &n_done) {
        const bool mine = mbar_wait(bar, uint32_t(n_done & 1), kSsdWaitCycles);
        const bool all = __syncthreads_and(mine) != 0;
        if (all) ++n_done;
        return all;
    };
    auto load_a = [&](int c) {
        const int t = c * Q + row;
        return (c < nchunk && t < L) ? p.a[(size_t(b) * L + t) * H + h] : 0.f;
    };
    int w_tma = 0, w_g = 0, w_d = 0, w_yi = 0;
    float a_next = load_a(0);
    // the decays of chunk cc: inclusive cumulative sum over the chunk (zero past L) into
    // cum[], e^{a} and e^{-a} into ea[], eai[]; this row's cum (cs), e^{cum} (el) and the
    // chunk's total (tot).  One barrier inside; cum[] is read after the next one.
    float cs = 0.f, el = 1.f, tot = 0.f;
    auto chunk_decays = [&](int cc) {
        cs = a_next;
        a_next = load_a(cc + 1);
        ea[row] = ex2_approx(cs * kLog2e);
        eai[row] = ex2_approx(-cs * kLog2e);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, cs, o);
            if (lane >= o) cs += u;
        }
        if (lane == 31) cum[Q + warp] = cs;
        __syncthreads();
        for (int w = 0; w < warp; ++w) cs += cum[Q + w];
        tot = cum[Q] + cum[Q + 1] + cum[Q + 2] + cum[Q + 3];
        cum[row] = cs;
        el = ex2_approx(cs * kLog2e);
    };
    // MMA 1 (G = C B^T) of chunk cc, whose tiles have landed; and the L2 prefetch of the
    // chunk after it
    auto issue_g = [&](int cc) {
        tc_fence_after_sync();
#pragma unroll
        for (int k = 0; k < N / 16; ++k) {
            const uint32_t koff = (k >> 2) * Cfg::BC_BLOCK + (k & 3) * 32;
            umma_bf16(tmem + Cfg::TM_G, at(dsc_cm, koff), at(dsc_b, koff), ID_G, k > 0);
        }
        if (cc + 1 < nchunk) {
            tma_prefetch_l2_4d(&tm_x, 0, h, (cc + 1) * Q, b);
#pragma unroll
            for (int k = 0; k < NB; ++k) {
                tma_prefetch_l2_4d(&tm_b, 64 * k, h, (cc + 1) * Q, b);
                tma_prefetch_l2_4d(&tm_c, 64 * k, h, (cc + 1) * Q, b);
            }
        }
    };
    // MMA 2 (Yc = C S^T, S the state entering the chunk), then one commit for MMAs 1 and 2:
    // the masking waits for both, since it overwrites C
    auto issue_yc = [&]() {
        tc_fence_after_sync();
#pragma unroll
        for (int k = 0; k < N / 16; ++k) {
            const uint32_t koff = (k >> 2) * Cfg::BC_BLOCK + (k & 3) * 32;
            umma_bf16(tmem + Cfg::TM_YC, at(dsc_cm, koff), at(dsc_s, k * MN_KSTEP), ID_YC, k > 0);
        }
        umma_commit(bar_g);
        ++n_g;
    };
    chunk_decays(0);
    bool ok = wait_all(bar_tma, w_tma);
    if (ok && tid == 0) {
        issue_g(0);
        issue_yc();
    }
    int c = 0;
    for (; ok && c < nchunk; ++c) {
        const int t = c * Q + row;

        // masked scores from G (row l): e^{cum_l - cum_s} for s <= l, 0 above, as bf16 over
        // C (its products are complete); then B's row s times w_s = e^{tot - cum_s}
        if (!(ok = wait_all(bar_g, w_g))) break;
        tc_fence_after_sync();
#pragma unroll
        for (int jb = 0; jb < Q / 32; ++jb) {
            const int s0b = 32 * jb;
            unsigned char *mblk = smem + Cfg::OFF_CM + (s0b >> 6) * Cfg::BC_BLOCK;
            if (s0b > 32 * warp + 31) {                  // wholly above this warp's rows
#pragma unroll
                for (int j8 = 0; j8 < 4; ++j8)
                    *reinterpret_cast<uint4 *>(mblk + swz<128>(row, 2 * ((s0b & 63) + 8 * j8))) =
                        make_uint4(0u, 0u, 0u, 0u);
                continue;
            }
            uint32_t graw[32];
            tmem_ld32_async(tmem + lane_base + Cfg::TM_G + s0b, graw);
            tmem_wait_ld();
            float m[32];
            if (s0b + 31 < 32 * warp) {
                // wholly below the diagonal: one exponential for the block's last column,
                // then e^{cum_l - cum_(s-1)} = e^{cum_l - cum_s} e^{a_s} down the columns
                // (decreasing, so an underflow to 0 is the true value's)
                float dec = ex2_approx((cs - cum[s0b + 31]) * kLog2e);
#pragma unroll
                for (int e = 31; e >= 0; --e) {
                    m[e] = __uint_as_float(graw[e]) * dec;
                    dec *= ea[s0b + e];
                }
            } else if (fabsf(cum[s0b] - cum[s0b + 31]) <= 80.f) {
                // the diagonal block, its 32 decays within a factor e^80: one exponential
                // for the first column, then e^{cum_l - cum_(s+1)} = e^{cum_l - cum_s} e^{-a_(s+1)}
                // up the columns (0 above the diagonal, whatever the product there)
                float dec = ex2_approx((cs - cum[s0b]) * kLog2e);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    m[e] = s0b + e <= row ? __uint_as_float(graw[e]) * dec : 0.f;
                    if (e < 31) dec *= eai[s0b + e + 1];
                }
            } else {
                // the diagonal block otherwise: one exponential per score
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int s = s0b + e;
                    const float dec = ex2_approx((cs - cum[s]) * kLog2e);
                    m[e] = s <= row ? __uint_as_float(graw[e]) * dec : 0.f;
                }
            }
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8) {
                uint4 v;
                v.x = pack_bf16x2(m[8 * j8 + 0], m[8 * j8 + 1]); v.y = pack_bf16x2(m[8 * j8 + 2], m[8 * j8 + 3]);
                v.z = pack_bf16x2(m[8 * j8 + 4], m[8 * j8 + 5]); v.w = pack_bf16x2(m[8 * j8 + 6], m[8 * j8 + 7]);
                *reinterpret_cast<uint4 *>(mblk + swz<128>(row, 2 * ((s0b & 63) + 8 * j8))) = v;
            }
        }
        {
            const float w = ex2_approx((tot - cs) * kLog2e);
#pragma unroll
            for (int k = 0; k < NB; ++k) {
                unsigned char *bblk = smem + Cfg::OFF_B + k * Cfg::BC_BLOCK;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 *q = reinterpret_cast<uint4 *>(bblk + swz<128>(row, 16 * j));
                    const uint4 v = *q;
                    const unsigned vv[4] = {v.x, v.y, v.z, v.w};
                    unsigned o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        o[e] = pack_bf16x2(__uint_as_float(vv[e] << 16) * w,
                                           __uint_as_float(vv[e] & 0xffff0000u) * w);
                    *q = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        // MMA 3: D = (w o B)^T x into G's columns (rows n: B^T MN-major, 64-state blocks LBO
        // apart); MMA 4: Yi = M x
        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int k = 0; k < Q / 16; ++k)
                umma_bf16(tmem + Cfg::TM_G, at(dsc_bt, k * 2048), at(dsc_x, k * MN_KSTEP), ID_D, k > 0);
            umma_commit(bar_d);
            ++n_d;
#pragma unroll
            for (int k = 0; k < Q / 16; ++k) {
                const uint32_t koff = (k >> 2) * Cfg::BC_BLOCK + (k & 3) * 32;
                umma_bf16(tmem + Cfg::TM_YI, at(dsc_cm, koff), at(dsc_x, k * MN_KSTEP), ID_YI, k > 0);
            }
            umma_commit(bar_yi);
            ++n_yi;
        }
        // every product reading this chunk's tiles is done: the next chunk's loads go out
        if (!(ok = wait_all(bar_d, w_d))) break;
        if (!(ok = wait_all(bar_yi, w_yi))) break;
        tc_fence_after_sync();
        if (tid == 0 && c + 1 < nchunk) issue_loads(c + 1);
        // the state: S' = e^{tot} S + D (row n); MMA 2 has read the old copy
        {
            const float dtot = ex2_approx(tot * kLog2e);
            uint32_t d[P];
#pragma unroll
            for (int j = 0; j < P; j += PW) tmem_ld_cols<PW>(tmem + lane_base + Cfg::TM_G + j, d + j);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < P; ++e) S[e] = fmaf(dtot, S[e], __uint_as_float(d[e]));
            write_state();
        }
        // the next chunk's decays, and its MMA 1 once its tiles land (G's columns are free:
        // D has been read), so that the product runs while this chunk's y is written
        const float el_c = el;
        const bool more = c + 1 < nchunk;
        if (more) {
            chunk_decays(c + 1);
            fence_async_smem();
            tc_fence_before_sync();
            if (!(ok = wait_all(bar_tma, w_tma))) break;
            if (tid == 0) issue_g(c + 1);
        }
        // y = Yi + e^{cum_l} Yc, row l
        {
            Tout *yrow = static_cast<Tout *>(p.y) + ((size_t(b) * L + t) * H + h) * P;
#pragma unroll
            for (int j = 0; j < P; j += PW) {
                uint32_t yir[PW], ycr[PW];
                tmem_ld_cols<PW>(tmem + lane_base + Cfg::TM_YI + j, yir);
                tmem_ld_cols<PW>(tmem + lane_base + Cfg::TM_YC + j, ycr);
                tmem_wait_ld();
                float yv[PW];
#pragma unroll
                for (int e = 0; e < PW; ++e) yv[e] = fmaf(el_c, __uint_as_float(ycr[e]), __uint_as_float(yir[e]));
                if (t < L) {
#pragma unroll
                    for (int e = 0; e < PW; e += 8) store_run<8>(yrow + j + e, yv + e);
                }
            }
        }
        // every tensor-memory read of Yc and Yi is done before the next chunk's MMA 2 and
        // MMA 4 overwrite them; the new S copy reaches MMA 2
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        if (more && tid == 0) issue_yc();
    }
    if (ok) {
        if (p.hN != nullptr && row < N) {
#pragma unroll
            for (int q = 0; q < P; ++q) p.hN[sbase + size_t(q) * N + row] = S[q];
        }
    } else if (tid == 0) {
        // a wait gave up: report it, then let whatever this CTA still has in flight finish,
        // each wait bounded
        if (p.timeouts != nullptr) atomicAdd(p.timeouts, 1u);
        for (int k = w_tma; k < n_tma; ++k) mbar_wait(bar_tma, uint32_t(k & 1), kSsdWaitCycles);
        for (int k = w_g; k < n_g; ++k) mbar_wait(bar_g, uint32_t(k & 1), kSsdWaitCycles);
        for (int k = w_d; k < n_d; ++k) mbar_wait(bar_d, uint32_t(k & 1), kSsdWaitCycles);
        for (int k = w_yi; k < n_yi; ++k) mbar_wait(bar_yi, uint32_t(k & 1), kSsdWaitCycles);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, Cfg::TM_COLS);
}

}  // namespace ssm
