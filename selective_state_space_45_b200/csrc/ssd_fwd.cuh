// ssd_fwd.cuh -- Mamba-2's state-space dual (SSD) forward by chunks, on tensor cores.
//
// What it computes (per sequence b and head h, a P x N state S, one decay per head):
//     S <- exp(a_t) S + x_t B_t^T,     y_t = S C_t
// with x already times the step and a = step * A ("Beyond attention with Mamba, state
// space models and hybrids", xmarva lesson 10, section 8 "Mamba-2: the same model as
// attention").  By chunks of Q tokens, with cum_l = a_0 + ... + a_l inside the chunk and
// S_in the state entering it:
//     y_l   = sum_{s<=l} (C_l . B_s) exp(cum_l - cum_s) x_s  +  exp(cum_l) S_in C_l
//     S_out = exp(cum_{Q-1}) S_in + sum_s exp(cum_{Q-1} - cum_s) x_s B_s^T
// -- attention with the decay as its mask inside the chunk, the recurrence between chunks.
//
// Layout of the work: one CTA (8 warps) per (sequence, head) walks its chunks in order,
// the state staying in shared memory (fp32) between chunks; the chunk inputs are staged by
// a 2-deep cp.async ring.  Per chunk four products on the tensor cores (bf16 operands,
// fp32 accumulation, 16x16x16 WMMA tiles): G = C B^T; Y = (G o mask) X; Y' = C S_in^T;
// S += B^T (w o X).  Masks, decays and the combination y = Y + exp(cum) Y' are fp32.
#pragma once

#include <mma.h>

#include "common.cuh"

namespace ssm {

struct SsdArgs {
    const __nv_bfloat16 *x;   // [batch][L][heads][P]
    const float *a;           // [batch][L][heads]
    const __nv_bfloat16 *B;   // [batch][L][heads][N]
    const __nv_bfloat16 *C;   // [batch][L][heads][N]
    void *y;                  // [batch][L][heads][P], Tout
    const float *h0;          // [batch][heads][P][N] or null
    float *hN;                // [batch][heads][P][N] or null
    int batch, seqlen, heads;
};

template <int P_, int N_, typename Tout_>
struct SsdCfg {
    using Tout = Tout_;
    static constexpr int P = P_, N = N_, Q = 64, NT = 256, NW = 8;
    static constexpr int LDP = P + 8;        // bf16 rows of P (x, w o x, S^T operand)
    static constexpr int LDN = N + 8;        // bf16 rows of N (B, C)
    static constexpr int LDQ = Q + 8;        // bf16 rows of Q (masked scores)
    static constexpr int LDF = P + 4;        // fp32 rows of P (Y, Y', state)
    static constexpr int LDG = Q + 4;        // fp32 rows of Q (scores)
    static_assert(P % 16 == 0 && N % 16 == 0, "whole 16x16 tiles");

    static constexpr size_t al(size_t v) { return (v + 127) & ~size_t(127); }
    static constexpr size_t XS = al(size_t(Q) * LDP * 2);
    static constexpr size_t BS = al(size_t(Q) * LDN * 2);
    static constexpr size_t AS = al(size_t(Q) * 4);
    static constexpr size_t STAGE = XS + 2 * BS + AS;
    static constexpr size_t OFF_STAGE = 0;                                   // 2 stages
    static constexpr size_t OFF_G = OFF_STAGE + 2 * STAGE;                   // fp32 [Q][LDG], then Y
    static constexpr size_t OFF_Y2 = OFF_G + al(size_t(Q) * (LDG > LDF ? LDG : LDF) * 4);  // fp32 [Q][LDF]
    static constexpr size_t OFF_M = OFF_Y2 + al(size_t(Q) * LDF * 4);         // bf16 [Q][LDQ]
    static constexpr size_t OFF_XW = OFF_M + al(size_t(Q) * LDQ * 2);         // bf16 [Q][LDP]
    static constexpr size_t OFF_SF = OFF_XW + al(size_t(Q) * LDP * 2);        // fp32 [N][LDF]
    static constexpr size_t OFF_SB = OFF_SF + al(size_t(N) * LDF * 4);        // bf16 [N][LDP]
    static constexpr size_t OFF_CUM = OFF_SB + al(size_t(N) * LDP * 2);       // fp32 [Q] + total
    static constexpr size_t SMEM_BYTES = OFF_CUM + al(size_t(Q + 4) * 4);
};

// Stage chunk c (tokens t0 .. t0+Q-1) of x, B, C and a for (b, h); rows past L are zero.
template <class Cfg>
__device__ __forceinline__ void ssd_load_chunk(const SsdArgs &p, unsigned char *smem, int st, int b,
                                               int h, int t0) {
    constexpr int P = Cfg::P, N = Cfg::N, Q = Cfg::Q, NT = Cfg::NT;
    unsigned char *base = smem + Cfg::OFF_STAGE + size_t(st) * Cfg::STAGE;
    __nv_bfloat16 *xs = reinterpret_cast<__nv_bfloat16 *>(base);
    __nv_bfloat16 *bs = reinterpret_cast<__nv_bfloat16 *>(base + Cfg::XS);
    __nv_bfloat16 *cs = reinterpret_cast<__nv_bfloat16 *>(base + Cfg::XS + Cfg::BS);
    float *as = reinterpret_cast<float *>(base + Cfg::XS + 2 * Cfg::BS);
    const int L = p.seqlen, H = p.heads;
    constexpr int XC = P / 8, BC = N / 8;     // 16-byte chunks per row
    for (int i = tid_x(); i < Q * XC; i += NT) {
        const int l = i / XC, k = i % XC;
        __nv_bfloat16 *dst = xs + l * Cfg::LDP + 8 * k;
        const int t = t0 + l;
        if (t < L)
            cp_async_16(dst, p.x + ((size_t(b) * L + t) * H + h) * P + 8 * k);
        else
            *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int i = tid_x(); i < 2 * Q * BC; i += NT) {
        const int which = i / (Q * BC);
        const int r = i % (Q * BC);
        const int l = r / BC, k = r % BC;
        __nv_bfloat16 *dst = (which ? cs : bs) + l * Cfg::LDN + 8 * k;
        const int t = t0 + l;
        if (t < L)
            cp_async_16(dst, (which ? p.C : p.B) + ((size_t(b) * L + t) * H + h) * N + 8 * k);
        else
            *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int l = tid_x(); l < Q; l += NT) {
        const int t = t0 + l;
        as[l] = t < L ? p.a[(size_t(b) * L + t) * H + h] : 0.f;   // no-op tokens: no decay
    }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::NT, 1) ssd_fwd_kernel(const SsdArgs p) {
    namespace wm = nvcuda::wmma;
    using Tout = typename Cfg::Tout;
    using bf16 = __nv_bfloat16;
    constexpr int P = Cfg::P, N = Cfg::N, Q = Cfg::Q, NT = Cfg::NT, NW = Cfg::NW;
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int b = bh / p.heads, h = bh - b * p.heads;
    const int L = p.seqlen, H = p.heads;
    const int nchunk = (L + Q - 1) / Q;

    float *G = reinterpret_cast<float *>(smem + Cfg::OFF_G);      // scores, later Y
    float *Y2 = reinterpret_cast<float *>(smem + Cfg::OFF_Y2);    // C S_in^T
    bf16 *M = reinterpret_cast<bf16 *>(smem + Cfg::OFF_M);        // masked scores
    bf16 *XW = reinterpret_cast<bf16 *>(smem + Cfg::OFF_XW);      // w o x
    float *SF = reinterpret_cast<float *>(smem + Cfg::OFF_SF);    // state, [N][P] (transposed)
    bf16 *SB = reinterpret_cast<bf16 *>(smem + Cfg::OFF_SB);      // state as a bf16 operand
    float *cum = reinterpret_cast<float *>(smem + Cfg::OFF_CUM);  // cum[0..Q), cum[Q] = total

    // the entering state of chunk 0, stored transposed: SF[n][p] = S[p][n]
    for (int i = tid; i < N * P; i += NT) {
        const int n = i / P, pp = i % P;
        SF[n * Cfg::LDF + pp] = p.h0 != nullptr ? p.h0[((size_t(b) * H + h) * P + pp) * N + n] : 0.f;
    }
    ssd_load_chunk<Cfg>(p, smem, 0, b, h, 0);
    cp_async_commit();

    for (int c = 0; c < nchunk; ++c) {
        const int t0 = c * Q;
        cp_async_wait<0>();
        __syncthreads();
        if (c + 1 < nchunk) ssd_load_chunk<Cfg>(p, smem, (c + 1) & 1, b, h, t0 + Q);
        cp_async_commit();
        unsigned char *sb = smem + Cfg::OFF_STAGE + size_t(c & 1) * Cfg::STAGE;
        const bf16 *xs = reinterpret_cast<const bf16 *>(sb);
        const bf16 *bs = reinterpret_cast<const bf16 *>(sb + Cfg::XS);
        const bf16 *cs = reinterpret_cast<const bf16 *>(sb + Cfg::XS + Cfg::BS);
        const float *as = reinterpret_cast<const float *>(sb + Cfg::XS + 2 * Cfg::BS);

        // cumulative decay inside the chunk (warp 0: two tokens per lane, one warp scan);
        // the other warps form G = C B^T meanwhile
        if (warp == 0) {
            const float v0 = as[2 * lane], v1 = as[2 * lane + 1];
            float s = v0 + v1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float o = __shfl_up_sync(0xffffffffu, s, off);
                if (lane >= off) s += o;
            }
            cum[2 * lane + 1] = s;
            cum[2 * lane] = s - v1;
            if (lane == 31) cum[Q] = s;
        }
        // G = C B^T: 16 tiles of 16x16 (rows l, columns s), K = N
        for (int tile = warp; tile < (Q / 16) * (Q / 16); tile += NW) {
            const int i = tile / (Q / 16), j = tile % (Q / 16);
            wm::fragment<wm::accumulator, 16, 16, 16, float> acc;
            wm::fill_fragment(acc, 0.f);
#pragma unroll
            for (int k = 0; k < N / 16; ++k) {
                wm::fragment<wm::matrix_a, 16, 16, 16, bf16, wm::row_major> fa;
                wm::fragment<wm::matrix_b, 16, 16, 16, bf16, wm::col_major> fb;
                wm::load_matrix_sync(fa, cs + (16 * i) * Cfg::LDN + 16 * k, Cfg::LDN);
                wm::load_matrix_sync(fb, bs + (16 * j) * Cfg::LDN + 16 * k, Cfg::LDN);
                wm::mma_sync(acc, fa, fb, acc);
            }
            wm::store_matrix_sync(G + (16 * i) * Cfg::LDG + 16 * j, acc, Cfg::LDG, wm::mem_row_major);
        }
        __syncthreads();

        // masked scores, w o x and the state as a bf16 operand (all fp32 arithmetic)
        const float total = cum[Q];
        for (int i = tid; i < Q * Q; i += NT) {
            const int l = i / Q, s = i % Q;
            const float v = s <= l ? G[l * Cfg::LDG + s] * ex2_approx((cum[l] - cum[s]) * kLog2e) : 0.f;
            M[l * Cfg::LDQ + s] = __float2bfloat16_rn(v);
        }
        for (int i = tid; i < Q * P; i += NT) {
            const int s = i / P, pp = i % P;
            const float w = ex2_approx((total - cum[s]) * kLog2e);
            XW[s * Cfg::LDP + pp] = __float2bfloat16_rn(w * __bfloat162float(xs[s * Cfg::LDP + pp]));
        }
        for (int i = tid; i < N * P; i += NT) {
            const int n = i / P, pp = i % P;
            SB[n * Cfg::LDP + pp] = __float2bfloat16_rn(SF[n * Cfg::LDF + pp]);
        }
        __syncthreads();

        // Y = M X (into G's space) and Y' = C S_in^T: 16 tiles each (rows l, columns p)
        for (int tile = warp; tile < 2 * (Q / 16) * (P / 16); tile += NW) {
            const int which = tile / ((Q / 16) * (P / 16));
            const int r = tile % ((Q / 16) * (P / 16));
            const int i = r / (P / 16), j = r % (P / 16);
            wm::fragment<wm::accumulator, 16, 16, 16, float> acc;
            wm::fill_fragment(acc, 0.f);
            if (which == 0) {
#pragma unroll
                for (int k = 0; k < Q / 16; ++k) {
                    wm::fragment<wm::matrix_a, 16, 16, 16, bf16, wm::row_major> fa;
                    wm::fragment<wm::matrix_b, 16, 16, 16, bf16, wm::row_major> fb;
                    wm::load_matrix_sync(fa, M + (16 * i) * Cfg::LDQ + 16 * k, Cfg::LDQ);
                    wm::load_matrix_sync(fb, xs + (16 * k) * Cfg::LDP + 16 * j, Cfg::LDP);
                    wm::mma_sync(acc, fa, fb, acc);
                }
                wm::store_matrix_sync(G + (16 * i) * Cfg::LDF + 16 * j, acc, Cfg::LDF, wm::mem_row_major);
            } else {
#pragma unroll
                for (int k = 0; k < N / 16; ++k) {
                    wm::fragment<wm::matrix_a, 16, 16, 16, bf16, wm::row_major> fa;
                    wm::fragment<wm::matrix_b, 16, 16, 16, bf16, wm::row_major> fb;
                    wm::load_matrix_sync(fa, cs + (16 * i) * Cfg::LDN + 16 * k, Cfg::LDN);
                    wm::load_matrix_sync(fb, SB + (16 * k) * Cfg::LDP + 16 * j, Cfg::LDP);
                    wm::mma_sync(acc, fa, fb, acc);
                }
                wm::store_matrix_sync(Y2 + (16 * i) * Cfg::LDF + 16 * j, acc, Cfg::LDF, wm::mem_row_major);
            }
        }
        __syncthreads();

        // y = Y + exp(cum_l) Y' to global; the state S <- exp(total) S + B^T (w o x)
        {
            constexpr int VP = 8;                   // outputs per thread per pass
            for (int i = tid; i < Q * (P / VP); i += NT) {
                const int l = i / (P / VP), k = i % (P / VP);
                const int t = t0 + l;
                if (t >= L) continue;
                const float e = ex2_approx(cum[l] * kLog2e);
                float o[VP];
#pragma unroll
                for (int u = 0; u < VP; ++u)
                    o[u] = fmaf(e, Y2[l * Cfg::LDF + VP * k + u], G[l * Cfg::LDF + VP * k + u]);
                Tout *dst = static_cast<Tout *>(p.y) + ((size_t(b) * L + t) * H + h) * P + VP * k;
                store8<Tout>(dst, o);
            }
        }
        {
            const float et = ex2_approx(total * kLog2e);
            for (int tile = warp; tile < (N / 16) * (P / 16); tile += NW) {
                const int i = tile / (P / 16), j = tile % (P / 16);     // rows n, columns p
                wm::fragment<wm::accumulator, 16, 16, 16, float> acc;
                wm::load_matrix_sync(acc, SF + (16 * i) * Cfg::LDF + 16 * j, Cfg::LDF, wm::mem_row_major);
#pragma unroll
                for (int e = 0; e < acc.num_elements; ++e) acc.x[e] *= et;
#pragma unroll
                for (int k = 0; k < Q / 16; ++k) {
                    wm::fragment<wm::matrix_a, 16, 16, 16, bf16, wm::col_major> fa;   // B^T
                    wm::fragment<wm::matrix_b, 16, 16, 16, bf16, wm::row_major> fb;   // w o x
                    wm::load_matrix_sync(fa, bs + (16 * k) * Cfg::LDN + 16 * i, Cfg::LDN);
                    wm::load_matrix_sync(fb, XW + (16 * k) * Cfg::LDP + 16 * j, Cfg::LDP);
                    wm::mma_sync(acc, fa, fb, acc);
                }
                wm::store_matrix_sync(SF + (16 * i) * Cfg::LDF + 16 * j, acc, Cfg::LDF, wm::mem_row_major);
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    if (p.hN != nullptr) {
        for (int i = tid; i < P * N; i += NT) {
            const int pp = i / N, n = i % N;
            p.hN[((size_t(b) * H + h) * P + pp) * N + n] = SF[n * Cfg::LDF + pp];
        }
    }
}

}  // namespace ssm
