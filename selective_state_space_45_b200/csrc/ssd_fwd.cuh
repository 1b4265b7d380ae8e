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
// Layout of the work: three kernels, the first and last with one CTA (8 warps) per
// (sequence, head, chunk), so the grid grows with the sequence length:
//   ssd_chunk_state_kernel  dS_c = B^T (w o x) with w_s = exp(cum_{Q-1} - cum_s): what the
//                           chunk adds to the state (fp32), and the chunk's total decay;
//   ssd_state_pass_kernel   the recurrence between chunks, elementwise over the P x N
//                           state: E_0 = h0, E_{c+1} = exp(total_c) E_c + dS_c (fp32 carry),
//                           E_c kept as a bf16 operand; the final state;
//   ssd_chunk_scan_kernel   G = C B^T, the masked scores M (bf16), Y = M x and
//                           Y' = C E_c^T on the tensor cores, y = Y + exp(cum) Y' (fp32).
// Products use bf16 operands with fp32 accumulation in 16x16x16 WMMA tiles.
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
    float *dS;                // scratch [batch*heads][nchunk][N][P]: chunk contributions
    __nv_bfloat16 *E;         // scratch [batch*heads][nchunk][N][P]: entering states
    float *tot;               // scratch [batch*heads][nchunk]: chunk total decays
    int batch, seqlen, heads, nchunk;
};

template <int P_, int N_, typename Tout_>
struct SsdCfg {
    using Tout = Tout_;
    static constexpr int P = P_, N = N_, Q = 64, NT = 256, NW = 8;
    static constexpr int LDP = P + 8;        // bf16 rows of P (x, w o x, E)
    static constexpr int LDN = N + 8;        // bf16 rows of N (B, C)
    static constexpr int LDQ = Q + 8;        // bf16 rows of Q (masked scores)
    static constexpr int LDF = P + 4;        // fp32 rows of P (Y, Y')
    static constexpr int LDG = Q + 4;        // fp32 rows of Q (scores)
    static_assert(P % 16 == 0 && N % 16 == 0, "whole 16x16 tiles");

    static constexpr size_t al(size_t v) { return (v + 127) & ~size_t(127); }
    static constexpr size_t XS = al(size_t(Q) * LDP * 2);
    static constexpr size_t BS = al(size_t(Q) * LDN * 2);
    static constexpr size_t ES = al(size_t(N) * LDP * 2);
    static constexpr size_t GS = al(size_t(Q) * (LDG > LDF ? LDG : LDF) * 4);
    static constexpr size_t FS = al(size_t(Q) * LDF * 4);
    static constexpr size_t MS = al(size_t(Q) * LDQ * 2);
    static constexpr size_t CUMS = al(size_t(Q + 4) * 4);
    // chunk-state kernel: x, B, w o x, cum, the [N][P] fp32 result staged for row stores
    static constexpr size_t ST_X = 0, ST_B = ST_X + XS, ST_XW = ST_B + BS, ST_CUM = ST_XW + XS;
    static constexpr size_t ST_OUT = ST_CUM + CUMS;
    static constexpr size_t ST_SMEM = ST_OUT + al(size_t(N) * LDF * 4);
    // chunk-scan kernel: x, B, C, E, scores / Y, Y', masked scores, cum
    static constexpr size_t SC_X = 0, SC_B = SC_X + XS, SC_C = SC_B + BS, SC_E = SC_C + BS;
    static constexpr size_t SC_G = SC_E + ES, SC_Y2 = SC_G + GS, SC_M = SC_Y2 + FS;
    static constexpr size_t SC_CUM = SC_M + MS;
    static constexpr size_t SC_SMEM = SC_CUM + CUMS;
};

// Stage rows t0 .. t0+Q-1 of a [batch][L][heads][W] bf16 tensor for (b, h) into rows of
// `ld` elements (16-byte cp.async copies); rows past L become zeros.
template <int W, int Q, int NT>
__device__ __forceinline__ void ssd_stage_rows(__nv_bfloat16 *dst, int ld, const __nv_bfloat16 *src,
                                               int b, int h, int t0, int L, int H) {
    constexpr int CPR = W / 8;
    for (int i = tid_x(); i < Q * CPR; i += NT) {
        const int l = i / CPR, k = i % CPR;
        __nv_bfloat16 *d = dst + l * ld + 8 * k;
        const int t = t0 + l;
        if (t < L)
            cp_async_16(d, src + ((size_t(b) * L + t) * H + h) * W + 8 * k);
        else
            *reinterpret_cast<uint4 *>(d) = make_uint4(0u, 0u, 0u, 0u);
    }
}

// cum[l] = a_{t0} + ... + a_{t0+l} for l < Q (zero decay past L), cum[Q] = the chunk total.
// One warp, two tokens per lane.
template <int Q>
__device__ __forceinline__ void ssd_chunk_cumsum(const SsdArgs &p, float *cum, int b, int h, int t0) {
    static_assert(Q == 64, "two tokens per lane of one warp");
    const int lane = tid_x() & 31;
    const int L = p.seqlen, H = p.heads;
    const int ta = t0 + 2 * lane, tb = ta + 1;
    const float v0 = ta < L ? p.a[(size_t(b) * L + ta) * H + h] : 0.f;
    const float v1 = tb < L ? p.a[(size_t(b) * L + tb) * H + h] : 0.f;
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

// What chunk c of (b, h) adds to the state, dS = B^T (w o x), and its total decay.
template <class Cfg>
__global__ void __launch_bounds__(Cfg::NT, 2) ssd_chunk_state_kernel(const SsdArgs p) {
    namespace wm = nvcuda::wmma;
    using bf16 = __nv_bfloat16;
    constexpr int P = Cfg::P, N = Cfg::N, Q = Cfg::Q, NT = Cfg::NT, NW = Cfg::NW;
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5;
    const int bh = blockIdx.x / p.nchunk, c = blockIdx.x - bh * p.nchunk;
    const int b = bh / p.heads, h = bh - b * p.heads;
    const int t0 = c * Q;
    bf16 *xs = reinterpret_cast<bf16 *>(smem + Cfg::ST_X);
    bf16 *bs = reinterpret_cast<bf16 *>(smem + Cfg::ST_B);
    bf16 *xw = reinterpret_cast<bf16 *>(smem + Cfg::ST_XW);
    float *cum = reinterpret_cast<float *>(smem + Cfg::ST_CUM);
    ssd_stage_rows<P, Q, NT>(xs, Cfg::LDP, p.x, b, h, t0, p.seqlen, p.heads);
    ssd_stage_rows<N, Q, NT>(bs, Cfg::LDN, p.B, b, h, t0, p.seqlen, p.heads);
    cp_async_commit();
    if (warp == 0) ssd_chunk_cumsum<Q>(p, cum, b, h, t0);
    cp_async_wait<0>();
    __syncthreads();
    const float total = cum[Q];
    if (tid == 0) p.tot[blockIdx.x] = total;
    for (int i = tid; i < Q * P; i += NT) {
        const int s = i / P, pp = i % P;
        const float w = ex2_approx((total - cum[s]) * kLog2e);
        xw[s * Cfg::LDP + pp] = __float2bfloat16_rn(w * __bfloat162float(xs[s * Cfg::LDP + pp]));
    }
    __syncthreads();
    float *outs = reinterpret_cast<float *>(smem + Cfg::ST_OUT);   // [N][LDF]
    for (int tile = warp; tile < (N / 16) * (P / 16); tile += NW) {
        const int i = tile / (P / 16), j = tile % (P / 16);   // rows n, columns p
        wm::fragment<wm::accumulator, 16, 16, 16, float> acc;
        wm::fill_fragment(acc, 0.f);
#pragma unroll
        for (int k = 0; k < Q / 16; ++k) {
            wm::fragment<wm::matrix_a, 16, 16, 16, bf16, wm::col_major> fa;   // B^T
            wm::fragment<wm::matrix_b, 16, 16, 16, bf16, wm::row_major> fb;   // w o x
            wm::load_matrix_sync(fa, bs + (16 * k) * Cfg::LDN + 16 * i, Cfg::LDN);
            wm::load_matrix_sync(fb, xw + (16 * k) * Cfg::LDP + 16 * j, Cfg::LDP);
            wm::mma_sync(acc, fa, fb, acc);
        }
        wm::store_matrix_sync(outs + (16 * i) * Cfg::LDF + 16 * j, acc, Cfg::LDF, wm::mem_row_major);
    }
    __syncthreads();
    float4 *dS = reinterpret_cast<float4 *>(p.dS + size_t(blockIdx.x) * N * P);   // [N][P]
    for (int i = tid; i < N * P / 4; i += NT) {
        const int n = i / (P / 4), k = i % (P / 4);
        dS[i] = *reinterpret_cast<const float4 *>(outs + n * Cfg::LDF + 4 * k);
    }
}

// The recurrence between chunks for (b, h): thread element e of the P x N state, over the
// chunks in order.  E_c (the state entering chunk c) is written as a bf16 operand.
template <class Cfg>
__global__ void __launch_bounds__(256) ssd_state_pass_kernel(const SsdArgs p) {
    constexpr int P = Cfg::P, N = Cfg::N;
    const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long total = static_cast<long long>(p.batch) * p.heads * N * P;
    if (e >= total) return;
    const long long bh = e / (N * P);
    const int r = int(e - bh * (N * P));                       // n * P + p
    const int n = r / P, pp = r % P;
    const long long sidx = (bh * P + pp) * N + n;              // [batch][heads][P][N]
    float S = p.h0 != nullptr ? p.h0[sidx] : 0.f;
    const size_t base = size_t(bh) * p.nchunk;
    const float *__restrict__ dS = p.dS;
    const float *__restrict__ tot = p.tot;
    __nv_bfloat16 *__restrict__ E = p.E;
    constexpr int K = 8;                         // chunks whose inputs are loaded together
    for (int c0 = 0; c0 < p.nchunk; c0 += K) {
        float dv[K], dec[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int c = c0 + k;
            const bool ok = c < p.nchunk;
            dv[k] = ok ? __ldg(dS + (base + c) * (N * P) + r) : 0.f;
            dec[k] = ok ? __ldg(tot + base + c) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int c = c0 + k;
            if (c < p.nchunk) {
                E[(base + c) * (N * P) + r] = __float2bfloat16_rn(S);
                S = fmaf(ex2_approx(dec[k] * kLog2e), S, dv[k]);
            }
        }
    }
    if (p.hN != nullptr) p.hN[sidx] = S;
}

// Outputs of chunk c of (b, h): attention with the decay mask inside the chunk plus what
// every position reads from the entering state.
template <class Cfg>
__global__ void __launch_bounds__(Cfg::NT, 2) ssd_chunk_scan_kernel(const SsdArgs p) {
    namespace wm = nvcuda::wmma;
    using Tout = typename Cfg::Tout;
    using bf16 = __nv_bfloat16;
    constexpr int P = Cfg::P, N = Cfg::N, Q = Cfg::Q, NT = Cfg::NT, NW = Cfg::NW;
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5;
    const int bh = blockIdx.x / p.nchunk, c = blockIdx.x - bh * p.nchunk;
    const int b = bh / p.heads, h = bh - b * p.heads;
    const int t0 = c * Q, L = p.seqlen, H = p.heads;
    bf16 *xs = reinterpret_cast<bf16 *>(smem + Cfg::SC_X);
    bf16 *bs = reinterpret_cast<bf16 *>(smem + Cfg::SC_B);
    bf16 *cs = reinterpret_cast<bf16 *>(smem + Cfg::SC_C);
    bf16 *es = reinterpret_cast<bf16 *>(smem + Cfg::SC_E);
    float *G = reinterpret_cast<float *>(smem + Cfg::SC_G);      // scores, later Y
    float *Y2 = reinterpret_cast<float *>(smem + Cfg::SC_Y2);    // C E^T
    bf16 *M = reinterpret_cast<bf16 *>(smem + Cfg::SC_M);
    float *cum = reinterpret_cast<float *>(smem + Cfg::SC_CUM);
    ssd_stage_rows<P, Q, NT>(xs, Cfg::LDP, p.x, b, h, t0, L, H);
    ssd_stage_rows<N, Q, NT>(bs, Cfg::LDN, p.B, b, h, t0, L, H);
    ssd_stage_rows<N, Q, NT>(cs, Cfg::LDN, p.C, b, h, t0, L, H);
    {   // E_c: N rows of P bf16
        const bf16 *src = p.E + size_t(blockIdx.x) * N * P;
        constexpr int CPR = P / 8;
        for (int i = tid; i < N * CPR; i += NT) {
            const int n = i / CPR, k = i % CPR;
            cp_async_16(es + n * Cfg::LDP + 8 * k, src + n * P + 8 * k);
        }
    }
    cp_async_commit();
    if (warp == 0) ssd_chunk_cumsum<Q>(p, cum, b, h, t0);
    cp_async_wait<0>();
    __syncthreads();

    // G = C B^T (rows l, columns s) and Y' = C E^T (rows l, columns p): independent tiles
    for (int tile = warp; tile < (Q / 16) * (Q / 16) + (Q / 16) * (P / 16); tile += NW) {
        wm::fragment<wm::accumulator, 16, 16, 16, float> acc;
        wm::fill_fragment(acc, 0.f);
        if (tile < (Q / 16) * (Q / 16)) {
            const int i = tile / (Q / 16), j = tile % (Q / 16);
#pragma unroll
            for (int k = 0; k < N / 16; ++k) {
                wm::fragment<wm::matrix_a, 16, 16, 16, bf16, wm::row_major> fa;
                wm::fragment<wm::matrix_b, 16, 16, 16, bf16, wm::col_major> fb;
                wm::load_matrix_sync(fa, cs + (16 * i) * Cfg::LDN + 16 * k, Cfg::LDN);
                wm::load_matrix_sync(fb, bs + (16 * j) * Cfg::LDN + 16 * k, Cfg::LDN);
                wm::mma_sync(acc, fa, fb, acc);
            }
            wm::store_matrix_sync(G + (16 * i) * Cfg::LDG + 16 * j, acc, Cfg::LDG, wm::mem_row_major);
        } else {
            const int r = tile - (Q / 16) * (Q / 16);
            const int i = r / (P / 16), j = r % (P / 16);
#pragma unroll
            for (int k = 0; k < N / 16; ++k) {
                wm::fragment<wm::matrix_a, 16, 16, 16, bf16, wm::row_major> fa;
                wm::fragment<wm::matrix_b, 16, 16, 16, bf16, wm::row_major> fb;
                wm::load_matrix_sync(fa, cs + (16 * i) * Cfg::LDN + 16 * k, Cfg::LDN);
                wm::load_matrix_sync(fb, es + (16 * k) * Cfg::LDP + 16 * j, Cfg::LDP);
                wm::mma_sync(acc, fa, fb, acc);
            }
            wm::store_matrix_sync(Y2 + (16 * i) * Cfg::LDF + 16 * j, acc, Cfg::LDF, wm::mem_row_major);
        }
    }
    __syncthreads();
    for (int i = tid; i < Q * Q; i += NT) {
        const int l = i / Q, s = i % Q;
        const float v = s <= l ? G[l * Cfg::LDG + s] * ex2_approx((cum[l] - cum[s]) * kLog2e) : 0.f;
        M[l * Cfg::LDQ + s] = __float2bfloat16_rn(v);
    }
    __syncthreads();
    for (int tile = warp; tile < (Q / 16) * (P / 16); tile += NW) {      // Y = M x into G
        const int i = tile / (P / 16), j = tile % (P / 16);
        wm::fragment<wm::accumulator, 16, 16, 16, float> acc;
        wm::fill_fragment(acc, 0.f);
#pragma unroll
        for (int k = 0; k < Q / 16; ++k) {
            wm::fragment<wm::matrix_a, 16, 16, 16, bf16, wm::row_major> fa;
            wm::fragment<wm::matrix_b, 16, 16, 16, bf16, wm::row_major> fb;
            wm::load_matrix_sync(fa, M + (16 * i) * Cfg::LDQ + 16 * k, Cfg::LDQ);
            wm::load_matrix_sync(fb, xs + (16 * k) * Cfg::LDP + 16 * j, Cfg::LDP);
            wm::mma_sync(acc, fa, fb, acc);
        }
        wm::store_matrix_sync(G + (16 * i) * Cfg::LDF + 16 * j, acc, Cfg::LDF, wm::mem_row_major);
    }
    __syncthreads();
    constexpr int VP = 8;
    for (int i = tid; i < Q * (P / VP); i += NT) {
        const int l = i / (P / VP), k = i % (P / VP);
        const int t = t0 + l;
        if (t >= L) continue;
        const float e = ex2_approx(cum[l] * kLog2e);
        float o[VP];
#pragma unroll
        for (int u = 0; u < VP; ++u)
            o[u] = fmaf(e, Y2[l * Cfg::LDF + VP * k + u], G[l * Cfg::LDF + VP * k + u]);
        store8<Tout>(static_cast<Tout *>(p.y) + ((size_t(b) * L + t) * H + h) * P + VP * k, o);
    }
}

}  // namespace ssm
