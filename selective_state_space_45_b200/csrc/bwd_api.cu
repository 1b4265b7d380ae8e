// bwd_api.cu -- C ABI of the backward of the selective scan (ssm_selective_scan_bwd).
//
// Arguments are checked on the host before anything is launched.  One call: a
// stream-ordered scratch buffer (tile checkpoints and partial sums), the backward kernel,
// then the fixed-order reductions of the partial sums, all on the caller's stream.
#include <algorithm>
#include <climits>

#include "api_host.cuh"
#include "scan_bwd.cuh"

using namespace ssm_host;

namespace {

template <typename To>
int launch_reduce(const float *in, To *out, long long outer, int K, long long R, int NPin, int Nout,
                  cudaStream_t s) {
    const long long total = outer * R * Nout;
    if (total == 0) return SSM_OK;
    if (NPin == Nout && Nout % 4 == 0) {   // whole 16-byte rows: the vectorised form
        const long long groups = total / 4;
        const long long blocks = std::min<long long>((groups + 255) / 256, 148LL * 16);
        ssm::reduce_partials_vec4_kernel<To><<<unsigned(blocks), 256, 0, s>>>(in, out, outer, K,
                                                                              R * Nout / 4);
        return status_of(cudaGetLastError());
    }
    const long long blocks = std::min<long long>((total + 255) / 256, 148LL * 16);
    ssm::reduce_partials_kernel<To><<<unsigned(blocks), 256, 0, s>>>(in, out, outer, K, R, NPin, Nout);
    return status_of(cudaGetLastError());
}

template <typename Tin, typename Tg, bool VEC>
int run_bwd(ssm::BwdArgs a, void *dB, void *dC, float *dA, float *dD, float *ddelta_bias,
            cudaStream_t stream) {
    using Cfg = ssm::BwdCfg<Tin, Tg, VEC>;
    const long long groups = (a.dim + Cfg::CH - 1) / Cfg::CH;
    const long long ctas = groups * a.batch;
    if (ctas > INT_MAX || groups > INT_MAX) return SSM_ERR_UNSUPPORTED;
    a.groups_per_seq = int(groups);
    a.ntiles = (a.seqlen + Cfg::T - 1) / Cfg::T;
    const size_t ck_floats = size_t(ctas) * a.ntiles * (Cfg::T / 4) * Cfg::NP * 32;
    const size_t bc_floats = 2 * size_t(ctas) * a.seqlen * Cfg::NP;
    const size_t pa_floats = size_t(a.batch) * a.dim * Cfg::NP;
    const size_t pd_floats = 2 * size_t(a.batch) * a.dim;
    void *ws = nullptr;
    if (cudaMallocAsync(&ws, (ck_floats + bc_floats + pa_floats + pd_floats) * sizeof(float), stream) !=
        cudaSuccess)
        return SSM_ERR_CUDA;
    a.ck = static_cast<float *>(ws);
    a.part_bc = a.ck + ck_floats;
    a.part_a = a.part_bc + bc_floats;
    a.part_dd = a.part_a + pa_floats;

    int st = SSM_OK;
    const size_t smem = Cfg::SMEM_BYTES;
    if (cudaFuncSetAttribute(ssm::scan_bwd_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem)) != cudaSuccess)
        st = SSM_ERR_CUDA;
    if (st == SSM_OK) {
        ssm::scan_bwd_kernel<Cfg><<<unsigned(ctas), Cfg::NT, smem, stream>>>(a);
        st = status_of(cudaGetLastError());
    }
    const long long L = a.seqlen, N = a.dstate;
    const int G = int(groups);
    if (st == SSM_OK)   // dB, dC: sum over the channel groups of each sequence
        st = launch_reduce<Tg>(a.part_bc, static_cast<Tg *>(dB), a.batch, G, L, Cfg::NP, int(N), stream);
    if (st == SSM_OK)
        st = launch_reduce<Tg>(a.part_bc + bc_floats / 2, static_cast<Tg *>(dC), a.batch, G, L, Cfg::NP,
                               int(N), stream);
    if (st == SSM_OK)   // dA: sum over sequences
        st = launch_reduce<float>(a.part_a, dA, 1, a.batch, a.dim, Cfg::NP, int(N), stream);
    if (st == SSM_OK && dD != nullptr)
        st = launch_reduce<float>(a.part_dd, dD, 1, a.batch, a.dim, 1, 1, stream);
    if (st == SSM_OK && ddelta_bias != nullptr)
        st = launch_reduce<float>(a.part_dd + pd_floats / 2, ddelta_bias, 1, a.batch, a.dim, 1, 1, stream);
    const cudaError_t fe = cudaFreeAsync(ws, stream);
    if (st == SSM_OK && fe != cudaSuccess) st = SSM_ERR_CUDA;
    return st;
}

template <typename Tin, typename Tg>
int dispatch_bwd(const ssm::BwdArgs &a, bool vec, void *dB, void *dC, float *dA, float *dD,
                 float *ddelta_bias, cudaStream_t s) {
    return vec ? run_bwd<Tin, Tg, true>(a, dB, dC, dA, dD, ddelta_bias, s)
               : run_bwd<Tin, Tg, false>(a, dB, dC, dA, dD, ddelta_bias, s);
}

}  // namespace

extern "C" {

int ssm_selective_scan_bwd(const void *x, const void *delta, const float *delta_bias,
                           int delta_softplus, const float *A, const void *B, const void *C,
                           const float *D, const void *z, const float *initial_state,
                           const void *dy, const float *dfinal_state,
                           void *dx, void *ddelta, float *dA, void *dB, void *dC, float *dD,
                           void *dz, float *ddelta_bias, float *dinitial_state,
                           int batch, int dim, int seqlen, int dstate,
                           int in_dtype, int grad_dtype, void *cuda_stream) {
    if (!valid_dtype(in_dtype) || !valid_dtype(grad_dtype)) return SSM_ERR_INVALID_ARG;
    if (batch < 0 || dim < 0 || seqlen < 0 || dstate < 1) return SSM_ERR_INVALID_ARG;
    if (dstate > 16) return SSM_ERR_UNSUPPORTED;
    if (dz != nullptr && z == nullptr) return SSM_ERR_INVALID_ARG;
    const long long channels = (long long)batch * dim;
    const bool work = channels > 0 && seqlen > 0;
    if (channels > 0 && !dA) return SSM_ERR_INVALID_ARG;
    if (work && (!x || !delta || !A || !B || !C || !dy || !dx || !ddelta || !dB || !dC))
        return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, delta, delta_bias, A, B, C, D, z, initial_state, dy, dfinal_state,
                          dx, ddelta, dA, dB, dC, dD, dz, ddelta_bias, dinitial_state};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSM_ERR_ALIGNMENT;
    if (dim == 0) return SSM_OK;

    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (!work) {   // no tokens or no sequences: parameter gradients are zero, dh0 = dfinal
        int st = status_of(cudaMemsetAsync(dA, 0, size_t(dim) * dstate * sizeof(float), stream));
        if (st == SSM_OK && dD) st = status_of(cudaMemsetAsync(dD, 0, size_t(dim) * sizeof(float), stream));
        if (st == SSM_OK && ddelta_bias)
            st = status_of(cudaMemsetAsync(ddelta_bias, 0, size_t(dim) * sizeof(float), stream));
        if (st == SSM_OK && dinitial_state && channels > 0) {
            const size_t bytes = size_t(channels) * dstate * sizeof(float);
            st = dfinal_state ? status_of(cudaMemcpyAsync(dinitial_state, dfinal_state, bytes,
                                                          cudaMemcpyDeviceToDevice, stream))
                              : status_of(cudaMemsetAsync(dinitial_state, 0, bytes, stream));
        }
        return st;
    }

    ssm::BwdArgs a{};
    a.x = x; a.delta = delta; a.delta_bias = delta_bias; a.A = A; a.B = B; a.C = C; a.D = D; a.z = z;
    a.h0 = initial_state; a.dy = dy; a.dfinal = dfinal_state;
    a.dx = dx; a.ddelta = ddelta; a.dz = dz; a.dh0 = dinitial_state;
    a.batch = batch; a.dim = dim; a.seqlen = seqlen; a.dstate = dstate;
    a.softplus = delta_softplus ? 1 : 0;
    // 16-byte staging needs every row start on a 16-byte boundary in both dtypes
    const int ein = in_dtype == SSM_F32 ? 4 : 8;
    const int eg = grad_dtype == SSM_F32 ? 4 : 8;
    const bool vec = seqlen % ein == 0 && seqlen % eg == 0;
    if (in_dtype == SSM_F32 && grad_dtype == SSM_F32)
        return dispatch_bwd<float, float>(a, vec, dB, dC, dA, dD, ddelta_bias, stream);
    if (in_dtype == SSM_BF16 && grad_dtype == SSM_BF16)
        return dispatch_bwd<__nv_bfloat16, __nv_bfloat16>(a, vec, dB, dC, dA, dD, ddelta_bias, stream);
    if (in_dtype == SSM_BF16)
        return dispatch_bwd<__nv_bfloat16, float>(a, vec, dB, dC, dA, dD, ddelta_bias, stream);
    return dispatch_bwd<float, __nv_bfloat16>(a, vec, dB, dC, dA, dD, ddelta_bias, stream);
}

}  // extern "C"
