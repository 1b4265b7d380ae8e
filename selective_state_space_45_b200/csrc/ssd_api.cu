// ssd_api.cu -- C ABI of Mamba-2's state-space dual by chunks (ssm_ssd_fwd).
//
// Arguments are checked on the host before anything is launched; the kernel runs on the
// caller's stream, asynchronously.
#include <climits>

#include "api_host.cuh"
#include "ssd_fwd.cuh"

using namespace ssm_host;

namespace {

template <int P, int N, typename Tout>
int launch_ssd(ssm::SsdArgs a, cudaStream_t s) {
    using Cfg = ssm::SsdCfg<P, N, Tout>;
    const long long bh = (long long)a.batch * a.heads;
    const long long nchunk = (a.seqlen + Cfg::Q - 1) / Cfg::Q;
    const long long ctas = bh * nchunk;
    const long long pass_blocks = (bh * N * P + 255) / 256;
    if (ctas > INT_MAX || pass_blocks > INT_MAX) return SSM_ERR_UNSUPPORTED;
    if (ctas == 0) return SSM_OK;
    a.nchunk = int(nchunk);
    // scratch: the chunks' state contributions (fp32), their total decays, the entering
    // states (bf16)
    const size_t ds_bytes = size_t(ctas) * N * P * sizeof(float);
    const size_t tot_bytes = (size_t(ctas) * sizeof(float) + 255) & ~size_t(255);
    const size_t e_bytes = size_t(ctas) * N * P * sizeof(__nv_bfloat16);
    void *ws = nullptr;
    if (cudaMallocAsync(&ws, ds_bytes + tot_bytes + e_bytes, s) != cudaSuccess) return SSM_ERR_CUDA;
    a.dS = static_cast<float *>(ws);
    a.tot = reinterpret_cast<float *>(static_cast<char *>(ws) + ds_bytes);
    a.E = reinterpret_cast<__nv_bfloat16 *>(static_cast<char *>(ws) + ds_bytes + tot_bytes);
    int st = SSM_OK;
    if (cudaFuncSetAttribute(ssm::ssd_chunk_scan_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(Cfg::SC_SMEM)) != cudaSuccess ||
        cudaFuncSetAttribute(ssm::ssd_chunk_state_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(Cfg::ST_SMEM)) != cudaSuccess)
        st = SSM_ERR_CUDA;
    if (st == SSM_OK) {
        ssm::ssd_chunk_state_kernel<Cfg><<<unsigned(ctas), Cfg::NT, Cfg::ST_SMEM, s>>>(a);
        ssm::ssd_state_pass_kernel<Cfg><<<unsigned(pass_blocks), 256, 0, s>>>(a);
        ssm::ssd_chunk_scan_kernel<Cfg><<<unsigned(ctas), Cfg::NT, Cfg::SC_SMEM, s>>>(a);
        st = status_of(cudaGetLastError());
    }
    const cudaError_t fe = cudaFreeAsync(ws, s);
    if (st == SSM_OK && fe != cudaSuccess) st = SSM_ERR_CUDA;
    return st;
}

template <typename Tout>
int dispatch_ssd(const ssm::SsdArgs &a, int P, int N, cudaStream_t s) {
    if (P == 64 && N == 128) return launch_ssd<64, 128, Tout>(a, s);
    if (P == 64 && N == 64) return launch_ssd<64, 64, Tout>(a, s);
    if (P == 32 && N == 128) return launch_ssd<32, 128, Tout>(a, s);
    if (P == 32 && N == 64) return launch_ssd<32, 64, Tout>(a, s);
    return SSM_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

int ssm_ssd_fwd(const void *x, const float *a, const void *B, const void *C, void *y,
                const float *initial_state, float *final_state,
                int batch, int seqlen, int heads, int headdim, int dstate,
                int in_dtype, int out_dtype, void *cuda_stream) {
    if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return SSM_ERR_INVALID_ARG;
    if (batch < 0 || seqlen < 0 || heads < 0 || headdim < 1 || dstate < 1) return SSM_ERR_INVALID_ARG;
    if (in_dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
    if (!((headdim == 32 || headdim == 64) && (dstate == 64 || dstate == 128))) return SSM_ERR_UNSUPPORTED;
    const long long heads_total = (long long)batch * heads;
    const bool work = heads_total > 0 && seqlen > 0;
    if (work && (!x || !a || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, a, B, C, y, initial_state, final_state};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSM_ERR_ALIGNMENT;
    if (heads_total == 0) return SSM_OK;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (!work) {   // no tokens: the final state is the start state
        if (!final_state) return SSM_OK;
        const size_t bytes = size_t(heads_total) * headdim * dstate * sizeof(float);
        if (initial_state)
            return status_of(cudaMemcpyAsync(final_state, initial_state, bytes, cudaMemcpyDeviceToDevice, stream));
        return status_of(cudaMemsetAsync(final_state, 0, bytes, stream));
    }
    ssm::SsdArgs s{};
    s.x = static_cast<const __nv_bfloat16 *>(x);
    s.a = a;
    s.B = static_cast<const __nv_bfloat16 *>(B);
    s.C = static_cast<const __nv_bfloat16 *>(C);
    s.y = y; s.h0 = initial_state; s.hN = final_state;
    s.batch = batch; s.seqlen = seqlen; s.heads = heads;
    if (out_dtype == SSM_F32) return dispatch_ssd<float>(s, headdim, dstate, stream);
    return dispatch_ssd<__nv_bfloat16>(s, headdim, dstate, stream);
}

}  // extern "C"
