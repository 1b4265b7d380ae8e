// ssd_api.cu -- C ABI of Mamba-2's state-space dual by chunks (ssm_ssd_fwd).
//
// Arguments are checked on the host before anything is launched; the kernel runs on the
// caller's stream, asynchronously.  The tile loads go through TMA tensor maps, built here
// per call (cuTensorMapEncodeTiled, reached through the runtime's driver entry point).
#include <climits>

#include "api_host.cuh"
#include "ssd_tc.cuh"

using namespace ssm_host;

// Kernels that give up waiting on an asynchronous copy or a tensor-core operation count it
// here (read by ssm_device_timeouts).
static __device__ unsigned g_wait_timeouts;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return EncodeTiledFn(nullptr);
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// Tensor map over a [batch][L][heads][W] bf16 tensor as the 4-D array (W, heads, L, batch),
// boxes of (bw, 1, rows, 1): one head's `rows` tokens of `bw` values.  Tokens past L read
// as zeros.  128-byte boxes use the 128-byte swizzle, 64-byte boxes the 64-byte one.
bool make_map(CUtensorMap *m, const void *base, int W, int H, int L, int batch, int bw, int rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {cuuint64_t(W), cuuint64_t(H), cuuint64_t(L), cuuint64_t(batch)};
    const cuuint64_t strides[3] = {cuuint64_t(W) * 2, cuuint64_t(W) * H * 2, cuuint64_t(W) * H * L * 2};
    const cuuint32_t box[4] = {cuuint32_t(bw), 1, cuuint32_t(rows), 1};
    const cuuint32_t unit[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, unit,
               CU_TENSOR_MAP_INTERLEAVE_NONE, bw * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int P, int N, typename Tout>
int launch_ssd(const void *x, const void *B, const void *C, ssm::SsdTcArgs a, cudaStream_t s) {
    using Cfg = ssm::SsdTcCfg<P, N, Tout>;
    const long long ctas = (long long)a.batch * a.heads;
    if (ctas > INT_MAX) return SSM_ERR_UNSUPPORTED;
    CUtensorMap mx, mb, mc;
    if (!make_map(&mx, x, P, a.heads, a.seqlen, a.batch, P, Cfg::Q) ||
        !make_map(&mb, B, N, a.heads, a.seqlen, a.batch, 64, Cfg::Q) ||
        !make_map(&mc, C, N, a.heads, a.seqlen, a.batch, 64, Cfg::Q))
        return SSM_ERR_CUDA;
    void *counter = nullptr;
    if (cudaGetSymbolAddress(&counter, g_wait_timeouts) != cudaSuccess) return SSM_ERR_CUDA;
    a.timeouts = static_cast<unsigned *>(counter);
    if (cudaFuncSetAttribute(ssm::ssd_tc_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(Cfg::SMEM_BYTES)) != cudaSuccess ||
        cudaFuncSetAttribute(ssm::ssd_tc_kernel<Cfg>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             int(cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
        return SSM_ERR_CUDA;
    ssm::ssd_tc_kernel<Cfg><<<unsigned(ctas), Cfg::NT, Cfg::SMEM_BYTES, s>>>(mx, mb, mc, a);
    return status_of(cudaGetLastError());
}

template <typename Tout>
int dispatch_ssd(const void *x, const void *B, const void *C, const ssm::SsdTcArgs &a, int P, int N,
                 cudaStream_t s) {
    if (P == 64 && N == 128) return launch_ssd<64, 128, Tout>(x, B, C, a, s);
    if (P == 64 && N == 64) return launch_ssd<64, 64, Tout>(x, B, C, a, s);
    if (P == 32 && N == 128) return launch_ssd<32, 128, Tout>(x, B, C, a, s);
    if (P == 32 && N == 64) return launch_ssd<32, 64, Tout>(x, B, C, a, s);
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
    ssm::SsdTcArgs s{};
    s.a = a;
    s.y = y; s.h0 = initial_state; s.hN = final_state;
    s.batch = batch; s.seqlen = seqlen; s.heads = heads;
    if (out_dtype == SSM_F32) return dispatch_ssd<float>(x, B, C, s, headdim, dstate, stream);
    return dispatch_ssd<__nv_bfloat16>(x, B, C, s, headdim, dstate, stream);
}

unsigned ssm_device_timeouts(void) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_wait_timeouts, sizeof(v)) != cudaSuccess) return ~0u;
    return v;
}

}  // extern "C"
