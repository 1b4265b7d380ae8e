// conv_api.cu -- C ABI of the causal depthwise convolution in front of the scan
// (ssm_causal_conv1d_fwd) and its one-token window form (ssm_causal_conv1d_step).
#include <algorithm>
#include <climits>

#include "api_host.cuh"
#include "conv1d.cuh"

using namespace ssm_host;

namespace {

template <typename Tin, typename Tout, int K>
int launch_conv_vec(const ssm::ConvArgs &a, cudaStream_t s) {
    // warp spans of 32*U vectors: U = 4 for rows of more than 64 vectors, else 1 so that
    // short rows do not leave most lanes idle
    const long long nvr = a.seqlen / ssm::Vec16<Tin>::kN;
    const int U = nvr > 64 ? 4 : 1;
    const long long spans_per_row = (nvr + 32 * U - 1) / (32 * U);
    const long long total_spans = a.rows * spans_per_row;
    const long long blocks = (total_spans * 32 + 255) / 256;
    if (blocks > INT_MAX) return SSM_ERR_UNSUPPORTED;
    if (U == 4)
        ssm::causal_conv1d_vec_kernel<Tin, Tout, K, 4><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
            a, nvr, spans_per_row, total_spans);
    else
        ssm::causal_conv1d_vec_kernel<Tin, Tout, K, 1><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
            a, nvr, spans_per_row, total_spans);
    return status_of(cudaGetLastError());
}

template <typename Tin, typename Tout>
int launch_conv(const ssm::ConvArgs &a, cudaStream_t s) {
    // the vector path needs every row to start on a 16-byte vector of inputs
    if (a.seqlen % ssm::Vec16<Tin>::kN == 0) {
        switch (a.K) {
            case 1: return launch_conv_vec<Tin, Tout, 1>(a, s);
            case 2: return launch_conv_vec<Tin, Tout, 2>(a, s);
            case 3: return launch_conv_vec<Tin, Tout, 3>(a, s);
            case 4: return launch_conv_vec<Tin, Tout, 4>(a, s);
            default: break;
        }
    }
    const long long total = a.rows * a.seqlen;
    const long long blocks = std::min<long long>((total + 255) / 256, INT_MAX);
    ssm::causal_conv1d_any_kernel<Tin, Tout><<<static_cast<unsigned>(blocks), 256, 0, s>>>(a);
    return status_of(cudaGetLastError());
}

template <typename Tin, typename Tout>
int launch_conv_step(float *window, const void *x, const float *w, const float *bias, void *u,
                     long long rows, int dim, int K, int silu, cudaStream_t s) {
    const long long blocks = (rows + 255) / 256;
    if (blocks > INT_MAX) return SSM_ERR_UNSUPPORTED;
    ssm::conv1d_step_kernel<Tin, Tout><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        window, static_cast<const Tin *>(x), w, bias, static_cast<Tout *>(u), rows, dim, K, silu);
    return status_of(cudaGetLastError());
}

}  // namespace

extern "C" {

int ssm_causal_conv1d_fwd(const void *x, const float *weight, const float *bias,
                          const float *initial_window, void *u, float *final_window,
                          int batch, int dim, int seqlen, int width, int silu,
                          int in_dtype, int out_dtype, void *cuda_stream) {
    if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return SSM_ERR_INVALID_ARG;
    if (batch < 0 || dim < 0 || seqlen < 0 || width < 1) return SSM_ERR_INVALID_ARG;
    if (width > ssm::kMaxConvWidth) return SSM_ERR_UNSUPPORTED;
    const long long rows = (long long)batch * dim;
    const int H = width - 1;
    const bool work = rows > 0 && seqlen > 0;
    if (work && (!x || !weight || !u)) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, weight, bias, initial_window, u, final_window};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSM_ERR_ALIGNMENT;
    const size_t xb = size_t(rows) * seqlen * dtype_size(in_dtype);
    const size_t ub = size_t(rows) * seqlen * dtype_size(out_dtype);
    const size_t wb = size_t(rows) * H * sizeof(float);
    if (overlaps(u, ub, x, xb) || overlaps(final_window, wb, initial_window, wb) ||
        overlaps(final_window, wb, x, xb) || overlaps(final_window, wb, u, ub))
        return SSM_ERR_INVALID_ARG;
    if (rows == 0) return SSM_OK;

    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (!work) {   // empty sequences: the window is the one carried in
        if (!final_window || H == 0) return SSM_OK;
        if (initial_window)
            return status_of(cudaMemcpyAsync(final_window, initial_window, wb, cudaMemcpyDeviceToDevice, stream));
        return status_of(cudaMemsetAsync(final_window, 0, wb, stream));
    }

    ssm::ConvArgs a{};
    a.x = x; a.w = weight; a.bias = bias; a.hist = initial_window; a.u = u;
    a.hist_out = final_window; a.rows = rows; a.dim = dim; a.seqlen = seqlen; a.K = width;
    a.silu = silu ? 1 : 0;
    if (in_dtype == SSM_F32 && out_dtype == SSM_F32) return launch_conv<float, float>(a, stream);
    if (in_dtype == SSM_BF16 && out_dtype == SSM_BF16)
        return launch_conv<__nv_bfloat16, __nv_bfloat16>(a, stream);
    if (in_dtype == SSM_BF16) return launch_conv<__nv_bfloat16, float>(a, stream);
    return launch_conv<float, __nv_bfloat16>(a, stream);
}

int ssm_causal_conv1d_step(float *window, const void *x, const float *weight, const float *bias,
                           void *u, int batch, int dim, int width, int silu,
                           int in_dtype, int out_dtype, void *cuda_stream) {
    if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return SSM_ERR_INVALID_ARG;
    if (batch < 0 || dim < 0 || width < 1) return SSM_ERR_INVALID_ARG;
    if (width > ssm::kMaxConvWidth) return SSM_ERR_UNSUPPORTED;
    const long long rows = (long long)batch * dim;
    const int H = width - 1;
    if (rows > 0 && (!x || !weight || !u || (H > 0 && !window))) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {window, x, weight, bias, u};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSM_ERR_ALIGNMENT;
    const size_t wb = size_t(rows) * H * sizeof(float);
    if (overlaps(window, wb, x, size_t(rows) * dtype_size(in_dtype)) ||
        overlaps(window, wb, u, size_t(rows) * dtype_size(out_dtype)))
        return SSM_ERR_INVALID_ARG;
    if (rows == 0) return SSM_OK;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    const int sf = silu ? 1 : 0;
    if (in_dtype == SSM_F32 && out_dtype == SSM_F32)
        return launch_conv_step<float, float>(window, x, weight, bias, u, rows, dim, width, sf, stream);
    if (in_dtype == SSM_BF16 && out_dtype == SSM_BF16)
        return launch_conv_step<__nv_bfloat16, __nv_bfloat16>(window, x, weight, bias, u, rows, dim, width, sf, stream);
    if (in_dtype == SSM_BF16)
        return launch_conv_step<__nv_bfloat16, float>(window, x, weight, bias, u, rows, dim, width, sf, stream);
    return launch_conv_step<float, __nv_bfloat16>(window, x, weight, bias, u, rows, dim, width, sf, stream);
}

}  // extern "C"
