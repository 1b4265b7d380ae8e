// step_api.cu -- C ABI of the decode steps: one token (ssm_state_step) and several tokens
// on the carried state (ssm_state_step_multi).
#include <algorithm>
#include <climits>

#include "api_host.cuh"
#include "state_step.cuh"

using namespace ssm_host;

namespace {

template <int NP, int J, typename Tin, typename Tout>
int launch_step_j(const ssm::StepArgs &a, cudaStream_t s) {
    constexpr int G = NP / 4;
    const long long quads = (long long)a.batch * a.dim * G;
    const long long blocks = (quads + 256LL * J - 1) / (256LL * J);
    if (blocks > INT_MAX) return SSM_ERR_UNSUPPORTED;
    if (a.dstate % 4 == 0)
        ssm::state_step_kernel<NP, Tin, Tout, true, J><<<unsigned(blocks), 256, 0, s>>>(a);
    else
        ssm::state_step_kernel<NP, Tin, Tout, false, J><<<unsigned(blocks), 256, 0, s>>>(a);
    return status_of(cudaGetLastError());
}

// One channel-quad per thread: at 32 registers the SM holds 2048 threads, each with its
// 16-byte state load in flight, which measured faster than several quads per thread.
template <int NP, typename Tin, typename Tout>
int launch_step_np(const ssm::StepArgs &a, cudaStream_t s) {
    return launch_step_j<NP, 1, Tin, Tout>(a, s);
}

template <typename Tin, typename Tout>
int launch_step(const ssm::StepArgs &a, cudaStream_t s) {
    if (a.dstate <= 4) return launch_step_np<4, Tin, Tout>(a, s);
    if (a.dstate <= 8) return launch_step_np<8, Tin, Tout>(a, s);
    return launch_step_np<16, Tin, Tout>(a, s);
}

// Several tokens: one channel per thread, kStepThreads consecutive channels per block; the
// blocks of a channel range share out the sequences, as many blocks in all as the GPU holds
// at once (or one per (sequence, channel range) if that is fewer).
template <int NP, typename Tin, typename Tout, bool VEC4>
int launch_steps_vec(const ssm::StepArgs &a, long long dblocks, cudaStream_t s) {
    const auto kernel = ssm::state_steps_kernel<NP, Tin, Tout, VEC4>;
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, ssm::kStepThreads, 0) != cudaSuccess)
        return SSM_ERR_CUDA;
    const long long resident = std::max(1LL, (long long)sms * per_sm);
    const long long slices = std::max(1LL, std::min<long long>(a.batch, resident / dblocks));
    const long long blocks = dblocks * slices;
    if (blocks > INT_MAX) return SSM_ERR_UNSUPPORTED;
    kernel<<<unsigned(blocks), ssm::kStepThreads, 0, s>>>(a, int(dblocks));
    return status_of(cudaGetLastError());
}

template <int NP, typename Tin, typename Tout>
int launch_steps_np(const ssm::StepArgs &a, cudaStream_t s) {
    const long long dblocks = (a.dim + ssm::kStepThreads - 1) / ssm::kStepThreads;
    if (dblocks == 0 || a.batch == 0) return SSM_OK;
    if (dblocks > INT_MAX) return SSM_ERR_UNSUPPORTED;
    return a.dstate % 4 == 0 ? launch_steps_vec<NP, Tin, Tout, true>(a, dblocks, s)
                             : launch_steps_vec<NP, Tin, Tout, false>(a, dblocks, s);
}

template <typename Tin, typename Tout>
int launch_steps(const ssm::StepArgs &a, cudaStream_t s) {
    if (a.dstate <= 4) return launch_steps_np<4, Tin, Tout>(a, s);
    if (a.dstate <= 8) return launch_steps_np<8, Tin, Tout>(a, s);
    return launch_steps_np<16, Tin, Tout>(a, s);
}

}  // namespace

extern "C" {

int ssm_state_step(float *state, const void *x, const void *delta, const float *A,
                   const void *B, const void *C, const float *D, const void *z, void *y,
                   int batch, int dim, int dstate, int in_dtype, int out_dtype,
                   void *cuda_stream) {
    if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return SSM_ERR_INVALID_ARG;
    if (batch < 0 || dim < 0 || dstate < 1) return SSM_ERR_INVALID_ARG;
    if (dstate > 16) return SSM_ERR_UNSUPPORTED;
    const long long channels = (long long)batch * dim;
    if (channels > 0 && (!state || !x || !delta || !A || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {state, x, delta, A, B, C, D, z, y};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSM_ERR_ALIGNMENT;
    if (channels == 0) return SSM_OK;

    ssm::StepArgs a{};
    a.state = state; a.x = x; a.delta = delta; a.A = A; a.B = B; a.C = C; a.D = D; a.z = z;
    a.y = y; a.batch = batch; a.dim = dim; a.dstate = dstate;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (in_dtype == SSM_F32 && out_dtype == SSM_F32) return launch_step<float, float>(a, stream);
    if (in_dtype == SSM_BF16 && out_dtype == SSM_BF16)
        return launch_step<__nv_bfloat16, __nv_bfloat16>(a, stream);
    if (in_dtype == SSM_BF16) return launch_step<__nv_bfloat16, float>(a, stream);
    return launch_step<float, __nv_bfloat16>(a, stream);
}

int ssm_state_step_multi(float *state, const void *x, const void *delta, const float *A,
                         const void *B, const void *C, const float *D, const void *z, void *y,
                         int ntok, int batch, int dim, int dstate, int in_dtype, int out_dtype,
                         void *cuda_stream) {
    if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return SSM_ERR_INVALID_ARG;
    if (ntok < 0 || batch < 0 || dim < 0 || dstate < 1) return SSM_ERR_INVALID_ARG;
    if (dstate > 16) return SSM_ERR_UNSUPPORTED;
    const long long channels = (long long)batch * dim;
    const bool work = channels > 0 && ntok > 0;
    if (work && (!state || !x || !delta || !A || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {state, x, delta, A, B, C, D, z, y};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSM_ERR_ALIGNMENT;
    if (!work) return SSM_OK;

    ssm::StepArgs a{};
    a.state = state; a.x = x; a.delta = delta; a.A = A; a.B = B; a.C = C; a.D = D; a.z = z;
    a.y = y; a.batch = batch; a.dim = dim; a.dstate = dstate; a.ntok = ntok;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (in_dtype == SSM_F32 && out_dtype == SSM_F32) return launch_steps<float, float>(a, stream);
    if (in_dtype == SSM_BF16 && out_dtype == SSM_BF16)
        return launch_steps<__nv_bfloat16, __nv_bfloat16>(a, stream);
    if (in_dtype == SSM_BF16) return launch_steps<__nv_bfloat16, float>(a, stream);
    return launch_steps<float, __nv_bfloat16>(a, stream);
}

}  // extern "C"
