// ssm_api.cu -- library-wide entry points of libssm.so: version and status strings, and
// the SFU throughput probe.  The operations live in scan_api.cu, step_api.cu,
// conv_api.cu, bwd_api.cu and ssd_api.cu.
#include "api_host.cuh"
#include "common.cuh"

using namespace ssm_host;

namespace {
constexpr int kVersion = 1 * 10000 + 1 * 100 + 0;
constexpr int kProbeThreads = 256;
constexpr int kProbeChains = 8;

// Each thread iterates kProbeChains independent chains v <- 2^(-v).  From v in [0.5, 1] the
// values stay in [0.5, 0.71], so every step is one ordinary SFU ex2 (the negation rides on
// its operand or costs one FP32 instruction, as the decay argument does in the scan).
__global__ void __launch_bounds__(kProbeThreads) sfu_probe_kernel(float *out, int iters) {
    float v[kProbeChains];
#pragma unroll
    for (int k = 0; k < kProbeChains; ++k) v[k] = 0.5f + 0.0625f * k;
#pragma unroll 4
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int k = 0; k < kProbeChains; ++k) v[k] = ssm::ex2_approx(-v[k]);
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kProbeChains; ++k) s += v[k];
    out[size_t(blockIdx.x) * kProbeThreads + threadIdx.x] = s;
}
}  // namespace

extern "C" {

int ssm_version(void) { return kVersion; }

int ssm_sfu_probe(float *out, int blocks, int iters, void *cuda_stream) {
    if (out == nullptr || blocks < 1 || iters < 0) return SSM_ERR_INVALID_ARG;
    if (!aligned16(out)) return SSM_ERR_ALIGNMENT;
    sfu_probe_kernel<<<unsigned(blocks), kProbeThreads, 0, static_cast<cudaStream_t>(cuda_stream)>>>(out, iters);
    return status_of(cudaGetLastError());
}

const char *ssm_status_string(int status) {
    switch (status) {
    case SSM_OK: return "ok";
    case SSM_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size or bad dtype)";
    case SSM_ERR_UNSUPPORTED: return "unsupported size (dstate above 16, conv width above 8, or a grid too large)";
    case SSM_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case SSM_ERR_CUDA: return "CUDA runtime error at launch";
    case SSM_ERR_SCRATCH:
        return "the allocation-free scan needs more scratch than its fixed 4 MiB device array";
    default: return "unknown status";
    }
}

}  // extern "C"
