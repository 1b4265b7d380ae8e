// ssm_api.cu -- library-wide entry points of libssm.so: version and status strings.
// The operations live in scan_api.cu, step_api.cu and conv_api.cu.
#include "api_host.cuh"

namespace {
constexpr int kVersion = 1 * 10000 + 1 * 100 + 0;
}  // namespace

extern "C" {

int ssm_version(void) { return kVersion; }

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
