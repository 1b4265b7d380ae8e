// ssm_api.cu -- the C ABI of libssm.so: argument checks, kernel choice, launch.
//
// Every entry point checks its arguments on the host before touching the GPU; a
// rejected call launches nothing.  Kernels run on the caller's stream, asynchronously.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "../../include/ssm.h"
#include "conv1d.cuh"
#include "scan_fwd.cuh"
#include "state_step.cuh"

namespace {

constexpr int kVersion = 1 * 10000 + 0 * 100 + 0;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_dtype(int t) { return t == SSM_F32 || t == SSM_BF16; }

int status_of(cudaError_t e) { return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA; }

size_t dtype_size(int t) { return t == SSM_F32 ? 4 : 2; }

// Do the byte ranges [p, p + pb) and [q, q + qb) share a byte?
bool overlaps(const void *p, size_t pb, const void *q, size_t qb) {
    if (!p || !q || pb == 0 || qb == 0) return false;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
    return a < b + qb && b < a + pb;
}

constexpr int kMinSegTokens = 4096;     // shortest segment worth a carry correction

// Segments per sequence: 1 while the channel groups alone fill every resident CTA slot
// (`slots` = SMs x resident CTAs per SM); otherwise as many as fit in one wave of slots,
// each at least kMinSegTokens long.  SSM_SCAN_SEGMENTS=k forces k (used by the tests to
// reach the two-pass path).
int choose_segments(long long channel_groups, int seqlen, long long slots) {
    if (const char *e = std::getenv("SSM_SCAN_SEGMENTS")) {
        const int v = std::atoi(e);
        if (v >= 1) return v;
    }
    if (2 * channel_groups >= slots) return 1;
    const long long want = slots / channel_groups;
    const long long room = seqlen / kMinSegTokens;
    return int(std::max(1LL, std::min(want, room)));
}

// Resident CTA slots of a kernel on the current device (0 if the query fails).
template <class Kernel>
long long resident_slots(Kernel kernel, int threads, size_t smem) {
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess)
        return 0;
    return (long long)sms * per_sm;
}

template <class Cfg, bool SEG, bool ZOH = false>
int launch_scan_kernel(const ssm::ScanArgs &a, long long blocks, cudaStream_t stream) {
    if (blocks > INT_MAX) return SSM_ERR_UNSUPPORTED;
    if (blocks == 0) return SSM_OK;
    ssm::scan_fwd_kernel<Cfg, SEG, ZOH><<<unsigned(blocks), Cfg::NTHREADS, Cfg::SMEM_BYTES, stream>>>(a);
    return status_of(cudaGetLastError());
}

// One scan: a single pass when the sequence fits one CTA per channel group, else the two
// segment passes with a stream-ordered scratch buffer of batch*dim*nseg*(NP+1) floats.
template <class Cfg, bool ZOH>
int run_scan(const ssm::ScanArgs &a0, cudaStream_t stream) {
    ssm::ScanArgs a = a0;
    const long long groups = (a.dim + Cfg::CH - 1) / Cfg::CH;
    if (groups > INT_MAX) return SSM_ERR_UNSUPPORTED;
    a.groups_per_seq = int(groups);
    const long long cgroups = groups * a.batch;
    const size_t smem = Cfg::SMEM_BYTES;
    if (smem > 48 * 1024) {   // opt in to large shared memory for both kernel variants
        if (cudaFuncSetAttribute(ssm::scan_fwd_kernel<Cfg, false, ZOH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem)) != cudaSuccess ||
            cudaFuncSetAttribute(ssm::scan_fwd_kernel<Cfg, true, ZOH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem)) != cudaSuccess)
            return SSM_ERR_CUDA;
    }
    const long long slots = resident_slots(ssm::scan_fwd_kernel<Cfg, true, ZOH>, Cfg::NTHREADS, smem);
    int nseg = choose_segments(cgroups, a.seqlen, slots > 0 ? slots : 2 * cgroups);
    long long seg_len = (a.seqlen + nseg - 1) / nseg;
    seg_len = (seg_len + Cfg::T - 1) / Cfg::T * Cfg::T;
    nseg = int((a.seqlen + seg_len - 1) / seg_len);
    if (nseg <= 1) {
        a.pass = 0;
        a.nseg = 1;
        a.seg_len = a.seqlen;
        return launch_scan_kernel<Cfg, false, ZOH>(a, cgroups, stream);
    }
    const size_t rows = size_t(a.batch) * a.dim * nseg;
    const size_t bytes = rows * Cfg::NP * sizeof(float) + rows * sizeof(float);
    void *ws = nullptr;
    if (cudaMallocAsync(&ws, bytes, stream) != cudaSuccess) return SSM_ERR_CUDA;
    a.nseg = nseg;
    a.seg_len = int(seg_len);
    a.seg_h = static_cast<float *>(ws);
    a.seg_s = a.seg_h + rows * Cfg::NP;
    a.pass = 1;
    int st = launch_scan_kernel<Cfg, true, ZOH>(a, cgroups * nseg, stream);
    if (st == SSM_OK) {
        a.pass = 2;
        st = launch_scan_kernel<Cfg, true, ZOH>(a, cgroups * (nseg - 1), stream);
    }
    const cudaError_t fe = cudaFreeAsync(ws, stream);
    if (st == SSM_OK && fe != cudaSuccess) st = SSM_ERR_CUDA;
    return st;
}

// Tile shape per padded state width: 32-token tiles; 32 channels per CTA (64 at N <= 4).
#ifndef SSM_SCAN16_MINB
#define SSM_SCAN16_MINB 4     // resident CTAs per SM the 16-state kernel's registers target
#endif
#ifndef SSM_SCAN16_NSTAGE
#define SSM_SCAN16_NSTAGE 3   // cp.async ring depth of the 16-state kernel
#endif

template <int NP, typename Tin, typename Tout, bool VEC>
int dispatch_cfg(const ssm::ScanArgs &a, cudaStream_t s) {
    using C16 = ssm::ScanCfg<16, 1, 32, SSM_SCAN16_NSTAGE, Tin, Tout, VEC, SSM_SCAN16_MINB>;
    using C8 = ssm::ScanCfg<8, 1, 32, 3, Tin, Tout, VEC, 6>;
    using C4 = ssm::ScanCfg<4, 2, 32, 3, Tin, Tout, VEC, 6>;
    using Cfg = std::conditional_t<NP == 16, C16, std::conditional_t<NP == 8, C8, C4>>;
    return a.zoh ? run_scan<Cfg, true>(a, s) : run_scan<Cfg, false>(a, s);
}

template <typename Tin, typename Tout>
int dispatch_np(const ssm::ScanArgs &a, bool vec, cudaStream_t s) {
    const int N = a.dstate;
    if (N <= 4) return vec ? dispatch_cfg<4, Tin, Tout, true>(a, s) : dispatch_cfg<4, Tin, Tout, false>(a, s);
    if (N <= 8) return vec ? dispatch_cfg<8, Tin, Tout, true>(a, s) : dispatch_cfg<8, Tin, Tout, false>(a, s);
    return vec ? dispatch_cfg<16, Tin, Tout, true>(a, s) : dispatch_cfg<16, Tin, Tout, false>(a, s);
}

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

// ---------------------------------------------------------------------------------
// Allocation-free variant (ssm_selective_scan_fwd_noalloc).  The segment aggregates of
// the two-pass scan live in this file-scope device array instead of a stream-ordered
// allocation.  Every GPU that loads the library holds it until the process exits.
// ---------------------------------------------------------------------------------
constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;      // 4 MiB per GPU
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
float *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code the array's
// name stands for a host-side shadow, not for device memory, so the address is looked up
// once per device (with that device current) and cached.
int noalloc_scratch(float **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SSM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
            return SSM_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<float *>(ptr);
    }
    *out = g_noalloc_ptr[dev];
    return SSM_OK;
}

// Same scan as run_scan, with the segment aggregates in the static array: nothing is
// allocated.  Pass 1 writes every (channel, segment) row that pass 2 reads within the
// same call, so the array needs no clearing between calls.
template <class Cfg>
int run_scan_noalloc(const ssm::ScanArgs &a0, cudaStream_t stream) {
    ssm::ScanArgs a = a0;
    const long long groups = (a.dim + Cfg::CH - 1) / Cfg::CH;
    if (groups > INT_MAX) return SSM_ERR_UNSUPPORTED;
    a.groups_per_seq = int(groups);
    const long long cgroups = groups * a.batch;
    const size_t smem = Cfg::SMEM_BYTES;
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(ssm::scan_fwd_kernel<Cfg, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem)) != cudaSuccess ||
            cudaFuncSetAttribute(ssm::scan_fwd_kernel<Cfg, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem)) != cudaSuccess)
            return SSM_ERR_CUDA;
    }
    const long long slots = resident_slots(ssm::scan_fwd_kernel<Cfg, true, false>, Cfg::NTHREADS, smem);
    int nseg = choose_segments(cgroups, a.seqlen, slots > 0 ? slots : 2 * cgroups);
    long long seg_len = (a.seqlen + nseg - 1) / nseg;
    seg_len = (seg_len + Cfg::T - 1) / Cfg::T * Cfg::T;
    nseg = int((a.seqlen + seg_len - 1) / seg_len);
    if (nseg <= 1) {
        a.pass = 0;
        a.nseg = 1;
        a.seg_len = a.seqlen;
        return launch_scan_kernel<Cfg, false>(a, cgroups, stream);
    }
    const size_t rows = size_t(a.batch) * a.dim * nseg;
    if (rows * (Cfg::NP + 1) > kNoAllocScratchFloats) return SSM_ERR_SCRATCH;
    float *ws = nullptr;
    const int st0 = noalloc_scratch(&ws);
    if (st0 != SSM_OK) return st0;
    a.nseg = nseg;
    a.seg_len = int(seg_len);
    a.seg_h = ws;
    a.seg_s = ws + rows * Cfg::NP;
    a.pass = 1;
    int st = launch_scan_kernel<Cfg, true>(a, cgroups * nseg, stream);
    if (st == SSM_OK) {
        a.pass = 2;
        st = launch_scan_kernel<Cfg, true>(a, cgroups * (nseg - 1), stream);
    }
    return st;
}

template <int NP, typename Tin, typename Tout, bool VEC>
int dispatch_cfg_noalloc(const ssm::ScanArgs &a, cudaStream_t s) {
    if constexpr (NP == 16)
        return run_scan_noalloc<ssm::ScanCfg<16, 1, 32, SSM_SCAN16_NSTAGE, Tin, Tout, VEC, SSM_SCAN16_MINB>>(a, s);
    else if constexpr (NP == 8) return run_scan_noalloc<ssm::ScanCfg<8, 1, 32, 3, Tin, Tout, VEC, 6>>(a, s);
    else return run_scan_noalloc<ssm::ScanCfg<4, 2, 32, 3, Tin, Tout, VEC, 6>>(a, s);
}

template <typename Tin, typename Tout>
int dispatch_np_noalloc(const ssm::ScanArgs &a, bool vec, cudaStream_t s) {
    const int N = a.dstate;
    if (N <= 4) return vec ? dispatch_cfg_noalloc<4, Tin, Tout, true>(a, s) : dispatch_cfg_noalloc<4, Tin, Tout, false>(a, s);
    if (N <= 8) return vec ? dispatch_cfg_noalloc<8, Tin, Tout, true>(a, s) : dispatch_cfg_noalloc<8, Tin, Tout, false>(a, s);
    return vec ? dispatch_cfg_noalloc<16, Tin, Tout, true>(a, s) : dispatch_cfg_noalloc<16, Tin, Tout, false>(a, s);
}

}  // namespace

extern "C" {

int ssm_version(void) { return kVersion; }

const char *ssm_status_string(int status) {
    switch (status) {
    case SSM_OK: return "ok";
    case SSM_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size or bad dtype)";
    case SSM_ERR_UNSUPPORTED: return "unsupported size (dstate must be 1..16; grid too large)";
    case SSM_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case SSM_ERR_CUDA: return "CUDA runtime error at launch";
    case SSM_ERR_SCRATCH:
        return "the allocation-free scan needs more scratch than its fixed 4 MiB device array";
    default: return "unknown status";
    }
}

int ssm_selective_scan_fwd(const void *x, const void *delta, const float *delta_bias,
                           int delta_softplus, const float *A, const void *B, const void *C,
                           const float *D, const void *z, void *y, float *final_state,
                           int batch, int dim, int seqlen, int dstate,
                           int in_dtype, int out_dtype, void *cuda_stream) {
    return ssm_selective_scan_fwd_ex(x, delta, delta_bias, delta_softplus, A, B, C, D, z, y,
                                     final_state, nullptr, 0, batch, dim, seqlen, dstate,
                                     in_dtype, out_dtype, cuda_stream);
}

int ssm_selective_scan_fwd_ex(const void *x, const void *delta, const float *delta_bias,
                              int delta_softplus, const float *A, const void *B, const void *C,
                              const float *D, const void *z, void *y, float *final_state,
                              const float *initial_state, int zoh_exact,
                              int batch, int dim, int seqlen, int dstate,
                              int in_dtype, int out_dtype, void *cuda_stream) {
    if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return SSM_ERR_INVALID_ARG;
    if (batch < 0 || dim < 0 || seqlen < 0 || dstate < 1) return SSM_ERR_INVALID_ARG;
    if (dstate > 16) return SSM_ERR_UNSUPPORTED;
    const long long channels = (long long)batch * dim;
    const bool work = channels > 0 && seqlen > 0;
    if (work && (!x || !delta || !A || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, delta, delta_bias, A, B, C, D, z, y, final_state, initial_state};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSM_ERR_ALIGNMENT;
    if (channels == 0) return SSM_OK;
    if (!work && !final_state) return SSM_OK;

    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (!work) {   // empty sequences: the final state is the start state
        const size_t bytes = size_t(channels) * dstate * sizeof(float);
        if (initial_state)
            return status_of(cudaMemcpyAsync(final_state, initial_state, bytes, cudaMemcpyDeviceToDevice, stream));
        return status_of(cudaMemsetAsync(final_state, 0, bytes, stream));
    }

    ssm::ScanArgs a{};
    a.x = x; a.delta = delta; a.delta_bias = delta_bias; a.A = A; a.B = B; a.C = C; a.D = D;
    a.z = z; a.y = y; a.final_state = final_state; a.h0 = initial_state;
    a.batch = batch; a.dim = dim; a.seqlen = seqlen; a.dstate = dstate;
    a.softplus = delta_softplus ? 1 : 0;
    a.zoh = zoh_exact ? 1 : 0;

    // 16-byte staging needs every row of x/delta/z/y and every sequence's B/C block to
    // start on a 16-byte boundary: seqlen a multiple of the 16-byte element count.
    const int ein = in_dtype == SSM_F32 ? 4 : 8;
    const int eout = out_dtype == SSM_F32 ? 4 : 8;
    const bool vec = (seqlen % ein == 0) && (seqlen % eout == 0);

    if (in_dtype == SSM_F32 && out_dtype == SSM_F32) return dispatch_np<float, float>(a, vec, stream);
    if (in_dtype == SSM_BF16 && out_dtype == SSM_BF16)
        return dispatch_np<__nv_bfloat16, __nv_bfloat16>(a, vec, stream);
    if (in_dtype == SSM_BF16) return dispatch_np<__nv_bfloat16, float>(a, vec, stream);
    return dispatch_np<float, __nv_bfloat16>(a, vec, stream);
}

int ssm_selective_scan_fwd_noalloc(const void *x, const void *delta, const float *delta_bias,
                                   int delta_softplus, const float *A, const void *B, const void *C,
                                   const float *D, const void *z, void *y, float *final_state,
                                   int batch, int dim, int seqlen, int dstate,
                                   int in_dtype, int out_dtype, void *cuda_stream) {
    if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return SSM_ERR_INVALID_ARG;
    if (batch < 0 || dim < 0 || seqlen < 0 || dstate < 1) return SSM_ERR_INVALID_ARG;
    if (dstate > 16) return SSM_ERR_UNSUPPORTED;
    const long long channels = (long long)batch * dim;
    const bool work = channels > 0 && seqlen > 0;
    if (work && (!x || !delta || !A || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, delta, delta_bias, A, B, C, D, z, y, final_state};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSM_ERR_ALIGNMENT;
    if (channels == 0) return SSM_OK;
    if (!work && !final_state) return SSM_OK;

    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (!work)   // empty sequences: the final state is the zero start state
        return status_of(cudaMemsetAsync(final_state, 0, size_t(channels) * dstate * sizeof(float), stream));

    ssm::ScanArgs a{};
    a.x = x; a.delta = delta; a.delta_bias = delta_bias; a.A = A; a.B = B; a.C = C; a.D = D;
    a.z = z; a.y = y; a.final_state = final_state;
    a.batch = batch; a.dim = dim; a.seqlen = seqlen; a.dstate = dstate;
    a.softplus = delta_softplus ? 1 : 0;
    const int ein = in_dtype == SSM_F32 ? 4 : 8;
    const int eout = out_dtype == SSM_F32 ? 4 : 8;
    const bool vec = (seqlen % ein == 0) && (seqlen % eout == 0);

    if (in_dtype == SSM_F32 && out_dtype == SSM_F32) return dispatch_np_noalloc<float, float>(a, vec, stream);
    if (in_dtype == SSM_BF16 && out_dtype == SSM_BF16)
        return dispatch_np_noalloc<__nv_bfloat16, __nv_bfloat16>(a, vec, stream);
    if (in_dtype == SSM_BF16) return dispatch_np_noalloc<__nv_bfloat16, float>(a, vec, stream);
    return dispatch_np_noalloc<float, __nv_bfloat16>(a, vec, stream);
}

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
