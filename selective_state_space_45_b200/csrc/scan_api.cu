// scan_api.cu -- C ABI of the selective scan: ssm_selective_scan_fwd, its _ex form (start
// state, exact zero-order-hold gain) and the allocation-free _noalloc form.
//
// Arguments are checked on the host before anything is launched; kernels run on the
// caller's stream, asynchronously.
#include <algorithm>
#include <atomic>
#include <climits>
#include <type_traits>

#include "api_host.cuh"
#include "scan_fwd.cuh"

using namespace ssm_host;

namespace {

constexpr int kMinSegTokens = 4096;     // shortest segment worth a carry correction

// Segment count forced by ssm_scan_force_segments (0: automatic).
std::atomic<int> g_forced_segments{0};

// Segments per sequence: 1 while the channel groups alone fill every resident CTA slot
// (`slots` = SMs x resident CTAs per SM); otherwise as many as fit in one wave of slots,
// each at least kMinSegTokens long.  A count forced through ssm_scan_force_segments wins.
int choose_segments(long long channel_groups, int seqlen, long long slots) {
    if (const int v = g_forced_segments.load(std::memory_order_relaxed); v >= 1) return v;
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

template <class Cfg, bool SEG, bool ZOH>
constexpr auto scan_kernel() {
    return &ssm::scan_fwd_kernel<Cfg, SEG, ZOH>;
}

template <class Cfg, bool SEG, bool ZOH>
int launch_scan_kernel(const ssm::ScanArgs &a, long long blocks, cudaStream_t stream) {
    if (blocks > INT_MAX) return SSM_ERR_UNSUPPORTED;
    if (blocks == 0) return SSM_OK;
    scan_kernel<Cfg, SEG, ZOH>()<<<unsigned(blocks), Cfg::NTHREADS, Cfg::SMEM_BYTES, stream>>>(a);
    return status_of(cudaGetLastError());
}

// The passes before the segment scans: each earlier segment's tail sum and step sum, then
// the fold of those into the carry of every segment.
template <class Cfg, bool ZOH>
int launch_tail_fold(const ssm::ScanArgs &a, cudaStream_t stream) {
    constexpr int NP = Cfg::NP;
    const long long rows = (long long)a.batch * a.dim;
    const long long tail_blocks = rows * (a.nseg - 1);
    const long long fold_blocks = (rows * NP + 255) / 256;
    if (tail_blocks > INT_MAX || fold_blocks > INT_MAX) return SSM_ERR_UNSUPPORTED;
    ssm::scan_tail_kernel<NP, typename Cfg::Tin, ZOH>
        <<<unsigned(tail_blocks), 32 * ssm::kTailWarps, 0, stream>>>(a);
    int st = status_of(cudaGetLastError());
    if (st != SSM_OK) return st;
    ssm::scan_fold_kernel<NP><<<unsigned(fold_blocks), 256, 0, stream>>>(a);
    return status_of(cudaGetLastError());
}

// The launch plan shared by the regular and the allocation-free scans: channel groups,
// the shared-memory opt-in of both kernel variants, and the segment count and length.
template <class Cfg, bool ZOH>
int plan_scan(ssm::ScanArgs &a, long long &cgroups) {
    const long long groups = (a.dim + Cfg::CH - 1) / Cfg::CH;
    if (groups > INT_MAX) return SSM_ERR_UNSUPPORTED;
    a.groups_per_seq = int(groups);
    cgroups = groups * a.batch;
    const size_t smem = Cfg::SMEM_BYTES;
    // both kernel variants: large shared memory where needed, and the whole unified L1 /
    // shared array given to shared memory so that every resident CTA the registers allow fits
    for (auto k : {scan_kernel<Cfg, false, ZOH>(), scan_kernel<Cfg, true, ZOH>()}) {
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
            return SSM_ERR_CUDA;
        if (cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 int(cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
            return SSM_ERR_CUDA;
    }
    const long long slots = resident_slots(scan_kernel<Cfg, true, ZOH>(), Cfg::NTHREADS, smem);
    int nseg = choose_segments(cgroups, a.seqlen, slots > 0 ? slots : 2 * cgroups);
    long long seg_len = (a.seqlen + nseg - 1) / nseg;
    seg_len = (seg_len + Cfg::T - 1) / Cfg::T * Cfg::T;
    a.nseg = int((a.seqlen + seg_len - 1) / seg_len);
    a.seg_len = a.nseg <= 1 ? a.seqlen : int(seg_len);
    if (a.nseg < 1) a.nseg = 1;
    return SSM_OK;
}

// One scan: a single pass when the sequence fits one CTA per channel group, else the tail
// and fold passes and one scan per segment from its carry, with a stream-ordered scratch
// buffer of batch*dim*nseg*(NP+1) floats.
template <class Cfg, bool ZOH>
int run_scan(const ssm::ScanArgs &a0, cudaStream_t stream) {
    ssm::ScanArgs a = a0;
    long long cgroups = 0;
    int st = plan_scan<Cfg, ZOH>(a, cgroups);
    if (st != SSM_OK) return st;
    if (a.nseg == 1) return launch_scan_kernel<Cfg, false, ZOH>(a, cgroups, stream);
    const size_t rows = size_t(a.batch) * a.dim * a.nseg;
    const size_t bytes = rows * Cfg::NP * sizeof(float) + rows * sizeof(float);
    void *ws = nullptr;
    if (cudaMallocAsync(&ws, bytes, stream) != cudaSuccess) return SSM_ERR_CUDA;
    a.seg_h = static_cast<float *>(ws);
    a.seg_s = a.seg_h + rows * Cfg::NP;
    st = launch_tail_fold<Cfg, ZOH>(a, stream);
    if (st == SSM_OK) st = launch_scan_kernel<Cfg, true, ZOH>(a, cgroups * a.nseg, stream);
    const cudaError_t fe = cudaFreeAsync(ws, stream);
    if (st == SSM_OK && fe != cudaSuccess) st = SSM_ERR_CUDA;
    return st;
}

// Tile shape per padded state width: 32-token tiles; 32 channels per CTA (64 at N <= 4).
// bf16 inputs at N = 16: a 2-stage ring, 42 KB of shared memory and at most 96 registers,
// so 5 CTAs share an SM (740 on the chip: 4 sequences x 5120 channels run in one wave).
#ifndef SSM_SCAN16_NSTAGE
#define SSM_SCAN16_NSTAGE 2   // ring depth of the bf16 N = 16 tile
#endif
#ifndef SSM_SCAN16_MINB
#define SSM_SCAN16_MINB 5     // resident CTAs per SM its registers target
#endif
template <int NP, typename Tin, typename Tout, bool VEC>
struct ScanConfig {
    using C16 = std::conditional_t<sizeof(Tin) == 2,
                                   ssm::ScanCfg<16, 1, 32, SSM_SCAN16_NSTAGE, Tin, Tout, VEC, SSM_SCAN16_MINB>,
                                   ssm::ScanCfg<16, 1, 32, 3, Tin, Tout, VEC, 4>>;
    using C8 = ssm::ScanCfg<8, 1, 32, 3, Tin, Tout, VEC, 6>;
    using C4 = ssm::ScanCfg<4, 2, 32, 3, Tin, Tout, VEC, 6>;
    using type = std::conditional_t<NP == 16, C16, std::conditional_t<NP == 8, C8, C4>>;
};

template <int NP, typename Tin, typename Tout, bool VEC>
int dispatch_cfg(const ssm::ScanArgs &a, cudaStream_t s) {
    using Cfg = typename ScanConfig<NP, Tin, Tout, VEC>::type;
    return a.zoh ? run_scan<Cfg, true>(a, s) : run_scan<Cfg, false>(a, s);
}

template <typename Tin, typename Tout>
int dispatch_np(const ssm::ScanArgs &a, bool vec, cudaStream_t s) {
    const int N = a.dstate;
    if (N <= 4) return vec ? dispatch_cfg<4, Tin, Tout, true>(a, s) : dispatch_cfg<4, Tin, Tout, false>(a, s);
    if (N <= 8) return vec ? dispatch_cfg<8, Tin, Tout, true>(a, s) : dispatch_cfg<8, Tin, Tout, false>(a, s);
    return vec ? dispatch_cfg<16, Tin, Tout, true>(a, s) : dispatch_cfg<16, Tin, Tout, false>(a, s);
}

// ---------------------------------------------------------------------------------
// Allocation-free variant (ssm_selective_scan_fwd_noalloc).  The segment aggregates of
// the two-pass scan live in this file-scope device array instead of a stream-ordered
// allocation.  Every GPU that loads the library holds it until the process exits.
// ---------------------------------------------------------------------------------
constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;      // 4 MiB per GPU
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// Device address of g_noalloc_scratch in the current device's context.  In host code the
// array's name stands for a host-side shadow, not for device memory, so the address is
// asked of the runtime with the device current.  It is asked on every call rather than
// cached: once the module is loaded this is a table lookup, and a context that was torn
// down and recreated (cudaDeviceReset) may place the array elsewhere, so a cached address
// could outlive the memory it named.  The first call on a device may load the module,
// which is why that first call should come before any stream capture.
int noalloc_scratch(float **out) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
        return SSM_ERR_CUDA;
    *out = static_cast<float *>(ptr);
    return SSM_OK;
}

// Same scan as run_scan, with the segment aggregates in the static array: nothing is
// allocated.  The tail pass writes every (channel, segment) row that the fold reads, and
// the fold every row that the segment scans read, within the same call, so the array
// needs no clearing between calls.
template <class Cfg>
int run_scan_noalloc(const ssm::ScanArgs &a0, cudaStream_t stream) {
    ssm::ScanArgs a = a0;
    long long cgroups = 0;
    int st = plan_scan<Cfg, false>(a, cgroups);
    if (st != SSM_OK) return st;
    if (a.nseg == 1) return launch_scan_kernel<Cfg, false, false>(a, cgroups, stream);
    const size_t rows = size_t(a.batch) * a.dim * a.nseg;
    if (rows * (Cfg::NP + 1) > kNoAllocScratchFloats) return SSM_ERR_SCRATCH;
    float *ws = nullptr;
    st = noalloc_scratch(&ws);
    if (st != SSM_OK) return st;
    a.seg_h = ws;
    a.seg_s = ws + rows * Cfg::NP;
    st = launch_tail_fold<Cfg, false>(a, stream);
    return st == SSM_OK ? launch_scan_kernel<Cfg, true, false>(a, cgroups * a.nseg, stream) : st;
}

template <int NP, typename Tin, typename Tout, bool VEC>
int dispatch_cfg_noalloc(const ssm::ScanArgs &a, cudaStream_t s) {
    return run_scan_noalloc<typename ScanConfig<NP, Tin, Tout, VEC>::type>(a, s);
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

int ssm_scan_force_segments(int segments) {
    if (segments < 0) return -1;
    return g_forced_segments.exchange(segments);
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

}  // extern "C"
