/*
 * ssm.h -- C ABI of the B200 selective state-space scan library (libssm.so).
 *
 * Operations:
 *   ssm_selective_scan_fwd  the selective scan (S6) over a whole sequence;
 *   ssm_state_step          one decode token on a carried state, updated in place;
 *   ssm_state_step_multi    several decode tokens on a carried state in one call;
 *   ssm_causal_conv1d_fwd   the causal depthwise convolution + SiLU that feeds the scan;
 *   ssm_causal_conv1d_step  its one-token form on a carried window, updated in place;
 *   ssm_selective_scan_bwd  the gradients of the scan (training), states recomputed;
 *   ssm_ssd_fwd             Mamba-2's state-space dual by chunks, on tensor cores.
 *
 * The scan and the state step compute, per sequence b and channel d, with an N-wide fp32 state h:
 *     Delta_t = softplus(delta[b,d,t] + delta_bias[d])   (bias and softplus optional)
 *     h_n    <- exp(Delta_t * A[d,n]) * h_n + Delta_t * B[b,t,n] * x[b,d,t]
 *     y[b,d,t] = (sum_n C[b,t,n] * h_n + D[d] * x[b,d,t]) * SiLU(z[b,d,t])
 * Sources: zero-order-hold decay Abar = exp(Delta A) and its Euler input gain
 * Bbar ~ Delta B ("Module 19: State-Space Models (Mamba)", learnllm, section "The Math:
 * The State-Space Recurrence"); input-dependent Delta, B, C ("Beyond attention with
 * Mamba, state space models and hybrids", xmarva lesson 10, section 3 "Selectivity");
 * softplus step with bias, the skip D*x and then the SiLU(z) gate (same lesson,
 * section 4 "The Mamba block"); the one-token update (section 7 "Generation with a
 * state of fixed size").
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library keeps
 *    no state between calls.  Two calls may take a temporary scratch buffer with
 *    cudaMallocAsync / cudaFreeAsync on cuda_stream: ssm_selective_scan_fwd (and _ex)
 *    for long sequences with few channels (see below), and ssm_selective_scan_bwd.
 *    ssm_selective_scan_fwd_noalloc is the scan's form that never allocates; every
 *    other call allocates nothing.
 *  - Every pointer must be 16-byte aligned (SSM_ERR_ALIGNMENT otherwise).
 *  - The call is asynchronous on `cuda_stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and never synchronises.  Argument errors are returned before
 *    anything is launched; a launch failure returns SSM_ERR_CUDA.  Faults inside a
 *    kernel surface, as usual for CUDA, at the caller's next synchronisation.
 *  - dtype codes: SSM_F32 (fp32) or SSM_BF16 (bf16).  A, D, delta_bias and the state
 *    are always fp32; the state arithmetic is fp32 whatever the input dtype.
 *  - For the S6 calls (scan, backward, state steps) dstate (N) must be in 1..16
 *    (SSM_ERR_UNSUPPORTED above 16); ssm_ssd_fwd takes its own sizes (below).
 *  - Output buffers must not overlap input buffers (the convolution checks and returns
 *    SSM_ERR_INVALID_ARG; for the scan the result of an overlap is undefined).
 */
#ifndef SSM_H_
#define SSM_H_

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSM_F32 = 0,
    SSM_BF16 = 1
} ssm_dtype;

typedef enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = 1,   /* null required pointer, negative size, bad dtype code   */
    SSM_ERR_UNSUPPORTED = 2,   /* dstate above 16, conv width above 8, sizes out of range */
    SSM_ERR_ALIGNMENT = 3,     /* a pointer not 16-byte aligned                            */
    SSM_ERR_CUDA = 4,          /* the CUDA runtime reported an error at launch             */
    SSM_ERR_SCRATCH = 5        /* ssm_selective_scan_fwd_noalloc: fixed scratch too small  */
} ssm_status;

/*
 * Selective scan forward over whole sequences, starting from a zero state.
 *
 *   x, delta, z : [batch][dim][seqlen], in_dtype, contiguous ("channels first").
 *                 delta is the raw step; z may be NULL (no gate).
 *   delta_bias  : [dim] fp32, or NULL (no bias).  Added to delta before the softplus.
 *   delta_softplus : nonzero -> Delta = softplus(delta + bias); zero -> Delta = delta + bias.
 *   A           : [dim][dstate] fp32 (Mamba keeps it negative; any value is accepted).
 *   B, C        : [batch][seqlen][dstate], in_dtype, shared by all channels of a sequence.
 *   D           : [dim] fp32, or NULL (no skip term).
 *   y           : [batch][dim][seqlen], out_dtype, written.
 *   final_state : [batch][dim][dstate] fp32, or NULL; receives h after the last token
 *                 (all zeros when seqlen == 0).
 * Sizes: batch, dim, seqlen >= 0 (a zero size launches nothing except the zero final
 * state); 1 <= dstate <= 16; batch*dim*seqlen and batch*seqlen*dstate must be below 2^62
 * and seqlen below 2^31.
 * The N-wide state never leaves the chip: only y and final_state are written.
 * When batch * ceil(dim / 32) CTAs cannot fill the GPU, each sequence is cut into segments
 * scanned in parallel, each from its true carry.  Before the scans, each earlier segment's
 * end state is summed from its last tokens, those whose decay is not yet 0 in fp32.  Those
 * end states and step sums (batch * dim * segments * (padded dstate + 1) floats, a few MiB
 * at most) go to a stream-ordered temporary buffer freed on the same stream before the
 * call returns.
 */
int ssm_selective_scan_fwd(const void *x, const void *delta, const float *delta_bias,
                           int delta_softplus, const float *A, const void *B, const void *C,
                           const float *D, const void *z, void *y, float *final_state,
                           int batch, int dim, int seqlen, int dstate,
                           int in_dtype, int out_dtype, void *cuda_stream);

/*
 * ssm_selective_scan_fwd with two options (ssm_selective_scan_fwd passes NULL and 0):
 *   initial_state : [batch][dim][dstate] fp32, or NULL.  The scan starts from this state
 *                   instead of zero, e.g. to continue a sequence whose earlier tokens
 *                   were scanned by a previous call (its final_state).  With seqlen == 0
 *                   the final state is a copy of it.
 *   zoh_exact     : nonzero -> exact zero-order-hold input gain
 *                   Bbar = (exp(Delta a) - 1) / a * B (the limit Delta * B where a == 0)
 *                   instead of the Euler gain Delta * B ("Module 19: State-Space Models
 *                   (Mamba)", learnllm, "The Math: The State-Space Recurrence"; the
 *                   understandingdata page's ZOH numbers use this gain).
 * All other arguments, layouts and errors as ssm_selective_scan_fwd.
 */
int ssm_selective_scan_fwd_ex(const void *x, const void *delta, const float *delta_bias,
                              int delta_softplus, const float *A, const void *B, const void *C,
                              const float *D, const void *z, void *y, float *final_state,
                              const float *initial_state, int zoh_exact,
                              int batch, int dim, int seqlen, int dstate,
                              int in_dtype, int out_dtype, void *cuda_stream);

/*
 * Allocation-free variant of ssm_selective_scan_fwd: same arguments, same results, and no
 * memory allocation of any kind (no cudaMalloc, cudaMallocAsync or cudaFree).  The pages
 * have no counterpart to this call; it exists for callers that are not allowed to
 * allocate device memory while they run: a serving engine that has handed all free
 * device memory to its own pool before the first request, code running under an
 * allocator policy that forbids the library to allocate behind its back, or a latency-
 * critical loop that must not touch the allocator after start-up.
 *
 * Where ssm_selective_scan_fwd takes a stream-ordered temporary buffer (long sequences
 * with few channels are scanned in segments whose end states must be kept between
 * launches), this call uses a fixed 4 MiB array in device memory instead.  That array
 * exists on every GPU that loads the library and stays there until the process exits.
 *  - Every call asks the runtime for the array's address in the current device's
 *    context (a lookup, no allocation), so the address stays right after a
 *    cudaDeviceReset.  The first call on a device may load the library's device code;
 *    make that first call before any CUDA stream capture on the device.
 *  - A call whose segmented scan would need more than 4 MiB of scratch (batch * dim *
 *    segments * (padded dstate + 1) floats, padded dstate = 4, 8 or 16) returns
 *    SSM_ERR_SCRATCH and launches nothing.  Calls that need no segments work at any size.
 *  - All calls share the array and it keeps the contents of the last call.  Nothing in it
 *    has to start at zero: each call writes every entry it later reads.  Two calls whose
 *    kernels may overlap on the GPU (different streams, or different host threads without
 *    ordering between their streams) race on the array and give wrong results; serialise
 *    them on one stream.
 */
int ssm_selective_scan_fwd_noalloc(const void *x, const void *delta, const float *delta_bias,
                                   int delta_softplus, const float *A, const void *B, const void *C,
                                   const float *D, const void *z, void *y, float *final_state,
                                   int batch, int dim, int seqlen, int dstate,
                                   int in_dtype, int out_dtype, void *cuda_stream);

/*
 * Testing and tuning only: force the number of time segments every following scan call
 * (ssm_selective_scan_fwd, _ex, _noalloc) cuts each sequence into, whatever its shape, so
 * that the long-sequence plan (tail sums, fold, segment scans) can be exercised on small
 * inputs.  segments = 0 restores the automatic choice; a value above the sequence's tile
 * count gives fewer, whole-tile segments.  Returns the previous setting, or -1 (nothing
 * changed) for a negative argument.  Process-wide: calls that race with a scan on another
 * host thread may see either setting.  The pages have no counterpart to this call.
 */
int ssm_scan_force_segments(int segments);

/*
 * One decode step: every (b, d) channel takes one token and its state is updated in place.
 *
 *   state       : [batch][dim][dstate] fp32, read and overwritten.
 *   x, delta, z : [batch][dim], in_dtype.  delta is the final step Delta (already
 *                 positive: no bias, no softplus is applied here).  z may be NULL.
 *   A           : [dim][dstate] fp32.   D: [dim] fp32 or NULL.
 *   B, C        : [batch][dstate], in_dtype.
 *   y           : [batch][dim], out_dtype, written.
 * Chaining L calls from a state h0 gives the same y and state as the scan over those L
 * tokens started from h0.
 */
int ssm_state_step(float *state, const void *x, const void *delta, const float *A,
                   const void *B, const void *C, const float *D, const void *z, void *y,
                   int batch, int dim, int dstate, int in_dtype, int out_dtype,
                   void *cuda_stream);

/*
 * Causal depthwise convolution, bias and SiLU over whole sequences (the filter in front of
 * the scan: "Module 19: State-Space Models (Mamba)", learnllm, section "The Causal
 * Convolution"; xmarva lesson 10, section 4 "The Mamba block").  Per sequence b, channel d
 * and position t, with K = width and xe the input preceded by the K-1 window values:
 *     u[b,d,t] = act( bias[d] + sum_{i<K} weight[d,i] * xe[b,d,t-K+1+i] )
 * act = SiLU when silu != 0, else the identity.  Output t never reads a later input.
 *
 *   x, u           : [batch][dim][seqlen], in_dtype / out_dtype (u written).
 *   weight         : [dim][width] fp32, tap i multiplies the input K-1-i steps back.
 *   bias           : [dim] fp32 or NULL (zero).
 *   initial_window : [batch][dim][width-1] fp32 or NULL: the width-1 inputs before
 *                    position 0, oldest first (NULL = zeros, the left pad).
 *   final_window   : [batch][dim][width-1] fp32 or NULL: receives the last width-1
 *                    inputs (window included when seqlen < width-1), the window that
 *                    ssm_causal_conv1d_step continues from.
 * width must be 1..8 (SSM_ERR_UNSUPPORTED above 8).  Widths 1..4 with seqlen a multiple
 * of 8 (bf16 input) or 4 (fp32 input) take the vectorised kernel; others a per-element
 * kernel with the same results.  u may not overlap x; final_window may not overlap
 * initial_window, x or u (SSM_ERR_INVALID_ARG).  seqlen = 0 copies the window through.
 */
int ssm_causal_conv1d_fwd(const void *x, const float *weight, const float *bias,
                          const float *initial_window, void *u, float *final_window,
                          int batch, int dim, int seqlen, int width, int silu,
                          int in_dtype, int out_dtype, void *cuda_stream);

/*
 * One decode token of the convolution (xmarva lesson 10, section 7 "Generation with a
 * state of fixed size": the block keeps the last inputs of its convolution next to h).
 *
 *   window : [batch][dim][width-1] fp32, the previous width-1 inputs, oldest first; read,
 *            then overwritten with the window shifted by one and x appended.  May be NULL
 *            when width = 1.
 *   x, u   : [batch][dim], in_dtype / out_dtype (u written).
 *   weight, bias, silu, width: as for ssm_causal_conv1d_fwd.
 * Chaining L calls from a window gives the same u and window as ssm_causal_conv1d_fwd
 * over those L tokens with that initial_window.  window may not overlap x or u.
 */
int ssm_causal_conv1d_step(float *window, const void *x, const float *weight, const float *bias,
                           void *u, int batch, int dim, int width, int silu,
                           int in_dtype, int out_dtype, void *cuda_stream);

/*
 * Backward of the scan (Euler gain): the gradients of
 *     loss = sum dy[b,d,t] * y[b,d,t] + sum dfinal_state[b,d,n] * final_state[b,d,n]
 * with respect to every input of ssm_selective_scan_fwd_ex (zoh_exact = 0), for the
 * training half that "Beyond attention with Mamba, state space models and hybrids"
 * (xmarva lesson 10, section 6) describes: the states are recomputed in the backward pass,
 * never stored.  Reverse-mode differentiation of the recurrence: with mu the adjoint
 * flowing into h_t, lambda_n = dypre_t C_t[n] + mu_n, dC_t[n] += dypre_t h_t[n],
 * dB_t[n] += lambda_n Delta_t x_t, dx_t = dypre_t D + sum_n lambda_n Delta_t B_t[n],
 * dDelta_t = sum_n lambda_n (B_t[n] x_t + h_{t-1}[n] Abar_t[n] A[n]), dA[n] +=
 * lambda_n h_{t-1}[n] Abar_t[n] Delta_t, mu_n <- Abar_t[n] lambda_n, where dypre_t =
 * dy_t SiLU(z_t) and dz_t = dy_t ypre_t SiLU'(z_t).
 *
 *   inputs     : as ssm_selective_scan_fwd_ex (x, delta, z, B, C in in_dtype; A, D,
 *                delta_bias, initial_state fp32; z, D, delta_bias, initial_state optional).
 *   dy         : [batch][dim][seqlen], grad_dtype.
 *   dfinal_state: [batch][dim][dstate] fp32 or NULL (zero).
 *   dx, ddelta : [batch][dim][seqlen], grad_dtype, written (ddelta is the gradient of the
 *                raw delta, through the bias and softplus).
 *   dz         : [batch][dim][seqlen], grad_dtype, or NULL (requires z when given).
 *   dB, dC     : [batch][seqlen][dstate], grad_dtype, written.
 *   dA         : [dim][dstate] fp32, written.   dD, ddelta_bias: [dim] fp32 or NULL.
 *   dinitial_state: [batch][dim][dstate] fp32 or NULL: the gradient of the start state.
 * Sums over channels (dB, dC) and over sequences and positions (dA, dD, ddelta_bias) are
 * formed from per-CTA partial sums added in a fixed order: results are deterministic.
 * Takes a stream-ordered scratch buffer of about batch*dim'*(20*L' + 72) bytes, dim' = dim
 * rounded up to 32 and L' = seqlen rounded up to 16 (the state before every 4th token,
 * 16*L' bytes per channel, and per-CTA partial sums), with cudaMallocAsync / cudaFreeAsync
 * on cuda_stream.
 * dstate must be 1..16; zoh_exact has no backward here.
 * seqlen = 0 writes zero parameter gradients and dinitial_state = dfinal_state.
 */
int ssm_selective_scan_bwd(const void *x, const void *delta, const float *delta_bias,
                           int delta_softplus, const float *A, const void *B, const void *C,
                           const float *D, const void *z, const float *initial_state,
                           const void *dy, const float *dfinal_state,
                           void *dx, void *ddelta, float *dA, void *dB, void *dC, float *dD,
                           void *dz, float *ddelta_bias, float *dinitial_state,
                           int batch, int dim, int seqlen, int dstate,
                           int in_dtype, int grad_dtype, void *cuda_stream);

/*
 * Several decode tokens on a carried state in one call (speculative or chunked decoding):
 * ntok chained ssm_state_step calls, with the state read and written once.
 *
 *   state       : [batch][dim][dstate] fp32, read and overwritten with the state after
 *                 the last token.
 *   x, delta, z : [ntok][batch][dim], in_dtype (delta already positive; z may be NULL).
 *   B, C        : [ntok][batch][dstate], in_dtype.   A, D: as for ssm_state_step.
 *   y           : [ntok][batch][dim], out_dtype, written.
 * Per token the arithmetic is that of ssm_state_step in the same order: the results are
 * bit-identical to ntok chained calls.  ntok = 0 does nothing.
 */
int ssm_state_step_multi(float *state, const void *x, const void *delta, const float *A,
                         const void *B, const void *C, const float *D, const void *z, void *y,
                         int ntok, int batch, int dim, int dstate, int in_dtype, int out_dtype,
                         void *cuda_stream);

/*
 * Mamba-2's state-space dual (SSD) by chunks ("Beyond attention with Mamba, state space
 * models and hybrids", xmarva lesson 10, section 8 "Mamba-2: the same model as
 * attention"): one decay per head and a headdim x dstate state per head,
 *     S <- exp(a_t) S + x_t B_t^T,    y_t = S C_t    (per sequence and head)
 * computed as attention with the decay mask inside chunks of 128 tokens and the
 * recurrence between chunks.  x already carries the step (x = Delta * input), a = Delta * A.
 *
 *   x, y          : [batch][seqlen][heads][headdim]; x bf16, y out_dtype (written).
 *   a             : [batch][seqlen][heads] fp32.
 *   B, C          : [batch][seqlen][heads][dstate] bf16.
 *   initial_state : [batch][heads][headdim][dstate] fp32 or NULL (zero).
 *   final_state   : [batch][heads][headdim][dstate] fp32 or NULL (not written).
 * in_dtype must be SSM_BF16 (the tensor-core operands); headdim 32 or 64 and dstate 64 or
 * 128 (SSM_ERR_UNSUPPORTED otherwise).  Products run on the tensor cores (tcgen05) on bf16
 * operands with fp32 accumulation; the masked scores, the decay-weighted inputs and the
 * state are rounded to bf16 where they enter a product.  The state stays on the chip
 * between chunks (fp32): the call allocates nothing and writes only y and final_state.
 * seqlen = 0 copies the start state through.  Uses about 100 KB of shared memory and 256
 * tensor-memory columns per CTA (two CTAs per SM).
 */
int ssm_ssd_fwd(const void *x, const float *a, const void *B, const void *C, void *y,
                const float *initial_state, float *final_state,
                int batch, int seqlen, int heads, int headdim, int dstate,
                int in_dtype, int out_dtype, void *cuda_stream);

/*
 * Number of times, since the library was loaded on the current device, that a kernel gave
 * up waiting on its own asynchronous copies or tensor-core operations (each such wait is
 * bounded, about a second).  0 in normal operation; a nonzero count means the results of
 * the call that timed out are not valid.  Synchronises with the device; ~0u if the count
 * cannot be read.  The pages have no counterpart to this call.
 */
unsigned ssm_device_timeouts(void);

/*
 * Diagnostic, not part of the path: the SFU exponential rate that the scan's roofline
 * counts against (decays are SFU ex2 operations).  Launches `blocks` CTAs of 256 threads;
 * each thread runs 8 independent chains v <- 2^(-v) for `iters` steps (one ex2 each, the
 * values staying in [0.5, 1]) and writes the sum of its chains to out[thread] (`out`:
 * device, blocks * 256 floats, 16-byte aligned, owned by the caller).  blocks * 256 * 8 *
 * iters ex2 in all; time the call with events on `cuda_stream`.  SSM_ERR_INVALID_ARG for a
 * NULL `out`, blocks < 1 or iters < 0; asynchronous like every call.
 */
int ssm_sfu_probe(float *out, int blocks, int iters, void *cuda_stream);

/* Static, NUL-terminated description of a status code (never NULL). */
const char *ssm_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
int ssm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSM_H_ */
