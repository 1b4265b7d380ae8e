"""ctypes binding of libssm.so (include/ssm.h): argument marshalling only.

Every step of the computation runs in the CUDA kernels behind the C ABI.  There is no
fallback: if the library is missing or was built for another architecture the calls
raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssm.so")

SSM_F32, SSM_BF16 = 0, 1
SSM_OK, SSM_ERR_INVALID_ARG, SSM_ERR_UNSUPPORTED, SSM_ERR_ALIGNMENT, SSM_ERR_CUDA, SSM_ERR_SCRATCH = range(6)

_DTYPE_CODE = {torch.float32: SSM_F32, torch.bfloat16: SSM_BF16}

_lib = None
_lock = threading.Lock()


class SsmError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__("%s (status %d)" % (msg, status))
        self.status = status


def load_library(path: str | None = None):
    """Load libssm.so once (raises if it is absent: build it with
    ``python -m selective_state_space_45_b200.build``)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError("libssm.so not found at %s; build it first "
                               "(python -m selective_state_space_45_b200.build)" % p)
        lib = ctypes.CDLL(p)
        vp, i = ctypes.c_void_p, ctypes.c_int
        lib.ssm_selective_scan_fwd.restype = i
        lib.ssm_selective_scan_fwd.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, vp, vp, vp,
                                               i, i, i, i, i, i, vp]
        lib.ssm_selective_scan_fwd_ex.restype = i
        lib.ssm_selective_scan_fwd_ex.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, vp, vp, vp, vp, i,
                                                  i, i, i, i, i, i, vp]
        lib.ssm_selective_scan_fwd_noalloc.restype = i
        lib.ssm_selective_scan_fwd_noalloc.argtypes = list(lib.ssm_selective_scan_fwd.argtypes)
        lib.ssm_state_step.restype = i
        lib.ssm_state_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
        lib.ssm_causal_conv1d_fwd.restype = i
        lib.ssm_causal_conv1d_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
        lib.ssm_causal_conv1d_step.restype = i
        lib.ssm_causal_conv1d_step.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
        lib.ssm_ssd_fwd.restype = i
        lib.ssm_ssd_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
        lib.ssm_state_step_multi.restype = i
        lib.ssm_state_step_multi.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
        lib.ssm_selective_scan_bwd.restype = i
        lib.ssm_selective_scan_bwd.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, vp, vp, vp, vp,
                                               vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                               i, i, i, i, i, i, vp]
        lib.ssm_status_string.restype = ctypes.c_char_p
        lib.ssm_status_string.argtypes = [i]
        lib.ssm_version.restype = i
        lib.ssm_version.argtypes = []
        lib.ssm_device_timeouts.restype = ctypes.c_uint
        lib.ssm_device_timeouts.argtypes = []
        lib.ssm_scan_force_segments.restype = i
        lib.ssm_scan_force_segments.argtypes = [i]
        lib.ssm_sfu_probe.restype = i
        lib.ssm_sfu_probe.argtypes = [vp, i, i, vp]
        _lib = lib
        return lib


def ssm_status_string(status: int) -> str:
    return load_library().ssm_status_string(int(status)).decode()


def ssm_version() -> int:
    return int(load_library().ssm_version())


def ssm_device_timeouts() -> int:
    """How many bounded waits inside the library's kernels gave up on this device (0 in
    normal operation; see include/ssm.h).  Synchronises with the device."""
    return int(load_library().ssm_device_timeouts())


def ssm_sfu_probe(out, blocks, iters, stream=None):
    """Diagnostic SFU throughput probe (see include/ssm.h): ``blocks`` CTAs of 256 threads,
    8 ex2 chains of ``iters`` steps per thread; ``out`` is a CUDA fp32 tensor of at least
    blocks * 256 elements.  Asynchronous on ``stream``."""
    if out.dtype.itemsize != 4 or out.numel() < int(blocks) * 256:
        raise ValueError("out must hold blocks * 256 fp32 values")
    _check(load_library().ssm_sfu_probe(_ptr(out), int(blocks), int(iters), _stream(stream, out)))


def ssm_scan_force_segments(segments: int) -> int:
    """Testing and tuning: force the time-segment count of the following scans (0 restores
    the automatic plan).  Returns the previous setting (see include/ssm.h)."""
    prev = int(load_library().ssm_scan_force_segments(int(segments)))
    if prev < 0:
        raise ValueError("segments must be >= 0")
    return prev


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to libssm must be contiguous")
    return t.data_ptr()


def _stream(stream, *tensors):
    if stream is None:
        dev = next((t.device for t in tensors if isinstance(t, torch.Tensor) and t.is_cuda), None)
        if dev is None:
            return None
        return torch.cuda.current_stream(dev).cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status):
    if status != SSM_OK:
        raise SsmError(status, ssm_status_string(status))


def ssm_selective_scan_fwd(x, delta, delta_bias, delta_softplus, A, B, C, D, z, y, final_state,
                           stream=None):
    """Selective scan forward (see include/ssm.h).  Tensors are CUDA tensors in the
    layouts of the header: x, delta, z, y [batch, dim, L]; B, C [batch, L, N]; A [dim, N];
    D, delta_bias [dim]; final_state [batch, dim, N].  Writes y and final_state in place."""
    batch, dim, L = x.shape
    N = A.shape[1]
    _check(load_library().ssm_selective_scan_fwd(
        _ptr(x), _ptr(delta), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(A), _ptr(B),
        _ptr(C), _ptr(D), _ptr(z), _ptr(y), _ptr(final_state), batch, dim, L, N,
        _DTYPE_CODE[x.dtype], _DTYPE_CODE[y.dtype], _stream(stream, x, y)))


def ssm_selective_scan_fwd_ex(x, delta, delta_bias, delta_softplus, A, B, C, D, z, y, final_state,
                              initial_state=None, zoh_exact=False, stream=None):
    """``ssm_selective_scan_fwd`` with a start state and the exact zero-order-hold gain
    (see include/ssm.h); initial_state is [batch, dim, N] fp32 or None."""
    batch, dim, L = x.shape
    N = A.shape[1]
    _check(load_library().ssm_selective_scan_fwd_ex(
        _ptr(x), _ptr(delta), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(A), _ptr(B),
        _ptr(C), _ptr(D), _ptr(z), _ptr(y), _ptr(final_state), _ptr(initial_state),
        int(bool(zoh_exact)), batch, dim, L, N, _DTYPE_CODE[x.dtype], _DTYPE_CODE[y.dtype],
        _stream(stream, x, y)))


def ssm_selective_scan_fwd_noalloc(x, delta, delta_bias, delta_softplus, A, B, C, D, z, y,
                                   final_state, stream=None):
    """Allocation-free variant of ``ssm_selective_scan_fwd`` (see include/ssm.h): same
    arguments and results; long sequences use a fixed device array for their scratch."""
    batch, dim, L = x.shape
    N = A.shape[1]
    _check(load_library().ssm_selective_scan_fwd_noalloc(
        _ptr(x), _ptr(delta), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(A), _ptr(B),
        _ptr(C), _ptr(D), _ptr(z), _ptr(y), _ptr(final_state), batch, dim, L, N,
        _DTYPE_CODE[x.dtype], _DTYPE_CODE[y.dtype], _stream(stream, x, y)))


def ssm_state_step(state, x, delta, A, B, C, D, z, y, stream=None):
    """One decode step (see include/ssm.h): state [batch, dim, N] fp32 updated in place;
    x, delta, z, y [batch, dim]; B, C [batch, N]."""
    batch, dim, N = state.shape
    _check(load_library().ssm_state_step(
        _ptr(state), _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(y),
        batch, dim, N, _DTYPE_CODE[x.dtype], _DTYPE_CODE[y.dtype], _stream(stream, state, y)))


def ssm_ssd_fwd(x, a, B, C, y, initial_state=None, final_state=None, stream=None):
    """Mamba-2 SSD by chunks (see include/ssm.h): x, y [batch, L, heads, P]; a [batch, L,
    heads] fp32; B, C [batch, L, heads, N] bf16; states [batch, heads, P, N] fp32."""
    batch, L, heads, P = x.shape
    N = B.shape[-1]
    _check(load_library().ssm_ssd_fwd(
        _ptr(x), _ptr(a), _ptr(B), _ptr(C), _ptr(y), _ptr(initial_state), _ptr(final_state),
        batch, L, heads, P, N, _DTYPE_CODE[x.dtype], _DTYPE_CODE[y.dtype], _stream(stream, x, y)))


def ssd(x, a, B, C, initial_state=None, out_dtype=None, return_final_state=True, stream=None):
    """Allocate y (and the final state) with torch and run ``ssm_ssd_fwd``."""
    batch, L, heads, P = x.shape
    y = torch.empty(x.shape, device=x.device, dtype=out_dtype or torch.float32)
    fs = (torch.empty((batch, heads, P, B.shape[-1]), device=x.device, dtype=torch.float32)
          if return_final_state else None)
    ssm_ssd_fwd(x, a, B, C, y, initial_state, fs, stream)
    return (y, fs) if return_final_state else y


def ssm_state_step_multi(state, x, delta, A, B, C, D, z, y, stream=None):
    """Several decode tokens on the carried state (see include/ssm.h): state [batch, dim, N]
    fp32 updated in place; x, delta, z, y [ntok, batch, dim]; B, C [ntok, batch, N]."""
    batch, dim, N = state.shape
    ntok = x.shape[0]
    _check(load_library().ssm_state_step_multi(
        _ptr(state), _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(y),
        ntok, batch, dim, N, _DTYPE_CODE[x.dtype], _DTYPE_CODE[y.dtype], _stream(stream, state, y)))


def ssm_selective_scan_bwd(x, delta, delta_bias, delta_softplus, A, B, C, D, z, initial_state,
                           dy, dfinal_state, dx, ddelta, dA, dB, dC, dD, dz, ddelta_bias,
                           dinitial_state, stream=None):
    """Backward of the scan (see include/ssm.h).  Gradient tensors share dy's dtype
    (dx, ddelta, dz, dB, dC); dA, dD, ddelta_bias, dinitial_state are fp32.  Optional
    arguments are None.  Writes the gradients in place."""
    batch, dim, L = x.shape
    N = A.shape[1]
    _check(load_library().ssm_selective_scan_bwd(
        _ptr(x), _ptr(delta), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(A), _ptr(B),
        _ptr(C), _ptr(D), _ptr(z), _ptr(initial_state), _ptr(dy), _ptr(dfinal_state),
        _ptr(dx), _ptr(ddelta), _ptr(dA), _ptr(dB), _ptr(dC), _ptr(dD), _ptr(dz),
        _ptr(ddelta_bias), _ptr(dinitial_state), batch, dim, L, N,
        _DTYPE_CODE[x.dtype], _DTYPE_CODE[dy.dtype], _stream(stream, x, dy)))


def selective_scan_bwd(dy, x, delta, A, B, C, D=None, z=None, delta_bias=None,
                       delta_softplus=False, initial_state=None, dfinal_state=None, stream=None):
    """Allocate the gradients with torch (dy's dtype for the tensor gradients) and run the
    backward; returns a dict dx, ddelta, dz, dA, dB, dC, dD, ddelta_bias, dinitial_state
    (None where the input was absent)."""
    batch, dim, L = x.shape
    N = A.shape[1]
    dev, gd, f32 = x.device, dy.dtype, torch.float32
    g = dict(dx=torch.empty((batch, dim, L), device=dev, dtype=gd),
             ddelta=torch.empty((batch, dim, L), device=dev, dtype=gd),
             dz=None if z is None else torch.empty((batch, dim, L), device=dev, dtype=gd),
             dA=torch.empty((dim, N), device=dev, dtype=f32),
             dB=torch.empty((batch, L, N), device=dev, dtype=gd),
             dC=torch.empty((batch, L, N), device=dev, dtype=gd),
             dD=None if D is None else torch.empty(dim, device=dev, dtype=f32),
             ddelta_bias=None if delta_bias is None else torch.empty(dim, device=dev, dtype=f32),
             dinitial_state=None if initial_state is None else
             torch.empty((batch, dim, N), device=dev, dtype=f32))
    ssm_selective_scan_bwd(x, delta, delta_bias, delta_softplus, A, B, C, D, z, initial_state,
                           dy, dfinal_state, g["dx"], g["ddelta"], g["dA"], g["dB"], g["dC"],
                           g["dD"], g["dz"], g["ddelta_bias"], g["dinitial_state"], stream)
    return g


def ssm_causal_conv1d_fwd(x, weight, bias, initial_window, u, final_window, silu=True,
                          stream=None):
    """Causal depthwise convolution + bias + SiLU (see include/ssm.h): x, u [batch, dim, L];
    weight [dim, width] fp32; bias [dim] fp32 or None; initial_window / final_window
    [batch, dim, width-1] fp32 or None.  Writes u (and final_window) in place."""
    batch, dim, L = x.shape
    width = weight.shape[1]
    _check(load_library().ssm_causal_conv1d_fwd(
        _ptr(x), _ptr(weight), _ptr(bias), _ptr(initial_window), _ptr(u), _ptr(final_window),
        batch, dim, L, width, int(bool(silu)), _DTYPE_CODE[x.dtype], _DTYPE_CODE[u.dtype],
        _stream(stream, x, u)))


def ssm_causal_conv1d_step(window, x, weight, bias, u, silu=True, stream=None):
    """One decode token of the convolution (see include/ssm.h): window [batch, dim, width-1]
    fp32 updated in place (may be None for width 1); x, u [batch, dim]."""
    batch, dim = x.shape
    width = weight.shape[1]
    _check(load_library().ssm_causal_conv1d_step(
        _ptr(window), _ptr(x), _ptr(weight), _ptr(bias), _ptr(u), batch, dim, width,
        int(bool(silu)), _DTYPE_CODE[x.dtype], _DTYPE_CODE[u.dtype], _stream(stream, x, u)))


def causal_conv1d(x, weight, bias=None, initial_window=None, silu=True, out_dtype=None,
                  return_final_window=False, stream=None):
    """Allocate u (and the final window) with torch and run the convolution."""
    batch, dim, L = x.shape
    u = torch.empty((batch, dim, L), device=x.device, dtype=out_dtype or x.dtype)
    fw = (torch.empty((batch, dim, weight.shape[1] - 1), device=x.device, dtype=torch.float32)
          if return_final_window else None)
    ssm_causal_conv1d_fwd(x, weight, bias, initial_window, u, fw, silu, stream)
    return (u, fw) if return_final_window else u


def selective_scan(x, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=False,
                   out_dtype=None, return_final_state=True, initial_state=None, zoh_exact=False,
                   stream=None):
    """Allocate y (and the final state) with torch and run the scan."""
    batch, dim, L = x.shape
    y = torch.empty((batch, dim, L), device=x.device, dtype=out_dtype or x.dtype)
    fs = (torch.empty((batch, dim, A.shape[1]), device=x.device, dtype=torch.float32)
          if return_final_state else None)
    ssm_selective_scan_fwd_ex(x, delta, delta_bias, delta_softplus, A, B, C, D, z, y, fs,
                              initial_state, zoh_exact, stream)
    return (y, fs) if return_final_state else y
