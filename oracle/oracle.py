"""fp64 CPU oracle for the selective state-space scan (S6) -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this module.  It shares no code with the CUDA library: the sequential scan
and the decode step are the plain C loops in ``ssm_oracle.c`` (built into
``libssm_oracle.so`` next to this file); everything else here is numpy written for
tiny inputs so that it can be read against the pages by eye.

Functions and the passages they follow:

``scan``            the full recurrence with discretisation, readout, skip and gate:
                    learnllm "Module 19", "The Math: The State-Space Recurrence";
                    xmarva lesson 10, sections 3 "Selectivity" and 4 "The Mamba block".
``step``            one token of the same recurrence on a carried state: xmarva
                    lesson 10, section 7 "Generation with a state of fixed size".
``affine_scan_loop``          h_t = a_t h_{t-1} + b_t left to right: learnllm "Module 19",
                              "The Parallel Scan".
``affine_scan_hillis_steele`` the same prefix computed in log2(L) rounds of the
                              associative composition (a2,b2)o(a1,b1) = (a2 a1, a2 b1 + b2):
                              learnllm "The Parallel Scan"; xmarva section 6 "The scan".
``scan_parallel_reference``   the whole selective scan routed through the Hillis-Steele
                              rounds over N-expanded pairs (tiny inputs only): an
                              implementation independent of the C loop.
``scan_bwd``        gradients of the scan by reverse-mode differentiation of the same
                    recurrence (Euler gain): the training half; xmarva lesson 10,
                    section 6 (Mamba's kernel recomputes the states in the backward pass).
``ssd_loop`` / ``ssd_chunked``  Mamba-2's state-space dual (scalar decay per head, a
                    P x N state per head): the step-by-step loop and the chunked form,
                    attention inside chunks and the recurrence between them; xmarva
                    lesson 10, section 8 "Mamba-2: the same model as attention".
``causal_conv1d`` / ``conv1d_step``  the causal depthwise convolution with SiLU in front of
                              the scan, and its one-token window form: learnllm "Module 19",
                              "The Causal Convolution"; xmarva lesson 10, sections 4 and 7.
``lti_kernel`` / ``lti_conv`` the convolutional face of a time-invariant SSM,
                              K = (C Bbar, C Abar Bbar, C Abar^2 Bbar, ...), y = K * x:
                              learnllm "Two Faces: Recurrent = Convolutional".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB = os.path.join(_HERE, "libssm_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``ssm_oracle.c`` into ``libssm_oracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            p = ctypes.c_void_p
            i64 = ctypes.c_int64
            lib.oracle_scan.restype = ctypes.c_int
            lib.oracle_scan.argtypes = [p, p, p, ctypes.c_int, p, p, p, p, p, p, ctypes.c_int,
                                        p, p, i64, i64, i64, i64, ctypes.c_int]
            lib.oracle_step.restype = None
            lib.oracle_step.argtypes = [p, p, p, p, p, p, p, p, p, i64, i64, i64]
            lib.oracle_scan_bwd.restype = ctypes.c_int
            lib.oracle_scan_bwd.argtypes = [p, p, p, ctypes.c_int, p, p, p, p, p, p, p, p,
                                            p, p, p, p, p, p, p, p, p, i64, i64, i64, i64]
            lib.oracle_ssd_loop.restype = ctypes.c_int
            lib.oracle_ssd_loop.argtypes = [p, p, p, p, p, p, p, i64, i64, i64, i64, i64]
            lib.oracle_causal_conv1d.restype = None
            lib.oracle_causal_conv1d.argtypes = [p, p, p, p, ctypes.c_int, p, p, i64, i64, i64, i64]
            lib.oracle_conv1d_step.restype = None
            lib.oracle_conv1d_step.argtypes = [p, p, p, p, ctypes.c_int, p, i64, i64, i64]
            _lib = lib
    return _lib


def _f64(a, shape=None):
    if a is None:
        return None
    if hasattr(a, "detach"):  # a torch tensor: widen exactly on the host
        a = a.detach().to("cpu").double().numpy()
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if shape is not None and a.shape != tuple(shape):
        raise ValueError("oracle: expected shape %s, got %s" % (tuple(shape), a.shape))
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def scan(x, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=False,
         h0=None, zoh_exact=False, nthreads=0, return_threads=False):
    """Sequential selective scan in fp64.

    Layouts: x, delta, z: [batch, dim, L]; B, C: [batch, L, N]; A: [dim, N];
    D, delta_bias: [dim]; h0: [batch, dim, N].  Returns ``(y, final_state)`` with y
    [batch, dim, L] and final_state [batch, dim, N], both float64.
    """
    x = _f64(x)
    if x.ndim != 3:
        raise ValueError("oracle.scan: x must be [batch, dim, L]")
    batch, dim, L = x.shape
    A = _f64(A)
    N = A.shape[1]
    delta = _f64(delta, (batch, dim, L))
    A = _f64(A, (dim, N))
    B = _f64(B, (batch, L, N))
    C = _f64(C, (batch, L, N))
    D = _f64(D, (dim,))
    z = _f64(z, (batch, dim, L))
    delta_bias = _f64(delta_bias, (dim,))
    h0 = _f64(h0, (batch, dim, N))
    y = np.empty((batch, dim, L), dtype=np.float64)
    hN = np.empty((batch, dim, N), dtype=np.float64)
    used = _load().oracle_scan(_ptr(x), _ptr(delta), _ptr(delta_bias), int(bool(delta_softplus)),
                               _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(h0),
                               int(bool(zoh_exact)), _ptr(y), _ptr(hN),
                               batch, dim, L, N, int(nthreads))
    if used < 0:
        raise ValueError("oracle.scan: unsupported sizes")
    if return_threads:
        return y, hN, used
    return y, hN


def step(state, x, delta, A, B, C, D=None, z=None):
    """One decode step in fp64: returns ``(y, new_state)``.

    Layouts: state [batch, dim, N]; x, delta, z: [batch, dim] (delta already the final
    step); B, C: [batch, N]; A: [dim, N]; D: [dim].
    """
    st = _f64(state).copy()
    batch, dim, N = st.shape
    x = _f64(x, (batch, dim))
    delta = _f64(delta, (batch, dim))
    A = _f64(A, (dim, N))
    B = _f64(B, (batch, N))
    C = _f64(C, (batch, N))
    D = _f64(D, (dim,))
    z = _f64(z, (batch, dim))
    y = np.empty((batch, dim), dtype=np.float64)
    _load().oracle_step(_ptr(st), _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                        _ptr(z), _ptr(y), batch, dim, N)
    return y, st


def scan_bwd(dy, x, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=False,
             h0=None, dfinal=None):
    """Gradients of  sum(dy * y) + sum(dfinal * final_state)  of the (Euler) scan, in fp64.

    Same layouts as ``scan``; dy [batch, dim, L], dfinal [batch, dim, N].  Returns a dict
    with dx, ddelta, dz (or None), dB, dC, dA, dD (or None), ddelta_bias (or None), dh0.
    """
    x = _f64(x)
    batch, dim, L = x.shape
    A = _f64(A)
    N = A.shape[1]
    dy = _f64(dy, (batch, dim, L))
    delta = _f64(delta, (batch, dim, L))
    B = _f64(B, (batch, L, N))
    C = _f64(C, (batch, L, N))
    D = _f64(D, (dim,))
    z = _f64(z, (batch, dim, L))
    delta_bias = _f64(delta_bias, (dim,))
    h0 = _f64(h0, (batch, dim, N))
    dfinal = _f64(dfinal, (batch, dim, N))
    out = dict(dx=np.empty((batch, dim, L)), ddelta=np.empty((batch, dim, L)),
               dz=None if z is None else np.empty((batch, dim, L)),
               dB=np.empty((batch, L, N)), dC=np.empty((batch, L, N)), dA=np.empty((dim, N)),
               dD=None if D is None else np.empty(dim),
               ddelta_bias=None if delta_bias is None else np.empty(dim),
               dh0=np.empty((batch, dim, N)))
    rc = _load().oracle_scan_bwd(
        _ptr(x), _ptr(delta), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(A), _ptr(B),
        _ptr(C), _ptr(D), _ptr(z), _ptr(h0), _ptr(dy), _ptr(dfinal),
        _ptr(out["dx"]), _ptr(out["ddelta"]), _ptr(out["dA"]), _ptr(out["dB"]), _ptr(out["dC"]),
        _ptr(out["dD"]), _ptr(out["dz"]), _ptr(out["ddelta_bias"]), _ptr(out["dh0"]),
        batch, dim, L, N)
    if rc != 0:
        raise ValueError("oracle.scan_bwd: unsupported sizes")
    return out


def ssd_loop(x, a, B, C, h0=None):
    """Mamba-2 SSD as its step-by-step recurrence, in fp64: returns ``(y, final_state)``.

    x [batch, L, heads, P] (already times the step), a [batch, L, heads] (= step * A),
    B, C [batch, L, heads, N], h0 [batch, heads, P, N].  y [batch, L, heads, P].
    """
    x = _f64(x)
    batch, L, heads, P = x.shape
    a = _f64(a, (batch, L, heads))
    B = _f64(B)
    N = B.shape[-1]
    B = _f64(B, (batch, L, heads, N))
    C = _f64(C, (batch, L, heads, N))
    h0 = _f64(h0, (batch, heads, P, N))
    y = np.empty((batch, L, heads, P))
    hN = np.empty((batch, heads, P, N))
    if _load().oracle_ssd_loop(_ptr(x), _ptr(a), _ptr(B), _ptr(C), _ptr(h0), _ptr(y), _ptr(hN),
                               batch, L, heads, P, N) != 0:
        raise ValueError("oracle.ssd_loop: bad sizes")
    return y, hN


def ssd_chunked(x, a, B, C, chunk=64, h0=None, dtype=np.float64):
    """Mamba-2 SSD by chunks (xmarva lesson 10, section 8): inside a chunk the outputs are
    masked attention, between chunks a recurrence on the P x N state.  Returns
    ``(y, final_state)`` with the layouts of ``ssd_loop``.

    Written per (sequence, head, chunk) with the chunk's own cumulative log-decay
    g_i = a_{c0} + ... + a_{c0+i}:
      within   y_i  = sum_{j<=i} (C_i . B_j) e^{g_i - g_j} x_j      (the decay-masked scores)
      entering y_i += e^{g_i} S C_i                                 (the state that entered)
      state    S    = e^{g_last} S + sum_j e^{g_last - g_j} x_j B_j^T
    ``dtype`` is the arithmetic type (fp64 by default; fp32 shows the rounding of the
    chunked order in single precision).
    """
    cast = lambda v: np.asarray(v, dtype=np.float64).astype(dtype)
    x, a, B, C = cast(x), cast(a), cast(B), cast(C)
    batch, L, heads, P = x.shape
    N = B.shape[-1]
    a = a.reshape(batch, L, heads)
    y = np.zeros((batch, L, heads, P), dtype=dtype)
    final = np.zeros((batch, heads, P, N), dtype=dtype)
    for bi in range(batch):
        for h in range(heads):
            S = np.zeros((P, N), dtype=dtype) if h0 is None else cast(h0)[bi, h].copy()
            for c0 in range(0, L, chunk):
                c1 = min(L, c0 + chunk)
                g = np.cumsum(a[bi, c0:c1, h], dtype=dtype)          # [l]
                xs, bs, cs = x[bi, c0:c1, h], B[bi, c0:c1, h], C[bi, c0:c1, h]
                n = c1 - c0
                scores = cs @ bs.T                                  # [i, j] = C_i . B_j
                mask = np.zeros((n, n), dtype=dtype)
                for i in range(n):
                    mask[i, :i + 1] = np.exp(g[i] - g[:i + 1])
                y[bi, c0:c1, h] = (scores * mask) @ xs + np.exp(g)[:, None] * (cs @ S.T)
                w = np.exp(g[-1] - g)                               # decay to the chunk end
                S = np.exp(g[-1]) * S + (xs * w[:, None]).T @ bs
            final[bi, h] = S
    return y, final


def causal_conv1d(x, weight, bias=None, hist=None, silu=True):
    """Causal depthwise convolution (+ bias, + SiLU) in fp64: returns ``(u, window)``.

    x: [batch, dim, L]; weight: [dim, K]; bias: [dim]; hist: [batch, dim, K-1] (the K-1
    inputs before x, oldest first; zeros if None).  window: the last K-1 inputs, [batch,
    dim, K-1], for a decode step to continue from.
    """
    x = _f64(x)
    batch, dim, L = x.shape
    w = _f64(weight)
    K = w.shape[1]
    w = _f64(weight, (dim, K))
    bias = _f64(bias, (dim,))
    hist = _f64(hist, (batch, dim, K - 1))
    u = np.empty((batch, dim, L))
    win = np.empty((batch, dim, K - 1))
    _load().oracle_causal_conv1d(_ptr(x), _ptr(w), _ptr(bias), _ptr(hist), int(bool(silu)),
                                 _ptr(u), _ptr(win), batch, dim, L, K)
    return u, win


def conv1d_step(window, x, weight, bias=None, silu=True):
    """One decode token of the convolution in fp64: returns ``(u, new_window)``.
    window: [batch, dim, K-1]; x: [batch, dim]; weight: [dim, K]."""
    win = _f64(window).copy()
    batch, dim, km1 = win.shape
    w = _f64(weight, (dim, km1 + 1))
    x = _f64(x, (batch, dim))
    bias = _f64(bias, (dim,))
    u = np.empty((batch, dim))
    _load().oracle_conv1d_step(_ptr(win), _ptr(x), _ptr(w), _ptr(bias), int(bool(silu)), _ptr(u),
                               batch, dim, km1 + 1)
    return u, win


# ----------------------------------------------------------------------------------
# numpy pieces for tiny inputs
# ----------------------------------------------------------------------------------

def affine_scan_loop(a, b, h0=0.0):
    """h_t = a_t * h_{t-1} + b_t, left to right, one step at a time (pure Python)."""
    h = float(h0)
    out = []
    for at, bt in zip(np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)):
        h = at * h + bt
        out.append(h)
    return np.array(out)


def affine_scan_hillis_steele(a, b):
    """Inclusive prefix of the affine maps along the LAST axis in ceil(log2 L) rounds.

    Round k combines every position with the one 2^k to its left through
    (a2, b2) o (a1, b1) = (a2*a1, a2*b1 + b2); positions left of the start take the
    identity map (1, 0).  Returns the b-component, which is h_t for h_{-1} = 0.
    """
    a = np.array(a, dtype=np.float64, copy=True)
    h = np.array(b, dtype=np.float64, copy=True)
    L = a.shape[-1]
    shift = 1
    while shift < L:
        a_left = np.ones_like(a)
        h_left = np.zeros_like(h)
        a_left[..., shift:] = a[..., :-shift]
        h_left[..., shift:] = h[..., :-shift]
        h = a * h_left + h          # uses the old a of this position
        a = a * a_left
        shift *= 2
    return h


def scan_parallel_reference(x, delta, A, B, C, D=None, z=None, delta_bias=None,
                            delta_softplus=False):
    """The selective scan through N-expanded affine pairs and Hillis-Steele rounds.

    Materialises Abar[b,d,t,n] = exp(Delta[b,d,t] A[d,n]) and
    w[b,d,t,n] = Delta[b,d,t] B[b,t,n] x[b,d,t] (Euler gain), scans each (b,d,n) row
    over t, reads out y = sum_n C[b,t,n] h[b,d,t,n], adds D x and applies the SiLU
    gate.  Independent of the C loop; tiny inputs only (memory is O(batch*dim*L*N)).
    """
    x = _f64(x)
    delta = _f64(delta)
    A = _f64(A)
    B = _f64(B)
    C = _f64(C)
    v = delta + (0.0 if delta_bias is None else _f64(delta_bias)[None, :, None])
    if delta_softplus:
        v = np.logaddexp(0.0, v)          # log(e^0 + e^v) = softplus(v)
    abar = np.exp(v[..., None] * A[None, :, None, :])            # [b,d,t,n]
    w = v[..., None] * B[:, None, :, :] * x[..., None]           # [b,d,t,n]
    h = affine_scan_hillis_steele(np.moveaxis(abar, 2, -1), np.moveaxis(w, 2, -1))
    h = np.moveaxis(h, -1, 2)                                     # back to [b,d,t,n]
    y = np.einsum("bdtn,btn->bdt", h, C)
    if D is not None:
        y = y + _f64(D)[None, :, None] * x
    if z is not None:
        zz = _f64(z)
        y = y * (zz / (1.0 + np.exp(-zz)))
    return y, h[:, :, -1, :]


def lti_kernel(abar, bbar, c, length):
    """Taps K_i = sum_n c_n * abar_n**i * bbar_n, i = 0 .. length-1 (diagonal SSM)."""
    abar = np.asarray(abar, dtype=np.float64)
    bbar = np.asarray(bbar, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    return np.array([np.sum(c * abar ** i * bbar) for i in range(length)])


def lti_conv(abar, bbar, c, x):
    """Causal convolution y_t = sum_{i=0..t} K_i x_{t-i}, written as the O(L^2) double sum."""
    x = np.asarray(x, dtype=np.float64)
    K = lti_kernel(abar, bbar, c, len(x))
    y = np.zeros(len(x))
    for t in range(len(x)):
        for i in range(t + 1):
            y[t] += K[i] * x[t - i]
    return y
