"""Seeded synthetic inputs for the selective scan, the decode step and the causal
convolution in front of the scan.

This module only draws random numbers in the shapes and distributions of the
workloads; it computes nothing of the scan itself, so the CUDA path and the fp64
oracle can both be fed from it.

Workloads (sizes follow the Mamba shapes the pages use: mamba-130m has
d_inner = 1536 and N = 16, xmarva lesson 10 section 4; the 2.8b shape has
d_inner = 5120; the million-token length follows the long-context claims in
learnllm "Module 19" and askaiml section 4):

=============  ======  =========  =======  ===  =====================================
name           batch   L          d_inner  N    dtype of x, delta, z, B, C
=============  ======  =========  =======  ===  =====================================
tiny           1       64         8        4    fp32
mamba130m      8       2048       1536     16   bf16 (A, D, bias, state fp32)
mamba2p8b      4       4096       5120     16   bf16
long1m         1       1048576    1536     16   bf16
long1m_slow    1       1048576    1536     16   bf16, A[d, n] = -exp(U[-5, 0]): slow decays
decode         256     1 x 64     5120     16   bf16 tokens, fp32 state
decode4        256     4 x 16     5120     16   as decode, 4 tokens per call
bwd130m        8       2048       1536     16   bf16 inputs, dy and gradients (backward)
ssd130m        8       2048       24 x 64  128  Mamba-2 SSD: bf16 x, B, C; fp32 a
conv130m       8       2048       1536     --   bf16 x and u; width 4, fp32 taps/bias
conv2p8b       4       4096       5120     --   bf16 x and u; width 4
convstep       256     1 x 64     5120     --   bf16 tokens, fp32 window (width 4)
=============  ======  =========  =======  ===  =====================================

Draw order (one generator seeded once): x, delta_raw, z, B, C, D, dt.
  x, z ~ N(0, 1);  delta_raw = 0.5 * N(0, 1);  B, C ~ N(0, 1) per (b, t, n);
  D ~ N(0, 1);  dt ~ U[1e-3, 1e-1] per channel (log-uniform on that range for the
  2.8b shape);  delta_bias = log(expm1(dt)), evaluated in fp64 and stored fp32, so
  that softplus(delta_bias) = dt;  A[d, n] = -(n + 1), or for long1m_slow
  A[d, n] = -exp(U[-5, 0]) drawn last (|A| between 0.0067 and 1: states that remember
  for up to ~10^5 tokens, the hardest case for cutting a sequence into segments).
The decode workload draws an N(0, 1) fp32 state and, per token, a positive step
delta = dt * exp(0.5 * N(0, 1)) (the step is an input of the decode call, already
positive), with x, z, B, C as above.
"""
from __future__ import annotations

import math

import torch

CONFIGS = {
    "tiny": dict(batch=1, seqlen=64, dim=8, dstate=4, dtype=torch.float32, dt_dist="uniform"),
    "mamba130m": dict(batch=8, seqlen=2048, dim=1536, dstate=16, dtype=torch.bfloat16,
                      dt_dist="uniform"),
    "mamba2p8b": dict(batch=4, seqlen=4096, dim=5120, dstate=16, dtype=torch.bfloat16,
                      dt_dist="loguniform"),
    # the 2.8b shape with d_inner set so that the grid of 32-channel CTAs fills the 148 SMs
    # evenly: 592 CTAs (4 per SM) and 740 CTAs (5 per SM); the 2.8b shape's own 640 CTAs
    # leave 48 SMs with a fifth CTA
    "mamba2p8b_d4736": dict(batch=4, seqlen=4096, dim=4736, dstate=16, dtype=torch.bfloat16,
                            dt_dist="loguniform"),
    "mamba2p8b_d5920": dict(batch=4, seqlen=4096, dim=5920, dstate=16, dtype=torch.bfloat16,
                            dt_dist="loguniform"),
    "long1m": dict(batch=1, seqlen=1 << 20, dim=1536, dstate=16, dtype=torch.bfloat16,
                   dt_dist="uniform"),
    "long1m_slow": dict(batch=1, seqlen=1 << 20, dim=1536, dstate=16, dtype=torch.bfloat16,
                        dt_dist="uniform", a_dist="slow"),
    "decode": dict(batch=256, steps=64, dim=5120, dstate=16, dtype=torch.bfloat16,
                   dt_dist="uniform"),
    # the decode workload with 4 tokens per call on the carried state (speculative decoding)
    "decode4": dict(batch=256, steps=64, dim=5120, dstate=16, dtype=torch.bfloat16,
                    dt_dist="uniform", ntok=4),
    # the backward of the mamba130m-shaped scan (training), bf16 inputs and gradients
    "bwd130m": dict(batch=8, seqlen=2048, dim=1536, dstate=16, dtype=torch.bfloat16,
                    dt_dist="uniform"),
    # Mamba-2's SSD in the 130m shape: 24 heads of 64 channels, state 128
    "ssd130m": dict(batch=8, seqlen=2048, heads=24, headdim=64, dstate=128, dtype=torch.bfloat16),
    # the causal convolution in front of the scan, in the same block shapes (width 4)
    "conv130m": dict(batch=8, seqlen=2048, dim=1536, width=4, dtype=torch.bfloat16),
    "conv2p8b": dict(batch=4, seqlen=4096, dim=5120, width=4, dtype=torch.bfloat16),
    "convstep": dict(batch=256, steps=64, dim=5120, width=4, dtype=torch.bfloat16),
}

DT_MIN, DT_MAX = 1e-3, 1e-1


def _generator(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _draw_dt(n, dist, g, device):
    u = torch.rand(n, generator=g, device=device, dtype=torch.float64)
    if dist == "uniform":
        return DT_MIN + (DT_MAX - DT_MIN) * u
    if dist == "loguniform":
        return torch.exp(math.log(DT_MIN) + (math.log(DT_MAX) - math.log(DT_MIN)) * u)
    raise ValueError("unknown dt distribution %r" % (dist,))


def make_scan_inputs(batch, dim, seqlen, dstate, dtype=torch.float32, device="cpu", seed=0,
                     dt_dist="uniform", a_dist="index"):
    """Inputs of one selective-scan call, as a dict of tensors on ``device``.

    Keys: x, delta, z ([batch, dim, seqlen], ``dtype``); B, C ([batch, seqlen, dstate],
    ``dtype``); A ([dim, dstate] fp32); D, delta_bias ([dim] fp32).  ``delta`` is the raw
    step: the scan adds ``delta_bias`` and applies softplus.
    """
    g = _generator(device, seed)
    f32 = torch.float32

    def normal(*shape, scale=1.0):
        t = torch.randn(*shape, generator=g, device=device, dtype=f32)
        if scale != 1.0:
            t.mul_(scale)
        return t.to(dtype)

    x = normal(batch, dim, seqlen)
    delta = normal(batch, dim, seqlen, scale=0.5)
    z = normal(batch, dim, seqlen)
    B = normal(batch, seqlen, dstate)
    C = normal(batch, seqlen, dstate)
    D = torch.randn(dim, generator=g, device=device, dtype=f32)
    dt = _draw_dt(dim, dt_dist, g, device)
    delta_bias = torch.log(torch.expm1(dt)).to(f32)
    if a_dist == "index":
        A = -torch.arange(1, dstate + 1, device=device, dtype=f32).repeat(dim, 1).contiguous()
    elif a_dist == "slow":
        u = torch.rand(dim, dstate, generator=g, device=device, dtype=f32)
        A = -torch.exp(-5.0 * u)
    else:
        raise ValueError("unknown A distribution %r" % (a_dist,))
    return dict(x=x, delta=delta, z=z, B=B, C=C, A=A, D=D, delta_bias=delta_bias)


def make_scan_bwd_inputs(batch, dim, seqlen, dstate, dtype=torch.bfloat16, device="cpu", seed=0,
                         dt_dist="uniform"):
    """Inputs of one backward call: those of ``make_scan_inputs`` (same seed) plus the
    output gradient dy ([batch, dim, seqlen], ``dtype``, N(0, 1)) from a second generator
    seeded seed + 1."""
    inp = make_scan_inputs(batch, dim, seqlen, dstate, dtype, device=device, seed=seed,
                           dt_dist=dt_dist)
    g = _generator(device, seed + 1)
    inp["dy"] = torch.randn(batch, dim, seqlen, generator=g, device=device,
                            dtype=torch.float32).to(dtype)
    return inp


def make_ssd_inputs(batch, seqlen, heads, headdim, dstate, dtype=torch.bfloat16, device="cpu",
                    seed=0):
    """Inputs of one SSD call, following the worked example of the Mamba-2 section: x, B, C
    ~ N(0, 1) in ``dtype`` (x [batch, L, heads, P], B, C [batch, L, heads, N]) and the
    per-head log-decay a = -U[0, 0.3) fp32 [batch, L, heads].  Draw order: x, a, B, C."""
    g = _generator(device, seed)
    f32 = torch.float32
    x = torch.randn(batch, seqlen, heads, headdim, generator=g, device=device, dtype=f32).to(dtype)
    a = -0.3 * torch.rand(batch, seqlen, heads, generator=g, device=device, dtype=f32)
    B = torch.randn(batch, seqlen, heads, dstate, generator=g, device=device, dtype=f32).to(dtype)
    C = torch.randn(batch, seqlen, heads, dstate, generator=g, device=device, dtype=f32).to(dtype)
    return dict(x=x, a=a, B=B, C=C)


def make_config_inputs(name, device="cpu", seed=0):
    c = CONFIGS[name]
    if name.startswith("ssd"):
        return make_ssd_inputs(c["batch"], c["seqlen"], c["heads"], c["headdim"], c["dstate"],
                               c["dtype"], device=device, seed=seed)
    if name == "convstep":
        return make_conv_step_inputs(c["batch"], c["dim"], c["steps"], c["width"], c["dtype"],
                                     device=device, seed=seed)
    if name.startswith("bwd"):
        return make_scan_bwd_inputs(c["batch"], c["dim"], c["seqlen"], c["dstate"], c["dtype"],
                                    device=device, seed=seed, dt_dist=c["dt_dist"])
    if name.startswith("conv"):
        return make_conv_inputs(c["batch"], c["dim"], c["seqlen"], c["width"], c["dtype"],
                                device=device, seed=seed)
    if name in ("decode", "decode4"):
        return make_decode_inputs(c["batch"], c["dim"], c["dstate"], c["steps"], c["dtype"],
                                  device=device, seed=seed)
    return make_scan_inputs(c["batch"], c["dim"], c["seqlen"], c["dstate"], c["dtype"],
                            device=device, seed=seed, dt_dist=c["dt_dist"],
                            a_dist=c.get("a_dist", "index"))


def make_decode_inputs(batch, dim, dstate, steps, dtype=torch.bfloat16, device="cpu", seed=0,
                       dt_dist="uniform"):
    """Inputs of ``steps`` chained decode calls.

    Keys: state ([batch, dim, dstate] fp32, N(0,1)); x, delta, z ([steps, batch, dim],
    ``dtype``; delta positive); B, C ([steps, batch, dstate], ``dtype``); A ([dim, dstate]
    fp32); D ([dim] fp32).
    """
    g = _generator(device, seed)
    f32 = torch.float32
    state = torch.randn(batch, dim, dstate, generator=g, device=device, dtype=f32)
    x = torch.randn(steps, batch, dim, generator=g, device=device, dtype=f32).to(dtype)
    noise = torch.randn(steps, batch, dim, generator=g, device=device, dtype=f32)
    z = torch.randn(steps, batch, dim, generator=g, device=device, dtype=f32).to(dtype)
    B = torch.randn(steps, batch, dstate, generator=g, device=device, dtype=f32).to(dtype)
    C = torch.randn(steps, batch, dstate, generator=g, device=device, dtype=f32).to(dtype)
    D = torch.randn(dim, generator=g, device=device, dtype=f32)
    dt = _draw_dt(dim, dt_dist, g, device).to(f32)
    delta = (dt[None, None, :] * torch.exp(0.5 * noise)).to(dtype)
    A = -torch.arange(1, dstate + 1, device=device, dtype=f32).repeat(dim, 1).contiguous()
    return dict(state=state, x=x, delta=delta, z=z, B=B, C=C, A=A, D=D)


def make_conv_inputs(batch, dim, seqlen, width=4, dtype=torch.bfloat16, device="cpu", seed=0,
                     with_window=False):
    """Inputs of one causal-convolution call (the filter in front of the scan).

    Keys: x ([batch, dim, seqlen], ``dtype``, N(0, 1)); weight ([dim, width] fp32) and bias
    ([dim] fp32), both U(-1/sqrt(width), 1/sqrt(width)) -- the default initialisation of a
    depthwise Conv1d, whose fan-in is the width; window ([batch, dim, width-1] fp32,
    N(0, 1), the inputs before position 0) when ``with_window``.
    Draw order: x, weight, bias, window.
    """
    g = _generator(device, seed)
    f32 = torch.float32
    bound = 1.0 / math.sqrt(width)
    x = torch.randn(batch, dim, seqlen, generator=g, device=device, dtype=f32).to(dtype)
    weight = (torch.rand(dim, width, generator=g, device=device, dtype=f32) * 2 - 1) * bound
    bias = (torch.rand(dim, generator=g, device=device, dtype=f32) * 2 - 1) * bound
    out = dict(x=x, weight=weight.contiguous(), bias=bias)
    if with_window:
        out["window"] = torch.randn(batch, dim, width - 1, generator=g, device=device, dtype=f32)
    return out


def make_conv_step_inputs(batch, dim, steps, width=4, dtype=torch.bfloat16, device="cpu", seed=0):
    """Inputs of ``steps`` chained convolution decode calls: window ([batch, dim, width-1]
    fp32, N(0, 1)); x ([steps, batch, dim], ``dtype``, N(0, 1)); weight, bias as in
    ``make_conv_inputs``.  Draw order: window, x, weight, bias."""
    g = _generator(device, seed)
    f32 = torch.float32
    bound = 1.0 / math.sqrt(width)
    window = torch.randn(batch, dim, width - 1, generator=g, device=device, dtype=f32)
    x = torch.randn(steps, batch, dim, generator=g, device=device, dtype=f32).to(dtype)
    weight = (torch.rand(dim, width, generator=g, device=device, dtype=f32) * 2 - 1) * bound
    bias = (torch.rand(dim, generator=g, device=device, dtype=f32) * 2 - 1) * bound
    return dict(window=window, x=x, weight=weight.contiguous(), bias=bias)
