"""GPU parity of the scan's backward (ssm_selective_scan_bwd) against the fp64 oracle.

Gradient bar (one reading of the parity tolerance for gradients): the kernel sees the
oracle's exact input values, so per gradient tensor the normwise relative error
max|g_gpu - g_ref| / max|g_ref| must stay within 1e-4; a gradient written in bf16 may
also carry its own output rounding, 2^-8 |g_ref| per element.
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_45_b200 as ssm
from selective_state_space_45_b200 import inputs
from tests.helpers import to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRAD_REL = 1e-4
NAMES = ("dx", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias", "dinitial_state")
ORACLE_NAME = {"dinitial_state": "dh0"}


def assert_grad(gpu, ref, grad_dtype, what):
    g = to64(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    if g.size == 0:
        return
    assert np.all(np.isfinite(g)), what
    scale = max(float(np.max(np.abs(r))), 1e-30)
    err = np.abs(g - r)
    bound = GRAD_REL * scale + (2.0 ** -8 * np.abs(r) if grad_dtype == torch.bfloat16 else 0.0)
    bad = err > bound
    assert not bad.any(), (what, int(bad.sum()), float(err.max()) / scale)


def make_case(batch, dim, L, N, din, dg, seed, with_h0=True, with_dfinal=True):
    inp = inputs.make_scan_inputs(batch, dim, L, N, din, device=DEV, seed=seed)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(seed + 1000)
    inp["dy"] = torch.randn(batch, dim, L, generator=gen, device=DEV).to(dg)
    inp["h0"] = torch.randn(batch, dim, N, generator=gen, device=DEV) if with_h0 else None
    inp["dfinal"] = torch.randn(batch, dim, N, generator=gen, device=DEV) if with_dfinal else None
    return inp


def run_both(inp, softplus=True, use_z=True, use_D=True, use_bias=True):
    z = inp["z"] if use_z else None
    D = inp["D"] if use_D else None
    bias = inp["delta_bias"] if use_bias else None
    g = ssm.selective_scan_bwd(inp["dy"], inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], D=D,
                               z=z, delta_bias=bias, delta_softplus=softplus,
                               initial_state=inp["h0"], dfinal_state=inp["dfinal"])
    torch.cuda.synchronize()
    r = oracle.scan_bwd(inp["dy"], inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], D=D, z=z,
                        delta_bias=bias, delta_softplus=softplus, h0=inp["h0"], dfinal=inp["dfinal"])
    return g, r


def check_all(g, r, dg):
    for name in NAMES:
        if g[name] is None:
            continue
        assert_grad(g[name], r[ORACLE_NAME.get(name, name)], dg, name)


# (batch, dim, L, N, input dtype, gradient dtype): multi-tile, ragged last tiles, partial
# channel groups, N below 16, and the scalar staging path (L not a multiple of 4 / 8)
CASES = [
    (1, 8, 64, 4, torch.float32, torch.float32),
    (2, 40, 100, 16, torch.float32, torch.float32),
    (2, 33, 77, 5, torch.float32, torch.float32),
    (1, 64, 256, 16, torch.bfloat16, torch.float32),
    (2, 48, 136, 16, torch.bfloat16, torch.bfloat16),
    (1, 16, 40, 8, torch.float32, torch.bfloat16),
    (3, 32, 33, 16, torch.bfloat16, torch.float32),
]


@pytest.mark.parametrize("batch,dim,L,N,din,dg", CASES)
def test_bwd_parity(cuda_lib, batch, dim, L, N, din, dg):
    inp = make_case(batch, dim, L, N, din, dg, seed=L + N)
    g, r = run_both(inp)
    check_all(g, r, dg)


@pytest.mark.parametrize("softplus,use_z,use_D,use_bias", [
    (False, True, True, True), (True, False, True, True), (True, True, False, False),
    (False, False, False, False)])
def test_bwd_optional_terms(cuda_lib, softplus, use_z, use_D, use_bias):
    inp = make_case(2, 36, 72, 16, torch.float32, torch.float32, seed=3)
    if not softplus:   # the raw step (plus bias) is then used as given: keep it positive
        inp["delta"] = inp["delta"].abs() * 0.1 + 0.01
        inp["delta_bias"] = torch.full_like(inp["delta_bias"], 0.02)
    g, r = run_both(inp, softplus, use_z, use_D, use_bias)
    check_all(g, r, torch.float32)


def test_bwd_without_start_state_or_final_gradient(cuda_lib):
    inp = make_case(2, 32, 96, 16, torch.bfloat16, torch.float32, seed=4, with_h0=False,
                    with_dfinal=False)
    g, r = run_both(inp)
    check_all(g, r, torch.float32)


def test_bwd_is_deterministic(cuda_lib):
    inp = make_case(2, 64, 200, 16, torch.bfloat16, torch.float32, seed=5)
    g1 = ssm.selective_scan_bwd(inp["dy"], inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                                delta_softplus=True, initial_state=inp["h0"],
                                dfinal_state=inp["dfinal"])
    g2 = ssm.selective_scan_bwd(inp["dy"], inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                                delta_softplus=True, initial_state=inp["h0"],
                                dfinal_state=inp["dfinal"])
    torch.cuda.synchronize()
    for name in NAMES:
        assert torch.equal(g1[name], g2[name]), name


def test_bwd_empty_sequence(cuda_lib):
    inp = make_case(2, 8, 0, 16, torch.float32, torch.float32, seed=6)
    g = ssm.selective_scan_bwd(inp["dy"], inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                               D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                               delta_softplus=True, initial_state=inp["h0"],
                               dfinal_state=inp["dfinal"])
    torch.cuda.synchronize()
    assert torch.count_nonzero(g["dA"]).item() == 0
    assert torch.count_nonzero(g["dD"]).item() == 0
    assert torch.count_nonzero(g["ddelta_bias"]).item() == 0
    assert torch.equal(g["dinitial_state"], inp["dfinal"])


def test_bwd_mamba130m_one_sequence(cuda_lib):
    # full-size run; the oracle checks every per-token gradient of sequence 0 (dB, dC sum over
    # all 1536 channels of it), and a batch-1 run of that sequence for dA, dD, dbias, dh0
    c = inputs.CONFIGS["mamba130m"]
    inp = make_case(c["batch"], c["dim"], c["seqlen"], c["dstate"], c["dtype"], torch.bfloat16, seed=0)
    g = ssm.selective_scan_bwd(inp["dy"], inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                               D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                               delta_softplus=True, initial_state=inp["h0"],
                               dfinal_state=inp["dfinal"])
    one = {k: (v[:1].contiguous() if k in ("x", "delta", "z", "B", "C", "dy", "h0", "dfinal") else v)
           for k, v in inp.items()}
    g1, r = run_both(one)
    for name in ("dx", "ddelta", "dz", "dB", "dC", "dinitial_state"):
        assert_grad(g[name][:1], r[ORACLE_NAME.get(name, name)], torch.bfloat16, name)
    for name in ("dA", "dD", "ddelta_bias", "dinitial_state", "dB"):
        assert_grad(g1[name], r[ORACLE_NAME.get(name, name)], torch.bfloat16, name + " (batch 1)")
