"""GPU parity of the causal depthwise convolution (ssm_causal_conv1d_fwd) and its decode
form (ssm_causal_conv1d_step) against the fp64 oracle.

Tolerance (the convolution's own bar, tighter than the scan's): the kernels see the same
input values as the oracle (bf16 inputs are widened exactly), so the only differences are
the fp32 accumulation of at most 8 products and the fp32 SiLU.  Both are bounded by a
small multiple of 2^-24 times the magnitude sum  m = |bias| + sum_i |w_i| |x_{t-K+1+i}|
(SiLU's slope is at most 1.1):  |gpu - ref| <= 1e-5 m, plus the output's own rounding
(2^-8 |ref| for a bf16 u, on top of twice the fp32 bound).  The magnitude sum is the
oracle's own convolution of |x| with |w| and |bias|, activation off.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_45_b200 import inputs
from tests.helpers import to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
CONV_ACC = 1e-5


def conv_ref(x, w, b, hist, silu):
    u, win = oracle.causal_conv1d(to64(x), to64(w), None if b is None else to64(b),
                                  None if hist is None else to64(hist), silu=silu)
    mag, _ = oracle.causal_conv1d(np.abs(to64(x)), np.abs(to64(w)),
                                  None if b is None else np.abs(to64(b)),
                                  None if hist is None else np.abs(to64(hist)), silu=False)
    return u, win, mag


def assert_conv_close(gpu, ref, mag, out_dtype, what="u"):
    g = to64(gpu)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    if g.size == 0:
        return
    assert np.all(np.isfinite(g)), what
    err = np.abs(g - ref)
    if out_dtype == torch.bfloat16:
        bound = 2 * CONV_ACC * mag + 2.0 ** -8 * np.abs(ref)
    else:
        bound = CONV_ACC * mag
    bad = err > bound
    assert not bad.any(), (what, int(bad.sum()), float(err.max()), float((err / (mag + 1e-30)).max()))


def run_conv(ssm, inp, silu=True, dout=None, use_bias=True, use_window=True, want_window=True):
    x = inp["x"]
    batch, dim, L = x.shape
    K = inp["weight"].shape[1]
    u = torch.empty(batch, dim, L, device=DEV, dtype=dout or x.dtype)
    fw = torch.full((batch, dim, K - 1), float("nan"), device=DEV) if want_window else None
    ssm.ssm_causal_conv1d_fwd(x, inp["weight"], inp["bias"] if use_bias else None,
                              inp.get("window") if use_window else None, u, fw, silu)
    torch.cuda.synchronize()
    return u, fw


# (batch, dim, L, width, in dtype, out dtype): widths 1-4 with L a multiple of the 16-byte
# vector take the vector kernel; the rest (ragged L, widths 5-8) the per-element kernel.
# L = 200 (bf16) or 100 (fp32) makes 13 chunks per row, so rows start at every lane.
CASES = [
    (2, 8, 64, 4, torch.float32, torch.float32),
    (2, 8, 64, 4, torch.bfloat16, torch.bfloat16),
    (3, 5, 200, 4, torch.bfloat16, torch.float32),
    (3, 5, 100, 4, torch.float32, torch.bfloat16),
    (1, 7, 8, 4, torch.bfloat16, torch.bfloat16),      # one half chunk per row
    (1, 7, 24, 3, torch.bfloat16, torch.bfloat16),     # a full chunk and a half one
    (2, 6, 48, 2, torch.float32, torch.float32),
    (2, 6, 40, 1, torch.bfloat16, torch.bfloat16),
    (2, 9, 37, 4, torch.bfloat16, torch.bfloat16),     # ragged: general kernel
    (2, 9, 37, 4, torch.float32, torch.float32),
    (1, 4, 1000, 4, torch.float32, torch.float32),
    (2, 3, 64, 5, torch.bfloat16, torch.bfloat16),     # width above 4: general kernel
    (2, 3, 29, 8, torch.float32, torch.bfloat16),
    (4, 96, 2048, 4, torch.bfloat16, torch.bfloat16),  # rows of 128 chunks: 4 warps each
]


@pytest.mark.parametrize("batch,dim,L,K,din,dout", CASES)
@pytest.mark.parametrize("window", [False, True])
def test_conv_parity(cuda_lib, batch, dim, L, K, din, dout, window):
    inp = inputs.make_conv_inputs(batch, dim, L, K, din, device=DEV, seed=L + K,
                                  with_window=window)
    u, fw = run_conv(cuda_lib, inp, dout=dout)
    ur, winr, mag = conv_ref(inp["x"], inp["weight"], inp["bias"], inp.get("window"), True)
    assert_conv_close(u, ur, mag, dout)
    # the final window holds input values, widened exactly: bit-exact
    assert np.array_equal(to64(fw), winr)


@pytest.mark.parametrize("silu,use_bias", [(False, True), (True, False), (False, False)])
@pytest.mark.parametrize("L", [64, 61])
def test_conv_optional_terms(cuda_lib, silu, use_bias, L):
    inp = inputs.make_conv_inputs(2, 12, L, 4, torch.float32, device=DEV, seed=5)
    u, _ = run_conv(cuda_lib, inp, silu=silu, use_bias=use_bias, want_window=False)
    ur, _, mag = conv_ref(inp["x"], inp["weight"], inp["bias"] if use_bias else None, None, silu)
    assert_conv_close(u, ur, mag, torch.float32)


@pytest.mark.parametrize("L", [1, 2, 3])
@pytest.mark.parametrize("din", [torch.float32, torch.bfloat16])
def test_conv_shorter_than_window(cuda_lib, L, din):
    # the final window mixes the carried window and the few new inputs
    inp = inputs.make_conv_inputs(2, 5, L, 4, din, device=DEV, seed=L, with_window=True)
    u, fw = run_conv(cuda_lib, inp)
    ur, winr, mag = conv_ref(inp["x"], inp["weight"], inp["bias"], inp["window"], True)
    assert_conv_close(u, ur, mag, din)
    assert np.array_equal(to64(fw), winr)


def test_conv_empty_sequences(cuda_lib):
    inp = inputs.make_conv_inputs(2, 5, 0, 4, torch.bfloat16, device=DEV, seed=1, with_window=True)
    u, fw = run_conv(cuda_lib, inp)
    assert u.shape == (2, 5, 0)
    assert torch.equal(fw, inp["window"])
    _, fw0 = run_conv(cuda_lib, inp, use_window=False)
    assert torch.count_nonzero(fw0).item() == 0
    # no rows: nothing to do, nothing written
    inp0 = inputs.make_conv_inputs(0, 5, 16, 4, torch.bfloat16, device=DEV, seed=1)
    u0, _ = run_conv(cuda_lib, inp0)
    assert u0.numel() == 0


@pytest.mark.parametrize("split", [8, 16, 40, 64, 120])
def test_conv_resume_is_bitwise(cuda_lib, split):
    # the same products in the same order: a split run reproduces the whole one exactly
    inp = inputs.make_conv_inputs(3, 10, 128, 4, torch.bfloat16, device=DEV, seed=2)
    u, fw = run_conv(cuda_lib, inp)
    a = dict(inp, x=inp["x"][..., :split].contiguous())
    u1, w1 = run_conv(cuda_lib, a)
    b = dict(inp, x=inp["x"][..., split:].contiguous(), window=w1)
    u2, w2 = run_conv(cuda_lib, b)
    assert torch.equal(torch.cat([u1, u2], dim=-1), u)
    assert torch.equal(w2, fw)


def test_conv_is_causal_and_deterministic(cuda_lib):
    inp = inputs.make_conv_inputs(2, 16, 256, 4, torch.bfloat16, device=DEV, seed=3)
    u, _ = run_conv(cuda_lib, inp)
    u_again, _ = run_conv(cuda_lib, inp)
    assert torch.equal(u, u_again)
    t0 = 100
    x2 = inp["x"].clone()
    x2[:, 3, t0] += 2.0
    u2, _ = run_conv(cuda_lib, dict(inp, x=x2))
    assert torch.equal(u2[..., :t0], u[..., :t0])
    assert torch.equal(u2[:, [0, 1, 2] + list(range(4, 16))], u[:, [0, 1, 2] + list(range(4, 16))])
    assert torch.equal(u2[:, 3, t0 + 4:], u[:, 3, t0 + 4:])
    assert not torch.equal(u2[:, 3, t0:t0 + 4], u[:, 3, t0:t0 + 4])


# ------------------------------------------------------------------------------------
# decode form
# ------------------------------------------------------------------------------------

def chain_steps(ssm, inp, dout, silu=True):
    window = inp["window"].clone()
    steps = inp["x"].shape[0]
    us = []
    for t in range(steps):
        u = torch.empty(inp["x"].shape[1:], device=DEV, dtype=dout)
        # a fresh copy: every pointer the library takes is 16-byte aligned, and the slice
        # x[t] starts at t * batch * dim elements
        ssm.ssm_causal_conv1d_step(window, inp["x"][t].clone(), inp["weight"], inp["bias"], u, silu)
        us.append(u)
    torch.cuda.synchronize()
    return torch.stack(us, dim=-1), window


@pytest.mark.parametrize("batch,dim,K,din,dout", [
    (3, 40, 4, torch.bfloat16, torch.bfloat16),
    (2, 33, 4, torch.float32, torch.float32),
    (2, 17, 2, torch.bfloat16, torch.float32),
    (1, 9, 8, torch.float32, torch.bfloat16),
    (2, 5, 1, torch.float32, torch.float32),
])
def test_conv_step_chain_matches_oracle_and_fwd(cuda_lib, batch, dim, K, din, dout):
    steps = 12
    inp = inputs.make_conv_step_inputs(batch, dim, steps, K, din, device=DEV, seed=dim + K)
    us, window = chain_steps(cuda_lib, inp, dout)
    xs = inp["x"].permute(1, 2, 0).contiguous()            # [batch, dim, steps]
    ur, winr, mag = conv_ref(xs, inp["weight"], inp["bias"], inp["window"], True)
    assert_conv_close(us, ur, mag, dout)
    assert np.array_equal(to64(window), winr)
    # and bit for bit what the whole-sequence kernel gives from the same window
    u_fwd = torch.empty(batch, dim, steps, device=DEV, dtype=dout)
    fw = torch.empty(batch, dim, K - 1, device=DEV)
    cuda_lib.ssm_causal_conv1d_fwd(xs, inp["weight"], inp["bias"], inp["window"], u_fwd, fw, True)
    torch.cuda.synchronize()
    assert torch.equal(u_fwd, us)
    assert torch.equal(fw, window)


def test_conv_step_single_against_oracle(cuda_lib):
    inp = inputs.make_conv_step_inputs(256, 512, 1, 4, torch.bfloat16, device=DEV, seed=9)
    us, window = chain_steps(cuda_lib, inp, torch.bfloat16)
    ur, wr = oracle.conv1d_step(to64(inp["window"]), to64(inp["x"][0]), to64(inp["weight"]),
                                to64(inp["bias"]))
    _, _, mag = conv_ref(inp["x"][0][..., None], inp["weight"], inp["bias"], inp["window"], False)
    assert_conv_close(us[..., 0], ur, mag[..., 0], torch.bfloat16)
    assert np.array_equal(to64(window), wr)


# ------------------------------------------------------------------------------------
# the Mamba block shapes
# ------------------------------------------------------------------------------------

def test_conv_mamba130m_full(cuda_lib):
    inp = inputs.make_conv_inputs(8, 1536, 2048, 4, torch.bfloat16, device=DEV, seed=0)
    u, fw = run_conv(cuda_lib, inp)
    ur, winr, mag = conv_ref(inp["x"], inp["weight"], inp["bias"], None, True)
    assert_conv_close(u, ur, mag, torch.bfloat16)
    assert np.array_equal(to64(fw), winr)


def test_conv_mamba2p8b_sampled_rows(cuda_lib):
    inp = inputs.make_conv_inputs(4, 5120, 4096, 4, torch.bfloat16, device=DEV, seed=0)
    u, fw = run_conv(cuda_lib, inp)
    dsel = torch.tensor([0, 1, 31, 32, 1000, 2047, 2048, 4095, 5087, 5119], device=DEV)
    xs = inp["x"].index_select(1, dsel)
    ur, winr, mag = conv_ref(xs, inp["weight"].index_select(0, dsel),
                             inp["bias"].index_select(0, dsel), None, True)
    assert_conv_close(u.index_select(1, dsel), ur, mag, torch.bfloat16)
    assert np.array_equal(to64(fw.index_select(1, dsel)), winr)
