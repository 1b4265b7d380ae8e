"""GPU parity of Mamba-2's chunked SSD (ssm_ssd_fwd) against the fp64 oracle loop.

SSD bar (one reading of the parity tolerance for this operation): the inputs are bf16 and
exact for the oracle, but three intermediate operands enter tensor-core products rounded to
bf16 -- the masked scores, the decay-weighted inputs and the state -- each carrying up to
2^-9 relative error.  Per output tensor: relative L2 error <= 3 * 2^-9 (= 5.9e-3) and
normwise max|y_gpu - y_ref| / max|y_ref| <= 1e-2; the final state (fp32, written from the
fp32 accumulators) likewise.
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
RELL2 = 3 * 2.0 ** -9
NORM_MAX = 1e-2


def assert_ssd_close(gpu, ref, what):
    g = to64(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), what
    rel_l2 = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))
    norm_max = float(np.abs(g - r).max() / max(np.abs(r).max(), 1e-30))
    assert rel_l2 <= RELL2 and norm_max <= NORM_MAX, (what, rel_l2, norm_max)
    return rel_l2, norm_max


CASES = [  # batch, L, heads, headdim, dstate (chunks of 128 tokens)
    (1, 150, 3, 64, 128),     # two chunks, the last ragged
    (2, 256, 4, 64, 64),      # exactly two chunks
    (1, 100, 2, 32, 128),     # one ragged chunk
    (2, 128, 3, 32, 64),      # exactly one chunk
    (1, 7, 2, 64, 128),       # shorter than a chunk
    (2, 421, 2, 64, 128),     # four chunks, more CTAs than one
    (1, 300, 5, 32, 64),
]


@pytest.mark.parametrize("batch,L,heads,P,N", CASES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_ssd_parity(cuda_lib, batch, L, heads, P, N, out_dtype):
    inp = inputs.make_ssd_inputs(batch, L, heads, P, N, device=DEV, seed=L + N)
    y, hN = ssm.ssd(inp["x"], inp["a"], inp["B"], inp["C"], out_dtype=out_dtype)
    torch.cuda.synchronize()
    yr, hr = oracle.ssd_loop(inp["x"], inp["a"], inp["B"], inp["C"])
    assert_ssd_close(y, yr, "y")
    assert_ssd_close(hN, hr, "final state")
    assert cuda_lib.ssm_device_timeouts() == 0


def test_ssd_from_a_start_state_and_resume(cuda_lib):
    inp = inputs.make_ssd_inputs(2, 200, 3, 64, 128, device=DEV, seed=3)
    g = torch.Generator(device=DEV)
    g.manual_seed(4)
    h0 = torch.randn(2, 3, 64, 128, generator=g, device=DEV)
    y, hN = ssm.ssd(inp["x"], inp["a"], inp["B"], inp["C"], initial_state=h0)
    torch.cuda.synchronize()
    yr, hr = oracle.ssd_loop(inp["x"], inp["a"], inp["B"], inp["C"], h0=h0)
    assert_ssd_close(y, yr, "y")
    assert_ssd_close(hN, hr, "final state")
    # two calls chained through the state: the second starts where the first stopped
    part = {k: v[:, :128].contiguous() for k, v in inp.items()}
    rest = {k: v[:, 128:].contiguous() for k, v in inp.items()}
    y1, h1 = ssm.ssd(part["x"], part["a"], part["B"], part["C"], initial_state=h0)
    y2, h2 = ssm.ssd(rest["x"], rest["a"], rest["B"], rest["C"], initial_state=h1)
    torch.cuda.synchronize()
    assert_ssd_close(torch.cat([y1, y2], dim=1), yr, "y (resumed)")
    assert_ssd_close(h2, hr, "final state (resumed)")


@pytest.mark.parametrize("scale", [5.0, 12.0])
def test_ssd_fast_decays(cuda_lib, scale):
    # decays scaled so that a chunk's cumulative log-decay passes -64: the in-chunk decay
    # factors span more than the fp32 range and the carried state all but vanishes between
    # chunks; the first chunk keeps the unscaled decays
    inp = inputs.make_ssd_inputs(2, 300, 2, 64, 128, device=DEV, seed=int(scale))
    a = inp["a"].clone()
    a[:, 128:] *= scale
    y, hN = ssm.ssd(inp["x"], a, inp["B"], inp["C"])
    torch.cuda.synchronize()
    yr, hr = oracle.ssd_loop(inp["x"], a, inp["B"], inp["C"])
    assert_ssd_close(y, yr, "y")
    assert_ssd_close(hN, hr, "final state")
    assert cuda_lib.ssm_device_timeouts() == 0


def test_ssd_empty_sequence_copies_the_state(cuda_lib):
    inp = inputs.make_ssd_inputs(1, 0, 2, 64, 128, device=DEV, seed=5)
    h0 = torch.randn(1, 2, 64, 128, device=DEV)
    y, hN = ssm.ssd(inp["x"], inp["a"], inp["B"], inp["C"], initial_state=h0)
    torch.cuda.synchronize()
    assert y.numel() == 0 and torch.equal(hN, h0)


def test_ssd_is_deterministic_and_causal(cuda_lib):
    inp = inputs.make_ssd_inputs(1, 300, 2, 64, 128, device=DEV, seed=6)
    y1 = ssm.ssd(inp["x"], inp["a"], inp["B"], inp["C"], return_final_state=False)
    y2 = ssm.ssd(inp["x"], inp["a"], inp["B"], inp["C"], return_final_state=False)
    x2 = inp["x"].clone()
    x2[:, 200] += 1.0
    y3 = ssm.ssd(x2, inp["a"], inp["B"], inp["C"], return_final_state=False)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert torch.equal(y3[:, :200], y1[:, :200])
    assert not torch.equal(y3[:, 200], y1[:, 200])


def test_ssd130m_sampled_heads(cuda_lib):
    c = inputs.CONFIGS["ssd130m"]
    inp = inputs.make_ssd_inputs(c["batch"], c["seqlen"], c["heads"], c["headdim"], c["dstate"],
                                 device=DEV, seed=0)
    y, hN = ssm.ssd(inp["x"], inp["a"], inp["B"], inp["C"])
    torch.cuda.synchronize()
    for b, h in [(0, 0), (3, 11), (7, 23)]:
        sl = {k: v[b:b + 1, :, h:h + 1].contiguous() for k, v in inp.items()}
        yr, hr = oracle.ssd_loop(sl["x"], sl["a"], sl["B"], sl["C"])
        assert_ssd_close(y[b:b + 1, :, h:h + 1], yr, "y (b=%d, h=%d)" % (b, h))
        assert_ssd_close(hN[b:b + 1, h:h + 1], hr, "final state (b=%d, h=%d)" % (b, h))
    assert cuda_lib.ssm_device_timeouts() == 0


def test_ssd_more_ctas_than_resident_slots(cuda_lib):
    # 16 x 24 = 384 (sequence, head) CTAs: more than two per SM, so a second wave starts as
    # CTAs of the first finish; sampled heads from both waves against the oracle
    inp = inputs.make_ssd_inputs(16, 300, 24, 64, 128, device=DEV, seed=9)
    y, hN = ssm.ssd(inp["x"], inp["a"], inp["B"], inp["C"])
    torch.cuda.synchronize()
    for b, h in [(0, 0), (6, 5), (12, 17), (15, 23)]:
        sl = {k: v[b:b + 1, :, h:h + 1].contiguous() for k, v in inp.items()}
        yr, hr = oracle.ssd_loop(sl["x"], sl["a"], sl["B"], sl["C"])
        assert_ssd_close(y[b:b + 1, :, h:h + 1], yr, "y (b=%d, h=%d)" % (b, h))
        assert_ssd_close(hN[b:b + 1, h:h + 1], hr, "final state (b=%d, h=%d)" % (b, h))
    assert cuda_lib.ssm_device_timeouts() == 0
