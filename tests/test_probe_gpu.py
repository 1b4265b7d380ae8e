"""The SFU probe (ssm_sfu_probe), a diagnostic beside the path: bench.py times it to report
the ex2 rate that the scan's roofline counts against.  Each thread runs 8 chains
v <- 2^(-v); the map is a contraction (slope -ln 2 * 2^(-v), about -0.44 at its fixed
point), so from any start in [0.5, 1] every chain settles on the fixed point
v* = 2^(-v*) = 0.64118574...  Its output is each thread's sum of the 8 chains."""
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda"


def fixed_point():
    v = 0.5
    for _ in range(200):
        v = 2.0 ** (-v)
    return v


def test_probe_chains_reach_the_fixed_point(cuda_lib):
    out = torch.full((3 * 256,), float("nan"), device=DEV)
    cuda_lib.ssm_sfu_probe(out, 3, 200)
    torch.cuda.synchronize()
    want = torch.full_like(out, 8 * fixed_point(), dtype=torch.float64)
    assert torch.allclose(out.double(), want, rtol=1e-5, atol=0.0)


def test_probe_with_no_steps_returns_the_starts(cuda_lib):
    out = torch.full((2 * 256,), float("nan"), device=DEV)
    cuda_lib.ssm_sfu_probe(out, 2, 0)
    torch.cuda.synchronize()
    starts = sum(0.5 + 0.0625 * k for k in range(8))
    assert torch.all(out.double() == starts)


def test_probe_rejects_a_short_buffer(cuda_lib):
    out = torch.empty(100, device=DEV)
    with pytest.raises(ValueError):
        cuda_lib.ssm_sfu_probe(out, 1, 1)
