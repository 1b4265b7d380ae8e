"""GPU parity of ssm_selective_scan_fwd against the fp64 oracle (called through the C ABI)."""

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_45_b200 import inputs
from tests.helpers import assert_parity, oracle_inputs_for, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(params=[None, 3], ids=["oneCTA", "segments3"])
def split(request, force_segments):
    """Both scan paths: one CTA per channel group over the whole sequence, and the
    sequence cut into (up to) 3 segments -- the tail sums of the earlier segments, their
    fold into every segment's carry, and one scan per segment from its carry."""
    force_segments(request.param)
    yield request.param


def run_gpu(ssm, inp, out_dtype, use_z=True, use_D=True, use_bias=True, softplus=True):
    x = inp["x"]
    y = torch.empty(x.shape, device=DEV, dtype=out_dtype)
    fs = torch.empty(x.shape[0], x.shape[1], inp["A"].shape[1], device=DEV, dtype=torch.float32)
    ssm.ssm_selective_scan_fwd(x, inp["delta"], inp["delta_bias"] if use_bias else None, softplus,
                               inp["A"], inp["B"], inp["C"], inp["D"] if use_D else None,
                               inp["z"] if use_z else None, y, fs)
    torch.cuda.synchronize()
    return y, fs


def run_oracle(inp, use_z=True, use_D=True, use_bias=True, softplus=True):
    return oracle.scan(x=inp["x"], delta=inp["delta"], A=inp["A"], B=inp["B"], C=inp["C"],
                       D=inp["D"] if use_D else None, z=inp["z"] if use_z else None,
                       delta_bias=inp["delta_bias"] if use_bias else None,
                       delta_softplus=softplus)


def test_tiny_config_full(cuda_lib, split):
    inp = inputs.make_config_inputs("tiny", device=DEV)
    y, fs = run_gpu(cuda_lib, inp, torch.float32)
    yr, fr = run_oracle(inp)
    assert_parity(y, yr, torch.float32, what="y")
    assert_parity(fs, fr, torch.float32, what="final_state")


CASES = [
    # batch, dim, L, N, in dtype, out dtype
    (2, 37, 1000, 16, torch.bfloat16, torch.bfloat16),   # several tiles, ragged dim
    (2, 19, 997, 16, torch.bfloat16, torch.bfloat16),    # ragged L: scalar staging path
    (1, 40, 256, 16, torch.bfloat16, torch.float32),
    (3, 21, 331, 5, torch.float32, torch.float32),       # odd N, ragged L
    (2, 33, 128, 8, torch.float32, torch.float32),
    (2, 70, 96, 4, torch.float32, torch.bfloat16),
    (1, 9, 77, 1, torch.float32, torch.float32),
    (2, 16, 520, 12, torch.bfloat16, torch.float32),
    (1, 3, 1, 16, torch.float32, torch.float32),         # a single token
    (4, 5, 33, 3, torch.bfloat16, torch.bfloat16),
]


@pytest.mark.parametrize("batch,dim,L,N,din,dout", CASES)
def test_ragged_multi_tile_parity(cuda_lib, split, batch, dim, L, N, din, dout):
    inp = inputs.make_scan_inputs(batch, dim, L, N, din, device=DEV, seed=batch * 1000 + L + N)
    y, fs = run_gpu(cuda_lib, inp, dout)
    yr, fr = run_oracle(inp)
    assert_parity(y, yr, din, dout, what="y")
    assert_parity(fs, fr, din, torch.float32, what="final_state")


@pytest.mark.parametrize("use_z,use_D,use_bias,softplus", [
    (False, True, True, True), (True, False, True, True), (True, True, False, True),
    (True, True, True, False), (False, False, False, False),
])
def test_optional_terms(cuda_lib, split, use_z, use_D, use_bias, softplus):
    inp = inputs.make_scan_inputs(2, 24, 200, 16, torch.float32, device=DEV, seed=5)
    if not softplus:   # a raw step must stay positive without the softplus
        inp["delta"] = inp["delta"].abs() * 0.1 + 1e-3
        inp["delta_bias"] = inp["delta_bias"].abs() * 0.0 + 1e-3
    kw = dict(use_z=use_z, use_D=use_D, use_bias=use_bias, softplus=softplus)
    y, fs = run_gpu(cuda_lib, inp, torch.float32, **kw)
    yr, fr = run_oracle(inp, **kw)
    assert_parity(y, yr, torch.float32, what="y")
    assert_parity(fs, fr, torch.float32, what="final_state")


def test_printed_toy_recurrence_through_gpu(cuda_lib):
    # Abar = 0.8, Bbar = 0.2, x = 5, 0, 0, 10 -> 1, 0.8, 0.64, 2.512 (understandingdata toy)
    L = 4
    delta = torch.full((1, 1, L), -float(np.log(0.8)), device=DEV)
    x = torch.tensor([5.0, 0.0, 0.0, 10.0], device=DEV).reshape(1, 1, L)
    A = torch.full((1, 1), -1.0, device=DEV)
    B = (0.2 / delta[0, 0]).reshape(1, L, 1).contiguous()
    C = torch.ones(1, L, 1, device=DEV)
    y, fs = cuda_lib.selective_scan(x, delta, A, B, C)
    torch.cuda.synchronize()
    np.testing.assert_allclose(to64(y)[0, 0], [1.0, 0.8, 0.64, 2.512], rtol=2e-6)
    assert abs(to64(fs)[0, 0, 0] - 2.512) < 1e-5


def test_impulse_response_through_gpu(cuda_lib, split):
    L = 5
    delta = torch.full((1, 1, L), float(np.log(2.0)), device=DEV)
    x = torch.tensor([1.0, 0, 0, 0, 0], device=DEV).reshape(1, 1, L)
    A = torch.full((1, 1), -1.0, device=DEV)
    B = (1.0 / delta[0, 0]).reshape(1, L, 1).contiguous()
    C = torch.ones(1, L, 1, device=DEV)
    y, _ = cuda_lib.selective_scan(x, delta, A, B, C)
    torch.cuda.synchronize()
    np.testing.assert_allclose(to64(y)[0, 0], [1.0, 0.5, 0.25, 0.125, 0.0625], rtol=2e-6)


def test_causality_bit_identical_before_edit(cuda_lib, split):
    inp = inputs.make_scan_inputs(2, 48, 300, 16, torch.bfloat16, device=DEV, seed=9)
    y1, _ = run_gpu(cuda_lib, inp, torch.bfloat16)
    t0 = 171
    ed = {k: v.clone() for k, v in inp.items()}
    ed["x"][..., t0] += 4.0
    ed["delta"][..., t0] -= 1.0
    ed["z"][..., t0] += 2.0
    ed["B"][:, t0, :] *= -3.0
    ed["C"][:, t0, :] += 1.0
    y2, _ = run_gpu(cuda_lib, ed, torch.bfloat16)
    assert torch.equal(y1[..., :t0], y2[..., :t0])
    assert not torch.equal(y1[..., t0], y2[..., t0])


def test_deterministic_repeat(cuda_lib):
    inp = inputs.make_scan_inputs(2, 64, 512, 16, torch.bfloat16, device=DEV, seed=3)
    y1, f1 = run_gpu(cuda_lib, inp, torch.bfloat16)
    y2, f2 = run_gpu(cuda_lib, inp, torch.bfloat16)
    assert torch.equal(y1, y2) and torch.equal(f1, f2)


def test_empty_and_degenerate_sizes(cuda_lib):
    # L = 0: y is empty and the final state is the zero start state
    x = torch.empty(2, 3, 0, device=DEV)
    A = -torch.ones(3, 16, device=DEV)
    Bm = torch.empty(2, 0, 16, device=DEV)
    y = torch.empty(2, 3, 0, device=DEV)
    fs = torch.full((2, 3, 16), 7.0, device=DEV)
    cuda_lib.ssm_selective_scan_fwd(x, x, None, True, A, Bm, Bm, None, None, y, fs)
    torch.cuda.synchronize()
    assert torch.count_nonzero(fs).item() == 0
    # batch = 0: nothing launched, nothing written
    x0 = torch.empty(0, 3, 8, device=DEV)
    B0 = torch.empty(0, 8, 16, device=DEV)
    cuda_lib.ssm_selective_scan_fwd(x0, x0, None, True, A, B0, B0, None, None, x0.clone(), None)
    torch.cuda.synchronize()


def _misaligned(shape):
    """A contiguous fp32 view whose data pointer is 4 bytes past a 16-byte boundary."""
    n = int(np.prod(shape))
    base = torch.empty(n + 4, device=DEV)
    v = base[1:1 + n].view(*shape)
    assert v.data_ptr() % 16 == 4
    return v


def test_misaligned_pointer_rejected_on_device(cuda_lib):
    inp = inputs.make_scan_inputs(1, 4, 64, 16, torch.float32, device=DEV)
    y = _misaligned((1, 4, 64))
    with pytest.raises(cuda_lib.SsmError) as e:
        cuda_lib.ssm_selective_scan_fwd(inp["x"], inp["delta"], None, True, inp["A"], inp["B"],
                                        inp["C"], None, None, y, None)
    assert e.value.status == cuda_lib.SSM_ERR_ALIGNMENT


@pytest.mark.parametrize("nseg", ["2", "5"])
def test_segment_carry_never_dies(cuda_lib, nseg, force_segments):
    """A = 0 keeps exp(A * S) = 1: the carry reaches every token of every later segment,
    so the carry pass must cover whole segments."""
    force_segments(int(nseg))
    inp = inputs.make_scan_inputs(1, 40, 700, 16, torch.float32, device=DEV, seed=21)
    inp["A"][:, :3] = 0.0
    inp["A"][:, 3:8] = 0.05          # a slowly growing state as well
    y, fs = run_gpu(cuda_lib, inp, torch.float32)
    yr, fr = run_oracle(inp)
    assert_parity(y, yr, torch.float32, what="y")
    assert_parity(fs, fr, torch.float32, what="final_state")


def test_segment_carry_dies_at_once(cuda_lib, force_segments):
    """Huge steps wipe the carry within one token: the carry pass stops in its first
    window and the pass-1 output stands."""
    force_segments(4)
    inp = inputs.make_scan_inputs(2, 33, 512, 16, torch.bfloat16, device=DEV, seed=22)
    inp["delta_bias"].fill_(60.0)
    y, fs = run_gpu(cuda_lib, inp, torch.bfloat16)
    yr, fr = run_oracle(inp)
    assert_parity(y, yr, torch.bfloat16, torch.bfloat16, what="y")
    assert_parity(fs, fr, torch.bfloat16, torch.float32, what="final_state")


@pytest.mark.parametrize("nseg", ["3", "7"])
def test_segment_carry_with_negative_steps(cuda_lib, nseg, force_segments):
    """Without the softplus a raw step can be negative, so the step sum S_t of a segment
    can fall again after rising: the carry's share exp(A S_t) h_in is checked against the
    oracle on every block, not cut off at the first small value."""
    force_segments(int(nseg))
    inp = inputs.make_scan_inputs(2, 24, 900, 16, torch.float32, device=DEV, seed=24)
    g = torch.Generator(DEV).manual_seed(25)
    inp["delta"] = (0.05 * torch.randn(inp["delta"].shape, device=DEV, generator=g) + 0.01).contiguous()
    inp["A"].mul_(0.25)
    y, fs = run_gpu(cuda_lib, inp, torch.float32, use_bias=False, softplus=False)
    yr, fr = run_oracle(inp, use_bias=False, softplus=False)
    assert (inp["delta"] < 0).float().mean().item() > 0.3
    assert_parity(y, yr, torch.float32, what="y")
    assert_parity(fs, fr, torch.float32, what="final_state")


def test_long_sequence_default_segmentation(cuda_lib):
    """Few channels and a long sequence choose the segmented path on their own."""
    inp = inputs.make_scan_inputs(1, 64, 40000, 16, torch.bfloat16, device=DEV, seed=23)
    y, fs = run_gpu(cuda_lib, inp, torch.float32)
    yr, fr = run_oracle(inp)
    assert_parity(y, yr, torch.bfloat16, torch.float32, what="y")
    assert_parity(fs, fr, torch.bfloat16, torch.float32, what="final_state")


def run_gpu_ex(ssm, inp, out_dtype, h0=None, zoh=False):
    x = inp["x"]
    y = torch.empty(x.shape, device=DEV, dtype=out_dtype)
    fs = torch.empty(x.shape[0], x.shape[1], inp["A"].shape[1], device=DEV, dtype=torch.float32)
    ssm.ssm_selective_scan_fwd_ex(x, inp["delta"], inp["delta_bias"], True, inp["A"], inp["B"],
                                  inp["C"], inp["D"], inp["z"], y, fs, h0, zoh)
    torch.cuda.synchronize()
    return y, fs


@pytest.mark.parametrize("batch,dim,L,N,din,dout", [
    (2, 37, 1000, 16, torch.bfloat16, torch.bfloat16),
    (3, 21, 331, 5, torch.float32, torch.float32),
    (1, 40, 256, 8, torch.bfloat16, torch.float32),
])
@pytest.mark.parametrize("h0,zoh", [(True, False), (False, True), (True, True)],
                         ids=["state", "zoh", "state+zoh"])
def test_initial_state_and_exact_zoh(cuda_lib, split, batch, dim, L, N, din, dout, h0, zoh):
    inp = inputs.make_scan_inputs(batch, dim, L, N, din, device=DEV, seed=batch + L + N + 7)
    if zoh:
        inp["A"][:, 0] = 0.0          # the a = 0 limit of the exact gain is Delta * B
    state = (torch.randn(batch, dim, N, device=DEV, generator=torch.Generator(DEV).manual_seed(8))
             if h0 else None)
    y, fs = run_gpu_ex(cuda_lib, inp, dout, state, zoh)
    yr, fr = oracle.scan(x=inp["x"], delta=inp["delta"], A=inp["A"], B=inp["B"], C=inp["C"],
                         D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=True,
                         h0=None if state is None else state, zoh_exact=zoh)
    assert_parity(y, yr, din, dout, what="y")
    assert_parity(fs, fr, din, torch.float32, what="final_state")


def test_continuation_equals_one_scan(cuda_lib):
    """Scanning L tokens, then the next L tokens from the returned state, gives the same
    outputs as one scan over 2L tokens (prefill continued across calls)."""
    inp = inputs.make_scan_inputs(2, 48, 1024, 16, torch.float32, device=DEV, seed=41)
    y_all, f_all = run_gpu_ex(cuda_lib, inp, torch.float32)
    half = {k: (v[..., :512].contiguous() if k in ("x", "delta", "z") else
                v[:, :512].contiguous() if k in ("B", "C") else v) for k, v in inp.items()}
    rest = {k: (v[..., 512:].contiguous() if k in ("x", "delta", "z") else
                v[:, 512:].contiguous() if k in ("B", "C") else v) for k, v in inp.items()}
    y1, f1 = run_gpu_ex(cuda_lib, half, torch.float32)
    y2, f2 = run_gpu_ex(cuda_lib, rest, torch.float32, h0=f1)
    assert_parity(torch.cat([y1, y2], dim=-1), to64(y_all), torch.float32, what="y halves vs whole")
    assert_parity(f2, to64(f_all), torch.float32, what="final state halves vs whole")


def test_empty_sequence_returns_initial_state(cuda_lib):
    h0 = torch.randn(2, 3, 16, device=DEV)
    x = torch.empty(2, 3, 0, device=DEV)
    y = torch.empty(2, 3, 0, device=DEV)
    fs = torch.zeros(2, 3, 16, device=DEV)
    Bm = torch.empty(2, 0, 16, device=DEV)
    cuda_lib.ssm_selective_scan_fwd_ex(x, x, None, True, -torch.ones(3, 16, device=DEV), Bm, Bm,
                                       None, None, y, fs, h0, False)
    torch.cuda.synchronize()
    assert torch.equal(fs, h0)
