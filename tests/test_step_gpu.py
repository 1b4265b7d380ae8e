"""GPU parity of ssm_state_step (one decode token, state in place) against the fp64 oracle,
and decode chaining against the full scan."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_45_b200 import inputs
from tests.helpers import assert_parity, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("batch,dim,N,din,dout", [
    (3, 40, 16, torch.float32, torch.float32),
    (5, 33, 5, torch.float32, torch.float32),
    (2, 17, 8, torch.bfloat16, torch.bfloat16),
    (4, 64, 16, torch.bfloat16, torch.float32),
    (1, 7, 1, torch.float32, torch.bfloat16),
    (2, 9, 12, torch.float32, torch.float32),
])
def test_single_step_parity(cuda_lib, batch, dim, N, din, dout):
    inp = inputs.make_decode_inputs(batch, dim, N, 1, din, device=DEV, seed=dim + N)
    state = inp["state"].clone()
    y = torch.empty(batch, dim, device=DEV, dtype=dout)
    cuda_lib.ssm_state_step(state, inp["x"][0], inp["delta"][0], inp["A"], inp["B"][0], inp["C"][0],
                            inp["D"], inp["z"][0], y)
    torch.cuda.synchronize()
    yr, sr = oracle.step(inp["state"], inp["x"][0], inp["delta"][0], inp["A"], inp["B"][0],
                         inp["C"][0], D=inp["D"], z=inp["z"][0])
    assert_parity(y, yr, din, dout, what="y")
    assert_parity(state, sr, din, torch.float32, what="state")


def test_step_without_optional_terms(cuda_lib):
    inp = inputs.make_decode_inputs(2, 24, 16, 1, torch.float32, device=DEV, seed=1)
    state = inp["state"].clone()
    y = torch.empty(2, 24, device=DEV)
    cuda_lib.ssm_state_step(state, inp["x"][0], inp["delta"][0], inp["A"], inp["B"][0], inp["C"][0],
                            None, None, y)
    torch.cuda.synchronize()
    yr, sr = oracle.step(inp["state"], inp["x"][0], inp["delta"][0], inp["A"], inp["B"][0], inp["C"][0])
    assert_parity(y, yr, torch.float32, what="y")
    assert_parity(state, sr, torch.float32, what="state")


def _chain(ssm, inp, state, dout):
    steps = inp["x"].shape[0]
    ys = []
    for t in range(steps):
        y = torch.empty(inp["x"].shape[1:], device=DEV, dtype=dout)
        ssm.ssm_state_step(state, inp["x"][t], inp["delta"][t], inp["A"], inp["B"][t], inp["C"][t],
                           inp["D"], inp["z"][t], y)
        ys.append(y)
    torch.cuda.synchronize()
    return torch.stack(ys, dim=-1)            # [batch, dim, steps]


def test_decode_config_chain_vs_oracle_scan(cuda_lib):
    """64 chained steps from an N(0,1) state, checked against the oracle's scan started from
    that state (sampled sequences x channels of the 256 x 5120 workload)."""
    inp = inputs.make_config_inputs("decode", device=DEV)
    state = inp["state"].clone()
    y = _chain(cuda_lib, inp, state, torch.bfloat16)
    rng = np.random.default_rng(5)
    bsel = torch.as_tensor(np.sort(rng.choice(256, 16, replace=False)), device=DEV)
    dsel = torch.as_tensor(np.sort(rng.choice(5120, 96, replace=False)), device=DEV)

    def sel(t):     # [steps, batch, dim] -> [b, d, steps]
        return to64(t.index_select(1, bsel).index_select(2, dsel).permute(1, 2, 0))

    yr, fr = oracle.scan(x=sel(inp["x"]), delta=sel(inp["delta"]), z=sel(inp["z"]),
                         B=to64(inp["B"].index_select(1, bsel).permute(1, 0, 2)),
                         C=to64(inp["C"].index_select(1, bsel).permute(1, 0, 2)),
                         A=to64(inp["A"].index_select(0, dsel)), D=to64(inp["D"].index_select(0, dsel)),
                         h0=to64(inp["state"].index_select(0, bsel).index_select(1, dsel)))
    assert_parity(y.index_select(0, bsel).index_select(1, dsel), yr, torch.bfloat16, torch.bfloat16,
                  what="decode y")
    assert_parity(state.index_select(0, bsel).index_select(1, dsel), fr, torch.bfloat16,
                  torch.float32, what="decode state")


@pytest.mark.parametrize("din,dout", [(torch.float32, torch.float32), (torch.bfloat16, torch.bfloat16)])
def test_chain_from_zero_equals_gpu_scan(cuda_lib, din, dout):
    """Decode chaining from a zero state equals the forward scan over the same tokens."""
    batch, dim, N, L = 8, 200, 16, 64
    inp = inputs.make_decode_inputs(batch, dim, N, L, din, device=DEV, seed=2)
    state = torch.zeros(batch, dim, N, device=DEV)
    y_step = _chain(cuda_lib, inp, state, dout)
    x = inp["x"].permute(1, 2, 0).contiguous()
    dl = inp["delta"].permute(1, 2, 0).contiguous()
    z = inp["z"].permute(1, 2, 0).contiguous()
    B = inp["B"].permute(1, 0, 2).contiguous()
    C = inp["C"].permute(1, 0, 2).contiguous()
    y_scan = torch.empty(batch, dim, L, device=DEV, dtype=dout)
    fs = torch.empty(batch, dim, N, device=DEV)
    cuda_lib.ssm_selective_scan_fwd(x, dl, None, False, inp["A"], B, C, inp["D"], z, y_scan, fs)
    torch.cuda.synchronize()
    assert_parity(y_step, to64(y_scan), din, dout, what="y chain vs scan")
    assert_parity(state, to64(fs), din, torch.float32, what="state chain vs scan")


@pytest.mark.parametrize("ntok,batch,dim,N,din,dout", [
    (4, 3, 40, 16, torch.bfloat16, torch.bfloat16),
    (1, 2, 33, 5, torch.float32, torch.float32),
    (7, 2, 17, 8, torch.float32, torch.bfloat16),
    (3, 4, 64, 16, torch.bfloat16, torch.float32),
])
def test_multi_token_step_matches_chained_steps_and_oracle(cuda_lib, ntok, batch, dim, N, din, dout):
    inp = inputs.make_decode_inputs(batch, dim, N, ntok, din, device=DEV, seed=ntok + dim)
    st_multi = inp["state"].clone()
    y_multi = torch.empty(ntok, batch, dim, device=DEV, dtype=dout)
    cuda_lib.ssm_state_step_multi(st_multi, inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                  inp["D"], inp["z"], y_multi)
    st_chain = inp["state"].clone()
    ys = []
    for t in range(ntok):
        # fresh copies: every pointer the library takes is 16-byte aligned
        y = torch.empty(batch, dim, device=DEV, dtype=dout)
        cuda_lib.ssm_state_step(st_chain, inp["x"][t].clone(), inp["delta"][t].clone(), inp["A"],
                                inp["B"][t].clone(), inp["C"][t].clone(), inp["D"],
                                inp["z"][t].clone(), y)
        ys.append(y)
    torch.cuda.synchronize()
    assert torch.equal(st_multi, st_chain)                 # same arithmetic, same order
    assert torch.equal(y_multi, torch.stack(ys))
    h = to64(inp["state"])
    for t in range(ntok):
        yr, h = oracle.step(h, inp["x"][t], inp["delta"][t], inp["A"], inp["B"][t], inp["C"][t],
                            D=inp["D"], z=inp["z"][t])
        assert_parity(y_multi[t], yr, din, dout, what="y[%d]" % t)
    assert_parity(st_multi, h, din, torch.float32, what="state")


def test_multi_token_step_with_no_tokens_keeps_state(cuda_lib):
    inp = inputs.make_decode_inputs(2, 8, 16, 1, torch.float32, device=DEV, seed=1)
    st = inp["state"].clone()
    cuda_lib.ssm_state_step_multi(st, inp["x"][:0], inp["delta"][:0], inp["A"], inp["B"][:0],
                                  inp["C"][:0], inp["D"], inp["z"][:0],
                                  torch.empty(0, 2, 8, device=DEV))
    torch.cuda.synchronize()
    assert torch.equal(st, inp["state"])


@pytest.mark.parametrize("batch,dim,N", [(40, 1, 16), (9, 3, 4), (5, 70, 8)])
def test_multi_token_step_small_dims_span_many_sequences(cuda_lib, batch, dim, N):
    # channel ranges narrower than a block (most lanes idle), sequences shared out over the
    # blocks, three rounds of staged B, C per sequence (the last one partial)
    ntok = 11
    inp = inputs.make_decode_inputs(batch, dim, N, ntok, torch.float32, device=DEV, seed=batch + dim)
    st = inp["state"].clone()
    y = torch.empty(ntok, batch, dim, device=DEV)
    cuda_lib.ssm_state_step_multi(st, inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                  inp["z"], y)
    torch.cuda.synchronize()
    h = to64(inp["state"])
    for t in range(ntok):
        yr, h = oracle.step(h, inp["x"][t], inp["delta"][t], inp["A"], inp["B"][t], inp["C"][t],
                            D=inp["D"], z=inp["z"][t])
        assert_parity(y[t], yr, torch.float32, torch.float32, what="y[%d]" % t)
    assert_parity(st, h, torch.float32, torch.float32, what="state")


@pytest.mark.parametrize("ntok,N,din,dout", [(6, 16, torch.bfloat16, torch.bfloat16),
                                             (9, 8, torch.float32, torch.float32),
                                             (5, 12, torch.bfloat16, torch.float32),
                                             (7, 5, torch.float32, torch.bfloat16)])
def test_multi_token_step_blocks_walk_many_sequences(cuda_lib, ntok, N, din, dout):
    # more sequences than the resident blocks of a channel range: each block walks several,
    # loading the next one's state and first tokens while it computes the current one (the
    # state through the shared ring when N is a multiple of 4, else through registers; N =
    # 12 leaves the last quad of the padded 16 empty); the last channel range is ragged
    # (3000 = 23 x 128 + 56)
    batch, dim = 96, 3000
    inp = inputs.make_decode_inputs(batch, dim, N, ntok, din, device=DEV, seed=ntok + N)
    st_multi = inp["state"].clone()
    y_multi = torch.empty(ntok, batch, dim, device=DEV, dtype=dout)
    cuda_lib.ssm_state_step_multi(st_multi, inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                  inp["D"], inp["z"], y_multi)
    st_chain = inp["state"].clone()
    for t in range(ntok):
        y = torch.empty(batch, dim, device=DEV, dtype=dout)
        cuda_lib.ssm_state_step(st_chain, inp["x"][t].clone(), inp["delta"][t].clone(), inp["A"],
                                inp["B"][t].clone(), inp["C"][t].clone(), inp["D"],
                                inp["z"][t].clone(), y)
        torch.cuda.synchronize()
        assert torch.equal(y_multi[t], y), t
    assert torch.equal(st_multi, st_chain)
    h = to64(inp["state"])
    for t in range(ntok):
        yr, h = oracle.step(h, inp["x"][t], inp["delta"][t], inp["A"], inp["B"][t], inp["C"][t],
                            D=inp["D"], z=inp["z"][t])
        assert_parity(y_multi[t], yr, din, dout, what="y[%d]" % t)
    assert_parity(st_multi, h, din, torch.float32, what="state")
