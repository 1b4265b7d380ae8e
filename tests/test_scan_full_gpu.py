"""Full-size workloads on the GPU, in the launch configuration the benchmark times,
checked against the fp64 oracle on sampled channels (every channel's scan is
independent, so a sample of (sequence, channel) rows is computed exactly)."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_45_b200 import inputs
from tests.helpers import assert_parity, oracle_inputs_for

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check_sampled(ssm, name, n_dims, out_dtypes=(torch.bfloat16, torch.float32), seed=0):
    inp = inputs.make_config_inputs(name, device=DEV, seed=seed)
    batch, dim, L = inp["x"].shape
    rng = np.random.default_rng(123)
    dsel = np.sort(rng.choice(dim, size=n_dims, replace=False))
    dsel[0] = 0
    dsel[-1] = dim - 1                      # include the first and the last channel group
    bsel = np.arange(batch)
    sub = oracle_inputs_for(inp, bsel, dsel)
    yr, fr = oracle.scan(delta_softplus=True, **sub)
    for dout in out_dtypes:
        y = torch.empty(inp["x"].shape, device=DEV, dtype=dout)
        fs = torch.empty(batch, dim, inp["A"].shape[1], device=DEV)
        ssm.ssm_selective_scan_fwd(inp["x"], inp["delta"], inp["delta_bias"], True, inp["A"],
                                   inp["B"], inp["C"], inp["D"], inp["z"], y, fs)
        torch.cuda.synchronize()
        ys = y[:, torch.as_tensor(dsel, device=DEV)]
        fss = fs[:, torch.as_tensor(dsel, device=DEV)]
        assert_parity(ys, yr, torch.bfloat16, dout, what="%s y (%s)" % (name, dout))
        assert_parity(fss, fr, torch.bfloat16, torch.float32, what="%s final_state" % name)
        del y, fs
    del inp
    torch.cuda.empty_cache()


def test_mamba130m_shape_sampled(cuda_lib):
    _check_sampled(cuda_lib, "mamba130m", 48)


def test_mamba2p8b_shape_sampled(cuda_lib):
    _check_sampled(cuda_lib, "mamba2p8b", 24)


def test_long_context_sampled(cuda_lib):
    # one sequence of 2^20 tokens, cut into segments scanned in parallel from their carries
    _check_sampled(cuda_lib, "long1m", 6, out_dtypes=(torch.bfloat16,))


def test_long_context_slow_decays_sampled(cuda_lib):
    # the same length with |A| down to 0.0067: a segment's carry outlives the segment
    _check_sampled(cuda_lib, "long1m_slow", 6, out_dtypes=(torch.bfloat16,))
