"""Shared test helpers: tolerances of the parity bar and channel sampling.

Tolerances (one reading of the parity bar, applied per output tensor):
  * fp32 inputs:  normwise relative error  max|gpu - ref| / max|ref|  <= 1e-4; when the
    output is written as bf16, each element may also carry its bf16 rounding
    (at most 2^-8 of its magnitude): |gpu - ref| <= 1e-4 max|ref| + 2^-8 |ref|.
  * bf16 inputs, fp32 state:  relative L2 error <= 5e-3, and max-abs <= 2e-2 on every
    fp32 output (final state; y when it is written in fp32).  A bf16 y is rounded to
    bf16 on the way out, so there the max-abs bound is applied as |gpu - ref| <=
    2e-2 + 2^-7 |ref|: the bound plus one bf16 rounding step of the output.
"""
import numpy as np
import torch

FP32_REL = 1e-4
BF16_MAXABS = 2e-2
BF16_RELL2 = 5e-3
BF16_ULP = 2.0 ** -7
BF16_HALF_ULP = 2.0 ** -8


def to64(t):
    return t.detach().to("cpu").double().numpy()


def assert_parity(gpu, ref, in_dtype, out_dtype=None, what="y"):
    """Compare a GPU result (torch tensor or numpy) with the fp64 oracle's (numpy)."""
    g = to64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    if g.size == 0:
        return {}
    assert np.all(np.isfinite(g)), "%s: non-finite values from the GPU" % what
    err = np.abs(g - r)
    scale = max(float(np.max(np.abs(r))), 1e-30)
    stats = dict(max_abs=float(err.max()), norm_rel=float(err.max()) / scale,
                 rel_l2=float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)))
    if in_dtype == torch.float32:
        if out_dtype == torch.bfloat16:
            bad = err > FP32_REL * scale + BF16_HALF_ULP * np.abs(r)
            assert not bad.any(), (what, stats, int(bad.sum()))
        else:
            assert stats["norm_rel"] <= FP32_REL, (what, stats)
    else:
        assert stats["rel_l2"] <= BF16_RELL2, (what, stats)
        if out_dtype == torch.bfloat16:
            bound = BF16_MAXABS + BF16_ULP * np.abs(r)
            bad = err > bound
            assert not bad.any(), (what, stats, int(bad.sum()))
        else:
            assert stats["max_abs"] <= BF16_MAXABS, (what, stats)
    return stats


def oracle_inputs_for(inp, bsel, dsel):
    """Slice a workload's inputs to sequences ``bsel`` x channels ``dsel`` (exact values)."""
    bsel = torch.as_tensor(bsel, dtype=torch.long)
    dsel = torch.as_tensor(dsel, dtype=torch.long)
    dev = inp["x"].device

    def rows(t):  # [batch, dim, L] -> [len(bsel), len(dsel), L]
        return t.index_select(0, bsel.to(dev)).index_select(1, dsel.to(dev))

    return dict(
        x=to64(rows(inp["x"])), delta=to64(rows(inp["delta"])), z=to64(rows(inp["z"])),
        B=to64(inp["B"].index_select(0, bsel.to(dev))), C=to64(inp["C"].index_select(0, bsel.to(dev))),
        A=to64(inp["A"].index_select(0, dsel.to(dev))), D=to64(inp["D"].index_select(0, dsel.to(dev))),
        delta_bias=to64(inp["delta_bias"].index_select(0, dsel.to(dev))),
    )
