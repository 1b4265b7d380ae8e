"""Host-side checks of the C ABI: the library loads, exports what include/ssm.h declares,
and rejects bad arguments before touching the GPU (no compute call is made here)."""
import ctypes
import os
import re

import pytest

import selective_state_space_45_b200 as ssm
from selective_state_space_45_b200 import build as ssm_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm.h")

# fake, 16-byte aligned "device" addresses: validation returns before any is dereferenced
P = 0x7F0000001000
MIS = 0x7F0000001004


@pytest.fixture(scope="module")
def lib():
    ssm_build.build()
    return ssm.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(ssm_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for expected in ("ssm_selective_scan_fwd", "ssm_selective_scan_fwd_ex", "ssm_selective_scan_fwd_noalloc",
                     "ssm_state_step", "ssm_causal_conv1d_fwd", "ssm_causal_conv1d_step",
                     "ssm_selective_scan_bwd", "ssm_state_step_multi",
                     "ssm_status_string", "ssm_version"):
        assert expected in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert getattr(lib, name) is not None


def test_status_strings_and_version(lib):
    assert ssm.ssm_status_string(ssm.SSM_OK) == "ok"
    for code in range(1, 6):
        s = ssm.ssm_status_string(code)
        assert s and s != "unknown status"
    assert ssm.ssm_status_string(99) == "unknown status"
    assert ssm.ssm_version() >= 10000


def scan(lib, **kw):
    args = dict(x=P, delta=P, bias=None, sp=1, A=P, B=P, C=P, D=P, z=P, y=P, fs=P,
                batch=2, dim=3, L=8, N=16, din=ssm.SSM_BF16, dout=ssm.SSM_BF16)
    args.update(kw)
    return lib.ssm_selective_scan_fwd(args["x"], args["delta"], args["bias"], args["sp"], args["A"],
                                      args["B"], args["C"], args["D"], args["z"], args["y"],
                                      args["fs"], args["batch"], args["dim"], args["L"], args["N"],
                                      args["din"], args["dout"], None)


def step(lib, **kw):
    args = dict(state=P, x=P, delta=P, A=P, B=P, C=P, D=P, z=P, y=P, batch=2, dim=3, N=16,
                din=ssm.SSM_BF16, dout=ssm.SSM_BF16)
    args.update(kw)
    return lib.ssm_state_step(args["state"], args["x"], args["delta"], args["A"], args["B"], args["C"],
                              args["D"], args["z"], args["y"], args["batch"], args["dim"], args["N"],
                              args["din"], args["dout"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(delta=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(A=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(B=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(C=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(y=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(batch=-1), ssm.SSM_ERR_INVALID_ARG),
    (dict(dim=-5), ssm.SSM_ERR_INVALID_ARG),
    (dict(L=-1), ssm.SSM_ERR_INVALID_ARG),
    (dict(N=0), ssm.SSM_ERR_INVALID_ARG),
    (dict(N=17), ssm.SSM_ERR_UNSUPPORTED),
    (dict(N=64), ssm.SSM_ERR_UNSUPPORTED),
    (dict(din=2), ssm.SSM_ERR_INVALID_ARG),
    (dict(dout=-1), ssm.SSM_ERR_INVALID_ARG),
    (dict(x=MIS), ssm.SSM_ERR_ALIGNMENT),
    (dict(B=MIS), ssm.SSM_ERR_ALIGNMENT),
    (dict(y=MIS), ssm.SSM_ERR_ALIGNMENT),
    (dict(fs=MIS), ssm.SSM_ERR_ALIGNMENT),
    (dict(bias=MIS), ssm.SSM_ERR_ALIGNMENT),
    # nothing to do: accepted without a launch, optional pointers may be absent
    (dict(batch=0), ssm.SSM_OK),
    (dict(dim=0, x=None, y=None), ssm.SSM_OK),
    (dict(L=0, fs=None), ssm.SSM_OK),
])
def test_scan_argument_checks(lib, kw, status):
    assert scan(lib, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(state=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(x=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(delta=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(y=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(batch=-2), ssm.SSM_ERR_INVALID_ARG),
    (dict(N=0), ssm.SSM_ERR_INVALID_ARG),
    (dict(N=17), ssm.SSM_ERR_UNSUPPORTED),
    (dict(din=7), ssm.SSM_ERR_INVALID_ARG),
    (dict(state=MIS), ssm.SSM_ERR_ALIGNMENT),
    (dict(A=MIS), ssm.SSM_ERR_ALIGNMENT),
    (dict(batch=0), ssm.SSM_OK),
])
def test_step_argument_checks(lib, kw, status):
    assert step(lib, **kw) == status


# distinct fake buffers, 1 MiB apart, for the calls that check overlaps
X, U, W, BIAS, H0, H1 = (0x7F0000000000 + k * (1 << 20) for k in range(6))


def conv(lib, **kw):
    args = dict(x=X, w=W, bias=BIAS, h0=H0, u=U, h1=H1, batch=2, dim=3, L=8, K=4, silu=1,
                din=ssm.SSM_BF16, dout=ssm.SSM_BF16)
    args.update(kw)
    return lib.ssm_causal_conv1d_fwd(args["x"], args["w"], args["bias"], args["h0"], args["u"],
                                     args["h1"], args["batch"], args["dim"], args["L"], args["K"],
                                     args["silu"], args["din"], args["dout"], None)


def conv_step(lib, **kw):
    args = dict(win=H0, x=X, w=W, bias=BIAS, u=U, batch=2, dim=3, K=4, silu=1,
                din=ssm.SSM_BF16, dout=ssm.SSM_BF16)
    args.update(kw)
    return lib.ssm_causal_conv1d_step(args["win"], args["x"], args["w"], args["bias"], args["u"],
                                      args["batch"], args["dim"], args["K"], args["silu"],
                                      args["din"], args["dout"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(w=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(u=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(K=0), ssm.SSM_ERR_INVALID_ARG),
    (dict(K=9), ssm.SSM_ERR_UNSUPPORTED),
    (dict(L=-1), ssm.SSM_ERR_INVALID_ARG),
    (dict(dim=-1), ssm.SSM_ERR_INVALID_ARG),
    (dict(din=3), ssm.SSM_ERR_INVALID_ARG),
    (dict(x=X + 8), ssm.SSM_ERR_ALIGNMENT),
    (dict(h1=H1 + 4), ssm.SSM_ERR_ALIGNMENT),
    (dict(w=W + 4), ssm.SSM_ERR_ALIGNMENT),
    # outputs overlapping inputs are refused: u over x, the new window over the old one
    (dict(u=X), ssm.SSM_ERR_INVALID_ARG),
    (dict(u=X + 16), ssm.SSM_ERR_INVALID_ARG),
    (dict(h1=H0), ssm.SSM_ERR_INVALID_ARG),
    (dict(h1=U + 32), ssm.SSM_ERR_INVALID_ARG),
    (dict(h1=X), ssm.SSM_ERR_INVALID_ARG),
    # x holds 2*3*8 bf16 = 96 bytes: a u that starts in its last 16 overlaps it
    (dict(u=X + 80), ssm.SSM_ERR_INVALID_ARG),
    (dict(batch=0), ssm.SSM_OK),
    (dict(dim=0, x=None, u=None, w=None), ssm.SSM_OK),
])
def test_conv_argument_checks(lib, kw, status):
    assert conv(lib, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(win=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(x=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(u=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(w=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(K=0), ssm.SSM_ERR_INVALID_ARG),
    (dict(K=9), ssm.SSM_ERR_UNSUPPORTED),
    (dict(win=H0 + 4), ssm.SSM_ERR_ALIGNMENT),
    (dict(win=X), ssm.SSM_ERR_INVALID_ARG),
    (dict(u=H0), ssm.SSM_ERR_INVALID_ARG),
    (dict(batch=0), ssm.SSM_OK),
])
def test_conv_step_argument_checks(lib, kw, status):
    assert conv_step(lib, **kw) == status


def bwd(lib, **kw):
    args = dict(x=P, delta=P, bias=None, sp=1, A=P, B=P, C=P, D=P, z=P, h0=None, dy=P, dfin=None,
                dx=P, ddelta=P, dA=P, dB=P, dC=P, dD=P, dz=P, dbias=None, dh0=None,
                batch=2, dim=3, L=8, N=16, din=ssm.SSM_BF16, dg=ssm.SSM_F32)
    args.update(kw)
    return lib.ssm_selective_scan_bwd(
        args["x"], args["delta"], args["bias"], args["sp"], args["A"], args["B"], args["C"],
        args["D"], args["z"], args["h0"], args["dy"], args["dfin"], args["dx"], args["ddelta"],
        args["dA"], args["dB"], args["dC"], args["dD"], args["dz"], args["dbias"], args["dh0"],
        args["batch"], args["dim"], args["L"], args["N"], args["din"], args["dg"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(dy=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(dx=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(ddelta=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(dA=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(dB=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(dC=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(z=None), ssm.SSM_ERR_INVALID_ARG),         # dz requested without a gate
    (dict(N=0), ssm.SSM_ERR_INVALID_ARG),
    (dict(N=17), ssm.SSM_ERR_UNSUPPORTED),
    (dict(L=-3), ssm.SSM_ERR_INVALID_ARG),
    (dict(dg=5), ssm.SSM_ERR_INVALID_ARG),
    (dict(dy=MIS), ssm.SSM_ERR_ALIGNMENT),
    (dict(dA=MIS), ssm.SSM_ERR_ALIGNMENT),
    (dict(dh0=MIS), ssm.SSM_ERR_ALIGNMENT),
    (dict(dim=0), ssm.SSM_OK),
])
def test_bwd_argument_checks(lib, kw, status):
    assert bwd(lib, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(state=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(ntok=-1), ssm.SSM_ERR_INVALID_ARG),
    (dict(N=17), ssm.SSM_ERR_UNSUPPORTED),
    (dict(y=MIS), ssm.SSM_ERR_ALIGNMENT),
    (dict(ntok=0), ssm.SSM_OK),
    (dict(batch=0), ssm.SSM_OK),
])
def test_step_multi_argument_checks(lib, kw, status):
    args = dict(state=P, x=P, delta=P, A=P, B=P, C=P, D=P, z=P, y=P, ntok=4, batch=2, dim=3, N=16,
                din=ssm.SSM_BF16, dout=ssm.SSM_BF16)
    args.update(kw)
    assert lib.ssm_state_step_multi(args["state"], args["x"], args["delta"], args["A"], args["B"],
                                    args["C"], args["D"], args["z"], args["y"], args["ntok"],
                                    args["batch"], args["dim"], args["N"], args["din"],
                                    args["dout"], None) == status


@pytest.mark.parametrize("kw,status", [
    (dict(out=None), ssm.SSM_ERR_INVALID_ARG),
    (dict(blocks=0), ssm.SSM_ERR_INVALID_ARG),
    (dict(iters=-1), ssm.SSM_ERR_INVALID_ARG),
    (dict(out=MIS), ssm.SSM_ERR_ALIGNMENT),
])
def test_sfu_probe_argument_checks(lib, kw, status):
    args = dict(out=P, blocks=1, iters=1)
    args.update(kw)
    assert lib.ssm_sfu_probe(args["out"], args["blocks"], args["iters"], None) == status


def test_python_binding_raises_on_error(lib):
    with pytest.raises(ssm.SsmError) as e:
        ssm._lib._check(ssm.SSM_ERR_UNSUPPORTED)
    assert e.value.status == ssm.SSM_ERR_UNSUPPORTED


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises((RuntimeError, OSError)):
        ctypes_path = str(tmp_path / "nope.so")
        saved = ssm._lib._lib
        ssm._lib._lib = None
        try:
            ssm.load_library(ctypes_path)
        finally:
            ssm._lib._lib = saved
