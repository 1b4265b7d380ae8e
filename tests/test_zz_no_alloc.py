"""The allocation-free scan entry point (ssm_selective_scan_fwd_noalloc).

Some callers may not allocate device memory while they run -- for instance an engine
that gave all free memory to its own pool at start-up.  For them the library offers a
variant of the selective scan whose segment scratch lives in a fixed device array.  These
tests call it through the C ABI and check it against the regular entry point on the same
inputs, with the parity tolerances of the rest of the suite, over consecutive calls that
share (and leave behind) the array's contents.  The file is collected last on purpose.
"""
import ctypes
import os

import pytest
import torch

from selective_state_space_45_b200 import inputs
from tests.helpers import assert_parity, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _outputs(inp, dout):
    batch, dim, L = inp["x"].shape
    y = torch.full((batch, dim, L), 7.0, device=DEV, dtype=dout)
    fs = torch.full((batch, dim, inp["A"].shape[1]), 7.0, device=DEV)
    return y, fs


def _call(fn, inp, y, fs):
    fn(inp["x"], inp["delta"], inp["delta_bias"], True, inp["A"], inp["B"], inp["C"], inp["D"],
       inp["z"], y, fs)


def _compare(ssm, inp, din, dout):
    y_ref, fs_ref = _outputs(inp, dout)
    _call(ssm.ssm_selective_scan_fwd, inp, y_ref, fs_ref)
    y, fs = _outputs(inp, dout)
    _call(ssm.ssm_selective_scan_fwd_noalloc, inp, y, fs)
    torch.cuda.synchronize()
    assert_parity(y, to64(y_ref), din, dout, what="y (no-alloc vs regular)")
    assert_parity(fs, to64(fs_ref), din, torch.float32, what="final_state (no-alloc vs regular)")


def _pool_watermark():
    """(reset, high): the used-memory high watermark of the device's default memory pool,
    the pool that stream-ordered allocations (cudaMallocAsync) draw from, read through the
    CUDA runtime that torch loads."""
    try:
        import nvidia.cuda_runtime as rt_pkg
        path = os.path.join(os.path.dirname(rt_pkg.__file__), "lib", "libcudart.so.12")
    except ImportError:
        path = "libcudart.so.12"
    rt = ctypes.CDLL(path)
    pool = ctypes.c_void_p()
    assert rt.cudaDeviceGetDefaultMemPool(ctypes.byref(pool), torch.cuda.current_device()) == 0
    used_mem_high = 8                      # cudaMemPoolAttrUsedMemHigh

    def reset():
        zero = ctypes.c_uint64(0)
        assert rt.cudaMemPoolSetAttribute(pool, used_mem_high, ctypes.byref(zero)) == 0

    def high():
        v = ctypes.c_uint64(0)
        assert rt.cudaMemPoolGetAttribute(pool, used_mem_high, ctypes.byref(v)) == 0
        return v.value

    return reset, high


def test_segmented_scan_two_calls_in_a_row(cuda_lib, force_segments):
    """Few channels, long sequences: the segmented path, which needs scratch.  The second
    call runs on different data over the array the first call left behind.  The regular
    call draws its scratch from the default memory pool (the positive control); the
    allocation-free call leaves the pool's high watermark at zero."""
    force_segments(0)
    first = inputs.make_scan_inputs(1, 64, 40000, 16, torch.bfloat16, device=DEV, seed=31)
    second = inputs.make_scan_inputs(2, 40, 24000, 16, torch.bfloat16, device=DEV, seed=32)
    reset, high = _pool_watermark()
    torch.cuda.synchronize()
    reset()
    y, fs = _outputs(first, torch.bfloat16)
    _call(cuda_lib.ssm_selective_scan_fwd, first, y, fs)
    torch.cuda.synchronize()
    assert high() > 0
    reset()
    _call(cuda_lib.ssm_selective_scan_fwd_noalloc, first, y, fs)
    torch.cuda.synchronize()
    assert high() == 0
    _compare(cuda_lib, first, torch.bfloat16, torch.bfloat16)
    _compare(cuda_lib, second, torch.bfloat16, torch.bfloat16)
    _compare(cuda_lib, first, torch.bfloat16, torch.float32)


def test_forced_segments_fp32_two_calls(cuda_lib, force_segments):
    force_segments(5)
    for seed in (33, 34):
        inp = inputs.make_scan_inputs(3, 21, 997, 5, torch.float32, device=DEV, seed=seed)
        _compare(cuda_lib, inp, torch.float32, torch.float32)


def test_unsegmented_sizes_need_no_scratch(cuda_lib, force_segments):
    force_segments(0)
    inp = inputs.make_scan_inputs(8, 1536, 256, 16, torch.bfloat16, device=DEV, seed=35)
    _compare(cuda_lib, inp, torch.bfloat16, torch.bfloat16)
    _compare(cuda_lib, inp, torch.bfloat16, torch.bfloat16)


def test_scratch_beyond_the_array_is_rejected(cuda_lib, force_segments):
    """2048 channels cut into 64 segments need 2048 * 64 * 17 floats > 4 MiB: the call
    returns SSM_ERR_SCRATCH and writes nothing."""
    force_segments(64)
    inp = inputs.make_scan_inputs(1, 2048, 8192, 16, torch.bfloat16, device=DEV, seed=36)
    y, fs = _outputs(inp, torch.bfloat16)
    with pytest.raises(cuda_lib.SsmError) as e:
        _call(cuda_lib.ssm_selective_scan_fwd_noalloc, inp, y, fs)
    assert e.value.status == cuda_lib.SSM_ERR_SCRATCH
    torch.cuda.synchronize()
    assert bool((y == 7.0).all()) and bool((fs == 7.0).all())
