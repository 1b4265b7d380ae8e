"""B200 (sm_100a) selective state-space scan (S6): forward scan, its backward and the decode
step, the causal depthwise convolution in front of it, and Mamba-2's chunked SSD.

The computation lives in ``libssm.so`` (C ABI in ``include/ssm.h``); this package only
loads it and marshals torch tensors into it.
"""
from ._lib import (  # noqa: F401
    LIB_PATH,
    SSM_BF16,
    SSM_ERR_ALIGNMENT,
    SSM_ERR_CUDA,
    SSM_ERR_INVALID_ARG,
    SSM_ERR_SCRATCH,
    SSM_ERR_UNSUPPORTED,
    SSM_F32,
    SSM_OK,
    SsmError,
    causal_conv1d,
    load_library,
    selective_scan,
    selective_scan_bwd,
    ssd,
    ssm_causal_conv1d_fwd,
    ssm_causal_conv1d_step,
    ssm_device_timeouts,
    ssm_selective_scan_bwd,
    ssm_selective_scan_fwd,
    ssm_selective_scan_fwd_ex,
    ssm_selective_scan_fwd_noalloc,
    ssm_scan_force_segments,
    ssm_sfu_probe,
    ssm_ssd_fwd,
    ssm_state_step,
    ssm_state_step_multi,
    ssm_status_string,
    ssm_version,
)
