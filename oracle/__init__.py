"""fp64 CPU oracle for the selective scan -- test infrastructure only.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The library itself never does.
"""
from .oracle import (  # noqa: F401
    affine_scan_hillis_steele,
    affine_scan_loop,
    build,
    causal_conv1d,
    conv1d_step,
    lti_conv,
    lti_kernel,
    scan,
    scan_bwd,
    scan_parallel_reference,
    ssd_chunked,
    ssd_loop,
    step,
)
