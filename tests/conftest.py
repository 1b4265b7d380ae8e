import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library, built in-tree; GPU tests fail loudly if it is missing."""
    import torch

    if not torch.cuda.is_available():
        pytest.fail("gpu test collected on a machine without CUDA")
    import selective_state_space_45_b200 as ssm

    ssm.load_library()
    return ssm


@pytest.fixture
def force_segments(cuda_lib):
    """Set the library's forced time-segment count for one test (None or 0: automatic);
    the automatic plan is restored afterwards."""
    def setter(k):
        cuda_lib.ssm_scan_force_segments(int(k or 0))
    yield setter
    cuda_lib.ssm_scan_force_segments(0)
