import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running CPU check")


def read_golden(name):
    """Parse ``key = v1 v2 ...`` lines of a golden fixture (``#`` starts a comment)."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = line.split("=", 1)
            out[k.strip()] = v.split()
    return out


@pytest.fixture
def golden():
    return read_golden


@pytest.fixture(autouse=True)
def _device_error_word_stays_clear(request):
    """Every GPU test must leave the library's device error word clear: a bounded
    in-kernel wait that ran out would otherwise only show up as a slow test."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    try:
        import torch
    except ImportError:  # pragma: no cover
        return
    if not torch.cuda.is_available():
        return
    from fp8_delayed_scaling_02_b200 import ops

    rc, where = ops.device_error(clear=True)
    assert rc == ops.FP8_OK, f"a bounded in-kernel wait ran out (site {where})"
