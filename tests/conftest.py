import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running full-size case")


def read_golden(name):
    """Rows of a golden text fixture, comments and blank lines dropped."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def kvq_lib():
    """The binding module; builds libkvq.so in-tree first if it is missing."""
    # build.py by path: importing the package would load a stale library first
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "kvq_build", os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                                  "bit_attention_decode_b200", "build.py"))
    _build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(_build)
    if not _build.up_to_date():
        _build.build()
    import bit_attention_decode_b200 as kvq
    return kvq


@pytest.fixture(scope="session")
def kvq(kvq_lib):
    """The binding module on a CUDA device (GPU tests only)."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    return kvq_lib
