import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


_PARITY_REPORT = []


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def parity_report():
    """Lines (one per checked workload) printed in the session's summary."""
    return _PARITY_REPORT


def pytest_terminal_summary(terminalreporter):
    if _PARITY_REPORT:
        terminalreporter.write_sep("-", "parity against the fp64 oracle")
        for line in _PARITY_REPORT:
            terminalreporter.write_line(line)


def read_golden(name: str) -> dict:
    """Parse a `key value...` fixture; '#' lines are comments (citations)."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            nums = [float(v) if "." in v else int(v) for v in vals]
            out[key] = nums if len(nums) > 1 else nums[0]
    return out


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def cuda_dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(autouse=True)
def _device_kernels_healthy(request):
    """After every GPU test: no bounded wait inside a library kernel expired."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    import paged_kv_cache_367_b200 as pkv
    assert pkv.pkv_device_status(clear=True) == 0, "a device-side wait expired"
