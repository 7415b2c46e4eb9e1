import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def lsq():
    """The C-ABI binding with a CUDA device; GPU tests only."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nf4_layer_streamed_blockwise_b200 import lib
    return lib


@pytest.fixture(autouse=True)
def _device_status_clean(request):
    """After every GPU test the library's device status word must read (0, 0):
    no bounded wait in any kernel ran out, so no result of the test came from
    a kernel that gave up (reading the word also clears it)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    from nf4_layer_streamed_blockwise_b200 import lib
    torch.cuda.synchronize()
    assert lib.lsq_device_status() == (0, 0), "a device-side bounded wait ran out during this test"


def pytest_sessionfinish(session, exitstatus):
    """With LSQ_PARITY_LOG set, write what every parity check measured."""
    path = os.environ.get("LSQ_PARITY_LOG")
    if not path:
        return
    import tolerances
    with open(path, "w") as f:
        json.dump(tolerances.RECORD, f, indent=0)
