import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU oracle run")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("gpu test run without a CUDA device")
    return True


@pytest.fixture(autouse=True)
def _device_error_word_clear(request):
    """After every GPU test the library's device error word must be clear: no
    bounded wait gave up and, on the bounds-checking build, no index check
    fired.  Tests that provoke an error on purpose read (and so clear) the
    word themselves."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    import context_attention_dits_cp_b200 as cp
    from context_attention_dits_cp_b200 import binding as bd
    st = cp.last_device_error()
    assert st == 0, f"device error word after the test: {bd.STATUS.get(st, st)}"
