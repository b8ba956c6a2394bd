import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle():
    import oracle as orc
    orc.build()
    return orc


@pytest.fixture(autouse=True)
def _device_status_clean(request):
    """After every GPU test: no bounded device-side wait of the library ran out."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    from trainable_block_sparse_v2_b200 import binding
    torch.cuda.synchronize()
    assert binding.infllmv2_device_status() == 0, "a device-side wait timed out"
