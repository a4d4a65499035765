import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload (minutes)")
    config.addinivalue_line("markers", "last: runs after every other test (collection order)")


def cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


# GPU parity files in the order they run: the cheap kernel-level checks first (router, dispatch),
# then the whole block and the expert half, then the sublayer, the dense MLP and the low-precision
# checkpoints.  Tests marked `last` run after all others.
_ORDER = ["test_gpu_route.py", "test_gpu_permute.py", "test_gpu_forward.py", "test_gpu_experts.py", "test_gpu_ep.py",
          "test_gpu_block.py", "test_gpu_dense.py", "test_gpu_fp8.py", "test_gpu_mxfp8.py", "test_gpu_nvfp4.py",
          "test_gpu_w4a4.py"]


def _rank(item) -> tuple:
    if item.get_closest_marker("last") is not None:
        return (2, 0)
    name = os.path.basename(str(item.fspath))
    return (1, _ORDER.index(name)) if name in _ORDER else (0, 0)


def pytest_collection_modifyitems(config, items):
    items[:] = [it for _, it in sorted(enumerate(items), key=lambda p: (_rank(p[1]), p[0]))]
    if cuda_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(scope="session")
def bank():
    """The shared Beam layer, its checkpoints, inputs and oracle results (tests/fullsize.py)."""
    from tests import fullsize
    return fullsize.bank()


@pytest.fixture(scope="session")
def beam_weights(bank):
    """The shared Beam layer's expert weights (20 GB bf16), drawn once per session on cuda:0."""
    return bank.gpu


@pytest.fixture(scope="session")
def beam_weights_fp8(bank):
    """MXFP8 copy of the shared Beam layer's expert weights (10 GB codes + scales) on cuda:0."""
    return bank.fp8()


@pytest.fixture(scope="session")
def beam_weights_nvfp4(bank):
    """NVFP4 copy of the shared Beam layer's expert weights (5.3 GB codes + scales) on cuda:0."""
    return bank.nvfp4()
