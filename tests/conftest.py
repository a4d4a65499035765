import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload (minutes)")


def cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if cuda_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(scope="session")
def beam_weights():
    """The shared Beam layer's expert weights (20 GB bf16), drawn once per session on cuda:0."""
    import beam_synth as bs
    wg, wu, wd = bs.make_experts(bs.WORKLOADS["prefill"], device="cuda")
    return wg, wu, wd


@pytest.fixture(scope="session")
def beam_weights_fp8(beam_weights):
    """MXFP8 copy of the shared Beam layer's expert weights (10 GB codes + scales) on cuda:0."""
    import beam_synth as bs
    return bs.quantize_experts(*beam_weights)


@pytest.fixture(scope="session")
def beam_weights_nvfp4(beam_weights):
    """NVFP4 copy of the shared Beam layer's expert weights (5.3 GB codes + scales) on cuda:0."""
    import beam_synth as bs
    return bs.quantize_experts_nvfp4(*beam_weights)
