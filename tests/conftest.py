import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))
for _p in (ROOT, TESTS):  # the repository modules, and helpers shared between test files
    if _p not in sys.path:
        sys.path.insert(0, _p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(params=["fused", "general"])
def both_paths(request):
    """Runs the test once on each tensor-core prefill path (tc_set_prefill_path),
    for the calls both take (bf16, d = 64, W a multiple of 128); other calls
    run where they always do."""
    import sliding_window_attention_tc_b200 as tc
    with tc.prefill_path(request.param):
        yield request.param
