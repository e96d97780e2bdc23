import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library through its Python binding; skips without a GPU."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_attention_24_b200 as ta
    ta.load()
    return ta


@pytest.fixture(autouse=True)
def _debug_build_bounds(request):
    """Under the debug build (TILEDATTN_LIB pointing at libtiledattn_debug.so)
    every test also fails if one of its launches recorded a bounds violation
    (a TMA coordinate or tensor-memory address that failed its check)."""
    yield
    if not os.environ.get("TILEDATTN_LIB", "").endswith("libtiledattn_debug.so"):
        return
    from tiled_attention_24_b200 import _binding
    if _binding._lib is None:
        return
    counters = _binding.attn_debug_counters(reset=False)
    assert counters[2] == 0, f"{request.node.nodeid}: {counters[2]} bounds violations"
