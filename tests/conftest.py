import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")


def _cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library, loaded. GPU tests fail (not skip) when it is missing."""
    if not _cuda_available():
        pytest.skip("no CUDA device in this process")
    import block_causal_attention_wave_b200 as wave
    wave.load()  # raises if libwave.so is absent
    return wave
