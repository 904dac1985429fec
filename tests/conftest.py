import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def gpu_available() -> bool:
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library's Python binding; fails loudly when the library or GPU is missing."""
    if not gpu_available():
        pytest.fail("a GPU test ran without a CUDA device")
    import sparse_query_attention_sqa_b200 as sqa

    sqa.load_library()
    return sqa
