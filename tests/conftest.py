import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a B200)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def cuda_ok():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def gpu():
    if not cuda_ok():
        pytest.skip("no CUDA device")
    import torch
    return torch.device("cuda:0")


@pytest.fixture(scope="session")
def lkv_built():
    """The binding with liblkv.so built in-tree first (nvcc cross-compiles; no GPU needed to load it)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("lkv_build", os.path.join(ROOT, "latent_kv_cache_split_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import latent_kv_cache_split_b200 as L
    return L
