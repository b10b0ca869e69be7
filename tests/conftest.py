import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")

import pytest  # noqa: E402


@pytest.fixture(scope="session")
def oracle_lib():
    from oracle import build as ob
    return ob.build()


@pytest.fixture(scope="session")
def tq_lib():
    """Build libtq.so in-tree (no-op when up to date) and return the binding.
    The build script is loaded by path: importing the package needs the
    library it builds."""
    import importlib.util
    path = os.path.join(ROOT, "kv_cache_embedding_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_tq_build", path)
    kb = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(kb)
    kb.build()
    import kv_cache_embedding_b200 as tq
    return tq


@pytest.fixture(scope="session")
def cuda(tq_lib):
    import torch
    if not torch.cuda.is_available():
        pytest.fail("test marked gpu but no CUDA device is visible")
    return torch.device("cuda:0")
