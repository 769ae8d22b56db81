import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# Guard bytes around every device buffer an index owns (a stand-in for a memory checker):
# set before the library makes its first allocation; checked after every GPU test below.
os.environ.setdefault("PARISKV_GUARD", "1")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running check")


def _has_gpu() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if _has_gpu():
        return
    skip = pytest.mark.skip(reason="no CUDA device in this environment")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


# The CUDA library and the oracle are compiled in-tree on first use (nvcc cross-compiles for
# sm_100a without a GPU); an up-to-date build is reused.
def pytest_sessionstart(session):
    from long_context_kv_srht_b200 import build as kbuild
    kbuild.build()
    import oracle
    oracle.build()


@pytest.fixture(autouse=True)
def _guard_bytes_intact(request):
    """After each GPU test: no kernel wrote past either end of an index buffer."""
    yield
    if "gpu" not in request.keywords or not _has_gpu() or os.environ.get("PARISKV_GUARD") != "1":
        return
    from long_context_kv_srht_b200 import pariskv as pk
    pk.check_guards()
