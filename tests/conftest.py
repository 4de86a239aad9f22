import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    oracle.set_mutation(0)
    return oracle


@pytest.fixture(scope="session")
def tam_lib():
    """The built C-ABI library (compiled on first use if it is missing)."""
    from top_attention_mass_b200 import build as tam_build
    tam_build.build_library()
    import top_attention_mass_b200 as tam
    return tam


def pytest_collection_modifyitems(config, items):
    # GPU tests need a device; skip them with a clear reason when there is none.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)
