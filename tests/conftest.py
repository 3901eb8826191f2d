import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.build_oracle()
    return oracle


def cuda_available() -> bool:
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:  # pragma: no cover
        return False


@pytest.fixture(params=["fused", "split"])
def bwd_mode(request):
    """Runs a test once per backward mode; restores the default (fused) afterwards."""
    import column_sparse_masked_b200 as fm

    fm.set_bwd_mode(request.param)
    try:
        yield request.param
    finally:
        fm.set_bwd_mode("fused")
