import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


@pytest.fixture(params=[False, True], ids=["row_stores", "tma_store"])
def store_path(request):
    """Runs a GPU test with each output path of the dense and grouped GEMMs: every
    thread storing its own row, and shared-memory staging with TMA stores."""
    import moe_grouped_gemm_quantize_b200 as lnq
    previous = lnq.lnq_set_tma_store(request.param)
    yield request.param
    lnq.lnq_set_tma_store(previous)


@pytest.fixture(params=[0, 1], ids=["one_cta", "cta_pairs"])
def mx_pairs(request):
    """Runs a block-scaled (UE8M0 / MXFP8) GEMM test with single CTAs on 128 x 256 tiles
    and with CTA pairs on 256 x 256 tiles (dense products of more than 128 rows)."""
    import moe_grouped_gemm_quantize_b200 as lnq
    previous = lnq.lnq_set_dense_cta_pairs(request.param)
    yield request.param
    lnq.lnq_set_dense_cta_pairs(previous)
