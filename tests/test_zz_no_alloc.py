"""The allocation-free entry point lnq_fp8_block_gemm_nt_static_ws.

Its K split keeps partial tiles in the library's fixed device array instead of a
caller's workspace.  Two consecutive calls must give the same bytes as the
workspace entry point on the same operands (the split plan, and so the order in
which partial tiles are added, is the same); a product whose split needs more than
the array holds is rejected before any launch.  This file is collected last, so it
also runs after every other test in the same process.
"""
import pytest
import torch

import moe_grouped_gemm_quantize_b200 as lnq
from moe_grouped_gemm_quantize_b200 import synthetic

pytestmark = pytest.mark.gpu
DEV = "cuda"
STATIC_BYTES = 10 << 20


def operands(M, N, K, seed):
    a = synthetic.gaussian_bf16((M, K), 1.0, seed)
    w = synthetic.gaussian_bf16((N, K), 0.02, seed + 1)
    wq, ws = lnq.quantize_weights(w.to(DEV))
    aq, sa = lnq.quantize_activations(a.to(DEV))
    return aq, sa, wq, ws


@pytest.mark.parametrize("M,N,K", [(8, 1152, 4096), (64, 12288, 4096), (33, 400, 2048), (1, 12288, 4096)])
def test_two_calls_match_the_workspace_entry_point(M, N, K):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    need = lnq.lnq_fp8_block_gemm_nt_workspace_bytes(M, N, K, sms)
    assert 0 < need <= STATIC_BYTES
    aq, sa, wq, ws = operands(M, N, K, seed=M + N)
    work = lnq.gemm_workspace(M, N, K, DEV)
    d_ref = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    lnq.lnq_fp8_block_gemm_nt_ws(aq, sa, wq, ws, d_ref, work)
    d1 = torch.full_like(d_ref, float("nan"))
    d2 = torch.full_like(d_ref, float("nan"))
    lnq.lnq_fp8_block_gemm_nt_static_ws(aq, sa, wq, ws, d1)
    lnq.lnq_fp8_block_gemm_nt_static_ws(aq, sa, wq, ws, d2)
    torch.cuda.synchronize()
    assert lnq.lnq_get_last_device_error() == 0
    assert torch.equal(d1.view(torch.int16), d_ref.view(torch.int16))
    assert torch.equal(d2.view(torch.int16), d_ref.view(torch.int16))


def test_products_that_do_not_split_run_the_plain_kernel():
    M, N, K = 256, 512, 1024
    aq, sa, wq, ws = operands(M, N, K, seed=5)
    d_ref = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    lnq.lnq_fp8_block_gemm_nt(aq, sa, wq, ws, d_ref)
    d = torch.empty_like(d_ref)
    lnq.lnq_fp8_block_gemm_nt_static_ws(aq, sa, wq, ws, d)
    torch.cuda.synchronize()
    assert torch.equal(d.view(torch.int16), d_ref.view(torch.int16))


def test_a_split_larger_than_the_array_is_rejected():
    M, N, K = 64, 16384, 4096
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert lnq.lnq_fp8_block_gemm_nt_workspace_bytes(M, N, K, sms) > STATIC_BYTES
    aq, sa, wq, ws = operands(M, N, K, seed=9)
    d = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(lnq.LnqError):
        lnq.lnq_fp8_block_gemm_nt_static_ws(aq, sa, wq, ws, d)
    assert lnq.lnq_get_last_device_error() == 0


def test_a_reported_timeout_leaves_the_array_usable():
    # lnq_get_last_device_error, on reporting a timeout, zeroes the tile counters of
    # the array (a split that gave up on a wait could have left some non-zero); the
    # timeout here comes from the self-test wait, so none is left, and the calls after
    # it must still give the workspace entry point's bytes
    M, N, K = 32, 12288, 4096
    aq, sa, wq, ws = operands(M, N, K, seed=11)
    work = lnq.gemm_workspace(M, N, K, DEV)
    d_ref = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    lnq.lnq_fp8_block_gemm_nt_ws(aq, sa, wq, ws, d_ref, work)
    d = torch.empty_like(d_ref)
    lnq.lnq_fp8_block_gemm_nt_static_ws(aq, sa, wq, ws, d)
    lnq.lnq_selftest_wait_timeout(5_000_000)
    assert lnq.lnq_get_last_device_error() == 6
    assert lnq.lnq_get_last_device_error() == 0
    for _ in range(2):
        d.fill_(float("nan"))
        lnq.lnq_fp8_block_gemm_nt_static_ws(aq, sa, wq, ws, d)
        torch.cuda.synchronize()
        assert lnq.lnq_get_last_device_error() == 0
        assert torch.equal(d.view(torch.int16), d_ref.view(torch.int16))
