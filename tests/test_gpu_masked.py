"""GPU parity of the M-grouped masked GEMM against the oracle.

Layout (deepgemm-rust README, "What's implemented", m_grouped_fp8_gemm_nt_masked):
every group has a buffer of M_max rows of which the first masked_m[g] hold tokens;
the counts stay on the device.  Rows of real tokens are compared with the oracle
element by element (all of them at the workload size); the other rows of
D must keep what was there before the call.  The rows past a count hold random
values, which must not reach any real row.
"""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_quantize_b200 as lnq
import oracle
from moe_grouped_gemm_quantize_b200 import synthetic
import full_refs
from parity import assert_gemm_close, oracle_quantize_a, oracle_quantize_w, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def oracle_quantize_w_grouped(w, G):
    N = w.shape[0] // G
    parts = [oracle_quantize_w(w[g * N:(g + 1) * N]) for g in range(G)]
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])


def make_inputs(G, M_max, N, K, seed):
    a = synthetic.gaussian_bf16((G * M_max, K), 1.0, seed)
    w = synthetic.gaussian_bf16((G * N, K), 0.02, seed + 1)
    return a, w


def run_gpu(a, w, masked, M_max, expected_m=0):
    G = len(masked)
    N = w.shape[0] // G
    aq, sa = lnq.quantize_activations(a.to(DEV))
    wq, ws = lnq.quantize_weights_grouped(w.to(DEV), G)
    d = torch.full((G * M_max, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    mm = torch.tensor(masked, dtype=torch.int32, device=DEV)
    lnq.lnq_m_grouped_fp8_gemm_masked(aq, sa, wq, ws, mm, d, expected_m)
    return d


@pytest.mark.parametrize("masked,M_max,N,K", [
    ([77], 128, 256, 256),
    ([256, 0, 129, 1], 256, 256, 512),
    ([128, 64, 0, 127, 5, 100, 128, 33], 128, 384, 256),
    ([200, 17], 256, 128, 1024),
    ([3, 128, 90], 128, 48, 256),
])
def test_masked_elementwise(masked, M_max, N, K, store_path):
    G = len(masked)
    a, w = make_inputs(G, M_max, N, K, seed=G * 10 + N)
    d = run_gpu(a, w, masked, M_max)
    assert lnq.lnq_get_last_device_error() == 0
    qa, sa = oracle_quantize_a(a)
    qb, sb = oracle_quantize_w_grouped(w, G)
    ref = oracle.m_grouped_gemm_masked(qa, sa, qb, sb, masked, M_max)
    got = to_f64(d)
    valid = ~np.isnan(ref[:, 0])
    if valid.any():
        assert_gemm_close(got[valid], ref[valid], f"masked G={G} M_max={M_max} {N}x{K}")
    # rows past each count are untouched
    assert np.all(np.isnan(got[~valid]))


def test_decode_moe_workload_full(store_path):
    # 32 experts with 128-row buffers, 2048 routed tokens (multinomial, seed 3): every
    # token row is compared, each group's rows with the dense oracle product of its
    # weights (the definition of the masked product)
    G, M_max, N, K = 32, 128, 4096, 7168
    counts = np.minimum(np.random.default_rng(3).multinomial(2048, [1.0 / G] * G), M_max)
    masked = [int(c) for c in counts]
    a, w = make_inputs(G, M_max, N, K, seed=71)
    d = run_gpu(a, w, masked, M_max, expected_m=64)
    assert lnq.lnq_get_last_device_error() == 0
    qa, sa = oracle_quantize_a(a)
    qb, sb = oracle_quantize_w_grouped(w, G)
    starts = np.arange(G) * M_max
    ref = full_refs.grouped_ref(qa, sa, qb, sb, starts, masked, N)
    real = np.concatenate([np.arange(g * M_max, g * M_max + c) for g, c in enumerate(masked)])
    got = to_f64(d)
    assert_gemm_close(got[real], ref[real], "masked decode MoE")
    pad = np.setdiff1d(np.arange(G * M_max), real)
    assert np.all(np.isnan(got[pad]))


def test_count_out_of_range_is_reported_and_clamped():
    G, M_max, N, K = 2, 128, 256, 256
    a, w = make_inputs(G, M_max, N, K, seed=81)
    d = run_gpu(a, w, [M_max + 5, 40], M_max)
    assert lnq.lnq_get_last_device_error() == 1          # LNQ_ERR_INVALID_ARG
    assert lnq.lnq_get_last_device_error() == 0
    qa, sa = oracle_quantize_a(a)
    qb, sb = oracle_quantize_w_grouped(w, G)
    ref = oracle.m_grouped_gemm_masked(qa, sa, qb, sb, [M_max, 40], M_max)
    got = to_f64(d)
    valid = ~np.isnan(ref[:, 0])
    assert_gemm_close(got[valid], ref[valid], "clamped count")
    assert np.all(np.isnan(got[~valid]))


def test_full_counts_equal_the_contiguous_product():
    # every row real: the masked and contiguous kernels compute the same products
    G, M_max, N, K = 3, 128, 256, 512
    a, w = make_inputs(G, M_max, N, K, seed=91)
    d = run_gpu(a, w, [M_max] * G, M_max)
    aq, sa = lnq.quantize_activations(a.to(DEV))
    wq, ws = lnq.quantize_weights_grouped(w.to(DEV), G)
    mi = torch.arange(G, dtype=torch.int32, device=DEV).repeat_interleave(M_max)
    d2 = torch.empty_like(d)
    lnq.lnq_m_grouped_fp8_gemm_contiguous(aq, sa, wq, ws, mi, G, d2)
    torch.cuda.synchronize()
    assert lnq.lnq_get_last_device_error() == 0
    assert torch.equal(d.view(torch.int16), d2.view(torch.int16))
