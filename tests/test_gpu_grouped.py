"""GPU parity of the M-grouped contiguous GEMM against the oracle.

Layout (deepgemm-rust README, "Grouped (contiguous) MoE GEMM"; Triton_Grouped_GEMM
README, "Example DeepGEMM layout creation"): each group's rows start at a multiple
of 128, pad rows carry id -1.  Rows of real tokens are compared with the oracle
element by element (all of them at the MoE workload size); pad rows inside a block
are unspecified; blocks whose first row is -1 must not be written at all.
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


def make_inputs(sizes, N, K, seed):
    m_indices, starts, M_total = synthetic.contiguous_layout(sizes)
    G = len(sizes)
    a = synthetic.gaussian_bf16((M_total, K), 1.0, seed)
    a = a.masked_fill(torch.from_numpy(m_indices < 0).unsqueeze(1), 0.0)
    w = synthetic.gaussian_bf16((G * N, K), 0.02, seed + 1)
    return a, w, m_indices, G


def run_gpu(a, w, m_indices, G, fill=float("nan")):
    aq, sa = lnq.quantize_activations(a.to(DEV))
    wq, ws = lnq.quantize_weights_grouped(w.to(DEV), G)
    N = w.shape[0] // G
    d = torch.full((a.shape[0], N), fill, dtype=torch.bfloat16, device=DEV)
    lnq.lnq_m_grouped_fp8_gemm_contiguous(aq, sa, wq, ws, torch.from_numpy(m_indices).to(DEV), G, d)
    assert lnq.lnq_get_last_device_error() == 0
    return to_f64(d)


def oracle_quantize_w_grouped(w, G):
    """Each group's [N, K] weights quantized on their own (blocks never span groups)."""
    N = w.shape[0] // G
    parts = [oracle_quantize_w(w[g * N:(g + 1) * N]) for g in range(G)]
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])


def run_oracle(a, w, m_indices, G):
    qa, sa = oracle_quantize_a(a)
    qb, sb = oracle_quantize_w_grouped(w, G)
    return oracle.m_grouped_gemm_contiguous(qa, sa, qb, sb, m_indices, G)


@pytest.mark.parametrize("sizes,N,K", [
    ([5, 130, 0, 64, 250], 256, 384),
    ([128], 512, 256),
    ([1, 1, 1], 128, 128),
    ([300, 17], 384, 1024),
    ([64, 200, 129, 3], 48, 256),
])
def test_grouped_elementwise(sizes, N, K, store_path):
    a, w, m_indices, G = make_inputs(sizes, N, K, seed=sum(sizes) + N)
    d = run_gpu(a, w, m_indices, G)
    ref = run_oracle(a, w, m_indices, G)
    real = m_indices >= 0
    assert_gemm_close(d[real], ref[real], f"grouped {sizes} N={N} K={K}")


def test_blocks_led_by_a_pad_row_are_not_written(store_path):
    sizes = [130, 60]
    N, K = 256, 256
    a, w, m_indices, G = make_inputs(sizes, N, K, seed=3)
    m_indices = m_indices.copy()
    m_indices[128:256] = -1      # the block starting at row 128 now leads with -1
    d = run_gpu(a, w, m_indices, G, fill=7.0)
    assert np.all(d[128:256] == 7.0)
    ref = run_oracle(a, w, m_indices, G)
    real = m_indices >= 0
    assert_gemm_close(d[real], ref[real], "grouped with a skipped block")


def test_single_group_equals_dense():
    a = synthetic.gaussian_bf16((256, 512), 1.0, 11)
    w = synthetic.gaussian_bf16((256, 512), 0.02, 12)
    d = run_gpu(a, w, np.zeros(256, np.int32), 1)
    aq, sa = lnq.quantize_activations(a.to(DEV))
    wq, ws = lnq.quantize_weights(w.to(DEV))
    dd = torch.empty((256, 256), dtype=torch.bfloat16, device=DEV)
    lnq.lnq_fp8_block_gemm_nt(aq, sa, wq, ws, dd)
    assert np.array_equal(d, to_f64(dd))


def test_moe_workload_full(store_path):
    # every token row of the 32-expert MoE workload, element by element
    cfg = synthetic.MOE
    a, w, m_indices, _, _ = full_refs.moe_inputs()
    d = run_gpu(a, w, m_indices, cfg.groups)
    ref = full_refs.moe_ref()
    real = m_indices >= 0
    assert np.array_equal(real, ~np.isnan(ref[:, 0]))
    assert_gemm_close(d[real], ref[real], cfg.name)
    led_by_pad = np.repeat(m_indices[::128] < 0, 128)
    assert np.all(np.isnan(d[led_by_pad]))
