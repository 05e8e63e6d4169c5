"""GPU parity of the gate_up linear with SiLU.mul fused into the epilogue.

h[m][j] = bf16( silu(D[m][j]) * D[m][I + j] ), the weight holding the I gate rows over
the I up rows (deepgemm-rust README, "What's implemented", moe_fp8_layer: grouped GEMM
-> SiLU.mul -> grouped GEMM).  Compared with the oracle's FP64 h within the GEMM
tolerance: the gate and up products carry the GEMM's FP32 error, silu is computed in
FP32, and h is rounded once to bf16.  Both schedules (CTA pairs for M > 128, single
CTAs) run every case; at the prefill size the whole of h is checked.
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


def run_gpu(a, w, pairs):
    M = a.shape[0]
    I = w.shape[0] // 2
    aq, sa = lnq.quantize_activations(a.to(DEV))
    wq, ws = lnq.quantize_weights(w.to(DEV))
    h = torch.full((M, I), float("nan"), dtype=torch.bfloat16, device=DEV)
    prev = lnq.lnq_set_dense_cta_pairs(pairs)
    try:
        lnq.lnq_fp8_block_gemm_nt_silu_mul(aq, sa, wq, ws, h)
    finally:
        lnq.lnq_set_dense_cta_pairs(prev)
    return h


@pytest.mark.parametrize("pairs", [0, 1])
@pytest.mark.parametrize("M,I,K", [(300, 256, 512), (129, 128, 256), (100, 384, 256), (8, 128, 1024),
                                   (1000, 512, 384), (1, 256, 128)])
def test_silu_mul_elementwise(M, I, K, pairs, store_path):
    a = synthetic.gaussian_bf16((M, K), 1.0, seed=M + I)
    w = synthetic.gaussian_bf16((2 * I, K), 0.05, seed=I + K)
    h = run_gpu(a, w, pairs)
    assert lnq.lnq_get_last_device_error() == 0
    qa, sa = oracle_quantize_a(a)
    qb, sb = oracle_quantize_w(w)
    ref = oracle.gemm_nt_silu_mul(qa, sa, qb, sb)
    assert_gemm_close(to_f64(h), ref, f"silu_mul {M}x{I}x{K} pairs={pairs}")


def test_gate_and_up_are_not_swapped():
    # gate products strongly negative (silu ~ 0) and up products large: swapped halves
    # would give silu(up) * gate, far from zero
    M, I, K = 256, 128, 256
    a = torch.ones((M, K), dtype=torch.bfloat16)
    w = torch.cat([torch.full((I, K), -0.5, dtype=torch.bfloat16),
                   torch.full((I, K), 0.25, dtype=torch.bfloat16)])
    h = to_f64(run_gpu(a, w, 1))
    qa, sa = oracle_quantize_a(a)
    qb, sb = oracle_quantize_w(w)
    ref = oracle.gemm_nt_silu_mul(qa, sa, qb, sb)     # silu(-128) * 64: about -2e-52
    assert np.all(np.abs(ref) < 1e-40)
    assert np.all(np.abs(h) < 1e-30)


def test_prefill_gate_up_full(store_path):
    # the prefill gate_up linear: M = 2048 tokens, I = 12288, K = 4096; h is compared
    # over the whole [M, I] output with silu(gate) * up of the full FP64 product
    cfg = synthetic.PREFILL[2]
    I = cfg.N // 2
    a, w = full_refs.linear_inputs(cfg.name)
    h = run_gpu(a, w, 1)
    assert lnq.lnq_get_last_device_error() == 0
    D = full_refs.linear_ref(cfg.name)
    ref = oracle.silu_mul(np.ascontiguousarray(D[:, :I]), np.ascontiguousarray(D[:, I:]))
    assert_gemm_close(to_f64(h), ref, "prefill gate_up silu_mul")
