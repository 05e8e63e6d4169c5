"""GPU parity of the block-scaled recipes in the M-grouped masked layout.

deepgemm-rust README, "What's implemented" (the masked_m scheduler of the DeepEP-style
dispatch output, zero CPU sync) and "Full recipes" (gran-32 and gran-128 on either side):
group g owns rows g*M_max .. g*M_max + M_max - 1 of A and D, of which the first
masked_m[g] are tokens.  Each group's token rows are compared, element by element, with the
oracle's FP64 product of the same codes and scales against that group's weights (the
UE8M0 gran-128 and the MXFP8 gran-32 recipe); rows past each count must stay untouched
(D is filled with NaN before the call).  Counts 0, 1, ragged and M_max are covered, a count
outside 0 .. M_max is clamped and reported, and the decode-time masked MoE workload (32
expert buffers of 128 rows) is compared in full.
"""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_quantize_b200 as lnq
import oracle
from moe_grouped_gemm_quantize_b200 import synthetic
from parity import assert_gemm_close, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def quantize(recipe, a, w):
    if recipe == "mxfp8":
        return lnq.quantize_mxfp8(a.to(DEV)), lnq.quantize_mxfp8(w.to(DEV))
    return lnq.quantize_activations_ue8m0(a.to(DEV)), lnq.quantize_weights_ue8m0(w.to(DEV))


def oracle_rows(recipe, a, w):
    """FP64 product of every row of a with every row of w under the recipe (rows of a
    quantized on their own, so per-row results do not depend on the other rows)."""
    if recipe == "mxfp8":
        qa, ea = oracle.quantize_mxfp8(synthetic.bf16_bits(a))
        qb, eb = oracle.quantize_mxfp8(synthetic.bf16_bits(w))
        return oracle.gemm_nt_mx32(qa, ea, qb, eb)
    qa, ea = oracle.quantize_ue8m0_groups(synthetic.bf16_bits(a))
    qb, eb = oracle.quantize_ue8m0_blocks(synthetic.bf16_bits(w))
    return oracle.gemm_nt(qa, oracle.ue8m0_value(ea), qb, oracle.ue8m0_value(eb))


def run_masked(recipe, a, w, counts, G, expected_m=0):
    (aq, sa), (wq, sw) = quantize(recipe, a, w)
    N = w.shape[0] // G
    d = torch.full((a.shape[0], N), float("nan"), dtype=torch.bfloat16, device=DEV)
    mm = torch.tensor(counts, dtype=torch.int32, device=DEV)
    fn = lnq.lnq_m_grouped_mxfp8_gemm_masked if recipe == "mxfp8" else lnq.lnq_m_grouped_mx_gemm_masked
    fn(aq, sa, wq, sw, mm, d, expected_m)
    return d


def check_groups(recipe, a, w, counts, G, M_max, d, what):
    N = w.shape[0] // G
    got = to_f64(d)
    for g, c in enumerate(counts):
        c = max(0, min(int(c), M_max))
        rows = slice(g * M_max, g * M_max + c)
        if c:
            ref = oracle_rows(recipe, a[rows], w[g * N:(g + 1) * N])
            assert_gemm_close(got[rows], ref, f"{what} group {g} ({c} rows)")
        assert np.all(np.isnan(got[g * M_max + c:(g + 1) * M_max])), f"{what}: rows past group {g}'s count written"


@pytest.mark.parametrize("recipe", ["ue8m0", "mxfp8"])
@pytest.mark.parametrize("counts,M_max,N,K", [
    ([0, 1, 130, 256], 256, 256, 512),
    ([128, 5, 64], 128, 384, 256),
    ([300, 0, 17], 384, 128, 1024),
])
def test_masked_layouts(recipe, counts, M_max, N, K):
    G = len(counts)
    a = synthetic.gaussian_bf16_with_outliers((G * M_max, K), 1.0, M_max + K, 5, frac=0.05)
    w = synthetic.gaussian_bf16((G * N, K), 0.02, seed=N + K + G)
    d = run_masked(recipe, a, w, counts, G, expected_m=sum(counts) // G)
    assert lnq.lnq_get_last_device_error() == 0
    check_groups(recipe, a, w, counts, G, M_max, d, f"{recipe} masked {counts}")


@pytest.mark.parametrize("recipe", ["ue8m0", "mxfp8"])
def test_count_past_the_buffer_is_clamped_and_reported(recipe):
    G, M_max, N, K = 2, 128, 256, 256
    counts = [200, 40]
    a = synthetic.gaussian_bf16((G * M_max, K), 1.0, seed=7)
    w = synthetic.gaussian_bf16((G * N, K), 0.02, seed=8)
    d = run_masked(recipe, a, w, counts, G)
    assert lnq.lnq_get_last_device_error() == 1          # LNQ_ERR_INVALID_ARG
    check_groups(recipe, a, w, [M_max, 40], G, M_max, d, f"{recipe} clamped count")


@pytest.mark.parametrize("recipe", ["ue8m0", "mxfp8"])
def test_masked_moe_workload_full(recipe):
    cfg = synthetic.MOE_MASKED
    a, w, counts = synthetic.make_moe_masked_inputs(cfg)
    d = run_masked(recipe, a, w, list(counts), cfg.groups, expected_m=cfg.tokens // cfg.groups)
    assert lnq.lnq_get_last_device_error() == 0
    check_groups(recipe, a, w, list(counts), cfg.groups, cfg.m_max, d, f"{recipe} masked MoE workload")
