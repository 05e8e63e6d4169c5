"""The whole-matrix references of the GPU tests (full_refs) against the oracle's own
grouped functions, on small layouts: the loop of dense products per group gives the
same FP64 values as the grouped oracle on token rows, and NaN elsewhere."""
import numpy as np

import full_refs
import oracle
from moe_grouped_gemm_quantize_b200 import synthetic
from parity import oracle_quantize_a


def test_grouped_ref_equals_the_contiguous_oracle():
    sizes, N, K = [5, 130, 0, 64, 250], 256, 384
    G = len(sizes)
    m_indices, starts, M_total = synthetic.contiguous_layout(sizes)
    a = synthetic.gaussian_bf16((M_total, K), 1.0, 3)
    w = synthetic.gaussian_bf16((G * N, K), 0.02, 4)
    qa, sa = oracle_quantize_a(a)
    qb, sb = full_refs.grouped_weights(w, G)
    ref = full_refs.grouped_ref(qa, sa, qb, sb, starts, sizes, N)
    want = oracle.m_grouped_gemm_contiguous(qa, sa, qb, sb, m_indices, G)
    real = m_indices >= 0
    assert np.array_equal(np.isnan(ref[:, 0]), ~real)
    assert np.array_equal(ref[real], want[real])


def test_grouped_ref_equals_the_masked_oracle():
    G, M_max, N, K = 3, 128, 128, 256
    masked = [77, 0, 128]
    a = synthetic.gaussian_bf16((G * M_max, K), 1.0, 5)
    w = synthetic.gaussian_bf16((G * N, K), 0.02, 6)
    qa, sa = oracle_quantize_a(a)
    qb, sb = full_refs.grouped_weights(w, G)
    ref = full_refs.grouped_ref(qa, sa, qb, sb, np.arange(G) * M_max, masked, N)
    want = oracle.m_grouped_gemm_masked(qa, sa, qb, sb, masked, M_max)
    assert np.array_equal(np.isnan(ref), np.isnan(want))
    v = ~np.isnan(want)
    assert np.array_equal(ref[v], want[v])
