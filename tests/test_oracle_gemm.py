"""Pins for the oracle's block-scaled product and its M-grouped contiguous variant.

The product is D[m,n] = sum_k (v(qa[m,k]) * sfa[k/128][m]) * (v(qb[n,k]) * sfb[n/128][k/128]),
with sfa stored column by column over padded rows (MN-major) and sfb as
(ceil(N/128), K/128) row-major (deepgemm-rust README, "Quick start" and
"What's implemented"; Linnet plugin docstring).  Pinned against:

* brute force with an independent decoder (torch float8_e4m3fn) and torch's
  float64 matmul on small ragged shapes;
* exact integer closed forms (all codes small integers, unit scales);
* a scale-only closed form that pins the MN-major sfa index and the
  [n/128][k/128] sfb index (shapes chosen so that a swapped index fails);
* the grouped variant: closed forms per expert, untouched -1 rows, and equality
  with a per-segment torch float64 product.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_quantize_b200 import synthetic

FINITE = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)


def torch_deq(codes: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64)


def torch_reference(qa, sfa, qb, sfb, M):
    """float64 (deq(qa) * Sa) @ (deq(qb) * Sb)^T with the scales expanded by broadcasting."""
    K = qa.shape[1]
    N = qb.shape[0]
    sa = torch.from_numpy(sfa[:, :M].astype(np.float64)).T                      # [M, K/128]
    sa = sa.repeat_interleave(128, dim=1)                                      # [M, K]
    sb = torch.from_numpy(sfb.astype(np.float64))                             # [NB, K/128]
    sb = sb.repeat_interleave(128, dim=0)[:N].repeat_interleave(128, dim=1)   # [N, K]
    A = torch_deq(qa) * sa
    B = torch_deq(qb) * sb
    return (A @ B.T).numpy()


def random_operands(M, N, K, seed):
    rng = np.random.default_rng(seed)
    M4 = -(-M // 4) * 4
    qa = rng.choice(FINITE, size=(M, K)).astype(np.uint8)
    qb = rng.choice(FINITE, size=(N, K)).astype(np.uint8)
    sfa = rng.uniform(0.001, 2.0, size=(K // 128, M4)).astype(np.float32)
    sfa[:, M:] = 0.0
    sfb = rng.uniform(0.001, 2.0, size=(-(-N // 128), K // 128)).astype(np.float32)
    return qa, sfa, qb, sfb


@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (3, 8, 256), (8, 16, 384), (16, 130, 128),
                                   (130, 7, 256), (5, 257, 512)])
def test_brute_force_against_torch(M, N, K):
    qa, sfa, qb, sfb = random_operands(M, N, K, seed=M * 1000 + N * 10 + K)
    D = oracle.gemm_nt(qa, sfa, qb, sfb)
    ref = torch_reference(qa, sfa, qb, sfb, M)
    assert D.shape == (M, N)
    np.testing.assert_allclose(D, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_integer_closed_form():
    # codes of the integers -15..15 with unit scales: D is the exact integer product
    ints = np.arange(-15, 16)
    codes = oracle.e4m3_encode(ints.astype(np.float32))
    assert np.array_equal(oracle.e4m3_value(codes), ints)
    rng = np.random.default_rng(7)
    M, N, K = 9, 33, 384
    ia = rng.integers(0, len(ints), size=(M, K))
    ib = rng.integers(0, len(ints), size=(N, K))
    qa, qb = codes[ia], codes[ib]
    sfa = np.ones((K // 128, 12), np.float32)
    sfb = np.ones((1, K // 128), np.float32)
    D = oracle.gemm_nt(qa, sfa, qb, sfb)
    exact = ints[ia].astype(np.int64) @ ints[ib].astype(np.int64).T
    assert np.array_equal(D, exact.astype(np.float64))


def test_scale_indexing_closed_form():
    # every code 1.0: D[m,n] = 128 * sum_g sfa[g][m] * sfb[n/128][g]
    M, N, K = 6, 384, 640          # M4 = 8, K/128 = 5, N/128 = 3: no two index spaces coincide
    one = np.uint8(0x38)
    qa = np.full((M, K), one, np.uint8)
    qb = np.full((N, K), one, np.uint8)
    rng = np.random.default_rng(8)
    sfa = np.exp2(rng.integers(-6, 6, size=(K // 128, 8))).astype(np.float32)
    sfa[:, M:] = 0
    sfb = np.exp2(rng.integers(-6, 6, size=(N // 128, K // 128))).astype(np.float32)
    D = oracle.gemm_nt(qa, sfa, qb, sfb)
    for m in range(M):
        for n in range(N):
            want = 128.0 * sum(float(sfa[g, m]) * float(sfb[n // 128, g]) for g in range(K // 128))
            assert D[m, n] == want


def test_operands_are_not_transposed():
    # A has a single non-zero column k0; B a single non-zero row n0: D is non-zero only
    # in column n0, with value v(qa[m,k0]) * v(qb[n0,k0])
    M, N, K = 4, 256, 256
    qa = np.zeros((M, K), np.uint8)
    qb = np.zeros((N, K), np.uint8)
    qa[:, 131] = oracle.e4m3_encode(np.array([1, 2, 3, 4], np.float32))
    qb[77, 131] = oracle.e4m3_encode(np.array([5.0], np.float32))[0]
    D = oracle.gemm_nt(qa, np.ones((2, 4), np.float32), qb, np.ones((2, 2), np.float32))
    want = np.zeros((M, N))
    want[:, 77] = [5, 10, 15, 20]
    assert np.array_equal(D, want)


def test_points_agree_with_full_product():
    qa, sfa, qb, sfb = random_operands(33, 260, 384, seed=9)
    D = oracle.gemm_nt(qa, sfa, qb, sfb)
    rng = np.random.default_rng(10)
    rows = rng.integers(0, 33, 500)
    cols = rng.integers(0, 260, 500)
    assert np.array_equal(oracle.gemm_nt_points(qa, sfa, qb, sfb, rows, cols), D[rows, cols])


def test_end_to_end_tiny_against_unquantized():
    # quantize A (1x128) and W (128x128), multiply: close to the bf16 product (the
    # pages report a few percent relative error for FP8 linears against bf16)
    a = synthetic.gaussian_bf16((64, 512), 1.0, 0)
    w = synthetic.gaussian_bf16((256, 512), 0.02, 1)
    qa, sfa = oracle.quantize_fp8_groups(synthetic.bf16_bits(a))
    qb, sfb = oracle.quantize_fp8_blocks(synthetic.bf16_bits(w))
    D = oracle.gemm_nt(qa, sfa, qb, sfb)
    ref = (a.to(torch.float64) @ w.to(torch.float64).T).numpy()
    rel = np.linalg.norm(D - ref) / np.linalg.norm(ref)
    assert 1e-3 < rel < 0.08


# ---------------------------------------------------------------- grouped

def grouped_operands(sizes, N, K, seed):
    m_indices, starts, M_total = synthetic.contiguous_layout(sizes)
    G = len(sizes)
    rng = np.random.default_rng(seed)
    qa = rng.choice(FINITE, size=(M_total, K)).astype(np.uint8)
    qb = rng.choice(FINITE, size=(G * N, K)).astype(np.uint8)
    sfa = rng.uniform(0.01, 1.0, size=(K // 128, M_total)).astype(np.float32)
    NB = -(-N // 128)
    sfb = rng.uniform(0.01, 1.0, size=(G * NB, K // 128)).astype(np.float32)
    return m_indices, starts, qa, sfa, qb, sfb


def test_layout_helper():
    m_indices, starts, M_total = synthetic.contiguous_layout([3, 0, 130, 128])
    assert M_total == 128 + 0 + 256 + 128
    assert list(starts) == [0, 128, 128, 384]
    assert np.all(m_indices[:3] == 0) and np.all(m_indices[3:128] == -1)
    assert np.all(m_indices[128:258] == 2) and np.all(m_indices[258:384] == -1)
    assert np.all(m_indices[384:] == 3)


def test_grouped_against_per_segment_torch():
    sizes = [5, 130, 0, 64]
    N, K = 256, 384
    m_indices, starts, qa, sfa, qb, sfb = grouped_operands(sizes, N, K, seed=11)
    G = len(sizes)
    D = oracle.m_grouped_gemm_contiguous(qa, sfa, qb, sfb, m_indices, G)
    NB = N // 128
    for g, (s, n) in enumerate(zip(starts, sizes)):
        if n == 0:
            continue
        ref = torch_reference(qa[s:s + n], np.ascontiguousarray(sfa[:, s:s + n]),
                              qb[g * N:(g + 1) * N], sfb[g * NB:(g + 1) * NB], n)
        np.testing.assert_allclose(D[s:s + n], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    assert np.all(np.isnan(D[m_indices < 0]))


def test_grouped_closed_form_per_expert():
    # expert g's weights are all the code of (g+1) with unit scales, so
    # D[m, n] = (g+1) * sum_k v(qa[m,k]) for a row of group g
    sizes = [128, 1, 200]
    N, K = 128, 256
    m_indices, starts, M_total = synthetic.contiguous_layout(sizes)
    G = len(sizes)
    rng = np.random.default_rng(12)
    ints = np.arange(-4, 5)
    codes = oracle.e4m3_encode(ints.astype(np.float32))
    ia = rng.integers(0, len(ints), size=(M_total, K))
    qa = codes[ia]
    qb = np.concatenate([np.full((N, K), oracle.e4m3_encode(np.array([g + 1.0], np.float32))[0],
                                 np.uint8) for g in range(G)])
    sfa = np.ones((K // 128, M_total), np.float32)
    sfb = np.ones((G, K // 128), np.float32)
    D = oracle.m_grouped_gemm_contiguous(qa, sfa, qb, sfb, m_indices, G)
    rowsum = ints[ia].sum(axis=1)
    for m in range(M_total):
        g = m_indices[m]
        if g >= 0:
            assert np.all(D[m] == (g + 1) * rowsum[m])
        else:
            assert np.all(np.isnan(D[m]))


def test_grouped_single_group_is_dense():
    qa, sfa, qb, sfb = random_operands(256, 128, 256, seed=13)
    D = oracle.m_grouped_gemm_contiguous(qa, sfa, qb, sfb, np.zeros(256, np.int32), 1)
    ref = torch_reference(qa, sfa, qb, sfb, 256)
    np.testing.assert_allclose(D, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_grouped_points_agree():
    sizes = [70, 129]
    N, K = 256, 256
    m_indices, starts, qa, sfa, qb, sfb = grouped_operands(sizes, N, K, seed=14)
    D = oracle.m_grouped_gemm_contiguous(qa, sfa, qb, sfb, m_indices, 2)
    rows = np.nonzero(m_indices >= 0)[0][::7]
    cols = (rows * 13) % N
    pts = oracle.m_grouped_gemm_points(qa, sfa, qb, sfb, m_indices, 2, rows, cols)
    assert np.array_equal(pts, D[rows, cols])
