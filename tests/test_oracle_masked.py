"""Pins for the oracle's M-grouped masked product.

Group g owns rows g*M_max .. g*M_max + M_max - 1 of A and D, of which only the first
masked_m[g] are computed; the weights and scales are laid out as in the contiguous
variant (deepgemm-rust README, "What's implemented", m_grouped_fp8_gemm_nt_masked).
Pinned against:

* per-group brute force with an independent decoder (torch float8_e4m3fn) and
  torch's float64 matmul;
* an exact closed form per group (integer codes, unit scales), which fails on a
  wrong group stride of A, of the weights or of the weight scales;
* the contiguous oracle, written separately, with the equivalent per-row group ids;
* counts of 0 and M_max, untouched rows past each count, and rejected counts.
"""
import numpy as np
import pytest
import torch

import oracle

FINITE = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)


def torch_deq(codes: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64)


def masked_operands(G, M_max, N, K, seed):
    rng = np.random.default_rng(seed)
    rows = G * M_max
    qa = rng.choice(FINITE, size=(rows, K)).astype(np.uint8)
    qb = rng.choice(FINITE, size=(G * N, K)).astype(np.uint8)
    sfa = rng.uniform(0.001, 2.0, size=(K // 128, rows)).astype(np.float32)
    sfb = rng.uniform(0.001, 2.0, size=(G * -(-N // 128), K // 128)).astype(np.float32)
    return qa, sfa, qb, sfb


def torch_group(qa, sfa, qb, sfb, g, M_max, n_rows, N, K):
    NB = -(-N // 128)
    r0 = g * M_max
    sa = torch.from_numpy(sfa[:, r0:r0 + n_rows].astype(np.float64)).T.repeat_interleave(128, dim=1)
    sb = torch.from_numpy(sfb[g * NB:(g + 1) * NB].astype(np.float64))
    sb = sb.repeat_interleave(128, dim=0)[:N].repeat_interleave(128, dim=1)
    A = torch_deq(qa[r0:r0 + n_rows]) * sa
    B = torch_deq(qb[g * N:(g + 1) * N]) * sb
    return (A @ B.T).numpy()


@pytest.mark.parametrize("G,M_max,N,K,masked", [
    (1, 8, 16, 128, [5]),
    (3, 16, 130, 256, [16, 0, 7]),
    (4, 12, 256, 384, [1, 12, 3, 9]),
])
def test_per_group_brute_force(G, M_max, N, K, masked):
    qa, sfa, qb, sfb = masked_operands(G, M_max, N, K, seed=G * 100 + M_max)
    D = oracle.m_grouped_gemm_masked(qa, sfa, qb, sfb, masked, M_max)
    assert D.shape == (G * M_max, N)
    for g in range(G):
        r0, n = g * M_max, masked[g]
        if n:
            ref = torch_group(qa, sfa, qb, sfb, g, M_max, n, N, K)
            np.testing.assert_allclose(D[r0:r0 + n], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
        assert np.all(np.isnan(D[r0 + n:r0 + M_max]))


def test_closed_form_per_group():
    # group g's weights are all the code of (g + 1), every scale is 1:
    # D[g*M_max + m, n] = (g + 1) * sum_k v(qa[g*M_max + m, k]) for m < masked[g]
    G, M_max, N, K = 3, 10, 128, 256
    masked = [10, 4, 7]
    ints = np.arange(-4, 5)
    codes = oracle.e4m3_encode(ints.astype(np.float32))
    rng = np.random.default_rng(7)
    ia = rng.integers(0, len(ints), size=(G * M_max, K))
    qa = codes[ia]
    qb = np.concatenate([np.full((N, K), oracle.e4m3_encode(np.array([g + 1.0], np.float32))[0], np.uint8)
                         for g in range(G)])
    sfa = np.ones((K // 128, G * M_max), np.float32)
    sfb = np.ones((G, K // 128), np.float32)
    D = oracle.m_grouped_gemm_masked(qa, sfa, qb, sfb, masked, M_max)
    rowsum = ints[ia].sum(axis=1)
    for g in range(G):
        for m in range(M_max):
            r = g * M_max + m
            if m < masked[g]:
                assert np.all(D[r] == (g + 1) * rowsum[r])
            else:
                assert np.all(np.isnan(D[r]))


def test_equals_the_contiguous_product_with_matching_group_ids():
    G, M_max, N, K = 4, 128, 256, 256
    masked = [128, 0, 77, 1]
    qa, sfa, qb, sfb = masked_operands(G, M_max, N, K, seed=21)
    m_indices = np.full(G * M_max, -1, np.int32)
    for g, n in enumerate(masked):
        m_indices[g * M_max:g * M_max + n] = g
    D = oracle.m_grouped_gemm_masked(qa, sfa, qb, sfb, masked, M_max)
    Dc = oracle.m_grouped_gemm_contiguous(qa, sfa, qb, sfb, m_indices, G)
    assert np.array_equal(np.isnan(D), np.isnan(Dc))
    valid = ~np.isnan(D)
    assert np.array_equal(D[valid], Dc[valid])


def test_points_agree_and_counts_are_checked():
    G, M_max, N, K = 2, 20, 140, 128
    masked = [13, 20]
    qa, sfa, qb, sfb = masked_operands(G, M_max, N, K, seed=22)
    D = oracle.m_grouped_gemm_masked(qa, sfa, qb, sfb, masked, M_max)
    rows = np.arange(0, G * M_max, 3)
    cols = (rows * 7) % N
    pts = oracle.m_grouped_gemm_masked_points(qa, sfa, qb, sfb, masked, M_max, rows, cols)
    ref = D[rows, cols]
    assert np.array_equal(np.isnan(pts), np.isnan(ref))
    assert np.array_equal(pts[~np.isnan(ref)], ref[~np.isnan(ref)])
    for bad in ([21, 0], [-1, 3]):
        with pytest.raises(ValueError):
            oracle.m_grouped_gemm_masked(qa, sfa, qb, sfb, bad, M_max)
