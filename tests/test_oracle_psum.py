"""Pins for the oracle's M-grouped contiguous product in the prefix-sum layout.

psum[g] counts the tokens of groups 0..g; group g's tokens start at an aligned row
of the A arena, the sum over earlier groups of their counts rounded up to the
alignment (deepgemm-rust README, "The mk_alignment knob (MoE tile width)", and the
psum-layout contiguous entry point of its device-level API).  Pinned against:

* hand-written layouts: for given counts and alignment the start rows are written
  out as literals, and an integer closed form (group g's weights all equal g + 1,
  unit scales) shows which group every row was computed with;
* per-group brute force with an independent decoder (torch float8_e4m3fn) and
  torch's float64 matmul;
* the contiguous oracle with per-row group ids;
* rejected prefix sums (decreasing, or groups that overrun the arena).
"""
import numpy as np
import pytest
import torch

import oracle

FINITE = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)


def torch_deq(codes: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64)


def operands(G, rows, N, K, seed):
    rng = np.random.default_rng(seed)
    qa = rng.choice(FINITE, size=(rows, K)).astype(np.uint8)
    qb = rng.choice(FINITE, size=(G * N, K)).astype(np.uint8)
    sfa = rng.uniform(0.001, 2.0, size=(K // 128, rows)).astype(np.float32)
    sfb = rng.uniform(0.001, 2.0, size=(G * -(-N // 128), K // 128)).astype(np.float32)
    return qa, sfa, qb, sfb


def closed_form_operands(G, rows, N, K, seed):
    # group g's weights are all the code of (g + 1), every scale is 1, so a row computed
    # with group g equals (g + 1) * (sum of its decoded A codes)
    ints = np.arange(-4, 5)
    codes = oracle.e4m3_encode(ints.astype(np.float32))
    ia = np.random.default_rng(seed).integers(0, len(ints), size=(rows, K))
    qb = np.concatenate([np.full((N, K), oracle.e4m3_encode(np.array([g + 1.0], np.float32))[0], np.uint8)
                         for g in range(G)])
    return codes[ia], np.ones((K // 128, rows), np.float32), qb, np.ones((G, K // 128), np.float32), ints[ia].sum(axis=1)


# counts, alignment, start rows written out by hand
LAYOUTS = [
    ([3, 0, 5], 4, [0, 4, 4]),
    ([4, 4, 1], 4, [0, 4, 8]),
    ([0, 0, 7], 8, [0, 0, 0]),
    ([9, 2, 8, 1], 8, [0, 16, 24, 32]),
    ([1, 1], 16, [0, 16]),
]


@pytest.mark.parametrize("counts,alignment,starts", LAYOUTS)
def test_hand_written_layouts(counts, alignment, starts):
    G, N, K = len(counts), 128, 256
    rows = 40
    qa, sfa, qb, sfb, rowsum = closed_form_operands(G, rows, N, K, seed=sum(counts))
    psum = np.cumsum(counts).astype(np.int32)
    D = oracle.m_grouped_gemm_psum(qa, sfa, qb, sfb, psum, alignment)
    owner = np.full(rows, -1)
    for g, (c, s) in enumerate(zip(counts, starts)):
        owner[s:s + c] = g
    for r in range(rows):
        if owner[r] < 0:
            assert np.all(np.isnan(D[r])), r
        else:
            assert np.all(D[r] == (owner[r] + 1) * rowsum[r]), r


@pytest.mark.parametrize("counts,alignment,N,K", [
    ([5, 0, 11], 8, 130, 256),
    ([16, 3], 16, 256, 384),
    ([1, 7, 2, 6], 4, 64, 128),
])
def test_per_group_brute_force(counts, alignment, N, K):
    G = len(counts)
    starts = np.concatenate([[0], np.cumsum([-(-c // alignment) * alignment for c in counts])[:-1]])
    rows = int(starts[-1] + -(-counts[-1] // alignment) * alignment) + 3
    qa, sfa, qb, sfb = operands(G, rows, N, K, seed=G * 31 + N)
    D = oracle.m_grouped_gemm_psum(qa, sfa, qb, sfb, np.cumsum(counts), alignment)
    NB = -(-N // 128)
    covered = np.zeros(rows, bool)
    for g, c in enumerate(counts):
        if c == 0:
            continue
        r0 = int(starts[g])
        sa = torch.from_numpy(sfa[:, r0:r0 + c].astype(np.float64)).T.repeat_interleave(128, dim=1)
        sb = torch.from_numpy(sfb[g * NB:(g + 1) * NB].astype(np.float64))
        sb = sb.repeat_interleave(128, dim=0)[:N].repeat_interleave(128, dim=1)
        ref = ((torch_deq(qa[r0:r0 + c]) * sa) @ (torch_deq(qb[g * N:(g + 1) * N]) * sb).T).numpy()
        np.testing.assert_allclose(D[r0:r0 + c], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
        covered[r0:r0 + c] = True
    assert np.all(np.isnan(D[~covered]))


def test_equals_the_contiguous_product_with_matching_group_ids():
    counts, alignment = [130, 0, 256, 7], 128
    G, N, K = len(counts), 256, 256
    rows = 128 * 2 + 256 + 128
    qa, sfa, qb, sfb = operands(G, rows, N, K, seed=41)
    m_indices = np.full(rows, -1, np.int32)
    m_indices[0:130] = 0
    m_indices[256:512] = 2
    m_indices[512:519] = 3
    D = oracle.m_grouped_gemm_psum(qa, sfa, qb, sfb, np.cumsum(counts), alignment)
    Dc = oracle.m_grouped_gemm_contiguous(qa, sfa, qb, sfb, m_indices, G)
    assert np.array_equal(np.isnan(D), np.isnan(Dc))
    assert np.array_equal(D[~np.isnan(D)], Dc[~np.isnan(Dc)])


def test_bad_prefix_sums_are_rejected():
    G, N, K, rows = 2, 128, 128, 16
    qa, sfa, qb, sfb = operands(G, rows, N, K, seed=43)
    with pytest.raises(ValueError):          # decreasing
        oracle.m_grouped_gemm_psum(qa, sfa, qb, sfb, [5, 3], 4)
    with pytest.raises(ValueError):          # 9 -> 12 rows, then 5 more: 17 > 16
        oracle.m_grouped_gemm_psum(qa, sfa, qb, sfb, [9, 14], 4)
    D = oracle.m_grouped_gemm_psum(qa, sfa, qb, sfb, [9, 13], 4)   # exactly 16 rows
    assert not np.isnan(D[15]).any() and np.isnan(D[9:12]).all()
