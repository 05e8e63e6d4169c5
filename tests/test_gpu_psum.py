"""GPU parity of the M-grouped contiguous GEMM in the prefix-sum layout.

psum[g] counts the tokens of groups 0..g on the device; group g's tokens start at the
sum of the earlier groups' counts rounded up to the alignment (deepgemm-rust README,
"The mk_alignment knob (MoE tile width)", and its psum-layout contiguous entry point).
Tiles are 128 rows, those of pad rows only skipped; with alignment 256, N >= 256 and
the grouped pairs knob set, 256 x 256 tiles on CTA pairs.  Both schedules run every
case.  Token rows are compared with the oracle element by element (all of them at the
workload size); pad rows and rows past the last group must keep what was there
before the call.
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


def run_gpu(a, w, psum, alignment, G, pairs=0):
    N = w.shape[0] // G
    aq, sa = lnq.quantize_activations(a.to(DEV))
    wq, ws = lnq.quantize_weights_grouped(w.to(DEV), G)
    d = torch.full((a.shape[0], N), float("nan"), dtype=torch.bfloat16, device=DEV)
    ps = torch.tensor(np.asarray(psum, dtype=np.int32), device=DEV)
    prev = lnq.lnq_set_grouped_cta_pairs(pairs)
    try:
        lnq.lnq_m_grouped_fp8_gemm_contiguous_psum(aq, sa, wq, ws, ps, d, alignment)
    finally:
        lnq.lnq_set_grouped_cta_pairs(prev)
    return d


def token_rows(sizes, starts):
    return np.concatenate([np.arange(s, s + n) for s, n in zip(starts, sizes)] + [np.zeros(0, np.int64)])


CASES = [
    # sizes, alignment, N, K, extra arena rows
    ([300, 0, 256, 17], 256, 256, 512, 0),      # a pair's second CTA (a 128-row tile) without tokens
    ([1], 256, 512, 256, 256),                  # one token, a tile past the last group
    ([257, 511, 3], 256, 768, 384, 0),          # three pair tiles per row band
    ([129, 128, 255, 1, 0, 513], 128, 384, 256, 128),  # 128-row tiles, ragged N tile
    ([200, 90], 256, 128, 1024, 0),             # N < 256: single-CTA 128-column tiles
    ([40, 600], 256, 272, 256, 0),              # N ragged inside the pair's second half
    # more groups than a warp's lanes: the lookup walks several runs of 32 groups
    ([int(x) for x in np.random.default_rng(40).integers(0, 300, 40)], 128, 256, 256, 0),
    ([int(x) for x in np.random.default_rng(70).integers(0, 200, 70)], 256, 256, 128, 256),
]


@pytest.mark.parametrize("pairs", [0, 1])
@pytest.mark.parametrize("sizes,alignment,N,K,extra", CASES)
def test_psum_elementwise(sizes, alignment, N, K, extra, pairs, store_path):
    G = len(sizes)
    psum, starts, M_total = synthetic.psum_layout(sizes, alignment)
    M_total += extra
    a = synthetic.gaussian_bf16((M_total, K), 1.0, seed=G * 7 + N)
    w = synthetic.gaussian_bf16((G * N, K), 0.02, seed=K + N)
    d = run_gpu(a, w, psum, alignment, G, pairs)
    assert lnq.lnq_get_last_device_error() == 0
    qa, sa = oracle_quantize_a(a)
    qb, sb = oracle_quantize_w_grouped(w, G)
    ref = oracle.m_grouped_gemm_psum(qa, sa, qb, sb, psum, alignment)
    got = to_f64(d)
    valid = ~np.isnan(ref[:, 0])
    assert np.array_equal(np.flatnonzero(valid), token_rows(sizes, starts))
    assert_gemm_close(got[valid], ref[valid], f"psum {sizes} align {alignment} {N}x{K}")
    assert np.all(np.isnan(got[~valid]))


def test_pairs_and_single_ctas_agree():
    sizes, alignment, N, K = [300, 700, 0, 256], 256, 512, 512
    G = len(sizes)
    psum, _, M_total = synthetic.psum_layout(sizes, alignment)
    a = synthetic.gaussian_bf16((M_total, K), 1.0, seed=3)
    w = synthetic.gaussian_bf16((G * N, K), 0.02, seed=4)
    d_pair = run_gpu(a, w, psum, alignment, G, pairs=1)
    d_one = run_gpu(a, w, psum, alignment, G, pairs=0)
    assert lnq.lnq_get_last_device_error() == 0
    x, y = to_f64(d_pair), to_f64(d_one)
    assert np.array_equal(np.isnan(x), np.isnan(y))
    v = ~np.isnan(x)
    assert_gemm_close(x[v], y[v], "pair vs single")


def test_128_alignment_matches_the_group_id_layout_bit_for_bit():
    # same tiles and groups as the per-row id layout: the same kernel schedule
    sizes, N, K = [130, 0, 256, 7, 128], 256, 512
    G = len(sizes)
    psum, starts, M_total = synthetic.psum_layout(sizes, 128)
    m_indices, starts2, M2 = synthetic.contiguous_layout(sizes, 128)
    assert M2 == M_total and np.array_equal(starts, starts2)
    a = synthetic.gaussian_bf16((M_total, K), 1.0, seed=11)
    w = synthetic.gaussian_bf16((G * N, K), 0.02, seed=12)
    d = run_gpu(a, w, psum, 128, G)
    aq, sa = lnq.quantize_activations(a.to(DEV))
    wq, ws = lnq.quantize_weights_grouped(w.to(DEV), G)
    d2 = torch.full_like(d, float("nan"))
    lnq.lnq_m_grouped_fp8_gemm_contiguous(aq, sa, wq, ws, torch.from_numpy(m_indices).to(DEV), G, d2)
    assert lnq.lnq_get_last_device_error() == 0
    rows = torch.from_numpy(token_rows(sizes, starts)).to(DEV)
    assert torch.equal(d[rows].view(torch.int16), d2[rows].view(torch.int16))


@pytest.mark.parametrize("pairs", [0, 1])
def test_moe_workload_full(pairs, store_path):
    # the 32-expert MoE workload (16384 tokens, multinomial seed 0) moved into the
    # prefix-sum arena with 256-row alignment: every token row is compared with the
    # group-id layout's full reference (the same tokens, the same weights)
    cfg = synthetic.MOE
    a128, w, _, sizes, starts128 = full_refs.moe_inputs()
    G, N, K = cfg.groups, cfg.N, cfg.K
    psum, starts, M_total = synthetic.psum_layout(sizes, 256)
    a = torch.zeros((M_total, K), dtype=torch.bfloat16)
    src = np.concatenate([np.arange(s, s + n) for s, n in zip(starts128, sizes)])
    dst = np.concatenate([np.arange(s, s + n) for s, n in zip(starts, sizes)])
    a[torch.from_numpy(dst)] = a128[torch.from_numpy(src)]
    d = run_gpu(a, w, psum, 256, G, pairs)
    assert lnq.lnq_get_last_device_error() == 0
    ref = full_refs.moe_ref()
    got = to_f64(d)
    assert np.array_equal(np.sort(dst), token_rows(sizes, starts))
    assert_gemm_close(got[dst], ref[src], f"psum MoE workload, pairs={pairs}")
    pad = np.setdiff1d(np.arange(M_total), dst)
    assert np.all(np.isnan(got[pad][:, :64]))


def test_bad_prefix_sums_are_reported():
    N, K = 256, 256
    a = synthetic.gaussian_bf16((512, K), 1.0, seed=21)
    w = synthetic.gaussian_bf16((2 * N, K), 0.02, seed=22)
    # decreasing: group 1's count is taken as zero, group 0 is still computed
    d = run_gpu(a, w, [100, 50], 256, 2)
    assert lnq.lnq_get_last_device_error() == 1          # LNQ_ERR_INVALID_ARG
    assert lnq.lnq_get_last_device_error() == 0
    qa, sa = oracle_quantize_a(a)
    qb, sb = oracle_quantize_w_grouped(w, 2)
    ref = oracle.m_grouped_gemm_psum(qa, sa, qb, sb, [100, 100], 256)
    got = to_f64(d)
    assert_gemm_close(got[:100], ref[:100], "decreasing psum")
    assert np.all(np.isnan(got[100:]))
    # group 1 starts at row 512 of a 512-row arena: nothing of it is written
    d = run_gpu(a, w, [300, 400], 256, 2)
    assert lnq.lnq_get_last_device_error() == 1
    got = to_f64(d)
    ref = oracle.m_grouped_gemm_psum(qa, sa, qb, sb, [300, 300], 256)
    assert_gemm_close(got[:300], ref[:300], "overrun")
    assert np.all(np.isnan(got[300:]))
