"""Pins for the oracle's SiLU.mul of a gate_up linear.

h[m][j] = silu(D[m][j]) * D[m][I + j], silu(x) = x / (1 + e^-x), with the gate_up
weight stacking the I gate rows over the I up rows (deepgemm-rust README, "What's
implemented", moe_fp8_layer: grouped GEMM -> SiLU.mul -> grouped GEMM).  Pinned against:

* the identity silu(x) - silu(-x) = x and silu's limits (0 at 0, x for large x,
  -0 for very negative x);
* torch's float64 SiLU (an independent implementation);
* brute force of the whole gate_up product with torch's float64 matmul and SiLU on
  an independent decoder (torch float8_e4m3fn), with gate and up weights drawn
  differently, so that swapped halves fail;
* the point-wise variant against the full one.
"""
import numpy as np
import pytest
import torch

import oracle

FINITE = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)


def test_odd_part_identity_and_limits():
    x = np.concatenate([np.linspace(-30, 30, 601), [1e-300, 1e-200, 3.5, -3.5]])
    one = np.ones_like(x)
    diff = oracle.silu_mul(x, one) - oracle.silu_mul(-x, one)
    np.testing.assert_allclose(diff, x, rtol=4e-16, atol=0)
    assert oracle.silu_mul(np.array([0.0]), np.array([5.0]))[0] == 0.0
    assert oracle.silu_mul(np.array([40.0]), np.array([1.0]))[0] == 40.0
    h = oracle.silu_mul(np.array([-800.0]), np.array([1.0]))[0]
    assert h == 0.0 and np.signbit(h)


def test_against_torch_silu():
    rng = np.random.default_rng(1)
    g = rng.normal(0, 4, 5000)
    u = rng.normal(0, 4, 5000)
    ref = (torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    np.testing.assert_allclose(oracle.silu_mul(g, u), ref, rtol=1e-15, atol=1e-300)


def torch_deq(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64)


@pytest.mark.parametrize("M,I,K", [(5, 128, 256), (33, 256, 128), (2, 384, 384)])
def test_gate_up_brute_force(M, I, K):
    rng = np.random.default_rng(M + I)
    qa = rng.choice(FINITE, size=(M, K)).astype(np.uint8)
    qb = rng.choice(FINITE, size=(2 * I, K)).astype(np.uint8)
    M4 = -(-M // 4) * 4
    sfa = rng.uniform(0.001, 0.01, size=(K // 128, M4)).astype(np.float32)
    sfb = np.concatenate([rng.uniform(0.001, 0.01, size=(I // 128, K // 128)),     # gate blocks
                          rng.uniform(0.02, 0.05, size=(I // 128, K // 128))]      # up blocks
                         ).astype(np.float32)
    h = oracle.gemm_nt_silu_mul(qa, sfa, qb, sfb)
    assert h.shape == (M, I)
    sa = torch.from_numpy(sfa[:, :M].astype(np.float64)).T.repeat_interleave(128, dim=1)
    sb = torch.from_numpy(sfb.astype(np.float64)).repeat_interleave(128, dim=0).repeat_interleave(128, dim=1)
    D = (torch_deq(qa) * sa) @ (torch_deq(qb) * sb).T
    ref = (torch.nn.functional.silu(D[:, :I]) * D[:, I:]).numpy()
    np.testing.assert_allclose(h, ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())
    swapped = (torch.nn.functional.silu(D[:, I:]) * D[:, :I]).numpy()
    assert not np.allclose(h, swapped, rtol=1e-3)


def test_points_agree():
    rng = np.random.default_rng(4)
    M, I, K = 20, 256, 256
    qa = rng.choice(FINITE, size=(M, K)).astype(np.uint8)
    qb = rng.choice(FINITE, size=(2 * I, K)).astype(np.uint8)
    sfa = rng.uniform(0.001, 0.01, size=(K // 128, M)).astype(np.float32)
    sfb = rng.uniform(0.001, 0.01, size=(2 * I // 128, K // 128)).astype(np.float32)
    h = oracle.gemm_nt_silu_mul(qa, sfa, qb, sfb)
    rows = rng.integers(0, M, 300)
    cols = rng.integers(0, I, 300)
    pts = oracle.gemm_nt_silu_mul_points(qa, sfa, qb, sfb, rows, cols)
    assert np.array_equal(pts, h[rows, cols])
    with pytest.raises(ValueError):
        oracle.gemm_nt_silu_mul_points(qa, sfa, qb, sfb, [0], [I])
