"""Pins for the oracle's MXFP8 gran-32 recipe.

deepgemm-rust README, benchmark block "SM100 FP8: DeepSeek gran-128 recipe and MXFP8
gran-32" and its kernel table (kind::mxf8f6f4 with UE8M0 scales).  The reading: every row
of an operand, activations and weights alike, in 1 x 32 blocks along K; each block's scale
is the smallest power of two p with 448 p >= amax (the gran-128 rule of the UE8M0 recipe),
stored as e + 127; codes are the E4M3 RNE of x / p.  Pinned against:

* the hand-worked row of tests/golden/mxfp8_worked_example.json (scales and codes);
* the defining inequalities 448 p >= amax > 448 p / 2, in exact rationals, block by block;
* torch's independent float32 -> float8_e4m3fn conversion of x / p;
* for the product: brute force in torch float64 with torch's own E4M3 decoder and scales
  2^(e - 127), and closed forms in which every 32-block carries its own scale, so a block
  index taken per 128 columns (or a scale taken from the other operand's row) fails.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_quantize_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "mxfp8_worked_example.json")


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    return synthetic.bf16_bits(x.to(torch.bfloat16))


def test_worked_example():
    g = json.load(open(GOLDEN))
    row = torch.zeros(g["K"], dtype=torch.float32)
    for k, v in g["inputs"].items():
        row[int(k)] = v
    q, sfe = oracle.quantize_mxfp8(bf16_bits(row[None, :]))
    assert sfe[0].tolist() == g["scale_bytes"]
    for k, code in g["codes"].items():
        assert int(q[0, int(k)]) == code, k


def test_defining_inequalities_block_by_block():
    x = synthetic.gaussian_bf16_with_outliers((64, 1024), 1.0, 3, 4, frac=0.2)
    x[0, :32] = 0.0
    x[1, 32:64] *= 2.0 ** -100
    q, sfe = oracle.quantize_mxfp8(synthetic.bf16_bits(x))
    xf = x.float().numpy()
    for r in range(x.shape[0]):
        for b in range(x.shape[1] // 32):
            amax = float(np.abs(xf[r, 32 * b:32 * b + 32]).max())
            p = Fraction(2) ** (int(sfe[r, b]) - 127)
            if amax == 0.0:
                assert sfe[r, b] == 127
            else:
                assert 448 * p >= Fraction(amax) > 224 * p or sfe[r, b] in (0, 254)


def test_codes_are_torch_conversions_of_x_over_p():
    x = synthetic.gaussian_bf16_with_outliers((128, 512), 1.0, 5, 6, frac=0.1)
    q, sfe = oracle.quantize_mxfp8(synthetic.bf16_bits(x))
    p = np.ldexp(1.0, np.repeat(sfe.astype(np.int32) - 127, 32, axis=1))
    t = torch.tensor(x.double().numpy() / p, dtype=torch.float64)   # exact: p is a power of two
    assert float(t.abs().max()) <= 448.0                              # never saturates
    want = t.float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, want)


def torch_product(qa, ea, qb, eb):
    da = torch.from_numpy(qa).view(torch.float8_e4m3fn).double() * torch.from_numpy(
        np.ldexp(1.0, np.repeat(ea.astype(np.int32) - 127, 32, axis=1)))
    db = torch.from_numpy(qb).view(torch.float8_e4m3fn).double() * torch.from_numpy(
        np.ldexp(1.0, np.repeat(eb.astype(np.int32) - 127, 32, axis=1)))
    return (da @ db.T).numpy()


@pytest.mark.parametrize("M,N,K", [(1, 1, 32), (3, 5, 64), (8, 16, 128), (7, 9, 256)])
def test_product_brute_force(M, N, K):
    a = synthetic.gaussian_f32((M, K), 1.0, M + 100)
    w = synthetic.gaussian_f32((N, K), 0.5, K + 200)
    a[:, ::7] *= 100.0                       # blocks of very different magnitudes
    w[:, 3::11] *= 0.01
    a, w = a.to(torch.bfloat16), w.to(torch.bfloat16)
    qa, ea = oracle.quantize_mxfp8(synthetic.bf16_bits(a))
    qb, eb = oracle.quantize_mxfp8(synthetic.bf16_bits(w))
    np.testing.assert_allclose(oracle.gemm_nt_mx32(qa, ea, qb, eb), torch_product(qa, ea, qb, eb),
                               rtol=1e-12, atol=1e-300)


def test_product_closed_form_per_block_scales():
    # codes all 1.0 (0x38); row m of A gives 32-block b the scale 2^(m + b), row n of B
    # gives block b the scale 2^(-n * b): D[m][n] = sum_b 32 * 2^(m + b - n b), exact
    M, N, K = 4, 3, 256
    B = K // 32
    qa = np.full((M, K), 0x38, np.uint8)
    qb = np.full((N, K), 0x38, np.uint8)
    ea = np.array([[127 + m + b for b in range(B)] for m in range(M)], np.uint8)
    eb = np.array([[127 - n * b for b in range(B)] for n in range(N)], np.uint8)
    D = oracle.gemm_nt_mx32(qa, ea, qb, eb)
    want = np.array([[sum(32.0 * 2.0 ** (m + b - n * b) for b in range(B)) for n in range(N)] for m in range(M)])
    assert np.array_equal(D, want)


def test_product_one_hot_block_picks_its_own_scales():
    # a single non-zero 32-block k in A's row and B's row: D is that block's product
    # with exactly that block's two scales
    K = 256
    for k in range(K // 32):
        qa = np.zeros((1, K), np.uint8)
        qb = np.zeros((1, K), np.uint8)
        qa[0, 32 * k:32 * k + 32] = 0x40            # 2.0
        qb[0, 32 * k:32 * k + 32] = 0x30            # 0.5
        ea = np.array([[127 + b for b in range(K // 32)]], np.uint8)
        eb = np.array([[127 - 2 * b for b in range(K // 32)]], np.uint8)
        D = oracle.gemm_nt_mx32(qa, ea, qb, eb)
        assert D[0, 0] == 32 * 1.0 * 2.0 ** (k - 2 * k)
