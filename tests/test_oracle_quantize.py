"""Pins for the oracle's 1x128 activation and 128x128 weight quantization.

Checked against the pages' definition (one scale per 128 inputs of a row, or per
128x128 weight block, scale = amax/448, codes on the E4M3 grid) and against things
other than the oracle itself:

* a hand-worked example (tests/golden/quantize_worked_example.json);
* the scale is the binary32 value nearest to amax/448, judged in float64;
* groups whose amax is 448 * 2^j have scale 2^j exactly, and their codes equal
  torch's independent fp32 -> e4m3fn conversion of x / 2^j;
* invariants: codes finite, the group maximum maps to +-448, and the dequantized
  value is within half an E4M3 ulp times the scale (plus the fp32 quotient rounding);
* pad scale entries (rows M .. ceil4(M)-1) are 0.0f; an all-zero group has scale 0.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_quantize_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quantize_worked_example.json")


def bf16_from_f64(vals) -> np.ndarray:
    t = torch.tensor(np.asarray(vals, dtype=np.float64)).to(torch.bfloat16)
    assert np.array_equal(t.to(torch.float64).numpy(), np.asarray(vals, np.float64)), "not bf16-exact"
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def e4m3_half_ulp(a: np.ndarray) -> np.ndarray:
    """Half the E4M3 grid spacing in the binade of |a| (2^-10 in the subnormal range)."""
    a = np.abs(a)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.exp2(e - 3) / 2


def check_group_invariants(x: np.ndarray, q: np.ndarray, s: np.ndarray):
    """x float64 [R, 128] bf16 values, q codes [R, 128], s scales [R]."""
    assert not np.any((q & 0x7F) == 0x7F), "NaN code produced"
    vals = oracle.e4m3_value(q)
    amax = np.abs(x).max(axis=1)
    # scale: the binary32 nearest to amax/448 (float64 judges the rounding)
    exact = amax / 448.0
    s64 = s.astype(np.float64)
    ulp32 = np.spacing(s.astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(s64 - exact) <= ulp32 / 2 * (1 + 1e-12))
    nz = amax > 0
    # the largest magnitude lands on +-448
    assert np.all(np.abs(vals[nz]).max(axis=1) == 448.0)
    # dequantization error: |x - v*s| <= (half ulp of the E4M3 binade) * s + |x| 2^-24
    t = np.where(nz[:, None], x / np.where(nz, s64, 1.0)[:, None], 0.0)
    bound = e4m3_half_ulp(t) * s64[:, None] + np.abs(x) * 2.0 ** -24
    err = np.abs(x - vals * s64[:, None])
    assert np.all(err <= bound * (1 + 1e-9) + 1e-300)
    # zero groups: scale 0, codes +-0 with the sign of x
    z = ~nz
    assert np.all(s[z] == 0)
    assert np.all((q[z] & 0x7F) == 0)
    assert np.array_equal(q[z] == 0x80, np.signbit(x[z]))


def test_worked_example():
    d = json.load(open(GOLDEN))
    K = 128 * len(d["groups"])
    x = np.zeros(K, dtype=np.float64)
    codes = np.zeros(K, dtype=np.uint8)
    for g, grp in enumerate(d["groups"]):
        n = len(grp["values"])
        x[g * 128:g * 128 + n] = grp["values"]
        codes[g * 128:g * 128 + n] = [int(c, 16) for c in grp["codes"]]
    q, sfa = oracle.quantize_fp8_groups(bf16_from_f64(x)[None, :])
    assert sfa.shape == (len(d["groups"]), 4)
    assert list(sfa[:, 0]) == [grp["scale"] for grp in d["groups"]]
    assert np.all(sfa[:, 1:] == 0) and not np.any(np.signbit(sfa[:, 1:]))
    assert np.array_equal(q[0], codes), [hex(c) for c in q[0][:20]]


@pytest.mark.parametrize("M,K", [(1, 128), (37, 384), (130, 512)])
def test_activation_invariants_random(M, K):
    x = synthetic.gaussian_bf16((M, K), 1.0, seed=M + K)
    bits = synthetic.bf16_bits(x)
    q, sfa = oracle.quantize_fp8_groups(bits)
    M4 = -(-M // 4) * 4
    assert sfa.shape == (K // 128, M4)
    xf = bf16_bits_to_f64(bits)
    G = K // 128
    check_group_invariants(xf.reshape(M * G, 128), q.reshape(M * G, 128), sfa[:, :M].T.reshape(-1))
    pad = sfa[:, M:]
    assert np.all(pad.view(np.uint32) == 0)


def test_activation_outliers_and_tiny_groups():
    # outlier groups (x100), tiny groups (subnormal-range bf16) and an all-zero group
    M, K = 9, 1024
    x = synthetic.gaussian_bf16_with_outliers((M, K), 1.0, seed=5, outlier_seed=6, frac=0.3)
    xf = x.to(torch.float64).numpy()
    xf[2, :128] *= 2.0 ** -130  # a group whose scale is subnormal in fp32
    xf[3, 128:256] = 0.0
    xf[3, 130] = -0.0
    xf[4, 256:384] = -0.0
    bits = torch.tensor(xf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q, sfa = oracle.quantize_fp8_groups(bits)
    xf = bf16_bits_to_f64(bits)
    G = K // 128
    check_group_invariants(xf.reshape(M * G, 128), q.reshape(M * G, 128), sfa[:, :M].T.reshape(-1))
    assert sfa[0, 2] > 0 and sfa[0, 2] < np.finfo(np.float32).tiny  # subnormal scale kept (no FTZ)
    assert np.all(q[4, 256:384] == 0x80)


@pytest.mark.parametrize("j", [-20, -3, 0, 1, 7])
def test_power_of_two_scale_matches_torch(j):
    rng = np.random.default_rng(100 + j)
    vals = rng.normal(size=(5, 128)) * 100.0
    vals = torch.tensor(vals).to(torch.bfloat16).to(torch.float64).numpy()
    vals = np.clip(vals, -447.0, 447.0)
    vals[:, 17] = 448.0  # amax exactly 448, so scale 2^j after the shift
    vals = vals * 2.0 ** j
    bits = bf16_from_f64(vals)
    q, sfa = oracle.quantize_fp8_groups(bits)
    assert np.all(sfa[0, :5] == np.float32(2.0 ** j))
    t = torch.tensor(vals / 2.0 ** j, dtype=torch.float32)
    ref = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


def check_block_invariants(wf: np.ndarray, q: np.ndarray, sfb: np.ndarray):
    N, K = wf.shape
    for nb in range(sfb.shape[0]):
        for kb in range(sfb.shape[1]):
            blk = wf[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            qb = q[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            check_group_invariants(blk.reshape(1, -1), qb.reshape(1, -1), sfb[nb:nb + 1, kb])


@pytest.mark.parametrize("N,K", [(128, 128), (200, 384), (384, 256)])
def test_weight_block_invariants(N, K):
    w = synthetic.gaussian_bf16((N, K), 0.02, seed=N * 7 + K)
    bits = synthetic.bf16_bits(w)
    q, sfb = oracle.quantize_fp8_blocks(bits)
    assert sfb.shape == (-(-N // 128), K // 128)
    check_block_invariants(bf16_bits_to_f64(bits), q, sfb)


def test_weight_block_is_not_a_row_group():
    # one outlier row inside a block moves the whole block's scale, not only its row
    w = np.full((128, 256), 0.5)
    w[5, 3] = 448.0
    w[9, 200] = 896.0
    q, sfb = oracle.quantize_fp8_blocks(bf16_from_f64(w))
    assert list(sfb[0]) == [1.0, 2.0]
    assert np.all(q[:, :128][np.arange(128) != 5] == 0x30)       # 0.5 / 1.0
    assert np.all(q[:, 128:][np.arange(128) != 9] == 0x28)       # 0.5 / 2.0 = 0.25
    assert q[5, 3] == 0x7E and q[9, 200] == 0x7E


def test_weight_ragged_edge_uses_existing_rows_only():
    N, K = 130, 128
    w = np.full((N, K), 1.0)
    w[128:, :] = 7.0
    w[0, 0] = 448.0
    q, sfb = oracle.quantize_fp8_blocks(bf16_from_f64(w))
    assert sfb[0, 0] == 1.0
    assert sfb[1, 0] == np.float32(7.0) / np.float32(448.0)
    assert np.all(q[128:] == 0x7E)
