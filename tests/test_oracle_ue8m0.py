"""Pins for the oracle's UE8M0 recipe (power-of-two scales stored as 8-bit exponents).

deepgemm-rust README, "Blackwell-native FP4/FP8 (SM100a, tcgen05)": UE8M0 scales consumed
by the block-scaled MMA; "What's implemented": the gran-128 recipe on either side.  The
reading: a group's (or block's) scale is the smallest power of two p with 448 p >= amax,
stored as e + 127; codes are the E4M3 RNE of x / p.  Pinned against:

* the defining inequalities 448 p >= amax > 448 p / 2, evaluated in exact rationals, over
  random and boundary amax values, and hand-worked examples (one of them the four-group
  row of tests/golden/ue8m0_worked_example.json);
* torch's independent float32 -> float8_e4m3fn conversion of x / p;
* properties: no code saturates, every non-zero group has a code of magnitude >= 224,
  dequantized values lie within half an E4M3 step of the input;
* blocks: the amax over a 128 x 128 block (ragged edges included), and the activation
  rule applied to a single-row block.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_quantize_b200 import synthetic


def bf16_bits_of(values) -> np.ndarray:
    t = torch.tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def group_with_amax(amax: float) -> np.ndarray:
    """One 1x128 row whose largest magnitude is exactly amax (a bf16 value)."""
    row = np.zeros(128, dtype=np.float32)
    row[5] = amax
    row[77] = -amax / 3
    return bf16_bits_of(row)[None, :]


@pytest.mark.parametrize("amax,byte", [
    (448.0, 127),        # p = 1
    (449.0, 127),        # 449 is not a bf16 value: the input rounds to 448, p = 1
    (1.0, 119),          # 448 * 2^-8 = 1.75 >= 1 > 0.875
    (14.0, 122),         # 448 * 2^-5 = 14
    (14.0625, 123),      # the next bf16 above 14: p = 2^-4
    (0.0, 127),          # all-zero group: p = 1
])
def test_hand_worked_scales(amax, byte):
    bits = group_with_amax(amax)
    a = float(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().abs().max())
    q, sfe = oracle.quantize_ue8m0_groups(bits)
    if amax == 449.0:
        assert a == 448.0
    assert sfe[0, 0] == byte


def exact_bounds_hold(amax: float, byte: int) -> bool:
    p = Fraction(2) ** (int(byte) - 127)
    a = Fraction(amax)
    if a == 0:
        return byte == 127
    return 448 * p >= a and (byte == 0 or 448 * p / 2 < a)


def test_scale_is_the_smallest_sufficient_power_of_two():
    rng = np.random.default_rng(3)
    mags = np.concatenate([
        np.exp(rng.uniform(-80, 80, 3000)),
        [448.0 * 2.0 ** k for k in range(-60, 60)],
        [1.75 * 2.0 ** k for k in range(-60, 60)],
        [1.7578125 * 2.0 ** k for k in range(-60, 60)],     # first bf16 above 1.75
        [1.7421875 * 2.0 ** k for k in range(-60, 60)],     # last bf16 below 1.75
        [2.0 ** -133, 2.0 ** -126, 3.3e38],
    ])
    rows = np.stack([group_with_amax(float(m))[0] for m in mags])
    q, sfe = oracle.quantize_ue8m0_groups(rows)
    amax = torch.from_numpy(rows.view(np.int16)).view(torch.bfloat16).float().abs().max(dim=1).values.numpy()
    for a, b in zip(amax, sfe[0]):
        assert exact_bounds_hold(float(a), int(b)), (a, b)


def test_codes_against_torch_conversion_and_properties():
    x = synthetic.gaussian_bf16((64, 512), 3.0, seed=9)
    x[3, :128] = 0.0
    x[4, 128:256] *= 1e-30
    bits = synthetic.bf16_bits(x)
    q, sfe = oracle.quantize_ue8m0_groups(bits)
    xf = x.float().numpy().astype(np.float64)
    p = np.repeat(oracle.ue8m0_value(sfe).T.astype(np.float64), 128, axis=1)
    ref = torch.from_numpy((xf / p).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)
    vals = torch.from_numpy(q).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.all(np.abs(vals) <= 448.0)
    g = np.abs(vals).reshape(64, 4, 128).max(axis=2)
    nonzero = np.abs(xf).reshape(64, 4, 128).max(axis=2) > 0
    assert np.all(g[nonzero] >= 224.0)
    assert np.all(q[3, :128] & 0x7F == 0) and sfe[0, 3] == 127
    # within half an E4M3 step (relative 2^-4) of the input, or the subnormal step
    err = np.abs(vals * p - xf)
    assert np.all(err <= np.maximum(np.abs(xf) * 2.0 ** -4, p * 2.0 ** -10) * 1.0000001)


@pytest.mark.parametrize("N,K", [(256, 256), (200, 384), (1, 128)])
def test_blocks(N, K):
    w = synthetic.gaussian_bf16((N, K), 0.02, seed=N + K)
    bits = synthetic.bf16_bits(w)
    q, sfe = oracle.quantize_ue8m0_blocks(bits)
    assert sfe.shape == (-(-N // 128), K // 128)
    wf = w.float().numpy()
    for nb in range(sfe.shape[0]):
        for kb in range(sfe.shape[1]):
            blk = wf[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            assert exact_bounds_hold(float(np.abs(blk).max()), int(sfe[nb, kb]))
    # one row: the block rule equals the activation rule
    q1, s1 = oracle.quantize_ue8m0_groups(bits[:1])
    if N == 1:
        assert np.array_equal(q1, q) and np.array_equal(s1[:, 0], sfe[0])
    p = np.repeat(np.repeat(oracle.ue8m0_value(sfe).astype(np.float64), 128, axis=0)[:N], 128, axis=1)
    ref = torch.from_numpy((wf.astype(np.float64) / p).astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(q, ref.view(torch.uint8).numpy())


def test_gemm_with_ue8m0_scales_is_the_plain_product():
    # the recipe changes only the scales: the block-scaled product of the UE8M0 operands is
    # the dense product of their dequantized values
    a = synthetic.gaussian_bf16((40, 256), 1.0, seed=1)
    w = synthetic.gaussian_bf16((256, 256), 0.02, seed=2)
    qa, ea = oracle.quantize_ue8m0_groups(synthetic.bf16_bits(a))
    qb, eb = oracle.quantize_ue8m0_blocks(synthetic.bf16_bits(w))
    sa, sb = oracle.ue8m0_value(ea), oracle.ue8m0_value(eb)
    D = oracle.gemm_nt(qa, sa, qb, sb)
    A = torch.from_numpy(qa).view(torch.float8_e4m3fn).double() * torch.from_numpy(
        np.repeat(sa.T, 128, axis=1).astype(np.float64))
    B = torch.from_numpy(qb).view(torch.float8_e4m3fn).double() * torch.from_numpy(
        np.repeat(np.repeat(sb, 128, axis=0), 128, axis=1).astype(np.float64))
    np.testing.assert_allclose(D, (A @ B.T).numpy(), rtol=1e-12, atol=1e-12)
    # and it is near the FP32-scale recipe's product: each recipe carries up to 2^-4 relative
    # rounding per code (about 2-3% RMS on a product of two quantized operands), so the
    # two differ by a few percent, never by a wrong scale (a factor of 2 or more)
    qa2, sa2 = oracle.quantize_fp8_groups(synthetic.bf16_bits(a))
    qb2, sb2 = oracle.quantize_fp8_blocks(synthetic.bf16_bits(w))
    D2 = oracle.gemm_nt(qa2, sa2, qb2, sb2)
    assert np.linalg.norm(D - D2) / np.linalg.norm(D2) < 0.1


def test_golden_worked_example():
    path = os.path.join(os.path.dirname(__file__), "golden", "ue8m0_worked_example.json")
    ex = json.load(open(path))
    row = np.zeros(ex["K"], dtype=np.float32)
    for k, v in ex["inputs"].items():
        row[int(k)] = v
    bits = bf16_bits_of(row)[None, :]
    assert np.array_equal(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()[0], row)
    q, sfe = oracle.quantize_ue8m0_groups(bits)
    assert list(sfe[:, 0]) == ex["scale_bytes"]
    expected = np.zeros(ex["K"], dtype=np.uint8)
    for k, c in ex["codes"].items():
        expected[int(k)] = c
    assert np.array_equal(q[0], expected)
