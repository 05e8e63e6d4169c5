"""GPU parity of the quantize kernels against the oracle: bit-exact codes and scales.

Covers the 1x128 activation kernel (lnq_quantize_fp8_groups) and the 128x128
weight kernel (lnq_quantize_fp8_blocks) on ragged and strided shapes, the edge
cases of the method (-0, subnormal bf16, tiny scales, all-zero groups, outlier
groups), every bf16 magnitude up to 448 with a unit scale, and the full
workloads' activations and weights.
"""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_quantize_b200 as lnq
import oracle
from moe_grouped_gemm_quantize_b200 import synthetic
from parity import codes, oracle_quantize_a, oracle_quantize_w

pytestmark = pytest.mark.gpu
DEV = "cuda"


def gpu_quantize_a(a: torch.Tensor, M4=None, ld_x=None, ld_q=None):
    M, K = a.shape
    M4 = lnq.ceil4(M) if M4 is None else M4
    if ld_x is not None:
        base = torch.zeros((M, ld_x), dtype=torch.bfloat16, device=DEV)
        base[:, :K] = a.to(DEV)
        x = base[:, :K]
    else:
        x = a.to(DEV)
    qb = torch.full((M, ld_q if ld_q else K), 0xAB, dtype=torch.uint8, device=DEV)
    q = qb[:, :K]
    sfa = torch.full((K // 128, M4), float("nan"), dtype=torch.float32, device=DEV)
    lnq.lnq_quantize_fp8_groups(x, q, sfa)
    torch.cuda.synchronize()
    if ld_q:
        assert np.all(codes(qb)[:, K:] == 0xAB), "wrote past K in the padded row stride"
    return codes(q), sfa.cpu().numpy()


def assert_same_a(a: torch.Tensor, **kw):
    q, s = gpu_quantize_a(a, **kw)
    qo, so = oracle_quantize_a(a, kw.get("M4"))
    assert np.array_equal(s.view(np.uint32), so.view(np.uint32)), "scales differ"
    if not np.array_equal(q, qo):
        bad = np.argwhere(q != qo)[:5]
        raise AssertionError(f"codes differ at {bad.tolist()}: gpu {[hex(q[tuple(i)]) for i in bad]}"
                             f" oracle {[hex(qo[tuple(i)]) for i in bad]}")


@pytest.mark.parametrize("M,K", [(1, 128), (3, 256), (4, 384), (37, 512), (130, 4096), (128, 512)])
def test_activation_shapes(M, K):
    assert_same_a(synthetic.gaussian_bf16((M, K), 1.0, seed=M * 31 + K))


def test_activation_strides_and_padded_scales():
    a = synthetic.gaussian_bf16((37, 384), 1.0, seed=3)
    assert_same_a(a, ld_x=520, ld_q=400)
    assert_same_a(a, M4=48)


def test_activation_edge_values():
    M, K = 12, 1024
    x = synthetic.gaussian_bf16_with_outliers((M, K), 1.0, 7, 8, frac=0.25).to(torch.float64)
    x[0, :128] *= 2.0 ** -128          # subnormal-range bf16 and a subnormal fp32 scale
    x[1, 128:256] = 0.0                # all-zero group
    x[1, 200] = -0.0
    x[2, 256:384] = -0.0
    x[3, :128] = torch.linspace(-448, 448, 128, dtype=torch.float64)
    x[4, :128] = 1e-3 * torch.sign(torch.randn(128, dtype=torch.float64))
    x[4, 5] = 3e4                      # one huge value: most codes round to +-0
    x[5, :] = 2.0 ** -133              # the smallest bf16 subnormals
    x[6, ::2] = 3.0e38                 # near the top of the bf16 range
    assert_same_a(x.to(torch.bfloat16))


def test_subnormal_values_under_the_smallest_reciprocal_scales():
    # scales just above 2^-125 (the smallest whose reciprocal is taken rather than the
    # division) with the rest of each group bf16 subnormals: their quotients reach the
    # E4M3 subnormal codes, so no input or product may be flushed to zero
    rows = []
    for m in (1.0, 1.25, 1.5, 3.0, 5.5, 7.9):
        for sign in (1.0, -1.0):
            row = np.zeros(128)
            row[0] = 448.0 * 2.0 ** -125 * m
            row[1:] = sign * np.arange(1, 128) * 2.0 ** -133
            rows.append(row)
    x = torch.tensor(np.stack(rows)).to(torch.bfloat16)
    assert_same_a(x)


def test_every_bf16_magnitude_with_unit_and_power_of_two_scales():
    # all non-negative finite bf16 bit patterns up to 448, both signs, in rows whose
    # amax is exactly 448 * 2^j: the scale is 2^j and each code is the E4M3 rounding
    # of the value itself
    bits = np.arange(0, 0x43E1, dtype=np.uint16)            # 0 .. 448 (0x43E0)
    vals = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    vals = np.concatenate([vals, -vals])
    per_row = 127
    rows = -(-vals.size // per_row)
    x = np.zeros((rows, 128))
    x[:, 0] = 448.0
    flat = np.zeros(rows * per_row)
    flat[:vals.size] = vals
    x[:, 1:] = flat.reshape(rows, per_row)
    for j in (0, -5, 3):
        assert_same_a(torch.tensor(x * 2.0 ** j).to(torch.bfloat16))


@pytest.mark.parametrize("name", ["tiny", "prefill_down", "decode", "square"])
def test_activation_workloads(name):
    if name == "tiny":
        cfgs = [synthetic.TINY]
    elif name == "prefill_down":
        cfgs = [synthetic.PREFILL[3], synthetic.PREFILL[0]]
    elif name == "decode":
        cfgs = list(synthetic.DECODE)
    else:
        cfgs = [synthetic.SQUARE]
    for cfg in cfgs:
        a, _ = synthetic.make_linear_inputs(cfg)
        assert_same_a(a)


def test_activation_moe_workload():
    a, _, _, _ = synthetic.make_moe_inputs(synthetic.MoE(groups=32, N=128))  # small weights
    assert_same_a(a)


def gpu_quantize_w(w: torch.Tensor):
    q, s = lnq.quantize_weights(w.to(DEV))
    torch.cuda.synchronize()
    return codes(q), s.cpu().numpy()


def assert_same_w(w: torch.Tensor):
    q, s = gpu_quantize_w(w)
    qo, so = oracle_quantize_w(w)
    assert np.array_equal(s.view(np.uint32), so.view(np.uint32)), "block scales differ"
    assert np.array_equal(q, qo), "weight codes differ"


@pytest.mark.parametrize("N,K", [(128, 128), (200, 384), (256, 512), (130, 4096)])
def test_weight_shapes(N, K):
    assert_same_w(synthetic.gaussian_bf16((N, K), 0.02, seed=N + K))


def test_weight_edge_values():
    w = synthetic.gaussian_bf16_with_outliers((256, 256), 1.0, 9, 10, frac=0.2).to(torch.float64)
    w[:128, :128] = 0.0
    w[5, 5] = -0.0
    w[128:, 128:] *= 2.0 ** -127
    assert_same_w(w.to(torch.bfloat16))


def test_weight_workloads():
    for cfg in (synthetic.TINY, synthetic.DECODE[0], synthetic.PREFILL[3]):
        _, w = synthetic.make_linear_inputs(cfg)
        assert_same_w(w)
    cfg = synthetic.SQUARE
    w = synthetic.gaussian_bf16_with_outliers((cfg.N, cfg.K), 1.0, cfg.w_seed, cfg.w_outlier_seed)
    assert_same_w(w)


def test_moe_weights_full_size():
    cfg = synthetic.MOE
    w = synthetic.gaussian_bf16((cfg.groups * cfg.N, cfg.K), cfg.w_std, cfg.w_seed)
    assert_same_w(w)


def near_midpoint_rows(max_rows=8192):
    """Rows whose quotients x/s land near E4M3 rounding midpoints under scales that are
    not powers of two: found by brute force over every bf16 amax in [1, 2) (every
    possible scale mantissa) x every bf16 x up to amax.  Kept: x where RN(x * RN(1/s))
    and RN(x / s) take different E4M3 codes, and x where RN(x / s) is within 256 ulps
    of a midpoint."""
    amax_bits = np.arange(0x3F80, 0x4000, dtype=np.uint16)           # bf16 values in [1, 2)
    x_bits = np.arange(0, 0x4000, dtype=np.uint16)                   # bf16 values in [0, 2)
    xs = (x_bits.astype(np.uint32) << 16).view(np.float32)
    chosen = []
    for ab in amax_bits:
        amax = np.float32((np.uint32(ab) << 16).view(np.float32))
        s = np.float32(amax / np.float32(448.0))
        r = np.float32(np.float32(1.0) / s)
        x = xs[xs <= amax]
        t = (x / s).astype(np.float32)
        f = (x * r).astype(np.float32)
        ct = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        cf = torch.from_numpy(f).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        low = t.view(np.uint32) & 0xFFFFF
        near = np.abs(low.astype(np.int64) - 0x80000) <= 256
        pick = x[(ct != cf) | near]
        for i in range(0, pick.size, 127):
            chosen.append((amax, pick[i:i + 127]))
    rows = chosen[:max_rows]
    out = np.zeros((len(rows), 128), np.float64)
    for k, (amax, vals) in enumerate(rows):
        out[k, 0] = amax
        out[k, 1:1 + vals.size] = vals
        out[k, 1 + vals.size:] = -vals[0] if vals.size else 0.0
    return out


def test_quotients_near_e4m3_midpoints():
    x = near_midpoint_rows()
    assert x.shape[0] > 100
    for scale in (1.0, -3.0, 2.0 ** 40, 2.0 ** -60):
        assert_same_a(torch.tensor(x * scale).to(torch.bfloat16))


def test_zero_rows_write_zero_pad_scales():
    x = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    q = torch.empty((0, 256), dtype=torch.uint8, device=DEV)
    sfa = torch.full((2, 8), float("nan"), dtype=torch.float32, device=DEV)
    lnq.lnq_quantize_fp8_groups(x, q, sfa)
    torch.cuda.synchronize()
    assert torch.all(sfa == 0)


@pytest.mark.parametrize("M,K", [(1, 4096), (33, 384), (100, 640), (4097, 256)])
def test_activation_more_ragged_shapes(M, K):
    # K not a multiple of 256 (a half-empty column tile) and row counts off the 32-row tile
    assert_same_a(synthetic.gaussian_bf16((M, K), 1.0, seed=M + K))


@pytest.mark.parametrize("M,K", [(8192, 8192), (2048, 12288)])
def test_activation_quantize_is_repeatable(M, K):
    # Every launch must write the same bytes, whatever the output buffers held before and
    # however the launches overlap: a consumer warp that handed a ring stage back before its
    # shared-memory reads completed would let some groups see the next tile (wrong scales at
    # places that change from run to run).  Inputs larger than L2 keep the producer ahead of
    # the consumers; twelve launches per shape, chained as a step chains them.
    g = torch.Generator(device=DEV)
    g.manual_seed(M + K)
    x = (torch.randn((M, K), generator=g, device=DEV)
         * torch.exp(torch.randn((M, 1), generator=g, device=DEV))).to(torch.bfloat16)
    M4 = lnq.ceil4(M)
    ref_q = torch.empty((M, K), dtype=torch.uint8, device=DEV)
    ref_s = torch.empty((K // 128, M4), dtype=torch.float32, device=DEV)
    lnq.lnq_quantize_fp8_groups(x, ref_q, ref_s)
    for fill in (0x00, 0xAB, 0x55, 0xFF):
        q = torch.full((M, K), fill, dtype=torch.uint8, device=DEV)
        s = torch.full((K // 128, M4), float(fill), dtype=torch.float32, device=DEV)
        for _ in range(3):
            lnq.lnq_quantize_fp8_groups(x, q, s)
        torch.cuda.synchronize()
        assert lnq.lnq_get_last_device_error() == 0
        bad = (q != ref_q).nonzero()
        assert bad.shape[0] == 0, f"fill {fill:#x}: {bad.shape[0]} codes differ, first {bad[:4].tolist()}"
        assert torch.equal(s.view(torch.int32), ref_s.view(torch.int32)), f"fill {fill:#x}: scales differ"
