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
