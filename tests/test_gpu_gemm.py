"""GPU parity of the block-scaled FP8 GEMM (dense and decode) against the oracle.

The oracle quantizes the same seeded bf16 inputs itself and computes D in FP64;
the CUDA path quantizes with its own kernels (bit-exact with the oracle, see
test_gpu_quantize) and multiplies.  Every output is compared element by element
over the whole of D: the small and ragged shapes, a shape of many more tiles than
SMs (so every persistent CTA runs several tiles), and the full workloads in every
launch configuration (the benchmark's included); the full-size references are
computed once per session (full_refs).
"""
import functools

import numpy as np
import pytest
import torch

import moe_grouped_gemm_quantize_b200 as lnq
import oracle
from moe_grouped_gemm_quantize_b200 import synthetic
import full_refs
from parity import assert_gemm_close, codes, oracle_quantize_a, oracle_quantize_w, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def gpu_linear(a: torch.Tensor, w: torch.Tensor):
    wq, ws = lnq.quantize_weights(w.to(DEV))
    aq, sa = lnq.quantize_activations(a.to(DEV))
    d = torch.full((a.shape[0], w.shape[0]), float("nan"), dtype=torch.bfloat16, device=DEV)
    lnq.lnq_fp8_block_gemm_nt(aq, sa, wq, ws, d)
    assert lnq.lnq_get_last_device_error() == 0
    return d, (aq, sa, wq, ws)


def oracle_linear(a, w):
    qa, sa = oracle_quantize_a(a)
    qb, sb = oracle_quantize_w(w)
    return oracle.gemm_nt(qa, sa, qb, sb), (qa, sa, qb, sb)


def check_full(a, w, what):
    d, _ = gpu_linear(a, w)
    ref, _ = oracle_linear(a, w)
    return assert_gemm_close(to_f64(d), ref, what)


def test_tiny_workload_elementwise():
    a, w = synthetic.make_linear_inputs(synthetic.TINY)
    check_full(a, w, "tiny 128x256x512")


@pytest.fixture(params=[0, 1, 2], ids=["one_cta", "cta_pairs_256", "cta_pairs_128"])
def dense_pairs(request):
    """Runs a test with each dense configuration: single CTAs, CTA pairs on 256x256
    tiles, CTA pairs on 256x128 tiles."""
    previous = lnq.lib().lnq_set_dense_cta_pairs(request.param)
    yield request.param
    lnq.lib().lnq_set_dense_cta_pairs(previous)


@pytest.fixture(params=[False, True], ids=["no_prefetch", "weight_prefetch"])
def weight_prefetch(request):
    """Runs a test with and without the weights' first stages streamed before the
    wait on the previous kernel (the weights here are written two kernels earlier,
    by a kernel that does not release its dependents early)."""
    previous = lnq.lnq_set_weight_prefetch(request.param)
    yield request.param
    lnq.lnq_set_weight_prefetch(previous)


@pytest.mark.parametrize("M,N,K", [
    (65, 256, 128), (100, 128, 256), (128, 16, 128), (130, 272, 384), (200, 640, 512),
    (257, 384, 640), (384, 1024, 1024), (129, 48, 256), (300, 4096, 128), (640, 768, 512),
])
def test_dense_shapes_elementwise(M, N, K, dense_pairs, weight_prefetch, store_path):
    a = synthetic.gaussian_bf16((M, K), 1.0, seed=M + 7 * N + K)
    w = synthetic.gaussian_bf16((N, K), 0.02, seed=M + N + 3 * K)
    check_full(a, w, f"{M}x{N}x{K}")


@pytest.mark.parametrize("M", [1, 2, 5, 8, 17, 31, 32, 33, 48, 63, 64])
@pytest.mark.parametrize("N,K", [(256, 512), (384, 1024)])
def test_decode_shapes_elementwise(M, N, K, weight_prefetch):
    a = synthetic.gaussian_bf16((M, K), 1.0, seed=M * 5 + N)
    w = synthetic.gaussian_bf16((N, K), 0.02, seed=N + K)
    check_full(a, w, f"decode {M}x{N}x{K}")


def test_outlier_groups_elementwise():
    a = synthetic.gaussian_bf16_with_outliers((256, 1024), 1.0, 1, 2)
    w = synthetic.gaussian_bf16_with_outliers((512, 1024), 1.0, 3, 4)
    check_full(a, w, "outliers 256x512x1024")


def test_oracle_quantized_operands_give_the_same_product():
    # feed the oracle's own codes and scales to the GEMM: the result must equal the
    # product of the GPU-quantized operands bit for bit (the quantize is bit-exact)
    a, w = synthetic.make_linear_inputs(synthetic.TINY)
    d, (aq, sa, wq, ws) = gpu_linear(a, w)
    qa, sao = oracle_quantize_a(a)
    qb, sbo = oracle_quantize_w(w)
    d2 = torch.empty_like(d)
    lnq.lnq_fp8_block_gemm_nt(torch.from_numpy(qa).to(DEV), torch.from_numpy(sao).to(DEV),
                              torch.from_numpy(qb).to(DEV), torch.from_numpy(sbo).to(DEV), d2)
    torch.cuda.synchronize()
    assert torch.equal(d.view(torch.int16), d2.view(torch.int16))


def test_deterministic():
    a = synthetic.gaussian_bf16((512, 2048), 1.0, 5)
    w = synthetic.gaussian_bf16((1024, 2048), 0.02, 6)
    d1, _ = gpu_linear(a, w)
    d2, _ = gpu_linear(a, w)
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))


def check_workload(name, what=None):
    """The named workload's whole D against its cached full oracle reference."""
    a, w = full_refs.linear_inputs(name)
    d, _ = gpu_linear(a, w)
    return assert_gemm_close(to_f64(d), full_refs.linear_ref(name), what or name)


@pytest.mark.parametrize("idx", range(4))
def test_prefill_workloads_full(idx, dense_pairs, store_path):
    check_workload(synthetic.PREFILL[idx].name)


@pytest.mark.parametrize("idx", range(4))
def test_decode_workloads_full(idx, weight_prefetch):
    check_workload(synthetic.DECODE[idx].name)


def test_square_outlier_workload_full(dense_pairs, store_path):
    check_workload(synthetic.SQUARE.name)


@functools.lru_cache(maxsize=None)
def many_tiles_case():
    # 4096 x 8192 output at K = 256: 1024 tiles of 128 x 256 (512 CTA-pair tiles of
    # 256 x 256), several per persistent CTA, so the accumulator ring, its phases and the
    # tile boundary are exercised under an element-by-element check
    M, N, K = 4096, 8192, 256
    a = synthetic.gaussian_bf16((M, K), 1.0, seed=401)
    w = synthetic.gaussian_bf16((N, K), 0.02, seed=402)
    qa, sa = oracle_quantize_a(a)
    qb, sb = oracle_quantize_w(w)
    return a, w, oracle.gemm_nt(qa, sa, qb, sb)


def test_many_tiles_per_cta_elementwise(dense_pairs, weight_prefetch, store_path):
    a, w, ref = many_tiles_case()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert (a.shape[0] // 256) * (w.shape[0] // 256) > 3 * sms // 2
    d, _ = gpu_linear(a, w)
    assert_gemm_close(to_f64(d), ref, f"many tiles, configuration {dense_pairs}")


def test_timeout_path_reports_and_recovers():
    # a wait that nobody satisfies gives up after 20 ms and reports LNQ_ERR_TIMEOUT;
    # the context stays usable and the status is cleared once read
    lnq.lnq_selftest_wait_timeout(20_000_000)
    assert lnq.lnq_get_last_device_error() == 6
    assert lnq.lnq_get_last_device_error() == 0
    a, w = synthetic.make_linear_inputs(synthetic.TINY)
    check_full(a, w, "tiny after timeout")


# ---------------------------------------------------------------- decode K split

def gpu_linear_split(a: torch.Tensor, w: torch.Tensor):
    wq, ws = lnq.quantize_weights(w.to(DEV))
    aq, sa = lnq.quantize_activations(a.to(DEV))
    M, N, K = a.shape[0], w.shape[0], a.shape[1]
    work = lnq.gemm_workspace(M, N, K, DEV)
    d = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    lnq.lnq_fp8_block_gemm_nt_ws(aq, sa, wq, ws, d, work)
    assert lnq.lnq_get_last_device_error() == 0
    return d, work, (aq, sa, wq, ws)


def counters_zero(work: torch.Tensor, M: int, N: int) -> bool:
    # the counters fill the workspace's first 4 KiB, one int32 per weight tile
    return bool((work[:4096].view(torch.int32) == 0).all())


@pytest.mark.parametrize("M", [1, 5, 32, 33, 64])
@pytest.mark.parametrize("N,K", [(256, 1024), (400, 2048), (1152, 4096)])
def test_decode_split_elementwise(M, N, K, weight_prefetch):
    a = synthetic.gaussian_bf16((M, K), 1.0, seed=3 * M + N)
    w = synthetic.gaussian_bf16((N, K), 0.02, seed=N + 7 * K)
    d, work, _ = gpu_linear_split(a, w)
    assert work is not None, "this product must take the split path"
    ref, _ = oracle_linear(a, w)
    assert_gemm_close(to_f64(d), ref, f"split {M}x{N}x{K}")
    torch.cuda.synchronize()
    assert counters_zero(work, M, N)


def test_decode_split_is_deterministic_and_reuses_its_workspace():
    M, N, K = 64, 1152, 4096
    a = synthetic.gaussian_bf16((M, K), 1.0, 11)
    w = synthetic.gaussian_bf16((N, K), 0.02, 12)
    d1, work, (aq, sa, wq, ws) = gpu_linear_split(a, w)
    d2 = torch.empty_like(d1)
    for _ in range(3):
        lnq.lnq_fp8_block_gemm_nt_ws(aq, sa, wq, ws, d2, work)
    torch.cuda.synchronize()
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))
    assert counters_zero(work, M, N)


def test_decode_split_workloads(weight_prefetch):
    for cfg in synthetic.DECODE:
        a, w = full_refs.linear_inputs(cfg.name)
        d, work, (aq, sa, wq, ws) = gpu_linear_split(a, w)
        assert work is not None
        assert_gemm_close(to_f64(d), full_refs.linear_ref(cfg.name), cfg.name + " split")
        torch.cuda.synchronize()
        assert counters_zero(work, cfg.M, cfg.N)


def test_workspace_call_without_a_split_is_the_plain_product():
    # no workspace, or a product that does not split, takes the unsplit kernel
    a = synthetic.gaussian_bf16((64, 1024), 1.0, 21)
    w = synthetic.gaussian_bf16((256, 1024), 0.02, 22)
    d_plain, (aq, sa, wq, ws) = gpu_linear(a, w)
    d = torch.empty_like(d_plain)
    lnq.lnq_fp8_block_gemm_nt_ws(aq, sa, wq, ws, d, None)
    torch.cuda.synchronize()
    assert torch.equal(d.view(torch.int16), d_plain.view(torch.int16))
    a2 = synthetic.gaussian_bf16((200, 512), 1.0, 23)
    w2 = synthetic.gaussian_bf16((256, 512), 0.02, 24)
    assert lnq.gemm_workspace(200, 256, 512, DEV) is None
    d2_plain, (aq2, sa2, wq2, ws2) = gpu_linear(a2, w2)
    d2 = torch.empty_like(d2_plain)
    lnq.lnq_fp8_block_gemm_nt_ws(aq2, sa2, wq2, ws2, d2, torch.zeros(256, dtype=torch.uint8, device=DEV))
    torch.cuda.synchronize()
    assert torch.equal(d2.view(torch.int16), d2_plain.view(torch.int16))


def test_workspace_errors_are_reported_before_launch():
    a = synthetic.gaussian_bf16((8, 1024), 1.0, 31)
    w = synthetic.gaussian_bf16((256, 1024), 0.02, 32)
    _, (aq, sa, wq, ws) = gpu_linear(a, w)
    d = torch.empty((8, 256), dtype=torch.bfloat16, device=DEV)
    need = lnq.lnq_fp8_block_gemm_nt_workspace_bytes(8, 256, 1024, torch.cuda.get_device_properties(0).multi_processor_count)
    assert need > 0
    small = torch.zeros(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(lnq.LnqError):
        lnq.lnq_fp8_block_gemm_nt_ws(aq, sa, wq, ws, d, small)
    big = torch.zeros(need + 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(lnq.LnqError):
        lnq.lnq_fp8_block_gemm_nt_ws(aq, sa, wq, ws, d, big[16:])   # not 256-byte aligned
    assert lnq.lnq_get_last_device_error() == 0


def test_one_workspace_serves_products_of_different_shapes():
    # sized for the largest product, zeroed once, then used by products whose
    # partial tiles and counters have other extents
    shapes = [(64, 12288, 4096), (8, 1152, 4096), (33, 400, 2048), (1, 2048, 8192), (64, 12288, 4096)]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    size = max(lnq.lnq_fp8_block_gemm_nt_workspace_bytes(M, N, K, sms) for M, N, K in shapes)
    work = torch.zeros(size, dtype=torch.uint8, device=DEV)
    for i, (M, N, K) in enumerate(shapes):
        a = synthetic.gaussian_bf16((M, K), 1.0, seed=100 + i)
        w = synthetic.gaussian_bf16((N, K), 0.02, seed=200 + i)
        wq, ws = lnq.quantize_weights(w.to(DEV))
        aq, sa = lnq.quantize_activations(a.to(DEV))
        d = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        lnq.lnq_fp8_block_gemm_nt_ws(aq, sa, wq, ws, d, work)
        torch.cuda.synchronize()
        assert lnq.lnq_get_last_device_error() == 0
        qa, sao = oracle_quantize_a(a)
        qb, sbo = oracle_quantize_w(w)
        ref = oracle.gemm_nt(qa, sao, qb, sbo)
        assert_gemm_close(to_f64(d), ref, f"shared workspace {M}x{N}x{K}")
        assert counters_zero(work, M, N)
