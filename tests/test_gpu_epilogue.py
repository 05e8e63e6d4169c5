"""GPU parity of the fused GEMM epilogues: bias, and the output quantized for a next linear.

* Bias: D = A.B^T + bias, compared with the oracle's FP64 product plus the bias within
  the GEMM tolerance, for dense and decode tiles.
* FP8 output, exact case: integer codes with unit scales make every D value (and
  D + bias) a small integer, exact in FP32 and in bf16.  The oracle's product is
  then exact, and its 1 x 128 quantize of that bf16 matrix gives the expected codes
  and scales bit for bit, pad-row scales (0.0) included.
* FP8 output, Gaussian case: each dequantized code lies within the E4M3 rounding
  error of the oracle's result, and almost all codes equal the oracle's quantize
  of its own bf16-rounded product (a code may differ where the FP32 and FP64 sums
  round to different bf16 values).
"""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_quantize_b200 as lnq
import oracle
from moe_grouped_gemm_quantize_b200 import synthetic
from parity import assert_gemm_close, oracle_quantize_a, oracle_quantize_w, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of float64 values (exact in float32) to bf16 bits."""
    f = x.astype(np.float32)
    assert np.array_equal(f.astype(np.float64), x), "values must be exact in float32"
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


@pytest.mark.parametrize("M,N,K", [(300, 384, 512), (129, 256, 256), (8, 256, 1024), (64, 4096, 512)])
def test_bias_bf16_output(M, N, K, store_path):
    a = synthetic.gaussian_bf16((M, K), 1.0, seed=M + N)
    w = synthetic.gaussian_bf16((N, K), 0.02, seed=N + K)
    bias = synthetic.gaussian_bf16((N,), 1.0, seed=K)
    wq, ws = lnq.quantize_weights(w.to(DEV))
    aq, sa = lnq.quantize_activations(a.to(DEV))
    d = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    lnq.lnq_fp8_block_gemm_nt_epilogue(aq, sa, wq, ws, bias=bias.to(DEV), d=d)
    assert lnq.lnq_get_last_device_error() == 0
    qa, sao = oracle_quantize_a(a)
    qb, sbo = oracle_quantize_w(w)
    ref = oracle.gemm_nt(qa, sao, qb, sbo) + bias.to(torch.float64).numpy()[None, :]
    assert_gemm_close(to_f64(d), ref, f"bias {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,with_bias", [(203, 384, True), (256, 256, False), (1000, 512, True)])
def test_fp8_output_exact_integer_case(M, N, with_bias, store_path):
    K = 128
    rng = np.random.default_rng(M + N)
    small = oracle.e4m3_encode(np.array([-1.0, 0.0, 1.0], np.float32))
    qa = small[rng.integers(0, 3, size=(M, K))]
    qb = small[rng.integers(0, 3, size=(N, K))]
    M4 = -(-M // 4) * 4
    sfa = np.ones((K // 128, M4), np.float32)
    sfb = np.ones((N // 128, K // 128), np.float32)
    bias_f = rng.integers(-8, 9, size=N).astype(np.float64) if with_bias else np.zeros(N)
    D = oracle.gemm_nt(qa, sfa, qb, sfb) + bias_f[None, :]            # small integers: exact
    q_ref, s_ref = oracle.quantize_fp8_groups(f64_to_bf16_bits(D), M4)
    q = torch.zeros((M, N), dtype=torch.uint8, device=DEV)
    s = torch.full((N // 128, M4), float("nan"), dtype=torch.float32, device=DEV)
    bias = torch.from_numpy(f64_to_bf16_bits(bias_f).view(np.int16)).view(torch.bfloat16).to(DEV) if with_bias else None
    lnq.lnq_fp8_block_gemm_nt_epilogue(torch.from_numpy(qa).to(DEV), torch.from_numpy(sfa).to(DEV),
                                       torch.from_numpy(qb).to(DEV), torch.from_numpy(sfb).to(DEV),
                                       bias=bias, q=q, sfa_out=s)
    assert lnq.lnq_get_last_device_error() == 0
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_fp8_output_gaussian_against_the_oracle(store_path):
    M, N, K = 512, 1024, 1024
    a = synthetic.gaussian_bf16((M, K), 1.0, seed=5)
    w = synthetic.gaussian_bf16((N, K), 0.02, seed=6)
    bias = synthetic.gaussian_bf16((N,), 0.5, seed=7)
    wq, ws = lnq.quantize_weights(w.to(DEV))
    aq, sa = lnq.quantize_activations(a.to(DEV))
    q = torch.zeros((M, N), dtype=torch.uint8, device=DEV)
    s = torch.empty((N // 128, M), dtype=torch.float32, device=DEV)
    lnq.lnq_fp8_block_gemm_nt_epilogue(aq, sa, wq, ws, bias=bias.to(DEV), q=q, sfa_out=s)
    assert lnq.lnq_get_last_device_error() == 0
    qa, sao = oracle_quantize_a(a)
    qb, sbo = oracle_quantize_w(w)
    D = oracle.gemm_nt(qa, sao, qb, sbo) + bias.to(torch.float64).numpy()[None, :]
    q_ref, s_ref = oracle.quantize_fp8_groups(f64_to_bf16_bits(D.astype(np.float32).astype(np.float64)), M)
    got_codes = q.cpu().numpy()
    got_s = s.cpu().numpy()
    # scales: amax of the bf16-rounded rows, so equal up to the rounding of the sums
    np.testing.assert_allclose(got_s, s_ref, rtol=2 ** -7)
    # dequantized values within half an E4M3 step (relative 2^-4) plus the bf16 rounding
    deq = oracle.e4m3_value(got_codes) * np.repeat(got_s.T, 128, axis=1)
    bound = (2.0 ** -4 + 2.0 ** -8) * np.abs(D) + np.repeat(got_s.T, 128, axis=1) * 2.0 ** -9 * 1.01
    assert np.all(np.abs(deq - D) <= bound)
    assert np.mean(got_codes == q_ref) > 0.99


def test_fp8_output_rejects_what_it_cannot_fuse():
    aq = torch.zeros((8, 256), dtype=torch.uint8, device=DEV)
    sa = torch.ones((2, 8), dtype=torch.float32, device=DEV)
    wq = torch.zeros((256, 256), dtype=torch.uint8, device=DEV)
    ws = torch.ones((2, 2), dtype=torch.float32, device=DEV)
    q = torch.zeros((8, 256), dtype=torch.uint8, device=DEV)
    s = torch.zeros((2, 8), dtype=torch.float32, device=DEV)
    with pytest.raises(lnq.LnqError):   # decode tiles keep a group across threads
        lnq.lnq_fp8_block_gemm_nt_epilogue(aq, sa, wq, ws, q=q, sfa_out=s)
    with pytest.raises(ValueError):
        lnq.lnq_fp8_block_gemm_nt_epilogue(aq, sa, wq, ws)
    assert lnq.lnq_get_last_device_error() == 0
