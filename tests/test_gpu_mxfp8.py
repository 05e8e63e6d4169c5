"""GPU parity of the MXFP8 gran-32 recipe: 1 x 32 UE8M0 blocks on both operands.

deepgemm-rust README, benchmark block "SM100 FP8: DeepSeek gran-128 recipe and MXFP8 gran-32"
and its kernel table (kind::mxf8f6f4 with UE8M0 scales).

* The quantizer is bit-exact against the oracle: E4M3 codes and exponent bytes.  The GPU
  writes a row's four 32-block exponents of a 128-wide K block into the four bytes of the
  row's atom word; the test reads them back into the oracle's [rows][K/32] layout.  Rows past
  the last real one in a 128-row block carry the byte of p = 1 in all four bytes.
* The GEMM (tcgen05.mma kind::mxf8f6f4.block_scale, the j-th K = 32 step reading scale byte
  j) is compared with the oracle's FP64 product of the same codes and scales within the
  GEMM tolerance, element by element on ragged shapes and over the whole output of a
  prefill linear; a product whose every 32-block has its own scale (a closed form) is
  exact.
* The M-grouped contiguous form is compared on every token row, on small layouts and on the
  32-expert MoE workload (each group's rows against the dense oracle product with its
  weights).
"""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_quantize_b200 as lnq
import oracle
from moe_grouped_gemm_quantize_b200 import synthetic
import full_refs
from parity import assert_gemm_close, codes, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def atom_bytes32(atoms: torch.Tensor, rows: int) -> np.ndarray:
    """Exponent bytes [rows, K/32] from scale atoms [K/128, ceil(rows/128)*128]."""
    w = atoms.cpu().numpy().view(np.uint32)
    r = np.arange(rows)
    idx = (r // 128) * 128 + ((r % 128) % 32) * 4 + ((r % 128) // 32)
    words = w[:, idx]                                   # [K/128, rows]
    b = np.stack([(words >> (8 * j)) & 0xFF for j in range(4)], axis=-1)   # [K/128, rows, 4]
    return b.transpose(1, 0, 2).reshape(rows, -1).astype(np.uint8)


def pad_words(atoms: torch.Tensor, rows: int) -> np.ndarray:
    w = atoms.cpu().numpy().view(np.uint32)
    pad = np.arange(rows, w.shape[1])
    idx = (pad // 128) * 128 + ((pad % 128) % 32) * 4 + ((pad % 128) // 32)
    return w[:, idx]


@pytest.mark.parametrize("R,K", [(1, 128), (130, 256), (300, 1024), (2048, 4096), (6144, 4096)])
def test_quantize_bit_exact(R, K):
    x = synthetic.gaussian_bf16((R, K), 1.0, seed=R + K)
    if R > 3:
        x[1, :32] = 0.0                        # all-zero block: p = 1
        x[2, 32:64] = 3e38                     # near the top of the bf16 range
        x[3, 64:96] *= 1e-38                   # tiny block: clamped exponent
        x[0, 96:128] *= 100.0
    q, sf = lnq.quantize_mxfp8(x.to(DEV))
    torch.cuda.synchronize()
    q_ref, e_ref = oracle.quantize_mxfp8(synthetic.bf16_bits(x))
    assert np.array_equal(codes(q), q_ref)
    assert np.array_equal(atom_bytes32(sf, R), e_ref)
    assert np.all(pad_words(sf, R) == 0x7F7F7F7F)


def run_gemm(a, w):
    aq, sa = lnq.quantize_mxfp8(a.to(DEV))
    wq, sw = lnq.quantize_mxfp8(w.to(DEV))
    d = torch.full((a.shape[0], w.shape[0]), float("nan"), dtype=torch.bfloat16, device=DEV)
    lnq.lnq_mxfp8_gemm_nt(aq, sa, wq, sw, d)
    return d


def oracle_gemm(a, w):
    qa, ea = oracle.quantize_mxfp8(synthetic.bf16_bits(a))
    qb, eb = oracle.quantize_mxfp8(synthetic.bf16_bits(w))
    return oracle.gemm_nt_mx32(qa, ea, qb, eb)


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (300, 384, 512), (1, 256, 128), (129, 16, 256),
                                   (64, 4096, 1024), (1000, 768, 384)])
def test_gemm_elementwise(M, N, K, mx_pairs):
    a = synthetic.gaussian_bf16_with_outliers((M, K), 1.0, M + N, 3, frac=0.1)
    w = synthetic.gaussian_bf16((N, K), 0.02, seed=N + K)
    d = run_gemm(a, w)
    assert lnq.lnq_get_last_device_error() == 0
    assert_gemm_close(to_f64(d), oracle_gemm(a, w), f"mxfp8 {M}x{N}x{K}")


@pytest.mark.parametrize("M", [128, 384])
def test_every_32_block_takes_its_own_scale(M, mx_pairs):
    # codes 1.0 throughout, 32-block b of A row m at 2^(m % 4 + b % 5) and of B row n at
    # 2^-(n % 3): every output is an exact small sum that a scale taken per 128 columns, or
    # from a neighbouring block (or from the other CTA of a pair), would change
    N, K = 256, 512
    B = K // 32
    a = torch.ones((M, K), dtype=torch.float32)
    w = torch.ones((N, K), dtype=torch.float32)
    for b in range(B):
        a[:, 32 * b:32 * b + 32] *= torch.tensor([2.0 ** (m % 4 + b % 5) for m in range(M)])[:, None]
    w *= torch.tensor([2.0 ** -(n % 3) for n in range(N)])[:, None]
    a, w = a.to(torch.bfloat16), w.to(torch.bfloat16)
    d = run_gemm(a, w)
    want = np.array([[sum(32.0 * 2.0 ** (m % 4 + b % 5) for b in range(B)) * 2.0 ** -(n % 3) for n in range(N)]
                     for m in range(M)])
    assert np.array_equal(to_f64(d), want)
    assert np.array_equal(oracle_gemm(a, w), want)


def test_gemm_prefill_full(mx_pairs):
    cfg = synthetic.PREFILL[0]
    a, w = full_refs.linear_inputs(cfg.name)
    d = run_gemm(a, w)
    assert lnq.lnq_get_last_device_error() == 0
    assert_gemm_close(to_f64(d), oracle_gemm(a, w), "mxfp8 prefill QKV")


def run_grouped(a, w, m_indices, G):
    aq, sa = lnq.quantize_mxfp8(a.to(DEV))
    wq, sw = lnq.quantize_mxfp8(w.to(DEV))
    N = w.shape[0] // G
    d = torch.full((a.shape[0], N), float("nan"), dtype=torch.bfloat16, device=DEV)
    lnq.lnq_m_grouped_mxfp8_gemm_contiguous(aq, sa, wq, sw, torch.from_numpy(m_indices).to(DEV), G, d)
    return d


def mx_grouped_ref(a, w, starts, sizes, N):
    qa, ea = oracle.quantize_mxfp8(synthetic.bf16_bits(a))
    qb, eb = oracle.quantize_mxfp8(synthetic.bf16_bits(w))
    D = np.full((a.shape[0], N), np.nan)
    for g, (s, n) in enumerate(zip(starts, sizes)):
        s, n = int(s), int(n)
        if n:
            D[s:s + n] = oracle.gemm_nt_mx32(qa[s:s + n], ea[s:s + n], qb[g * N:(g + 1) * N], eb[g * N:(g + 1) * N])
    return D


@pytest.mark.parametrize("sizes,N,K", [([130, 0, 256, 7, 300], 256, 256), ([1], 384, 512),
                                       ([128, 128, 5], 128, 1024), ([200, 90, 129], 512, 256)])
def test_grouped_elementwise(sizes, N, K):
    G = len(sizes)
    m_indices, starts, M_total = synthetic.contiguous_layout(sizes)
    a = synthetic.gaussian_bf16((M_total, K), 1.0, seed=G + N)
    w = synthetic.gaussian_bf16((G * N, K), 0.02, seed=K + N)
    d = run_grouped(a, w, m_indices, G)
    assert lnq.lnq_get_last_device_error() == 0
    ref = mx_grouped_ref(a, w, starts, sizes, N)
    got = to_f64(d)
    real = m_indices >= 0
    assert_gemm_close(got[real], ref[real], f"mxfp8 grouped {sizes} {N}x{K}")
    led_by_pad = np.repeat(m_indices[::128] < 0, 128)
    assert np.all(np.isnan(got[led_by_pad]))


def test_grouped_moe_workload_full():
    cfg = synthetic.MOE
    a, w, m_indices, sizes, starts = full_refs.moe_inputs()
    d = run_grouped(a, w, m_indices, cfg.groups)
    assert lnq.lnq_get_last_device_error() == 0
    ref = mx_grouped_ref(a, w, starts, sizes, cfg.N)
    real = m_indices >= 0
    assert_gemm_close(to_f64(d)[real], ref[real], "mxfp8 MoE workload")
