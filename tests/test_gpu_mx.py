"""GPU parity of the UE8M0 recipe: power-of-two scales applied by the tensor core.

deepgemm-rust README, "Blackwell-native FP4/FP8 (SM100a, tcgen05)" (UE8M0 scales consumed
by the block-scaled MMA) and "What's implemented" (gran-128 on either side).

* The quantizers are bit-exact against the oracle: E4M3 codes and exponent bytes.  The
  GPU writes the bytes into 512-byte scale atoms (row r = r0 + 32 r1 of a 128-row block in
  word 4 r0 + r1, low byte); the test reads them back into the oracle's [K/128][rows]
  layout.  Pad rows of the last block carry the byte of p = 1.
* The GEMM (tcgen05.mma kind::mxf8f6f4.block_scale) is compared with the oracle's FP64
  product of the same codes and power-of-two scales, within the GEMM tolerance, element by
  element on ragged shapes and over the whole output of a prefill linear.
* The M-grouped contiguous form (each 128-row block takes the group of its first row) is
  compared with the oracle's grouped product on rows with a group id, element by element on
  small layouts and on every token row of the 32-expert MoE workload; blocks led by -1
  stay untouched.
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


def atom_bytes(atoms: torch.Tensor, rows: int) -> np.ndarray:
    """Exponent bytes [K/128, rows] from scale atoms [K/128, ceil(rows/128)*128]."""
    w = atoms.cpu().numpy().view(np.uint32)
    r = np.arange(rows)
    idx = (r // 128) * 128 + ((r % 128) % 32) * 4 + ((r % 128) // 32)
    assert np.all((w & 0xFFFFFF00) == 0), "only the low byte of a word is used"
    return (w[:, idx] & 0xFF).astype(np.uint8)


def pad_bytes(atoms: torch.Tensor, rows: int) -> np.ndarray:
    w = atoms.cpu().numpy().view(np.uint32)
    pad = np.arange(rows, w.shape[1])
    idx = (pad // 128) * 128 + ((pad % 128) % 32) * 4 + ((pad % 128) // 32)
    return w[:, idx]


@pytest.mark.parametrize("M,K", [(1, 128), (130, 256), (300, 1024), (2048, 4096)])
def test_activation_quantize_bit_exact(M, K):
    x = synthetic.gaussian_bf16((M, K), 1.0, seed=M + K)
    if M > 3:
        x[1, :128] = 0.0                       # all-zero group: p = 1
        x[2, 128:256] = 3e38 if K > 128 else x[2, 128:256]
        x[3, :128] *= 1e-38                    # tiny group: clamped exponent
    q, sf = lnq.quantize_activations_ue8m0(x.to(DEV))
    torch.cuda.synchronize()
    q_ref, e_ref = oracle.quantize_ue8m0_groups(synthetic.bf16_bits(x))
    assert np.array_equal(codes(q), q_ref)
    assert np.array_equal(atom_bytes(sf, M), e_ref)
    assert np.all(pad_bytes(sf, M) == 127)


@pytest.mark.parametrize("N,K", [(256, 256), (200, 384), (1, 128), (6144, 4096)])
def test_weight_quantize_bit_exact(N, K):
    w = synthetic.gaussian_bf16((N, K), 0.02, seed=N + 3 * K)
    q, sf = lnq.quantize_weights_ue8m0(w.to(DEV))
    torch.cuda.synchronize()
    q_ref, e_ref = oracle.quantize_ue8m0_blocks(synthetic.bf16_bits(w))
    assert np.array_equal(codes(q), q_ref)
    rows = atom_bytes(sf, -(-N // 128) * 128)          # every row of a block: the block's byte
    assert np.array_equal(rows, np.repeat(e_ref.T, 128, axis=1))


def run_gemm(a, w):
    aq, sa = lnq.quantize_activations_ue8m0(a.to(DEV))
    wq, sw = lnq.quantize_weights_ue8m0(w.to(DEV))
    d = torch.full((a.shape[0], w.shape[0]), float("nan"), dtype=torch.bfloat16, device=DEV)
    lnq.lnq_mx_block_gemm_nt(aq, sa, wq, sw, d)
    return d


def oracle_gemm(a, w):
    qa, ea = oracle.quantize_ue8m0_groups(synthetic.bf16_bits(a))
    qb, eb = oracle.quantize_ue8m0_blocks(synthetic.bf16_bits(w))
    return oracle.gemm_nt(qa, oracle.ue8m0_value(ea), qb, oracle.ue8m0_value(eb))


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (300, 384, 512), (1, 256, 128), (129, 16, 256),
                                   (64, 4096, 1024), (1000, 768, 384)])
def test_gemm_elementwise(M, N, K, mx_pairs):
    a = synthetic.gaussian_bf16((M, K), 1.0, seed=M + N)
    w = synthetic.gaussian_bf16((N, K), 0.02, seed=N + K)
    d = run_gemm(a, w)
    assert lnq.lnq_get_last_device_error() == 0
    assert_gemm_close(to_f64(d), oracle_gemm(a, w), f"ue8m0 {M}x{N}x{K}")


def test_gemm_prefill_full(mx_pairs):
    cfg = synthetic.PREFILL[0]
    a, w = full_refs.linear_inputs(cfg.name)
    d = run_gemm(a, w)
    assert lnq.lnq_get_last_device_error() == 0
    assert_gemm_close(to_f64(d), oracle_gemm(a, w), "ue8m0 prefill QKV")


def test_repeated_runs_are_identical(mx_pairs):
    a = synthetic.gaussian_bf16((256, 512), 1.0, seed=5)
    w = synthetic.gaussian_bf16((512, 512), 0.02, seed=6)
    d1, d2 = run_gemm(a, w), run_gemm(a, w)
    torch.cuda.synchronize()
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))


def test_many_tiles_per_cta_elementwise(mx_pairs):
    # 4096 x 8192 at K = 256: 1024 tiles of 128 x 256 (512 pair tiles of 256 x 256), several
    # per persistent CTA, so the accumulator hand-over between tiles is checked element by
    # element
    a = synthetic.gaussian_bf16((4096, 256), 1.0, seed=411)
    w = synthetic.gaussian_bf16((8192, 256), 0.02, seed=412)
    d = run_gemm(a, w)
    assert lnq.lnq_get_last_device_error() == 0
    assert_gemm_close(to_f64(d), oracle_gemm(a, w), "ue8m0 many tiles")


def run_grouped(a, w, m_indices, G):
    aq, sa = lnq.quantize_activations_ue8m0(a.to(DEV))
    wq, sw = lnq.quantize_weights_ue8m0(w.to(DEV))
    N = w.shape[0] // G
    d = torch.full((a.shape[0], N), float("nan"), dtype=torch.bfloat16, device=DEV)
    lnq.lnq_m_grouped_mx_gemm_contiguous(aq, sa, wq, sw, torch.from_numpy(m_indices).to(DEV), G, d)
    return d


@pytest.mark.parametrize("sizes,N,K", [([130, 0, 256, 7, 300], 256, 256), ([1], 384, 512),
                                       ([128, 128, 5], 128, 1024), ([200, 90, 129], 512, 256)])
def test_grouped_elementwise(sizes, N, K):
    G = len(sizes)
    m_indices, _, M_total = synthetic.contiguous_layout(sizes)
    a = synthetic.gaussian_bf16((M_total, K), 1.0, seed=G + N)
    w = synthetic.gaussian_bf16((G * N, K), 0.02, seed=K + N)
    d = run_grouped(a, w, m_indices, G)
    assert lnq.lnq_get_last_device_error() == 0
    qa, ea = oracle.quantize_ue8m0_groups(synthetic.bf16_bits(a))
    qb, eb = oracle.quantize_ue8m0_blocks(synthetic.bf16_bits(w))
    ref = oracle.m_grouped_gemm_contiguous(qa, oracle.ue8m0_value(ea), qb, oracle.ue8m0_value(eb), m_indices, G)
    got = to_f64(d)
    real = m_indices >= 0
    assert_gemm_close(got[real], ref[real], f"ue8m0 grouped {sizes} {N}x{K}")
    led_by_pad = np.repeat(m_indices[::128] < 0, 128)
    assert np.all(np.isnan(got[led_by_pad]))


def test_grouped_moe_workload_full():
    # every token row of the 32-expert MoE workload; each group's rows against the
    # dense oracle product with its weights and power-of-two scales
    cfg = synthetic.MOE
    a, w, m_indices, sizes, starts = full_refs.moe_inputs()
    d = run_grouped(a, w, m_indices, cfg.groups)
    assert lnq.lnq_get_last_device_error() == 0
    qa, ea = oracle.quantize_ue8m0_groups(synthetic.bf16_bits(a))
    qb, eb = oracle.quantize_ue8m0_blocks(synthetic.bf16_bits(w))
    ref = full_refs.grouped_ref(qa, oracle.ue8m0_value(ea), qb, oracle.ue8m0_value(eb), starts, sizes, cfg.N)
    real = m_indices >= 0
    assert_gemm_close(to_f64(d)[real], ref[real], "ue8m0 MoE workload")
