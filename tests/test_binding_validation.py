"""Host-only checks of the Python binding's argument marshalling (no GPU, no compute).

Each call validates dtypes, contiguity and shapes before it reaches the C ABI, and raises
TypeError or ValueError; arguments that pass reach the library, which on a host without a
usable GPU answers with an error status (LnqError), never a silent result (the default
stream comes from torch.cuda, so those calls pass stream 0 explicitly).
"""
import pytest
import torch

import moe_grouped_gemm_quantize_b200 as lnq
from moe_grouped_gemm_quantize_b200 import build


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def f8(*shape):
    return torch.zeros(shape, dtype=torch.float8_e4m3fn)


def f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def i32(*shape):
    return torch.zeros(shape, dtype=torch.int32)


def test_psum_binding():
    a, sa = f8(256, 256), f32(2, 256)
    b, sb = f8(2 * 256, 256), f32(4, 2)
    ps, d = i32(2), bf16(256, 256)
    with pytest.raises(TypeError):
        lnq.lnq_m_grouped_fp8_gemm_contiguous_psum(a, sa, b, sb, ps.to(torch.int64), d)
    with pytest.raises(TypeError):
        lnq.lnq_m_grouped_fp8_gemm_contiguous_psum(a, sa, b, sb, ps, d.float())
    with pytest.raises(ValueError):
        lnq.lnq_m_grouped_fp8_gemm_contiguous_psum(a, sa, f8(3 * 256, 256), sb, ps, d)
    with pytest.raises(ValueError):
        lnq.lnq_m_grouped_fp8_gemm_contiguous_psum(a, sa, b, sb, i32(0), d)
    with pytest.raises(ValueError):
        lnq.lnq_m_grouped_fp8_gemm_contiguous_psum(a, sa.t(), b, sb, ps, d)
    if not torch.cuda.is_available():
        with pytest.raises(lnq.LnqError):
            lnq.lnq_m_grouped_fp8_gemm_contiguous_psum(a, sa, b, sb, ps, d, alignment=256, stream=0)


def test_silu_mul_binding():
    a, sa = f8(64, 256), f32(2, 64)
    b, sb = f8(512, 256), f32(4, 2)
    h = bf16(64, 256)
    with pytest.raises(TypeError):
        lnq.lnq_fp8_block_gemm_nt_silu_mul(a, sa, b, sb, h.float())
    with pytest.raises(ValueError):
        lnq.lnq_fp8_block_gemm_nt_silu_mul(a, sa, b, sb, bf16(64, 128))      # I != rows of b / 2
    with pytest.raises(ValueError):
        lnq.lnq_fp8_block_gemm_nt_silu_mul(a, sa, b, f32(2, 2), h)           # sfb rows for 2I
    if not torch.cuda.is_available():
        with pytest.raises(lnq.LnqError):
            lnq.lnq_fp8_block_gemm_nt_silu_mul(a, sa, b, sb, h, stream=0)


def test_ue8m0_bindings():
    with pytest.raises(TypeError):
        lnq.quantize_activations_ue8m0(torch.zeros(4, 128))
    with pytest.raises(TypeError):
        lnq.quantize_weights_ue8m0(torch.zeros(4, 128))
    a, b = f8(200, 256), f8(384, 256)
    sa, sb = i32(2, 256), i32(2, 384)
    d = bf16(200, 384)
    with pytest.raises(TypeError):
        lnq.lnq_mx_block_gemm_nt(a, sa.float(), b, sb, d)
    with pytest.raises(ValueError):
        lnq.lnq_mx_block_gemm_nt(a, i32(2, 200), b, sb, d)                  # atoms cover 256 rows
    with pytest.raises(ValueError):
        lnq.lnq_mx_block_gemm_nt(a, sa, b, sb, bf16(200, 256))
    assert tuple(lnq.ue8m0_atoms(200, 256, "cpu").shape) == (2, 256)
    mi = i32(256)
    with pytest.raises(TypeError):
        lnq.lnq_m_grouped_mx_gemm_contiguous(f8(256, 256), sa, f8(512, 256), i32(2, 512), mi.long(), 2,
                                             bf16(256, 256))
    with pytest.raises(ValueError):
        lnq.lnq_m_grouped_mx_gemm_contiguous(f8(256, 256), sa, f8(512, 256), i32(2, 512), mi, 3, bf16(256, 256))
    if not torch.cuda.is_available():
        with pytest.raises(lnq.LnqError):
            lnq.lnq_mx_block_gemm_nt(a, sa, b, sb, d, stream=0)
