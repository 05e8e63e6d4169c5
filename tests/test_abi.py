"""Host-only checks of the C ABI (no GPU needed, no compute launched).

* liblnq.so loads and exports every function include/lnq.h declares;
* argument validation answers before any CUDA call, with the documented codes;
* with valid arguments and no usable GPU the call fails loudly (LNQ_ERR_CUDA or
  LNQ_ERR_UNSUPPORTED_ARCH), never silently.
"""
import ctypes
import os
import re

import pytest
import torch

import moe_grouped_gemm_quantize_b200 as lnq
from moe_grouped_gemm_quantize_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lnq.h")

OK, INVALID, SHAPE, MISALIGNED, ARCH, CUDA, TIMEOUT = range(7)
A16 = 0x10000   # fake, 16-byte aligned addresses: validation rejects before any use
A16b = 0x20000
A16c = 0x30000
A16d = 0x40000
A16e = 0x50000


@pytest.fixture(scope="module")
def L():
    build.build()
    return lnq.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:lnq_status|const char\*|int32_t|int64_t)\s+(lnq_\w+)\s*\(", text,
                                 flags=re.M)))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("lnq_quantize_fp8_groups", "lnq_fp8_block_gemm_nt",
              "lnq_m_grouped_fp8_gemm_contiguous", "lnq_quantize_fp8_blocks",
              "lnq_status_string", "lnq_get_last_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    assert L.lnq_abi_version() == 10000


def test_library_exports_nothing_undeclared(L):
    # every lnq_* symbol the library exports is part of the declared ABI
    import shutil
    import subprocess
    if shutil.which("nm") is None:
        pytest.skip("nm not available")
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.split() and line.split()[-1].startswith("lnq_")}
    assert exported == set(declared_functions())


def test_status_strings(L):
    for code in range(7):
        assert lnq.lnq_status_string(code)
    assert "timed out" in lnq.lnq_status_string(TIMEOUT)


def test_quantize_argument_errors(L):
    f = L.lnq_quantize_fp8_groups
    s = None
    assert f(A16, -1, 128, 128, A16b, 128, A16c, 4, s) == INVALID
    assert f(A16, 4, 100, 128, A16b, 128, A16c, 4, s) == SHAPE          # K % 128
    assert f(A16, 4, 128, 64, A16b, 128, A16c, 4, s) == INVALID          # ld_x < K
    assert f(A16, 5, 128, 128, A16b, 128, A16c, 4, s) == SHAPE           # M4 < ceil4(M)
    assert f(A16, 4, 128, 128, A16b, 128, A16c, 6, s) == SHAPE           # M4 % 4
    assert f(None, 4, 128, 128, A16b, 128, A16c, 4, s) == INVALID
    assert f(A16 + 2, 4, 128, 128, A16b, 128, A16c, 4, s) == MISALIGNED
    assert f(A16, 4, 128, 132, A16b, 128, A16c, 4, s) == MISALIGNED      # ld_x % 8
    assert f(A16, 4, 128, 128, A16b, 136, A16c, 4, s) == MISALIGNED      # ld_q % 16
    assert f(A16, 0, 128, 128, A16b, 128, A16c, 0, s) == OK              # nothing to do


def test_block_quantize_argument_errors(L):
    f = L.lnq_quantize_fp8_blocks
    assert f(A16, 0, 128, A16b, A16c, None) == INVALID
    assert f(A16, 128, 130, A16b, A16c, None) == SHAPE
    assert f(A16, 128, 128, None, A16c, None) == INVALID
    assert f(A16, 128, 128, A16b, A16c + 2, None) == MISALIGNED
    assert f(A16, 128, 128, A16b + 8, A16c, None) == MISALIGNED


def test_gemm_argument_errors(L):
    f = L.lnq_fp8_block_gemm_nt
    args = dict(a=A16, sfa=A16b, M4=8, b=A16c, sfb=A16d, d=A16e, M=8, N=256, K=512)

    def call(**kw):
        v = dict(args, **kw)
        return f(v["a"], v["sfa"], v["M4"], v["b"], v["sfb"], v["d"], v["M"], v["N"], v["K"], None)

    assert call(M=0) == INVALID
    assert call(K=500) == SHAPE
    assert call(N=8) == SHAPE
    assert call(N=264 + 4) == SHAPE
    assert call(M4=4) == SHAPE
    assert call(M4=10) == SHAPE
    assert call(a=None) == INVALID
    assert call(d=A16e + 8) == MISALIGNED
    assert call(sfb=A16d + 2) == MISALIGNED
    assert call(sfa=A16b + 4) == MISALIGNED


@pytest.mark.parametrize("entry", ["lnq_fp8_block_gemm_nt_static_ws", "lnq_fp8_block_gemm_nt_ws"])
def test_split_entry_points_reject_arguments_before_any_cuda_call(L, entry):
    # the allocation-free and the workspace entry points validate exactly as
    # lnq_fp8_block_gemm_nt does, before touching a device (here there is none)
    f = getattr(L, entry)
    args = dict(a=A16, sfa=A16b, M4=8, b=A16c, sfb=A16d, d=A16e, M=8, N=256, K=512)

    def call(**kw):
        v = dict(args, **kw)
        tail = (None,) if entry.endswith("static_ws") else (None, 0, None)
        return f(v["a"], v["sfa"], v["M4"], v["b"], v["sfb"], v["d"], v["M"], v["N"], v["K"], *tail)

    assert call(M=0) == INVALID
    assert call(M=-3) == INVALID
    assert call(K=500) == SHAPE
    assert call(N=8) == SHAPE
    assert call(M4=4) == SHAPE
    assert call(a=None) == INVALID
    assert call(d=None) == INVALID
    assert call(d=A16e + 8) == MISALIGNED
    assert call(sfa=A16b + 4) == MISALIGNED


def test_grouped_argument_errors(L):
    f = L.lnq_m_grouped_fp8_gemm_contiguous

    def call(M_total=256, N=256, K=512, G=4, mi=A16e + 0x1000, a=A16):
        return f(a, A16b, A16c, A16d, mi, G, A16e, M_total, N, K, None)

    assert call(G=0) == INVALID
    assert call(M_total=200) == SHAPE
    assert call(K=100) == SHAPE
    assert call(N=20) == SHAPE
    assert call(mi=None) == INVALID
    assert call(mi=A16e + 0x1002) == MISALIGNED
    assert call(a=A16 + 1) == MISALIGNED


def test_masked_argument_errors(L):
    f = L.lnq_m_grouped_fp8_gemm_masked

    def call(M_max=256, N=256, K=512, G=4, mm=A16e + 0x1000, a=A16, expected=64):
        return f(a, A16b, A16c, A16d, mm, G, M_max, expected, A16e, N, K, None)

    assert call(G=0) == INVALID
    assert call(expected=-1) == INVALID
    assert call(M_max=200) == SHAPE            # M_max % 128
    assert call(K=100) == SHAPE
    assert call(N=20) == SHAPE
    assert call(mm=None) == INVALID
    assert call(mm=A16e + 0x1002) == MISALIGNED
    assert call(a=A16 + 1) == MISALIGNED


def test_psum_argument_errors(L):
    f = L.lnq_m_grouped_fp8_gemm_contiguous_psum

    def call(M_total=512, N=256, K=512, G=4, ps=A16e + 0x1000, align=256, a=A16):
        return f(a, A16b, A16c, A16d, ps, G, align, A16e, M_total, N, K, None)

    assert call(G=0) == INVALID
    assert call(align=64) == INVALID
    assert call(align=512) == INVALID
    assert call(M_total=384) == SHAPE           # M_total % alignment
    assert call(K=100) == SHAPE
    assert call(N=20) == SHAPE
    assert call(ps=None) == INVALID
    assert call(ps=A16e + 0x1002) == MISALIGNED
    assert call(a=A16 + 1) == MISALIGNED


def test_silu_mul_argument_errors(L):
    f = L.lnq_fp8_block_gemm_nt_silu_mul

    def call(M=256, I=256, K=512, M4=256, h=A16e, a=A16):
        return f(a, A16b, M4, A16c, A16d, h, M, I, K, None)

    assert call(M=0) == INVALID
    assert call(h=None) == INVALID
    assert call(I=200) == SHAPE                 # I % 128
    assert call(K=100) == SHAPE
    assert call(M4=252) == SHAPE                # M4 < ceil4(M)
    assert call(h=A16e + 8) == MISALIGNED
    assert call(a=A16 + 1) == MISALIGNED


def test_ue8m0_argument_errors(L):
    q = L.lnq_quantize_ue8m0_groups
    assert q(A16, 0, 128, 128, A16b, 128, A16c, None) == INVALID
    assert q(A16, 4, 256, 128, A16b, 256, A16c, None) == INVALID      # ld_x < K
    assert q(A16, 4, 200, 256, A16b, 256, A16c, None) == SHAPE        # K % 128
    assert q(A16, 4, 128, 132, A16b, 128, A16c, None) == MISALIGNED   # ld_x % 8
    assert q(A16, 4, 128, 128, A16b, 128, A16c + 4, None) == MISALIGNED
    b = L.lnq_quantize_ue8m0_blocks
    assert b(A16, 0, 128, A16b, A16c, None) == INVALID
    assert b(A16, 4, 100, A16b, A16c, None) == SHAPE
    assert b(A16, 4, 128, A16b, None, None) == INVALID
    g = L.lnq_mx_block_gemm_nt
    assert g(A16, A16b, A16c, A16d, A16e, 0, 256, 128, None) == INVALID
    assert g(A16, A16b, A16c, A16d, A16e, 8, 20, 128, None) == SHAPE   # N % 16
    assert g(A16, A16b, A16c, A16d, A16e, 8, 256, 100, None) == SHAPE  # K % 128
    assert g(A16, A16b + 4, A16c, A16d, A16e, 8, 256, 128, None) == MISALIGNED
    h = L.lnq_m_grouped_mx_gemm_contiguous
    assert h(A16, A16b, A16c, A16d, A16e + 0x100, 0, A16e, 256, 256, 128, None) == INVALID
    assert h(A16, A16b, A16c, A16d, A16e + 0x100, 2, A16e, 200, 256, 128, None) == SHAPE    # M_total % 128
    assert h(A16, A16b, A16c, A16d, A16e + 0x100, 2, A16e, 256, 192, 128, None) == SHAPE    # N % 128
    assert h(A16, A16b, A16c, A16d, None, 2, A16e, 256, 256, 128, None) == INVALID
    assert h(A16, A16b, A16c, A16d, A16e + 0x102, 2, A16e, 256, 256, 128, None) == MISALIGNED


def test_epilogue_argument_errors(L):
    f = L.lnq_fp8_block_gemm_nt_epilogue

    def call(M=256, N=256, K=512, bias=None, d=A16e, q=None, so=None, M4o=256):
        return f(A16, A16b, ((M + 3) // 4) * 4, A16c, A16d, bias, d, q, so, M4o, M, N, K, None)

    assert call(d=None) == INVALID                         # no output
    assert call(q=A16e + 0x2000, so=A16e + 0x4000) == INVALID      # both outputs
    assert call(d=None, q=A16e + 0x2000) == INVALID         # codes without scales
    assert call(M=8, d=None, q=A16e + 0x2000, so=A16e + 0x4000, M4o=8) == SHAPE     # decode tiles
    assert call(N=320, d=None, q=A16e + 0x2000, so=A16e + 0x4000) == SHAPE          # N % 128
    assert call(N=128, d=None, q=A16e + 0x2000, so=A16e + 0x4000) == SHAPE          # N < 256
    assert call(d=None, q=A16e + 0x2000, so=A16e + 0x4000, M4o=252) == SHAPE       # M4_out < ceil4(M)
    assert call(bias=A16e + 0x2002) == MISALIGNED
    assert call(d=None, q=A16e + 0x2001, so=A16e + 0x4000) == MISALIGNED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU failure path")
def test_valid_arguments_without_gpu_fail_loudly(L):
    rc = L.lnq_fp8_block_gemm_nt(A16, A16b, 8, A16c, A16d, A16e, 8, 256, 512, None)
    assert rc in (CUDA, ARCH)
    rc = L.lnq_quantize_fp8_groups(A16, 4, 128, 128, A16b, 128, A16c, 4, None)
    assert rc in (CUDA, ARCH)
    with pytest.raises(lnq.LnqError):
        lnq._check(rc, "probe")


def test_python_binding_rejects_wrong_dtypes(L):
    x = torch.zeros(4, 128, dtype=torch.float32)
    with pytest.raises(TypeError):
        lnq.lnq_quantize_fp8_groups(x, torch.zeros(4, 128, dtype=torch.uint8),
                                    torch.zeros(1, 4, dtype=torch.float32))


def test_no_cpu_fallback_in_the_product():
    # the product package never imports the oracle or any CPU path
    pkg = os.path.join(ROOT, "moe_grouped_gemm_quantize_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "lnq_oracle" not in text, fn


def test_mxfp8_argument_errors(L):
    q = L.lnq_quantize_mxfp8
    assert q(A16, 0, 128, 128, A16b, 128, A16c, None) == INVALID
    assert q(A16, 4, 256, 128, A16b, 256, A16c, None) == INVALID       # ld_x < K
    assert q(A16, 4, 96, 96, A16b, 96, A16c, None) == SHAPE            # K % 128
    assert q(None, 4, 128, 128, A16b, 128, A16c, None) == INVALID
    assert q(A16, 4, 128, 128, A16b + 4, 128, A16c, None) == MISALIGNED
    g = L.lnq_mxfp8_gemm_nt
    assert g(A16, A16b, A16c, A16d, A16e, 0, 256, 128, None) == INVALID
    assert g(A16, A16b, A16c, A16d, A16e, 4, 250, 128, None) == SHAPE   # N % 16
    assert g(A16, A16b, A16c, A16d, None, 4, 256, 128, None) == INVALID
    assert g(A16, A16b, A16c, A16d, A16e + 8, 4, 256, 128, None) == MISALIGNED
    h = L.lnq_m_grouped_mxfp8_gemm_contiguous
    assert h(A16, A16b, A16c, A16d, None, 2, A16e, 256, 256, 128, None) == INVALID
    assert h(A16, A16b, A16c, A16d, A16e + 0x100, 0, A16e, 256, 256, 128, None) == INVALID
    assert h(A16, A16b, A16c, A16d, A16e + 0x100, 2, A16e, 200, 256, 128, None) == SHAPE   # M_total % 128
    assert h(A16, A16b, A16c, A16d, A16e + 0x102, 2, A16e, 256, 256, 128, None) == MISALIGNED


@pytest.mark.parametrize("entry", ["lnq_m_grouped_mx_gemm_masked", "lnq_m_grouped_mxfp8_gemm_masked"])
def test_block_scaled_masked_argument_errors(L, entry):
    f = getattr(L, entry)

    def call(M_max=256, N=256, K=512, G=4, mm=A16e + 0x1000, a=A16, expected=64):
        return f(a, A16b, A16c, A16d, mm, G, M_max, expected, A16e, N, K, None)

    assert call(G=0) == INVALID
    assert call(expected=-1) == INVALID
    assert call(M_max=200) == SHAPE            # M_max % 128
    assert call(K=100) == SHAPE
    assert call(N=144) == SHAPE                # grouped weights: N % 128
    assert call(mm=None) == INVALID
    assert call(mm=A16e + 0x1002) == MISALIGNED
    assert call(a=A16 + 1) == MISALIGNED
