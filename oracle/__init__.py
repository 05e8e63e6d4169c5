"""CPU oracle for the block-scaled FP8 linear and its M-grouped contiguous variant.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  The product path (the CUDA
library and its Python binding) never imports, links or runs anything here, and
this package never imports the product.

The arithmetic lives in ``lnq_oracle.c`` (plain C, FP64 accumulation, IEEE
single-precision division for the scales and quotients); this module only builds
it with gcc and marshals numpy arrays.  Every function cites the page passage it
follows in the C source.  Pins against the pages and the mathematics live in
``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lnq_oracle.c")
_LIB = os.path.join(_HERE, "liblnq_oracle.so")
# The mutation tests point this at a compiled copy of the oracle with one planted
# mistake, to show that the pins catch it; unset, the oracle is built from _SRC.
_LIB_OVERRIDE = os.environ.get("LNQ_ORACLE_LIB")
_lock = threading.Lock()
_lib = None

GROUP = 128


def compile_source(src: str, out: str) -> str:
    """Compile an oracle source file with gcc (OpenMP, no FMA contraction, no fast-math)."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = [
        "gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
        "-fPIC", "-shared", "-Wall", "-o", tmp, src, "-lm",
    ]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Build the oracle library next to its source (when out of date)."""
    if _LIB_OVERRIDE:
        return _LIB_OVERRIDE
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    return compile_source(_SRC, _LIB)


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode_array.argtypes = [P, I64, P]
        lib.oracle_e4m3_value_array.argtypes = [P, I64, P]
        lib.oracle_quantize_fp8_groups.restype = ctypes.c_int
        lib.oracle_quantize_fp8_groups.argtypes = [P, I64, I64, I64, P, I64, P, I64]
        lib.oracle_quantize_fp8_blocks.restype = ctypes.c_int
        lib.oracle_quantize_fp8_blocks.argtypes = [P, I64, I64, P, P]
        lib.oracle_gemm_nt.restype = ctypes.c_int
        lib.oracle_gemm_nt.argtypes = [P, P, I64, P, P, I64, I64, I64, P]
        lib.oracle_gemm_nt_points.restype = ctypes.c_int
        lib.oracle_gemm_nt_points.argtypes = [P, P, I64, P, P, I64, I64, I64, P, P, I64, P]
        lib.oracle_m_grouped_gemm_contiguous.restype = ctypes.c_int
        lib.oracle_m_grouped_gemm_contiguous.argtypes = [P, P, P, P, P, ctypes.c_int32, I64, I64, I64, P]
        lib.oracle_m_grouped_gemm_points.restype = ctypes.c_int
        lib.oracle_m_grouped_gemm_points.argtypes = [
            P, P, P, P, P, ctypes.c_int32, I64, I64, I64, P, P, I64, P]
        lib.oracle_quantize_ue8m0_groups.restype = ctypes.c_int
        lib.oracle_quantize_ue8m0_groups.argtypes = [P, I64, I64, I64, P, I64, P]
        lib.oracle_quantize_ue8m0_blocks.restype = ctypes.c_int
        lib.oracle_quantize_ue8m0_blocks.argtypes = [P, I64, I64, P, P]
        lib.oracle_silu_mul.restype = None
        lib.oracle_silu_mul.argtypes = [P, P, I64, P]
        lib.oracle_m_grouped_gemm_psum.restype = ctypes.c_int
        lib.oracle_m_grouped_gemm_psum.argtypes = [P, P, P, P, P, ctypes.c_int32, I64, I64, I64, I64, P]
        lib.oracle_m_grouped_gemm_masked.restype = ctypes.c_int
        lib.oracle_m_grouped_gemm_masked.argtypes = [P, P, I64, P, P, P, ctypes.c_int32, I64, I64, I64, P]
        lib.oracle_m_grouped_gemm_masked_points.restype = ctypes.c_int
        lib.oracle_m_grouped_gemm_masked_points.argtypes = [
            P, P, I64, P, P, P, ctypes.c_int32, I64, I64, I64, P, P, I64, P]
        lib.oracle_quantize_mxfp8.restype = ctypes.c_int
        lib.oracle_quantize_mxfp8.argtypes = [P, I64, I64, I64, P, I64, P]
        lib.oracle_gemm_nt_mx32.restype = ctypes.c_int
        lib.oracle_gemm_nt_mx32.argtypes = [P, P, P, P, I64, I64, I64, P]
        _lib = lib
        return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return np.ascontiguousarray(a)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use."""
    return int(_load().oracle_num_threads())


def ceil4(m: int) -> int:
    return -(-m // 4) * 4


def e4m3_value(codes) -> np.ndarray:
    """Exact value (float64) of each E4M3 code; NaN for 0x7F / 0xFF."""
    c = _c(np.asarray(codes, dtype=np.uint8), np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    _load().oracle_e4m3_value_array(_ptr(c), c.size, _ptr(out))
    return out


def e4m3_encode(t) -> np.ndarray:
    """E4M3 code of each float32 value: RNE, ties to even, saturating at 448."""
    a = _c(np.asarray(t, dtype=np.float32), np.float32)
    out = np.empty(a.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(a), a.size, _ptr(out))
    return out


def quantize_fp8_groups(x_bf16_bits: np.ndarray, M4: int | None = None):
    """1x128 activation quantization of a bf16 matrix given as uint16 bits [M, K].

    Returns (q uint8 [M, K], sfa float32 [K/128, M4]) with M4 = ceil4(M) unless given.
    """
    x = _c(x_bf16_bits, np.uint16)
    M, K = x.shape
    M4 = ceil4(M) if M4 is None else int(M4)
    q = np.empty((M, K), dtype=np.uint8)
    sfa = np.empty((K // GROUP, M4), dtype=np.float32)
    _check(_load().oracle_quantize_fp8_groups(_ptr(x), M, K, K, _ptr(q), K, _ptr(sfa), M4),
           "quantize_fp8_groups")
    return q, sfa


def quantize_fp8_blocks(w_bf16_bits: np.ndarray):
    """128x128 weight quantization of a bf16 matrix given as uint16 bits [N, K].

    Returns (q uint8 [N, K], sfb float32 [ceil(N/128), K/128]).
    """
    w = _c(w_bf16_bits, np.uint16)
    N, K = w.shape
    q = np.empty((N, K), dtype=np.uint8)
    sfb = np.empty((-(-N // GROUP), K // GROUP), dtype=np.float32)
    _check(_load().oracle_quantize_fp8_blocks(_ptr(w), N, K, _ptr(q), _ptr(sfb)),
           "quantize_fp8_blocks")
    return q, sfb


def gemm_nt(qa, sfa, qb, sfb, M: int | None = None) -> np.ndarray:
    """FP64 D [M, N] of the dequantized operands (qa [M, K], qb [N, K])."""
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    sfa = _c(sfa, np.float32)
    sfb = _c(sfb, np.float32)
    M = qa.shape[0] if M is None else M
    K = qa.shape[1]
    N = qb.shape[0]
    D = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_gemm_nt(_ptr(qa), _ptr(sfa), sfa.shape[1], _ptr(qb), _ptr(sfb),
                                  M, N, K, _ptr(D)), "gemm_nt")
    return D


def gemm_nt_points(qa, sfa, qb, sfb, rows, cols) -> np.ndarray:
    """FP64 D at the points (rows[i], cols[i])."""
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    sfa = _c(sfa, np.float32)
    sfb = _c(sfb, np.float32)
    rows = _c(np.asarray(rows, dtype=np.int64), np.int64)
    cols = _c(np.asarray(cols, dtype=np.int64), np.int64)
    out = np.empty(rows.shape, dtype=np.float64)
    _check(_load().oracle_gemm_nt_points(_ptr(qa), _ptr(sfa), sfa.shape[1], _ptr(qb), _ptr(sfb),
                                         qa.shape[0], qb.shape[0], qa.shape[1], _ptr(rows),
                                         _ptr(cols), rows.size, _ptr(out)), "gemm_nt_points")
    return out


def m_grouped_gemm_contiguous(qa, sfa, qb, sfb, m_indices, num_groups: int) -> np.ndarray:
    """FP64 D [M_total, N]; rows with a negative group id are NaN."""
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    sfa = _c(sfa, np.float32)
    sfb = _c(sfb, np.float32)
    mi = _c(np.asarray(m_indices, dtype=np.int32), np.int32)
    M_total, K = qa.shape
    N = qb.shape[0] // num_groups
    D = np.full((M_total, N), np.nan, dtype=np.float64)
    _check(_load().oracle_m_grouped_gemm_contiguous(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb),
                                                    _ptr(mi), num_groups, M_total, N, K, _ptr(D)),
           "m_grouped_gemm_contiguous")
    return D


def m_grouped_gemm_points(qa, sfa, qb, sfb, m_indices, num_groups: int, rows, cols) -> np.ndarray:
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    sfa = _c(sfa, np.float32)
    sfb = _c(sfb, np.float32)
    mi = _c(np.asarray(m_indices, dtype=np.int32), np.int32)
    rows = _c(np.asarray(rows, dtype=np.int64), np.int64)
    cols = _c(np.asarray(cols, dtype=np.int64), np.int64)
    M_total, K = qa.shape
    N = qb.shape[0] // num_groups
    out = np.empty(rows.shape, dtype=np.float64)
    _check(_load().oracle_m_grouped_gemm_points(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), _ptr(mi),
                                                num_groups, M_total, N, K, _ptr(rows), _ptr(cols),
                                                rows.size, _ptr(out)), "m_grouped_gemm_points")
    return out


def m_grouped_gemm_masked(qa, sfa, qb, sfb, masked_m, M_max: int) -> np.ndarray:
    """FP64 D [G*M_max, N] of the masked grouped product: group g's first masked_m[g]
    rows (rows g*M_max ...) against group g's weights; other rows are NaN.  qa is
    [G*M_max, K], sfa [K/128, M4] over those rows, qb [G*N, K]."""
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    sfa = _c(sfa, np.float32)
    sfb = _c(sfb, np.float32)
    mm = _c(np.asarray(masked_m, dtype=np.int32), np.int32)
    G = mm.size
    total, K = qa.shape
    if total != G * M_max:
        raise ValueError("qa must hold G * M_max rows")
    N = qb.shape[0] // G
    D = np.full((total, N), np.nan, dtype=np.float64)
    _check(_load().oracle_m_grouped_gemm_masked(_ptr(qa), _ptr(sfa), sfa.shape[1], _ptr(qb), _ptr(sfb),
                                                _ptr(mm), G, M_max, N, K, _ptr(D)), "m_grouped_gemm_masked")
    return D


def m_grouped_gemm_masked_points(qa, sfa, qb, sfb, masked_m, M_max: int, rows, cols) -> np.ndarray:
    """The masked grouped product at (rows[i], cols[i]); NaN past a group's count."""
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    sfa = _c(sfa, np.float32)
    sfb = _c(sfb, np.float32)
    mm = _c(np.asarray(masked_m, dtype=np.int32), np.int32)
    rows = _c(np.asarray(rows, dtype=np.int64), np.int64)
    cols = _c(np.asarray(cols, dtype=np.int64), np.int64)
    G = mm.size
    total, K = qa.shape
    N = qb.shape[0] // G
    out = np.empty(rows.shape, dtype=np.float64)
    _check(_load().oracle_m_grouped_gemm_masked_points(_ptr(qa), _ptr(sfa), sfa.shape[1], _ptr(qb), _ptr(sfb),
                                                       _ptr(mm), G, M_max, N, K, _ptr(rows), _ptr(cols),
                                                       rows.size, _ptr(out)), "m_grouped_gemm_masked_points")
    return out


def m_grouped_gemm_psum(qa, sfa, qb, sfb, psum, alignment: int) -> np.ndarray:
    """FP64 D [M_total, N] of the prefix-sum grouped layout: group g's psum[g] - psum[g-1]
    tokens start at the aligned row sum_{j<g} align_up(count_j, alignment); other rows NaN."""
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    sfa = _c(sfa, np.float32)
    sfb = _c(sfb, np.float32)
    ps = _c(np.asarray(psum, dtype=np.int32), np.int32)
    G = ps.size
    M_total, K = qa.shape
    N = qb.shape[0] // G
    D = np.full((M_total, N), np.nan, dtype=np.float64)
    _check(_load().oracle_m_grouped_gemm_psum(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), _ptr(ps), G,
                                              alignment, M_total, N, K, _ptr(D)), "m_grouped_gemm_psum")
    return D


def silu_mul(g, u) -> np.ndarray:
    """FP64 silu(g) * u elementwise, silu(x) = x / (1 + e^-x)."""
    g = np.ascontiguousarray(g, dtype=np.float64)
    u = np.ascontiguousarray(u, dtype=np.float64)
    if g.shape != u.shape:
        raise ValueError("gate and up shapes differ")
    h = np.empty_like(g)
    _load().oracle_silu_mul(_ptr(g), _ptr(u), g.size, _ptr(h))
    return h


def gemm_nt_silu_mul(qa, sfa, qb, sfb) -> np.ndarray:
    """FP64 h [M, I] of a gate_up linear: D = A.B^T with B [2I, K] (gate rows, then up
    rows), h = silu(D[:, :I]) * D[:, I:]."""
    D = gemm_nt(qa, sfa, qb, sfb)
    I = D.shape[1] // 2
    if D.shape[1] != 2 * I:
        raise ValueError("the gate_up weight needs an even row count")
    return silu_mul(D[:, :I], D[:, I:])


def gemm_nt_silu_mul_points(qa, sfa, qb, sfb, rows, cols) -> np.ndarray:
    """FP64 h at the points (rows[i], cols[i]), cols < I."""
    I = qb.shape[0] // 2
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.asarray(cols, dtype=np.int64)
    if np.any(cols < 0) or np.any(cols >= I):
        raise ValueError("columns must lie below I")
    g = gemm_nt_points(qa, sfa, qb, sfb, rows, cols)
    u = gemm_nt_points(qa, sfa, qb, sfb, rows, cols + I)
    return silu_mul(g, u)


def quantize_ue8m0_groups(x_bf16_bits: np.ndarray):
    """UE8M0 recipe, 1x128 activation groups of a bf16 matrix given as uint16 bits [M, K].

    Returns (q uint8 [M, K], sfe uint8 [K/128, M]): each group's scale is 2^(sfe - 127),
    the smallest power of two p with 448 p >= amax.
    """
    x = _c(x_bf16_bits, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.uint8)
    sfe = np.empty((K // GROUP, M), dtype=np.uint8)
    _check(_load().oracle_quantize_ue8m0_groups(_ptr(x), M, K, K, _ptr(q), K, _ptr(sfe)),
           "quantize_ue8m0_groups")
    return q, sfe


def quantize_ue8m0_blocks(w_bf16_bits: np.ndarray):
    """UE8M0 recipe, 128x128 weight blocks: (q uint8 [N, K], sfe uint8 [ceil(N/128), K/128])."""
    w = _c(w_bf16_bits, np.uint16)
    N, K = w.shape
    q = np.empty((N, K), dtype=np.uint8)
    sfe = np.empty((-(-N // GROUP), K // GROUP), dtype=np.uint8)
    _check(_load().oracle_quantize_ue8m0_blocks(_ptr(w), N, K, _ptr(q), _ptr(sfe)),
           "quantize_ue8m0_blocks")
    return q, sfe


def ue8m0_value(sfe) -> np.ndarray:
    """The scale 2^(b - 127) of UE8M0 bytes, as float32 (exact for b in 0..254)."""
    b = np.asarray(sfe, dtype=np.int32)
    return np.ldexp(np.float32(1.0), b - 127).astype(np.float32)


MX_BLOCK = 32


def quantize_mxfp8(x_bf16_bits: np.ndarray):
    """MXFP8 gran-32: every row of a bf16 matrix (uint16 bits [R, K]) in 1x32 blocks
    along K, each with the UE8M0 scale 2^(sfe - 127), the smallest power of two p with
    448 p >= amax (deepgemm-rust README, benchmark block "SM100 FP8: DeepSeek gran-128
    recipe and MXFP8 gran-32").  Returns (q uint8 [R, K], sfe uint8 [R, K/32])."""
    x = _c(x_bf16_bits, np.uint16)
    R, K = x.shape
    q = np.empty((R, K), dtype=np.uint8)
    sfe = np.empty((R, K // MX_BLOCK), dtype=np.uint8)
    _check(_load().oracle_quantize_mxfp8(_ptr(x), R, K, K, _ptr(q), K, _ptr(sfe)), "quantize_mxfp8")
    return q, sfe


def gemm_nt_mx32(qa, ea, qb, eb) -> np.ndarray:
    """FP64 D [M, N] of two MXFP8 gran-32 operands: codes qa [M, K], qb [N, K] with
    exponent bytes ea [M, K/32], eb [N, K/32]."""
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    ea = _c(ea, np.uint8)
    eb = _c(eb, np.uint8)
    M, K = qa.shape
    N = qb.shape[0]
    D = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_gemm_nt_mx32(_ptr(qa), _ptr(ea), _ptr(qb), _ptr(eb), M, N, K, _ptr(D)), "gemm_nt_mx32")
    return D
