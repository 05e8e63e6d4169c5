"""Block-scaled FP8 linear for NVIDIA B200 (sm_100a): Python binding of liblnq.so.

The functions named ``lnq_*`` mirror the C ABI in ``include/lnq.h`` one to one;
they only marshal torch tensors to pointers, sizes and the current CUDA stream
and raise :class:`LnqError` on a non-zero status.  Every step of the path runs
in the CUDA kernels of ``liblnq.so``; there is no CPU fallback, and a missing
library raises.

Numerics: activations quantized per row in 1x128 groups and weights in
128x128 blocks to E4M3 with FP32 scales amax/448; the product of each 128-wide
K block accumulated in FP32 on the tensor cores and promoted by sa*sb in FP32;
BF16 output (Linnet "Backend plugins", DeepGEMM plugin; deepgemm-rust README,
"What's implemented").

The helpers below the ABI wrappers (``quantize_activations``,
``quantize_weights``, ``linear``, ``m_grouped_linear``) allocate their outputs
with torch and call the same entry points.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "LnqError", "library_path", "lib",
    "lnq_quantize_fp8_groups", "lnq_quantize_fp8_blocks", "lnq_fp8_block_gemm_nt",
    "lnq_m_grouped_fp8_gemm_contiguous", "lnq_m_grouped_fp8_gemm_contiguous_psum",
    "lnq_fp8_block_gemm_nt_silu_mul", "lnq_mx_block_gemm_nt", "lnq_m_grouped_mx_gemm_contiguous", "quantize_activations_ue8m0",
    "quantize_weights_ue8m0", "ue8m0_atoms", "quantize_mxfp8", "lnq_mxfp8_gemm_nt",
    "lnq_m_grouped_mxfp8_gemm_contiguous", "lnq_m_grouped_mx_gemm_masked", "lnq_m_grouped_mxfp8_gemm_masked",
    "lnq_m_grouped_fp8_gemm_masked", "lnq_get_last_device_error", "lnq_status_string",
    "lnq_selftest_wait_timeout", "lnq_set_dense_cta_pairs", "lnq_set_grouped_cta_pairs",
    "lnq_set_weight_prefetch", "lnq_set_tma_store",
    "quantize_activations", "quantize_weights",
    "quantize_weights_grouped", "linear",
    "m_grouped_linear", "ceil4",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liblnq.so")
_lock = threading.Lock()
_lib = None

LNQ_OK = 0
STATUS_NAMES = {
    0: "LNQ_OK", 1: "LNQ_ERR_INVALID_ARG", 2: "LNQ_ERR_UNSUPPORTED_SHAPE", 3: "LNQ_ERR_MISALIGNED",
    4: "LNQ_ERR_UNSUPPORTED_ARCH", 5: "LNQ_ERR_CUDA", 6: "LNQ_ERR_TIMEOUT",
}


class LnqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS_NAMES.get(self.status, self.status)} "
                         f"({lnq_status_string(self.status)})")


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded liblnq.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m moe_grouped_gemm_quantize_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        sigs = {
            "lnq_quantize_fp8_groups": [P, I64, I64, I64, P, I64, P, I64, P],
            "lnq_quantize_fp8_blocks": [P, I64, I64, P, P, P],
            "lnq_fp8_block_gemm_nt": [P, P, I64, P, P, P, I64, I64, I64, P],
            "lnq_fp8_block_gemm_nt_ws": [P, P, I64, P, P, P, I64, I64, I64, P, I64, P],
            "lnq_fp8_block_gemm_nt_epilogue": [P, P, I64, P, P, P, P, P, P, I64, I64, I64, I64, P],
            "lnq_fp8_block_gemm_nt_static_ws": [P, P, I64, P, P, P, I64, I64, I64, P],
            "lnq_m_grouped_fp8_gemm_contiguous": [P, P, P, P, P, I32, P, I64, I64, I64, P],
            "lnq_m_grouped_fp8_gemm_masked": [P, P, P, P, P, I32, I64, I64, P, I64, I64, P],
            "lnq_m_grouped_fp8_gemm_contiguous_psum": [P, P, P, P, P, I32, I64, P, I64, I64, I64, P],
            "lnq_fp8_block_gemm_nt_silu_mul": [P, P, I64, P, P, P, I64, I64, I64, P],
            "lnq_quantize_ue8m0_groups": [P, I64, I64, I64, P, I64, P, P],
            "lnq_quantize_ue8m0_blocks": [P, I64, I64, P, P, P],
            "lnq_mx_block_gemm_nt": [P, P, P, P, P, I64, I64, I64, P],
            "lnq_m_grouped_mx_gemm_contiguous": [P, P, P, P, P, I32, P, I64, I64, I64, P],
            "lnq_quantize_mxfp8": [P, I64, I64, I64, P, I64, P, P],
            "lnq_mxfp8_gemm_nt": [P, P, P, P, P, I64, I64, I64, P],
            "lnq_m_grouped_mxfp8_gemm_contiguous": [P, P, P, P, P, I32, P, I64, I64, I64, P],
            "lnq_m_grouped_mx_gemm_masked": [P, P, P, P, P, I32, I64, I64, P, I64, I64, P],
            "lnq_m_grouped_mxfp8_gemm_masked": [P, P, P, P, P, I32, I64, I64, P, I64, I64, P],
            "lnq_get_last_device_error": [P],
            "lnq_selftest_wait_timeout": [I64, P],
        }
        for name, args in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.lnq_status_string.argtypes = [ctypes.c_int]
        L.lnq_status_string.restype = ctypes.c_char_p
        L.lnq_abi_version.restype = ctypes.c_int32
        L.lnq_fp8_block_gemm_nt_workspace_bytes.argtypes = [I64, I64, I64, I32]
        L.lnq_fp8_block_gemm_nt_workspace_bytes.restype = I64
        for knob in ("lnq_set_dense_cta_pairs", "lnq_set_grouped_cta_pairs", "lnq_set_weight_prefetch",
                     "lnq_set_tma_store"):
            getattr(L, knob).argtypes = [ctypes.c_int32]
            getattr(L, knob).restype = ctypes.c_int32
        _lib = L
        return L


def lnq_status_string(status: int) -> str:
    return lib().lnq_status_string(int(status)).decode()


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


def _check(rc: int, where: str) -> None:
    if rc != LNQ_OK:
        raise LnqError(rc, where)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _is_fp8(t: torch.Tensor) -> bool:
    return t.dtype in (torch.float8_e4m3fn, torch.uint8)


def ceil4(m: int) -> int:
    return -(-int(m) // 4) * 4


# ----------------------------------------------------------------- the C ABI

def lnq_quantize_fp8_groups(x: torch.Tensor, q: torch.Tensor, sfa: torch.Tensor, stream=None) -> None:
    """x bf16 [M, K] (row stride ld_x), q e4m3 [M, K] (row stride ld_q), sfa fp32 [K/128, M4]."""
    if x.dtype != torch.bfloat16 or not _is_fp8(q) or sfa.dtype != torch.float32:
        raise TypeError("x must be bf16, q float8_e4m3fn/uint8, sfa float32")
    M, K = x.shape
    if x.stride(1) != 1 or q.stride(1) != 1 or not sfa.is_contiguous() or tuple(q.shape) != (M, K):
        raise ValueError("x, q need unit column stride, sfa must be contiguous, q shaped like x")
    if sfa.shape[0] != K // 128:
        raise ValueError("sfa must be [K/128, M4]")
    _check(lib().lnq_quantize_fp8_groups(_ptr(x), M, K, x.stride(0), _ptr(q), q.stride(0),
                                         _ptr(sfa), sfa.shape[1], _stream(stream)),
           "lnq_quantize_fp8_groups")


def lnq_quantize_fp8_blocks(w: torch.Tensor, q: torch.Tensor, sfb: torch.Tensor, stream=None) -> None:
    """w bf16 [N, K], q e4m3 [N, K], sfb fp32 [ceil(N/128), K/128], all contiguous."""
    if w.dtype != torch.bfloat16 or not _is_fp8(q) or sfb.dtype != torch.float32:
        raise TypeError("w must be bf16, q float8_e4m3fn/uint8, sfb float32")
    N, K = w.shape
    if not (w.is_contiguous() and q.is_contiguous() and sfb.is_contiguous()):
        raise ValueError("w, q, sfb must be contiguous")
    if tuple(q.shape) != (N, K) or tuple(sfb.shape) != (-(-N // 128), K // 128):
        raise ValueError("q must be [N, K] and sfb [ceil(N/128), K/128]")
    _check(lib().lnq_quantize_fp8_blocks(_ptr(w), N, K, _ptr(q), _ptr(sfb), _stream(stream)),
           "lnq_quantize_fp8_blocks")


def lnq_fp8_block_gemm_nt(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                          d: torch.Tensor, stream=None) -> None:
    """a e4m3 [M, K], sfa fp32 [K/128, M4], b e4m3 [N, K], sfb fp32 [ceil(N/128), K/128], d bf16 [M, N]."""
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.float32 or \
            sfb.dtype != torch.float32 or d.dtype != torch.bfloat16:
        raise TypeError("a, b float8_e4m3fn/uint8; sfa, sfb float32; d bf16")
    M, K = a.shape
    N = b.shape[0]
    for t in (a, sfa, b, sfb, d):
        if not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    if b.shape[1] != K or tuple(d.shape) != (M, N) or sfa.shape[0] != K // 128 or \
            tuple(sfb.shape) != (-(-N // 128), K // 128):
        raise ValueError("inconsistent shapes")
    _check(lib().lnq_fp8_block_gemm_nt(_ptr(a), _ptr(sfa), sfa.shape[1], _ptr(b), _ptr(sfb), _ptr(d),
                                       M, N, K, _stream(stream)), "lnq_fp8_block_gemm_nt")


def lnq_fp8_block_gemm_nt_epilogue(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                                   bias: torch.Tensor | None = None, d: torch.Tensor | None = None,
                                   q: torch.Tensor | None = None, sfa_out: torch.Tensor | None = None,
                                   stream=None) -> None:
    """The GEMM with a fused epilogue: bias (bf16 [N] or None) added in FP32, and either d
    (bf16 [M, N]) or q (E4M3 [M, N]) with sfa_out (fp32 [N/128, M4_out]) written."""
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.float32 or sfb.dtype != torch.float32:
        raise TypeError("a, b float8_e4m3fn/uint8; sfa, sfb float32")
    if (d is None) == (q is None):
        raise ValueError("give exactly one of d and q")
    if d is not None and d.dtype != torch.bfloat16:
        raise TypeError("d bf16")
    if q is not None and (not _is_fp8(q) or sfa_out is None or sfa_out.dtype != torch.float32):
        raise TypeError("q float8_e4m3fn/uint8 with sfa_out float32")
    if bias is not None and bias.dtype != torch.bfloat16:
        raise TypeError("bias bf16")
    M, K = a.shape
    N = b.shape[0]
    for t in (a, sfa, b, sfb, bias, d, q, sfa_out):
        if t is not None and not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    out = d if d is not None else q
    if b.shape[1] != K or tuple(out.shape) != (M, N) or sfa.shape[0] != K // 128 or \
            tuple(sfb.shape) != (-(-N // 128), K // 128) or (bias is not None and bias.numel() != N) or \
            (sfa_out is not None and sfa_out.shape[0] != N // 128):
        raise ValueError("inconsistent shapes")
    nul = ctypes.c_void_p(0)
    _check(lib().lnq_fp8_block_gemm_nt_epilogue(
        _ptr(a), _ptr(sfa), sfa.shape[1], _ptr(b), _ptr(sfb), _ptr(bias) if bias is not None else nul,
        _ptr(d) if d is not None else nul, _ptr(q) if q is not None else nul,
        _ptr(sfa_out) if sfa_out is not None else nul, sfa_out.shape[1] if sfa_out is not None else 0,
        M, N, K, _stream(stream)), "lnq_fp8_block_gemm_nt_epilogue")


def lnq_fp8_block_gemm_nt_workspace_bytes(M: int, N: int, K: int, num_sms: int) -> int:
    """Workspace bytes for the decode K split over num_sms CTAs (0: the product does not split)."""
    return int(lib().lnq_fp8_block_gemm_nt_workspace_bytes(M, N, K, num_sms))


def gemm_workspace(M: int, N: int, K: int, device) -> torch.Tensor | None:
    """A zeroed workspace for lnq_fp8_block_gemm_nt_ws on `device`, or None when the
    product does not split.  The library leaves it zeroed after every call."""
    dev = torch.device(device)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    n = lnq_fp8_block_gemm_nt_workspace_bytes(M, N, K, sms)
    if n == 0:
        return None
    return torch.zeros(n, dtype=torch.uint8, device=dev)


def lnq_fp8_block_gemm_nt_static_ws(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                                    d: torch.Tensor, stream=None) -> None:
    """lnq_fp8_block_gemm_nt_ws with the library's fixed 10 MiB device scratch (no allocation;
    calls must not overlap in time)."""
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.float32 or \
            sfb.dtype != torch.float32 or d.dtype != torch.bfloat16:
        raise TypeError("a, b float8_e4m3fn/uint8; sfa, sfb float32; d bf16")
    M, K = a.shape
    N = b.shape[0]
    for t in (a, sfa, b, sfb, d):
        if not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    if b.shape[1] != K or tuple(d.shape) != (M, N) or sfa.shape[0] != K // 128 or \
            tuple(sfb.shape) != (-(-N // 128), K // 128):
        raise ValueError("inconsistent shapes")
    _check(lib().lnq_fp8_block_gemm_nt_static_ws(_ptr(a), _ptr(sfa), sfa.shape[1], _ptr(b), _ptr(sfb),
                                                 _ptr(d), M, N, K, _stream(stream)),
           "lnq_fp8_block_gemm_nt_static_ws")


def lnq_fp8_block_gemm_nt_ws(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                             d: torch.Tensor, workspace: torch.Tensor | None, stream=None) -> None:
    """lnq_fp8_block_gemm_nt with the decode K split over a caller-owned workspace
    (uint8 tensor from gemm_workspace, or None for the unsplit product)."""
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.float32 or \
            sfb.dtype != torch.float32 or d.dtype != torch.bfloat16:
        raise TypeError("a, b float8_e4m3fn/uint8; sfa, sfb float32; d bf16")
    M, K = a.shape
    N = b.shape[0]
    for t in (a, sfa, b, sfb, d):
        if not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    if b.shape[1] != K or tuple(d.shape) != (M, N) or sfa.shape[0] != K // 128 or \
            tuple(sfb.shape) != (-(-N // 128), K // 128):
        raise ValueError("inconsistent shapes")
    if workspace is None:
        ws, ws_bytes = ctypes.c_void_p(0), 0
    else:
        if workspace.dtype != torch.uint8 or not workspace.is_contiguous():
            raise TypeError("workspace: contiguous uint8 tensor")
        ws, ws_bytes = _ptr(workspace), workspace.numel()
    _check(lib().lnq_fp8_block_gemm_nt_ws(_ptr(a), _ptr(sfa), sfa.shape[1], _ptr(b), _ptr(sfb), _ptr(d),
                                          M, N, K, ws, ws_bytes, _stream(stream)), "lnq_fp8_block_gemm_nt_ws")


def lnq_m_grouped_fp8_gemm_contiguous(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor,
                                      sfb: torch.Tensor, m_indices: torch.Tensor, num_groups: int,
                                      d: torch.Tensor, stream=None) -> None:
    """a e4m3 [M_total, K], sfa [K/128, M_total], b e4m3 [G*N, K], sfb [G*ceil(N/128), K/128],
    m_indices int32 [M_total], d bf16 [M_total, N]."""
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.float32 or \
            sfb.dtype != torch.float32 or d.dtype != torch.bfloat16 or m_indices.dtype != torch.int32:
        raise TypeError("a, b e4m3; sfa, sfb float32; m_indices int32; d bf16")
    for t in (a, sfa, b, sfb, m_indices, d):
        if not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    M_total, K = a.shape
    G = int(num_groups)
    N = d.shape[1]
    if b.shape[0] != G * N or b.shape[1] != K or tuple(sfa.shape) != (K // 128, M_total) or \
            tuple(sfb.shape) != (G * -(-N // 128), K // 128) or m_indices.shape[0] != M_total or \
            d.shape[0] != M_total:
        raise ValueError("inconsistent shapes")
    _check(lib().lnq_m_grouped_fp8_gemm_contiguous(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb),
                                                   _ptr(m_indices), G, _ptr(d), M_total, N, K,
                                                   _stream(stream)),
           "lnq_m_grouped_fp8_gemm_contiguous")


def lnq_fp8_block_gemm_nt_silu_mul(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                                   h: torch.Tensor, stream=None) -> None:
    """Gate_up linear with SiLU.mul: a e4m3 [M, K], sfa [K/128, M4], b e4m3 [2I, K] (gate rows
    then up rows), sfb [2I/128, K/128], h bf16 [M, I] = silu(D[:, :I]) * D[:, I:]."""
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.float32 or sfb.dtype != torch.float32 or \
            h.dtype != torch.bfloat16:
        raise TypeError("a, b e4m3; sfa, sfb float32; h bf16")
    for t in (a, sfa, b, sfb, h):
        if not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    M, K = a.shape
    I = h.shape[1]
    if b.shape[0] != 2 * I or b.shape[1] != K or h.shape[0] != M or sfa.shape[0] != K // 128 or \
            tuple(sfb.shape) != (-(-2 * I // 128), K // 128):
        raise ValueError("inconsistent shapes")
    _check(lib().lnq_fp8_block_gemm_nt_silu_mul(_ptr(a), _ptr(sfa), sfa.shape[1], _ptr(b), _ptr(sfb), _ptr(h),
                                                M, I, K, _stream(stream)),
           "lnq_fp8_block_gemm_nt_silu_mul")


def ue8m0_atoms(rows: int, K: int, device) -> torch.Tensor:
    """Scale-atom storage of the UE8M0 recipe: uint32-valued int32 [K/128, ceil(rows/128)*128]."""
    return torch.empty((K // 128, -(-rows // 128) * 128), dtype=torch.int32, device=device)


def quantize_activations_ue8m0(x: torch.Tensor, stream=None):
    """UE8M0 recipe, 1x128 groups: (q e4m3 [M, K], scale atoms int32 [K/128, ceil(M/128)*128])."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise TypeError("x must be a row-major bf16 matrix")
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    sf = ue8m0_atoms(M, K, x.device)
    _check(lib().lnq_quantize_ue8m0_groups(_ptr(x), M, K, x.stride(0), _ptr(q), K, _ptr(sf), _stream(stream)),
           "lnq_quantize_ue8m0_groups")
    return q, sf


def quantize_weights_ue8m0(w: torch.Tensor, stream=None):
    """UE8M0 recipe, 128x128 blocks: (q e4m3 [N, K], scale atoms int32 [K/128, ceil(N/128)*128])."""
    if w.dtype != torch.bfloat16 or w.dim() != 2 or not w.is_contiguous():
        raise TypeError("w must be a contiguous bf16 matrix")
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.float8_e4m3fn, device=w.device)
    sf = ue8m0_atoms(N, K, w.device)
    _check(lib().lnq_quantize_ue8m0_blocks(_ptr(w), N, K, _ptr(q), _ptr(sf), _stream(stream)),
           "lnq_quantize_ue8m0_blocks")
    return q, sf


def lnq_mx_block_gemm_nt(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                         d: torch.Tensor, stream=None) -> None:
    """UE8M0 recipe GEMM: a e4m3 [M, K], b e4m3 [N, K], their scale atoms, d bf16 [M, N]."""
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.int32 or sfb.dtype != torch.int32 or \
            d.dtype != torch.bfloat16:
        raise TypeError("a, b e4m3; sfa, sfb int32 scale atoms; d bf16")
    for t in (a, sfa, b, sfb, d):
        if not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K or tuple(d.shape) != (M, N) or tuple(sfa.shape) != (K // 128, -(-M // 128) * 128) or \
            tuple(sfb.shape) != (K // 128, -(-N // 128) * 128):
        raise ValueError("inconsistent shapes")
    _check(lib().lnq_mx_block_gemm_nt(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), M, N, K, _stream(stream)),
           "lnq_mx_block_gemm_nt")


def lnq_m_grouped_mx_gemm_contiguous(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                                     m_indices: torch.Tensor, num_groups: int, d: torch.Tensor,
                                     stream=None) -> None:
    """UE8M0 recipe, M-grouped contiguous: a e4m3 [M_total, K] and its scale atoms, b e4m3 [G*N, K]
    and its scale atoms, m_indices int32 [M_total], d bf16 [M_total, N]."""
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.int32 or sfb.dtype != torch.int32 or \
            d.dtype != torch.bfloat16 or m_indices.dtype != torch.int32:
        raise TypeError("a, b e4m3; sfa, sfb int32 scale atoms; m_indices int32; d bf16")
    for t in (a, sfa, b, sfb, m_indices, d):
        if not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    M_total, K = a.shape
    G = int(num_groups)
    N = d.shape[1]
    if b.shape[0] != G * N or b.shape[1] != K or d.shape[0] != M_total or m_indices.shape[0] != M_total or \
            tuple(sfa.shape) != (K // 128, -(-M_total // 128) * 128) or \
            tuple(sfb.shape) != (K // 128, -(-G * N // 128) * 128):
        raise ValueError("inconsistent shapes")
    _check(lib().lnq_m_grouped_mx_gemm_contiguous(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(m_indices), G,
                                                  _ptr(d), M_total, N, K, _stream(stream)),
           "lnq_m_grouped_mx_gemm_contiguous")


def quantize_mxfp8(x: torch.Tensor, stream=None):
    """MXFP8 gran-32: every row in 1x32 blocks along K (activations and weights alike):
    (q e4m3 [rows, K], scale atoms int32 [K/128, ceil(rows/128)*128], four exponent bytes
    per word)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise TypeError("x must be a row-major bf16 matrix")
    R, K = x.shape
    q = torch.empty((R, K), dtype=torch.float8_e4m3fn, device=x.device)
    sf = ue8m0_atoms(R, K, x.device)
    _check(lib().lnq_quantize_mxfp8(_ptr(x), R, K, x.stride(0), _ptr(q), K, _ptr(sf), _stream(stream)),
           "lnq_quantize_mxfp8")
    return q, sf


def lnq_mxfp8_gemm_nt(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                      d: torch.Tensor, stream=None) -> None:
    """MXFP8 gran-32 GEMM: a e4m3 [M, K], b e4m3 [N, K], their scale atoms, d bf16 [M, N]."""
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.int32 or sfb.dtype != torch.int32 or \
            d.dtype != torch.bfloat16:
        raise TypeError("a, b e4m3; sfa, sfb int32 scale atoms; d bf16")
    for t in (a, sfa, b, sfb, d):
        if not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K or tuple(d.shape) != (M, N) or tuple(sfa.shape) != (K // 128, -(-M // 128) * 128) or \
            tuple(sfb.shape) != (K // 128, -(-N // 128) * 128):
        raise ValueError("inconsistent shapes")
    _check(lib().lnq_mxfp8_gemm_nt(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), M, N, K, _stream(stream)),
           "lnq_mxfp8_gemm_nt")


def lnq_m_grouped_mxfp8_gemm_contiguous(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                                        m_indices: torch.Tensor, num_groups: int, d: torch.Tensor,
                                        stream=None) -> None:
    """MXFP8 gran-32, M-grouped contiguous: as lnq_m_grouped_mx_gemm_contiguous with the scale
    atoms of lnq_quantize_mxfp8 on both operands."""
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.int32 or sfb.dtype != torch.int32 or \
            d.dtype != torch.bfloat16 or m_indices.dtype != torch.int32:
        raise TypeError("a, b e4m3; sfa, sfb int32 scale atoms; m_indices int32; d bf16")
    for t in (a, sfa, b, sfb, m_indices, d):
        if not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    M_total, K = a.shape
    G = int(num_groups)
    N = d.shape[1]
    if b.shape[0] != G * N or b.shape[1] != K or d.shape[0] != M_total or m_indices.shape[0] != M_total or \
            tuple(sfa.shape) != (K // 128, -(-M_total // 128) * 128) or \
            tuple(sfb.shape) != (K // 128, -(-G * N // 128) * 128):
        raise ValueError("inconsistent shapes")
    _check(lib().lnq_m_grouped_mxfp8_gemm_contiguous(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(m_indices), G,
                                                     _ptr(d), M_total, N, K, _stream(stream)),
           "lnq_m_grouped_mxfp8_gemm_contiguous")


def _mx_masked(fn_name: str, a, sfa, b, sfb, masked_m, d, expected_m, stream) -> None:
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.int32 or sfb.dtype != torch.int32 or \
            d.dtype != torch.bfloat16 or masked_m.dtype != torch.int32:
        raise TypeError("a, b e4m3; sfa, sfb int32 scale atoms; masked_m int32; d bf16")
    G = masked_m.numel()
    if a.dim() == 3:
        if a.shape[0] != G:
            raise ValueError("a's first dimension must be the number of groups")
        M_max, K = a.shape[1], a.shape[2]
    else:
        M_max, K = a.shape[0] // G, a.shape[1]
    N = (b.shape[1] if b.dim() == 3 else b.shape[0] // G)
    for t in (a, sfa, b, sfb, masked_m, d):
        if not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    if a.numel() != G * M_max * K or b.numel() != G * N * K or d.numel() != G * M_max * N or \
            tuple(sfa.shape) != (K // 128, -(-G * M_max // 128) * 128) or \
            tuple(sfb.shape) != (K // 128, -(-G * N // 128) * 128):
        raise ValueError("inconsistent shapes")
    _check(getattr(lib(), fn_name)(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(masked_m), G, M_max,
                                   int(expected_m), _ptr(d), N, K, _stream(stream)), fn_name)


def lnq_m_grouped_mx_gemm_masked(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                                 masked_m: torch.Tensor, d: torch.Tensor, expected_m: int = 0,
                                 stream=None) -> None:
    """UE8M0 recipe, M-grouped masked: a e4m3 [G, M_max, K] (or [G*M_max, K]) and its scale atoms
    over G*M_max rows, b e4m3 [G*N, K] and its atoms, masked_m int32 [G] on the device, d bf16
    [G*M_max, N]: group g's first masked_m[g] rows of d are written."""
    _mx_masked("lnq_m_grouped_mx_gemm_masked", a, sfa, b, sfb, masked_m, d, expected_m, stream)


def lnq_m_grouped_mxfp8_gemm_masked(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                                    masked_m: torch.Tensor, d: torch.Tensor, expected_m: int = 0,
                                    stream=None) -> None:
    """MXFP8 gran-32, M-grouped masked: as lnq_m_grouped_mx_gemm_masked with the scale atoms of
    lnq_quantize_mxfp8 on both operands."""
    _mx_masked("lnq_m_grouped_mxfp8_gemm_masked", a, sfa, b, sfb, masked_m, d, expected_m, stream)


def lnq_m_grouped_fp8_gemm_contiguous_psum(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor,
                                           sfb: torch.Tensor, psum: torch.Tensor, d: torch.Tensor,
                                           alignment: int = 128, stream=None) -> None:
    """a e4m3 [M_total, K], sfa [K/128, M_total], b e4m3 [G*N, K], sfb [G*ceil(N/128), K/128],
    psum int32 [G] on the device (tokens of groups 0..g), d bf16 [M_total, N]; group g's tokens
    start at the sum of the earlier groups' counts rounded up to `alignment` (128 or 256)."""
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.float32 or \
            sfb.dtype != torch.float32 or d.dtype != torch.bfloat16 or psum.dtype != torch.int32:
        raise TypeError("a, b e4m3; sfa, sfb float32; psum int32; d bf16")
    for t in (a, sfa, b, sfb, psum, d):
        if not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    M_total, K = a.shape
    G = psum.numel()
    N = d.shape[1]
    if G == 0 or b.shape[0] != G * N or b.shape[1] != K or tuple(sfa.shape) != (K // 128, M_total) or \
            tuple(sfb.shape) != (G * -(-N // 128), K // 128) or d.shape[0] != M_total:
        raise ValueError("inconsistent shapes")
    _check(lib().lnq_m_grouped_fp8_gemm_contiguous_psum(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(psum), G,
                                                        int(alignment), _ptr(d), M_total, N, K, _stream(stream)),
           "lnq_m_grouped_fp8_gemm_contiguous_psum")


def lnq_m_grouped_fp8_gemm_masked(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                                  masked_m: torch.Tensor, d: torch.Tensor, expected_m: int = 0,
                                  stream=None) -> None:
    """a e4m3 [G, M_max, K] (or [G*M_max, K]), sfa fp32 [K/128, G*M_max], b e4m3 [G*N, K] (or
    [G, N, K]), sfb fp32 [G*ceil(N/128), K/128], masked_m int32 [G] on the device, d bf16
    [G, M_max, N] (or [G*M_max, N]): group g's first masked_m[g] rows of d are written."""
    if not (_is_fp8(a) and _is_fp8(b)) or sfa.dtype != torch.float32 or sfb.dtype != torch.float32 or \
            d.dtype != torch.bfloat16 or masked_m.dtype != torch.int32:
        raise TypeError("a, b float8_e4m3fn/uint8; sfa, sfb float32; masked_m int32; d bf16")
    G = masked_m.numel()
    if a.dim() == 3:
        if a.shape[0] != G:
            raise ValueError("a's first dimension must be the number of groups")
        M_max, K = a.shape[1], a.shape[2]
    else:
        M_max, K = a.shape[0] // G, a.shape[1]
    N = (b.shape[1] if b.dim() == 3 else b.shape[0] // G)
    for t in (a, sfa, b, sfb, masked_m, d):
        if not t.is_contiguous():
            raise ValueError("all operands must be contiguous")
    if a.numel() != G * M_max * K or b.numel() != G * N * K or d.numel() != G * M_max * N or \
            tuple(sfa.shape) != (K // 128, G * M_max) or tuple(sfb.shape) != (G * -(-N // 128), K // 128):
        raise ValueError("inconsistent shapes")
    _check(lib().lnq_m_grouped_fp8_gemm_masked(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(masked_m), G,
                                               M_max, expected_m, _ptr(d), N, K, _stream(stream)),
           "lnq_m_grouped_fp8_gemm_masked")


def lnq_get_last_device_error(stream=None) -> int:
    """Synchronizes the stream; returns (and clears) the device-reported status."""
    return int(lib().lnq_get_last_device_error(_stream(stream)))


def lnq_set_dense_cta_pairs(mode: int) -> int:
    """Dense GEMM configuration for M > 128: 0 one CTA per 128x256 tile, 1 CTA pairs on
    256x256 tiles, 2 CTA pairs on 256x128 tiles (the block-scaled UE8M0 / MXFP8 GEMMs:
    0 single CTAs, otherwise CTA pairs on 256x256 tiles).  Returns the previous setting."""
    return int(lib().lnq_set_dense_cta_pairs(int(mode)))


def lnq_set_grouped_cta_pairs(mode: int) -> int:
    """Prefix-sum grouped GEMM with 256-row alignment: 1 runs 256x256 tiles on CTA pairs,
    0 (the default) 128-row tiles on single CTAs.  Returns the previous setting."""
    return int(lib().lnq_set_grouped_cta_pairs(int(mode)))


def lnq_set_weight_prefetch(enable: bool) -> bool:
    """Let GEMMs stream their first weight stages before the previous kernel of the
    stream completes (weights must not be written by still-running kernels)."""
    return bool(lib().lnq_set_weight_prefetch(1 if enable else 0))


def lnq_set_tma_store(enable: bool) -> bool:
    """Dense and grouped GEMM outputs through shared memory and TMA stores (True, the
    default) or stored row by row from registers (False).  Returns the previous setting."""
    return bool(lib().lnq_set_tma_store(1 if enable else 0))


def lnq_selftest_wait_timeout(timeout_ns: int, stream=None) -> None:
    _check(lib().lnq_selftest_wait_timeout(int(timeout_ns), _stream(stream)),
           "lnq_selftest_wait_timeout")


# ----------------------------------------------------------------- helpers

def quantize_activations(x: torch.Tensor, stream=None):
    """(q e4m3 [M, K], sfa fp32 [K/128, ceil4(M)]) of a bf16 [M, K] CUDA tensor."""
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    sfa = torch.empty((K // 128, ceil4(M)), dtype=torch.float32, device=x.device)
    lnq_quantize_fp8_groups(x, q, sfa, stream)
    return q, sfa


def quantize_weights(w: torch.Tensor, stream=None):
    """(q e4m3 [N, K], sfb fp32 [ceil(N/128), K/128]) of a bf16 [N, K] CUDA tensor."""
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.float8_e4m3fn, device=w.device)
    sfb = torch.empty((-(-N // 128), K // 128), dtype=torch.float32, device=w.device)
    lnq_quantize_fp8_blocks(w.contiguous(), q, sfb, stream)
    return q, sfb


def quantize_weights_grouped(w: torch.Tensor, num_groups: int, stream=None):
    """Per-group 128x128 quantization of grouped weights [G*N, K]:
    (q e4m3 [G*N, K], sfb fp32 [G*ceil(N/128), K/128]).  Each group is quantized on
    its own, so no block spans two groups when N is not a multiple of 128."""
    GN, K = w.shape
    G = int(num_groups)
    N = GN // G
    NB = -(-N // 128)
    w = w.contiguous()
    q = torch.empty((GN, K), dtype=torch.float8_e4m3fn, device=w.device)
    sfb = torch.empty((G * NB, K // 128), dtype=torch.float32, device=w.device)
    for g in range(G):
        lnq_quantize_fp8_blocks(w[g * N:(g + 1) * N], q[g * N:(g + 1) * N],
                                sfb[g * NB:(g + 1) * NB], stream)
    return q, sfb


def linear(x: torch.Tensor, w_q: torch.Tensor, w_s: torch.Tensor, stream=None) -> torch.Tensor:
    """y = x . W^T in bf16 with x quantized on the fly (1x128) and W pre-quantized (128x128)."""
    q, sfa = quantize_activations(x, stream)
    d = torch.empty((x.shape[0], w_q.shape[0]), dtype=torch.bfloat16, device=x.device)
    lnq_fp8_block_gemm_nt(q, sfa, w_q, w_s, d, stream)
    return d


def m_grouped_linear(x: torch.Tensor, w_q: torch.Tensor, w_s: torch.Tensor, m_indices: torch.Tensor,
                     num_groups: int, stream=None) -> torch.Tensor:
    """Grouped y for the contiguous MoE layout (x rows already padded per group to 128)."""
    q, sfa = quantize_activations(x, stream)
    N = w_q.shape[0] // num_groups
    d = torch.empty((x.shape[0], N), dtype=torch.bfloat16, device=x.device)
    lnq_m_grouped_fp8_gemm_contiguous(q, sfa, w_q, w_s, m_indices, num_groups, d, stream)
    return d
