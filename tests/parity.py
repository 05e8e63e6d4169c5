"""Shared parity helpers for the GPU tests: the tolerance check and the oracle side.

Tolerances (the benchmark spec of the method): the quantize outputs are
bit-exact; a GEMM output D (bf16) against the oracle's FP64 D_ref satisfies
    ||D - D_ref||_F / ||D_ref||_F <= 4e-3,
    max |D - D_ref| / |D_ref| <= 2e-2 over |D_ref| > 1e-2 * max |D_ref|.
bf16 rounding of the output alone is at most 2^-9 relative per element, and FP32
accumulation over K <= 12288 adds well under 1e-4, so a failure means a bug.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from moe_grouped_gemm_quantize_b200 import synthetic

REL_FRO = 4e-3
REL_MAX = 2e-2
MASK_FRAC = 1e-2


def gemm_errors(d: np.ndarray, ref: np.ndarray, ref_absmax: float | None = None):
    """(Frobenius relative error, max relative error over the masked elements).  The mask
    keeps |D_ref| > 1e-2 * max|D_ref|, the max taken over the whole product: pass
    `ref_absmax` when d and ref are a part of it (rows of a grouped product)."""
    d = np.asarray(d, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert d.shape == ref.shape
    assert np.all(np.isfinite(d)), "non-finite output"
    fro = np.linalg.norm(d - ref) / max(np.linalg.norm(ref), 1e-300)
    top = np.abs(ref).max() if ref_absmax is None else ref_absmax
    mask = np.abs(ref) > MASK_FRAC * top
    mx = float((np.abs(d - ref)[mask] / np.abs(ref)[mask]).max()) if mask.any() else 0.0
    return float(fro), mx


def assert_gemm_close(d, ref, what="", ref_absmax: float | None = None):
    fro, mx = gemm_errors(d, ref, ref_absmax)
    assert fro <= REL_FRO, f"{what}: Frobenius relative error {fro:.3e} > {REL_FRO}"
    assert mx <= REL_MAX, f"{what}: max relative error {mx:.3e} > {REL_MAX}"
    return fro, mx


def to_f64(d: torch.Tensor) -> np.ndarray:
    return d.detach().float().cpu().numpy().astype(np.float64)


def codes(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def oracle_quantize_a(a_bf16: torch.Tensor, M4=None):
    return oracle.quantize_fp8_groups(synthetic.bf16_bits(a_bf16), M4)


def oracle_quantize_w(w_bf16: torch.Tensor):
    return oracle.quantize_fp8_blocks(synthetic.bf16_bits(w_bf16))


def sample_points(M: int, N: int, count: int, seed: int, full_row=None, full_col=None):
    """Random (row, col) points plus, optionally, one whole row and one whole column."""
    rng = np.random.default_rng(seed)
    rows = [rng.integers(0, M, count)]
    cols = [rng.integers(0, N, count)]
    if full_row is not None:
        rows.append(np.full(N, full_row))
        cols.append(np.arange(N))
    if full_col is not None:
        rows.append(np.arange(M))
        cols.append(np.full(M, full_col))
    return np.concatenate(rows).astype(np.int64), np.concatenate(cols).astype(np.int64)
