"""Whole-matrix oracle references of the full-size workloads, computed once per test
session and shared by the GPU parity tests.

Every full-size GEMM output is compared with the oracle element by element: the
whole of D, not sampled points.  The oracle is the plain FP64 definition
(``oracle.gemm_nt``), which takes tens of seconds per workload on the host cores,
so each reference is computed once and reused by every launch configuration that
produces the same product.

The M-grouped references are the definition of the grouped product itself: each
group's token rows times that group's weights, one dense oracle product per group
(deepgemm-rust README, "Grouped (contiguous) MoE GEMM").  The oracle's own grouped
functions agree with this loop of dense products on every layout the CPU tests pin.
"""
from __future__ import annotations

import functools

import numpy as np

import oracle
from moe_grouped_gemm_quantize_b200 import synthetic
from parity import oracle_quantize_a, oracle_quantize_w


@functools.lru_cache(maxsize=None)
def linear_inputs(name: str):
    """(A, W) bf16 CPU tensors of the named dense workload."""
    cfg = workload(name)
    return synthetic.make_linear_inputs(cfg)


def workload(name: str) -> synthetic.Linear:
    for cfg in (synthetic.TINY, *synthetic.PREFILL, *synthetic.DECODE, synthetic.SQUARE):
        if cfg.name == name:
            return cfg
    raise KeyError(name)


@functools.lru_cache(maxsize=None)
def linear_operands(name: str):
    """The oracle's own codes and scales (qa, sa, qb, sb) of the named workload."""
    a, w = linear_inputs(name)
    qa, sa = oracle_quantize_a(a)
    qb, sb = oracle_quantize_w(w)
    return qa, sa, qb, sb


@functools.lru_cache(maxsize=None)
def linear_ref(name: str) -> np.ndarray:
    """FP64 D_ref [M, N] of the named dense workload."""
    return oracle.gemm_nt(*linear_operands(name))


def grouped_weights(w, G: int):
    """Each group's [N, K] weights quantized on their own (blocks never span groups)."""
    N = w.shape[0] // G
    parts = [oracle_quantize_w(w[g * N:(g + 1) * N]) for g in range(G)]
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])


def grouped_ref(qa, sa, qb, sb, starts, counts, N: int) -> np.ndarray:
    """FP64 D [rows of qa, N]: rows starts[g] .. starts[g] + counts[g] - 1 get the dense
    oracle product with group g's weights; every other row is NaN."""
    M_total, K = qa.shape
    nb = -(-N // 128)
    D = np.full((M_total, N), np.nan, dtype=np.float64)
    for g, (s, n) in enumerate(zip(starts, counts)):
        s, n = int(s), int(n)
        if n == 0:
            continue
        D[s:s + n] = oracle.gemm_nt(qa[s:s + n], np.ascontiguousarray(sa[:, s:s + n]),
                                    qb[g * N:(g + 1) * N], sb[g * nb:(g + 1) * nb])
    return D


@functools.lru_cache(maxsize=None)
def moe_inputs():
    """The 32-expert MoE workload in the per-row group-id layout (128-row alignment):
    (A, W, m_indices, sizes, starts)."""
    a, w, m_indices, sizes = synthetic.make_moe_inputs(synthetic.MOE)
    _, starts, _ = synthetic.contiguous_layout(sizes)
    return a, w, m_indices, sizes, starts


@functools.lru_cache(maxsize=None)
def moe_ref() -> np.ndarray:
    """FP64 D_ref of the MoE workload over its arena rows (pad rows NaN)."""
    a, w, _, sizes, starts = moe_inputs()
    cfg = synthetic.MOE
    qa, sa = oracle_quantize_a(a)
    qb, sb = grouped_weights(w, cfg.groups)
    return grouped_ref(qa, sa, qb, sb, starts, sizes, cfg.N)
