"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds input recipes only: random normal matrices rounded to bf16,
outlier 1x128 groups, seeded MoE group sizes and the padded contiguous group-id
layout.  It holds none of the quantization or product arithmetic, so both the
CUDA path and the CPU oracle can take their inputs from it without sharing any
of the method.

Recipes (the workloads of the block-scaled FP8 linear):
  * activations  A ~ N(0, 1), weights W ~ N(0, 0.02), drawn in fp32 with a
    seeded ``torch.Generator`` and rounded to bf16 (round to nearest even);
  * outliers: a seeded Bernoulli(p) over the 1x128 row groups of a matrix; the
    chosen groups are multiplied by a factor in fp32 before the bf16 rounding;
  * MoE sizes: ``numpy.random.default_rng(seed).multinomial(total, [1/G]*G)``;
  * contiguous layout: each group's rows start at a multiple of 128, pad rows
    carry group id -1 (the padded group-id layout of the Triton_Grouped_GEMM
    README, "Example DeepGEMM layout creation", and the deepgemm-rust README,
    "Grouped (contiguous) MoE GEMM").
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK = 128


def gaussian_f32(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device) * float(std)


def gaussian_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) drawn in fp32 and rounded to bf16."""
    return gaussian_f32(shape, std, seed, device).to(torch.bfloat16)


def outlier_group_mask(rows: int, cols: int, frac: float, seed: int, device="cpu") -> torch.Tensor:
    """Bool [rows, cols/128]: a seeded Bernoulli(frac) over the 1x128 row groups."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.rand((rows, cols // BLOCK), generator=g, device=device) < frac


def gaussian_bf16_with_outliers(shape, std: float, seed: int, outlier_seed: int,
                                frac: float = 0.05, factor: float = 100.0,
                                device="cpu") -> torch.Tensor:
    """N(0, std^2) in fp32, chosen 1x128 groups scaled by `factor` in fp32, then bf16."""
    rows, cols = shape
    x = gaussian_f32(shape, std, seed, device)
    mask = outlier_group_mask(rows, cols, frac, outlier_seed, device)
    scale = torch.where(mask, torch.tensor(factor, device=device), torch.tensor(1.0, device=device))
    x = (x.view(rows, cols // BLOCK, BLOCK) * scale.unsqueeze(-1)).view(rows, cols)
    return x.to(torch.bfloat16)


def moe_group_sizes(total: int = 16384, groups: int = 32, seed: int = 0) -> np.ndarray:
    return np.random.default_rng(seed).multinomial(total, [1.0 / groups] * groups).astype(np.int64)


def contiguous_layout(sizes, block: int = BLOCK):
    """Padded group-id layout: (m_indices int32 [M_total], starts int64 [G], M_total).

    Group g occupies rows starts[g] .. starts[g]+sizes[g]-1; the following rows up to
    the next multiple of `block` carry id -1.
    """
    sizes = np.asarray(sizes, dtype=np.int64)
    padded = -(-sizes // block) * block
    starts = np.concatenate([[0], np.cumsum(padded)[:-1]]).astype(np.int64)
    M_total = int(padded.sum())
    m_indices = np.full(M_total, -1, dtype=np.int32)
    for g, (s, n) in enumerate(zip(starts, sizes)):
        m_indices[s:s + n] = g
    return m_indices, starts, M_total


def psum_layout(sizes, alignment: int = 256):
    """Prefix-sum layout: (psum int32 [G], starts int64 [G], M_total).

    psum[g] counts the tokens of groups 0..g; group g occupies rows starts[g] ..
    starts[g]+sizes[g]-1, starts being the running sum of the sizes rounded up to
    `alignment`, and M_total the sum of all rounded sizes.
    """
    m_indices, starts, M_total = contiguous_layout(sizes, alignment)
    psum = np.cumsum(np.asarray(sizes, dtype=np.int64)).astype(np.int32)
    return psum, starts, M_total


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """The uint16 bit patterns of a CPU bf16 tensor (what the oracle reads)."""
    assert x.dtype == torch.bfloat16
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------------------
# The workloads, by name and size.

@dataclass(frozen=True)
class Linear:
    name: str
    M: int
    N: int
    K: int
    a_std: float = 1.0
    w_std: float = 0.02
    a_seed: int = 0
    w_seed: int = 1
    outliers: bool = False
    a_outlier_seed: int = 1
    w_outlier_seed: int = 2

    @property
    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.K


@dataclass(frozen=True)
class MoE:
    name: str = "moe_32x_n4096_k7168"
    total_rows: int = 16384
    groups: int = 32
    N: int = 4096
    K: int = 7168
    a_std: float = 1.0
    w_std: float = 0.02
    sizes_seed: int = 0
    a_seed: int = 0
    w_seed: int = 1
    sizes: tuple = field(default=None, compare=False)

    def group_sizes(self) -> np.ndarray:
        return moe_group_sizes(self.total_rows, self.groups, self.sizes_seed)

    @property
    def flops(self) -> float:
        return 2.0 * self.total_rows * self.N * self.K


@dataclass(frozen=True)
class MoEMasked:
    """Decode-time MoE after a token dispatch: every expert has a buffer of m_max rows,
    of which the first count[g] hold tokens (multinomial over the experts, capped)."""
    name: str = "moe_masked_32x128_n4096_k7168"
    tokens: int = 2048
    groups: int = 32
    m_max: int = 128
    N: int = 4096
    K: int = 7168
    a_std: float = 1.0
    w_std: float = 0.02
    counts_seed: int = 3
    a_seed: int = 70
    w_seed: int = 71

    def counts(self) -> np.ndarray:
        c = np.random.default_rng(self.counts_seed).multinomial(self.tokens, [1.0 / self.groups] * self.groups)
        return np.minimum(c, self.m_max).astype(np.int32)

    @property
    def real_rows(self) -> int:
        return int(self.counts().sum())

    @property
    def flops(self) -> float:
        return 2.0 * self.real_rows * self.N * self.K


TINY = Linear("tiny_128x256x512", 128, 256, 512)
PREFILL = (
    Linear("prefill_qkv_2048x6144x4096", 2048, 6144, 4096, a_seed=10, w_seed=11),
    Linear("prefill_o_2048x4096x4096", 2048, 4096, 4096, a_seed=20, w_seed=21),
    Linear("prefill_gate_up_2048x24576x4096", 2048, 24576, 4096, a_seed=30, w_seed=31),
    Linear("prefill_down_2048x4096x12288", 2048, 4096, 12288, a_seed=40, w_seed=41),
)
DECODE = tuple(Linear(f"decode_m{m}_12288x4096", m, 12288, 4096, a_seed=50 + m, w_seed=49)
               for m in (1, 8, 32, 64))
MOE = MoE()
MOE_MASKED = MoEMasked()
SQUARE = Linear("square_8192", 8192, 8192, 8192, a_std=1.0, w_std=1.0, a_seed=60, w_seed=61,
                outliers=True, a_outlier_seed=1, w_outlier_seed=2)


def make_linear_inputs(cfg: Linear, device="cpu"):
    """(A bf16 [M, K], W bf16 [N, K]) for a dense workload."""
    if cfg.outliers:
        a = gaussian_bf16_with_outliers((cfg.M, cfg.K), cfg.a_std, cfg.a_seed, cfg.a_outlier_seed,
                                        device=device)
        w = gaussian_bf16_with_outliers((cfg.N, cfg.K), cfg.w_std, cfg.w_seed, cfg.w_outlier_seed,
                                        device=device)
    else:
        a = gaussian_bf16((cfg.M, cfg.K), cfg.a_std, cfg.a_seed, device)
        w = gaussian_bf16((cfg.N, cfg.K), cfg.w_std, cfg.w_seed, device)
    return a, w


def make_moe_inputs(cfg: MoE = MOE, device="cpu", alignment: int = BLOCK):
    """(A bf16 [M_total, K] with zero pad rows, W bf16 [G*N, K], m_indices, sizes); each
    group's rows start at a multiple of `alignment`."""
    sizes = cfg.group_sizes()
    m_indices, _, M_total = contiguous_layout(sizes, alignment)
    a = gaussian_bf16((M_total, cfg.K), cfg.a_std, cfg.a_seed, device)
    pad = torch.from_numpy(m_indices < 0).to(device)
    a = a.masked_fill(pad.unsqueeze(1), 0.0)
    w = gaussian_bf16((cfg.groups * cfg.N, cfg.K), cfg.w_std, cfg.w_seed, device)
    return a, w, m_indices, sizes


def make_moe_masked_inputs(cfg: MoEMasked = MOE_MASKED, device="cpu"):
    """(A bf16 [G*m_max, K] with random rows past each count, W bf16 [G*N, K], counts)."""
    a = gaussian_bf16((cfg.groups * cfg.m_max, cfg.K), cfg.a_std, cfg.a_seed, device)
    w = gaussian_bf16((cfg.groups * cfg.N, cfg.K), cfg.w_std, cfg.w_seed, device)
    return a, w, cfg.counts()
