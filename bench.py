#!/usr/bin/env python
"""Benchmark of the block-scaled FP8 linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload all|prefill|decode|moe|moe_psum|moe_masked|square|tiny]

One step is one pass of the hot path over one batch of synthetic input: for each
linear of the workload, the 1x128 activation quantize (lnq_quantize_fp8_groups)
and the block-scaled FP8 GEMM (lnq_fp8_block_gemm_nt, or the M-grouped
contiguous GEMM for `moe` (per-row group ids) and `moe_psum` (prefix sums, groups
aligned to 256 rows), or the masked one for `moe_masked`).  Weights are model
parameters: quantized to 128x128 blocks once, before timing
(lnq_quantize_fp8_blocks).

Default (`--workload all`): every timed workload, one after the other, in one JSON
line.  The headline (the line's own value, roofline, e2e and cpu_baseline) is the
largest single-GPU workload, the square 8192^3 GEMM with 5% outlier groups; the
prefill linears at M = 2048 (QKV N=6144, O N=4096, gate_up N=24576, down K=12288 ->
N=4096), the decode linears (M = 1, 8, 32, 64; N=12288, K=4096) and the 32-expert
MoE GEMM follow under `configs`, each with the same keys.  A ~ N(0,1), W ~
N(0,0.02) (square: N(0,1) with outliers), bf16, seeded.  Every workload's step
touches more than the 126 MB L2, so no extra L2 flush is used between steps.

Multi-GPU (torchrun): every rank runs its own replica of the workload (its own
tokens, replicated weights); no collective is on the data path.  The timed
region is bracketed by a barrier and a device synchronize on every rank; the
reported time is the max over ranks (an all-reduce of one number).

Output: one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "block-scaled FP8 GEMM TFLOP/s (and GB/s for decode) + % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0   # nominal dense ratio (4.5 / 2.25 PFLOP/s)
_CSRC = "moe_grouped_gemm_quantize_b200/csrc/"
# the files each GEMM kernel is built and launched from: a recorded ncu traffic figure
# stands only while these are unchanged
KERNEL_SOURCES = {
    "k_fp8_block_gemm": [_CSRC + f for f in ("lnq_gemm.cuh", "lnq_ptx.cuh", "lnq_quantize.cuh", "lnq_api.cu")],
    "k_mx_block_gemm": [_CSRC + f for f in ("lnq_mx.cuh", "lnq_ptx.cuh", "lnq_quantize.cuh", "lnq_api.cu")],
}


# --------------------------------------------------------------------------- setup

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str = "nccl"):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, dist, device) -> float:
    """Max of a per-rank number over all ranks (identity on one process)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist):
    if dist is not None:
        dist.barrier()


def job_throughput(work_per_rank_step: float, steps: int, world: int, ms_max: float,
                   scale: float) -> float:
    """Whole-job throughput of a weak-scaling run: every rank processed `steps` steps of
    `work_per_rank_step` units (FLOPs or bytes) in at most `ms_max` milliseconds (the max
    over ranks); `scale` converts units per second to the reported unit (1e12 for TFLOP/s,
    1e9 for GB/s)."""
    return work_per_rank_step * steps * world / (ms_max * 1e-3) / scale


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(kernel: str = "k_fp8_block_gemm") -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    e = rec.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples = []
        self.reasons = set()
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self._nv = None
            self.error = f"nvml unavailable: {e}"

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception as e:
                self.error = str(e)
                return
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.error}
        med = statistics.median(self.samples) if self.samples else None
        out = {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
               "samples": len(self.samples)}
        if self.error:
            out["note"] = self.error
        return out


# --------------------------------------------------------------------------- workloads

class Linear:
    """One dense linear: bf16 activations resident on the device, weights pre-quantized."""

    def __init__(self, cfg, dev, split: bool = False, fp8_out: bool = False, silu: bool = False,
                 recipe: str = "fp32"):
        import moe_grouped_gemm_quantize_b200 as lnq
        from moe_grouped_gemm_quantize_b200 import synthetic
        self.cfg = cfg
        a, w = synthetic.make_linear_inputs(cfg)
        self.x = a.to(dev)
        # UE8M0 recipes: power-of-two scales applied by the tensor core (no promotion), in
        # 1x128 / 128x128 blocks (ue8m0) or 1x32 blocks on both operands (mxfp8)
        self.recipe = recipe
        self.ue8m0 = recipe in ("ue8m0", "mxfp8")
        if recipe == "mxfp8":
            self.wq, self.ws = lnq.quantize_mxfp8(w.to(dev))
        elif self.ue8m0:
            self.wq, self.ws = lnq.quantize_weights_ue8m0(w.to(dev))
        else:
            self.wq, self.ws = lnq.quantize_weights(w.to(dev))
        del w
        M, N, K = cfg.M, cfg.N, cfg.K
        self.M4 = lnq.ceil4(M)
        self.q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=dev)
        self.sfa = torch.empty((K // 128, self.M4), dtype=torch.float32, device=dev)
        self.d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.flops = 2.0 * M * N * K
        self.gemm_bytes = (M * K + 4 * (K // 128) * self.M4 + N * K
                           + 4 * (-(-N // 128)) * (K // 128) + 2 * M * N)
        self.quant_bytes = 2 * M * K + M * K + 4 * (K // 128) * self.M4
        self.h2d_bytes = 2 * M * K
        self.d2h_bytes = 2 * M * N
        self.host_x = self.x.cpu().pin_memory()
        self.host_d = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        # decode shapes: a workspace lets every SM share the weight stream (K split)
        self.work = lnq.gemm_workspace(M, N, K, dev) if split and not self.ue8m0 else None
        if self.ue8m0:
            Mp, Np = -(-M // 128) * 128, -(-N // 128) * 128
            self.sfa = lnq.ue8m0_atoms(M, K, dev)
            self.gemm_bytes = M * K + 4 * (K // 128) * Mp + N * K + 4 * (K // 128) * Np + 2 * M * N
            self.quant_bytes = 2 * M * K + M * K + 4 * (K // 128) * Mp
            fp8_out = silu = False
        # fused epilogue: the output quantized (E4M3 + 1x128 scales) for a next linear
        self.fp8_out = fp8_out and M > 64 and N % 128 == 0 and N >= 256
        if self.fp8_out:
            self.qo = torch.empty((M, N), dtype=torch.float8_e4m3fn, device=dev)
            self.so = torch.empty((N // 128, self.M4), dtype=torch.float32, device=dev)
            self.gemm_bytes += -2 * M * N + M * N + 4 * (N // 128) * self.M4
            self.d2h_bytes = M * N + 4 * (N // 128) * self.M4
            self.host_qo = torch.empty((M, N), dtype=torch.uint8).pin_memory()
            self.host_so = torch.empty((N // 128, self.M4), dtype=torch.float32).pin_memory()
        # fused epilogue of a gate_up linear: h = silu(gate) * up, N/2 bf16 columns
        self.silu = silu and not self.fp8_out and "gate_up" in cfg.name and N % 256 == 0
        if self.silu:
            self.d = torch.empty((M, N // 2), dtype=torch.bfloat16, device=dev)
            self.gemm_bytes -= M * N
            self.d2h_bytes = M * N
            self.host_d = torch.empty((M, N // 2), dtype=torch.bfloat16).pin_memory()

    def out_pairs(self):
        """(device tensor, pinned host tensor) of each output the step reads back."""
        if self.fp8_out:
            return [(self.qo.view(torch.uint8), self.host_qo), (self.so, self.host_so)]
        return [(self.d, self.host_d)]

    OUTPUTS = ("d", "qo", "so")

    def calls(self, stream_ptr):
        """Pre-marshalled C-ABI calls (quantize, gemm)."""
        import ctypes
        import moe_grouped_gemm_quantize_b200 as lnq
        L = lnq.lib()
        P = ctypes.c_void_p
        c = self.cfg
        s = P(stream_ptr)
        if self.ue8m0:
            qargs = (P(self.x.data_ptr()), c.M, c.K, self.x.stride(0), P(self.q.data_ptr()), c.K,
                     P(self.sfa.data_ptr()), s)
            margs = (P(self.q.data_ptr()), P(self.sfa.data_ptr()), P(self.wq.data_ptr()), P(self.ws.data_ptr()),
                     P(self.d.data_ptr()), c.M, c.N, c.K, s)
            if self.recipe == "mxfp8":
                return (L.lnq_quantize_mxfp8, qargs), (L.lnq_mxfp8_gemm_nt, margs)
            return (L.lnq_quantize_ue8m0_groups, qargs), (L.lnq_mx_block_gemm_nt, margs)
        qargs = (P(self.x.data_ptr()), c.M, c.K, self.x.stride(0), P(self.q.data_ptr()), c.K,
                 P(self.sfa.data_ptr()), self.M4, s)
        gargs = (P(self.q.data_ptr()), P(self.sfa.data_ptr()), self.M4, P(self.wq.data_ptr()),
                 P(self.ws.data_ptr()), P(self.d.data_ptr()), c.M, c.N, c.K)
        if self.fp8_out:
            eargs = (P(self.q.data_ptr()), P(self.sfa.data_ptr()), self.M4, P(self.wq.data_ptr()),
                     P(self.ws.data_ptr()), P(0), P(0), P(self.qo.data_ptr()), P(self.so.data_ptr()),
                     self.M4, c.M, c.N, c.K, s)
            return (L.lnq_quantize_fp8_groups, qargs), (L.lnq_fp8_block_gemm_nt_epilogue, eargs)
        if self.silu:
            sargs = (P(self.q.data_ptr()), P(self.sfa.data_ptr()), self.M4, P(self.wq.data_ptr()),
                     P(self.ws.data_ptr()), P(self.d.data_ptr()), c.M, c.N // 2, c.K, s)
            return (L.lnq_quantize_fp8_groups, qargs), (L.lnq_fp8_block_gemm_nt_silu_mul, sargs)
        if self.work is not None:
            return (L.lnq_quantize_fp8_groups, qargs), \
                (L.lnq_fp8_block_gemm_nt_ws, gargs + (P(self.work.data_ptr()), self.work.numel(), s))
        return (L.lnq_quantize_fp8_groups, qargs), (L.lnq_fp8_block_gemm_nt, gargs + (s,))


class Grouped:
    """The M-grouped contiguous MoE GEMM: 16384 routed rows over 32 experts, described
    by per-row group ids (128-row alignment) or, with `alignment` set, by the prefix
    sums of the group sizes (group starts aligned to that many rows)."""

    def __init__(self, cfg, dev, alignment=None, recipe: str = "fp32"):
        import moe_grouped_gemm_quantize_b200 as lnq
        from moe_grouped_gemm_quantize_b200 import synthetic
        self.cfg = cfg
        self.alignment = alignment
        # UE8M0 recipes (group-id layout only): power-of-two scales applied by the tensor core
        self.recipe = recipe
        self.ue8m0 = recipe in ("ue8m0", "mxfp8") and alignment is None
        a, w, m_indices, sizes = synthetic.make_moe_inputs(cfg, alignment=alignment or 128)
        self.M = a.shape[0]
        self.x = a.to(dev)
        if self.ue8m0 and recipe == "mxfp8":
            self.wq, self.ws = lnq.quantize_mxfp8(w.to(dev))
        elif self.ue8m0:
            self.wq, self.ws = lnq.quantize_weights_ue8m0(w.to(dev))
        else:
            self.wq, self.ws = lnq.quantize_weights_grouped(w.to(dev), cfg.groups)
        del w
        if alignment is None:
            self.mi = torch.from_numpy(m_indices).to(dev)
        else:
            self.mi = torch.from_numpy(synthetic.psum_layout(sizes, alignment)[0]).to(dev)
        K, N, G = cfg.K, cfg.N, cfg.groups
        self.q = torch.empty((self.M, K), dtype=torch.float8_e4m3fn, device=dev)
        self.sfa = torch.empty((K // 128, self.M), dtype=torch.float32, device=dev)
        self.d = torch.empty((self.M, N), dtype=torch.bfloat16, device=dev)
        self.flops = cfg.flops   # real rows only
        self.gemm_bytes = (self.M * K + 4 * (K // 128) * self.M + G * N * K
                           + 4 * G * (-(-N // 128)) * (K // 128) + 2 * self.M * N
                           + 4 * (self.M if alignment is None else G))
        self.quant_bytes = 3 * self.M * K + 4 * (K // 128) * self.M
        if self.ue8m0:
            self.sfa = lnq.ue8m0_atoms(self.M, K, dev)
            self.gemm_bytes += 4 * (K // 128) * G * N - 4 * G * (-(-N // 128)) * (K // 128)
        self.h2d_bytes = 2 * self.M * K
        self.d2h_bytes = 2 * self.M * N
        self.host_x = self.x.cpu().pin_memory()
        self.host_d = torch.empty((self.M, N), dtype=torch.bfloat16).pin_memory()

    def out_pairs(self):
        return [(self.d, self.host_d)]

    OUTPUTS = ("d",)

    def calls(self, stream_ptr):
        import ctypes
        import moe_grouped_gemm_quantize_b200 as lnq
        L = lnq.lib()
        P = ctypes.c_void_p
        c = self.cfg
        s = P(stream_ptr)
        if self.ue8m0:
            qargs = (P(self.x.data_ptr()), self.M, c.K, c.K, P(self.q.data_ptr()), c.K, P(self.sfa.data_ptr()), s)
            gargs = (P(self.q.data_ptr()), P(self.sfa.data_ptr()), P(self.wq.data_ptr()), P(self.ws.data_ptr()),
                     P(self.mi.data_ptr()), c.groups, P(self.d.data_ptr()), self.M, c.N, c.K, s)
            if self.recipe == "mxfp8":
                return (L.lnq_quantize_mxfp8, qargs), (L.lnq_m_grouped_mxfp8_gemm_contiguous, gargs)
            return (L.lnq_quantize_ue8m0_groups, qargs), (L.lnq_m_grouped_mx_gemm_contiguous, gargs)
        qargs = (P(self.x.data_ptr()), self.M, c.K, c.K, P(self.q.data_ptr()), c.K,
                 P(self.sfa.data_ptr()), self.M, s)
        if self.alignment is not None:
            gargs = (P(self.q.data_ptr()), P(self.sfa.data_ptr()), P(self.wq.data_ptr()),
                     P(self.ws.data_ptr()), P(self.mi.data_ptr()), c.groups, self.alignment,
                     P(self.d.data_ptr()), self.M, c.N, c.K, s)
            return (L.lnq_quantize_fp8_groups, qargs), (L.lnq_m_grouped_fp8_gemm_contiguous_psum, gargs)
        gargs = (P(self.q.data_ptr()), P(self.sfa.data_ptr()), P(self.wq.data_ptr()),
                 P(self.ws.data_ptr()), P(self.mi.data_ptr()), c.groups, P(self.d.data_ptr()),
                 self.M, c.N, c.K, s)
        return (L.lnq_quantize_fp8_groups, qargs), (L.lnq_m_grouped_fp8_gemm_contiguous, gargs)


class Masked:
    """The M-grouped masked MoE GEMM: 32 expert buffers of 128 rows, 2048 routed tokens;
    in the FP32-scale recipe or (recipe ue8m0 / mxfp8) with power-of-two scales applied
    by the tensor core."""

    def __init__(self, cfg, dev, recipe: str = "fp32"):
        import moe_grouped_gemm_quantize_b200 as lnq
        from moe_grouped_gemm_quantize_b200 import synthetic
        self.cfg = cfg
        self.recipe = recipe
        self.ue8m0 = recipe in ("ue8m0", "mxfp8")
        a, w, counts = synthetic.make_moe_masked_inputs(cfg)
        G, Mm, N, K = cfg.groups, cfg.m_max, cfg.N, cfg.K
        self.M = G * Mm
        self.x = a.to(dev)
        if recipe == "mxfp8":
            self.wq, self.ws = lnq.quantize_mxfp8(w.to(dev))
        elif self.ue8m0:
            self.wq, self.ws = lnq.quantize_weights_ue8m0(w.to(dev))
        else:
            self.wq, self.ws = lnq.quantize_weights_grouped(w.to(dev), G)
        del w
        self.mm = torch.from_numpy(counts).to(dev)
        real = int(counts.sum())
        busy = int((counts > 0).sum())
        self.q = torch.empty((self.M, K), dtype=torch.float8_e4m3fn, device=dev)
        self.sfa = torch.empty((K // 128, self.M), dtype=torch.float32, device=dev)
        self.d = torch.empty((self.M, N), dtype=torch.bfloat16, device=dev)
        self.flops = cfg.flops   # real rows only
        # algorithmic: real activation rows and their scales, the weights and weight
        # scales of the experts with tokens, the real output rows, the counts
        self.gemm_bytes = (real * K + 4 * (K // 128) * real + busy * N * K
                           + 4 * busy * (-(-N // 128)) * (K // 128) + 2 * real * N + 4 * G)
        self.quant_bytes = 3 * self.M * K + 4 * (K // 128) * self.M
        if self.ue8m0:
            # scale atoms: 4 bytes per row per K block on both operands
            self.sfa = lnq.ue8m0_atoms(self.M, K, dev)
            self.gemm_bytes += 4 * (K // 128) * busy * N - 4 * busy * (-(-N // 128)) * (K // 128)
        self.h2d_bytes = 2 * self.M * K
        self.d2h_bytes = 2 * self.M * N
        self.host_x = self.x.cpu().pin_memory()
        self.host_d = torch.empty((self.M, N), dtype=torch.bfloat16).pin_memory()

    def out_pairs(self):
        return [(self.d, self.host_d)]

    OUTPUTS = ("d",)

    def calls(self, stream_ptr):
        import ctypes
        import moe_grouped_gemm_quantize_b200 as lnq
        L = lnq.lib()
        P = ctypes.c_void_p
        c = self.cfg
        s = P(stream_ptr)
        gargs = (P(self.q.data_ptr()), P(self.sfa.data_ptr()), P(self.wq.data_ptr()),
                 P(self.ws.data_ptr()), P(self.mm.data_ptr()), c.groups, c.m_max,
                 c.tokens // c.groups, P(self.d.data_ptr()), c.N, c.K, s)
        if self.ue8m0:
            qargs = (P(self.x.data_ptr()), self.M, c.K, c.K, P(self.q.data_ptr()), c.K, P(self.sfa.data_ptr()), s)
            if self.recipe == "mxfp8":
                return (L.lnq_quantize_mxfp8, qargs), (L.lnq_m_grouped_mxfp8_gemm_masked, gargs)
            return (L.lnq_quantize_ue8m0_groups, qargs), (L.lnq_m_grouped_mx_gemm_masked, gargs)
        qargs = (P(self.x.data_ptr()), self.M, c.K, c.K, P(self.q.data_ptr()), c.K,
                 P(self.sfa.data_ptr()), self.M, s)
        return (L.lnq_quantize_fp8_groups, qargs), (L.lnq_m_grouped_fp8_gemm_masked, gargs)


def workload_units(name: str):
    from moe_grouped_gemm_quantize_b200 import synthetic
    if name == "prefill":
        return list(synthetic.PREFILL), "linear"
    if name == "decode":
        return list(synthetic.DECODE), "linear"
    if name == "square":
        return [synthetic.SQUARE], "linear"
    if name == "tiny":
        return [synthetic.TINY], "linear"
    if name == "moe":
        return [synthetic.MOE], "grouped"
    if name == "moe_masked":
        return [synthetic.MOE_MASKED], "masked"
    if name == "moe_psum":
        return [synthetic.MOE], "psum"
    raise ValueError(name)


WORKLOAD_DESC = {
    "prefill": "prefill linears M=2048: QKV 6144x4096, O 4096x4096, gate_up 24576x4096, down 4096x12288",
    "decode": "decode linears M in {1,8,32,64}, N=12288, K=4096",
    "moe": "M-grouped contiguous MoE: 16384 rows over 32 experts (multinomial seed 0), N=4096, K=7168",
    "square": "square 8192^3 with 5% outlier 1x128 groups (x100)",
    "tiny": "tiny 128x256x512",
    "moe_psum": "M-grouped contiguous MoE, prefix-sum layout with 256-row group alignment "
                "(256x256 tiles on CTA pairs): 16384 rows over 32 experts (multinomial seed 0), "
                "N=4096, K=7168",
    "moe_masked": "M-grouped masked MoE: 32 expert buffers of 128 rows, 2048 routed tokens "
                  "(multinomial seed 3), N=4096, K=7168",
}


def is_hbm_bound(name: str) -> bool:
    return name in ("decode", "moe_masked")


# The default run: every timed workload of the block-scaled FP8 linear, the largest
# single-GPU one (square 8192^3) first as the headline.
ALL_WORKLOADS = ("square", "prefill", "decode", "moe")

# How each workload keeps the timed kernels reading their operands from HBM rather than L2.
L2_NOTE = {
    "square": "inputs larger than L2: A and W E4M3 67 MB each, D 134 MB, and the step's quantize "
              "reads 134 MB of bf16 between GEMMs (126 MB L2); no extra flush",
    "prefill": "working set per step ~500 MB > 126 MB L2 (four linears); no extra flush",
    "decode": "four distinct 50 MB weights per step (200 MB > 126 MB L2), each read once per step; "
              "no extra flush",
    "moe": "1.1 GB of expert weights and activations per step > 126 MB L2; no extra flush",
    "moe_psum": "1.1 GB of expert weights and activations per step > 126 MB L2; no extra flush",
    "moe_masked": "32 experts' weights (940 MB) per step > 126 MB L2; no extra flush",
    "tiny": "tiny: fits in L2 (parity-only workload)",
}


# --------------------------------------------------------------------------- our arm

def make_units(name: str, args, dev):
    cfgs, kind = workload_units(name)
    return [Grouped(c, dev, recipe=args.recipe) if kind == "grouped"
            else Grouped(c, dev, alignment=256) if kind == "psum"
            else Masked(c, dev, recipe=args.recipe) if kind == "masked"
            else Linear(c, dev, split=args.split, fp8_out=args.epilogue == "fp8",
                        silu=args.epilogue == "silu", recipe=args.recipe) for c in cfgs]


def describe_times(ms):
    """min / median / mean of a list of per-launch milliseconds."""
    return {"min": round(min(ms), 5), "median": round(statistics.median(ms), 5),
            "mean": round(statistics.mean(ms), 5), "reps": len(ms)}


class IoSlot:
    """One set of a unit's input and output device buffers for the end-to-end loop, with
    the unit's calls marshalled against them (the quantized activations and the weights
    are shared: the compute stream runs the steps in order)."""

    def __init__(self, u, stream_ptr, fresh: bool):
        names = ["x"] + [n for n in u.OUTPUTS if getattr(u, n, None) is not None]
        saved = {n: getattr(u, n) for n in names}
        self.bufs = {n: (torch.empty_like(t) if fresh else t) for n, t in saved.items()}
        for n, t in self.bufs.items():
            setattr(u, n, t)
        try:
            self.calls = u.calls(stream_ptr)
            self.outs = u.out_pairs()
        finally:
            for n, t in saved.items():
                setattr(u, n, t)
        self.x = self.bufs["x"]
        self.host_x = u.host_x


def measure_workload(name: str, args, dev, dist, world: int, rank: int, cpu_seconds: float):
    """Everything the bench reports for one workload, as a dict (the same keys as the
    top-level JSON line, without `metric`).

    * value: the step (quantize + GEMM of every linear) captured once in a CUDA graph
      and replayed K times between two events, every kernel chained by programmatic
      dependent launch; max over ranks.
    * kernels: each kernel alone, a graph of that one launch replayed max(K, 50) times,
      each replay between its own two events (min and median per launch); and the GEMMs
      alone, max(K, 50) rounds of the workload's GEMMs back to back in one graph (chained
      as in the step, no quantize between them): their mean period per launch is the
      duration `roofline.achieved` divides by.  Graphs keep the host's launch cost (the
      argument marshalling and tensor-map encoding of each C-ABI call) out of the
      device timeline, which would otherwise starve the GPU on the microsecond decode
      kernels.
    * e2e: the step through the public calls, issued from the host every step (no graph),
      with every step's bf16 activations copied in from pinned host memory and its outputs
      copied back.  With large transfers the copies in, the kernels and the copies out run
      on three streams over two sets of input and output buffers, so that step i+1's inputs
      and step i-1's outputs cross PCIe while step i computes (events order every buffer's
      reuse); with small ones (decode) the step is captured once in a CUDA graph, its
      copies included, and replayed.
    """
    import moe_grouped_gemm_quantize_b200 as lnq

    units = make_units(name, args, dev)
    # every call is marshalled for one dedicated stream, on which the graphs are captured
    # and replayed
    stream = torch.cuda.Stream(dev)
    calls = [u.calls(stream.cuda_stream) for u in units]
    n_units = len(units)
    flops_step = sum(u.flops for u in units)
    bytes_step = sum(u.gemm_bytes for u in units)
    hbm = is_hbm_bound(name)

    def run(fn_args, what):
        fn, a = fn_args
        rc = fn(*a)
        if rc:
            raise lnq.LnqError(rc, f"{name} {what}")

    def launch_step():
        for q, g in calls:
            run(q, "quantize")
            run(g, "gemm")

    def capture(fn):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            fn()
        return graph

    for _ in range(args.warmup):
        launch_step()
    torch.cuda.synchronize()
    if lnq.lnq_get_last_device_error() != 0:
        raise RuntimeError(f"{name}: device reported an error during warm-up")

    K = args.steps
    R = max(K, args.kernel_reps)
    g_step = capture(launch_step)
    g_chain = capture(lambda: [run(g, "gemm") for _ in range(R) for _, g in calls])
    g_qchain = capture(lambda: [run(q, "quantize") for _ in range(R) for q, _ in calls])
    g_quant = [capture(lambda q=q: run(q, "quantize")) for q, _ in calls]
    g_gemm = [capture(lambda g=g: run(g, "gemm")) for _, g in calls]
    torch.cuda.synchronize()

    def replay(graph, times=1):
        with torch.cuda.stream(stream):
            for _ in range(times):
                graph.replay()

    replay(g_step, 3)
    replay(g_chain)
    replay(g_qchain)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        # ---- the timed region: K replays of the step between two events on its stream
        barrier(dist)
        torch.cuda.synchronize()
        t0.record(stream)
        replay(g_step, K)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(dist)
        ms_local = t0.elapsed_time(t1)
        if lnq.lnq_get_last_device_error() != 0:
            raise RuntimeError(f"{name}: device reported an error in the timed region")

        # ---- each kernel alone, between its own events
        per_gemm = [[] for _ in range(n_units)]
        per_quant = [[] for _ in range(n_units)]
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4 * n_units)] for _ in range(R)]
        for r in range(R):
            e = evs[r]
            for i in range(n_units):
                e[4 * i].record(stream)
                replay(g_quant[i])
                e[4 * i + 1].record(stream)
                e[4 * i + 2].record(stream)
                replay(g_gemm[i])
                e[4 * i + 3].record(stream)
        torch.cuda.synchronize()
        for r in range(R):
            for i in range(n_units):
                per_quant[i].append(evs[r][4 * i].elapsed_time(evs[r][4 * i + 1]))
                per_gemm[i].append(evs[r][4 * i + 2].elapsed_time(evs[r][4 * i + 3]))

        # ---- the GEMMs alone, R rounds back to back as the step chains them
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        c0.record(stream)
        replay(g_chain)
        c1.record(stream)
        torch.cuda.synchronize()
        chained_ms = c0.elapsed_time(c1)
        # ---- the activation quantizes alone, R rounds back to back
        torch.cuda.synchronize()
        c0.record(stream)
        replay(g_qchain)
        c1.record(stream)
        torch.cuda.synchronize()
        qchained_ms = c0.elapsed_time(c1)
        if lnq.lnq_get_last_device_error() != 0:
            raise RuntimeError(f"{name}: device reported an error in the kernel loops")
    del g_step, g_chain, g_qchain, g_quant, g_gemm
    ms = max_over_ranks(ms_local, dist, dev)
    chained_ms = max_over_ranks(chained_ms, dist, dev)

    # ---- end to end through the public calls: host inputs in, host outputs back
    e2e = None
    if not args.no_e2e:
        Ke = max(1, min(K, args.e2e_steps))
        # a step whose PCIe transfers are small (decode) gains nothing from overlapping them and
        # would pay the cross-stream waits: it runs copies and kernels in order on one stream
        pipelined = sum(u.h2d_bytes + u.d2h_bytes for u in units) >= (32 << 20)
        s_in = torch.cuda.Stream(dev) if pipelined else stream
        s_out = torch.cuda.Stream(dev) if pipelined else stream
        slots = [[IoSlot(u, stream.cuda_stream, fresh=(k == 1)) for u in units]
                 for k in range(2 if pipelined else 1)]
        ev = lambda: torch.cuda.Event()
        in_done = [[ev() for _ in units] for _ in range(2)]      # slot's inputs landed
        comp_done = [[ev() for _ in units] for _ in range(2)]    # slot's kernels done
        out_done = [[ev() for _ in units] for _ in range(2)]     # slot's outputs read back

        def e2e_step(i):
            k = i % 2 if pipelined else 0
            for j, (u, sl) in enumerate(zip(units, slots[k])):
                q, g = sl.calls
                with torch.cuda.stream(s_in):
                    if i >= 2 and pipelined:
                        s_in.wait_event(comp_done[k][j])      # step i-2 has read this input buffer
                    sl.x.copy_(sl.host_x, non_blocking=True)
                    in_done[k][j].record(s_in)
                with torch.cuda.stream(stream):
                    if pipelined:
                        stream.wait_event(in_done[k][j])
                        if i >= 2:
                            stream.wait_event(out_done[k][j])  # step i-2's outputs are read back
                    run(q, "e2e quantize")
                    run(g, "e2e gemm")
                    comp_done[k][j].record(stream)
                with torch.cuda.stream(s_out):
                    if pipelined:
                        s_out.wait_event(comp_done[k][j])
                    for dev_t, host_t in sl.outs:
                        host_t.copy_(dev_t, non_blocking=True)
                    out_done[k][j].record(s_out)

        def serial_step():
            # copies in, kernels and copies out of every linear in order on one stream
            with torch.cuda.stream(stream):
                for sl in slots[0]:
                    q, g = sl.calls
                    sl.x.copy_(sl.host_x, non_blocking=True)
                    run(q, "e2e quantize")
                    run(g, "e2e gemm")
                    for dev_t, host_t in sl.outs:
                        host_t.copy_(dev_t, non_blocking=True)

        for i in range(2):                    # warm the copy paths and both buffer sets
            e2e_step(i) if pipelined else serial_step()
        torch.cuda.synchronize()
        g_e2e = None
        if not pipelined:
            # small transfers: the step (its copies in, kernels and copies out) is captured
            # once through the public calls and replayed, as a decode server does, so the
            # host's per-call cost stays out of the device timeline
            g_e2e = capture(serial_step)
            replay(g_e2e)
            torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        barrier(dist)
        torch.cuda.synchronize()
        e0.record(s_in)
        if pipelined:
            stream.wait_event(e0)
            s_out.wait_event(e0)
            for i in range(Ke):
                e2e_step(i)
            s_out.wait_stream(stream)
            s_out.wait_stream(s_in)
        else:
            replay(g_e2e, Ke)
        e1.record(s_out)
        torch.cuda.synchronize()
        barrier(dist)
        if lnq.lnq_get_last_device_error() != 0:
            raise RuntimeError(f"{name}: device reported an error in the end-to-end loop")
        e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
        del slots, g_e2e
        if hbm:
            ev_val, ev_unit = job_throughput(bytes_step, Ke, world, e_ms, 1e9), "GB/s"
        else:
            ev_val, ev_unit = job_throughput(flops_step, Ke, world, e_ms, 1e12), "TFLOP/s"
        e2e = {"value": round(ev_val, 3), "unit": ev_unit, "steps": Ke,
               "h2d_bytes_per_step": int(sum(u.h2d_bytes for u in units)),
               "d2h_bytes_per_step": int(sum(u.d2h_bytes for u in units)),
               "schedule": ("copies in, kernels and copies out on three streams over two buffer sets"
                            if pipelined else "copies in, kernels and copies out in order on one stream, "
                                              "the step captured once in a CUDA graph and replayed"),
               "note": "every step: pinned host bf16 activations copied in and the outputs copied back "
                       "(weights resident, model parameters); with 32 MB or more of PCIe transfers per "
                       "step, those of neighbouring steps overlap the kernels; with less, the step's "
                       "copies and calls replay from one CUDA graph"}

    # ---- numbers
    peaks, peak_src = load_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    gemm_period_ms = chained_ms / (R * n_units)
    if hbm:
        value = job_throughput(bytes_step, K, world, ms, 1e9)
        unit = "GB/s"
        ach = bytes_step * R / (chained_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / peaks["hbm_gbs"], 4)}
        peak_note = f"HBM copy bandwidth ({peak_src}; burst)"
        iso = [bytes_step / n_units / (statistics.median(t) * 1e-3) / 1e9 for t in per_gemm]
    else:
        value = job_throughput(flops_step, K, world, ms, 1e12)
        unit = "TFLOP/s"
        ach = flops_step * R / (chained_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": round(fp8_peak, 1),
                "unit": "TFLOP/s", "frac": round(ach / fp8_peak, 4)}
        peak_note = (f"dense FP8 = {FP8_OVER_BF16:g} x bf16 cuBLAS burst {peaks['bf16_tflops']} "
                     f"TFLOP/s ({peak_src})")
        iso = [u.flops / (statistics.median(t) * 1e-3) / 1e12 for u, t in zip(units, per_gemm)]
    ue8m0 = any(getattr(u, "ue8m0", False) for u in units)
    kernel_name = "k_mx_block_gemm" if ue8m0 else "k_fp8_block_gemm"
    roof["traffic"] = recorded_traffic(kernel_name, name if args.recipe == "fp32" else f"{name}_{args.recipe}")
    roof["kernel"] = kernel_name
    roof["peak_source"] = peak_note
    roof["duration"] = ("mean period per GEMM launch over the workload's GEMMs captured back to "
                        f"back {R} times in one CUDA graph (chained by programmatic dependent launch "
                        "as in the step)")
    roof["algorithmic_per_launch"] = ({"bytes": [int(u.gemm_bytes) for u in units]} if hbm
                                      else {"flops": [float(u.flops) for u in units]})
    roof["isolated_median"] = {"value": [round(x, 1) for x in iso], "unit": roof["unit"],
                               "note": "each GEMM alone (a one-launch graph between its own two events)"}
    q_total = sum(statistics.median(t) for t in per_quant)
    g_total = sum(statistics.median(t) for t in per_gemm)
    quant_gbs_isolated = sum(u.quant_bytes for u in units) / (q_total * 1e-3) / 1e9
    quant_gbs = sum(u.quant_bytes for u in units) * R / (qchained_ms * 1e-3) / 1e9
    out = {
        "value": round(value, 3),
        "unit": unit,
        "ms_per_step": round(ms / K, 5),
        "steps": K,
        "roofline": roof,
        "kernels": {
            "gemm_ms_per_launch": [describe_times(t) for t in per_gemm],
            "quantize_ms_per_launch": [describe_times(t) for t in per_quant],
            "gemm_chained_ms_per_launch": round(gemm_period_ms, 5),
            "quantize_chained_ms_per_launch": round(qchained_ms / (R * n_units), 5),
            "quantize_gbs": round(quant_gbs, 1),
            "quantize_frac_of_hbm": round(quant_gbs / peaks["hbm_gbs"], 4),
            "quantize_gbs_isolated": round(quant_gbs_isolated, 1),
            "quantize_note": ("quantize_gbs: algorithmic bytes (bf16 in, E4M3 and scales out) over the mean "
                              "period of the quantizes launched back to back in one graph; _isolated: each "
                              "launch alone between two events, which adds several microseconds of launch "
                              "latency to these microsecond kernels"),
            "gemm_share_of_step": round(g_total / (g_total + q_total), 4),
        },
        "gpu_launches": K * 2 * n_units,
        "clocks": clocks.summary(),
        "e2e": e2e,
        "desc": WORKLOAD_DESC[name],
        "recipe": ("MXFP8 gran-32: UE8M0 scales per 1x32 block on both operands, in the tensor core"
                   if args.recipe == "mxfp8" else
                   "UE8M0 power-of-two scales (gran-128) in the tensor core" if ue8m0
                   else "FP32 scales, per-128-K-block promotion"),
        "epilogue": ("fp8 output (E4M3 + 1x128 scales)" if any(getattr(u, "fp8_out", False) for u in units)
                     else "gate_up with SiLU.mul (bf16 h)" if any(getattr(u, "silu", False) for u in units)
                     else "bf16 output"),
        "decode_k_split": any(getattr(u, "work", None) is not None for u in units),
        "l2": L2_NOTE[name],
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(name, target_s=cpu_seconds)
    del calls, units
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def run_ours(args, world, rank, local):
    import moe_grouped_gemm_quantize_b200 as lnq
    from moe_grouped_gemm_quantize_b200 import build as lnq_build

    dist = init_dist(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if rank == 0:
        lnq_build.build()
    barrier(dist)
    lnq.lib()
    lnq.lib().lnq_set_dense_cta_pairs(args.cta_pairs)
    lnq.lib().lnq_set_grouped_cta_pairs(args.grouped_cta_pairs)
    # the weights are model parameters quantized before timing: nothing in the step
    # writes them, so the GEMMs may stream them before the previous kernel completes
    lnq.lnq_set_weight_prefetch(not args.no_weight_prefetch)
    lnq.lnq_set_tma_store(bool(args.tma_store))

    names = list(ALL_WORKLOADS) if args.workload == "all" else [args.workload]
    results = {}
    for name in names:
        # the headline's oracle sample takes about cpu_seconds / 2 of host time, every other
        # workload's about a third of that
        share = args.cpu_seconds if name == names[0] else args.cpu_seconds / 3
        results[name] = measure_workload(name, args, dev, dist, world, rank, share)
    head_name = names[0]
    head = results[head_name]
    out = {
        "metric": METRIC,
        "value": head["value"],
        "unit": head["unit"],
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("e4m3 x e4m3 with UE8M0 block scales -> f32 accumulate, bf16 out" if args.recipe != "fp32"
                  else "e4m3 x e4m3 -> f32 accumulate, bf16 out"),
        "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights, bf16)",
        "config": {"workload": (f"{head_name} (headline; every workload under `configs`)"
                                if len(names) > 1 else head_name),
                   "desc": head["desc"],
                   "workloads": names,
                   "dense_cta_pairs": args.cta_pairs,
                   "grouped_cta_pairs": args.grouped_cta_pairs,
                   "weight_prefetch": not args.no_weight_prefetch,
                   "output_store": "TMA store through shared memory" if args.tma_store else "row stores from registers",
                   "decode_k_split": head["decode_k_split"],
                   "epilogue": head["epilogue"],
                   "recipe": head["recipe"],
                   "parallelism": f"replicas x{world} (independent tokens per rank)",
                   "l2": head["l2"]},
        "roofline": head["roofline"],
        "kernels": head["kernels"],
        "gpu_launches": head["gpu_launches"],
        "timing": ("value: one step captured in a CUDA graph, replayed K times between two events "
                   "(kernels chained by programmatic dependent launch), max over ranks; roofline: "
                   "max(K, 50) rounds of the GEMMs back to back in one graph, mean period per launch; "
                   "kernels: each kernel alone in a graph, each replay between its own events "
                   "(min, median over max(K, 50)); e2e: host-issued calls with host copies"),
        "clocks": head["clocks"],
        "e2e": head["e2e"],
    }
    if "cpu_baseline" in head:
        out["cpu_baseline"] = head["cpu_baseline"]
    if len(names) > 1:
        out["configs"] = {n: {k: v for k, v in r.items() if k not in ("desc",)} | {"desc": r["desc"]}
                          for n, r in results.items()}
        out["gpu_launches_all_workloads"] = sum(r["gpu_launches"] for r in results.values())
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.destroy_process_group()


# --------------------------------------------------------------------------- the oracle (CPU)

def oracle_inputs(workload: str, max_rows: int):
    """Oracle inputs for every linear of the workload: up to `max_rows` activation rows
    (bf16 bits) and the pre-quantized weights of the product."""
    import oracle
    from moe_grouped_gemm_quantize_b200 import synthetic
    cfgs, kind = workload_units(workload)
    items = []
    for c in cfgs:
        if kind == "masked":
            a, w, counts = synthetic.make_moe_masked_inputs(c)
            r = min(max_rows, int(counts[0]))
            # group 0's real rows against group 0's weights
            wq, ws = oracle.quantize_fp8_blocks(synthetic.bf16_bits(w[:c.N]))
            items.append((synthetic.bf16_bits(a[:r]), wq, ws, 2.0 * c.N * c.K))
        elif kind in ("grouped", "psum"):
            a, w, m_indices, _ = synthetic.make_moe_inputs(c)
            r = min(max_rows, a.shape[0])
            # the first rows of the arena against group 0's weights: the product of one
            # expert, per row the same work as every row of the grouped product
            wq, ws = oracle.quantize_fp8_blocks(synthetic.bf16_bits(w[:c.N]))
            items.append((synthetic.bf16_bits(a[:r]), wq, ws, 2.0 * c.N * c.K))
        else:
            a, w = synthetic.make_linear_inputs(c)
            r = min(max_rows, c.M)
            wq, ws = oracle.quantize_fp8_blocks(synthetic.bf16_bits(w))
            items.append((synthetic.bf16_bits(a[:r]), wq, ws, 2.0 * c.N * c.K))
    return items


def oracle_sample(items, rows: int, cols: int | None = None):
    """The first `rows` activation rows of each linear, and of its output columns the
    first `cols` (a multiple of 128; all when None).  FLOPs are counted for the sample."""
    out = []
    for a_bits, wq, ws, flops_per_row in items:
        r = min(rows, a_bits.shape[0])
        n = wq.shape[0]
        if cols is not None and cols < n:
            wq, ws = wq[:cols], ws[:-(-cols // 128)]
        out.append((a_bits[:r], wq, ws, flops_per_row * r * wq.shape[0] / n))
    return out


def oracle_step(items):
    import oracle
    for a_bits, wq, ws, _ in items:
        qa, sa = oracle.quantize_fp8_groups(a_bits)
        oracle.gemm_nt(qa, sa, wq, ws)


def measure_oracle(items, dt_s: float, steps: int = 1):
    flops = sum(it[3] for it in items) * steps
    byts = sum(it[0].size * 3 + it[1].size + 2 * it[0].shape[0] * it[1].shape[0]
               for it in items) * steps
    return flops, byts


def cpu_baseline(workload: str, target_s: float = 10.0):
    """The oracle, as it stands, timed on this host on a bounded sample of the workload.

    The sample grows (the first r activation rows of every linear) until one timed pass
    takes at least half of `target_s`; a workload whose every row fits in less (decode) is
    passed over whole, as many times as that takes.  The last timed run is the reported one."""
    import oracle
    full = oracle_inputs(workload, 1 << 30)
    max_rows = max(it[0].shape[0] for it in full)
    rows = 1
    while True:
        items = oracle_sample(full, rows)
        t = time.perf_counter()
        oracle_step(items)
        dt = time.perf_counter() - t
        if dt >= 0.5 * target_s or rows >= max_rows:
            break
        rows = min(max_rows, max(2 * rows, int(rows * 0.8 * target_s / max(dt, 1e-3))))
    passes = 1
    if dt < 0.5 * target_s:
        passes = max(1, int(np.ceil(0.5 * target_s / max(dt, 1e-3))))
        t = time.perf_counter()
        for _ in range(passes):
            oracle_step(items)
        dt = time.perf_counter() - t
    flops, byts = measure_oracle(items, dt, passes)
    if is_hbm_bound(workload):
        val, unit = byts / dt / 1e9, "GB/s"
    else:
        val, unit = flops / dt / 1e12, "TFLOP/s"
    what = "each linear of the workload" if workload != "moe" else "the MoE arena against one expert's weights"
    return {"value": val, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {rows} activation row(s) of {what} (quantize + FP64 product, weights "
                      f"pre-quantized), {passes} pass(es), {dt:.2f} s"}


def reference_sample(workload: str, steps: int, warmup: int):
    """The oracle on one bounded sample per step: the first 16 activation rows x the first
    1024 output columns of every linear of the workload (fewer where it has fewer)."""
    rows, cols = 16, 1024
    items = oracle_sample(oracle_inputs(workload, rows), rows, cols)
    for _ in range(warmup):
        oracle_step(items)
    t = time.perf_counter()
    for _ in range(steps):
        oracle_step(items)
    dt = time.perf_counter() - t
    flops, byts = measure_oracle(items, dt, steps)
    if is_hbm_bound(workload):
        val, unit = byts / dt / 1e9, "GB/s"
    else:
        val, unit = flops / dt / 1e12, "TFLOP/s"
    return val, unit, dt / steps * 1e3, (f"first {rows} activation rows x first {cols} output columns of "
                                         f"each linear per step (quantize + FP64 product, weights "
                                         f"pre-quantized)")


def run_reference(args, world, rank, local):
    """The reference arm: the CPU oracle on a bounded sample, on rank 0 only."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    names = list(ALL_WORKLOADS) if args.workload == "all" else [args.workload]
    results = {n: reference_sample(n, args.steps, args.warmup) for n in names}
    val, unit, ms_step, sample = results[names[0]]
    cores = oracle.num_threads()
    out = {
        "impl": "reference",
        "metric": METRIC,
        "value": val,
        "unit": unit,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": (f"{names[0]} (headline; every workload under `configs`)"
                                if len(names) > 1 else names[0]),
                   "desc": WORKLOAD_DESC[names[0]], "workloads": names},
        "cpu_baseline": {"value": val, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    if len(names) > 1:
        out["configs"] = {n: {"value": v, "unit": u, "ms_per_step": m, "desc": WORKLOAD_DESC[n],
                              "cpu_baseline": {"value": v, "unit": u, "cores": cores, "kind": "oracle",
                                               "sample": smp}}
                          for n, (v, u, m, smp) in results.items()}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["all", "prefill", "decode", "moe", "moe_psum", "moe_masked", "square",
                                           "tiny"],
                    default="all", help="all (the default): square (headline), prefill, decode and moe")
    ap.add_argument("--kernel-reps", type=int, default=50,
                    help="repetitions of the per-kernel timing loops (at least the number of steps)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--epilogue", choices=["bf16", "fp8", "silu"], default="bf16",
                    help="dense GEMM output: bf16 D, E4M3 codes + 1x128 scales for a next linear, or "
                         "(silu) h = silu(gate) * up of the gate_up linear in bf16")
    ap.add_argument("--split", action="store_true",
                    help="decode GEMMs through the workspace K split (slower than whole weight tiles "
                         "per CTA at N = 12288 on B200)")
    ap.add_argument("--no-weight-prefetch", action="store_true",
                    help="GEMMs wait for the previous kernel before streaming weights")
    ap.add_argument("--recipe", choices=["fp32", "ue8m0", "mxfp8"], default="fp32",
                    help="dense and moe workloads: FP32 scales with promotion (the default), UE8M0 "
                         "power-of-two scales in 1x128 / 128x128 blocks, or MXFP8 gran-32 (1x32 UE8M0 "
                         "blocks on both operands), both applied by the block-scaled MMA")
    ap.add_argument("--grouped-cta-pairs", type=int, default=0, choices=[0, 1],
                    help="moe_psum: 256x256 tiles on CTA pairs (1) or 128-row tiles (0)")
    ap.add_argument("--tma-store", type=int, default=1, choices=[0, 1],
                    help="dense and grouped GEMM outputs: 1 through shared memory and TMA stores, 0 each "
                         "thread stores its own row")
    ap.add_argument("--cta-pairs", type=int, default=1, choices=[0, 1, 2],
                    help="dense GEMMs with M > 128: 0 one CTA per 128x256 tile, 1 CTA pairs on "
                         "256x256 tiles, 2 CTA pairs on 256x128 tiles")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank, local)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
