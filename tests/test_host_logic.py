"""Host-side logic that reported numbers depend on (no GPU).

* bench.recorded_traffic reports a committed ncu DRAM figure only while the sources of
  that kernel are unchanged since the capture, per kernel;
* the synthetic prefix-sum layout agrees with the padded group-id layout built from the
  same sizes, and its prefix sums are the running token counts;
* bench.job_throughput counts every rank's work over the slowest rank's time.
"""
import json
import os

import numpy as np

import bench
from moe_grouped_gemm_quantize_b200 import synthetic


def test_recorded_traffic_follows_its_kernel_sources(tmp_path, monkeypatch):
    rec = {"prefill": {
        "k_fp8_block_gemm": {"source_hash": bench.kernel_source_hash("k_fp8_block_gemm"), "bytes_per_launch": 11},
        "k_mx_block_gemm": {"source_hash": "0" * 16, "bytes_per_launch": 22},
    }}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the hash is still computed over the real sources (their paths are relative to ROOT)
    for k, files in bench.KERNEL_SOURCES.items():
        for f in files:
            dst = tmp_path / f
            dst.parent.mkdir(parents=True, exist_ok=True)
            dst.write_bytes(open(os.path.join(os.path.dirname(bench.__file__), f), "rb").read())
    assert bench.recorded_traffic("k_fp8_block_gemm", "prefill") == 11
    assert bench.recorded_traffic("k_mx_block_gemm", "prefill") is None        # stale hash
    assert bench.recorded_traffic("k_fp8_block_gemm", "decode") is None        # no record
    # a change to the UE8M0 kernel's own file leaves the FP32 kernel's record valid
    mx = tmp_path / bench.KERNEL_SOURCES["k_mx_block_gemm"][0]
    mx.write_bytes(mx.read_bytes() + b"\n")
    assert bench.recorded_traffic("k_fp8_block_gemm", "prefill") == 11
    # a change to a shared file invalidates it
    shared = tmp_path / bench.KERNEL_SOURCES["k_fp8_block_gemm"][1]
    shared.write_bytes(shared.read_bytes() + b"\n")
    assert bench.recorded_traffic("k_fp8_block_gemm", "prefill") is None


def test_committed_traffic_records_are_consistent():
    # a record goes stale (and reads as null) when its kernel changes; it must never be
    # internally inconsistent
    rec = json.load(open(os.path.join(os.path.dirname(bench.__file__), "profiles", "traffic.json")))
    for workload, kernels in rec.items():
        for kernel, e in kernels.items():
            assert kernel in bench.KERNEL_SOURCES
            assert e["bytes_per_launch"] == sum(e["bytes_per_launch_list"]) // len(e["bytes_per_launch_list"])
            assert "--clock-control none" in e["command"]


def test_psum_layout_matches_the_group_id_layout():
    rng = np.random.default_rng(5)
    for alignment in (128, 256):
        sizes = rng.integers(0, 700, 17)
        sizes[3] = 0
        psum, starts, M_total = synthetic.psum_layout(sizes, alignment)
        m_indices, starts2, M2 = synthetic.contiguous_layout(sizes, alignment)
        assert M_total == M2 and np.array_equal(starts, starts2)
        assert np.array_equal(psum, np.cumsum(sizes))
        assert np.all(starts % alignment == 0) and M_total % alignment == 0
        for g, (s, n) in enumerate(zip(starts, sizes)):
            assert np.all(m_indices[s:s + n] == g)
        assert (m_indices >= 0).sum() == sizes.sum()


def test_job_throughput_counts_all_ranks_over_the_slowest():
    # 2 ranks, each 1e12 units per step, 10 steps in 5 ms (max over ranks): 4e15 units/s
    assert abs(bench.job_throughput(1e12, 10, 2, 5.0, 1.0) - 4e15) < 1e3


class _FakeUnit:
    """A unit with the attributes the end-to-end loop's buffer sets swap."""

    OUTPUTS = ("d", "qo")

    def __init__(self):
        import torch
        self.x = torch.arange(12, dtype=torch.float32).reshape(3, 4)
        self.d = torch.zeros((3, 5), dtype=torch.float32)
        self.qo = None                       # an output this configuration does not produce
        self.host_x = self.x.clone()
        self.host_d = torch.zeros_like(self.d)

    def calls(self, stream_ptr):
        return ("quantize", self.x.data_ptr(), stream_ptr), ("gemm", self.d.data_ptr(), stream_ptr)

    def out_pairs(self):
        return [(self.d, self.host_d)]


def test_io_slot_marshals_calls_against_its_own_buffers():
    u = _FakeUnit()
    x0, d0 = u.x, u.d
    first = bench.IoSlot(u, 7, fresh=False)
    second = bench.IoSlot(u, 7, fresh=True)
    # the unit keeps its own buffers
    assert u.x is x0 and u.d is d0 and u.qo is None
    # the first set is the unit's; the second has buffers of its own, of the same shapes
    assert first.x is x0 and first.calls[1][1] == d0.data_ptr()
    assert second.x is not x0 and second.x.shape == x0.shape and second.x.dtype == x0.dtype
    assert second.calls[0][1] == second.x.data_ptr() != x0.data_ptr()
    assert second.calls[1][1] == second.bufs["d"].data_ptr() != d0.data_ptr()
    # both read back into the same pinned host buffer, from their own device buffer
    (dev0, host0), = first.outs
    (dev1, host1), = second.outs
    assert dev0 is d0 and dev1 is second.bufs["d"] and host0 is host1 is u.host_d
    assert "qo" not in second.bufs
