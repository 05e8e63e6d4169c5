"""The C-ABI calls captured in a CUDA graph and replayed.

The calls allocate nothing and never synchronize, so a sequence of them (activation
quantize, then the GEMM) can be captured once and replayed, which is how a decode
step avoids paying the host's launch cost per kernel.  A replayed graph must give the
same bytes as the same calls issued directly (the kernels are deterministic), for the
dense CTA-pair, decode and grouped configurations, and the programmatic-dependent-launch
chaining between the captured kernels must keep its ordering: the GEMM of a replay
reads the codes that the replay's own quantize wrote.
"""
import pytest
import torch

import moe_grouped_gemm_quantize_b200 as lnq
from moe_grouped_gemm_quantize_b200 import synthetic

pytestmark = pytest.mark.gpu
DEV = "cuda"


def dense_case(M, N, K, seed):
    a = synthetic.gaussian_bf16((M, K), 1.0, seed).to(DEV)
    w = synthetic.gaussian_bf16((N, K), 0.02, seed + 1).to(DEV)
    wq, ws = lnq.quantize_weights(w)
    q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=DEV)
    sfa = torch.empty((K // 128, lnq.ceil4(M)), dtype=torch.float32, device=DEV)
    d = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    return a, wq, ws, q, sfa, d


@pytest.mark.parametrize("M,N,K", [(2048, 1024, 1024), (8, 12288, 4096), (64, 4096, 2048), (300, 768, 512)])
def test_replayed_step_matches_direct_calls(M, N, K):
    a, wq, ws, q, sfa, d = dense_case(M, N, K, seed=M + N)
    stream = torch.cuda.Stream()

    def step():
        lnq.lnq_quantize_fp8_groups(a, q, sfa, stream)
        lnq.lnq_fp8_block_gemm_nt(q, sfa, wq, ws, d, stream)

    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    want = d.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for _ in range(3):
        d.fill_(float("nan"))
        q.zero_()
        sfa.zero_()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            graph.replay()
        torch.cuda.synchronize()
        assert lnq.lnq_get_last_device_error() == 0
        assert torch.equal(d.view(torch.int16), want.view(torch.int16))


def test_replayed_step_follows_new_inputs():
    # the graph holds pointers, not values: new activations written into the same
    # buffer before a replay give that input's product
    M, N, K = 256, 512, 1024
    a, wq, ws, q, sfa, d = dense_case(M, N, K, seed=3)
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        lnq.lnq_quantize_fp8_groups(a, q, sfa, stream)
        lnq.lnq_fp8_block_gemm_nt(q, sfa, wq, ws, d, stream)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, stream=stream):
        lnq.lnq_quantize_fp8_groups(a, q, sfa, stream)
        lnq.lnq_fp8_block_gemm_nt(q, sfa, wq, ws, d, stream)
    a2 = synthetic.gaussian_bf16((M, K), 1.0, 99).to(DEV)
    a.copy_(a2)
    with torch.cuda.stream(stream):
        graph.replay()
    torch.cuda.synchronize()
    want = lnq.linear(a2, wq, ws)
    torch.cuda.synchronize()
    assert torch.equal(d.view(torch.int16), want.view(torch.int16))


def test_replayed_grouped_gemm_matches_direct_call():
    sizes, N, K = [130, 0, 256, 7, 300], 256, 512
    G = len(sizes)
    m_indices, _, M_total = synthetic.contiguous_layout(sizes)
    a = synthetic.gaussian_bf16((M_total, K), 1.0, 5).to(DEV)
    w = synthetic.gaussian_bf16((G * N, K), 0.02, 6).to(DEV)
    wq, ws = lnq.quantize_weights_grouped(w, G)
    mi = torch.from_numpy(m_indices).to(DEV)
    q = torch.empty((M_total, K), dtype=torch.float8_e4m3fn, device=DEV)
    sfa = torch.empty((K // 128, M_total), dtype=torch.float32, device=DEV)
    d = torch.zeros((M_total, N), dtype=torch.bfloat16, device=DEV)
    stream = torch.cuda.Stream()

    def step():
        lnq.lnq_quantize_fp8_groups(a, q, sfa, stream)
        lnq.lnq_m_grouped_fp8_gemm_contiguous(q, sfa, wq, ws, mi, G, d, stream)

    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    want = d.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    d.zero_()
    with torch.cuda.stream(stream):
        graph.replay()
    torch.cuda.synchronize()
    assert lnq.lnq_get_last_device_error() == 0
    assert torch.equal(d.view(torch.int16), want.view(torch.int16))
