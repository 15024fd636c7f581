"""GPU: the prefill captured in a CUDA graph and replayed with new inputs.

Every step of a call is stream-ordered (scratch from cudaMallocAsync, the
clearing of the chunk scan's counters, the kernel, cudaFreeAsync), so a stream
capture records it as graph nodes and each replay must compute the current
contents of the captured buffers.  The hand-over and the split scan publish a
per-launch tag outside captures; a captured launch reuses one tag, so each
replay must start from cleared flags.  Checked element by element against the
float64 oracle for each way the kernel splits the work, over three replays
with fresh inputs, through both the allocating and the allocation-free entry.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_fwd_b200 import inputs as I
from long_context_fwd_b200 import ops
from parity import TOL_BF16, rel, worst_head

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")

CASES = [
    # B, H, N, mode the plan must pick (2 split scan, 1 hand-over, 0 chunk scan)
    (1, 64, 2500, 2),
    (2, 80, 1100, 1),
    (1, 4, 3000, 0),
]


def _fill(bufs, B, H, N, seed):
    """New seeded inputs copied into the captured buffers; returns the host bits."""
    w = I.Workload(f"graph{seed}", B, H, N, 128, 128, "bf16", index=1200 + seed)
    host = I.prefill_inputs(w)
    for dst, x in zip(bufs, host):
        dst.copy_(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16))
    return host


@pytest.mark.parametrize("noalloc", [False, True])
@pytest.mark.parametrize("B,H,N,mode", CASES)
def test_prefill_graph_replays_with_new_inputs(B, H, N, mode, noalloc):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert ops.fwd_plan(B, H, N, 0, sms)[0]["mode"] == mode
    q, k, v = (torch.empty((B, H, N, 128), dtype=torch.bfloat16, device=DEV) for _ in range(3))
    out = torch.empty((B, H, N, 128), dtype=torch.float32, device=DEV)
    sl_host = I.alibi_slopes(H)
    sl_host[::5] = 0.0
    sl = torch.from_numpy(sl_host).to(DEV)
    call = (lambda: ops.fwd_noalloc(q, k, v, sl, out)) if noalloc else (lambda: ops.fwd(q, k, v, sl, out))

    _fill((q, k, v), B, H, N, 0)
    call()  # first call outside the capture (one-time setup)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for seed in (1, 2, 3):
        hq, hk, hv = _fill((q, k, v), B, H, N, seed)
        out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert ops.device_status(reset=True) == 0
        got = out.cpu().numpy()
        ref = oracle.recurrent(hq, hk, hv, sl_host)
        assert np.isfinite(got).all(), seed
        assert rel(got, ref) <= TOL_BF16, seed
        assert worst_head(got, ref) <= TOL_BF16, seed
    del graph


@pytest.mark.parametrize("B,H,N", [(2, 80, 600), (1, 64, 2000), (1, 4, 3000)])
def test_backward_graph_replays_with_new_inputs(B, H, N):
    """The backward pass (dq launch + paired dk/dv launch, each role with its own
    cleared control block) captured once and replayed with fresh inputs."""
    q, k, v, g = (torch.empty((B, H, N, 128), dtype=torch.bfloat16, device=DEV) for _ in range(4))
    dq, dk, dv = (torch.empty((B, H, N, 128), dtype=torch.float32, device=DEV) for _ in range(3))
    sl_host = I.alibi_slopes(H)
    sl = torch.from_numpy(sl_host).to(DEV)
    call = lambda: ops.bwd(q, k, v, g, sl, dq, dk, dv)

    def fill(seed):
        host = _fill((q, k, v), B, H, N, 10 + seed)
        gh = I.f32_to_bf16_bits(np.random.default_rng(seed).standard_normal((B, H, N, 128))
                                .astype(np.float32))
        g.copy_(torch.from_numpy(gh.view(np.int16)).view(torch.bfloat16))
        return (*host, gh)

    fill(0)
    call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for seed in (1, 2):
        hq, hk, hv, hg = fill(seed)
        for t in (dq, dk, dv):
            t.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert ops.device_status(reset=True) == 0
        for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv),
                                  oracle.backward(hq, hk, hv, hg, sl_host)):
            a = got.cpu().numpy()
            assert np.isfinite(a).all(), (seed, name)
            assert rel(a, ref) <= TOL_BF16, (seed, name)
    del graph


def _captured_node_types(call):
    """Node types of the graph that capturing call(stream) records."""
    from cuda.bindings import runtime as rt

    ok = rt.cudaError_t.cudaSuccess
    s = torch.cuda.Stream(device=DEV)
    torch.cuda.synchronize()
    (err,) = rt.cudaStreamBeginCapture(s.cuda_stream,
                                       rt.cudaStreamCaptureMode.cudaStreamCaptureModeThreadLocal)
    assert err == ok
    try:
        call(s)
    finally:
        err, graph = rt.cudaStreamEndCapture(s.cuda_stream)
    assert err == ok
    err, _, n = rt.cudaGraphGetNodes(graph, 0)
    assert err == ok
    err, nodes, n = rt.cudaGraphGetNodes(graph, n)
    assert err == ok
    types = [rt.cudaGraphNodeGetType(node)[1] for node in nodes[:n]]
    rt.cudaGraphDestroy(graph)
    return types, rt.cudaGraphNodeType


@pytest.mark.parametrize("noalloc", [False, True])
@pytest.mark.parametrize("B,H,N,mode", CASES + [(1, 148, 1000, 1)])
def test_captured_call_clears_the_flags(B, H, N, mode, noalloc):
    """Inside a capture every split that uses scratch clears its flags (a memset
    node before the kernel); with 148 sequences on 148 SMs no sequence is split
    and nothing is cleared."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    info = ops.fwd_plan(B, H, N, 0, sms)[0]
    assert info["mode"] == mode
    q, k, v = (torch.zeros((B, H, N, 128), dtype=torch.bfloat16, device=DEV) for _ in range(3))
    out = torch.empty((B, H, N, 128), dtype=torch.float32, device=DEV)
    sl = torch.zeros((H,), dtype=torch.float32, device=DEV)
    fn = ops.fwd_noalloc if noalloc else ops.fwd
    fn(q, k, v, sl, out)  # first call outside the capture (one-time setup)
    torch.cuda.synchronize()
    types, T = _captured_node_types(lambda s: fn(q, k, v, sl, out, stream=s))
    assert types.count(T.cudaGraphNodeTypeKernel) == 1
    uses_scratch = info["slots"] > 0
    if (B, H, sms) == (1, 148, 148):
        assert not uses_scratch  # one whole sequence per SM
    assert types.count(T.cudaGraphNodeTypeMemset) == (1 if uses_scratch else 0), types
