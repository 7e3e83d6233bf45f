"""The layer's forward and backward captured in a CUDA graph and replayed.

A training loop drives the library through CUDA graphs to drop launch latency; the calls
enqueue on the caller's stream and allocate nothing, so the whole step (fused referral and
attention forward, then the attention backward with its count, scan, row pass and gather,
the last four launched with programmatic stream serialization) can be captured once and
replayed. The replays must give what the eager calls give: the same edges and forward
outputs bit for bit, and gradients equal up to the order of their fp32 sums (the bucket
order of the gather path comes from integer atomics).
"""
import pytest
import torch

import sparse_dynamic_routing_b200 as gm
from sparse_dynamic_routing_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    gm.load_library()
    gm.gm_check_device_errors()
    yield


def _close(a, b, what):
    ref = b.double()
    err = (a.double() - ref).abs().max().item()
    assert err <= 1e-5 * max(ref.abs().max().item(), 1e-30), (what, err)


@pytest.mark.parametrize("name,B", [("layer_b8_n4096_s4_local", 1), ("layer_b8_n4096_s2", 1)])
def test_step_captured_in_a_graph_matches_eager_calls(name, B):
    wl = I.WORKLOADS[name].with_(B=B)
    dev = torch.device("cuda", 0)
    x = {k: v.to(dev) for k, v in I.make(wl, grad=True).items()}
    n, hq, hkv, d = wl.n, wl.hq, wl.hkv, wl.d
    f32 = torch.float32
    ai = torch.empty((B, n, hkv, wl.s1), dtype=torch.int32, device=dev)
    aw = torch.empty((B, n, hkv, wl.s1), dtype=f32, device=dev)
    o = torch.empty_like(x["q"])
    lse = torch.empty((B, n, hq), dtype=f32, device=dev)
    dq = torch.empty((B, n, hq, d), dtype=f32, device=dev)
    dk = torch.empty((B, n, hkv, d), dtype=f32, device=dev)
    dv = torch.empty_like(dk)
    dlw = torch.empty((B, n, hkv, wl.s1), dtype=f32, device=dev)
    ws = torch.empty(gm.gm_sea_backward_workspace_size(x["q"].dtype, wl.s1, B, n, hq, hkv, d),
                     dtype=torch.uint8, device=dev)

    def step(stream):
        gm.gm_ser_sea_forward(x["q"], x["k"], x["v"], x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"],
                              wl.s1, wl.scale, out_idx=ai, out_w=aw, o=o, lse=lse, stream=stream)
        gm.gm_sea_backward(x["q"], x["k"], x["v"], x["dout"], ai, aw, wl.scale, dq=dq, dk=dk, dv=dv,
                           dlogw=dlw, workspace=ws, stream=stream)

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step(side)  # eager, on the stream the graph is captured from
    torch.cuda.synchronize(dev)
    gm.gm_check_device_errors()
    eager = [t.clone() for t in (ai, aw, o, lse, dq, dk, dv, dlw)]
    for t in (ai, aw, o, lse, dq, dk, dv, dlw):
        t.zero_()

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step(side)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize(dev)
    gm.gm_check_device_errors()
    for got, want, what in zip((ai, aw, o, lse), eager[:4], ("A' idx", "A' w", "o", "lse")):
        assert torch.equal(got, want), what
    for got, want, what in zip((dq, dk, dv, dlw), eager[4:], ("dq", "dk", "dv", "dlogw")):
        _close(got, want, what)
    del graph
