"""GPU parity of the timed layer step at its full size, on every output element.

The step the benchmark times on layer_b8_n4096_s4_local (B = 8, n = 4096, 16 query / 8 KV
heads, d = 128, s = 4, bf16): the fused SER->SEA forward into caller buffers, then the SEA
backward on the refreshed edges through a workspace (the gather path), both on one
non-default stream, as the benchmark launches them. Every element is compared with the
oracle: SER bit for bit, SEA outputs and all four gradients within the bf16 bar (2e-2
max-abs against fp64 on the same bf16 inputs). A second case runs the same shapes with the
edges collapsed onto a few positions per sequence, so that most targets hold thousands of
records and the gather pass takes its split (hot target) route at full size.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_dynamic_routing_b200 as gm
from sparse_dynamic_routing_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    gm.load_library()
    gm.gm_check_device_errors()
    yield


def assert_close(got, want, tol, what):
    got = got.detach().cpu().double().numpy().reshape(want.shape)
    both_inf = np.isneginf(got) & np.isneginf(want)
    with np.errstate(invalid="ignore"):
        diff = np.where(both_inf, 0.0, np.abs(got - want))
    assert not np.isnan(diff).any(), f"{what}: NaN"
    err = float(np.nanmax(diff)) if diff.size else 0.0
    assert err <= tol, f"{what}: max-abs error {err:.3g} > {tol}"


def run_step(wl, x):
    """The benchmark's step: caller buffers, a workspace, one side stream."""
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in x.items()}
    B, n, hq, hkv, d, s1 = wl.B, wl.n, wl.hq, wl.hkv, wl.d, wl.s1
    f32 = torch.float32
    ap_i = torch.empty((B, n, hkv, s1), dtype=torch.int32, device=dev)
    ap_w = torch.empty((B, n, hkv, s1), dtype=f32, device=dev)
    o = torch.empty_like(g["q"])
    lse = torch.empty((B, n, hq), dtype=f32, device=dev)
    # stale contents in every output: the step must overwrite all of them
    dq = torch.full((B, n, hq, d), 7.0, dtype=f32, device=dev)
    dk = torch.full((B, n, hkv, d), 7.0, dtype=f32, device=dev)
    dv = torch.full_like(dk, -7.0)
    dlw = torch.full((B, n, hkv, s1), 7.0, dtype=f32, device=dev)
    ws = torch.full((gm.gm_sea_backward_workspace_size(g["q"].dtype, s1, B, n, hq, hkv, d),),
                    0xAB, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for _ in range(2):  # a second step over the same buffers and workspace
            gm.gm_ser_sea_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"], g["a2_idx"],
                                  g["a2_w"], s1, wl.scale, out_idx=ap_i, out_w=ap_w, o=o,
                                  lse=lse, stream=stream)
            gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], ap_i, ap_w, wl.scale, dq=dq,
                               dk=dk, dv=dv, dlogw=dlw, workspace=ws, stream=stream)
    stream.synchronize()
    gm.gm_check_device_errors()
    return ap_i, ap_w, o, lse, dq, dk, dv, dlw


def check_step(wl, x):
    ap_i, ap_w, o, lse, dq, dk, dv, dlw = run_step(wl, x)
    oi, ow, bad = oracle.ser(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], wl.s1)
    assert bad == 0
    np.testing.assert_array_equal(ap_i.cpu().numpy(), oi)
    np.testing.assert_array_equal(ap_w.cpu().numpy().view(np.uint32), ow.view(np.uint32))
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], oi, ow, wl.scale)
    assert_close(o, o_ref, TOL, "o")
    assert_close(lse, lse_ref, TOL, "lse")
    ref = oracle.sea_backward(x["q"], x["k"], x["v"], x["dout"], oi, ow, wl.scale)
    for name, got, want in zip(("dq", "dk", "dv", "dlogw"), (dq, dk, dv, dlw), ref[:4]):
        assert_close(got, want, TOL, name)
    return oi, ow


def test_bench_step_full_size_every_element():
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"]
    check_step(wl, I.make(wl, grad=True))


def test_bench_step_full_size_collapsed_edges():
    # Both legs point every slot at one of the first four positions of its sequence (or at
    # the token itself): the referral then keeps a handful of targets per sequence and KV
    # head, each with thousands of records.
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"]
    x = I.make(wl, grad=True)
    for leg in ("a1_idx", "a2_idx"):
        idx = x[leg]
        pos = torch.arange(wl.n, dtype=idx.dtype).view(1, wl.n, 1, 1)
        x[leg] = torch.minimum(idx % 4, pos)
    oi, ow = check_step(wl, x)
    # records per target row (b, t, h): far above the split threshold of a few hundred
    b = np.arange(wl.B).reshape(wl.B, 1, 1, 1)
    h = np.arange(wl.hkv).reshape(1, 1, wl.hkv, 1)
    keys = ((b * wl.n + oi) * wl.hkv + h)[ow > 0]
    assert np.bincount(keys.ravel()).max() > 1000, "the case should reach the split route"
