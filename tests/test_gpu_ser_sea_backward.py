"""GPU parity of gm_ser_sea_backward: the attention backward on A' with the referral backward
of its d ln w fused into the row pass, through the C ABI.

Bars: dq, dK, dV, d ln w as the SEA backward parity (2e-2 max-abs for bf16 features against
the fp64 oracle, 1e-4 for fp32); dw1, dw2 against the oracle's referral backward fed the
kernel's own d ln w (relative, a few fp32 ulps of the largest term; dw2 is an fp32 atomic
sum). Against the unfused pair (gm_sea_backward then gm_ser_backward) dq, d ln w and dw1 are
identical bit for bit. Sources: "Graph Machine: Towards Better Pretraining via Edges", ai.info
summary, "Key Contributions" item 3 and "Methodology in Plain English", referral paragraph.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_dynamic_routing_b200 as gm
from sparse_dynamic_routing_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    gm.load_library()
    gm.gm_check_device_errors()
    yield


def host(t):
    return t.detach().cpu().double().numpy()


def assert_close(got, want, tol, what):
    err = np.abs(host(got).reshape(want.shape) - want).max()
    assert np.isfinite(err) and err <= tol, f"{what}: {err:.3g} > {tol}"


def assert_rel(got, want, what, rtol=1e-5):
    got = host(got).reshape(want.shape)
    scale = max(float(np.abs(want).max()), 1e-30)
    err = np.abs(got - want)
    assert not (err > rtol * np.abs(want) + rtol * scale).any(), f"{what}: {err.max():.3g}"


def run_case(wl):
    x = I.make(wl, grad=True)
    g = {k: v.cuda() for k, v in x.items()}
    ai, aw, _, _ = gm.gm_ser_sea_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"], g["a2_idx"],
                                         g["a2_w"], wl.s1, wl.scale)
    fused = gm.gm_ser_sea_backward(g["q"], g["k"], g["v"], g["dout"], g["a1_idx"], g["a1_w"],
                                   g["a2_idx"], g["a2_w"], ai, aw, wl.scale)
    gm.gm_check_device_errors()
    return x, g, ai, aw, fused


@pytest.mark.parametrize("name,B,n,s", [("layer_b8_n4096_s4_local", 2, 300, 4),
                                        ("layer_b8_n4096_s2", 1, 257, 2),
                                        ("layer_b8_n4096_s4_local", 1, 64, 4)])
def test_fused_backward_matches_oracle(name, B, n, s):
    wl = I.WORKLOADS[name].with_(B=B, n=n, s1=s, s2=s, s3=s)
    x, g, ai, aw, (dq, dk, dv, dlw, dw1, dw2) = run_case(wl)
    oi, ow = ai.cpu().numpy(), aw.cpu().numpy()
    want = oracle.sea_backward(x["q"], x["k"], x["v"], x["dout"], oi, ow, wl.scale)
    tol = TOL[wl.dtype]
    for got, ref, what in zip((dq, dk, dv, dlw), want[:4], ("dq", "dk", "dv", "dlogw")):
        assert_close(got, ref, tol, what)
    r1, r2, bad = oracle.ser_backward(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], dlw.cpu(),
                                      grad_is_log=True)
    assert bad == 0
    assert_rel(dw1, r1, "dw1")
    assert_rel(dw2, r2, "dw2")


def test_fused_backward_equals_the_unfused_pair_at_full_size():
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"]
    x, g, ai, aw, (dq, dk, dv, dlw, dw1, dw2) = run_case(wl)
    sq, sk, sv, slw = gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], ai, aw, wl.scale)
    s1, s2 = gm.gm_ser_backward(g["a1_idx"], g["a1_w"], g["a2_idx"], g["a2_w"], slw, grad_is_log=True)
    gm.gm_check_device_errors()
    assert torch.equal(dq, sq) and torch.equal(dlw, slw) and torch.equal(dw1, s1)
    for a, b, what in ((dk, sk, "dk"), (dv, sv, "dv"), (dw2, s2, "dw2")):  # fp32 sums in varying order
        err = float((a - b).abs().max())
        assert err <= 1e-5 * float(b.abs().max()), f"{what}: {err:.3g}"


def test_accumulate_adds_to_every_output():
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"].with_(B=1, n=200)
    x, g, ai, aw, first = run_case(wl)
    outs = [t.clone() for t in first]
    gm.gm_ser_sea_backward(g["q"], g["k"], g["v"], g["dout"], g["a1_idx"], g["a1_w"], g["a2_idx"],
                           g["a2_w"], ai, aw, wl.scale, *outs, accumulate=True)
    gm.gm_check_device_errors()
    for a, b, what in zip(outs, first, ("dq", "dk", "dv", "dlogw", "dw1", "dw2")):
        err = float((a - 2 * b).abs().max())
        assert err <= 1e-5 * max(float(b.abs().max()), 1e-20), f"{what}: {err:.3g}"


def test_unfused_fallback_for_other_budgets():
    """s2 = 3 is not a fused shape: the call runs the two backward passes one after the other."""
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"].with_(B=1, n=150, s1=4, s2=3, s3=3)
    x, g, ai, aw, (dq, dk, dv, dlw, dw1, dw2) = run_case(wl)
    want = oracle.sea_backward(x["q"], x["k"], x["v"], x["dout"], ai.cpu(), aw.cpu(), wl.scale)
    assert_close(dq, want[0], TOL["bf16"], "dq")
    r1, r2, _ = oracle.ser_backward(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], dlw.cpu(),
                                    grad_is_log=True)
    assert_rel(dw1, r1, "dw1")
    assert_rel(dw2, r2, "dw2")
    with pytest.raises(gm.GMError):  # accumulation needs the fused path
        gm.gm_ser_sea_backward(g["q"], g["k"], g["v"], g["dout"], g["a1_idx"], g["a1_w"],
                               g["a2_idx"], g["a2_w"], ai, aw, wl.scale, dq, dk, dv, dlw, dw1, dw2,
                               accumulate=True)
