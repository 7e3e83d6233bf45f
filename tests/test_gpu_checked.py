"""The checked build (libgm_b200_checked.so) on the GPU, through the C ABI.

It must give the regular build's results bit for bit on valid edges, and report through
gm_check_device_errors (GM_ERR_EDGE_INVALID) an input edge whose weight is negative, NaN or
infinite, or whose active index lies beyond its own row's position (edges are causal: the
pages' padding token sits at position 0 of every sequence, "Graph Machine: Towards Better
Pretraining via Edges", ai.info summary, "Methodology in Plain English", hybrid paragraph).
The regular build reports none of these (only indices outside [0, n)).
"""
import contextlib

import numpy as np
import pytest
import torch

import sparse_dynamic_routing_b200 as gm
from sparse_dynamic_routing_b200 import _binding as bnd
from sparse_dynamic_routing_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    regular = bnd.load_library()
    checked = bnd.open_library(bnd.CHECKED_LIB_PATH)
    assert checked.gm_checked_build() == 1 and regular.gm_checked_build() == 0
    for lib in (regular, checked):
        with using(lib):
            gm.gm_check_device_errors()
    return regular, checked


@contextlib.contextmanager
def using(lib):
    saved = bnd._lib
    bnd._lib = lib
    try:
        yield
    finally:
        bnd._lib = saved


def layer(B=1, n=96):
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"].with_(B=B, n=n)
    x = I.make(wl, grad=True)
    return wl, {k: v.clone().cuda() for k, v in x.items()}


def step(wl, g):
    ai, aw, o, lse = gm.gm_ser_sea_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"], g["a2_idx"],
                                           g["a2_w"], wl.s1, wl.scale)
    grads = gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], ai, aw, wl.scale)
    return (ai, aw, o, lse) + tuple(grads)


def test_checked_build_matches_the_regular_build_on_valid_edges(libs):
    regular, checked = libs
    wl, g = layer(B=2, n=200)
    with using(regular):
        want = step(wl, g)
        gm.gm_check_device_errors()
    with using(checked):
        got = step(wl, g)
        gm.gm_check_device_errors()  # valid edges: nothing reported
    for name, a, b in zip(("idx", "w", "o", "lse"), got[:4], want[:4]):
        assert torch.equal(a, b), name
    # dq and d ln w come from the row pass in a fixed order: the same bits; dK/dV are fp32
    # scatter sums whose order varies run to run
    for name, a, b in zip(("dq", "dk", "dv", "dlogw"), got[4:], want[4:]):
        scale = float(b.abs().max())
        err = float((a - b).abs().max())
        if name in ("dq", "dlogw"):
            assert torch.equal(a, b), f"{name}: max diff {err:.3g}"
        else:
            assert err <= 1e-5 * scale, f"{name}: max diff {err:.3g} (scale {scale:.3g})"


def corrupt(name, value):
    """A (tensor key, edit) pair applied to the layer's first-leg or second-leg edges."""
    def edit(g):
        if name == "noncausal":
            g["a1_idx"][0, 10, 3, 1] = 11     # row i = 10 points at position 11 (< n)
            g["a1_w"][0, 10, 3, 1] = 0.25
        else:
            g["a2_w"][0, 20, 5, 2] = value    # negative / NaN / inf weight
    return edit


@pytest.mark.parametrize("case,value", [("noncausal", None), ("weight", -0.5),
                                        ("weight", float("nan")), ("weight", float("inf"))])
def test_bad_leg_edges_are_reported_by_the_checked_build_only(libs, case, value):
    regular, checked = libs
    for lib, expect in ((regular, False), (checked, True)):
        wl, g = layer()
        corrupt(case, value)(g)
        with using(lib):
            gm.gm_ser_sea_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"], g["a2_idx"],
                                  g["a2_w"], wl.s1, wl.scale)
            if expect:
                with pytest.raises(gm.GMEdgeInvalidError):
                    gm.gm_check_device_errors()
            else:
                gm.gm_check_device_errors()


def test_bad_sea_and_backward_edges_are_reported(libs):
    _, checked = libs
    wl, g = layer()
    idx = torch.zeros((1, wl.n, wl.hkv, 4), dtype=torch.int32, device="cuda")
    w = torch.full((1, wl.n, wl.hkv, 4), 0.25, device="cuda")
    idx[0, 5, 2, 3] = 40  # row 5 points at position 40
    with using(checked):
        gm.gm_sea_forward(g["q"], g["k"], g["v"], idx, w, wl.scale)
        with pytest.raises(gm.GMEdgeInvalidError):
            gm.gm_check_device_errors()
        idx[0, 5, 2, 3] = 0
        w[0, 7, 1, 0] = float("nan")
        gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], idx, w, wl.scale)
        with pytest.raises(gm.GMEdgeInvalidError):
            gm.gm_check_device_errors()
        w[0, 7, 1, 0] = 0.25
        gm.gm_sea_forward(g["q"], g["k"], g["v"], idx, w, wl.scale)
        gm.gm_check_device_errors()  # clean again


def test_bad_stored_refresh_and_chain_edges_are_reported(libs):
    _, checked = libs
    wl, g = layer()
    le = {k: v.clone().cuda() for k, v in I.leg_inputs(wl).items()}
    with using(checked):
        le["e_idx"][0, 3, 0, 0] = 9
        le["e_w"][0, 3, 0, 0] = 0.5
        gm.gm_leg_sparsify(le["e_idx"], le["e_w"], le["mix1"], le["mix2"], wl.s2, wl.s3)
        with pytest.raises(gm.GMEdgeInvalidError):
            gm.gm_check_device_errors()
        f_idx = torch.zeros_like(g["a1_idx"])
        f_w = torch.full_like(g["a1_w"], 0.1)
        f_idx[0, 30, 0, 0] = 31
        gm.gm_ser_refresh_forward(g["a1_idx"], g["a1_w"], g["a2_idx"], g["a2_w"], f_idx, f_w, wl.s1)
        with pytest.raises(gm.GMEdgeInvalidError):
            gm.gm_check_device_errors()
        leg3_i, leg3_w = g["a2_idx"].clone(), g["a2_w"].clone()
        leg3_w[0, 50, 4, 0] = -1.0
        gm.gm_ser_chain_forward(g["a1_idx"], g["a1_w"], [(g["a2_idx"], g["a2_w"]), (leg3_i, leg3_w)],
                                wl.s2, wl.s1)
        with pytest.raises(gm.GMEdgeInvalidError):
            gm.gm_check_device_errors()
