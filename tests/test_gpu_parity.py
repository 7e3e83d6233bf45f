"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Every input comes from the seeded generators; every expected value from the oracle. Bars:
SER indices bit-exact and SER weights bit-exact (the kernels claim identical fp32 rounding;
the required bar is 1e-6 relative); SEA outputs and gradients within 1e-4 max-abs for fp32
features and 2e-2 max-abs for bf16 features, against fp64 on the same (bf16) inputs.
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
    gm.gm_check_device_errors()  # start with a clear error flag
    yield


def cuda(x):
    return {k: v.cuda() for k, v in x.items()}


def host(t):
    return t.detach().cpu()


def assert_ser_equal(gi, gw, oi, ow):
    gi, gw = host(gi).numpy(), host(gw).numpy()
    np.testing.assert_array_equal(gi, oi)
    np.testing.assert_allclose(gw, ow, rtol=1e-6, atol=0)
    np.testing.assert_array_equal(gw.view(np.uint32), ow.view(np.uint32))


def assert_close(got, want, tol, what):
    got = host(got).double().numpy().reshape(want.shape)
    both_inf = np.isneginf(got) & np.isneginf(want)
    with np.errstate(invalid="ignore"):
        diff = np.where(both_inf, 0.0, np.abs(got - want))
    err = float(np.nanmax(diff)) if diff.size else 0.0
    assert not np.isnan(diff).any(), f"{what}: NaN"
    assert err <= tol, f"{what}: max-abs error {err:.3g} > {tol}"
    return err


# ---- the five workloads ------------------------------------------------------------------


def test_tiny_ser_then_sea_f32():
    wl = I.WORKLOADS["tiny_b1_n128_s2_f32"]
    x = I.make(wl)
    oi, ow, bad = oracle.ser(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], wl.s1)
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], oi, ow, wl.scale)
    g = cuda(x)
    gi, gw = gm.gm_ser_forward(g["a1_idx"], g["a1_w"], g["a2_idx"], g["a2_w"], wl.s1)
    assert_ser_equal(gi, gw, oi, ow)
    o, lse = gm.gm_sea_forward(g["q"], g["k"], g["v"], gi, gw, wl.scale)
    assert_close(o, o_ref, TOL["f32"], "o")
    assert_close(lse, lse_ref, TOL["f32"], "lse")
    fi, fw, fo, flse = gm.gm_ser_sea_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"],
                                             g["a2_idx"], g["a2_w"], wl.s1, wl.scale)
    assert_ser_equal(fi, fw, oi, ow)
    assert torch.equal(fo, o) and torch.equal(flse, lse), "fused != SER then SEA"
    gm.gm_check_device_errors()


@pytest.mark.parametrize("name", ["layer_b8_n4096_s2", "layer_b8_n4096_s4_local"])
def test_layer_fused_forward_full_size(name):
    wl = I.WORKLOADS[name]
    x = I.make(wl)
    oi, ow, bad = oracle.ser(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], wl.s1)
    assert bad == 0
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], oi, ow, wl.scale)
    g = cuda(x)
    fi, fw, fo, flse = gm.gm_ser_sea_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"],
                                             g["a2_idx"], g["a2_w"], wl.s1, wl.scale)
    assert_ser_equal(fi, fw, oi, ow)
    assert_close(fo, o_ref, TOL["bf16"], "o")
    assert_close(flse, lse_ref, TOL["bf16"], "lse")
    # the unfused entry points give the same bits
    gi, gw = gm.gm_ser_forward(g["a1_idx"], g["a1_w"], g["a2_idx"], g["a2_w"], wl.s1)
    assert torch.equal(gi, fi) and torch.equal(gw, fw)
    o, lse = gm.gm_sea_forward(g["q"], g["k"], g["v"], gi, gw, wl.scale)
    assert torch.equal(o, fo) and torch.equal(lse, flse)
    gm.gm_check_device_errors()


def test_stack_of_21_layers_carries_edges():
    wl = I.WORKLOADS["stack21_b16_n4096_s4"]
    x = I.make(wl)
    e_idx, e_w = x["idx"].numpy(), x["w"].numpy()
    g_idx, g_w = x["idx"].cuda(), x["w"].cuda()
    rng = np.random.default_rng(4)
    for layer in range(wl.layers):
        f = I.layer_features(wl, layer) if layer else {k: x[k] for k in ("q", "k", "v")}
        gf = cuda(f)
        ni, nw, o, lse = gm.gm_ser_sea_forward(gf["q"], gf["k"], gf["v"], g_idx, g_w, g_idx,
                                               g_w, wl.s1, wl.scale)
        e_idx, e_w, bad = oracle.ser(e_idx, e_w, e_idx, e_w, wl.s1)
        assert bad == 0
        assert_ser_equal(ni, nw, e_idx, e_w)
        if layer in (0, wl.layers - 1):
            # the first layer and the last (edges collapsed toward the first positions: hot
            # rows, heavy merges) on every row
            o_ref, lse_ref, _ = oracle.sea_forward(f["q"], f["k"], f["v"], e_idx, e_w, wl.scale)
            assert_close(o, o_ref, TOL["bf16"], f"o L{layer}")
            assert_close(lse, lse_ref, TOL["bf16"], f"lse L{layer}")
        else:
            rows = np.sort(rng.choice(wl.B * wl.n, size=512, replace=False))
            rows[:2] = [0, wl.B * wl.n - 1]
            o_ref, lse_ref, _ = oracle.sea_forward(f["q"], f["k"], f["v"], e_idx, e_w, wl.scale,
                                                   rows=rows)
            sel = torch.from_numpy(rows).cuda()
            assert_close(o.reshape(wl.B * wl.n, wl.hq, wl.d)[sel], o_ref, TOL["bf16"], f"o L{layer}")
            assert_close(lse.reshape(wl.B * wl.n, wl.hq)[sel], lse_ref, TOL["bf16"], f"lse L{layer}")
        g_idx, g_w = ni, nw
    gm.gm_check_device_errors()


def test_long_sequence_forward_and_backward():
    wl = I.WORKLOADS["long_b1_n32768_s4_train"]
    x = I.make(wl, grad=True)
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], x["idx"], x["w"], wl.scale)
    dq_ref, dk_ref, dv_ref, dlw_ref, _ = oracle.sea_backward(
        x["q"], x["k"], x["v"], x["dout"], x["idx"], x["w"], wl.scale)
    g = cuda(x)
    o, lse = gm.gm_sea_forward(g["q"], g["k"], g["v"], g["idx"], g["w"], wl.scale)
    assert_close(o, o_ref, TOL["bf16"], "o")
    assert_close(lse, lse_ref, TOL["bf16"], "lse")
    assert gm.gm_sea_backward_workspace_size(torch.bfloat16, wl.s, wl.B, wl.n, wl.hq, wl.hkv,
                                             wl.d) > 0
    for ws in ("auto", None):  # gather path, atomic path
        dq, dk, dv, dlw = gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], g["idx"], g["w"],
                                             wl.scale, workspace=ws)
        assert_close(dq, dq_ref, TOL["bf16"], f"dq ({ws})")
        assert_close(dk, dk_ref, TOL["bf16"], f"dk ({ws})")
        assert_close(dv, dv_ref, TOL["bf16"], f"dv ({ws})")
        assert_close(dlw, dlw_ref, TOL["bf16"], f"dlogw ({ws})")
        # accumulate = 1 adds onto the buffers' contents
        gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], g["idx"], g["w"], wl.scale,
                           dq=dq, dk=dk, dv=dv, dlogw=dlw, accumulate=True, workspace=ws)
        assert_close(dq, 2 * dq_ref, 2 * TOL["bf16"], f"2 dq ({ws})")
        assert_close(dk, 2 * dk_ref, 2 * TOL["bf16"], f"2 dk ({ws})")
        assert_close(dv, 2 * dv_ref, 2 * TOL["bf16"], f"2 dv ({ws})")
        assert_close(dlw, 2 * dlw_ref, 2 * TOL["bf16"], f"2 dlogw ({ws})")
    gm.gm_check_device_errors()


def test_backward_paths_on_hot_rows():
    # Every slot of a sequence points at a handful of rows (the padding row 0 included): the
    # gather path meets buckets with thousands of edges, the atomic path heavy contention.
    B, n, hq, hkv, d, s = 2, 700, 16, 8, 128, 4
    x = random_case(21, B, n, hq, hkv, d, s, "bf16", zero_frac=0.1)
    idx = x["idx"].clone()
    idx[..., 0] = 0
    idx[..., 1] = torch.minimum(torch.full_like(idx[..., 1], 5), idx[..., 1])
    x["idx"] = idx
    scale = 1.0 / np.sqrt(d)
    ref = oracle.sea_backward(x["q"], x["k"], x["v"], x["dout"], x["idx"], x["w"], scale)
    g = cuda(x)
    for ws in ("auto", None):
        got = gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], g["idx"], g["w"], scale,
                                 workspace=ws)
        for name, a_, b_ in zip(("dq", "dk", "dv", "dlogw"), got, ref[:4]):
            assert_close(a_, b_, TOL["bf16"], f"{name} ({ws})")
        # accumulating onto the first result: the hot rows (more than a few hundred records
        # each here) take the gather pass's atomic route without the zero-fill
        again = gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], g["idx"], g["w"], scale,
                                   dq=got[0], dk=got[1], dv=got[2], dlogw=got[3], workspace=ws,
                                   accumulate=True)
        for name, a_, b_ in zip(("dq", "dk", "dv", "dlogw"), again, ref[:4]):
            assert_close(a_, 2.0 * b_, 2 * TOL["bf16"], f"{name} accumulated ({ws})")
    gm.gm_check_device_errors()


# ---- shapes, ragged tails and degenerate cases -------------------------------------------


def random_case(seed, B, n, hq, hkv, d, s, dtype, zero_frac=0.2, causal=True):
    rng = np.random.default_rng(seed)
    hi = np.arange(1, n + 1)[None, :, None, None] if causal else n
    idx = rng.integers(0, np.broadcast_to(hi, (B, n, hkv, s))).astype(np.int32)
    if s > 1:
        idx[..., 1] = np.where(rng.random((B, n, hkv)) < 0.3, idx[..., 0], idx[..., 1])
    w = rng.random((B, n, hkv, s)).astype(np.float32)
    w[rng.random(w.shape) < zero_frac] = 0.0
    if n > 3:
        w[:, 3] = 0.0  # rows with no active slot
    td = torch.bfloat16 if dtype == "bf16" else torch.float32

    def feat(shape):
        return torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(td)

    return dict(q=feat((B, n, hq, d)), k=feat((B, n, hkv, d)), v=feat((B, n, hkv, d)),
                dout=feat((B, n, hq, d)), idx=torch.from_numpy(idx), w=torch.from_numpy(w))


SHAPES = [
    # B, n, hq, hkv, d, s, dtype
    (1, 1, 2, 1, 64, 2, "f32"),
    (3, 37, 2, 1, 64, 3, "f32"),
    (2, 45, 4, 4, 32, 5, "f32"),
    (1, 29, 8, 1, 128, 8, "f32"),
    (2, 33, 16, 8, 128, 4, "bf16"),
    (1, 50, 8, 2, 256, 13, "bf16"),
    (2, 17, 4, 1, 32, 32, "bf16"),
    (1, 70, 8, 8, 64, 1, "bf16"),
    (1, 21, 16, 2, 128, 6, "bf16"),
]


@pytest.mark.parametrize("B,n,hq,hkv,d,s,dtype", SHAPES)
def test_sea_shapes_forward_backward(B, n, hq, hkv, d, s, dtype):
    x = random_case(B * 1000 + n * 10 + s, B, n, hq, hkv, d, s, dtype)
    scale = 1.0 / np.sqrt(d)
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], x["idx"], x["w"], scale)
    ref = oracle.sea_backward(x["q"], x["k"], x["v"], x["dout"], x["idx"], x["w"], scale)
    g = cuda(x)
    o, lse = gm.gm_sea_forward(g["q"], g["k"], g["v"], g["idx"], g["w"], scale)
    tol = TOL[dtype]
    assert_close(o, o_ref, tol, "o")
    assert_close(lse, lse_ref, tol, "lse")
    for ws in ("auto", None):
        got = gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], g["idx"], g["w"], scale,
                                 workspace=ws)
        for name, a, b in zip(("dq", "dk", "dv", "dlogw"), got, ref[:4]):
            assert_close(a, b, tol, f"{name} ({ws})")
    gm.gm_check_device_errors()


@pytest.mark.parametrize("s2,s3,s1", [(1, 1, 1), (2, 2, 2), (4, 4, 4), (4, 4, 16), (8, 4, 32),
                                      (3, 5, 7), (2, 16, 3), (1, 32, 5), (32, 1, 32)])
def test_ser_shapes_and_fused(s2, s3, s1):
    rng = np.random.default_rng(s2 * 100 + s3 * 10 + s1)
    B, n, hkv, hq, d = 2, 53, 4, 8, 64

    def legs(s):
        hi = np.broadcast_to(np.arange(1, n + 1)[None, :, None, None], (B, n, hkv, s))
        idx = rng.integers(0, hi).astype(np.int32)
        # dyadic weights: exact products and sums, many ties
        w = np.array([0.0, 0.5, 0.25, 0.125], np.float32)[rng.integers(0, 4, (B, n, hkv, s))]
        return idx, w

    i1, w1 = legs(s2)
    i2, w2 = legs(s3)
    oi, ow, bad = oracle.ser(i1, w1, i2, w2, s1)
    assert bad == 0
    t = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    gi, gw = gm.gm_ser_forward(t(i1), t(w1), t(i2), t(w2), s1)
    assert_ser_equal(gi, gw, oi, ow)
    x = random_case(7, B, n, hq, hkv, d, 1, "bf16")
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], oi, ow)
    g = cuda(x)
    fi, fw, fo, flse = gm.gm_ser_sea_forward(g["q"], g["k"], g["v"], t(i1), t(w1), t(i2), t(w2),
                                             s1)
    assert_ser_equal(fi, fw, oi, ow)
    assert_close(fo, o_ref, TOL["bf16"], "o")
    assert_close(flse, lse_ref, TOL["bf16"], "lse")
    # the fused kernel may skip writing the edges
    _, _, fo2, _ = gm.gm_ser_sea_forward(g["q"], g["k"], g["v"], t(i1), t(w1), t(i2), t(w2), s1,
                                         want_edges=False, want_lse=False)
    assert torch.equal(fo2, fo)
    gm.gm_check_device_errors()


def test_ser_random_weights_non_causal_and_repeatable():
    rng = np.random.default_rng(99)
    B, n, k, s2, s3, s1 = 3, 301, 5, 4, 4, 4
    i1 = rng.integers(0, n, (B, n, k, s2)).astype(np.int32)
    i2 = rng.integers(0, n, (B, n, k, s3)).astype(np.int32)
    i2[..., 1] = i2[..., 0]
    w1 = rng.dirichlet(np.ones(s2) * 0.3, (B, n, k)).astype(np.float32)
    w2 = rng.dirichlet(np.ones(s3) * 0.3, (B, n, k)).astype(np.float32)
    w2[rng.random(w2.shape) < 0.1] = 0.0
    oi, ow, _ = oracle.ser(i1, w1, i2, w2, s1)
    t = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    a = gm.gm_ser_forward(t(i1), t(w1), t(i2), t(w2), s1)
    b = gm.gm_ser_forward(t(i1), t(w1), t(i2), t(w2), s1)
    assert_ser_equal(*a, oi, ow)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_empty_problems_launch_nothing():
    e = torch.empty((0, 16, 2, 2), dtype=torch.int32, device="cuda")
    ew = torch.empty((0, 16, 2, 2), dtype=torch.float32, device="cuda")
    oi, ow = gm.gm_ser_forward(e, ew, e, ew, 2)
    assert oi.shape == (0, 16, 2, 2)
    q = torch.empty((2, 0, 4, 64), dtype=torch.bfloat16, device="cuda")
    kv = torch.empty((2, 0, 2, 64), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((2, 0, 2, 3), dtype=torch.int32, device="cuda")
    w = torch.empty((2, 0, 2, 3), dtype=torch.float32, device="cuda")
    o, lse = gm.gm_sea_forward(q, kv, kv, idx, w)
    assert o.shape == q.shape
    gm.gm_sea_backward(q, kv, kv, q, idx, w)
    gm.gm_check_device_errors()


def test_out_of_range_index_is_skipped_and_flagged():
    x = random_case(5, 1, 40, 4, 2, 64, 4, "bf16", zero_frac=0.0)
    bad_idx = x["idx"].clone()
    bad_idx[0, 10, 1, 2] = 40      # == n
    bad_idx[0, 20, 0, 0] = -3
    ref_w = x["w"].clone()
    ref_w[0, 10, 1, 2] = 0.0
    ref_w[0, 20, 0, 0] = 0.0
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], x["idx"], ref_w)
    _, _, bad = oracle.sea_forward(x["q"], x["k"], x["v"], bad_idx, x["w"])
    assert bad > 0
    g = cuda(x)
    gm.gm_check_device_errors()
    o, lse = gm.gm_sea_forward(g["q"], g["k"], g["v"], bad_idx.cuda(), g["w"])
    with pytest.raises(gm.GMIndexRangeError):
        gm.gm_check_device_errors()
    gm.gm_check_device_errors()  # the flag was cleared
    assert_close(o, o_ref, TOL["bf16"], "o")
    assert_close(lse, lse_ref, TOL["bf16"], "lse")
    # SER: an active first-leg slot pointing outside [0, n)
    i1, w1 = x["idx"].numpy().copy(), x["w"].numpy().copy()
    i1[0, 7, 0, 1] = 1 << 20
    oi, ow, bad = oracle.ser(i1, w1, x["idx"].numpy(), x["w"].numpy(), 4)
    assert bad == 1
    gi, gw = gm.gm_ser_forward(torch.from_numpy(i1).cuda(), g["w"], g["idx"], g["w"], 4)
    with pytest.raises(gm.GMIndexRangeError):
        gm.gm_check_device_errors()
    assert_ser_equal(gi, gw, oi, ow)


# ---- SER backward -------------------------------------------------------------------------------


def assert_rel(got, want, what, rtol=1e-5):
    """fp32 sums of a few products per entry: relative error bounded by a few ulps of the
    largest term; atol scales with the largest magnitude."""
    got = host(got).double().numpy().reshape(want.shape)
    scale = max(float(np.abs(want).max()), 1e-30)
    err = np.abs(got - want)
    bad = err > rtol * np.abs(want) + rtol * scale
    assert not bad.any(), f"{what}: max error {err.max():.3g} (scale {scale:.3g})"


@pytest.mark.parametrize("s2,s3,s1,n", [(2, 2, 2, 128), (4, 4, 4, 300), (4, 4, 2, 97),
                                        (3, 5, 7, 61), (8, 4, 32, 40), (1, 1, 1, 33)])
def test_ser_backward_shapes(s2, s3, s1, n):
    rng = np.random.default_rng(s2 * 100 + s3 * 10 + s1)
    B, k = 2, 3

    def legs(s):
        hi = np.broadcast_to(np.arange(1, n + 1)[None, :, None, None], (B, n, k, s))
        idx = rng.integers(0, hi).astype(np.int32)
        w = rng.dirichlet(np.ones(s) * 0.7, (B, n, k)).astype(np.float32)
        w[rng.random(w.shape) < 0.1] = 0.0
        return idx, w

    i1, w1 = legs(s2)
    i2, w2 = legs(s3)
    g = rng.standard_normal((B, n, k, s1)).astype(np.float32)
    want1, want2, _ = oracle.ser_backward(i1, w1, i2, w2, g)
    t = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    d1, d2 = gm.gm_ser_backward(t(i1), t(w1), t(i2), t(w2), t(g))
    assert_rel(d1, want1, "dw1")
    assert_rel(d2, want2, "dw2")
    # accumulate adds onto the buffers
    gm.gm_ser_backward(t(i1), t(w1), t(i2), t(w2), t(g), dw1=d1, dw2=d2, accumulate=True)
    assert_rel(d1, 2 * want1, "2 dw1")
    assert_rel(d2, 2 * want2, "2 dw2")
    gm.gm_check_device_errors()


def test_ser_backward_full_size_layer():
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"]
    x = I.make(wl)
    rng = np.random.default_rng(77)
    g = rng.standard_normal((wl.B, wl.n, wl.hkv, wl.s1)).astype(np.float32)
    want1, want2, _ = oracle.ser_backward(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], g)
    d1, d2 = gm.gm_ser_backward(x["a1_idx"].cuda(), x["a1_w"].cuda(), x["a2_idx"].cuda(),
                                x["a2_w"].cuda(), torch.from_numpy(g).cuda())
    assert_rel(d1, want1, "dw1")
    assert_rel(d2, want2, "dw2", rtol=1e-4)  # up to thousands of fp32 atomic terms per entry
    gm.gm_check_device_errors()


def test_training_chain_through_both_backwards_f32():
    # forward SER -> SEA, backward SEA -> d ln w -> SER backward, against the oracle's chain
    wl = I.WORKLOADS["tiny_b1_n128_s2_f32"]
    x = I.make(wl, grad=True)
    oi, ow, _ = oracle.ser(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], wl.s1)
    _, _, _, dlw_ref, _ = oracle.sea_backward(x["q"], x["k"], x["v"], x["dout"], oi, ow, wl.scale)
    want1, want2, _ = oracle.ser_backward(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"],
                                          dlw_ref.astype(np.float32), grad_is_log=True)
    g = cuda(x)
    ai, aw, _, _ = gm.gm_ser_sea_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"],
                                         g["a2_idx"], g["a2_w"], wl.s1, wl.scale)
    _, _, _, dlw = gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], ai, aw, wl.scale)
    d1, d2 = gm.gm_ser_backward(g["a1_idx"], g["a1_w"], g["a2_idx"], g["a2_w"], dlw,
                                grad_is_log=True)
    assert_rel(d1, want1, "dw1", rtol=1e-3)
    assert_rel(d2, want2, "dw2", rtol=1e-3)
    # d ln w / W through the flag equals dividing first
    e1, e2 = gm.gm_ser_backward(g["a1_idx"], g["a1_w"], g["a2_idx"], g["a2_w"],
                                torch.where(aw > 0, dlw / aw, torch.zeros_like(dlw)))
    assert torch.allclose(d1, e1, rtol=1e-6, atol=1e-6) and torch.allclose(d2, e2, rtol=1e-6, atol=1e-6)
    gm.gm_check_device_errors()
