"""GPU parity of the leg sparsification and its backward (through the C ABI) against the oracle.

Bars: leg indices and weights bit-exact (the kernel claims the oracle's fp32 roundings in the
oracle's order); gradients (fp32 on the GPU, fp64 in the oracle) within a relative bound of a
few fp32 ulps of the largest term. A full training chain (legs -> fused SER/SEA -> SEA
backward -> SER backward -> leg backward) is checked against the oracle's chain.
"""
import numpy as np
import pytest
import torch

import oracle
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


def t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(x):
    return x.detach().cpu().numpy()


def assert_legs_equal(got, want):
    for g, w, name in zip(got, want, ("a1_idx", "a1_w", "a2_idx", "a2_w")):
        g = host(g)
        if g.dtype == np.float32:
            np.testing.assert_array_equal(g.view(np.uint32), w.view(np.uint32), err_msg=name)
        else:
            np.testing.assert_array_equal(g, w, err_msg=name)


def assert_rel(got, want, what, rtol=1e-5):
    got = host(got).astype(np.float64).reshape(want.shape)
    scale = max(float(np.abs(want).max()), 1e-30)
    err = np.abs(got - want)
    bad = err > rtol * np.abs(want) + rtol * scale
    assert not bad.any(), f"{what}: max error {err.max():.3g} (scale {scale:.3g})"


def random_legs_case(seed, B, n, k, s0, shared=False, zero_frac=0.1, mix_zero_frac=0.1):
    rng = np.random.default_rng(seed)
    hi = np.broadcast_to(np.arange(1, n + 1)[None, :, None, None], (B, n, k, s0))
    ei = rng.integers(0, hi).astype(np.int32)
    ew = rng.dirichlet(np.ones(s0) * 0.7, (B, n, k)).astype(np.float32)
    ew[rng.random(ew.shape) < zero_frac] = 0.0
    shape = (k, k) if shared else (B, n, k, k)
    m1 = rng.dirichlet(np.ones(k), shape[:-1]).astype(np.float32)
    m2 = rng.dirichlet(np.ones(k), shape[:-1]).astype(np.float32)
    m1[rng.random(m1.shape) < mix_zero_frac] = 0.0
    return ei, ew, m1, m2, rng


LEG_SHAPES = [  # k, s0, s2, s3, n, shared
    (8, 4, 4, 4, 300, False), (8, 2, 2, 2, 128, False), (4, 4, 4, 16, 97, False),
    (2, 3, 5, 1, 61, True), (1, 1, 1, 1, 33, False), (16, 2, 4, 4, 50, False),
    (32, 1, 8, 3, 40, True), (3, 5, 2, 7, 45, False), (8, 4, 32, 1, 70, False),
    # thread-per-row shapes with ragged token counts
    (8, 4, 4, 4, 301, False), (8, 2, 3, 2, 97, True), (4, 4, 4, 1, 45, False),
    (4, 2, 2, 3, 63, False), (16, 2, 4, 4, 51, True), (16, 2, 1, 2, 7, False),
]


@pytest.mark.parametrize("k,s0,s2,s3,n,shared", LEG_SHAPES)
def test_leg_forward_and_backward_shapes(k, s0, s2, s3, n, shared):
    B = 2
    ei, ew, m1, m2, rng = random_legs_case(k * 1000 + s0 * 100 + s2 * 10 + s3, B, n, k, s0, shared)
    want = oracle.leg_sparsify(ei, ew, m1, m2, s2, s3)
    assert want[4] == 0
    got = gm.gm_leg_sparsify(t(ei), t(ew), t(m1), t(m2), s2, s3)
    assert_legs_equal(got, want[:4])
    g1 = rng.standard_normal((B, n, k, s2)).astype(np.float32)
    g2 = rng.standard_normal((B, n, k, s3)).astype(np.float32)
    dew_r, dm1_r, dm2_r, _ = oracle.leg_backward(ei, ew, m1, m2, g1, g2)
    dew, dm1, dm2 = gm.gm_leg_backward(t(ei), t(ew), t(m1), t(m2), t(g1), t(g2))
    assert_rel(dew, dew_r, "dew")
    assert_rel(dm1, dm1_r, "dmix1")
    assert_rel(dm2, dm2_r, "dmix2")
    assert np.all(host(dew)[ew == 0] == 0)
    gm.gm_leg_backward(t(ei), t(ew), t(m1), t(m2), t(g1), t(g2), dew=dew, dmix1=dm1, dmix2=dm2,
                       accumulate=True)
    assert_rel(dew, 2 * dew_r, "2 dew")
    assert_rel(dm1, 2 * dm1_r, "2 dmix1")
    gm.gm_check_device_errors()


def test_leg_full_size_layer_inputs():
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"]
    x = I.leg_inputs(wl)
    want = oracle.leg_sparsify(x["e_idx"], x["e_w"], x["mix1"], x["mix2"], wl.s2, wl.s3)
    g = {key: v.cuda() for key, v in x.items()}
    got = gm.gm_leg_sparsify(g["e_idx"], g["e_w"], g["mix1"], g["mix2"], wl.s2, wl.s3)
    assert_legs_equal(got, want[:4])
    rng = np.random.default_rng(5)
    g1 = rng.standard_normal(want[1].shape).astype(np.float32)
    g2 = rng.standard_normal(want[3].shape).astype(np.float32)
    ref = oracle.leg_backward(x["e_idx"], x["e_w"], x["mix1"], x["mix2"], g1, g2)
    out = gm.gm_leg_backward(g["e_idx"], g["e_w"], g["mix1"], g["mix2"], t(g1), t(g2))
    for o, r, name in zip(out, ref[:3], ("dew", "dmix1", "dmix2")):
        assert_rel(o, r, name)
    gm.gm_check_device_errors()


def test_leg_dyadic_ties_bit_exact():
    rng = np.random.default_rng(11)
    B, n, k, s0 = 2, 64, 8, 4
    hi = np.broadcast_to(np.arange(1, n + 1)[None, :, None, None], (B, n, k, s0))
    ei = np.minimum(rng.integers(0, 6, (B, n, k, s0)), hi - 1).astype(np.int32)  # many repeats
    vals = np.array([0.0, 0.5, 0.25, 0.125], np.float32)
    ew = vals[rng.integers(0, 4, ei.shape)]
    m1 = vals[rng.integers(0, 4, (B, n, k, k))]
    m2 = vals[rng.integers(0, 4, (B, n, k, k))]
    want = oracle.leg_sparsify(ei, ew, m1, m2, 3, 4)
    got = gm.gm_leg_sparsify(t(ei), t(ew), t(m1), t(m2), 3, 4)
    assert_legs_equal(got, want[:4])
    g1 = rng.standard_normal((B, n, k, 3)).astype(np.float32)
    g2 = rng.standard_normal((B, n, k, 4)).astype(np.float32)
    ref = oracle.leg_backward(ei, ew, m1, m2, g1, g2)
    out = gm.gm_leg_backward(t(ei), t(ew), t(m1), t(m2), t(g1), t(g2))
    for o, r, name in zip(out, ref[:3], ("dew", "dmix1", "dmix2")):
        assert_rel(o, r, name)
    gm.gm_check_device_errors()


def test_leg_out_of_range_and_empty():
    ei, ew, m1, m2, _ = random_legs_case(3, 1, 40, 4, 2, zero_frac=0.0)
    ei[0, 12, 1, 0] = 40
    ei[0, 30, 3, 1] = -7
    ei[0, 5, 0, 1] = 1 << 24
    ew[0, 5, 0, 1] = 0.0  # inactive: ignored, not flagged on its own
    want = oracle.leg_sparsify(ei, ew, m1, m2, 4, 4)
    assert want[4] == 2
    gm.gm_check_device_errors()
    got = gm.gm_leg_sparsify(t(ei), t(ew), t(m1), t(m2), 4, 4)
    with pytest.raises(gm.GMIndexRangeError):
        gm.gm_check_device_errors()
    assert_legs_equal(got, want[:4])
    e = torch.empty((0, 16, 8, 4), dtype=torch.int32, device="cuda")
    w = torch.empty((0, 16, 8, 4), dtype=torch.float32, device="cuda")
    m = torch.empty((8, 8), dtype=torch.float32, device="cuda")
    a1i, _, _, a2w = gm.gm_leg_sparsify(e, w, m, m, 4, 2)
    assert a1i.shape == (0, 16, 8, 4) and a2w.shape == (0, 16, 8, 2)
    gm.gm_check_device_errors()


def test_training_chain_from_stored_edges_f32():
    # stored edges -> legs -> fused SER/SEA -> SEA backward -> SER backward -> leg backward
    # two edge channels: with one, the coefficient gradient is zero up to rounding (scaling a
    # first leg's row scales its referral row, and attention ignores a common factor)
    wl = I.WORKLOADS["tiny_b1_n128_s2_f32"].with_(hq=4, hkv=2)
    x = I.make(wl, grad=True)
    le = I.leg_inputs(wl)
    a1i, a1w, a2i, a2w, _ = oracle.leg_sparsify(le["e_idx"], le["e_w"], le["mix1"], le["mix2"],
                                                wl.s2, wl.s3)
    oi, ow, _ = oracle.ser(a1i, a1w, a2i, a2w, wl.s1)
    _, _, _, dlw, _ = oracle.sea_backward(x["q"], x["k"], x["v"], x["dout"], oi, ow, wl.scale)
    d1, d2, _ = oracle.ser_backward(a1i, a1w, a2i, a2w, dlw.astype(np.float32), grad_is_log=True)
    want = oracle.leg_backward(le["e_idx"], le["e_w"], le["mix1"], le["mix2"],
                               d1.astype(np.float32), d2.astype(np.float32))

    g = {key: v.cuda() for key, v in list(x.items()) + list(le.items())}
    legs = gm.gm_leg_sparsify(g["e_idx"], g["e_w"], g["mix1"], g["mix2"], wl.s2, wl.s3)
    assert_legs_equal(legs, (a1i, a1w, a2i, a2w))
    ai, aw, _, _ = gm.gm_ser_sea_forward(g["q"], g["k"], g["v"], *legs, wl.s1, wl.scale)
    _, _, _, dl = gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], ai, aw, wl.scale)
    e1, e2 = gm.gm_ser_backward(*legs, dl, grad_is_log=True)
    got = gm.gm_leg_backward(g["e_idx"], g["e_w"], g["mix1"], g["mix2"], e1, e2)
    for o, r, name in zip(got, want[:3], ("dew", "dmix1", "dmix2")):
        assert_rel(o, r, name, rtol=1e-3)
    gm.gm_check_device_errors()
