"""GPU parity of the referral with refresh edges (through the C ABI) against the oracle.

Bars: referral indices and weights bit-exact; attention outputs within 1e-4 (fp32 features)
or 2e-2 (bf16) max-abs of the fp64 oracle on the oracle's edges; gradients within a relative
bound of a few fp32 ulps of the largest term (fp32 atomics on the second leg).
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
    x = x.detach()
    return (x.float() if x.dtype == torch.bfloat16 else x).cpu().numpy()


def assert_bits(gi, gw, oi, ow):
    np.testing.assert_array_equal(host(gi), oi)
    np.testing.assert_array_equal(host(gw).view(np.uint32), ow.view(np.uint32))


def assert_close(got, want, tol, what):
    got = host(got).astype(np.float64).reshape(want.shape)
    both = np.isneginf(got) & np.isneginf(want)
    with np.errstate(invalid="ignore"):
        err = np.where(both, 0.0, np.abs(got - want))
    assert not np.isnan(err).any() and err.max() <= tol, f"{what}: {err.max():.3g} > {tol}"


def assert_rel(got, want, what, rtol=1e-5):
    got = host(got).astype(np.float64).reshape(want.shape)
    scale = max(float(np.abs(want).max()), 1e-30)
    err = np.abs(got - want)
    assert not (err > rtol * np.abs(want) + rtol * scale).any(), f"{what}: {err.max():.3g}"


def case(seed, B, n, k, s2, s3, sf, zero_frac=0.1):
    rng = np.random.default_rng(seed)

    def e(s):
        hi = np.broadcast_to(np.arange(1, n + 1)[None, :, None, None], (B, n, k, s))
        idx = rng.integers(0, hi).astype(np.int32)
        w = rng.dirichlet(np.ones(s) * 0.7, (B, n, k)).astype(np.float32)
        w[rng.random(w.shape) < zero_frac] = 0.0
        return idx, w

    return e(s2), e(s3), e(sf), rng


# (2,2,2,2), (4,4,4,4), (2,2,4,3), (4,4,2,2), (4,4,4,1) reach the per-thread backward (s1 < s2
# leaves slots unkept); the others the warp-per-row kernel
@pytest.mark.parametrize("s2,s3,sf,s1,n", [(2, 2, 2, 2, 128), (4, 4, 4, 4, 300), (4, 4, 8, 8, 97),
                                           (2, 2, 1, 3, 61), (1, 1, 6, 4, 33), (3, 3, 5, 8, 45),
                                           (2, 2, 4, 3, 150), (4, 4, 2, 2, 77), (4, 4, 4, 1, 64)])
def test_refresh_referral_forward_and_backward(s2, s3, sf, s1, n):
    B, k = 2, 3
    (i1, w1), (i2, w2), (fi, fw), rng = case(s2 * 100 + s3 * 10 + sf, B, n, k, s2, s3, sf)
    oi, ow, bad = oracle.ser_refresh(i1, w1, i2, w2, fi, fw, s1)
    assert bad == 0
    gi, gw = gm.gm_ser_refresh_forward(t(i1), t(w1), t(i2), t(w2), t(fi), t(fw), s1)
    assert_bits(gi, gw, oi, ow)
    g = rng.standard_normal((B, n, k, s1)).astype(np.float32)
    r1, r2, rf, _ = oracle.ser_refresh_backward(i1, w1, i2, w2, fi, fw, g)
    d1, d2, df = gm.gm_ser_refresh_backward(t(i1), t(w1), t(i2), t(w2), t(fi), t(fw), t(g))
    assert_rel(d1, r1, "dw1")
    assert_rel(d2, r2, "dw2")
    assert_rel(df, rf, "dfw")
    gm.gm_ser_refresh_backward(t(i1), t(w1), t(i2), t(w2), t(fi), t(fw), t(g), dw1=d1, dw2=d2,
                               dfw=df, accumulate=True)
    assert_rel(df, 2 * rf, "2 dfw")
    assert_rel(d1, 2 * r1, "2 dw1")
    gm.gm_check_device_errors()


def test_fused_refresh_forward_tiny_f32():
    wl = I.WORKLOADS["tiny_b1_n128_s2_f32"]
    x = I.make(wl)
    fi, fw = I.leg_inputs(wl)["e_idx"], I.leg_inputs(wl)["e_w"]  # the stored edges as refresh
    oi, ow, _ = oracle.ser_refresh(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], fi, fw, wl.s1)
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], oi, ow, wl.scale)
    g = {key: v.cuda() for key, v in x.items()}
    ai, aw, o, lse = gm.gm_ser_sea_refresh_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"],
                                                   g["a2_idx"], g["a2_w"], fi.cuda(), fw.cuda(),
                                                   wl.s1, wl.scale)
    assert_bits(ai, aw, oi, ow)
    assert_close(o, o_ref, 1e-4, "o")
    assert_close(lse, lse_ref, 1e-4, "lse")
    gm.gm_check_device_errors()


def test_fused_refresh_forward_full_size_layer():
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"]
    x = I.make(wl)
    le = I.leg_inputs(wl)
    fi, fw = le["e_idx"], le["e_w"]
    oi, ow, bad = oracle.ser_refresh(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], fi, fw, wl.s1)
    assert bad == 0
    rows = np.random.default_rng(8).choice(wl.B * wl.n, 2048, replace=False)
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], oi, ow, wl.scale, rows=rows)
    g = {key: v.cuda() for key, v in x.items()}
    ai, aw, o, lse = gm.gm_ser_sea_refresh_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"],
                                                   g["a2_idx"], g["a2_w"], fi.cuda(), fw.cuda(),
                                                   wl.s1, wl.scale)
    assert_bits(ai, aw, oi, ow)
    sel = torch.from_numpy(rows).cuda()
    assert_close(o.reshape(wl.B * wl.n, wl.hq, wl.d)[sel], o_ref, 2e-2, "o")
    assert_close(lse.reshape(wl.B * wl.n, wl.hq)[sel], lse_ref, 2e-2, "lse")
    gi, gw = gm.gm_ser_refresh_forward(g["a1_idx"], g["a1_w"], g["a2_idx"], g["a2_w"], fi.cuda(),
                                       fw.cuda(), wl.s1)
    assert torch.equal(gi, ai) and torch.equal(gw, aw)
    gm.gm_check_device_errors()


def test_refresh_out_of_range_is_skipped_and_flagged():
    (i1, w1), (i2, w2), (fi, fw), _ = case(5, 1, 50, 2, 2, 2, 3, zero_frac=0.0)
    fi[0, 20, 1, 2] = 50
    oi, ow, bad = oracle.ser_refresh(i1, w1, i2, w2, fi, fw, 4)
    assert bad == 1
    gm.gm_check_device_errors()
    gi, gw = gm.gm_ser_refresh_forward(t(i1), t(w1), t(i2), t(w2), t(fi), t(fw), 4)
    with pytest.raises(gm.GMIndexRangeError):
        gm.gm_check_device_errors()
    assert_bits(gi, gw, oi, ow)


@pytest.mark.parametrize("s,sf,s1", [(2, 2, 2), (2, 4, 4), (4, 2, 3), (4, 4, 4)])
def test_fused_refresh_forward_bf16_tile_shapes(s, sf, s1):
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"].with_(B=2, n=300, s1=s1, s2=s, s3=s)
    x = I.make(wl)
    (_, _), (_, _), (fi, fw), _ = case(77 + s + sf, wl.B, wl.n, wl.hkv, 1, 1, sf)
    oi, ow, _ = oracle.ser_refresh(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], fi, fw, s1)
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], oi, ow, wl.scale)
    g = {key: v.cuda() for key, v in x.items()}
    ai, aw, o, lse = gm.gm_ser_sea_refresh_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"],
                                                   g["a2_idx"], g["a2_w"], t(fi), t(fw), s1, wl.scale)
    assert_bits(ai, aw, oi, ow)
    assert_close(o, o_ref, 2e-2, "o")
    assert_close(lse, lse_ref, 2e-2, "lse")
    gm.gm_check_device_errors()


def misaligned(a):
    """`a` copied to the GPU at a data pointer 4 bytes past a 16-byte boundary: the dispatch
    then takes the warp-per-row kernels instead of the per-thread ones."""
    src = torch.from_numpy(np.ascontiguousarray(a))
    flat = torch.empty(src.numel() + 4, dtype=src.dtype, device="cuda")
    view = flat[1:1 + src.numel()].view(src.shape)
    view.copy_(src)
    assert view.data_ptr() % 16 == 4
    return view


def tie_case(seed, n, k, s2, s3, sf):
    """Targets from {0..3} and weights from {0, 1/8, 1/4, 1/2}: duplicate targets in most rows
    and exact ties between merged weights, so the tie-break decides the kept set."""
    rng = np.random.default_rng(seed)

    def e(s):
        idx = np.minimum(rng.integers(0, 4, (1, n, k, s)), np.arange(n)[None, :, None, None])
        w = rng.choice(np.float32([0.0, 0.125, 0.25, 0.5]), (1, n, k, s))
        return idx.astype(np.int32), w.astype(np.float32)

    return e(s2), e(s3), e(sf), rng.standard_normal((1, n, k, 4)).astype(np.float32)


@pytest.mark.parametrize("s,sf", [(2, 0), (4, 0), (2, 2), (2, 4), (4, 2), (4, 4)])
def test_thread_and_warp_backward_agree_bit_for_bit_on_ties(s, sf):
    """The per-thread and warp-per-row referral backwards are chosen by shape and alignment
    alone, so they must keep the same slots and give the same first-leg and refresh-slot
    gradient bits; the second-leg gradient (fp32 atomics) only to rounding order."""
    n, k, s1 = 96, 2, 4
    (i1, w1), (i2, w2), (fi, fw), g = tie_case(500 + 10 * s + sf, n, k, s, s, max(sf, 1))
    if sf:
        args = (i1, w1, i2, w2, fi, fw)
        thread = gm.gm_ser_refresh_backward(*[t(a) for a in args], t(g), grad_is_log=True)
        warp = gm.gm_ser_refresh_backward(*[misaligned(a) for a in args], t(g), grad_is_log=True)
        ref = oracle.ser_refresh_backward(*args, g, grad_is_log=True)
        names = ("dw1", "dw2", "dfw")
    else:
        args = (i1, w1, i2, w2)
        thread = gm.gm_ser_backward(*[t(a) for a in args], t(g), grad_is_log=True)
        warp = gm.gm_ser_backward(*[misaligned(a) for a in args], t(g), grad_is_log=True)
        ref = oracle.ser_backward(*args, g, grad_is_log=True)
        names = ("dw1", "dw2")
    for name, a, b, r in zip(names, thread, warp, ref):
        assert_rel(a, r, f"thread {name}")
        assert_rel(b, r, f"warp {name}")
        if name != "dw2":
            np.testing.assert_array_equal(host(a).view(np.uint32), host(b).view(np.uint32),
                                          err_msg=name)
    # the forward: the fused tile kernel's per-thread referral against the warp kernel
    gen = torch.Generator().manual_seed(s + sf)
    q = torch.randn((1, n, 2 * k, 128), generator=gen).to(torch.bfloat16).cuda()
    kv = torch.randn((1, n, k, 128), generator=gen).to(torch.bfloat16).cuda()
    if sf:
        wi, ww = gm.gm_ser_refresh_forward(*[t(a) for a in args], s1)
        fi_, fw_, _, _ = gm.gm_ser_sea_refresh_forward(q, kv, kv, *[t(a) for a in args], s1)
        oi, ow, _ = oracle.ser_refresh(*args, s1)
    else:
        wi, ww = gm.gm_ser_forward(*[t(a) for a in args], s1)
        fi_, fw_, _, _ = gm.gm_ser_sea_forward(q, kv, kv, *[t(a) for a in args], s1)
        oi, ow, _ = oracle.ser(*args, s1)
    assert_bits(wi, ww, oi, ow)
    assert_bits(fi_, fw_, oi, ow)
    # the standalone referral on misaligned legs takes the warp-per-row kernel
    if sf:
        mi, mw = gm.gm_ser_refresh_forward(*[misaligned(a) for a in args], s1)
    else:
        mi, mw = gm.gm_ser_forward(*[misaligned(a) for a in args], s1)
    assert_bits(mi, mw, oi, ow)
    gm.gm_check_device_errors()
