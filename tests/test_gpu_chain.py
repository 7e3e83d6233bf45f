"""GPU parity of the multi-step referral (through the C ABI) against the oracle.

Bars: referral indices and weights bit-exact at every shape (each step claims the oracle's
fp32 roundings and order); gradients within a relative bound of a few fp32 ulps of the
largest term (fp32 atomics on every leg); attention outputs of the fused call within 2e-2
(bf16) or 1e-4 (fp32) max-abs of the fp64 oracle on the oracle's edges.
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


def edges(rng, B, n, k, s, zero_frac=0.1):
    hi = np.broadcast_to(np.arange(1, n + 1)[None, :, None, None], (B, n, k, s))
    idx = rng.integers(0, hi).astype(np.int32)
    w = rng.dirichlet(np.ones(s) * 0.7, (B, n, k)).astype(np.float32)
    w[rng.random(w.shape) < zero_frac] = 0.0
    return idx, w


# budgets s2 = s3 = s_mid in {2, 4} with s1 <= 4 and up to 4 legs run the per-thread backward
@pytest.mark.parametrize("s2,s3,s_mid,s1,nlegs,n", [(2, 2, 2, 2, 2, 128), (4, 4, 4, 4, 3, 300),
                                                    (4, 4, 4, 2, 2, 97), (2, 3, 5, 4, 4, 61),
                                                    (1, 2, 2, 3, 7, 45), (3, 3, 3, 3, 1, 40),
                                                    (2, 2, 2, 3, 4, 150), (4, 4, 4, 1, 1, 70)])
def test_chain_forward_and_backward(s2, s3, s_mid, s1, nlegs, n):
    rng = np.random.default_rng(s2 * 1000 + s3 * 100 + s_mid * 10 + nlegs)
    B, k = 2, 3
    a1 = edges(rng, B, n, k, s2)
    legs = [edges(rng, B, n, k, s3) for _ in range(nlegs)]
    oi, ow, bad = oracle.ser_chain(*a1, legs, s_mid, s1)
    assert bad == 0
    g_legs = [(t(i), t(w)) for i, w in legs]
    gi, gw = gm.gm_ser_chain_forward(t(a1[0]), t(a1[1]), g_legs, s_mid, s1)
    assert_bits(gi, gw, oi, ow)
    g = rng.standard_normal((B, n, k, s1)).astype(np.float32)
    d1_ref, dl_ref, _ = oracle.ser_chain_backward(*a1, legs, s_mid, g)
    d1, dl = gm.gm_ser_chain_backward(t(a1[0]), t(a1[1]), g_legs, s_mid, t(g))
    assert_rel(d1, d1_ref, "dw1", rtol=1e-4)
    for m, (got, want) in enumerate(zip(dl, dl_ref)):
        assert_rel(got, want, f"dleg{m}", rtol=1e-4)
    # the log-weight form and accumulation
    glog = (g.astype(np.float64) * ow).astype(np.float32)
    e1_ref, el_ref, _ = oracle.ser_chain_backward(*a1, legs, s_mid, glog, grad_is_log=True)
    e1, el = gm.gm_ser_chain_backward(t(a1[0]), t(a1[1]), g_legs, s_mid, t(glog), grad_is_log=True)
    assert_rel(e1, e1_ref, "dw1 (log)", rtol=1e-4)
    gm.gm_ser_chain_backward(t(a1[0]), t(a1[1]), g_legs, s_mid, t(g), dw1=d1, dlegs=dl, accumulate=True)
    assert_rel(d1, 2 * d1_ref, "2 dw1", rtol=1e-4)
    assert_rel(dl[-1], 2 * dl_ref[-1], "2 dleg", rtol=1e-4)
    gm.gm_check_device_errors()


def test_power_of_one_matrix_with_aliased_gradients():
    # A^3: every leg is A, and the legs' gradients land in one buffer (they add up)
    rng = np.random.default_rng(9)
    B, n, k, s = 2, 200, 2, 4
    A = edges(rng, B, n, k, s)
    oi, ow, _ = oracle.ser_chain(*A, [A, A], s, s)
    gA = (t(A[0]), t(A[1]))
    gi, gw = gm.gm_ser_chain_forward(*gA, [gA, gA], s, s)
    assert_bits(gi, gw, oi, ow)
    g = rng.standard_normal((B, n, k, s)).astype(np.float32)
    d1_ref, dl_ref, _ = oracle.ser_chain_backward(*A, [A, A], s, g)
    shared = torch.empty((B, n, k, s), dtype=torch.float32, device="cuda")
    d1, _ = gm.gm_ser_chain_backward(*gA, [gA, gA], s, t(g), dlegs=[shared, shared])
    assert_rel(d1, d1_ref, "dw1", rtol=1e-4)
    assert_rel(shared, dl_ref[0] + dl_ref[1], "dA (both legs)", rtol=1e-4)
    gm.gm_check_device_errors()


@pytest.mark.parametrize("s,nlegs,s1", [(2, 2, 2), (4, 2, 4), (4, 3, 4), (2, 3, 3)])
def test_fused_chain_forward_bf16_tile(s, nlegs, s1):
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"].with_(B=2, n=300, s1=s1, s2=s, s3=s)
    x = I.make(wl)
    rng = np.random.default_rng(50 + s + nlegs)
    legs = [(x["a2_idx"].numpy(), x["a2_w"].numpy())] + \
        [edges(rng, wl.B, wl.n, wl.hkv, s) for _ in range(nlegs - 1)]
    oi, ow, _ = oracle.ser_chain(x["a1_idx"], x["a1_w"], legs, s, s1)
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], oi, ow, wl.scale)
    g = {key: v.cuda() for key, v in x.items()}
    ai, aw, o, lse = gm.gm_ser_sea_chain_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"],
                                                 [(t(i), t(w)) for i, w in legs], s, s1, wl.scale)
    assert_bits(ai, aw, oi, ow)
    assert_close(o, o_ref, 2e-2, "o")
    assert_close(lse, lse_ref, 2e-2, "lse")
    gm.gm_check_device_errors()


def test_fused_chain_forward_other_shapes_run_chain_then_attention():
    wl = I.WORKLOADS["tiny_b1_n128_s2_f32"]
    x = I.make(wl)
    rng = np.random.default_rng(4)
    legs = [(x["a2_idx"].numpy(), x["a2_w"].numpy()), edges(rng, wl.B, wl.n, wl.hkv, wl.s3)]
    oi, ow, _ = oracle.ser_chain(x["a1_idx"], x["a1_w"], legs, 3, wl.s1)
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], oi, ow, wl.scale)
    g = {key: v.cuda() for key, v in x.items()}
    ai, aw, o, lse = gm.gm_ser_sea_chain_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"],
                                                 [(t(i), t(w)) for i, w in legs], 3, wl.s1, wl.scale)
    assert_bits(ai, aw, oi, ow)
    assert_close(o, o_ref, 1e-4, "o")
    assert_close(lse, lse_ref, 1e-4, "lse")
    gm.gm_check_device_errors()


def test_fused_chain_full_size_layer():
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"]
    x = I.make(wl)
    a3 = [v.numpy() for v in I.edges(wl, 2, wl.s3, layer=1)]
    legs = [(x["a2_idx"].numpy(), x["a2_w"].numpy()), tuple(a3)]
    oi, ow, bad = oracle.ser_chain(x["a1_idx"], x["a1_w"], legs, wl.s2, wl.s1)
    assert bad == 0
    rows = np.random.default_rng(12).choice(wl.B * wl.n, 2048, replace=False)
    o_ref, lse_ref, _ = oracle.sea_forward(x["q"], x["k"], x["v"], oi, ow, wl.scale, rows=rows)
    g = {key: v.cuda() for key, v in x.items()}
    g_legs = [(t(i), t(w)) for i, w in legs]
    ai, aw, o, lse = gm.gm_ser_sea_chain_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"],
                                                 g_legs, wl.s2, wl.s1, wl.scale)
    assert_bits(ai, aw, oi, ow)
    sel = torch.from_numpy(rows).cuda()
    assert_close(o.reshape(wl.B * wl.n, wl.hq, wl.d)[sel], o_ref, 2e-2, "o")
    assert_close(lse.reshape(wl.B * wl.n, wl.hq)[sel], lse_ref, 2e-2, "lse")
    ci, cw = gm.gm_ser_chain_forward(g["a1_idx"], g["a1_w"], g_legs, wl.s2, wl.s1)
    assert torch.equal(ci, ai) and torch.equal(cw, aw)
    gm.gm_check_device_errors()


def misaligned(a):
    """`a` on the GPU at a data pointer 4 bytes past a 16-byte boundary (forces the warp kernels)."""
    src = torch.from_numpy(np.ascontiguousarray(a))
    flat = torch.empty(src.numel() + 4, dtype=src.dtype, device="cuda")
    view = flat[1:1 + src.numel()].view(src.shape)
    view.copy_(src)
    assert view.data_ptr() % 16 == 4
    return view


@pytest.mark.parametrize("s,nlegs", [(2, 2), (4, 2), (4, 3)])
def test_chain_backward_thread_and_warp_agree(s, nlegs):
    """The per-thread and warp-per-row chain backwards are picked by shape and alignment
    alone: the first-leg gradient must match bit for bit (leg gradients: fp32 atomics)."""
    rng = np.random.default_rng(40 + s * 10 + nlegs)
    B, n, k = 1, 160, 2
    a1 = edges(rng, B, n, k, s)
    legs = [edges(rng, B, n, k, s) for _ in range(nlegs)]
    g = rng.standard_normal((B, n, k, 4)).astype(np.float32)
    thread = gm.gm_ser_chain_backward(t(a1[0]), t(a1[1]), [(t(i), t(w)) for i, w in legs], s, t(g))
    warp = gm.gm_ser_chain_backward(misaligned(a1[0]), misaligned(a1[1]),
                                    [(misaligned(i), misaligned(w)) for i, w in legs], s, t(g))
    np.testing.assert_array_equal(thread[0].cpu().numpy().view(np.uint32),
                                  warp[0].cpu().numpy().view(np.uint32))
    for a, b in zip(thread[1], warp[1]):
        ref = b.cpu().double().numpy()
        err = np.abs(a.cpu().double().numpy() - ref).max()
        assert err <= 1e-5 * max(np.abs(ref).max(), 1e-30)
    # the forward: one thread per row (aligned legs) against one warp per row, bit for bit
    ft = gm.gm_ser_chain_forward(t(a1[0]), t(a1[1]), [(t(i), t(w)) for i, w in legs], s, 4)
    fw = gm.gm_ser_chain_forward(misaligned(a1[0]), misaligned(a1[1]),
                                 [(misaligned(i), misaligned(w)) for i, w in legs], s, 4)
    for a, b in zip(ft, fw):
        np.testing.assert_array_equal(a.cpu().numpy().view(np.uint32), b.cpu().numpy().view(np.uint32))
    gm.gm_check_device_errors()
