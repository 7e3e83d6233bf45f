"""GPU parity on order-sensitive merges: every sparsify kernel against the oracle, bit for bit.

The cases (tests/merge_order_cases.py) merge four candidates into one target with plain
three-decimal fp32 weights whose fp32 sum depends on the order of the adds. The oracle sums in
ascending candidate order (its CPU pins fix that); here each kernel that merges (the warp and
the per-thread referral, fused or not, with refresh edges, through a chain, and both leg
kernels) must return the same bits. Source of the operations: "Graph Machine: Towards Better
Pretraining via Edges", ai.info summary, "Key Contributions" item 3 and "Methodology in Plain
English", referral paragraph.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_dynamic_routing_b200 as gm
from merge_order_cases import asc, leg_case, refresh_case, ser_case

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


def assert_bits(gi, gw, oi, ow, what):
    np.testing.assert_array_equal(gi.cpu().numpy(), oi, err_msg=what)
    np.testing.assert_array_equal(gw.cpu().numpy().view(np.uint32), ow.view(np.uint32), err_msg=what)


def features(n, hkv, G=2, d=128, seed=0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((1, n, G * hkv, d), generator=g).to(torch.bfloat16).cuda()
    k = torch.randn((1, n, hkv, d), generator=g).to(torch.bfloat16).cuda()
    v = torch.randn((1, n, hkv, d), generator=g).to(torch.bfloat16).cuda()
    return q, k, v


@pytest.mark.parametrize("k", [1, 8])
def test_referral_merge_order(k):
    args, u, _ = ser_case(k=k)
    oi, ow, bad = oracle.ser(*args, 2)
    assert bad == 0 and ow[0, 7, 0, 0] == asc(u)
    g = [t(a) for a in args]
    gi, gw = gm.gm_ser_forward(*g, 2)
    assert_bits(gi, gw, oi, ow, "gm_ser_forward")
    q, kk, v = features(args[0].shape[1], k)
    for s1 in (2, 4):  # per-thread referral of the fused tile kernel, budgets 2 and 4
        oi1, ow1, _ = oracle.ser(*args, s1)
        fi, fw, _, _ = gm.gm_ser_sea_forward(q, kk, v, *g, s1)
        assert_bits(fi, fw, oi1, ow1, f"gm_ser_sea_forward s1={s1}")
    gm.gm_check_device_errors()


def test_chain_merge_order():
    args, u, _ = ser_case(k=8)
    a1_idx, a1_w, a2_idx, a2_w = args
    n = a1_idx.shape[1]
    ident_i = np.broadcast_to(np.arange(n, dtype=np.int32)[None, :, None, None], (1, n, 8, 2)).copy()
    ident_w = np.zeros((1, n, 8, 2), np.float32)
    ident_w[..., 0] = 1.0
    legs_np = [(a2_idx, a2_w), (ident_i, ident_w)]
    oi, ow, bad = oracle.ser_chain(a1_idx, a1_w, legs_np, 2, 2)
    assert bad == 0 and ow[0, 7, 0, 0] == asc(u)
    legs = [(t(i), t(w)) for i, w in legs_np]
    ci, cw = gm.gm_ser_chain_forward(t(a1_idx), t(a1_w), legs, 2, 2)
    assert_bits(ci, cw, oi, ow, "gm_ser_chain_forward")
    q, kk, v = features(n, 8)
    fi, fw, _, _ = gm.gm_ser_sea_chain_forward(q, kk, v, t(a1_idx), t(a1_w), legs, 2, 2)
    assert_bits(fi, fw, oi, ow, "gm_ser_sea_chain_forward")
    gm.gm_check_device_errors()


@pytest.mark.parametrize("k", [1, 8])
def test_refresh_merge_order(k):
    args, u, _ = refresh_case(k=k, s3=2)
    oi, ow, bad = oracle.ser_refresh(*args, 2)
    assert bad == 0 and ow[0, 7, 0, 0] == asc(u)
    g = [t(a) for a in args]
    gi, gw = gm.gm_ser_refresh_forward(*g, 2)
    assert_bits(gi, gw, oi, ow, "gm_ser_refresh_forward")
    q, kk, v = features(args[0].shape[1], k)
    fi, fw, _, _ = gm.gm_ser_sea_refresh_forward(q, kk, v, *g, 2)
    assert_bits(fi, fw, oi, ow, "gm_ser_sea_refresh_forward")
    gm.gm_check_device_errors()


@pytest.mark.parametrize("k", [2, 4, 8])  # 2: warp-per-token kernel; 4, 8: tiled kernel
def test_leg_merge_order(k):
    args, u, _ = leg_case(k=k)
    want = oracle.leg_sparsify(*args, 2, 2)
    assert want[4] == 0 and want[1][0, 3, 0, 0] == asc(u)
    got = gm.gm_leg_sparsify(*[t(a) for a in args], 2, 2)
    for x, (gg, ww) in enumerate(zip(got, want[:4])):
        gg = gg.cpu().numpy()
        if gg.dtype == np.float32:
            np.testing.assert_array_equal(gg.view(np.uint32), ww.view(np.uint32), err_msg=str(x))
        else:
            np.testing.assert_array_equal(gg, ww, err_msg=str(x))
    gm.gm_check_device_errors()
