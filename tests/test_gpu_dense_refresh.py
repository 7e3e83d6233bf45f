"""GPU parity of gm_dense_refresh_edges (through the C ABI) against the oracle.

The kernel picks, per (b, i, KV head), the sf causal positions of largest attention mass of a
dense layer (the mean over the head's query group of exp(scale q.k - lse)). Scores run on the
tensor cores (bf16 products, fp32 sums) and masses in fp32, the oracle in fp64, so a position
whose mass lies within rounding of the sf-th largest may legitimately be exchanged: the bar is
what is unique, exactly - every position whose mass clears the sf-th largest by more than the
rounding bound is kept, none below it by more than that is, slots are distinct, causal,
ordered and padded as specified - and weights within 1e-4 relative of the fp64 masses. Exact
ties (uniform attention) must go to the smaller positions, bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_dynamic_routing_b200 as gm
from sparse_dynamic_routing_b200 import inputs as I

pytestmark = pytest.mark.gpu

RTOL = 1e-4  # masses: fp32 scores and exponentials against fp64


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    gm.load_library()
    gm.gm_check_device_errors()
    yield


def qk(seed, B, n, hq, hkv, d):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, n, hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, n, hkv, d, generator=g).to(torch.bfloat16)
    return q, k


def check_valid(gi, gw, mass, rows, n, sf):
    """gi, gw [nrows, hkv, sf] from the kernel; mass [nrows, hkv, n] fp64 from the oracle."""
    for r_idx, r in enumerate(rows):
        i = int(r) % n
        kept = min(sf, i + 1)
        for h in range(mass.shape[1]):
            m = mass[r_idx, h, : i + 1]
            idx, w = gi[r_idx, h], gw[r_idx, h]
            what = f"row {r} head {h}"
            np.testing.assert_array_equal(idx[kept:], 0, err_msg=what)
            np.testing.assert_array_equal(w[kept:], 0.0, err_msg=what)
            sel = idx[:kept]
            assert len(set(sel.tolist())) == kept, what + ": repeated position"
            assert (sel >= 0).all() and (sel <= i).all(), what + ": non-causal position"
            assert (np.diff(w[:kept]) <= 0).all(), what + ": weights not in descending order"
            np.testing.assert_allclose(w[:kept], m[sel], rtol=RTOL, atol=1e-12, err_msg=what)
            tau = np.sort(m)[::-1][kept - 1]
            tol = RTOL * tau + 1e-12
            assert (m[sel] >= tau - tol).all(), what + ": kept a position below the cut"
            must = np.nonzero(m > tau + tol)[0]
            assert set(must.tolist()) <= set(sel.tolist()), what + ": dropped a position above the cut"


@pytest.mark.parametrize("B,n,hq,hkv,d,sf", [
    (2, 300, 4, 2, 128, 4),    # G = 2, ragged last query block, two sequences
    (1, 130, 2, 2, 64, 2),     # G = 1, head_dim 64
    (1, 257, 8, 2, 128, 8),    # G = 4 (64-key blocks)
    (1, 129, 4, 2, 64, 1),     # sf = 1
    (3, 64, 4, 2, 128, 3),     # sequences shorter than a block
])
def test_dense_refresh_matches_oracle(B, n, hq, hkv, d, sf):
    q, k = qk(B * 1000 + n + sf, B, n, hq, hkv, d)
    scale = float(np.float32(1 / np.sqrt(d)))
    lse = oracle.dense_lse(q, k, scale).astype(np.float32)
    mass = oracle.dense_mass(q, k, lse, scale)
    gi, gw = gm.gm_dense_refresh_edges(q.cuda(), k.cuda(), torch.from_numpy(lse).cuda(), sf, scale)
    gm.gm_check_device_errors()
    gi = gi.cpu().numpy().reshape(B * n, hkv, sf)
    gw = gw.cpu().numpy().reshape(B * n, hkv, sf)
    check_valid(gi, gw, mass, np.arange(B * n), n, sf)
    # where the selection is unambiguous the oracle's indices are matched exactly
    oi, _ = oracle.dense_refresh(q, k, lse, sf, scale)
    agree = (gi == oi.reshape(B * n, hkv, sf)).all(-1).mean()
    assert agree > 0.99, f"only {agree:.3f} of rows agree with the oracle's order exactly"


def test_uniform_attention_ties_go_to_the_smaller_positions():
    B, n, hq, hkv, d, sf = 1, 200, 4, 2, 128, 4
    q = torch.zeros(B, n, hq, d, dtype=torch.bfloat16)
    k = torch.randn(B, n, hkv, d).to(torch.bfloat16)
    lse = oracle.dense_lse(q, k, 0.1).astype(np.float32)
    oi, ow = oracle.dense_refresh(q, k, lse, sf, 0.1)
    gi, gw = gm.gm_dense_refresh_edges(q.cuda(), k.cuda(), torch.from_numpy(lse).cuda(), sf, 0.1)
    gm.gm_check_device_errors()
    np.testing.assert_array_equal(gi.cpu().numpy(), oi)
    np.testing.assert_allclose(gw.cpu().numpy(), ow, rtol=1e-5, atol=0)


def test_bench_shape_sampled_rows_and_refresh_chain():
    """The bench layer's shape (B=8, n=4096, 16/8 heads, d=128), sf=4, checked on sampled rows;
    the produced edges then feed the fused referral with refresh edges, which must match the
    oracle's referral on the same edges bit for bit."""
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"]
    x = I.make(wl)
    scale = wl.scale
    q, k = x["q"], x["k"]
    rows = np.concatenate([[0, 1, 2, 127, 128, 4095, 4096, wl.B * wl.n - 1],
                           np.random.default_rng(3).choice(wl.B * wl.n, 120, replace=False)])
    # the oracle's normaliser on the sampled rows (the other rows' lse is 0: their edges are
    # still causal and finite, and only feed the referral check below)
    lse = np.zeros((wl.B * wl.n, wl.hq), np.float32)
    lse[rows] = oracle.dense_lse(q, k, scale, rows=rows).astype(np.float32)
    lse = lse.reshape(wl.B, wl.n, wl.hq)
    mass = oracle.dense_mass(q, k, lse, scale, rows=rows)
    gq, gk, glse = q.cuda(), k.cuda(), torch.from_numpy(lse).cuda()
    fi, fw = gm.gm_dense_refresh_edges(gq, gk, glse, 4, scale)
    gm.gm_check_device_errors()
    sel = torch.from_numpy(rows).cuda()
    check_valid(fi.reshape(-1, wl.hkv, 4)[sel].cpu().numpy(), fw.reshape(-1, wl.hkv, 4)[sel].cpu().numpy(),
                mass, rows, wl.n, 4)
    g = {key: v.cuda() for key, v in x.items()}
    ai, aw, _, _ = gm.gm_ser_sea_refresh_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"],
                                                 g["a2_idx"], g["a2_w"], fi, fw, wl.s1, scale)
    oi, ow, bad = oracle.ser_refresh(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], fi.cpu(), fw.cpu(),
                                     wl.s1)
    assert bad == 0
    np.testing.assert_array_equal(ai.cpu().numpy(), oi)
    np.testing.assert_array_equal(aw.cpu().numpy().view(np.uint32), ow.view(np.uint32))
    gm.gm_check_device_errors()


def test_rejects_unsupported_shapes():
    q = torch.zeros(1, 8, 4, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 8, 2, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 8, 4, device="cuda")
    with pytest.raises(gm.GMError):
        gm.gm_dense_refresh_edges(q, k, lse, 9)  # sf > 8
    with pytest.raises(gm.GMError):
        gm.gm_dense_refresh_edges(q.float(), k.float(), lse, 4)  # fp32 features
