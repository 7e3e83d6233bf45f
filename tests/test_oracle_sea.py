"""Pins of the oracle's sparse edge attention (SEA) forward against the mathematics.

SEA (Graph Machine: Towards Better Pretraining via Edges, ai.info summary, "Key
Contributions" item 3 and "Methodology in Plain English", SEA paragraph) reads K/V at each
position's edge indices per KV head and scores entry j as scale * q.k_j + ln w_j, then takes
a softmax over the entries and a weighted sum of V. Pins here:

* closed form: with every causal predecessor as a slot and equal weights per row, SEA is
  dense causal softmax attention (torch SDPA, fp64, K/V repeated over the GQA group);
* with arbitrary weights (zeros and duplicate indices included) SEA equals dense attention
  with the additive mask ln(sum of the row's weights at each position) - this pins the ln w
  term, the w = 0 rule and the duplicate rule;
* special cases: s = 1 returns V[t] exactly, a constant factor on a row's weights shifts lse
  by its log and leaves o unchanged, permuting slots changes nothing, a row with no active
  slot gives o = 0 and lse = -inf, the row-subset form equals the full form.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def rand_feats(rng, B, n, hq, hkv, d):
    q = rng.standard_normal((B, n, hq, d)).astype(np.float32)
    k = rng.standard_normal((B, n, hkv, d)).astype(np.float32)
    v = rng.standard_normal((B, n, hkv, d)).astype(np.float32)
    return q, k, v


def sdpa(q, k, v, scale, mask=None, causal=False):
    """torch SDPA in fp64; q [B,n,hq,d], k/v [B,n,hkv,d] -> o [B,n,hq,d]."""
    hq, hkv = q.shape[2], k.shape[2]
    G = hq // hkv
    Q = torch.from_numpy(q).double().transpose(1, 2)
    K = torch.from_numpy(k).double().transpose(1, 2).repeat_interleave(G, dim=1)
    V = torch.from_numpy(v).double().transpose(1, 2).repeat_interleave(G, dim=1)
    o = F.scaled_dot_product_attention(Q, K, V, attn_mask=mask, is_causal=causal, scale=scale)
    return o.transpose(1, 2).numpy()


@pytest.mark.parametrize("hq,hkv,d", [(2, 1, 64), (4, 2, 8), (8, 8, 16), (16, 8, 32)])
def test_sea_with_all_causal_slots_is_causal_attention(hq, hkv, d):
    rng = np.random.default_rng(hq * 100 + d)
    B, n = 2, 13
    q, k, v = rand_feats(rng, B, n, hq, hkv, d)
    idx = np.broadcast_to(np.arange(n, dtype=np.int32), (B, n, hkv, n)).copy()
    pos = np.arange(n)[None, :, None, None]
    w = np.where(idx <= pos, 1.0 / (pos + 1), 0.0).astype(np.float32)
    scale = 1.0 / math.sqrt(d)
    o, lse, bad = oracle.sea_forward(q, k, v, idx, w, scale)
    assert bad == 0
    want = sdpa(q, k, v, scale, causal=True)
    np.testing.assert_allclose(o.reshape(want.shape), want, rtol=0, atol=1e-12)
    # lse = logsumexp_t<=i(scale q.k_t) + ln w_i, w_i = fl32(1/(i+1)) the stored weight
    G = hq // hkv
    Q = torch.from_numpy(q).double()
    K = torch.from_numpy(k).double().repeat_interleave(G, dim=2)
    s = torch.einsum("bihd,bthd->bhit", Q, K) * scale
    s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    lnw = torch.log(torch.from_numpy(w[0, :, 0, 0]).double())
    want_lse = (torch.logsumexp(s, -1) + lnw).transpose(1, 2)
    np.testing.assert_allclose(lse.reshape(B, n, hq), want_lse.numpy(), rtol=0, atol=1e-12)


def test_sea_with_arbitrary_weights_is_attention_with_log_weight_mask():
    rng = np.random.default_rng(11)
    B, n, hq, hkv, d, s = 2, 10, 4, 2, 16, 5
    q, k, v = rand_feats(rng, B, n, hq, hkv, d)
    idx = rng.integers(0, n, (B, n, hkv, s)).astype(np.int32)
    idx[:, :, :, 1] = idx[:, :, :, 0]  # duplicate index in every row
    w = rng.random((B, n, hkv, s)).astype(np.float32)
    w[rng.random(w.shape) < 0.25] = 0.0
    w[:, :, :, 0] = np.maximum(w[:, :, :, 0], 0.1)  # keep one slot active per row
    scale = 0.3
    o, lse, bad = oracle.sea_forward(q, k, v, idx, w, scale)
    assert bad == 0
    # dense additive mask: ln(sum of active weights at t), -inf where none
    Wd = np.zeros((B, hkv, n, n))
    for b in range(B):
        for i in range(n):
            for h in range(hkv):
                for j in range(s):
                    if w[b, i, h, j] > 0:
                        Wd[b, h, i, idx[b, i, h, j]] += float(w[b, i, h, j])
    with np.errstate(divide="ignore"):
        M = torch.from_numpy(np.log(Wd)).repeat_interleave(hq // hkv, dim=1)
    want = sdpa(q, k, v, scale, mask=M)
    np.testing.assert_allclose(o.reshape(want.shape), want, rtol=0, atol=1e-12)
    G = hq // hkv
    Q = torch.from_numpy(q).double()
    K = torch.from_numpy(k).double().repeat_interleave(G, dim=2)
    sc = torch.einsum("bihd,bthd->bhit", Q, K) * scale + M
    want_lse = torch.logsumexp(sc, -1).transpose(1, 2).numpy()
    np.testing.assert_allclose(lse.reshape(B, n, hq), want_lse, rtol=0, atol=1e-12)


def test_sea_single_slot_returns_the_gathered_value_row():
    rng = np.random.default_rng(12)
    B, n, hq, hkv, d = 2, 9, 4, 2, 8
    q, k, v = rand_feats(rng, B, n, hq, hkv, d)
    idx = rng.integers(0, n, (B, n, hkv, 1)).astype(np.int32)
    w = (rng.random((B, n, hkv, 1)) + 0.1).astype(np.float32)
    o, lse, _ = oracle.sea_forward(q, k, v, idx, w, 0.25)
    o = o.reshape(B, n, hq, d)
    lse = lse.reshape(B, n, hq)
    for b in range(B):
        for i in range(n):
            for hqi in range(hq):
                h = hqi // (hq // hkv)
                t = idx[b, i, h, 0]
                assert np.array_equal(o[b, i, hqi], v[b, t, h].astype(np.float64))
                z = 0.25 * float(np.dot(q[b, i, hqi].astype(np.float64), k[b, t, h])) \
                    + math.log(float(w[b, i, h, 0]))
                assert abs(lse[b, i, hqi] - z) < 1e-12


def test_sea_row_weight_scale_permutation_and_empty_rows():
    rng = np.random.default_rng(13)
    B, n, hq, hkv, d, s = 1, 12, 2, 1, 16, 4
    q, k, v = rand_feats(rng, B, n, hq, hkv, d)
    idx = rng.integers(0, n, (B, n, hkv, s)).astype(np.int32)
    w = (rng.random((B, n, hkv, s)) + 0.05).astype(np.float32)
    o, lse, _ = oracle.sea_forward(q, k, v, idx, w, 0.2)
    # scaling a row's weights by 2^3 (exact in fp32) shifts lse by 3 ln 2, o unchanged
    o2, lse2, _ = oracle.sea_forward(q, k, v, idx, w * np.float32(8.0), 0.2)
    np.testing.assert_allclose(o2, o, atol=1e-13, rtol=0)
    np.testing.assert_allclose(lse2, lse + 3 * math.log(2.0), atol=1e-12, rtol=0)
    # slot order does not matter
    perm = rng.permutation(s)
    o3, lse3, _ = oracle.sea_forward(q, k, v, idx[..., perm].copy(), w[..., perm].copy(), 0.2)
    np.testing.assert_allclose(o3, o, atol=1e-13, rtol=0)
    np.testing.assert_allclose(lse3, lse, atol=1e-13, rtol=0)
    # a row with no active slot: o = 0, lse = -inf; its garbage indices are never read
    w0, i0 = w.copy(), idx.copy()
    w0[0, 4] = 0.0
    i0[0, 4] = 10 ** 6
    o4, lse4, bad = oracle.sea_forward(q, k, v, i0, w0, 0.2)
    assert bad == 0
    assert np.all(o4.reshape(B, n, hq, d)[0, 4] == 0)
    assert np.all(np.isneginf(lse4.reshape(B, n, hq)[0, 4]))
    keep = np.arange(n) != 4
    np.testing.assert_array_equal(o4[keep], o[keep])
    # an active slot outside [0, n) is skipped (same as w = 0) and counted
    w5, i5 = w.copy(), idx.copy()
    i5[0, 6, 0, 2] = n
    o5, _, bad = oracle.sea_forward(q, k, v, i5, w5, 0.2)
    w5[0, 6, 0, 2] = 0.0
    o6, _, _ = oracle.sea_forward(q, k, v, idx, w5, 0.2)
    assert bad == hq // hkv  # counted once per query head that reads the slot
    np.testing.assert_array_equal(o5, o6)


def test_sea_row_subset_equals_full():
    rng = np.random.default_rng(14)
    B, n, hq, hkv, d, s = 3, 20, 4, 2, 8, 3
    q, k, v = rand_feats(rng, B, n, hq, hkv, d)
    idx = rng.integers(0, n, (B, n, hkv, s)).astype(np.int32)
    w = rng.random((B, n, hkv, s)).astype(np.float32)
    o, lse, _ = oracle.sea_forward(q, k, v, idx, w, 0.5)
    rows = np.array([59, 0, 17, 33, 33])
    os_, ls, _ = oracle.sea_forward(q, k, v, idx, w, 0.5, rows=rows)
    np.testing.assert_array_equal(os_, o[rows])
    np.testing.assert_array_equal(ls, lse[rows])
