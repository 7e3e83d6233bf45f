"""Pins of the oracle's refresh edges from a dense attention layer.

Refresh edges may come from "the top positions of the most recent dense attention layer"
("Graph Machine: Towards Better Pretraining via Edges", ai.info summary, "Methodology in Plain
English", referral paragraph, last sentence; "Main Findings", bullet on refresh and
realignment). Readings fixed here: the dense layer is causal softmax attention; a KV head's
attention mass at position t is the mean over its query heads of the softmax probability;
the sf positions of largest mass are kept (ties: smaller position), weighted by that mass.

Pins, each independent of the oracle's code:
* the normaliser equals torch.logsumexp of fp64 causal scores, and equals the SEA oracle's lse
  when every causal predecessor is a slot with weight 1 (a different route to the same value);
* the masses equal torch's fp64 causal softmax averaged over the group, and sum to one;
* the kept positions are the first sf of a stable descending sort of the masses (brute force);
* uniform attention (q = 0) gives masses 1/(i+1) and keeps positions 0..sf-1 (every tie goes
  to the smaller position), padding rows with i + 1 < sf;
* a constructed case where the group's two heads prefer different positions.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def causal_scores(q, k, scale):
    """[B, hq, n, n] fp64 scores with -inf above the diagonal (GQA by repeat_interleave)."""
    B, n, hq, d = q.shape
    G = hq // k.shape[2]
    qq = q.double().permute(0, 2, 1, 3)
    kk = k.double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    s = scale * qq @ kk.transpose(-1, -2)
    mask = torch.ones(n, n, dtype=torch.bool).triu(1)
    return s.masked_fill(mask, float("-inf"))


def rand_qk(seed, B, n, hq, hkv, d):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(B, n, hq, d, generator=g), torch.randn(B, n, hkv, d, generator=g)


@pytest.mark.parametrize("hq,hkv", [(2, 1), (4, 2), (8, 2)])
def test_lse_is_causal_logsumexp(hq, hkv):
    q, k = rand_qk(1, 2, 37, hq, hkv, 16)
    scale = 1 / math.sqrt(16)
    want = torch.logsumexp(causal_scores(q, k, scale), dim=-1).permute(0, 2, 1).numpy()
    got = oracle.dense_lse(q, k, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_lse_equals_sea_over_all_predecessors():
    B, n, hq, hkv, d = 1, 20, 4, 2, 8
    q, k = rand_qk(2, B, n, hq, hkv, d)
    v = torch.randn(B, n, hkv, d)
    idx = np.broadcast_to(np.arange(n, dtype=np.int32)[None, None, None, :], (B, n, hkv, n)).copy()
    w = np.broadcast_to((np.arange(n)[None, :, None, None] >= np.arange(n)[None, None, None, :]),
                        (B, n, hkv, n)).astype(np.float32)
    _, lse_sea, _ = oracle.sea_forward(q, k, v, idx, w, 0.3)
    np.testing.assert_allclose(oracle.dense_lse(q, k, 0.3).reshape(lse_sea.shape), lse_sea, rtol=0,
                               atol=1e-12)


@pytest.mark.parametrize("hq,hkv", [(2, 1), (4, 2), (6, 3)])
def test_mass_is_group_mean_of_softmax(hq, hkv):
    B, n, d = 2, 29, 16
    q, k = rand_qk(3, B, n, hq, hkv, d)
    scale = 0.25
    lse = oracle.dense_lse(q, k, scale).astype(np.float32)
    # torch: softmax from the same fp32 normaliser the layer returned
    p = torch.exp(causal_scores(q, k, scale) - torch.from_numpy(lse).double().permute(0, 2, 1)[..., None])
    want = p.reshape(B, hkv, hq // hkv, n, n).mean(2).permute(0, 2, 1, 3).reshape(B * n, hkv, n)
    got = oracle.dense_mass(q, k, lse, scale)
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-12, atol=1e-15)
    # the masses of a row sum to one (up to the fp32 rounding of lse)
    np.testing.assert_allclose(got.sum(-1), 1.0, rtol=0, atol=1e-6)
    # rows list: same values for a subset, in the listed order
    rows = [5, 0, B * n - 1, 31]
    np.testing.assert_allclose(oracle.dense_mass(q, k, lse, scale, rows=rows), got[rows], rtol=0,
                               atol=0)
    np.testing.assert_allclose(oracle.dense_lse(q, k, scale, rows=rows),
                               oracle.dense_lse(q, k, scale).reshape(B * n, hq)[rows], rtol=0, atol=0)


@pytest.mark.parametrize("sf", [1, 2, 4, 8])
def test_kept_positions_are_the_heaviest_by_brute_force(sf):
    B, n, hq, hkv, d = 2, 40, 4, 2, 16
    q, k = rand_qk(10 + sf, B, n, hq, hkv, d)
    scale = 0.3
    lse = oracle.dense_lse(q, k, scale).astype(np.float32)
    mass = oracle.dense_mass(q, k, lse, scale)
    oi, ow = oracle.dense_refresh(q, k, lse, sf, scale)
    for r in range(B * n):
        i = r % n
        for h in range(hkv):
            m = torch.from_numpy(mass[r, h, : i + 1])
            order = torch.sort(-m, stable=True).indices.numpy()[:sf]  # ties: smaller t first
            want_i = np.zeros(sf, np.int32)
            want_w = np.zeros(sf, np.float32)
            want_i[: order.size] = order
            want_w[: order.size] = m.numpy()[order].astype(np.float32)
            np.testing.assert_array_equal(oi.reshape(B * n, hkv, sf)[r, h], want_i)
            np.testing.assert_array_equal(ow.reshape(B * n, hkv, sf)[r, h], want_w)


def test_uniform_attention_keeps_the_first_positions_and_pads():
    B, n, hq, hkv, d, sf = 1, 12, 4, 2, 8, 4
    q = torch.zeros(B, n, hq, d)
    k = torch.randn(B, n, hkv, d)
    lse = oracle.dense_lse(q, k, 1.0).astype(np.float32)
    np.testing.assert_allclose(lse[0, :, 0], np.log(np.arange(1, n + 1)), rtol=1e-7)
    oi, ow = oracle.dense_refresh(q, k, lse, sf, 1.0)
    for i in range(n):
        kept = min(sf, i + 1)
        np.testing.assert_array_equal(oi[0, i, :, :kept], np.broadcast_to(np.arange(kept), (hkv, kept)))
        np.testing.assert_array_equal(oi[0, i, :, kept:], 0)
        np.testing.assert_allclose(ow[0, i, :, :kept], 1.0 / (i + 1), rtol=1e-6)
        np.testing.assert_array_equal(ow[0, i, :, kept:], 0.0)


def test_group_mean_decides_between_heads():
    """One KV head, two query heads at token 3: head 0 puts mass (0.1, 0.2, 0.6, 0.1) on
    positions 0..3, head 1 puts (0.5, 0.1, 0.2, 0.2). Means: (0.3, 0.15, 0.4, 0.15): kept
    top-3 = 2, 0, then 1 (tie with 3, smaller position)."""
    n, d = 4, 4
    q = torch.zeros(1, n, 2, d, dtype=torch.float64)
    k = torch.zeros(1, n, 1, d, dtype=torch.float64)
    for t in range(n):
        k[0, t, 0, t] = 1.0  # one-hot keys: score of (hq, t) = q[hq, t]
    p0 = np.array([0.1, 0.2, 0.6, 0.1])
    p1 = np.array([0.5, 0.1, 0.2, 0.2])
    q[0, 3, 0] = torch.from_numpy(np.log(p0))
    q[0, 3, 1] = torch.from_numpy(np.log(p1))
    lse = oracle.dense_lse(q.float(), k.float(), 1.0).astype(np.float32)
    mass = oracle.dense_mass(q.float(), k.float(), lse, 1.0)
    np.testing.assert_allclose(mass[3, 0], (p0 + p1) / 2, rtol=1e-6)
    oi, ow = oracle.dense_refresh(q.float(), k.float(), lse, 3, 1.0)
    assert oi[0, 3, 0].tolist() == [2, 0, 1] or oi[0, 3, 0].tolist() == [2, 0, 3]
    # the last slot is a near-tie in fp32 inputs (0.15 vs 0.15): the mass decides exactly
    m1, m3 = mass[3, 0, 1], mass[3, 0, 3]
    assert oi[0, 3, 0, 2] == (1 if m1 >= m3 else 3)
    np.testing.assert_allclose(ow[0, 3, 0], [0.4, 0.3, 0.15], rtol=1e-6)
