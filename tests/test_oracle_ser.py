"""Pins of the oracle's sparse edge referral (SER) against the mathematics.

SER (Graph Machine: Towards Better Pretraining via Edges, ai.info summary, "Key
Contributions" item 3 and "Methodology in Plain English", referral paragraph) is
A' = Sparsify_s1(A1 A2): a product of two sparse adjacency matrices followed by a top-s1
cut. Pins here:

* closed form: with s1 >= s2*s3 nothing is cut, so scattering A' into a dense n x n matrix
  gives the dense product A1 @ A2 (numpy fp64), within the fp32 rounding bound;
* brute force: with dyadic weights every product and sum is exact in fp32, so the kept
  entries are exactly the s1 largest nonzero entries of the dense row, ties by smaller index;
* a hand-worked example, special cases (s2 = s3 = 1, padding, out-of-range indices) and
  invariants on the workload generators' causal edges.
"""
import numpy as np
import pytest

import oracle
from sparse_dynamic_routing_b200 import inputs as I


def dense(idx, w, n):
    """[B, k, n, n] fp64: M[b, h, i, t] = sum of the active weights of row (b, i, h) at t."""
    B, _, k, s = idx.shape
    M = np.zeros((B, k, n, n))
    for b in range(B):
        for i in range(n):
            for h in range(k):
                for j in range(s):
                    if w[b, i, h, j] > 0:
                        M[b, h, i, idx[b, i, h, j]] += float(w[b, i, h, j])
    return M


def random_edges(rng, B, n, k, s, causal=True, zero_frac=0.2):
    hi = np.arange(1, n + 1)[None, :, None, None] if causal else n
    idx = rng.integers(0, np.broadcast_to(hi, (B, n, k, s))).astype(np.int32)
    w = rng.random((B, n, k, s)).astype(np.float32)
    w[rng.random((B, n, k, s)) < zero_frac] = 0.0
    return idx, w


@pytest.mark.parametrize("s2,s3,causal", [(2, 2, True), (3, 2, True), (4, 4, True),
                                          (2, 3, False), (5, 6, False)])
def test_ser_equals_dense_product_when_nothing_is_cut(s2, s3, causal):
    rng = np.random.default_rng(7 + s2 * 10 + s3)
    B, n, k = 2, 16, 3
    i1, w1 = random_edges(rng, B, n, k, s2, causal)
    i2, w2 = random_edges(rng, B, n, k, s3, causal)
    s1 = s2 * s3
    oi, ow, bad = oracle.ser(i1, w1, i2, w2, s1)
    assert bad == 0
    got = dense(oi, ow, n)
    want = np.einsum("bhij,bhjt->bhit", dense(i1, w1, n), dense(i2, w2, n))
    # fp32: one rounding per product, m-1 per sum of m positive terms -> rel. error <= m*2^-24
    rtol = s1 * 2.0 ** -24 * 1.001
    assert np.all((got > 0) == (want > 0)), "support differs from the dense product"
    np.testing.assert_allclose(got, want, rtol=rtol, atol=0)
    # rows with fewer distinct targets than s1 are padded with (0, 0.0) at the tail
    nnz = (ow > 0).sum(-1)
    for r in range(s1):
        tail = r >= nnz
        assert np.all(oi[..., r][tail] == 0) and np.all(ow[..., r][tail] == 0)


@pytest.mark.parametrize("s2,s3,s1", [(2, 2, 2), (4, 4, 4), (4, 4, 3), (3, 5, 1), (8, 4, 7)])
def test_ser_top_s1_matches_brute_force_on_dyadic_weights(s2, s3, s1):
    rng = np.random.default_rng(100 + s1)
    B, n, k = 2, 12, 2
    dy = np.array([0.0, 0.5, 0.25, 0.125, 0.0625], np.float32)
    i1 = rng.integers(0, n, (B, n, k, s2)).astype(np.int32)
    i2 = rng.integers(0, n, (B, n, k, s3)).astype(np.int32)
    w1 = dy[rng.integers(0, len(dy), (B, n, k, s2))]
    w2 = dy[rng.integers(0, len(dy), (B, n, k, s3))]
    oi, ow, bad = oracle.ser(i1, w1, i2, w2, s1)
    assert bad == 0
    P = np.einsum("bhij,bhjt->bhit", dense(i1, w1, n), dense(i2, w2, n))  # exact here
    ties = 0
    for b in range(B):
        for h in range(k):
            for i in range(n):
                row = P[b, h, i]
                ts = [t for t in range(n) if row[t] > 0]
                ts.sort(key=lambda t: (-row[t], t))
                ws = [row[t] for t in ts]
                ties += sum(1 for a, c in zip(ws, ws[1:]) if a == c)
                ts, ws = (ts + [0] * s1)[:s1], (ws + [0.0] * s1)[:s1]
                assert list(oi[b, i, h]) == ts
                assert list(ow[b, i, h].astype(np.float64)) == ws
    assert ties > 10, "fixture should exercise the tie-break"


def test_ser_hand_worked_example():
    # n = 4, one channel, s2 = s3 = 2, s1 = 2.
    #   A1[3] = {2: .5, 1: .5}   A1[2] = {1: .5, 0: .5}   A1[1] = {0: 1}   A1[0] = {}
    #   A2[2] = {1: .5, 0: .5}   A2[1] = {1: .75, 0: .25} A2[0] = {}
    # Row 3, candidates in order c = a*s3 + e: (1, .25) (0, .25) (1, .375) (0, .125);
    #   merged t=1: .25 + .375 = .625, t=0: .25 + .125 = .375   -> [(1, .625), (0, .375)]
    # Row 2: via j=1 (1, .375) (0, .125); j=0 has no active slot -> [(1, .375), (0, .125)]
    # Row 1: via j=0 only, which has no active slot -> padded      [(0, 0), (0, 0)]
    # Row 0: no active slot                                        [(0, 0), (0, 0)]
    i1 = np.zeros((1, 4, 1, 2), np.int32)
    w1 = np.zeros((1, 4, 1, 2), np.float32)
    i2 = np.zeros((1, 4, 1, 2), np.int32)
    w2 = np.zeros((1, 4, 1, 2), np.float32)
    i1[0, 3, 0], w1[0, 3, 0] = [2, 1], [0.5, 0.5]
    i1[0, 2, 0], w1[0, 2, 0] = [1, 0], [0.5, 0.5]
    i1[0, 1, 0], w1[0, 1, 0] = [0, 0], [1.0, 0.0]
    i2[0, 2, 0], w2[0, 2, 0] = [1, 0], [0.5, 0.5]
    i2[0, 1, 0], w2[0, 1, 0] = [1, 0], [0.75, 0.25]
    oi, ow, bad = oracle.ser(i1, w1, i2, w2, 2)
    assert bad == 0
    assert oi[0, 3, 0].tolist() == [1, 0] and ow[0, 3, 0].tolist() == [0.625, 0.375]
    assert oi[0, 2, 0].tolist() == [1, 0] and ow[0, 2, 0].tolist() == [0.375, 0.125]
    assert oi[0, 1, 0].tolist() == [0, 0] and ow[0, 1, 0].tolist() == [0.0, 0.0]
    assert oi[0, 0, 0].tolist() == [0, 0] and ow[0, 0, 0].tolist() == [0.0, 0.0]

    # A tie and a one-target row:
    #   A2[1] = {1: .5}, A2[0] = {0: .5}
    #   Row 2 = {1: .5, 0: .5}: (1, .25) via j=1, (0, .25) via j=0 -> tie, smaller index
    #   first: [(0, .25), (1, .25)]
    #   Row 1 = {0: 1}: (0, .5) via j=0 -> [(0, .5), (0, 0.0)], padded
    #   Row 3 = {2: .5, 1: .5}: via j=2 (1, .25) (0, .25); via j=1 (1, .25)
    #   -> t=1: .5, t=0: .25 -> [(1, .5), (0, .25)]
    i2[0, 1, 0], w2[0, 1, 0] = [1, 0], [0.5, 0.0]
    i2[0, 0, 0], w2[0, 0, 0] = [0, 0], [0.5, 0.0]
    oi, ow, _ = oracle.ser(i1, w1, i2, w2, 2)
    assert oi[0, 2, 0].tolist() == [0, 1] and ow[0, 2, 0].tolist() == [0.25, 0.25]
    assert oi[0, 1, 0].tolist() == [0, 0] and ow[0, 1, 0].tolist() == [0.5, 0.0]
    assert oi[0, 3, 0].tolist() == [1, 0] and ow[0, 3, 0].tolist() == [0.5, 0.25]


def test_ser_single_slot_legs_is_pointer_chasing():
    # s2 = s3 = 1: A'[i] = (A2.idx[A1.idx[i]], fl32(w1 * w2)), exactly
    rng = np.random.default_rng(3)
    B, n, k = 2, 20, 4
    i1, w1 = random_edges(rng, B, n, k, 1, zero_frac=0.0)
    i2, w2 = random_edges(rng, B, n, k, 1, zero_frac=0.0)
    oi, ow, _ = oracle.ser(i1, w1, i2, w2, 1)
    for b in range(B):
        for i in range(n):
            for h in range(k):
                j = i1[b, i, h, 0]
                assert oi[b, i, h, 0] == i2[b, j, h, 0]
                assert ow[b, i, h, 0] == np.float32(w1[b, i, h, 0] * w2[b, j, h, 0])


def test_ser_out_of_range_active_slots_are_skipped_and_counted():
    rng = np.random.default_rng(5)
    B, n, k, s = 1, 8, 1, 2
    i1, w1 = random_edges(rng, B, n, k, s, zero_frac=0.0)
    i2, w2 = random_edges(rng, B, n, k, s, zero_frac=0.0)
    ref_i, ref_w, bad = oracle.ser(i1, w1, i2, w2, 4)
    assert bad == 0
    # an inactive slot's index is never read: garbage there changes nothing
    i1b, w1b = i1.copy(), w1.copy()
    i1b[0, 5, 0, 1], w1b[0, 5, 0, 1] = -7, 0.0
    oi, ow, bad = oracle.ser(i1b, w1b, i2, w2, 4)
    assert bad == 0
    i1c, w1c = i1.copy(), w1.copy()
    w1c[0, 5, 0, 1] = 0.0
    ci, cw, _ = oracle.ser(i1c, w1c, i2, w2, 4)
    assert np.array_equal(oi, ci) and np.array_equal(ow, cw)
    # an active slot pointing outside [0, n) is skipped like a zero weight, and counted
    i1b[0, 5, 0, 1], w1b[0, 5, 0, 1] = n, 0.3
    oi, ow, bad = oracle.ser(i1b, w1b, i2, w2, 4)
    assert bad == 1
    assert np.array_equal(oi, ci) and np.array_equal(ow, cw)


@pytest.mark.parametrize("name", ["tiny_b1_n128_s2_f32", "layer_b8_n4096_s4_local"])
def test_ser_invariants_on_workload_edges(name):
    wl = I.WORKLOADS[name]
    if wl.n > 1024:
        wl = wl.with_(B=1, n=1024)
    x = I.make(wl)
    i1, w1 = x["a1_idx"].numpy(), x["a1_w"].numpy()
    i2, w2 = x["a2_idx"].numpy(), x["a2_w"].numpy()
    oi, ow, bad = oracle.ser(i1, w1, i2, w2, wl.s1)
    assert bad == 0
    pos = np.arange(wl.n)[None, :, None, None]
    assert np.all(oi <= pos) and np.all(oi >= 0), "composition keeps causality"
    assert np.all(np.diff(ow, axis=-1) <= 0), "slots ordered by weight"
    nz = ow > 0
    # nonzero targets in one row are distinct
    for row_i, row_nz in zip(oi.reshape(-1, wl.s1), nz.reshape(-1, wl.s1)):
        t = row_i[row_nz]
        assert len(set(t.tolist())) == len(t)
    # kept mass never exceeds the mass of all two-hop paths
    tot = np.einsum("bnka->bnk", w1.astype(np.float64)) * np.max(
        np.einsum("bnka->bnk", w2.astype(np.float64)))
    assert np.all(ow.astype(np.float64).sum(-1) <= tot * (1 + 1e-6))
