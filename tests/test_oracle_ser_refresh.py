"""Pins of the oracle's referral with refresh edges, A' = Sparsify_s1(A1 A2 + F).

Refresh edges (the input edges, or the top positions of the latest dense attention layer)
join the referral's candidates ("Graph Machine: Towards Better Pretraining via Edges", ai.info
summary, "Methodology in Plain English", referral paragraph, last sentence; "Main Findings",
bullet on refresh and realignment). Pins here:

* with no refresh weight the result is the plain referral, bit for bit;
* closed form: with s1 >= s2*s3 + sf nothing is cut and the dense scatter of A' equals
  dense(A1) @ dense(A2) + dense(F) (numpy fp64) within the fp32 rounding bound;
* brute force: with dyadic weights every sum is exact, and the kept entries are the largest
  entries of the dense row of A1 A2 + F, ties by smaller index; with an empty first leg they
  are the largest entries of F's own row;
* backward: torch.autograd (fp64) through dense(A1) @ dense(A2) + dense(F) with the kept set
  held fixed, and a hand-worked example.
"""
import numpy as np
import pytest
import torch

import oracle


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


def edges(rng, B, n, k, s, zero_frac=0.2, vals=None):
    hi = np.broadcast_to(np.arange(1, n + 1)[None, :, None, None], (B, n, k, s))
    idx = rng.integers(0, hi).astype(np.int32)
    if vals is None:
        w = rng.random((B, n, k, s)).astype(np.float32)
    else:
        w = vals[rng.integers(0, len(vals), (B, n, k, s))]
    w[rng.random(w.shape) < zero_frac] = 0.0
    return idx, w


def test_no_refresh_weight_is_the_plain_referral():
    rng = np.random.default_rng(1)
    B, n, k = 2, 40, 3
    i1, w1 = edges(rng, B, n, k, 4)
    i2, w2 = edges(rng, B, n, k, 4)
    fi, fw = edges(rng, B, n, k, 3)
    want = oracle.ser(i1, w1, i2, w2, 4)
    got = oracle.ser_refresh(i1, w1, i2, w2, fi, np.zeros_like(fw), 4)
    assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])


@pytest.mark.parametrize("s2,s3,sf", [(2, 2, 2), (4, 4, 4), (3, 2, 1), (1, 1, 5)])
def test_equals_dense_product_plus_refresh_when_nothing_is_cut(s2, s3, sf):
    rng = np.random.default_rng(10 + s2 * 7 + s3 * 3 + sf)
    B, n, k = 2, 16, 2
    i1, w1 = edges(rng, B, n, k, s2)
    i2, w2 = edges(rng, B, n, k, s3)
    fi, fw = edges(rng, B, n, k, sf)
    s1 = s2 * s3 + sf
    oi, ow, bad = oracle.ser_refresh(i1, w1, i2, w2, fi, fw, s1)
    assert bad == 0
    got = dense(oi, ow, n)
    want = np.einsum("bhij,bhjt->bhit", dense(i1, w1, n), dense(i2, w2, n)) + dense(fi, fw, n)
    assert np.all((got > 0) == (want > 0)), "support differs from A1 A2 + F"
    np.testing.assert_allclose(got, want, rtol=s1 * 2.0 ** -24 * 1.001, atol=0)


@pytest.mark.parametrize("s2,s3,sf,s1", [(2, 2, 2, 2), (4, 4, 4, 4), (2, 3, 4, 3)])
def test_kept_entries_are_the_largest_of_the_dense_row_dyadic(s2, s3, sf, s1):
    rng = np.random.default_rng(20 + s1 + sf)
    B, n, k = 2, 12, 2
    vals = np.array([0.5, 0.25, 0.125], np.float32)
    i1, w1 = edges(rng, B, n, k, s2, vals=vals)
    i2, w2 = edges(rng, B, n, k, s3, vals=vals)
    fi, fw = edges(rng, B, n, k, sf, vals=vals)
    oi, ow, _ = oracle.ser_refresh(i1, w1, i2, w2, fi, fw, s1)
    full = np.einsum("bhij,bhjt->bhit", dense(i1, w1, n), dense(i2, w2, n)) + dense(fi, fw, n)
    ties = 0
    for b in range(B):
        for h in range(k):
            for i in range(n):
                row = full[b, h, i]
                nz = sorted((-row[t], t) for t in range(n) if row[t] > 0)
                ties += sum(1 for x, y in zip(nz, nz[1:]) if x[0] == y[0])
                want_t = [t for _, t in nz[:s1]] + [0] * max(0, s1 - len(nz))
                want_w = [-v for v, _ in nz[:s1]] + [0.0] * max(0, s1 - len(nz))
                assert oi[b, i, h].tolist() == want_t
                assert ow[b, i, h].tolist() == want_w
    assert ties > 0


def test_empty_first_leg_keeps_the_heaviest_refresh_edges():
    rng = np.random.default_rng(3)
    B, n, k = 1, 30, 2
    i1, w1 = edges(rng, B, n, k, 2)
    i2, w2 = edges(rng, B, n, k, 2)
    fi, fw = edges(rng, B, n, k, 5)
    oi, ow, _ = oracle.ser_refresh(i1, np.zeros_like(w1), i2, w2, fi, fw, 3)
    F = dense(fi, fw, n)
    for h in range(k):
        for i in range(n):
            nz = sorted((-F[0, h, i, t], t) for t in range(n) if F[0, h, i, t] > 0)[:3]
            assert oi[0, i, h, :len(nz)].tolist() == [t for _, t in nz]
            np.testing.assert_allclose(ow[0, i, h, :len(nz)], [-v for v, _ in nz], rtol=1e-6)


def test_hand_worked_example():
    # row 3: the path 3 -> 2 -> 1 carries .5 * .5 = .25; refresh slots (1, .5) and (2, .5):
    # t = 1 merges to .25 + .5 = .75 (path first, then refresh), t = 2 keeps .5
    z = lambda s: (np.zeros((1, 4, 1, s), np.int32), np.zeros((1, 4, 1, s), np.float32))  # noqa: E731
    (i1, w1), (i2, w2), (fi, fw) = z(1), z(1), z(2)
    i1[0, 3, 0], w1[0, 3, 0] = [2], [0.5]
    i2[0, 2, 0], w2[0, 2, 0] = [1], [0.5]
    fi[0, 3, 0], fw[0, 3, 0] = [1, 2], [0.5, 0.5]
    oi, ow, _ = oracle.ser_refresh(i1, w1, i2, w2, fi, fw, 2)
    assert oi[0, 3, 0].tolist() == [1, 2] and ow[0, 3, 0].tolist() == [0.75, 0.5]
    g = np.zeros((1, 4, 1, 2), np.float32)
    g[0, 3, 0] = [2.0, -1.0]
    dw1, dw2, dfw, _ = oracle.ser_refresh_backward(i1, w1, i2, w2, fi, fw, g)
    assert dw1[0, 3, 0].tolist() == [2.0 * 0.5]          # g_t1 * w2
    assert dw2[0, 2, 0].tolist() == [2.0 * 0.5]          # g_t1 * w1
    assert dfw[0, 3, 0].tolist() == [2.0, -1.0]          # each refresh slot gets its target's g
    # with s1 = 1 the refresh slot reaching t = 2 is cut and gets nothing
    _, _, dfw1, _ = oracle.ser_refresh_backward(i1, w1, i2, w2, fi, fw, g[..., :1])
    assert dfw1[0, 3, 0].tolist() == [2.0, 0.0]


@pytest.mark.parametrize("s2,s3,sf,s1", [(2, 2, 2, 2), (4, 4, 4, 4), (3, 2, 3, 6)])
def test_backward_matches_autograd_of_masked_dense_sum(s2, s3, sf, s1):
    rng = np.random.default_rng(40 + s2 + s3 + sf + s1)
    B, n, k = 2, 11, 2
    i1, w1 = edges(rng, B, n, k, s2, zero_frac=0.15)
    i2, w2 = edges(rng, B, n, k, s3, zero_frac=0.15)
    fi, fw = edges(rng, B, n, k, sf, zero_frac=0.15)
    oi, ow, _ = oracle.ser_refresh(i1, w1, i2, w2, fi, fw, s1)
    g = rng.standard_normal((B, n, k, s1)).astype(np.float32)
    dw1, dw2, dfw, bad = oracle.ser_refresh_backward(i1, w1, i2, w2, fi, fw, g)
    assert bad == 0
    W = [torch.tensor(x.astype(np.float64), requires_grad=True) for x in (w1, w2, fw)]
    loss = torch.zeros((), dtype=torch.float64)
    for b in range(B):
        for h in range(k):
            mats = []
            for (idx, w, Wt, s) in ((i1, w1, W[0], s2), (i2, w2, W[1], s3), (fi, fw, W[2], sf)):
                act = torch.from_numpy(w[b, :, h] > 0)
                rows = torch.arange(n)[:, None].expand(n, s)
                M = torch.zeros(n, n, dtype=torch.float64).index_put(
                    (rows[act], torch.from_numpy(idx[b, :, h]).long()[act]), Wt[b, :, h][act],
                    accumulate=True)
                mats.append(M)
            P = mats[0] @ mats[1] + mats[2]
            for i in range(n):
                for r in range(s1):
                    if ow[b, i, h, r] > 0:
                        loss = loss + float(g[b, i, h, r]) * P[i, oi[b, i, h, r]]
    loss.backward()
    for got, Wt in zip((dw1, dw2, dfw), W):
        np.testing.assert_allclose(got, Wt.grad.numpy(), rtol=0, atol=1e-12)
