"""Pins of the oracle's multi-step referral (a chain of referral steps within one layer).

"Graph Machine: Towards Better Pretraining via Edges" (ai.info summary, "Key Contributions"
item 2: the soft sparse adjacency matrix is raised to the l-th power and the result
sparsified; "Main Findings", bullet on referral: more referral steps, R3 vs R4). The chain
B_1 = A1, B_{m+1} = Sparsify(B_m A_{m+1}) cuts every intermediate to s_mid slots and the last
to s1. Pins here, each a dense restatement:

* closed form: with budgets that cut nothing, the dense scatter of the result equals the
  product of the dense legs (numpy fp64), within the fp32 rounding bound; with every leg the
  same matrix A that is dense(A)^l;
* brute force: with dyadic weights every product and sum is exact, and each step keeps the
  largest entries of the dense row of (kept previous step) @ (next leg), ties by smaller index;
* backward: torch.autograd (fp64) through the dense chain with every step's kept set held
  fixed.
"""
import numpy as np
import pytest
import torch

import oracle


def dense(idx, w, n):
    B, _, k, s = idx.shape
    M = np.zeros((B, k, n, n))
    for b in range(B):
        for i in range(n):
            for h in range(k):
                for j in range(s):
                    if w[b, i, h, j] > 0:
                        M[b, h, i, idx[b, i, h, j]] += float(w[b, i, h, j])
    return M


def edges(rng, B, n, k, s, vals=None, zero_frac=0.15):
    hi = np.broadcast_to(np.arange(1, n + 1)[None, :, None, None], (B, n, k, s))
    idx = rng.integers(0, hi).astype(np.int32)
    w = rng.random((B, n, k, s)).astype(np.float32) if vals is None else \
        vals[rng.integers(0, len(vals), (B, n, k, s))]
    w[rng.random(w.shape) < zero_frac] = 0.0
    return idx, w


def top_dense(M, s):
    """Keep the s largest entries of every row of M [B, k, n, n] (ties: smaller index)."""
    out = np.zeros_like(M)
    B, k, n, _ = M.shape
    for b in range(B):
        for h in range(k):
            for i in range(n):
                nz = sorted((-M[b, h, i, t], t) for t in range(n) if M[b, h, i, t] > 0)[:s]
                for v, t in nz:
                    out[b, h, i, t] = -v
    return out


def test_one_leg_is_the_plain_referral():
    rng = np.random.default_rng(0)
    a1 = edges(rng, 2, 30, 2, 4)
    leg = edges(rng, 2, 30, 2, 4)
    got = oracle.ser_chain(*a1, [leg], 4, 3)
    want = oracle.ser(*a1, *leg, 3)
    assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])


@pytest.mark.parametrize("s2,s3,nlegs", [(2, 2, 2), (2, 2, 3), (3, 2, 2), (1, 3, 3)])
def test_uncut_chain_is_the_dense_product(s2, s3, nlegs):
    rng = np.random.default_rng(10 + s2 * 10 + s3 + nlegs)
    B, n, k = 2, 12, 2
    a1 = edges(rng, B, n, k, s2)
    legs = [edges(rng, B, n, k, s3) for _ in range(nlegs)]
    s_mid = s2 * s3 ** (nlegs - 1)          # no intermediate is ever cut
    s1 = s_mid * s3
    oi, ow, bad = oracle.ser_chain(*a1, legs, s_mid, s1)
    assert bad == 0
    want = dense(*a1, n)
    for leg in legs:
        want = np.einsum("bhij,bhjt->bhit", want, dense(*leg, n))
    got = dense(oi, ow, n)
    assert np.all((got > 0) == (want > 0))
    # every entry is a sum of at most s1 products of nlegs + 1 factors, each step rounding
    np.testing.assert_allclose(got, want, rtol=(nlegs + 1) * s1 * 2.0 ** -24, atol=0)


def test_power_of_one_matrix():
    rng = np.random.default_rng(5)
    B, n, k, s = 1, 14, 1, 2
    A = edges(rng, B, n, k, s)
    oi, ow, _ = oracle.ser_chain(*A, [A, A], s * s, s ** 3)
    D = dense(*A, n)
    np.testing.assert_allclose(dense(oi, ow, n), D @ D @ D, rtol=3 * s ** 3 * 2.0 ** -24, atol=0)


@pytest.mark.parametrize("s2,s3,s_mid,s1,nlegs", [(2, 2, 2, 2, 2), (4, 4, 4, 4, 3), (2, 3, 3, 2, 3)])
def test_each_step_keeps_the_largest_entries_dyadic(s2, s3, s_mid, s1, nlegs):
    rng = np.random.default_rng(20 + s2 + s3 + s_mid + s1 + nlegs)
    B, n, k = 2, 11, 2
    vals = np.array([0.5, 0.25], np.float32)
    a1 = edges(rng, B, n, k, s2, vals)
    legs = [edges(rng, B, n, k, s3, vals) for _ in range(nlegs)]
    oi, ow, _ = oracle.ser_chain(*a1, legs, s_mid, s1)
    cur = dense(*a1, n)
    for m, leg in enumerate(legs):
        cur = top_dense(np.einsum("bhij,bhjt->bhit", cur, dense(*leg, n)),
                        s1 if m == nlegs - 1 else s_mid)
    assert np.array_equal(dense(oi, ow, n), cur)
    # the stored order is weight desc, then index asc
    for b in range(B):
        for i in range(n):
            for h in range(k):
                row = [(-ow[b, i, h, r], oi[b, i, h, r]) for r in range(s1) if ow[b, i, h, r] > 0]
                assert row == sorted(row)


@pytest.mark.parametrize("s2,s3,s_mid,nlegs,log", [(2, 2, 2, 2, False), (3, 2, 3, 3, True),
                                                  (4, 4, 4, 2, False)])
def test_chain_backward_matches_autograd(s2, s3, s_mid, nlegs, log):
    rng = np.random.default_rng(30 + s2 + s3 + nlegs)
    B, n, k = 2, 10, 2
    a1 = edges(rng, B, n, k, s2)
    legs = [edges(rng, B, n, k, s3) for _ in range(nlegs)]
    s1 = s_mid
    # forward with every step's kept set, for the dense restatement
    kept = []
    cur = a1
    for m, leg in enumerate(legs):
        cur = oracle.ser(*cur, *leg, s1 if m == nlegs - 1 else s_mid)[:2]
        kept.append(cur)
    g = rng.standard_normal((B, n, k, s1)).astype(np.float32)
    gin = (g.astype(np.float64) * kept[-1][1]).astype(np.float32) if log else g
    d1, dlegs, bad = oracle.ser_chain_backward(*a1, legs, s_mid, gin, grad_is_log=log)
    assert bad == 0
    W = [torch.tensor(a1[1].astype(np.float64), requires_grad=True)] + \
        [torch.tensor(leg[1].astype(np.float64), requires_grad=True) for leg in legs]
    loss = torch.zeros((), dtype=torch.float64)
    for b in range(B):
        for h in range(k):
            def dm(idx, w, Wt, s):
                act = torch.from_numpy(w[b, :, h] > 0)
                rows = torch.arange(n)[:, None].expand(n, s)
                return torch.zeros(n, n, dtype=torch.float64).index_put(
                    (rows[act], torch.from_numpy(idx[b, :, h]).long()[act]), Wt[b, :, h][act],
                    accumulate=True)
            cur = dm(a1[0], a1[1], W[0], s2)
            for m, leg in enumerate(legs):
                prod = cur @ dm(leg[0], leg[1], W[m + 1], s3)
                ki, kw = kept[m]
                mask = torch.zeros(n, n, dtype=torch.float64)
                for i in range(n):
                    for r in range(ki.shape[3]):
                        if kw[b, i, h, r] > 0:
                            mask[i, ki[b, i, h, r]] = 1.0
                cur = prod * mask              # the step's kept set, held fixed
            ki, kw = kept[-1]
            for i in range(n):
                for r in range(s1):
                    if kw[b, i, h, r] > 0:
                        loss = loss + float(g[b, i, h, r]) * cur[i, ki[b, i, h, r]]
    loss.backward()
    # intermediate gradients are rounded to fp32 between steps: a few fp32 ulps
    np.testing.assert_allclose(d1, W[0].grad.numpy(), rtol=1e-6, atol=1e-6)
    for dl, Wt in zip(dlegs, W[1:]):
        np.testing.assert_allclose(dl, Wt.grad.numpy(), rtol=1e-6, atol=1e-6)
