"""Pins of the oracle's leg sparsification (forward and backward) against the mathematics.

Before the two-hop composition, each sparse layer mixes the stored edges of a token into a
pair of legs and sparsifies each leg ("Graph Machine: Towards Better Pretraining via Edges",
ai.info summary, "Methodology in Plain English", referral paragraph; the mixing is full
across the k edge channels, "Main Findings", bullet on more edges). As a matrix statement:
row i of leg L, channel h is Sparsify_s(sum_c M_L[i, h, c] * E_c[i, :]), where E_c is the
dense adjacency matrix of stored channel c. Pins here:

* closed form: with a budget >= k*s0 nothing is cut, so the dense leg row equals the mixed
  dense rows (numpy fp64), within the fp32 rounding bound;
* brute force: with dyadic weights and coefficients every product and sum is exact, so the
  kept entries are exactly the largest entries of the dense mixed row, ties by smaller index;
* special cases: identity mixing returns a sorted, duplicate-free edge set unchanged; a shared
  [k, k] matrix equals its per-token broadcast; power-of-two scaling scales the weights only;
* backward: torch.autograd (fp64) through the dense restatement with the kept set held fixed,
  and a hand-worked example.
"""
import numpy as np
import pytest
import torch

import oracle


def dense_rows(e_idx, e_w, n):
    """[B, n, k, n] fp64: D[b, i, c, t] = sum of the active weights of stored row (b, i, c) at t."""
    B, _, k, s0 = e_idx.shape
    D = np.zeros((B, n, k, n))
    for b in range(B):
        for i in range(n):
            for c in range(k):
                for a in range(s0):
                    if e_w[b, i, c, a] > 0:
                        D[b, i, c, e_idx[b, i, c, a]] += float(e_w[b, i, c, a])
    return D


def leg_dense(idx, w, n):
    """[B, n, k, n] fp64 scatter of a leg (same layout as dense_rows)."""
    return dense_rows(idx, w, n)


def random_stored(rng, B, n, k, s0, zero_frac=0.15, causal=True):
    hi = np.arange(1, n + 1)[None, :, None, None] if causal else n
    idx = rng.integers(0, np.broadcast_to(hi, (B, n, k, s0))).astype(np.int32)
    w = rng.random((B, n, k, s0)).astype(np.float32)
    w[rng.random(w.shape) < zero_frac] = 0.0
    return idx, w


@pytest.mark.parametrize("k,s0,shared", [(2, 2, False), (3, 2, False), (4, 4, False),
                                         (2, 3, True), (8, 4, False)])
def test_legs_equal_mixed_dense_rows_when_nothing_is_cut(k, s0, shared):
    rng = np.random.default_rng(100 + 10 * k + s0)
    B, n = 2, 12
    ei, ew = random_stored(rng, B, n, k, s0)
    shape = (k, k) if shared else (B, n, k, k)
    m1 = rng.random(shape).astype(np.float32)
    m2 = rng.random(shape).astype(np.float32)
    m1[rng.random(shape) < 0.2] = 0.0
    s = k * s0
    a1i, a1w, a2i, a2w, bad = oracle.leg_sparsify(ei, ew, m1, m2, s, s)
    assert bad == 0
    D = dense_rows(ei, ew, n)
    for (ai, aw, m) in ((a1i, a1w, m1), (a2i, a2w, m2)):
        mb = np.broadcast_to(m, (B, n, k, k)).astype(np.float64)
        want = np.einsum("bihc,bict->biht", mb, D)
        got = leg_dense(ai, aw, n)
        assert np.all((got > 0) == (want > 0)), "support differs from the mixed dense rows"
        # one rounding per product and at most k*s0 - 1 per sum of positive terms
        np.testing.assert_allclose(got, want, rtol=s * 2.0 ** -24 * 1.001, atol=0)
        # distinct targets per row, stored by weight descending
        assert np.all(np.diff(aw, axis=-1) <= 0)


@pytest.mark.parametrize("k,s0,s2,s3", [(2, 2, 1, 3), (4, 2, 2, 4), (8, 4, 4, 4), (3, 3, 5, 2)])
def test_kept_entries_are_the_largest_of_the_dense_row_dyadic(k, s0, s2, s3):
    rng = np.random.default_rng(200 + k * s0 + s2)
    B, n = 2, 10
    ei, _ = random_stored(rng, B, n, k, s0)
    # weights and coefficients from {0, 1/2, 1/4, 1/8}: every product and sum is exact in fp32,
    # and equal merged weights (ties) are common
    vals = np.array([0.0, 0.5, 0.25, 0.125], np.float32)
    ew = vals[rng.integers(0, 4, ei.shape)]
    m1 = vals[rng.integers(0, 4, (B, n, k, k))]
    m2 = vals[rng.integers(0, 4, (B, n, k, k))]
    a1i, a1w, a2i, a2w, bad = oracle.leg_sparsify(ei, ew, m1, m2, s2, s3)
    assert bad == 0
    D = dense_rows(ei, ew, n)
    ties = 0
    for (ai, aw, m, sl) in ((a1i, a1w, m1, s2), (a2i, a2w, m2, s3)):
        mixed = np.einsum("bihc,bict->biht", m.astype(np.float64), D)
        for b in range(B):
            for i in range(n):
                for h in range(k):
                    row = mixed[b, i, h]
                    nz = [(-row[t], t) for t in range(n) if row[t] > 0]
                    nz.sort()
                    ties += sum(1 for x, y in zip(nz, nz[1:]) if x[0] == y[0])
                    want_t = [t for _, t in nz[:sl]] + [0] * max(0, sl - len(nz))
                    want_w = [-v for v, _ in nz[:sl]] + [0.0] * max(0, sl - len(nz))
                    assert ai[b, i, h].tolist() == want_t
                    assert aw[b, i, h].tolist() == want_w
    assert ties > 0, "the draw should exercise the tie-break"


def test_identity_mixing_returns_sorted_distinct_edges_unchanged():
    rng = np.random.default_rng(3)
    B, n, k, s0 = 2, 40, 4, 3
    ei = np.zeros((B, n, k, s0), np.int32)
    ew = np.zeros((B, n, k, s0), np.float32)
    for b in range(B):
        for i in range(n):
            for c in range(k):
                ei[b, i, c] = rng.choice(n, s0, replace=False)
                ew[b, i, c] = np.sort(rng.random(s0).astype(np.float32) + 0.01)[::-1]
    eye = np.eye(k, dtype=np.float32)
    a1i, a1w, a2i, a2w, _ = oracle.leg_sparsify(ei, ew, eye, np.broadcast_to(eye, (k, k)), s0, s0 + 2)
    assert np.array_equal(a1i, ei) and np.array_equal(a1w, ew)
    assert np.array_equal(a2i[..., :s0], ei) and np.array_equal(a2w[..., :s0], ew)
    assert np.all(a2i[..., s0:] == 0) and np.all(a2w[..., s0:] == 0.0)


def test_shared_matrix_equals_its_broadcast_and_power_of_two_scaling():
    rng = np.random.default_rng(4)
    B, n, k, s0 = 2, 24, 4, 4
    ei, ew = random_stored(rng, B, n, k, s0)
    m1 = rng.random((k, k)).astype(np.float32)
    m2 = rng.random((k, k)).astype(np.float32)
    r_shared = oracle.leg_sparsify(ei, ew, m1, m2, 3, 4)
    r_tok = oracle.leg_sparsify(ei, ew, np.broadcast_to(m1, (B, n, k, k)).copy(),
                                np.broadcast_to(m2, (B, n, k, k)).copy(), 3, 4)
    for x, y in zip(r_shared, r_tok):
        assert np.array_equal(x, y)
    r_scaled = oracle.leg_sparsify(ei, ew, m1 * 4.0, m2 * 0.5, 3, 4)
    assert np.array_equal(r_scaled[0], r_shared[0]) and np.array_equal(r_scaled[2], r_shared[2])
    assert np.array_equal(r_scaled[1], r_shared[1] * 4.0)
    assert np.array_equal(r_scaled[3], r_shared[3] * 0.5)


def test_out_of_range_stored_edges_are_skipped_and_counted_once():
    B, n, k, s0 = 1, 6, 2, 2
    ei = np.zeros((B, n, k, s0), np.int32)
    ew = np.zeros((B, n, k, s0), np.float32)
    ei[0, 5, 0], ew[0, 5, 0] = [4, 9], [0.5, 0.25]     # 9 is out of range and active
    ei[0, 5, 1], ew[0, 5, 1] = [-1, 3], [0.0, 0.75]    # -1 is inactive: not counted
    m = np.ones((k, k), np.float32)
    a1i, a1w, a2i, a2w, bad = oracle.leg_sparsify(ei, ew, m, m, 3, 3)
    assert bad == 1
    assert a1i[0, 5, 0].tolist() == [3, 4, 0] and a1w[0, 5, 0].tolist() == [0.75, 0.5, 0.0]
    *_, bad_b = oracle.leg_backward(ei, ew, m, m, np.ones_like(a1w), np.ones_like(a2w))
    assert bad_b == 1


def autograd_leg_grads(ei, ew, m1, m2, legs, g1, g2):
    """d/dE.w, d/dM1, d/dM2 of sum over kept slots of g * mixed dense row at the kept target."""
    B, n, k, s0 = ei.shape
    W = torch.tensor(ew.astype(np.float64), requires_grad=True)
    M = [torch.tensor(m.astype(np.float64), requires_grad=True) for m in (m1, m2)]
    loss = torch.zeros((), dtype=torch.float64)
    for b in range(B):
        for i in range(n):
            D = torch.zeros(k, n, dtype=torch.float64)
            act = torch.from_numpy(ew[b, i] > 0)
            rows = torch.arange(k)[:, None].expand(k, s0)
            D = D.index_put((rows[act], torch.from_numpy(ei[b, i]).long()[act]), W[b, i][act],
                            accumulate=True)
            for L, (ai, aw) in enumerate(legs):
                mixed = M[L][b, i] @ D                      # [k (leg channel h), n]
                g = (g1, g2)[L]
                for h in range(k):
                    for r in range(ai.shape[3]):
                        if aw[b, i, h, r] > 0:
                            loss = loss + float(g[b, i, h, r]) * mixed[h, ai[b, i, h, r]]
    loss.backward()
    return W.grad.numpy(), M[0].grad.numpy(), M[1].grad.numpy()


@pytest.mark.parametrize("k,s0,s2,s3", [(2, 2, 2, 2), (4, 4, 4, 4), (3, 2, 1, 5), (8, 4, 4, 2)])
def test_leg_backward_matches_autograd_of_masked_dense_mix(k, s0, s2, s3):
    rng = np.random.default_rng(300 + k * s0 * s2 + s3)
    B, n = 2, 9
    ei, ew = random_stored(rng, B, n, k, s0)
    m1 = rng.random((B, n, k, k)).astype(np.float32)
    m2 = rng.random((B, n, k, k)).astype(np.float32)
    m2[rng.random(m2.shape) < 0.2] = 0.0
    a1i, a1w, a2i, a2w, _ = oracle.leg_sparsify(ei, ew, m1, m2, s2, s3)
    g1 = rng.standard_normal(a1w.shape).astype(np.float32)
    g2 = rng.standard_normal(a2w.shape).astype(np.float32)
    dew, dm1, dm2, bad = oracle.leg_backward(ei, ew, m1, m2, g1, g2)
    assert bad == 0
    want_w, want_1, want_2 = autograd_leg_grads(ei, ew, m1, m2, [(a1i, a1w), (a2i, a2w)], g1, g2)
    np.testing.assert_allclose(dew, want_w, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dm1, want_1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dm2, want_2, rtol=0, atol=1e-12)
    assert np.all(dew[ew == 0] == 0)


def test_leg_backward_hand_worked_example():
    # one token, k = 2 stored channels with s0 = 2 slots:
    #   channel 0: (t=3, .5), (t=1, .25)      channel 1: (t=3, .25), (t=2, .75)
    # leg 1 of channel h = 0 with coefficients (1, .5): candidates 3:.5, 1:.25, 3:.125, 2:.375
    #   merged: 3 -> .625, 2 -> .375, 1 -> .25; with s2 = 2 it keeps (3, .625) and (2, .375)
    # upstream g = (2, -1) on those slots:
    #   dE.w[0,0] = 2*1, dE.w[1,0] = 2*.5, dE.w[1,1] = -1*.5; dE.w[0,1] (t=1, cut) = 0
    #   dM1[0, 0] = 2*.5 = 1;  dM1[0, 1] = 2*.25 + (-1)*.75 = -.25
    ei = np.array([[[[3, 1], [3, 2]]]], np.int32).reshape(1, 1, 2, 2)
    ew = np.array([[[[.5, .25], [.25, .75]]]], np.float32).reshape(1, 1, 2, 2)
    ei = np.concatenate([np.zeros_like(ei)] * 3 + [ei], axis=1)     # token 3 (causal), n = 4
    ew = np.concatenate([np.zeros_like(ew)] * 3 + [ew], axis=1)
    m1 = np.zeros((2, 2), np.float32)
    m1[0] = [1.0, 0.5]
    m2 = np.zeros((2, 2), np.float32)
    a1i, a1w, _, _, _ = oracle.leg_sparsify(ei, ew, m1, m2, 2, 1)
    assert a1i[0, 3, 0].tolist() == [3, 2] and a1w[0, 3, 0].tolist() == [0.625, 0.375]
    assert a1w[0, 3, 1].tolist() == [0.0, 0.0]
    g1 = np.zeros((1, 4, 2, 2), np.float32)
    g1[0, 3, 0] = [2.0, -1.0]
    dew, dm1, dm2, _ = oracle.leg_backward(ei, ew, m1, m2, g1, np.zeros((1, 4, 2, 1), np.float32))
    assert dew[0, 3].tolist() == [[2.0, 0.0], [1.0, -0.5]]
    assert dm1[0, 3].tolist() == [[1.0, -0.25], [0.0, 0.0]]
    assert not dm2.any()


def test_chain_gradient_of_first_leg_coefficients_respects_softmax_shift_invariance():
    # Scaling leg 1's row (i, h) by a factor scales every candidate of referral row (i, h) and so
    # the whole referral row; attention adds ln of it to every score and is unchanged. Hence
    # sum_c M1[i,h,c] * dM1[i,h,c] = 0 for every row, while the entries themselves are not zero.
    from sparse_dynamic_routing_b200 import inputs as I
    wl = I.WORKLOADS["tiny_b1_n128_s2_f32"].with_(hq=4, hkv=2, n=48)
    x = I.make(wl, grad=True)
    le = I.leg_inputs(wl)
    a1i, a1w, a2i, a2w, _ = oracle.leg_sparsify(le["e_idx"], le["e_w"], le["mix1"], le["mix2"],
                                                wl.s2, wl.s3)
    oi, ow, _ = oracle.ser(a1i, a1w, a2i, a2w, wl.s1)
    _, _, _, dlw, _ = oracle.sea_backward(x["q"], x["k"], x["v"], x["dout"], oi, ow, wl.scale)
    d1, d2, _ = oracle.ser_backward(a1i, a1w, a2i, a2w, dlw.astype(np.float32), grad_is_log=True)
    _, dm1, dm2, _ = oracle.leg_backward(le["e_idx"], le["e_w"], le["mix1"], le["mix2"],
                                         d1.astype(np.float32), d2.astype(np.float32))
    m1 = le["mix1"].numpy().astype(np.float64)
    terms = m1 * dm1
    assert np.abs(dm1).max() > 1e-3
    # fp32 rounding of the intermediate gradients (d ln w, dw1) bounds the residue
    np.testing.assert_allclose(terms.sum(-1), 0.0, atol=1e-5 * np.abs(terms).sum(-1).max())
