"""Pins of the oracle's SER backward against the mathematics.

The referral keeps the s1 heaviest entries of A1 A2 ("Graph Machine: Towards Better
Pretraining via Edges", ai.info summary, "Methodology in Plain English": hard top-s
selection, only retained weights get gradients, indices get none). So the gradient of the
kept weights is that of a masked dense product, L = sum over kept (i, t) of g[i, t] (A1 A2)[i, t]
with the kept set held fixed. Pins here: torch.autograd through that dense restatement
(index_add into dense adjacency matrices, matmul), a hand-worked example, and the
ln-weight form of the upstream gradient.
"""
import numpy as np
import pytest
import torch

import oracle


def dense_loss_grads(i1, w1, i2, w2, kept_idx, kept_w, gout):
    """d/dw1, d/dw2 of sum_kept g * (A1 A2)[i, t] by autograd (fp64, dense per (b, h))."""
    B, n, k, s2 = i1.shape
    s3, s1 = i2.shape[3], kept_idx.shape[3]
    W1 = torch.tensor(w1.astype(np.float64), requires_grad=True)
    W2 = torch.tensor(w2.astype(np.float64), requires_grad=True)
    loss = torch.zeros((), dtype=torch.float64)
    for b in range(B):
        for h in range(k):
            M1 = torch.zeros(n, n, dtype=torch.float64)
            M2 = torch.zeros(n, n, dtype=torch.float64)
            act1 = torch.from_numpy(w1[b, :, h] > 0)
            act2 = torch.from_numpy(w2[b, :, h] > 0)
            rows1 = torch.arange(n)[:, None].expand(n, s2)
            rows2 = torch.arange(n)[:, None].expand(n, s3)
            M1 = M1.index_put((rows1[act1], torch.from_numpy(i1[b, :, h]).long()[act1]),
                              W1[b, :, h][act1], accumulate=True)
            M2 = M2.index_put((rows2[act2], torch.from_numpy(i2[b, :, h]).long()[act2]),
                              W2[b, :, h][act2], accumulate=True)
            P = M1 @ M2
            for i in range(n):
                for r in range(s1):
                    if kept_w[b, i, h, r] > 0:
                        loss = loss + float(gout[b, i, h, r]) * P[i, kept_idx[b, i, h, r]]
    loss.backward()
    return W1.grad.numpy(), W2.grad.numpy()


@pytest.mark.parametrize("s2,s3,s1,causal", [(2, 2, 2, True), (4, 4, 4, True), (3, 2, 6, False),
                                             (4, 4, 2, False), (2, 5, 3, True)])
def test_ser_backward_matches_autograd_of_masked_dense_product(s2, s3, s1, causal):
    rng = np.random.default_rng(s2 * 31 + s3 * 7 + s1)
    B, n, k = 2, 14, 2
    def draw(s):
        hi = np.arange(1, n + 1)[None, :, None, None] if causal else n
        return rng.integers(0, np.broadcast_to(hi, (B, n, k, s))).astype(np.int32)

    i1, i2 = draw(s2), draw(s3)
    w1 = rng.random((B, n, k, s2)).astype(np.float32)
    w2 = rng.random((B, n, k, s3)).astype(np.float32)
    w1[rng.random(w1.shape) < 0.15] = 0.0
    w2[rng.random(w2.shape) < 0.15] = 0.0
    oi, ow, _ = oracle.ser(i1, w1, i2, w2, s1)
    g = rng.standard_normal((B, n, k, s1)).astype(np.float32)
    dw1, dw2, bad = oracle.ser_backward(i1, w1, i2, w2, g)
    assert bad == 0
    want1, want2 = dense_loss_grads(i1, w1, i2, w2, oi, ow, g)
    np.testing.assert_allclose(dw1, want1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dw2, want2, rtol=0, atol=1e-12)
    # inactive slots get nothing
    assert np.all(dw1[w1 == 0] == 0)


def test_ser_backward_hand_worked_example():
    # the forward example of the SER pins: row 3 keeps t=1 (.625 = .5*.5 + .5*.75) and
    # t=0 (.375 = .5*.5 + .5*.25); upstream gradients g1 (slot 0) and g0 (slot 1):
    #   dw1[3] = [g1*.5 + g0*.5, g1*.75 + g0*.25]     (first-leg slots j=2, j=1)
    #   dw2[2] += [g1*.5, g0*.5],  dw2[1] += [g1*.5, g0*.5]
    i1 = np.zeros((1, 4, 1, 2), np.int32)
    w1 = np.zeros((1, 4, 1, 2), np.float32)
    i2 = np.zeros((1, 4, 1, 2), np.int32)
    w2 = np.zeros((1, 4, 1, 2), np.float32)
    i1[0, 3, 0], w1[0, 3, 0] = [2, 1], [0.5, 0.5]
    i2[0, 2, 0], w2[0, 2, 0] = [1, 0], [0.5, 0.5]
    i2[0, 1, 0], w2[0, 1, 0] = [1, 0], [0.75, 0.25]
    g1, g0 = 2.0, -3.0
    g = np.zeros((1, 4, 1, 2), np.float32)
    g[0, 3, 0] = [g1, g0]
    dw1, dw2, _ = oracle.ser_backward(i1, w1, i2, w2, g)
    assert dw1[0, 3, 0].tolist() == [g1 * .5 + g0 * .5, g1 * .75 + g0 * .25]
    assert dw2[0, 2, 0].tolist() == [g1 * .5, g0 * .5]
    assert dw2[0, 1, 0].tolist() == [g1 * .5, g0 * .5]
    assert np.count_nonzero(dw1) == 2 and np.count_nonzero(dw2) == 4
    # with s1 = 1 only t=1 is kept: the paths to t=0 get no gradient
    dw1, dw2, _ = oracle.ser_backward(i1, w1, i2, w2, g[..., :1])
    assert dw1[0, 3, 0].tolist() == [g1 * .5, g1 * .75]
    assert dw2[0, 2, 0].tolist() == [g1 * .5, 0.0] and dw2[0, 1, 0].tolist() == [g1 * .5, 0.0]


def test_ser_backward_log_weight_gradient():
    # g w.r.t. ln W is g_W * W: feeding that with grad_is_log gives the same result
    rng = np.random.default_rng(9)
    B, n, k, s = 1, 30, 3, 4
    i1 = rng.integers(0, np.broadcast_to(np.arange(1, n + 1)[None, :, None, None], (B, n, k, s))).astype(np.int32)
    i2 = rng.integers(0, np.broadcast_to(np.arange(1, n + 1)[None, :, None, None], (B, n, k, s))).astype(np.int32)
    w1 = (rng.random((B, n, k, s)) + 0.05).astype(np.float32)
    w2 = (rng.random((B, n, k, s)) + 0.05).astype(np.float32)
    oi, ow, _ = oracle.ser(i1, w1, i2, w2, s)
    g = rng.standard_normal((B, n, k, s)).astype(np.float32)
    glog = (g.astype(np.float64) * ow).astype(np.float32)
    a1, a2, _ = oracle.ser_backward(i1, w1, i2, w2, g)
    b1, b2, _ = oracle.ser_backward(i1, w1, i2, w2, glog, grad_is_log=True)
    np.testing.assert_allclose(b1, a1, rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(b2, a2, rtol=1e-6, atol=1e-9)
