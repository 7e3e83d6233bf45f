"""Pins of the oracle's SEA backward against the mathematics.

The backward is the derivative of the SEA forward (Graph Machine: Towards Better Pretraining
via Edges, ai.info summary, "Methodology in Plain English": only soft weights carry the
learning signal, indices get none). Pins here:

* torch.autograd in fp64 through an independent restatement of the forward (advanced
  indexing gather, masked softmax, batched products) - gradients w.r.t. q, K, V and ln w;
* central finite differences of the oracle's own forward, on a scalar loss <dO, o>.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def restated_forward(q, k, v, idx, logw, scale):
    """SEA forward in torch fp64 (independent of the oracle's C code).

    q [B,n,hq,d]; k/v [B,n,hkv,d]; idx [B,n,hkv,s] long; logw [B,n,hkv,s] (-inf = inactive).
    """
    B, n, hq, d = q.shape
    hkv = k.shape[2]
    G = hq // hkv
    b = torch.arange(B)[:, None, None, None]
    h = torch.arange(hkv)[None, None, :, None]
    Kg = k[b, idx, h]  # [B,n,hkv,s,d]
    Vg = v[b, idx, h]
    Kq = Kg.repeat_interleave(G, dim=2)  # [B,n,hq,s,d]
    Vq = Vg.repeat_interleave(G, dim=2)
    z = scale * torch.einsum("bnhd,bnhsd->bnhs", q, Kq) + logw.repeat_interleave(G, dim=2)
    p = torch.softmax(z, dim=-1)
    return torch.einsum("bnhs,bnhsd->bnhd", p, Vq)


def make_case(seed, B, n, hq, hkv, d, s, zero_frac=0.25):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, n, hq, d)).astype(np.float32)
    k = rng.standard_normal((B, n, hkv, d)).astype(np.float32)
    v = rng.standard_normal((B, n, hkv, d)).astype(np.float32)
    g = rng.standard_normal((B, n, hq, d)).astype(np.float32)
    idx = rng.integers(0, n, (B, n, hkv, s)).astype(np.int32)
    idx[..., -1] = idx[..., 0]  # a duplicate index in every row
    w = (rng.random((B, n, hkv, s)) + 0.02).astype(np.float32)
    w[rng.random(w.shape) < zero_frac] = 0.0
    w[..., 0] = np.maximum(w[..., 0], 0.1)  # every row keeps an active slot
    return q, k, v, g, idx, w


@pytest.mark.parametrize("B,n,hq,hkv,d,s", [(1, 9, 2, 1, 16, 3), (2, 11, 4, 2, 8, 5),
                                            (1, 7, 8, 8, 4, 1), (2, 6, 6, 2, 12, 4)])
def test_sea_backward_matches_autograd_of_restated_forward(B, n, hq, hkv, d, s):
    q, k, v, g, idx, w = make_case(B * 100 + n, B, n, hq, hkv, d, s)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv, dlw, bad = oracle.sea_backward(q, k, v, g, idx, w, scale)
    assert bad == 0

    Q = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    K = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    V = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    wt = torch.from_numpy(w).double()
    active = wt > 0
    LW = torch.where(active, torch.log(torch.where(active, wt, torch.ones_like(wt))),
                     torch.zeros_like(wt)).requires_grad_(True)
    logw = torch.where(active, LW, torch.full_like(LW, float("-inf")))
    o = restated_forward(Q, K, V, torch.from_numpy(idx).long(), logw, scale)
    (o * torch.from_numpy(g).double()).sum().backward()

    np.testing.assert_allclose(dq, Q.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, K.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, V.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dlw, LW.grad.numpy(), rtol=0, atol=1e-12)
    assert np.all(dlw[w == 0] == 0)


def test_sea_backward_matches_finite_differences_of_oracle_forward():
    B, n, hq, hkv, d, s = 1, 8, 4, 2, 6, 3
    q, k, v, g, idx, w = make_case(77, B, n, hq, hkv, d, s, zero_frac=0.2)
    scale = 0.37
    dq, dk, dv, dlw, _ = oracle.sea_backward(q, k, v, g, idx, w, scale)
    q64, k64, v64 = q.astype(np.float64), k.astype(np.float64), v.astype(np.float64)
    lw64 = np.log(np.where(w > 0, w, 1.0).astype(np.float64))

    # The oracle takes fp32 inputs: perturb, round to fp32, and divide by the step that
    # survived the rounding.
    def loss(qq, kk, vv, ww):
        o, _, _ = oracle.sea_forward(qq, kk, vv, idx, ww, scale)
        return float((o.reshape(g.shape) * g.astype(np.float64)).sum())

    rng = np.random.default_rng(0)
    h = 1e-3
    for name, arr, grad in (("q", q64, dq), ("k", k64, dk), ("v", v64, dv)):
        for _ in range(6):
            pos = tuple(rng.integers(0, m) for m in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[pos] += h
            minus[pos] -= h
            p32, m32 = plus.astype(np.float32), minus.astype(np.float32)
            step = float(p32[pos]) - float(m32[pos])
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name], args_m[name] = p32, m32
            fd = (loss(args_p["q"], args_p["k"], args_p["v"], w)
                  - loss(args_m["q"], args_m["k"], args_m["v"], w)) / step
            assert abs(fd - grad[pos]) < 2e-4 * max(1.0, abs(grad[pos])), (name, pos)
    # ln w: w * exp(+-h) on active slots
    for _ in range(6):
        pos = tuple(rng.integers(0, m) for m in w.shape)
        if w[pos] == 0:
            assert dlw[pos] == 0
            continue
        wp, wm = w.copy(), w.copy()
        wp[pos] = np.float32(math.exp(lw64[pos] + h))
        wm[pos] = np.float32(math.exp(lw64[pos] - h))
        step = math.log(float(wp[pos])) - math.log(float(wm[pos]))
        fd = (loss(q, k, v, wp) - loss(q, k, v, wm)) / step
        assert abs(fd - dlw[pos]) < 2e-4 * max(1.0, abs(dlw[pos])), pos
