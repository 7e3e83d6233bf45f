"""The synthetic workloads: recipe properties and the pages' KV-access figure.

The golden file tests/golden/kv_access_fraction.txt holds the two percentages the pages
print for SEA's KV access ("Main Findings", "KV access reduction"); the workloads that stand
in for those model families must read exactly s rows per (token, KV head), which gives those
percentages against the (n+1)/2 rows of dense causal attention.
"""
import os

import numpy as np
import pytest
import torch

from sparse_dynamic_routing_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_access_fraction.txt")


def golden_rows():
    rows = []
    for line in open(GOLDEN):
        if line.strip() and not line.startswith("#"):
            fam, s, n, pct = line.split()
            rows.append((fam, int(s), int(n), float(pct)))
    return rows


def test_kv_access_fraction_matches_the_pages():
    rows = golden_rows()
    assert [r[0] for r in rows] == ["Theia", "Hyperion"]
    by_s = {2: "layer_b8_n4096_s2", 4: "layer_b8_n4096_s4_local"}
    for fam, s, n, pct in rows:
        wl = I.WORKLOADS[by_s[s]]
        assert wl.n == n and wl.s == s
        small = wl.with_(B=1)
        x = I.make(small)
        # the edges SEA reads are the referral output, s1 slots per (token, KV head)
        assert x["a1_idx"].shape[-1] == wl.s2 and wl.s1 == s
        assert round(100.0 * s / ((n + 1) / 2), 3) == pct


@pytest.mark.parametrize("name", I.WORKLOAD_ORDER)
def test_workload_recipe(name):
    wl = I.WORKLOADS[name]
    small = wl.with_(B=1, n=min(wl.n, 2048))
    x = I.make(small, grad=True)
    dt = small.torch_dtype
    assert x["q"].shape == (1, small.n, wl.hq, wl.d) and x["q"].dtype == dt
    assert x["k"].shape == (1, small.n, wl.hkv, wl.d) and x["v"].dtype == dt
    assert x["dout"].shape == x["q"].shape
    qf = x["q"].float().numpy()
    assert abs(qf.mean()) < 0.02 and abs(qf.std() - 1.0) < 0.02
    keys = [("a1_idx", "a1_w"), ("a2_idx", "a2_w")] if wl.kind == "ser_sea" else [("idx", "w")]
    pos = np.arange(small.n)[None, :, None, None]
    for ki, kw in keys:
        idx, w = x[ki].numpy(), x[kw].numpy()
        assert idx.dtype == np.int32 and w.dtype == np.float32
        assert np.all(idx >= 0) and np.all(idx <= pos), "causal: t in [0, i]"
        assert np.allclose(w.astype(np.float64).sum(-1), 1.0, atol=1e-5), "Dirichlet rows"
        assert np.all(w >= 0)
        dist = pos - idx
        if wl.local_frac > 0:
            # half the slots from the 64-token window, half uniform over [0, i]
            late = pos[0, :, 0, 0] >= 1024
            frac_local = (dist[:, late] < wl.window).mean()
            expect = wl.local_frac + (1 - wl.local_frac) * wl.window / 1536.0
            assert abs(frac_local - expect) < 0.03
        else:
            # uniform over [0, i]: mean distance i/2
            lo = small.n // 4
            rel = (dist[:, lo:] / pos[:, lo:]).mean()
            assert abs(rel - 0.5) < 4.0 / np.sqrt(dist[:, lo:].size)
    # Dirichlet(alpha): E[w] = 1/s, Var[w] = (s-1)/(s^2 (s*alpha + 1))
    w = x[keys[0][1]].numpy().astype(np.float64)
    s = w.shape[-1]
    assert abs(w.mean() - 1.0 / s) < 1e-3
    var = (s - 1) / (s * s * (s * wl.alpha + 1))
    assert abs(w.var() - var) < 0.05 * var + 1e-4


def test_streams_are_independent_and_reproducible():
    wl = I.WORKLOADS["tiny_b1_n128_s2_f32"]
    a, b = I.make(wl), I.make(wl)
    for key in a:
        assert np.array_equal(a[key].numpy(), b[key].numpy())
    assert not np.array_equal(a["a1_idx"].numpy(), a["a2_idx"].numpy())
    st = I.WORKLOADS["stack21_b16_n4096_s4"].with_(B=1, n=64)
    l0, l1 = I.layer_features(st, 0), I.layer_features(st, 1)
    assert not np.array_equal(l0["q"].float().numpy(), l1["q"].float().numpy())


def test_leg_inputs_recipe():
    wl = I.WORKLOADS["layer_b8_n4096_s4_local"].with_(B=2, n=256)
    x = I.leg_inputs(wl)
    assert x["e_idx"].shape == (2, 256, 8, 4) and x["e_w"].shape == (2, 256, 8, 4)
    assert x["mix1"].shape == (2, 256, 8, 8) and x["mix1"].dtype == torch.float32
    i = torch.arange(256)[None, :, None, None]
    assert bool((x["e_idx"] >= 0).all()) and bool((x["e_idx"] <= i).all())
    for m in (x["mix1"], x["mix2"]):
        assert bool((m >= 0).all())
        assert torch.allclose(m.double().sum(-1), torch.ones(2, 256, 8, dtype=torch.float64), atol=1e-6)
    assert not torch.equal(x["mix1"], x["mix2"])
    y = I.leg_inputs(wl)
    assert all(torch.equal(x[key], y[key]) for key in x)
