"""The bench's byte accounting (the roofline's numerator), checked on the host.

`distinct_rows` counts the K/V (or second-leg) rows an edge tensor really touches; the
roofline's compulsory bytes are built from it, so a miscount would inflate or deflate every
reported fraction. It is checked against a plain Python set, and the forward's compulsory
bytes against the sum of their terms written out for a tiny case.
"""
import numpy as np

import bench
from sparse_dynamic_routing_b200 import inputs as I


def test_distinct_rows_matches_a_set():
    rng = np.random.default_rng(1)
    B, n, H, s = 2, 50, 3, 4
    idx = rng.integers(0, n, (B, n, H, s)).astype(np.int32)
    w = rng.random((B, n, H, s)).astype(np.float32)
    w[rng.random(w.shape) < 0.3] = 0.0
    want = {(b, int(idx[b, i, h, j]), h) for b in range(B) for i in range(n) for h in range(H)
            for j in range(s) if w[b, i, h, j] > 0}
    assert bench.distinct_rows(idx, w, n) == len(want)


def test_compulsory_forward_bytes_written_out():
    wl = I.WORKLOADS["tiny_b1_n128_s2_f32"].with_(B=2, n=40)
    x = I.make(wl)
    rng = np.random.default_rng(2)
    ap_idx = rng.integers(0, wl.n, (wl.B, wl.n, wl.hkv, wl.s1)).astype(np.int32)
    ap_w = rng.random((wl.B, wl.n, wl.hkv, wl.s1)).astype(np.float32)
    cb = bench.compulsory_bytes(wl, x["a1_idx"].numpy(), x["a1_w"].numpy(), ap_idx, ap_w)
    tok, es = wl.B * wl.n, 4
    kv = bench.distinct_rows(ap_idx, ap_w, wl.n)
    a2 = bench.distinct_rows(x["a1_idx"].numpy(), x["a1_w"].numpy(), wl.n)
    want = (2 * tok * wl.hq * wl.d * es          # q read, o written
            + tok * wl.hq * 4                    # lse
            + tok * wl.hkv * wl.s2 * 8           # first leg
            + a2 * wl.s3 * 8                     # second-leg rows reached
            + tok * wl.hkv * wl.s1 * 8           # A' written
            + kv * wl.d * es * 2)                # K and V rows touched
    assert cb["fused_forward"] == want
    assert cb["kv_rows_touched"] == kv and cb["kv_rows_total"] == tok * wl.hkv
