"""CPU oracle of the Graph Machine sparse layer (leg sparsification, SER, SEA, their backward
passes, and refresh edges from a dense attention layer).

TEST INFRASTRUCTURE. Only the tests, the package smoke check and the benchmark's CPU-baseline
leg import this module. It wraps the plain C library built from gm_oracle.c (compiled on
first use if missing or stale); the CUDA library shares no code with it.

Every function takes CPU tensors or numpy arrays in the library's layouts (features
[B, n, H, d] fp32 or bf16, edges [B, n, k, s] int32 + fp32) and returns numpy arrays.
Features are widened exactly to fp32 before the call; SEA and its backward compute in fp64.
The definitions, the citations and the readings of the pages are in gm_oracle.c's header.
"""
from __future__ import annotations

import ctypes
import math

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        ci = ctypes.c_int
        lib.oracle_num_threads.restype = ci
        lib.oracle_set_num_threads.restype = None
        lib.oracle_set_num_threads.argtypes = [ci]
        lib.oracle_ser.restype = ctypes.c_int64
        lib.oracle_ser.argtypes = [i32p, f32p, ci, i32p, f32p, ci, i32p, f32p, ci, ci, ci, ci]
        lib.oracle_ser_backward.restype = ctypes.c_int64
        lib.oracle_ser_backward.argtypes = [i32p, f32p, ci, i32p, f32p, ci, f32p, ci, ci, ci, ci, ci,
                                            f64p, f64p]
        lib.oracle_sea_forward.restype = ctypes.c_int64
        lib.oracle_sea_forward.argtypes = [f32p, f32p, f32p, i32p, f32p, ci, ci, ci, ci, ci, ci,
                                           ctypes.c_double, ctypes.c_void_p, ctypes.c_int64,
                                           f64p, f64p]
        lib.oracle_sea_backward.restype = ctypes.c_int64
        lib.oracle_sea_backward.argtypes = [f32p, f32p, f32p, f32p, i32p, f32p, ci, ci, ci, ci,
                                            ci, ci, ctypes.c_double, f64p, f64p, f64p, f64p]
        lib.oracle_leg_sparsify.restype = ctypes.c_int64
        lib.oracle_leg_sparsify.argtypes = [i32p, f32p, ci, ci, f32p, f32p, ctypes.c_int64,
                                            i32p, f32p, ci, i32p, f32p, ci, ci, ci]
        lib.oracle_leg_backward.restype = ctypes.c_int64
        lib.oracle_leg_backward.argtypes = [i32p, f32p, ci, ci, f32p, f32p, ctypes.c_int64,
                                            f32p, ci, f32p, ci, ci, ci, f64p, f64p, f64p]
        lib.oracle_ser_refresh.restype = ctypes.c_int64
        lib.oracle_ser_refresh.argtypes = [i32p, f32p, ci, i32p, f32p, ci, i32p, f32p, ci, i32p, f32p,
                                           ci, ci, ci, ci]
        lib.oracle_ser_refresh_backward.restype = ctypes.c_int64
        lib.oracle_ser_refresh_backward.argtypes = [i32p, f32p, ci, i32p, f32p, ci, i32p, f32p, ci,
                                                    f32p, ci, ci, ci, ci, ci, f64p, f64p, f64p]
        lib.oracle_dense_lse.restype = None
        lib.oracle_dense_lse.argtypes = [f32p, f32p, ci, ci, ci, ci, ci, ctypes.c_double,
                                         ctypes.c_void_p, ctypes.c_int64, f64p]
        lib.oracle_dense_mass.restype = None
        lib.oracle_dense_mass.argtypes = [f32p, f32p, f32p, ci, ci, ci, ci, ci, ctypes.c_double,
                                          ctypes.c_void_p, ctypes.c_int64, f64p]
        lib.oracle_dense_refresh.restype = None
        lib.oracle_dense_refresh.argtypes = [f32p, f32p, f32p, ci, ci, ci, ci, ci, ctypes.c_double,
                                             ci, ctypes.c_void_p, ctypes.c_int64, i32p, f32p]
        _lib = lib
    return _lib


def num_threads() -> int:
    """Threads the oracle's parallel loops use (OMP_NUM_THREADS or all cores)."""
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of the oracle's parallel loops from now on."""
    _load().oracle_set_num_threads(int(n))


def _np(x, dtype):
    """CPU tensor / array -> contiguous numpy array of `dtype` (bf16 widened exactly)."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if dtype == np.float32:
            x = x.float()
        x = x.numpy()
    return np.ascontiguousarray(np.asarray(x), dtype=dtype)


def ser(a1_idx, a1_w, a2_idx, a2_w, s1: int):
    """A' = Sparsify_s1(A1 A2) per (b, i, h). Returns (idx int32, w fp32, bad_refs)."""
    i1, w1 = _np(a1_idx, np.int32), _np(a1_w, np.float32)
    i2, w2 = _np(a2_idx, np.int32), _np(a2_w, np.float32)
    B, n, k, s2 = i1.shape
    s3 = i2.shape[3]
    assert i2.shape[:3] == (B, n, k) and w1.shape == i1.shape and w2.shape == i2.shape
    out_i = np.zeros((B, n, k, s1), np.int32)
    out_w = np.zeros((B, n, k, s1), np.float32)
    bad = _load().oracle_ser(i1, w1, s2, i2, w2, s3, out_i, out_w, s1, B, n, k)
    if bad < 0:
        raise ValueError("s2*s3 exceeds the oracle's candidate buffer")
    return out_i, out_w, int(bad)


def ser_backward(a1_idx, a1_w, a2_idx, a2_w, gout, grad_is_log: bool = False):
    """Gradients of the kept referral weights with respect to both legs' weights (fp64).

    gout [B, n, k, s1]: gradient w.r.t. A'.w (or w.r.t. ln A'.w when grad_is_log).
    Returns (dw1 [B,n,k,s2], dw2 [B,n,k,s3], bad_refs).
    """
    i1, w1 = _np(a1_idx, np.int32), _np(a1_w, np.float32)
    i2, w2 = _np(a2_idx, np.int32), _np(a2_w, np.float32)
    g = _np(gout, np.float32)
    B, n, k, s2 = i1.shape
    s3, s1 = i2.shape[3], g.shape[3]
    assert i2.shape[:3] == (B, n, k) and g.shape[:3] == (B, n, k)
    dw1 = np.zeros(i1.shape, np.float64)
    dw2 = np.zeros(i2.shape, np.float64)
    bad = _load().oracle_ser_backward(i1, w1, s2, i2, w2, s3, g, s1, int(bool(grad_is_log)),
                                      B, n, k, dw1, dw2)
    if bad < 0:
        raise ValueError("s2*s3 exceeds the oracle's candidate buffer")
    return dw1, dw2, int(bad)


def sea_forward(q, k, v, idx, w, scale: float | None = None, rows=None):
    """SEA forward in fp64. Returns (o [R,hq,d], lse [R,hq], bad_refs).

    R = B*n rows in order, or len(rows) for the flat positions b*n+i listed in `rows`.
    """
    qa, ka, va = _np(q, np.float32), _np(k, np.float32), _np(v, np.float32)
    ia, wa = _np(idx, np.int32), _np(w, np.float32)
    B, n, hq, d = qa.shape
    hkv, s = ia.shape[2], ia.shape[3]
    assert ka.shape == (B, n, hkv, d) and va.shape == ka.shape and wa.shape == ia.shape
    assert hq % hkv == 0
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if rows is None:
        R, rp, keep = B * n, None, None
    else:
        keep = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        R, rp = len(keep), keep.ctypes.data_as(ctypes.c_void_p)
    o = np.zeros((R, hq, d), np.float64)
    lse = np.zeros((R, hq), np.float64)
    bad = _load().oracle_sea_forward(qa, ka, va, ia, wa, s, B, n, hq, hkv, d, float(scale),
                                     rp, R, o, lse)
    return o, lse, int(bad)


def sea_backward(q, k, v, dout, idx, w, scale: float | None = None):
    """SEA backward in fp64. Returns (dq, dk, dv, dlogw, bad_refs) in the input layouts."""
    qa, ka, va = _np(q, np.float32), _np(k, np.float32), _np(v, np.float32)
    ga = _np(dout, np.float32)
    ia, wa = _np(idx, np.int32), _np(w, np.float32)
    B, n, hq, d = qa.shape
    hkv, s = ia.shape[2], ia.shape[3]
    assert ga.shape == qa.shape and ka.shape == (B, n, hkv, d) and va.shape == ka.shape
    assert hq % hkv == 0
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = np.zeros(qa.shape, np.float64)
    dk = np.zeros(ka.shape, np.float64)
    dv = np.zeros(va.shape, np.float64)
    dlw = np.zeros(ia.shape, np.float64)
    bad = _load().oracle_sea_backward(qa, ka, va, ga, ia, wa, s, B, n, hq, hkv, d,
                                      float(scale), dq, dk, dv, dlw)
    return dq, dk, dv, dlw, int(bad)


def ser_sea_forward(q, k, v, a1_idx, a1_w, a2_idx, a2_w, s1: int, scale=None, rows=None):
    """SER followed by SEA on its output. Returns (idx, w, o, lse, bad_refs)."""
    oi, ow, bad1 = ser(a1_idx, a1_w, a2_idx, a2_w, s1)
    o, lse, bad2 = sea_forward(q, k, v, oi, ow, scale, rows)
    return oi, ow, o, lse, bad1 + bad2


def _mix(m, B, n, k):
    """Mixing coefficients [B, n, k, k] (per token) or [k, k] (shared) -> (array, token stride)."""
    m = _np(m, np.float32)
    if m.shape == (k, k):
        return m, 0
    assert m.shape == (B, n, k, k), m.shape
    return m, k * k


def leg_sparsify(e_idx, e_w, mix1, mix2, s2: int, s3: int):
    """The pair of legs of every (b, i, h) from the stored edges E [B, n, k, s0].

    Leg 1 = Sparsify_s2 of the stored edges of the same token mixed by mix1[.., h, :], leg 2
    the same with mix2 and s3. Returns (a1_idx, a1_w, a2_idx, a2_w, bad_refs).
    """
    ei, ew = _np(e_idx, np.int32), _np(e_w, np.float32)
    B, n, k, s0 = ei.shape
    assert ew.shape == ei.shape
    m1, st1 = _mix(mix1, B, n, k)
    m2, st2 = _mix(mix2, B, n, k)
    assert st1 == st2, "both legs' coefficients must be per token, or both shared"
    a1i = np.zeros((B, n, k, s2), np.int32)
    a1w = np.zeros((B, n, k, s2), np.float32)
    a2i = np.zeros((B, n, k, s3), np.int32)
    a2w = np.zeros((B, n, k, s3), np.float32)
    bad = _load().oracle_leg_sparsify(ei, ew, s0, k, m1, m2, st1, a1i, a1w, s2, a2i, a2w, s3,
                                      B, n)
    if bad < 0:
        raise ValueError("k*s0 exceeds the oracle's candidate buffer")
    return a1i, a1w, a2i, a2w, int(bad)


def leg_backward(e_idx, e_w, mix1, mix2, g1, g2):
    """Gradients of the kept leg weights w.r.t. the stored weights and both mixes (fp64).

    g1 [B, n, k, s2], g2 [B, n, k, s3]. Returns (dew [B,n,k,s0], dmix1 [B,n,k,k],
    dmix2 [B,n,k,k], bad_refs); the mixes' gradients are per token even when shared.
    """
    ei, ew = _np(e_idx, np.int32), _np(e_w, np.float32)
    B, n, k, s0 = ei.shape
    m1, st1 = _mix(mix1, B, n, k)
    m2, st2 = _mix(mix2, B, n, k)
    assert st1 == st2
    ga, gb = _np(g1, np.float32), _np(g2, np.float32)
    s2, s3 = ga.shape[3], gb.shape[3]
    assert ga.shape[:3] == (B, n, k) and gb.shape[:3] == (B, n, k)
    dew = np.zeros(ei.shape, np.float64)
    dm1 = np.zeros((B, n, k, k), np.float64)
    dm2 = np.zeros((B, n, k, k), np.float64)
    bad = _load().oracle_leg_backward(ei, ew, s0, k, m1, m2, st1, ga, s2, gb, s3, B, n,
                                      dew, dm1, dm2)
    if bad < 0:
        raise ValueError("k*s0 exceeds the oracle's candidate buffer")
    return dew, dm1, dm2, int(bad)


def ser_refresh(a1_idx, a1_w, a2_idx, a2_w, f_idx, f_w, s1: int):
    """A' = Sparsify_s1(A1 A2 + F) per (b, i, h): the referral with refresh edges F [B,n,k,sf]
    joining its candidates after the two-hop paths. Returns (idx int32, w fp32, bad_refs)."""
    i1, w1 = _np(a1_idx, np.int32), _np(a1_w, np.float32)
    i2, w2 = _np(a2_idx, np.int32), _np(a2_w, np.float32)
    fi, fw = _np(f_idx, np.int32), _np(f_w, np.float32)
    B, n, k, s2 = i1.shape
    s3, sf = i2.shape[3], fi.shape[3]
    assert i2.shape[:3] == (B, n, k) and fi.shape[:3] == (B, n, k) and fw.shape == fi.shape
    out_i = np.zeros((B, n, k, s1), np.int32)
    out_w = np.zeros((B, n, k, s1), np.float32)
    bad = _load().oracle_ser_refresh(i1, w1, s2, i2, w2, s3, fi, fw, sf, out_i, out_w, s1, B, n, k)
    if bad < 0:
        raise ValueError("s2*s3 + sf exceeds the oracle's candidate buffer")
    return out_i, out_w, int(bad)


def ser_refresh_backward(a1_idx, a1_w, a2_idx, a2_w, f_idx, f_w, gout, grad_is_log: bool = False):
    """Gradients of the kept weights of ser_refresh w.r.t. both legs and the refresh weights.

    Returns (dw1 [B,n,k,s2], dw2 [B,n,k,s3], dfw [B,n,k,sf], bad_refs), fp64.
    """
    i1, w1 = _np(a1_idx, np.int32), _np(a1_w, np.float32)
    i2, w2 = _np(a2_idx, np.int32), _np(a2_w, np.float32)
    fi, fw = _np(f_idx, np.int32), _np(f_w, np.float32)
    g = _np(gout, np.float32)
    B, n, k, s2 = i1.shape
    s3, sf, s1 = i2.shape[3], fi.shape[3], g.shape[3]
    dw1 = np.zeros(i1.shape, np.float64)
    dw2 = np.zeros(i2.shape, np.float64)
    dfw = np.zeros(fi.shape, np.float64)
    bad = _load().oracle_ser_refresh_backward(i1, w1, s2, i2, w2, s3, fi, fw, sf, g, s1,
                                              int(bool(grad_is_log)), B, n, k, dw1, dw2, dfw)
    if bad < 0:
        raise ValueError("s2*s3 + sf exceeds the oracle's candidate buffer")
    return dw1, dw2, dfw, int(bad)


def ser_chain(a1_idx, a1_w, legs, s_mid: int, s1: int):
    """Multi-step referral: B_1 = A1, B_{m+1} = Sparsify(B_m A_{m+1}) for the legs A_2..A_l in
    `legs` (a list of (idx, w) [B, n, k, s3]); every intermediate is cut to s_mid slots, the
    last to s1. Each step is oracle_ser. Returns (idx, w, bad_refs)."""
    cur_i, cur_w, bad = a1_idx, a1_w, 0
    for m, (li, lw) in enumerate(legs):
        s_out = s1 if m == len(legs) - 1 else s_mid
        cur_i, cur_w, b = ser(cur_i, cur_w, li, lw, s_out)
        bad += b
    return cur_i, cur_w, bad


def ser_chain_backward(a1_idx, a1_w, legs, s_mid: int, gout, grad_is_log: bool = False):
    """Gradients of ser_chain's kept weights w.r.t. A1's weights and every leg's weights.

    The forward is recomputed step by step; the gradient then runs back through the steps,
    each one oracle_ser_backward (the gradient w.r.t. a step's first leg is the upstream
    gradient of the previous step's kept weights, rounded to fp32 between steps). Returns
    (dw1 [B,n,k,s2], [dleg_2, ..., dleg_l], bad_refs), fp64.
    """
    firsts = [(_np(a1_idx, np.int32), _np(a1_w, np.float32))]
    for li, lw in legs[:-1]:
        oi, ow, _ = ser(firsts[-1][0], firsts[-1][1], li, lw, s_mid)
        firsts.append((oi, ow))
    g = _np(gout, np.float32)
    dlegs = [None] * len(legs)
    d_first, bad = None, 0
    for m in range(len(legs) - 1, -1, -1):
        d_first, d_leg, b = ser_backward(firsts[m][0], firsts[m][1], legs[m][0], legs[m][1], g,
                                         grad_is_log and m == len(legs) - 1)
        bad += b
        dlegs[m] = d_leg
        g = d_first.astype(np.float32)
    return d_first, dlegs, bad


def _rows(rows):
    if rows is None:
        return None, None, 0
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, r.ctypes.data_as(ctypes.c_void_p), int(r.size)


def dense_lse(q, k, scale: float | None = None, rows=None):
    """Normaliser of causal softmax attention per (b, i, hq), fp64 [B, n, hq] (or [nrows, hq]
    for a list of flat rows b*n + i): the lse a dense attention layer's forward returns."""
    qf, kf = _np(q, np.float32), _np(k, np.float32)
    B, n, hq, d = qf.shape
    hkv = kf.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    r, rp, nr = _rows(rows)
    out = np.zeros((B, n, hq) if r is None else (nr, hq), np.float64)
    _load().oracle_dense_lse(qf, kf, B, n, hq, hkv, d, scale, rp, nr, out)
    return out


def dense_mass(q, k, lse, scale: float | None = None, rows=None):
    """Attention mass of each KV head at every position, the mean over its query heads of the
    causal softmax probabilities, fp64 [nrows, hkv, n] (zero for t > i). rows: flat b*n + i."""
    qf, kf, lf = _np(q, np.float32), _np(k, np.float32), _np(lse, np.float32)
    B, n, hq, d = qf.shape
    hkv = kf.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    r, rp, nr = _rows(rows)
    nrows = B * n if r is None else nr
    out = np.zeros((nrows, hkv, n), np.float64)
    _load().oracle_dense_mass(qf, kf, lf, B, n, hq, hkv, d, scale, rp, nr, out)
    return out


def dense_refresh(q, k, lse, sf: int, scale: float | None = None, rows=None):
    """Refresh edges from a dense attention layer: per (b, i, h) the sf positions t <= i with
    the largest attention mass of KV head h (ties: smaller t), weights = that mass in fp32,
    padded with (0, 0.0). lse is the dense layer's fp32 normaliser [B, n, hq]. Returns
    (idx int32, w fp32), [B, n, hkv, sf], or [nrows, hkv, sf] for a list of flat rows."""
    qf, kf, lf = _np(q, np.float32), _np(k, np.float32), _np(lse, np.float32)
    B, n, hq, d = qf.shape
    hkv = kf.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    r, rp, nr = _rows(rows)
    shape = (B, n, hkv, sf) if r is None else (nr, hkv, sf)
    oi = np.zeros(shape, np.int32)
    ow = np.zeros(shape, np.float32)
    _load().oracle_dense_refresh(qf, kf, lf, B, n, hq, hkv, d, scale, sf, rp, nr, oi, ow)
    return oi, ow
