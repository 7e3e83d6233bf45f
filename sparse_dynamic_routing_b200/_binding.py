"""Python binding of the C ABI in include/gm.h (ctypes).

Argument marshalling only: every step of SER, SEA and the SEA backward runs in the CUDA
library libgm_b200.so. PyTorch supplies device memory (outputs are allocated with
torch.empty when not given) and the stream (the current torch stream unless one is passed).
There is no fallback: if the library is missing, or a tensor is not on a CUDA device, the
call raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgm_b200.so")
CHECKED_LIB_PATH = os.path.join(_HERE, "libgm_b200_checked.so")  # verifies input edges

(GM_OK, GM_ERR_INVALID_ARG, GM_ERR_UNSUPPORTED, GM_ERR_CUDA, GM_ERR_INDEX_RANGE,
 GM_ERR_SCRATCH_TOO_SMALL, GM_ERR_WAIT_TIMEOUT, GM_ERR_EDGE_INVALID) = range(8)
GM_F32, GM_BF16 = 0, 1

# Entry points of include/gm.h with their ctypes signatures.
_vp, _ci, _cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
SIGNATURES = {
    "gm_leg_sparsify": [_vp, _vp, _ci, _vp, _vp, ctypes.c_int64, _vp, _vp, _ci, _vp, _vp, _ci,
                        _ci, _ci, _ci, _vp],
    "gm_leg_backward": [_vp, _vp, _ci, _vp, _vp, ctypes.c_int64, _vp, _ci, _vp, _ci, _ci, _ci,
                        _ci, _vp, _vp, _vp, _ci, _vp],
    "gm_ser_forward": [_vp, _vp, _ci, _vp, _vp, _ci, _vp, _vp, _ci, _ci, _ci, _ci, _vp],
    "gm_ser_chain_forward": [_vp, _vp, _ci, _vp, _vp, _ci, _ci, _ci, _vp, _vp, _ci, _ci, _ci, _ci, _vp],
    "gm_ser_chain_backward": [_vp, _vp, _ci, _vp, _vp, _ci, _ci, _ci, _vp, _ci, _ci, _ci, _ci, _ci, _vp,
                              _vp, _ci, _vp],
    "gm_ser_sea_chain_forward": [_vp, _vp, _ci, _vp, _vp, _ci, _ci, _ci, _vp, _vp, _ci, _vp, _vp, _vp,
                                 _ci, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _vp, _vp],
    "gm_ser_refresh_forward": [_vp, _vp, _ci, _vp, _vp, _ci, _vp, _vp, _ci, _vp, _vp, _ci, _ci, _ci,
                               _ci, _vp],
    "gm_ser_refresh_backward": [_vp, _vp, _ci, _vp, _vp, _ci, _vp, _vp, _ci, _vp, _ci, _ci, _ci, _ci,
                                _ci, _vp, _vp, _vp, _ci, _vp],
    "gm_ser_sea_refresh_forward": [_vp, _vp, _ci, _vp, _vp, _ci, _vp, _vp, _ci, _vp, _vp, _ci, _vp,
                                   _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _vp, _vp],
    "gm_ser_backward": [_vp, _vp, _ci, _vp, _vp, _ci, _vp, _ci, _ci, _ci, _ci, _ci, _vp, _vp, _ci,
                        _vp],
    "gm_sea_forward": [_vp, _vp, _vp, _ci, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _vp,
                       _vp],
    "gm_ser_sea_forward": [_vp, _vp, _ci, _vp, _vp, _ci, _vp, _vp, _ci, _vp, _vp, _vp, _ci, _ci,
                           _ci, _ci, _ci, _ci, _cf, _vp, _vp, _vp],
    "gm_sea_backward": [_vp, _vp, _vp, _vp, _ci, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _cf,
                        _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _ci, _vp],
    "gm_sea_backward_workspace_size": [_ci, _ci, _ci, _ci, _ci, _ci, _ci],
    "gm_sea_backward_noalloc": [_vp, _vp, _vp, _vp, _ci, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci,
                                _cf, _vp, _vp, _vp, _vp, _ci, _vp],
    "gm_sea_backward_noalloc_max_scratch": [],
    "gm_ser_sea_backward": [_vp, _vp, _vp, _vp, _ci, _vp, _vp, _ci, _vp, _vp, _ci, _vp, _vp, _ci, _ci,
                            _ci, _ci, _ci, _ci, _cf, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                            _ci, _vp],
    "gm_dense_refresh_edges": [_vp, _vp, _ci, _vp, _ci, _ci, _ci, _ci, _ci, _cf, _ci, _vp, _vp, _vp],
    "gm_check_device_errors": [_vp],
    "gm_status_string": [_ci],
    "gm_version": [],
    "gm_checked_build": [],
    "gm_selftest_wait_timeout": [_vp],
}


class GMError(RuntimeError):
    """A library call returned a status other than GM_OK."""

    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


class GMIndexRangeError(GMError):
    """A kernel met an active edge slot whose index was outside [0, n)."""


class GMEdgeInvalidError(GMError):
    """(Checked build) an input edge had a bad weight or a non-causal index."""


_lib = None


def open_library(path: str) -> ctypes.CDLL:
    """A library built from csrc/ (regular or checked) with the ctypes signatures set."""
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m sparse_dynamic_routing_b200.build`")
    lib = ctypes.CDLL(path)
    for name, args in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = {"gm_status_string": ctypes.c_char_p,
                      "gm_sea_backward_workspace_size": ctypes.c_size_t,
                      "gm_sea_backward_noalloc_max_scratch": ctypes.c_size_t}.get(name, ctypes.c_int)
    return lib


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library the wrappers below call (once; libgm_b200.so unless the environment
    variable GM_CHECKED=1 selects the checked build). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if path == LIB_PATH and os.environ.get("GM_CHECKED") == "1":
            path = CHECKED_LIB_PATH
        _lib = open_library(path)
    return _lib


def status_string(status: int) -> str:
    return load_library().gm_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != GM_OK:
        cls = {GM_ERR_INDEX_RANGE: GMIndexRangeError, GM_ERR_EDGE_INVALID: GMEdgeInvalidError}.get(status, GMError)
        raise cls(status, f"{what}: {status_string(status)}")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None, dtype=None, name="tensor") -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _fdtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GM_BF16
    if t.dtype == torch.float32:
        return GM_F32
    raise ValueError(f"features must be bfloat16 or float32, got {t.dtype}")


def _scale(scale, d):
    return float(1.0 / math.sqrt(d)) if scale is None else float(scale)


def _leg_shapes(e_idx, e_w, mix1, mix2):
    B, n, k, s0 = e_idx.shape
    if e_w.shape != e_idx.shape:
        raise ValueError("stored edge weights disagree with their indices")
    if mix1.shape != mix2.shape:
        raise ValueError("both legs' coefficients must have the same shape")
    if tuple(mix1.shape) == (k, k):
        stride = 0
    elif tuple(mix1.shape) == (B, n, k, k):
        stride = k * k
    else:
        raise ValueError("mixing coefficients must be [B, n, k, k] or [k, k]")
    return B, n, k, s0, stride


def gm_leg_sparsify(e_idx, e_w, mix1, mix2, s2: int, s3: int, a1_idx=None, a1_w=None,
                    a2_idx=None, a2_w=None, stream=None):
    """Both referral legs from the stored edges. Returns (a1_idx, a1_w, a2_idx, a2_w)."""
    B, n, k, s0, stride = _leg_shapes(e_idx, e_w, mix1, mix2)
    dev = e_idx.device
    i32, f32 = torch.int32, torch.float32
    a1_idx = torch.empty((B, n, k, s2), dtype=i32, device=dev) if a1_idx is None else a1_idx
    a1_w = torch.empty((B, n, k, s2), dtype=f32, device=dev) if a1_w is None else a1_w
    a2_idx = torch.empty((B, n, k, s3), dtype=i32, device=dev) if a2_idx is None else a2_idx
    a2_w = torch.empty((B, n, k, s3), dtype=f32, device=dev) if a2_w is None else a2_w
    st = load_library().gm_leg_sparsify(
        _ptr(e_idx, i32, "e_idx"), _ptr(e_w, f32, "e_w"), s0,
        _ptr(mix1, f32, "mix1"), _ptr(mix2, f32, "mix2"), stride,
        _ptr(a1_idx, i32, "a1_idx"), _ptr(a1_w, f32, "a1_w"), s2,
        _ptr(a2_idx, i32, "a2_idx"), _ptr(a2_w, f32, "a2_w"), s3, B, n, k, _stream(stream))
    _check(st, "gm_leg_sparsify")
    return a1_idx, a1_w, a2_idx, a2_w


def gm_leg_backward(e_idx, e_w, mix1, mix2, g1, g2, dew=None, dmix1=None, dmix2=None,
                    accumulate=False, stream=None):
    """Gradients of the kept leg weights. Returns (dew [B,n,k,s0], dmix1, dmix2 [B,n,k,k])."""
    B, n, k, s0, stride = _leg_shapes(e_idx, e_w, mix1, mix2)
    s2, s3 = g1.shape[3], g2.shape[3]
    if tuple(g1.shape[:3]) != (B, n, k) or tuple(g2.shape[:3]) != (B, n, k):
        raise ValueError("leg gradients must be [B, n, k, s]")
    dev = e_idx.device
    f32 = torch.float32
    dew = torch.empty((B, n, k, s0), dtype=f32, device=dev) if dew is None else dew
    dmix1 = torch.empty((B, n, k, k), dtype=f32, device=dev) if dmix1 is None else dmix1
    dmix2 = torch.empty((B, n, k, k), dtype=f32, device=dev) if dmix2 is None else dmix2
    st = load_library().gm_leg_backward(
        _ptr(e_idx, torch.int32, "e_idx"), _ptr(e_w, f32, "e_w"), s0,
        _ptr(mix1, f32, "mix1"), _ptr(mix2, f32, "mix2"), stride,
        _ptr(g1, f32, "g1"), s2, _ptr(g2, f32, "g2"), s3, B, n, k,
        _ptr(dew, f32, "dew"), _ptr(dmix1, f32, "dmix1"), _ptr(dmix2, f32, "dmix2"),
        int(bool(accumulate)), _stream(stream))
    _check(st, "gm_leg_backward")
    return dew, dmix1, dmix2


def gm_ser_forward(a1_idx, a1_w, a2_idx, a2_w, s1: int, out_idx=None, out_w=None, stream=None):
    """Sparse edge referral A' = Sparsify_s1(A1 A2). Returns (out_idx, out_w) [B,n,k,s1]."""
    B, n, k, s2 = a1_idx.shape
    s3 = a2_idx.shape[3]
    if a2_idx.shape[:3] != (B, n, k) or a1_w.shape != a1_idx.shape or a2_w.shape != a2_idx.shape:
        raise ValueError("edge tensor shapes disagree")
    dev = a1_idx.device
    if out_idx is None:
        out_idx = torch.empty((B, n, k, s1), dtype=torch.int32, device=dev)
    if out_w is None:
        out_w = torch.empty((B, n, k, s1), dtype=torch.float32, device=dev)
    lib = load_library()
    st = lib.gm_ser_forward(
        _ptr(a1_idx, torch.int32, "a1_idx"), _ptr(a1_w, torch.float32, "a1_w"), s2,
        _ptr(a2_idx, torch.int32, "a2_idx"), _ptr(a2_w, torch.float32, "a2_w"), s3,
        _ptr(out_idx, torch.int32, "out_idx"), _ptr(out_w, torch.float32, "out_w"), s1,
        B, n, k, _stream(stream))
    _check(st, "gm_ser_forward")
    return out_idx, out_w


def gm_ser_backward(a1_idx, a1_w, a2_idx, a2_w, gout, grad_is_log=False, dw1=None, dw2=None,
                    accumulate=False, stream=None):
    """Gradients of the kept referral weights w.r.t. both legs' weights. Returns (dw1, dw2)."""
    B, n, k, s2 = a1_idx.shape
    s3, s1 = a2_idx.shape[3], gout.shape[3]
    if a2_idx.shape[:3] != (B, n, k) or gout.shape[:3] != (B, n, k):
        raise ValueError("edge tensor shapes disagree")
    if a1_w.shape != a1_idx.shape or a2_w.shape != a2_idx.shape:
        raise ValueError("edge weight shapes disagree with their indices")
    dev = a1_idx.device
    f32 = torch.float32
    dw1 = torch.empty((B, n, k, s2), dtype=f32, device=dev) if dw1 is None else dw1
    dw2 = torch.empty((B, n, k, s3), dtype=f32, device=dev) if dw2 is None else dw2
    st = load_library().gm_ser_backward(
        _ptr(a1_idx, torch.int32, "a1_idx"), _ptr(a1_w, f32, "a1_w"), s2,
        _ptr(a2_idx, torch.int32, "a2_idx"), _ptr(a2_w, f32, "a2_w"), s3,
        _ptr(gout, f32, "gout"), s1, int(bool(grad_is_log)), B, n, k,
        _ptr(dw1, f32, "dw1"), _ptr(dw2, f32, "dw2"), int(bool(accumulate)), _stream(stream))
    _check(st, "gm_ser_backward")
    return dw1, dw2


def _refresh_shapes(a1_idx, a1_w, a2_idx, a2_w, f_idx, f_w):
    B, n, k, s2 = a1_idx.shape
    s3, sf = a2_idx.shape[3], f_idx.shape[3]
    if a2_idx.shape[:3] != (B, n, k) or f_idx.shape[:3] != (B, n, k):
        raise ValueError("edge tensor shapes disagree")
    if a1_w.shape != a1_idx.shape or a2_w.shape != a2_idx.shape or f_w.shape != f_idx.shape:
        raise ValueError("edge weight shapes disagree with their indices")
    return B, n, k, s2, s3, sf


def gm_ser_refresh_forward(a1_idx, a1_w, a2_idx, a2_w, f_idx, f_w, s1: int, out_idx=None,
                           out_w=None, stream=None):
    """Referral with refresh edges, A' = Sparsify_s1(A1 A2 + F). Returns (out_idx, out_w)."""
    B, n, k, s2, s3, sf = _refresh_shapes(a1_idx, a1_w, a2_idx, a2_w, f_idx, f_w)
    dev = a1_idx.device
    i32, f32 = torch.int32, torch.float32
    out_idx = torch.empty((B, n, k, s1), dtype=i32, device=dev) if out_idx is None else out_idx
    out_w = torch.empty((B, n, k, s1), dtype=f32, device=dev) if out_w is None else out_w
    st = load_library().gm_ser_refresh_forward(
        _ptr(a1_idx, i32, "a1_idx"), _ptr(a1_w, f32, "a1_w"), s2,
        _ptr(a2_idx, i32, "a2_idx"), _ptr(a2_w, f32, "a2_w"), s3,
        _ptr(f_idx, i32, "f_idx"), _ptr(f_w, f32, "f_w"), sf,
        _ptr(out_idx, i32, "out_idx"), _ptr(out_w, f32, "out_w"), s1, B, n, k, _stream(stream))
    _check(st, "gm_ser_refresh_forward")
    return out_idx, out_w


def gm_ser_refresh_backward(a1_idx, a1_w, a2_idx, a2_w, f_idx, f_w, gout, grad_is_log=False,
                            dw1=None, dw2=None, dfw=None, accumulate=False, stream=None):
    """Gradients of the kept weights of the referral with refresh edges. Returns (dw1, dw2, dfw)."""
    B, n, k, s2, s3, sf = _refresh_shapes(a1_idx, a1_w, a2_idx, a2_w, f_idx, f_w)
    s1 = gout.shape[3]
    if tuple(gout.shape[:3]) != (B, n, k):
        raise ValueError("gout must be [B, n, k, s1]")
    dev = a1_idx.device
    i32, f32 = torch.int32, torch.float32
    dw1 = torch.empty((B, n, k, s2), dtype=f32, device=dev) if dw1 is None else dw1
    dw2 = torch.empty((B, n, k, s3), dtype=f32, device=dev) if dw2 is None else dw2
    dfw = torch.empty((B, n, k, sf), dtype=f32, device=dev) if dfw is None else dfw
    st = load_library().gm_ser_refresh_backward(
        _ptr(a1_idx, i32, "a1_idx"), _ptr(a1_w, f32, "a1_w"), s2,
        _ptr(a2_idx, i32, "a2_idx"), _ptr(a2_w, f32, "a2_w"), s3,
        _ptr(f_idx, i32, "f_idx"), _ptr(f_w, f32, "f_w"), sf,
        _ptr(gout, f32, "gout"), s1, int(bool(grad_is_log)), B, n, k,
        _ptr(dw1, f32, "dw1"), _ptr(dw2, f32, "dw2"), _ptr(dfw, f32, "dfw"),
        int(bool(accumulate)), _stream(stream))
    _check(st, "gm_ser_refresh_backward")
    return dw1, dw2, dfw


def gm_ser_sea_refresh_forward(q, k, v, a1_idx, a1_w, a2_idx, a2_w, f_idx, f_w, s1: int,
                               scale=None, out_idx=None, out_w=None, o=None, lse=None,
                               want_edges=True, want_lse=True, stream=None):
    """Fused referral with refresh edges -> SEA forward. Returns (out_idx, out_w, o, lse)."""
    B, n, hq, d = q.shape
    hkv = k.shape[2]
    _, _, kk, s2, s3, sf = _refresh_shapes(a1_idx, a1_w, a2_idx, a2_w, f_idx, f_w)
    if kk != hkv or tuple(a1_idx.shape[:2]) != (B, n):
        raise ValueError("edge tensors must be [B, n, hkv, s]")
    if k.shape != (B, n, hkv, d) or v.shape != k.shape:
        raise ValueError("k/v shapes disagree with q")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share a dtype")
    dev = q.device
    i32, f32 = torch.int32, torch.float32
    if want_edges:
        out_idx = torch.empty((B, n, hkv, s1), dtype=i32, device=dev) if out_idx is None else out_idx
        out_w = torch.empty((B, n, hkv, s1), dtype=f32, device=dev) if out_w is None else out_w
    o = torch.empty_like(q) if o is None else o
    if lse is None and want_lse:
        lse = torch.empty((B, n, hq), dtype=f32, device=dev)
    st = load_library().gm_ser_sea_refresh_forward(
        _ptr(a1_idx, i32, "a1_idx"), _ptr(a1_w, f32, "a1_w"), s2,
        _ptr(a2_idx, i32, "a2_idx"), _ptr(a2_w, f32, "a2_w"), s3,
        _ptr(f_idx, i32, "f_idx"), _ptr(f_w, f32, "f_w"), sf,
        _ptr(out_idx, i32, "out_idx"), _ptr(out_w, f32, "out_w"), s1,
        _ptr(q, name="q"), _ptr(k, name="k"), _ptr(v, name="v"), _fdtype(q),
        B, n, hq, hkv, d, _scale(scale, d), _ptr(o, q.dtype, "o"), _ptr(lse, f32, "lse"),
        _stream(stream))
    _check(st, "gm_ser_sea_refresh_forward")
    return out_idx, out_w, o, lse


def _chain_legs(a1_idx, a1_w, legs):
    B, n, k, s2 = a1_idx.shape
    if a1_w.shape != a1_idx.shape or not legs:
        raise ValueError("first leg shapes disagree, or no chain legs")
    s3 = legs[0][0].shape[3]
    for li, lw in legs:
        if tuple(li.shape) != (B, n, k, s3) or lw.shape != li.shape:
            raise ValueError("every chain leg must be [B, n, k, s3]")
    pi = (ctypes.c_void_p * len(legs))(*[_ptr(li, torch.int32, "leg_idx") for li, _ in legs])
    pw = (ctypes.c_void_p * len(legs))(*[_ptr(lw, torch.float32, "leg_w") for _, lw in legs])
    return B, n, k, s2, s3, pi, pw


def gm_ser_chain_forward(a1_idx, a1_w, legs, s_mid: int, s1: int, out_idx=None, out_w=None,
                         stream=None):
    """Multi-step referral through `legs` [(idx, w), ...]. Returns (out_idx, out_w) [B,n,k,s1]."""
    B, n, k, s2, s3, pi, pw = _chain_legs(a1_idx, a1_w, legs)
    dev = a1_idx.device
    out_idx = torch.empty((B, n, k, s1), dtype=torch.int32, device=dev) if out_idx is None else out_idx
    out_w = torch.empty((B, n, k, s1), dtype=torch.float32, device=dev) if out_w is None else out_w
    st = load_library().gm_ser_chain_forward(
        _ptr(a1_idx, torch.int32, "a1_idx"), _ptr(a1_w, torch.float32, "a1_w"), s2,
        ctypes.cast(pi, ctypes.c_void_p), ctypes.cast(pw, ctypes.c_void_p), len(legs), s3, s_mid,
        _ptr(out_idx, torch.int32, "out_idx"), _ptr(out_w, torch.float32, "out_w"), s1, B, n, k,
        _stream(stream))
    _check(st, "gm_ser_chain_forward")
    return out_idx, out_w


def gm_ser_chain_backward(a1_idx, a1_w, legs, s_mid: int, gout, grad_is_log=False, dw1=None,
                          dlegs=None, accumulate=False, stream=None):
    """Gradients of the multi-step referral's kept weights. Returns (dw1, [dleg, ...])."""
    B, n, k, s2, s3, pi, pw = _chain_legs(a1_idx, a1_w, legs)
    s1 = gout.shape[3]
    dev = a1_idx.device
    f32 = torch.float32
    dw1 = torch.empty((B, n, k, s2), dtype=f32, device=dev) if dw1 is None else dw1
    if dlegs is None:
        dlegs = [torch.empty((B, n, k, s3), dtype=f32, device=dev) for _ in legs]
    pd = (ctypes.c_void_p * len(legs))(*[_ptr(d, f32, "dleg") for d in dlegs])
    st = load_library().gm_ser_chain_backward(
        _ptr(a1_idx, torch.int32, "a1_idx"), _ptr(a1_w, f32, "a1_w"), s2,
        ctypes.cast(pi, ctypes.c_void_p), ctypes.cast(pw, ctypes.c_void_p), len(legs), s3, s_mid,
        _ptr(gout, f32, "gout"), s1, int(bool(grad_is_log)), B, n, k, _ptr(dw1, f32, "dw1"),
        ctypes.cast(pd, ctypes.c_void_p), int(bool(accumulate)), _stream(stream))
    _check(st, "gm_ser_chain_backward")
    return dw1, dlegs


def gm_ser_sea_chain_forward(q, k, v, a1_idx, a1_w, legs, s_mid: int, s1: int, scale=None,
                             out_idx=None, out_w=None, o=None, lse=None, want_lse=True,
                             stream=None):
    """Multi-step referral -> SEA forward. Returns (out_idx, out_w, o, lse)."""
    B, n, hq, d = q.shape
    hkv = k.shape[2]
    _, _, kk, s2, s3, pi, pw = _chain_legs(a1_idx, a1_w, legs)
    if kk != hkv or tuple(a1_idx.shape[:2]) != (B, n):
        raise ValueError("edge tensors must be [B, n, hkv, s]")
    if k.shape != (B, n, hkv, d) or v.shape != k.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("k/v must match q")
    dev = q.device
    out_idx = torch.empty((B, n, hkv, s1), dtype=torch.int32, device=dev) if out_idx is None else out_idx
    out_w = torch.empty((B, n, hkv, s1), dtype=torch.float32, device=dev) if out_w is None else out_w
    o = torch.empty_like(q) if o is None else o
    if lse is None and want_lse:
        lse = torch.empty((B, n, hq), dtype=torch.float32, device=dev)
    st = load_library().gm_ser_sea_chain_forward(
        _ptr(a1_idx, torch.int32, "a1_idx"), _ptr(a1_w, torch.float32, "a1_w"), s2,
        ctypes.cast(pi, ctypes.c_void_p), ctypes.cast(pw, ctypes.c_void_p), len(legs), s3, s_mid,
        _ptr(out_idx, torch.int32, "out_idx"), _ptr(out_w, torch.float32, "out_w"), s1,
        _ptr(q, name="q"), _ptr(k, name="k"), _ptr(v, name="v"), _fdtype(q), B, n, hq, hkv, d,
        _scale(scale, d), _ptr(o, q.dtype, "o"), _ptr(lse, torch.float32, "lse"), _stream(stream))
    _check(st, "gm_ser_sea_chain_forward")
    return out_idx, out_w, o, lse


def gm_sea_forward(q, k, v, idx, w, scale=None, o=None, lse=None, want_lse=True, stream=None):
    """Sparse edge attention. Returns (o [B,n,hq,d] in q's dtype, lse fp32 [B,n,hq] or None)."""
    B, n, hq, d = q.shape
    hkv, s = idx.shape[2], idx.shape[3]
    if k.shape != (B, n, hkv, d) or v.shape != k.shape or w.shape != idx.shape:
        raise ValueError("tensor shapes disagree")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share a dtype")
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, n, hq), dtype=torch.float32, device=q.device)
    lib = load_library()
    st = lib.gm_sea_forward(
        _ptr(q, name="q"), _ptr(k, name="k"), _ptr(v, name="v"), _fdtype(q),
        _ptr(idx, torch.int32, "idx"), _ptr(w, torch.float32, "w"), s,
        B, n, hq, hkv, d, _scale(scale, d), _ptr(o, q.dtype, "o"),
        _ptr(lse, torch.float32, "lse"), _stream(stream))
    _check(st, "gm_sea_forward")
    return o, lse


def gm_ser_sea_forward(q, k, v, a1_idx, a1_w, a2_idx, a2_w, s1: int, scale=None,
                       out_idx=None, out_w=None, o=None, lse=None, want_edges=True,
                       want_lse=True, stream=None):
    """Fused SER -> SEA forward. Returns (out_idx, out_w, o, lse); edges/lse None if not wanted."""
    B, n, hq, d = q.shape
    hkv = k.shape[2]
    s2, s3 = a1_idx.shape[3], a2_idx.shape[3]
    if a1_idx.shape[:3] != (B, n, hkv) or a2_idx.shape[:3] != (B, n, hkv):
        raise ValueError("edge tensors must be [B, n, hkv, s]")
    if a1_w.shape != a1_idx.shape or a2_w.shape != a2_idx.shape:
        raise ValueError("edge weight shapes disagree with their indices")
    if k.shape != (B, n, hkv, d) or v.shape != k.shape:
        raise ValueError("k/v shapes disagree with q")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share a dtype")
    dev = q.device
    if want_edges:
        if out_idx is None:
            out_idx = torch.empty((B, n, hkv, s1), dtype=torch.int32, device=dev)
        if out_w is None:
            out_w = torch.empty((B, n, hkv, s1), dtype=torch.float32, device=dev)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, n, hq), dtype=torch.float32, device=dev)
    lib = load_library()
    st = lib.gm_ser_sea_forward(
        _ptr(a1_idx, torch.int32, "a1_idx"), _ptr(a1_w, torch.float32, "a1_w"), s2,
        _ptr(a2_idx, torch.int32, "a2_idx"), _ptr(a2_w, torch.float32, "a2_w"), s3,
        _ptr(out_idx, torch.int32, "out_idx"), _ptr(out_w, torch.float32, "out_w"), s1,
        _ptr(q, name="q"), _ptr(k, name="k"), _ptr(v, name="v"), _fdtype(q),
        B, n, hq, hkv, d, _scale(scale, d), _ptr(o, q.dtype, "o"),
        _ptr(lse, torch.float32, "lse"), _stream(stream))
    _check(st, "gm_ser_sea_forward")
    return out_idx, out_w, o, lse


def gm_sea_backward_workspace_size(dtype, s: int, B: int, n: int, hq: int, hkv: int,
                                   d: int) -> int:
    """Workspace bytes of the gather path of gm_sea_backward (0: not covered, pass None)."""
    dt = GM_BF16 if dtype == torch.bfloat16 else GM_F32 if dtype == torch.float32 else -1
    return int(load_library().gm_sea_backward_workspace_size(dt, s, B, n, hq, hkv, d))


def gm_sea_backward(q, k, v, dout, idx, w, scale=None, dq=None, dk=None, dv=None, dlogw=None,
                    accumulate=False, workspace="auto", stream=None):
    """SEA backward. Returns (dq, dk, dv, dlogw), all fp32.

    workspace: "auto" allocates the gather path's scratch with torch (when the shape is
    covered); None forces the atomic path; or a uint8 CUDA tensor of at least
    gm_sea_backward_workspace_size(...) bytes.
    """
    B, n, hq, d = q.shape
    hkv, s = idx.shape[2], idx.shape[3]
    if k.shape != (B, n, hkv, d) or v.shape != k.shape or w.shape != idx.shape:
        raise ValueError("tensor shapes disagree")
    if dout.shape != q.shape or dout.dtype != q.dtype:
        raise ValueError("dout must match q")
    dev = q.device
    f32 = torch.float32
    dq = torch.empty((B, n, hq, d), dtype=f32, device=dev) if dq is None else dq
    dk = torch.empty((B, n, hkv, d), dtype=f32, device=dev) if dk is None else dk
    dv = torch.empty((B, n, hkv, d), dtype=f32, device=dev) if dv is None else dv
    dlogw = torch.empty((B, n, hkv, s), dtype=f32, device=dev) if dlogw is None else dlogw
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be 'auto', None or a CUDA tensor")
        nbytes = gm_sea_backward_workspace_size(q.dtype, s, B, n, hq, hkv, d)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes else None
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (
        _ptr(workspace, name="workspace"), workspace.numel() * workspace.element_size())
    lib = load_library()
    st = lib.gm_sea_backward(
        _ptr(q, name="q"), _ptr(k, name="k"), _ptr(v, name="v"), _ptr(dout, name="dout"),
        _fdtype(q), _ptr(idx, torch.int32, "idx"), _ptr(w, f32, "w"), s,
        B, n, hq, hkv, d, _scale(scale, d), _ptr(dq, f32, "dq"), _ptr(dk, f32, "dk"),
        _ptr(dv, f32, "dv"), _ptr(dlogw, f32, "dlogw"), ws_ptr, ws_bytes,
        int(bool(accumulate)), _stream(stream))
    _check(st, "gm_sea_backward")
    return dq, dk, dv, dlogw


def gm_sea_backward_noalloc(q, k, v, dout, idx, w, scale=None, dq=None, dk=None, dv=None,
                            dlogw=None, accumulate=False, stream=None):
    """gm_sea_backward on the library's fixed device scratch (no workspace is allocated).

    For callers that may not allocate device memory where they run the backward; see
    include/gm.h. Output tensors are allocated here only when not given. Calls on one device
    share the scratch: do not let them overlap on the GPU.
    """
    B, n, hq, d = q.shape
    hkv, s = idx.shape[2], idx.shape[3]
    if k.shape != (B, n, hkv, d) or v.shape != k.shape or w.shape != idx.shape:
        raise ValueError("tensor shapes disagree")
    if dout.shape != q.shape or dout.dtype != q.dtype:
        raise ValueError("dout must match q")
    dev = q.device
    f32 = torch.float32
    dq = torch.empty((B, n, hq, d), dtype=f32, device=dev) if dq is None else dq
    dk = torch.empty((B, n, hkv, d), dtype=f32, device=dev) if dk is None else dk
    dv = torch.empty((B, n, hkv, d), dtype=f32, device=dev) if dv is None else dv
    dlogw = torch.empty((B, n, hkv, s), dtype=f32, device=dev) if dlogw is None else dlogw
    st = load_library().gm_sea_backward_noalloc(
        _ptr(q, name="q"), _ptr(k, name="k"), _ptr(v, name="v"), _ptr(dout, name="dout"),
        _fdtype(q), _ptr(idx, torch.int32, "idx"), _ptr(w, f32, "w"), s,
        B, n, hq, hkv, d, _scale(scale, d), _ptr(dq, f32, "dq"), _ptr(dk, f32, "dk"),
        _ptr(dv, f32, "dv"), _ptr(dlogw, f32, "dlogw"), int(bool(accumulate)), _stream(stream))
    _check(st, "gm_sea_backward_noalloc")
    return dq, dk, dv, dlogw


def gm_ser_sea_backward(q, k, v, dout, a1_idx, a1_w, a2_idx, a2_w, idx, w, scale=None, dq=None,
                        dk=None, dv=None, dlogw=None, dw1=None, dw2=None, accumulate=False,
                        workspace="auto", stream=None):
    """Backward of the referral and the attention in one call (A' = idx/w as the forward
    returned it). Returns (dq, dk, dv, dlogw, dw1, dw2), all fp32."""
    B, n, hq, d = q.shape
    hkv, s1 = idx.shape[2], idx.shape[3]
    s2, s3 = a1_idx.shape[3], a2_idx.shape[3]
    if tuple(a1_idx.shape[:3]) != (B, n, hkv) or tuple(a2_idx.shape[:3]) != (B, n, hkv):
        raise ValueError("legs must be [B, n, hkv, s]")
    if a1_w.shape != a1_idx.shape or a2_w.shape != a2_idx.shape or w.shape != idx.shape:
        raise ValueError("edge weight shapes disagree with their indices")
    if k.shape != (B, n, hkv, d) or v.shape != k.shape or dout.shape != q.shape or dout.dtype != q.dtype:
        raise ValueError("feature shapes disagree")
    dev = q.device
    f32 = torch.float32
    dq = torch.empty((B, n, hq, d), dtype=f32, device=dev) if dq is None else dq
    dk = torch.empty((B, n, hkv, d), dtype=f32, device=dev) if dk is None else dk
    dv = torch.empty((B, n, hkv, d), dtype=f32, device=dev) if dv is None else dv
    dlogw = torch.empty((B, n, hkv, s1), dtype=f32, device=dev) if dlogw is None else dlogw
    dw1 = torch.empty((B, n, hkv, s2), dtype=f32, device=dev) if dw1 is None else dw1
    dw2 = torch.empty((B, n, hkv, s3), dtype=f32, device=dev) if dw2 is None else dw2
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be 'auto', None or a CUDA tensor")
        nbytes = gm_sea_backward_workspace_size(q.dtype, s1, B, n, hq, hkv, d)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes else None
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (
        _ptr(workspace, name="workspace"), workspace.numel() * workspace.element_size())
    st = load_library().gm_ser_sea_backward(
        _ptr(q, name="q"), _ptr(k, name="k"), _ptr(v, name="v"), _ptr(dout, name="dout"), _fdtype(q),
        _ptr(a1_idx, torch.int32, "a1_idx"), _ptr(a1_w, f32, "a1_w"), s2,
        _ptr(a2_idx, torch.int32, "a2_idx"), _ptr(a2_w, f32, "a2_w"), s3,
        _ptr(idx, torch.int32, "idx"), _ptr(w, f32, "w"), s1, B, n, hq, hkv, d, _scale(scale, d),
        _ptr(dq, f32, "dq"), _ptr(dk, f32, "dk"), _ptr(dv, f32, "dv"), _ptr(dlogw, f32, "dlogw"),
        _ptr(dw1, f32, "dw1"), _ptr(dw2, f32, "dw2"), ws_ptr, ws_bytes, int(bool(accumulate)),
        _stream(stream))
    _check(st, "gm_ser_sea_backward")
    return dq, dk, dv, dlogw, dw1, dw2


def gm_dense_refresh_edges(q, k, lse, sf: int, scale=None, out_idx=None, out_w=None, stream=None):
    """Refresh edges from a dense attention layer: per (b, i, KV head) the sf positions t <= i of
    largest attention mass (mean over the head's query group), weighted by that mass.
    q [B, n, hq, d], k [B, n, hkv, d] bf16; lse [B, n, hq] fp32. Returns (idx, w) [B, n, hkv, sf]."""
    B, n, hq, d = q.shape
    hkv = k.shape[2]
    if tuple(k.shape) != (B, n, hkv, d) or k.dtype != q.dtype:
        raise ValueError("k must be [B, n, hkv, d] with q's dtype")
    if tuple(lse.shape) != (B, n, hq):
        raise ValueError("lse must be [B, n, hq]")
    dev = q.device
    if out_idx is None:
        out_idx = torch.empty((B, n, hkv, sf), dtype=torch.int32, device=dev)
    if out_w is None:
        out_w = torch.empty((B, n, hkv, sf), dtype=torch.float32, device=dev)
    st = load_library().gm_dense_refresh_edges(
        _ptr(q, name="q"), _ptr(k, name="k"), _fdtype(q), _ptr(lse, torch.float32, "lse"),
        B, n, hq, hkv, d, _scale(scale, d), sf, _ptr(out_idx, torch.int32, "out_idx"),
        _ptr(out_w, torch.float32, "out_w"), _stream(stream))
    _check(st, "gm_dense_refresh_edges")
    return out_idx, out_w


def gm_check_device_errors(stream=None):
    """Synchronise the stream; raise GMIndexRangeError if a kernel met a bad index, GMError if a
    kernel gave up on a bounded wait (GM_ERR_WAIT_TIMEOUT)."""
    _check(load_library().gm_check_device_errors(_stream(stream)), "gm_check_device_errors")


def gm_selftest_wait_timeout(stream=None):
    """Launch the bounded-wait diagnostic (about one second); gm_check_device_errors then
    raises GMError with status GM_ERR_WAIT_TIMEOUT."""
    _check(load_library().gm_selftest_wait_timeout(_stream(stream)), "gm_selftest_wait_timeout")


def gm_version() -> int:
    return int(load_library().gm_version())
