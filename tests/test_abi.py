"""The C ABI without a GPU: the library builds, loads, exports every symbol include/gm.h
declares, and rejects bad arguments on the host before any CUDA call.

Only argument combinations that fail validation are passed here, so no kernel is ever
launched (and no pointer below is ever dereferenced).
"""
import ctypes
import os
import re

import pytest

from sparse_dynamic_routing_b200 import _binding as bnd
from sparse_dynamic_routing_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "gm.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return bnd.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gm_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"gm_ser_forward", "gm_sea_forward", "gm_ser_sea_forward", "gm_sea_backward",
            "gm_check_device_errors"} <= set(names)
    for name in names:
        assert hasattr(lib, name), name
        assert name in bnd.SIGNATURES, f"{name} has no binding"


def test_workspace_size(lib):
    size = lib.gm_sea_backward_workspace_size
    R, s = 8 * 4096 * 8, 4
    got = size(bnd.GM_BF16, s, 8, 4096, 16, 8, 128)
    # 8 B per target row (counts + offsets); per edge a 4 B rank and a 32 B sorted record
    # (target, source, 2G = 4 coefficients, padding)
    assert got >= 8 * R + 36 * R * s and got < 8 * R + 36 * R * s + 4096
    assert size(bnd.GM_BF16, 8, 8, 4096, 16, 8, 128) == 0  # s > 4: atomic path only
    assert size(bnd.GM_BF16, 4, 8, 4096, 16, 8, 256) == 0
    assert size(bnd.GM_F32, 2, 1, 128, 2, 1, 64) > 0
    assert size(bnd.GM_BF16, 4, 0, 4096, 16, 8, 128) == 0


def test_status_strings(lib):
    for st in range(8):
        assert bnd.status_string(st).startswith("GM_")
    assert "unknown" in bnd.status_string(99)
    assert lib.gm_version() >= 100


NULL = None
FAKE = 0x1000  # never dereferenced: every call below fails validation first


def test_ser_argument_checks(lib):
    f = lib.gm_ser_forward
    ok_empty = f(NULL, NULL, 2, NULL, NULL, 2, NULL, NULL, 2, 0, 128, 1, NULL)
    assert ok_empty == bnd.GM_OK  # B = 0: nothing to do
    assert f(NULL, NULL, 2, NULL, NULL, 2, NULL, NULL, 2, 4, 0, 1, NULL) == bnd.GM_OK  # n = 0
    assert f(NULL, NULL, 2, NULL, NULL, 2, NULL, NULL, 2, 1, 8, 1, NULL) == bnd.GM_ERR_INVALID_ARG
    bad = [
        dict(s2=8, s3=5),  # 40 candidates > 32
        dict(s1=33),
        dict(s1=0),
        dict(k=0),
        dict(B=-1),
    ]
    for b in bad:
        a = dict(s2=2, s3=2, s1=2, B=1, n=8, k=1)
        a.update(b)
        st = f(FAKE, FAKE, a["s2"], FAKE, FAKE, a["s3"], FAKE, FAKE, a["s1"], a["B"], a["n"],
               a["k"], NULL)
        assert st == bnd.GM_ERR_INVALID_ARG, b
    # null outputs
    assert f(FAKE, FAKE, 2, FAKE, FAKE, 2, NULL, FAKE, 2, 1, 8, 1, NULL) == bnd.GM_ERR_INVALID_ARG


def sea_call(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dt=bnd.GM_BF16, idx=FAKE, w=FAKE, s=4, B=1, n=8, hq=4,
             hkv=2, d=128, scale=0.1, o=FAKE + 1, lse=NULL)  # o misaligned: never launches
    a.update(kw)
    return lib.gm_sea_forward(a["q"], a["k"], a["v"], a["dt"], a["idx"], a["w"], a["s"], a["B"],
                              a["n"], a["hq"], a["hkv"], a["d"], a["scale"], a["o"], a["lse"],
                              NULL)


def test_sea_argument_checks(lib):
    assert sea_call(lib) == bnd.GM_ERR_INVALID_ARG  # misaligned o
    assert sea_call(lib, B=0) == bnd.GM_OK
    assert sea_call(lib, hq=3) == bnd.GM_ERR_INVALID_ARG
    assert sea_call(lib, s=0) == bnd.GM_ERR_INVALID_ARG
    assert sea_call(lib, s=33) == bnd.GM_ERR_INVALID_ARG
    assert sea_call(lib, scale=float("nan")) == bnd.GM_ERR_INVALID_ARG
    assert sea_call(lib, scale=float("inf")) == bnd.GM_ERR_INVALID_ARG
    assert sea_call(lib, dt=7) == bnd.GM_ERR_INVALID_ARG
    assert sea_call(lib, d=96) == bnd.GM_ERR_UNSUPPORTED
    assert sea_call(lib, dt=bnd.GM_F32, d=256) == bnd.GM_ERR_UNSUPPORTED
    assert sea_call(lib, hq=32, hkv=2) == bnd.GM_ERR_UNSUPPORTED  # group of 16
    assert sea_call(lib, q=FAKE + 8) == bnd.GM_ERR_INVALID_ARG  # misaligned q
    assert sea_call(lib, k=NULL) == bnd.GM_ERR_INVALID_ARG


def test_backward_and_fused_argument_checks(lib):
    f = lib.gm_sea_backward
    # dout misaligned in every case: a call that got past the checks under test would still
    # be rejected before its launch
    base = [FAKE, FAKE, FAKE, FAKE + 2, bnd.GM_BF16, FAKE, FAKE, 4, 1, 8, 4, 2, 128, 0.1,
            FAKE, FAKE, FAKE, FAKE, NULL, 0, 0, NULL]
    a = list(base)
    a[20] = 2  # accumulate must be 0 or 1
    assert f(*a) == bnd.GM_ERR_INVALID_ARG
    a = list(base)
    a[14] = FAKE + 4  # misaligned dq
    assert f(*a) == bnd.GM_ERR_INVALID_ARG
    a = list(base)
    a[17] = NULL  # no dlogw
    assert f(*a) == bnd.GM_ERR_INVALID_ARG
    a = list(base)
    a[3] = FAKE  # aligned dout: now a too-small workspace is what fails
    a[18], a[19] = FAKE, 16
    assert f(*a) == bnd.GM_ERR_INVALID_ARG
    g = lib.gm_ser_sea_forward
    fb = [FAKE, FAKE, 4, FAKE, FAKE, 4, FAKE, NULL, 4, FAKE, FAKE, FAKE, bnd.GM_BF16, 1, 8, 4,
          2, 128, 0.1, FAKE + 1, NULL, NULL]  # o misaligned: never launches
    assert g(*fb) == bnd.GM_ERR_INVALID_ARG  # out_idx given without out_w
    fb2 = list(fb)
    fb2[2], fb2[5] = 8, 8  # 64 candidates
    assert g(*fb2) == bnd.GM_ERR_INVALID_ARG


def test_leg_argument_checks(lib):
    f = lib.gm_leg_sparsify
    # e_idx, e_w, s0, mix1, mix2, stride, a1_idx, a1_w, s2, a2_idx, a2_w, s3, B, n, k, stream
    good = dict(s0=4, stride=64, s2=4, s3=4, B=1, n=8, k=8)
    bad_cases = [dict(s0=0), dict(s0=5), dict(k=0), dict(s2=0), dict(s3=33), dict(stride=63),
                 dict(stride=8), dict(n=-1), dict(B=-2)]
    for change in bad_cases:
        a = dict(good, **change)
        st = f(FAKE, FAKE, a["s0"], FAKE, FAKE, a["stride"], FAKE, FAKE, a["s2"], FAKE, FAKE,
               a["s3"], a["B"], a["n"], a["k"], NULL)
        assert st == bnd.GM_ERR_INVALID_ARG, change
    # null outputs / inputs
    assert f(FAKE, FAKE, 4, FAKE, NULL, 64, FAKE, FAKE, 4, FAKE, FAKE, 4, 1, 8, 8, NULL) == bnd.GM_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 4, FAKE, FAKE, 0, FAKE, FAKE, 4, NULL, FAKE, 4, 1, 8, 8, NULL) == bnd.GM_ERR_INVALID_ARG
    # an empty problem is a no-op that succeeds without touching any pointer
    assert f(NULL, NULL, 4, NULL, NULL, 64, NULL, NULL, 4, NULL, NULL, 4, 0, 8, 8, NULL) == bnd.GM_OK
    g = lib.gm_leg_backward
    # e_idx, e_w, s0, mix1, mix2, stride, g1, s2, g2, s3, B, n, k, dew, dmix1, dmix2, acc, stream
    assert g(FAKE, FAKE, 4, FAKE, FAKE, 64, FAKE, 4, FAKE, 4, 1, 8, 8, FAKE, FAKE, NULL, 0, NULL) == bnd.GM_ERR_INVALID_ARG
    assert g(FAKE, FAKE, 4, FAKE, FAKE, 64, FAKE, 4, FAKE, 4, 1, 8, 8, FAKE, FAKE, FAKE, 2, NULL) == bnd.GM_ERR_INVALID_ARG
    assert g(FAKE, FAKE, 9, FAKE, FAKE, 64, FAKE, 4, FAKE, 4, 1, 8, 8, FAKE, FAKE, FAKE, 0, NULL) == bnd.GM_ERR_INVALID_ARG
    assert g(NULL, NULL, 4, NULL, NULL, 0, NULL, 4, NULL, 4, 3, 0, 8, NULL, NULL, NULL, 0, NULL) == bnd.GM_OK


def test_refresh_argument_checks(lib):
    f = lib.gm_ser_refresh_forward
    # a1_idx, a1_w, s2, a2_idx, a2_w, s3, f_idx, f_w, sf, out_idx, out_w, s1, B, n, k, stream
    assert f(FAKE, FAKE, 4, FAKE, FAKE, 4, FAKE, FAKE, 0, FAKE, FAKE, 4, 1, 8, 2, NULL) == bnd.GM_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 4, FAKE, FAKE, 4, FAKE, FAKE, 17, FAKE, FAKE, 4, 1, 8, 2, NULL) == bnd.GM_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 4, FAKE, FAKE, 4, NULL, FAKE, 4, FAKE, FAKE, 4, 1, 8, 2, NULL) == bnd.GM_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 4, FAKE, FAKE, 4, FAKE, FAKE, 4, NULL, FAKE, 4, 1, 8, 2, NULL) == bnd.GM_ERR_INVALID_ARG
    g = lib.gm_ser_refresh_backward
    # ..., f_idx, f_w, sf, gout, s1, grad_is_log, B, n, k, dw1, dw2, dfw, accumulate, stream
    assert g(FAKE, FAKE, 2, FAKE, FAKE, 2, FAKE, FAKE, 2, FAKE, 2, 0, 1, 8, 2, FAKE, FAKE, NULL, 0, NULL) == bnd.GM_ERR_INVALID_ARG
    assert g(FAKE, FAKE, 2, FAKE, FAKE, 2, FAKE, FAKE, 2, FAKE, 2, 3, 1, 8, 2, FAKE, FAKE, FAKE, 0, NULL) == bnd.GM_ERR_INVALID_ARG
    h = lib.gm_ser_sea_refresh_forward
    base = [FAKE, FAKE, 2, FAKE, FAKE, 2, FAKE, FAKE, 2, FAKE, FAKE, 2, FAKE, FAKE, FAKE,
            bnd.GM_BF16, 1, 8, 4, 2, 128, 0.1, FAKE + 1, NULL, NULL]  # o misaligned
    assert h(*base) == bnd.GM_ERR_INVALID_ARG
    a = list(base)
    a[8] = 31  # s2*s3 + sf > 32
    a[22] = FAKE
    assert h(*a) == bnd.GM_ERR_INVALID_ARG


def test_chain_argument_checks(lib):
    legs_i = (ctypes.c_void_p * 8)(*([FAKE] * 8))
    legs_w = (ctypes.c_void_p * 8)(*([FAKE] * 8))
    f = lib.gm_ser_chain_forward
    # a1_idx, a1_w, s2, leg_idx[], leg_w[], nlegs, s3, s_mid, out_idx, out_w, s1, B, n, k, stream
    li, lw = ctypes.cast(legs_i, ctypes.c_void_p), ctypes.cast(legs_w, ctypes.c_void_p)
    assert f(FAKE, FAKE, 4, li, lw, 0, 4, 4, FAKE, FAKE, 4, 1, 8, 2, NULL) == bnd.GM_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 4, li, lw, 8, 4, 4, FAKE, FAKE, 4, 1, 8, 2, NULL) == bnd.GM_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 4, li, lw, 2, 4, 9, FAKE, FAKE, 4, 1, 8, 2, NULL) == bnd.GM_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 4, NULL, lw, 2, 4, 4, FAKE, FAKE, 4, 1, 8, 2, NULL) == bnd.GM_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 4, li, lw, 2, 4, 4, NULL, FAKE, 4, 1, 8, 2, NULL) == bnd.GM_ERR_INVALID_ARG
    legs_i[1] = None
    assert f(FAKE, FAKE, 4, li, lw, 2, 4, 4, FAKE, FAKE, 4, 1, 8, 2, NULL) == bnd.GM_ERR_INVALID_ARG
    g = lib.gm_ser_chain_backward
    # ..., s_mid, gout, s1, grad_is_log, B, n, k, dw1, dleg[], accumulate, stream
    assert g(FAKE, FAKE, 4, li, lw, 1, 4, 4, FAKE, 4, 0, 1, 8, 2, FAKE, NULL, 0, NULL) == bnd.GM_ERR_INVALID_ARG
    assert g(FAKE, FAKE, 4, li, lw, 1, 4, 4, FAKE, 4, 2, 1, 8, 2, FAKE, li, 0, NULL) == bnd.GM_ERR_INVALID_ARG


def test_binding_signatures_match_the_header():
    """Every declaration's parameter count equals the ctypes signature's (no GPU needed)."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decls = re.findall(r"\b(gm_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", src, flags=re.S)
    assert decls
    for name, params in decls:
        params = params.strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert len(bnd.SIGNATURES[name]) == n, f"{name}: header has {n} parameters"


def test_checked_build_exports_the_same_symbols(lib):
    """The checked build (input edges verified before every call) is the same ABI."""
    build.build(checked=True)
    checked = bnd.open_library(bnd.CHECKED_LIB_PATH)
    for name in declared_functions():
        assert hasattr(checked, name), name
    assert checked.gm_checked_build() == 1
    assert lib.gm_checked_build() == 0
    assert "checked" in checked.gm_status_string(bnd.GM_ERR_EDGE_INVALID).decode()
