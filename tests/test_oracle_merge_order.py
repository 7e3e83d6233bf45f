"""Pins of the fp32 merge order of the oracle's sparsify step.

Duplicate targets are summed in fp32, each add rounded to nearest, in ascending candidate
order, starting from the first occurrence. The pages leave the order open; this reading fixes
it (SER: candidate c = a*s3 + e; referral with refresh edges: the s2*s3 paths, then the
refresh slots in ascending f; leg sparsification: stored channel, then slot, c*s0 + a).
Sources: "Graph Machine: Towards Better Pretraining via Edges", ai.info summary, "Key
Contributions" item 3 (A' = Sparsify_s1(A1 A2)), "Methodology in Plain English", referral
paragraph (legs, refresh edges), "Main Findings", bullet on refresh and realignment.

The weights (tests/merge_order_cases.py) are plain three-decimal fp32 values, not dyadic, chosen so that four
candidates with one shared target give a different fp32 sum in ascending order than in any
other plausible order: reversed, transposed enumeration, pairwise tree, one fp64 sum rounded
once, or sorted by weight. Each case first checks that it is order-sensitive in this way, then
that the oracle returns the ascending-order sum written out with explicit np.float32 adds.
The last tests compile a copy of the oracle with the merge loops reversed and check that
these pins reject it.
"""
import ctypes
import re
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from merge_order_cases import asc, f32, leg_case, refresh_case, ser_case
from oracle import build as obuild


def tree(vals):
    v = [f32(x) for x in vals]
    while len(v) > 1:
        v = [f32(v[i] + v[i + 1]) if i + 1 < len(v) else v[i] for i in range(0, len(v), 2)]
    return v[0]


def alternatives(u, transposed):
    return {
        "reversed": asc(u[::-1]), "transposed": asc(transposed), "tree": tree(u),
        "fp64 once": f32(sum(float(x) for x in u)), "ascending weight": asc(sorted(u)),
        "descending weight": asc(sorted(u, reverse=True)),
    }


def assert_order_sensitive(u, transposed):
    want = asc(u)
    for name, got in alternatives(u, transposed).items():
        assert got != want, f"case does not separate ascending order from {name}"


# ---- SER: four two-hop paths to one target (token 7 -> {5, 6} -> 2) ---------------------------


def check_ser_order():
    args, u, ut = ser_case()
    assert_order_sensitive(u, ut)
    oi, ow, bad = oracle.ser(*args, 2)
    assert bad == 0
    want = f32(f32(f32(u[0] + u[1]) + u[2]) + u[3])
    assert oi[0, 7, 0].tolist() == [2, 0]
    assert ow[0, 7, 0, 0] == want, (ow[0, 7, 0, 0], want)
    assert ow[0, 7, 0, 1] == 0.0


def test_ser_merge_sums_in_ascending_candidate_order():
    check_ser_order()


def test_chain_step_merges_in_ascending_order():
    """A second step through an identity leg keeps the merged weight's bits (multiplying by 1.0
    is exact), so a chain merges its first step in the referral's order."""
    args, u, _ = ser_case()
    a1_idx, a1_w, a2_idx, a2_w = args
    n = a1_idx.shape[1]
    ident_i = np.broadcast_to(np.arange(n, dtype=np.int32)[None, :, None, None], (1, n, 1, 2)).copy()
    ident_w = np.zeros((1, n, 1, 2), np.float32)
    ident_w[..., 0] = 1.0
    ci, cw, bad = oracle.ser_chain(a1_idx, a1_w, [(a2_idx, a2_w), (ident_i, ident_w)], 2, 2)
    assert bad == 0
    assert ci[0, 7, 0, 0] == 2 and cw[0, 7, 0, 0] == asc(u)


# ---- referral with refresh edges: two paths, then two refresh slots, one target --------------


def check_refresh_order():
    args, u, refresh_first = refresh_case()
    assert_order_sensitive(u, refresh_first)
    assert asc([u[0], u[2], u[1], u[3]]) != asc(u), "interleaved order not separated"
    oi, ow, bad = oracle.ser_refresh(*args, 2)
    assert bad == 0
    want = f32(f32(f32(u[0] + u[1]) + u[2]) + u[3])
    assert oi[0, 7, 0].tolist() == [3, 0]
    assert ow[0, 7, 0, 0] == want, (ow[0, 7, 0, 0], want)


def test_refresh_slots_merge_after_the_paths_in_ascending_order():
    check_refresh_order()


# ---- leg sparsification: two stored channels x two slots, one target --------------------------


def check_leg_order():
    args, u, ut = leg_case()
    assert_order_sensitive(u, ut)
    a1i, a1w, _, _, bad = oracle.leg_sparsify(*args, 2, 2)
    assert bad == 0
    want = f32(f32(f32(u[0] + u[1]) + u[2]) + u[3])
    assert a1i[0, 3, 0].tolist() == [1, 0]
    assert a1w[0, 3, 0, 0] == want, (a1w[0, 3, 0, 0], want)


def test_leg_candidates_merge_in_ascending_channel_slot_order():
    check_leg_order()


# ---- the pins reject an oracle whose merge runs in reverse -----------------------------------

MERGE_LOOP = re.compile(r"for \(int c = 0; c < nc; \+\+c\) \{(\s*)int m = 0;")
REVERSED = r"for (int c = nc - 1; c >= 0; --c) {\1int m = 0;"


def build_mutant(tmp_path, patch):
    src = open(obuild.SRC).read()
    mutated = patch(src)
    assert mutated != src, "the mutation did not apply: the oracle's merge loop changed"
    path = tmp_path / "gm_oracle_mutant.c"
    path.write_text(mutated)
    lib = tmp_path / "libgm_oracle_mutant.so"
    subprocess.run(["gcc", *obuild.CFLAGS, str(path), "-o", str(lib), "-lm"], check=True)
    good = oracle._load()
    mutant = ctypes.CDLL(str(lib))
    for name in ("oracle_ser", "oracle_ser_refresh", "oracle_leg_sparsify", "oracle_num_threads"):
        fn, ref = getattr(mutant, name), getattr(good, name)
        fn.restype, fn.argtypes = ref.restype, ref.argtypes
    return mutant


def with_lib(lib, check):
    saved = oracle._lib
    oracle._lib = lib
    try:
        check()
    finally:
        oracle._lib = saved


def reverse_merge_in(function):
    """Reverse the first merge loop inside the body of `function` (up to the next function)."""
    def patch(src):
        head, sep, tail = src.partition(function)
        body, nxt, rest = tail.partition("\n}\n")
        return head + sep + MERGE_LOOP.sub(REVERSED, body, count=1) + nxt + rest
    return patch


reverse_ser_merge = reverse_merge_in("int64_t oracle_ser(")
reverse_shared_merge = reverse_merge_in("static int merge_and_order(")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_reversed_ser_merge_fails_the_pin(tmp_path):
    mutant = build_mutant(tmp_path, reverse_ser_merge)
    with pytest.raises(AssertionError):
        with_lib(mutant, check_ser_order)
    # the mutation touches the plain referral only
    with_lib(mutant, check_refresh_order)
    with_lib(mutant, check_leg_order)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_reversed_shared_merge_fails_the_refresh_and_leg_pins(tmp_path):
    mutant = build_mutant(tmp_path, reverse_shared_merge)
    with pytest.raises(AssertionError):
        with_lib(mutant, check_refresh_order)
    with pytest.raises(AssertionError):
        with_lib(mutant, check_leg_order)
    with_lib(mutant, check_ser_order)
