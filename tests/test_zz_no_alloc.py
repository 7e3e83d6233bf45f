"""gm_sea_backward_noalloc: the SEA backward for callers that may not allocate device memory.

Such callers (code inside an allocator's own hooks, runtimes whose device memory all belongs
to their own pool, step loops that forbid allocation because it can synchronise the device)
cannot hand gm_sea_backward a workspace. The no-alloc entry point runs the same gather path
on a fixed scratch array the library keeps on each device. This file checks, through the C
ABI, that two calls in a row give what the workspace entry point gives and what the fp64
oracle gives, and that a problem too large for the array is refused before anything runs. It
is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_dynamic_routing_b200 as gm
from sparse_dynamic_routing_b200 import _binding as bnd
from sparse_dynamic_routing_b200 import inputs as I

TOL = 2e-2  # bf16 features, as in the parity tests


def _max_abs(a, b):
    return float((a.double() - b.double()).abs().max())


@pytest.mark.gpu
def test_noalloc_backward_matches_workspace_backward_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    wl = I.WORKLOADS["long_b1_n32768_s4_train"].with_(n=8192)
    x = {k: v.cuda() for k, v in I.make(wl, grad=True).items()}
    need = gm.gm_sea_backward_workspace_size(torch.bfloat16, wl.s, wl.B, wl.n, wl.hq, wl.hkv,
                                             wl.d)
    assert 0 < need <= bnd.load_library().gm_sea_backward_noalloc_max_scratch()
    ref = gm.gm_sea_backward(x["q"], x["k"], x["v"], x["dout"], x["idx"], x["w"], wl.scale,
                             workspace="auto")
    # both GPU paths are also held to the fp64 oracle on the same bf16 inputs
    host = I.make(wl, grad=True)
    want = oracle.sea_backward(host["q"], host["k"], host["v"], host["dout"], host["idx"],
                               host["w"], wl.scale)[:4]
    for call in range(2):
        got = gm.gm_sea_backward_noalloc(x["q"], x["k"], x["v"], x["dout"], x["idx"], x["w"],
                                         wl.scale)
        gm.gm_check_device_errors()
        for name, a, b, w in zip(("dq", "dk", "dv", "dlogw"), got, ref, want):
            err = _max_abs(a, b)
            assert np.isfinite(err) and err <= TOL, f"call {call}: {name} differs by {err}"
            w = torch.from_numpy(w).reshape(a.shape)
            err = _max_abs(a.cpu(), w)
            assert np.isfinite(err) and err <= TOL, f"call {call}: {name} vs oracle: {err}"
        # dq and d ln w come from the same row pass in the same order: identical bits
        assert torch.equal(got[0], ref[0]) and torch.equal(got[3], ref[3])


def test_noalloc_refuses_problems_larger_than_its_scratch():
    lib = bnd.load_library()
    fake = 0x1000  # never dereferenced: the size check fails before anything is launched
    # 16 x 32768 tokens x 8 KV heads x 4 slots needs far more than the fixed scratch; dout is
    # misaligned as a second guard, so no path could reach a launch with these pointers
    st = lib.gm_sea_backward_noalloc(fake, fake, fake, fake + 2, bnd.GM_BF16, fake, fake, 4,
                                     16, 32768, 16, 8, 128, 0.088, fake, fake, fake, fake, 0, None)
    assert st == bnd.GM_ERR_SCRATCH_TOO_SMALL
    assert "scratch" in bnd.status_string(st)
    st = lib.gm_sea_backward_noalloc(fake, fake, fake, fake + 2, bnd.GM_BF16, fake, fake, 8,
                                     1, 64, 16, 8, 128, 0.088, fake, fake, fake, fake, 0, None)
    assert st == bnd.GM_ERR_UNSUPPORTED  # s > 4: the gather path does not cover it
