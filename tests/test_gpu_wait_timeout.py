"""A bounded wait that runs out is reported, and the device stays usable.

Every wait a kernel of the library spins on (the dense refresh kernel's copies and tensor-core
operations, the backward scan's look-back) gives up after about one second, sets the device
error flag and returns instead of hanging. gm_selftest_wait_timeout runs one such wait on a
shared-memory barrier that nothing arrives at; the test checks the status the host reads and
that the next calls run normally. No GPU fault is involved.
"""
import time

import pytest
import torch

import sparse_dynamic_routing_b200 as gm
from sparse_dynamic_routing_b200 import _binding as bnd
from sparse_dynamic_routing_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    gm.load_library()
    gm.gm_check_device_errors()
    yield


def test_wait_that_runs_out_is_reported_and_the_device_stays_usable():
    t0 = time.perf_counter()
    gm.gm_selftest_wait_timeout()
    with pytest.raises(gm.GMError) as err:
        gm.gm_check_device_errors()
    waited = time.perf_counter() - t0
    assert err.value.status == bnd.GM_ERR_WAIT_TIMEOUT
    assert 0.5 < waited < 30.0  # the one-second limit, not a hang
    gm.gm_check_device_errors()  # the flag was cleared by the read
    # the device still runs the library's kernels and gives the right answers
    wl = I.WORKLOADS["tiny_b1_n128_s2_f32"]
    x = {k: v.cuda() for k, v in I.make(wl).items()}
    ai, aw = gm.gm_ser_forward(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], wl.s1)
    ai2, aw2, o, lse = gm.gm_ser_sea_forward(x["q"], x["k"], x["v"], x["a1_idx"], x["a1_w"],
                                             x["a2_idx"], x["a2_w"], wl.s1, wl.scale)
    gm.gm_check_device_errors()
    assert torch.equal(ai, ai2) and torch.equal(aw, aw2)
    assert torch.isfinite(o).all()
