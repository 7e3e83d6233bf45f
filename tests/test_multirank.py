"""Host logic of the multi-GPU bench path, as two gloo ranks on CPU.

The path shards over independent sequences, so ranks exchange nothing on the data path:
each rank draws its own workload (seed offset by rank, same shapes), and the only
collectives are the timing barrier and the max-over-ranks reduction of the elapsed time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, store_path, out):
    # the variables torchrun sets (read by bench.dist_env); the rendezvous itself goes through
    # a file store and the loopback interface, so no port can be taken in between
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank), GLOO_SOCKET_IFNAME="lo")
    import bench
    from sparse_dynamic_routing_b200 import inputs as I

    dist.init_process_group("gloo", init_method=f"file://{store_path}", rank=rank,
                            world_size=world)
    try:
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        wl = bench.shard_seed(I.WORKLOADS["layer_b8_n4096_s2"].with_(B=1, n=64), rank)
        x = I.make(wl)
        # each rank's elapsed time; the bench reports the max over ranks
        t = bench.max_over_ranks(10.0 + rank, world, torch.device("cpu"))
        digest = float(x["q"].float().sum()) + float(x["a1_idx"].sum())
        out[rank] = (t, wl.seed, wl.B, wl.n, digest)
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_and_max_timing(tmp_path):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    store = str(tmp_path / "store")
    procs = [ctx.Process(target=_worker, args=(r, 2, port, store, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("rank did not finish")
        assert p.exitcode == 0
    (t0, s0, b0, n0, d0), (t1, s1, b1, n1, d1) = out[0], out[1]
    assert t0 == t1 == 11.0  # max over ranks, seen by every rank
    assert (b0, n0) == (b1, n1)  # same per-GPU work: weak scaling
    assert s0 != s1 and d0 != d1  # independent draws per rank
