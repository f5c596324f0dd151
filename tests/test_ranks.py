"""The multi-GPU benchmark path on CPU: world size 2 over gloo.

Under torchrun each rank quantizes and decodes its own batch (weak scaling,
no collective on the data path); the only collectives are the barriers around
the timed region and the max over ranks of the step time.  These checks run
that reduction in two gloo processes and check that the ranks' workloads are
distinct draws of the same shape.
"""
import os
import socket

import numpy as np
import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        torch.distributed.barrier()
        ms = bench.max_over_ranks(1.5 + 2.0 * rank, world, "cpu")
        torch.distributed.barrier()
        out.put((rank, ms))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 3.5, 1: 3.5}


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(2.25, 1, "cpu") == 2.25


def test_rank_workloads_are_distinct_draws_of_one_shape():
    import bench
    from kv_cache_bit_b200 import synth
    w0 = bench.rank_workload(0, batch=1, stream=0)
    w1 = bench.rank_workload(1, batch=1, stream=0)
    assert (w0.B, w0.Hq, w0.Hkv, w0.d, w0.S) == (w1.B, w1.Hq, w1.Hkv, w1.d, w1.S)
    k0, _ = synth.kv(w0.scaled(S=128))
    k1, _ = synth.kv(w1.scaled(S=128))
    assert k0.shape == k1.shape and not np.array_equal(k0, k1)
