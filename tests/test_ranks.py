"""The multi-GPU benchmark path on CPU: world size 2 over gloo.

Under torchrun each rank quantizes and decodes its own batch (weak scaling,
no collective on the data path), or, with --split-batch, its shard of one
workload's batch (strong scaling); the only collectives are the barriers
around the timed regions, the max over ranks of the step time and the sum
of the bytes moved.  These checks run those reductions in two gloo
processes, check that the ranks' workloads are distinct draws of the same
shape, and that a batch split over two ranks reproduces one rank's outputs
(the oracle stands in for the GPU path on the CPU).
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


def test_batch_shards_cover_the_batch_once():
    import bench
    for B in (1, 2, 5, 64, 67):
        for world in (1, 2, 3, 4, 8):
            spans = [bench.batch_shard(B, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == B
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1


def _shard_outputs(rows):
    """A bench-shaped step on the CPU for the batch rows [lo, hi) of one
    small throughput-shaped workload: the oracle quantizes the prefill, then
    three tokens are streamed and the oracle's decode attention runs after
    each (quantized blocks + fp16 residual tokens)."""
    import oracle
    from kv_cache_bit_b200 import synth
    from tests.modes import f16bits, oracle_cfg
    lo, hi = rows
    w = synth.WORKLOADS["throughput"].scaled(B=4, Hkv=2, Hq=8, S=256, stream=3)
    K, V = synth.kv(w)
    ks, vs = synth.stream_tokens(w)
    qs = synth.queries(w, steps=3)
    K, V, ks, vs, qs = K[lo:hi], V[lo:hi], ks[:, lo:hi], vs[:, lo:hi], qs[:, lo:hi]
    cfg = oracle_cfg("nsn+hadamard", w.d, 4)
    ck = oracle.quantize(cfg, f16bits(K), 384)
    cv = oracle.quantize(cfg, f16bits(V), 384)
    outs = []
    for i in range(3):
        rk = f16bits(np.ascontiguousarray(ks[:i + 1].transpose(1, 2, 0, 3)))
        rv = f16bits(np.ascontiguousarray(vs[:i + 1].transpose(1, 2, 0, 3)))
        outs.append(oracle.cache_attention(cfg, f16bits(qs[i]), ck, cv, rk, rv, w.S + i + 1))
    return np.stack(outs)


def _split_main(rank, world, port, out):
    import datetime
    import torch
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        mine = _shard_outputs(bench.batch_shard(4, rank, world))
        got = [None] * world
        torch.distributed.all_gather_object(got, mine)
        total = bench.sum_over_ranks(float(mine.shape[1]), world, "cpu")
        if rank == 0:
            out.put((np.concatenate(got, axis=1), total))
    finally:
        torch.distributed.destroy_process_group()


def test_split_batch_on_two_ranks_reproduces_one_rank_outputs():
    """One workload's batch split over two gloo ranks: each rank runs the
    bench-shaped step (quantize, stream, decode) on its rows; the gathered
    outputs equal those of one rank running the whole batch, bit for bit
    (every (batch row, kv head) pair is an independent problem)."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    # read before joining: rank 0 cannot exit until its result has left the queue
    split, total = q.get(timeout=300)
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    whole = _shard_outputs((0, 4))
    assert total == 4.0
    assert split.shape == whole.shape == (3, 4, 8, 128)
    assert np.array_equal(split, whole)
