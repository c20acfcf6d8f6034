"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

Every rank owns an independent layer (weak scaling, no data-path
collective); the only collective is the max-over-ranks of the timings.
This test runs that logic in two CPU processes: the per-rank seeds differ,
the compressed layers differ and each round-trips through the oracle, the
max reduction returns the slowest rank's time, and the aggregate throughput
counts every rank's bytes over that time.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from decode_gemm_exponent_b200 import synth
        from oracle import oracle as O
        seeds = [bench.rank_seed(i, rank) for i in range(3)]
        w = synth.weights_bf16(64, 256, 0.02, 0.001, 1.0, seed=seeds[0])
        enc = O.encode(w)
        assert np.array_equal(O.decode(enc), w)
        local_ms = 1.0 + rank                       # rank 1 is the slower one
        mx = bench.max_over_ranks(local_ms, world)
        out[rank] = (seeds, int(enc.stream_bits), mx, bench.aggregate_gbs(10**9, world, mx))
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_logic():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")     # no fork anywhere: the parent may hold threads (or a CUDA context)
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    (s0, b0, m0, v0), (s1, b1, m1, v1) = out[0], out[1]
    assert set(s0).isdisjoint(s1)                   # independent layers per rank
    assert b0 != b1                                 # different data, different streams
    assert m0 == m1 == 2.0                          # max over ranks
    assert v0 == pytest.approx(2 * 1e9 / 2e-3 / 1e9)
