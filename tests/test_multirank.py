"""The benchmark's multi-rank logic with two gloo ranks on the CPU.

Decode shards by sequence with no data exchange: each rank decodes its own
batch and only the timing is combined (max of step time, sum of units).
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        step_ms = [3.0, 5.0][rank]
        units = [[100.0, 7.0], [250.0, 9.0]][rank]
        t, u = bench.reduce_over_ranks(step_ms, units, world, "cpu")
        w = bench.rank_workload("llama70b", rank)
        out[rank] = (t, tuple(u), w.seed, w.num_seqs, tuple(w.context_lens[:3]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_combine_timings_and_split_batches():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        t, u, seed, nseq, head = res[rank]
        assert t == 5.0                       # max over ranks
        assert u == (350.0, 16.0)             # units summed over ranks
        assert nseq == 256
    assert res[0][2] != res[1][2]             # each rank has its own batch ...
    assert res[0][4] != res[1][4]             # ... with its own lengths (weak scaling)


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_over_ranks(2.5, [1, 2], 1, "cpu") == (2.5, [1.0, 2.0])
