"""The multi-rank host logic of bench.py on CPU: two gloo ranks, each with its
own time, agree on the max; whole-job throughput counts every rank's tokens."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        t = bench.max_over_ranks(0.5 + rank, dist, torch.device("cpu"))
        out[rank] = t
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert dict(out) == {0: 1.5, 1: 1.5}


def test_throughput_counts_every_rank():
    import bench
    one = bench.throughput_mtok(1, 1, 32768, 10, 0.01)
    assert abs(one - 32.768) < 1e-9
    assert abs(bench.throughput_mtok(4, 1, 32768, 10, 0.01) - 4 * one) < 1e-9
    assert bench.max_over_ranks(3.0) == 3.0


def _gather_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from linear_attention_11_b200 import seqpar
        state = torch.full((2, 3, 4, 4), float(rank + 1))
        got = seqpar.gather_states(state)
        out[rank] = [float(x) for x in got[:, 0, 0, 0, 0]]
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_sequence_sharding_gathers_states_in_rank_order():
    """The states of a sharded sequence arrive stacked in rank (= token) order
    on every rank: gloo, three ranks on CPU."""
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, 3, port, out)) for r in range(3)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert dict(out) == {r: [1.0, 2.0, 3.0] for r in range(3)}
