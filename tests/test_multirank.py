"""The multi-GPU path of bench.py on CPU: two gloo ranks, each with its own independent batch
(seed + rank) and no collective on the data path; only the timing bookkeeping is reduced
(max of the step time, sum of the tokens) -- the weak-scaling aggregation the bench reports."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    from bit_paged_kv_append_b200 import synth

    assert bench._init_dist() == world
    w_lengths = synth.seq_lengths("batch16", seed=0 + rank)  # each rank: its own batch
    tokens = float(sum(w_lengths))
    step_ms = 1.0 + rank  # rank 1 is the slow one
    mx = bench.reduce_over_ranks(step_ms, "max", torch.device("cpu"))
    sm = bench.reduce_over_ranks(tokens, "sum", torch.device("cpu"))
    q.put((rank, mx, sm, tokens))
    dist.destroy_process_group()


def test_two_ranks_aggregate_like_the_bench():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    toks = {r: t for r, _, _, t in out}
    assert toks[0] != toks[1]  # independent batches
    for _, mx, sm, _ in out:
        assert mx == 2.0  # the max over ranks of the step time
        assert sm == toks[0] + toks[1]  # whole-job tokens
