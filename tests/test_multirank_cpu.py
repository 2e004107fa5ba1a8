"""The multi-rank bench path on CPU: two gloo ranks reduce their timings to the
max over ranks, and the weak-scaling throughput counts every rank's batch."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench

    # each rank reports its own (step time, attention time); rank 1 is slower
    mine = [10.0 + 5.0 * rank, 7.0 - rank]
    q.put((rank, bench.max_over_ranks(mine, "cpu")))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got[0] == got[1] == [15.0, 7.0]


def test_weak_scaling_throughput():
    import bench

    # 2 ranks x 16 sequences x 64 steps in 100 ms (max over ranks)
    assert bench.weak_scaling_tokens_per_s(2, 16, 64, 100.0) == pytest.approx(20480.0)
    assert bench.max_over_ranks([1.0, 2.0], "cpu") == [1.0, 2.0]  # single process: identity


def test_attention_bytes_formula():
    import bench
    import synth

    w = synth.WORKLOADS["llama3_8b_gqa_8k"]
    # S = 8192: 252 groups of 3072 B + 128 residual tokens x 512 B per (seq, kv head)
    per_seq = 252 * 3072 + 128 * 128 * 4
    assert bench.attention_bytes(w, 8192) == 16 * 8 * per_seq + 16 * 32 * 128 * 6
