"""Host logic of the multi-GPU (weak scaling) bench on CPU: two gloo ranks.

Each rank quantises its own shard (its own seeded batch), nothing crosses
ranks on the data path, and the reported time is the max over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from kv_cache_quantization_03_b200 import workloads as W
    wr, rk, lr = bench.rank_env()
    w = bench.shard(W.WORKLOADS["gqa"].scaled(batch=1, seq_len=64), rk)
    k = W.kv_inputs(w, "k")
    # rank r pretends its timed region took r + 1 ms; everybody must see the max
    m = bench.max_over_ranks([1.0 + rk, 10.0 - rk], wr)
    out[rank] = (wr, rk, w.seed, int(k[0, 0, 0, 0]), m)
    dist.barrier()
    dist.destroy_process_group()


def test_weak_scaling_shards_and_max_over_ranks():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    r0, r1 = out[0], out[1]
    assert (r0[0], r0[1]) == (2, 0) and (r1[0], r1[1]) == (2, 1)
    assert r0[2] != r1[2] and r0[3] != r1[3]          # distinct seeded shards
    assert r0[4] == r1[4] == [2.0, 10.0]              # max over ranks, element-wise


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup, gpus = 1, 0, 2

    from kv_cache_quantization_03_b200 import workloads as W
    bench.run_reference(A, W.WORKLOADS["gqa"])
    assert capsys.readouterr().out == ""
