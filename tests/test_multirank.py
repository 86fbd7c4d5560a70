"""Multi-process host logic of the benchmark on CPU (gloo, world size 2): the layer runs as
independent replicas, one per GPU, and the job's time is the slowest rank's, reduced over the
process group; only rank 0 runs the oracle reference arm."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=timedelta(seconds=60))
    import bench
    ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
    got = bench.max_over_ranks(ms, "cpu")
    q.put((rank, got))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 15.0, 1: 15.0}


def test_max_over_ranks_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


def test_reference_arm_other_ranks_do_no_work(monkeypatch):
    import argparse
    import bench
    from moe_workloads import WORKLOADS
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(steps=1, warmup=0, gpus=2, ref_tokens=1)
    assert bench.run_reference(args, WORKLOADS["e128_bf16"]) == 0
