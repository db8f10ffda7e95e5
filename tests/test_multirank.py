"""The multi-GPU replica plumbing of bench.py, on CPU: two gloo ranks.

Under torchrun every rank runs one independent replica of the step (the
path has no exchange step); the job's time is the slowest rank's, its
throughput the FLOPs of all replicas over that time, and only rank 0 of the
reference arm does any work.  No GPU is used here."""
import json
import os
import socket
import sys
import tempfile

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank timings (ms): rank r is slower on the first, faster on the second
        mine = [1.0 + rank, 10.0 - rank, 3.0]
        got = bench.max_over_ranks(torch, mine, "cpu")
        ref = bench.run_reference(None, rank) if rank != 0 else None
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"got": got, "ref": ref}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_replica():
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_worker, args=(world, _free_port(), d), nprocs=world, join=True)
        res = [json.load(open(os.path.join(d, f"rank{r}.json"))) for r in range(world)]
    for r in res:
        assert r["got"] == [2.0, 10.0, 3.0]           # element-wise max over ranks
    assert res[1]["ref"] == 0                          # reference arm: other ranks exit 0


def test_job_throughput_counts_every_replica():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_tflops(2.0e12, 1, 1000.0) == 2.0
    assert bench.job_tflops(2.0e12, 8, 1000.0) == 16.0
    assert bench.max_over_ranks(torch, [4.0, 5.0], "cpu") == [4.0, 5.0]   # single process
