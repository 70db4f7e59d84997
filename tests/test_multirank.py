"""The multi-rank host logic on CPU, world size 2 over gloo: the job totals
bench.py reports (units summed over ranks, time of the slowest rank), the
per-rank input shards (each rank draws its own batch of the same shape:
the path is data-parallel, with no exchange), and the reference arm, which
only rank 0 runs."""
import json
import os
import socket
import sys
from datetime import timedelta
from types import SimpleNamespace

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    sys.path.insert(0, ROOT)
    import bench
    from sparse_paged_attention_build_b200 import workloads
    units, ms = bench.job_totals(100 * (rank + 1), 2.0 + rank, world, "cpu")
    w = workloads.make("c1", seed_offset=rank)
    rec = {"units": units, "ms": ms, "N": int(w.N), "q_sum": float(np.asarray(w.q, dtype=np.float64).sum()),
           "topk_sum": int(w.topk.sum())}
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(rec, f)
    dist.barrier()
    dist.destroy_process_group()


def test_job_totals_and_shards_two_ranks(tmp_path):
    mp.spawn(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    r0 = json.load(open(tmp_path / "r0.json"))
    r1 = json.load(open(tmp_path / "r1.json"))
    # units of both ranks (100 + 200), time of the slower (3.0 ms), on both
    assert r0["units"] == r1["units"] == 300.0
    assert r0["ms"] == r1["ms"] == 3.0
    # same shape, different draws
    assert r0["N"] == r1["N"]
    assert r0["q_sum"] != r1["q_sum"] and r0["topk_sum"] != r1["topk_sum"]


def test_single_rank_totals_are_local():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_totals(123, 4.5, 1, "cpu") == (123.0, 4.5)


def test_reference_arm_runs_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import bench
    args = SimpleNamespace(workload="c1", steps=1, warmup=0, ref_rows=0, gpus=2)
    assert bench.run_reference(args, 1, 2) == 0
