"""The N>1 host path of bench.py on CPU: two ranks over ``gloo`` (no GPU).

The hot path shards by sequence with no exchange step, so ``bench.py --gpus N``
runs N independent replicas: each rank times the same seeded workload, the
job reports the slowest rank's device time (max over ranks) and the whole-job
rate world x work / that time.  Checked here with world_size 2: the max
reduction, the barrier, the aggregation, and that the ranks' replicas are the
same seeded problem (identical oracle outputs).
"""

from __future__ import annotations

import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, outdir: str):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        from paged_kv_attention_35_b200 import synth
        from tests.problems import decode_problem
        # a timed region that differs per rank: the job reports the slowest
        mine = 10.0 + 5.0 * rank
        slowest = bench.max_over_ranks(torch, dist, world, mine)
        bench.barrier(torch, dist, world)
        # every rank's replica is the same seeded problem
        pr = decode_problem([5, 40, 77], hq=4, hkv=2, d=64, bs=16, seed=synth.SEED_BASE + 31)
        f64 = oracle.bf16_bits_to_f64
        out = oracle.ref_decode(f64(pr["q"]), f64(pr["k_pool"]), f64(pr["v_pool"]),
                                pr["block_tables"], pr["lens"])
        digest = float(np.abs(out).sum())
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "digests": digests}, f)
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["slowest"] == 15.0                      # max over ranks, on every rank
        assert r["digests"][0] == r["digests"][1]        # identical replicas
    import bench
    # whole-job rate: world x per-rank work over the slowest rank's time
    one = bench.whole_job_rate(1, 1e6, 10, 20.0)
    assert bench.whole_job_rate(2, 1e6, 10, 20.0) == pytest.approx(2 * one)
    assert bench.whole_job_rate(2, 1e6, 10, 40.0) == pytest.approx(one)
