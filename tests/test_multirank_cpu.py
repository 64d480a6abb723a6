"""The bench's multi-rank plumbing on CPU: two gloo ranks on 127.0.0.1.

Under torchrun each rank runs its own batch (replicas; no collective on the
data path), the step time is the maximum over ranks, and the job throughput
counts every rank's bytes.  The reference arm prints from rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(1.5 + rank, dist, "cpu")
        dist.barrier()
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_job_throughput_is_weak_scaling():
    import bench
    one = bench.job_throughput(1_000_000, 1, 0.5)
    assert abs(one - 2.0) < 1e-12            # 1 MB per 0.5 ms = 2 GB/s
    assert abs(bench.job_throughput(1_000_000, 4, 0.5) - 4 * one) < 1e-9


def test_reference_arm_prints_from_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "tiny", "--gpus", "2"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "tiny", "--gpus", "2"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["cores"] == 1


def _counts_main(rank, world, port, out):
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from combine_route_meta_b200.ep import exchange_counts
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        counts = torch.from_numpy(np.arange(8, dtype=np.int32) * (rank + 1))
        got = exchange_counts(counts)
        dist.barrier()
        out[rank] = got.numpy().tolist()
    finally:
        dist.destroy_process_group()


def test_expert_parallel_count_exchange_two_gloo_ranks():
    # the count exchange that precedes expert-parallel dispatch: every rank ends
    # with every rank's per-expert counts, in rank order
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_counts_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    want = [[i * (r + 1) for i in range(8)] for r in range(2)]
    assert out[0] == want and out[1] == want


def test_expert_parallel_bench_plumbing():
    # the host-side parts of `bench.py --parallelism ep`: which rank counts can
    # share the experts, the per-rank byte model, and the config both arms print
    sys.path.insert(0, ROOT)
    import bench
    from workloads import WORKLOADS
    for n in (1, 2, 4, 8):
        bench.ep_ranks_check(256, n)
    for bad in (3, 0, 128):
        with pytest.raises(SystemExit):
            bench.ep_ranks_check(256, bad)
    w = WORKLOADS["dsv3_decode"]
    d, c = bench.algorithmic_bytes(w.T, w.H, w.E, 1, w.k, w.fp8)
    assert bench.ep_step_bytes(w) == d + c
    cfg = bench.config_for(w, 8, w.T * w.k, "ep")
    assert cfg["parallelism"] == "ep x8" and cfg["workload"] == "dsv3_decode"


def test_reference_arm_prints_the_ep_config():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
                        "--workload", "tiny", "--parallelism", "ep"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["config"]["parallelism"] == "ep x1"
