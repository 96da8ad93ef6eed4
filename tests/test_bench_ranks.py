"""Multi-rank host logic of bench.py on CPU: gloo ranks, world size 2."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r measured (r + 1) ms of steps and (10 - r) ms end to end
        out[rank] = bench.max_over_ranks([rank + 1.0, 10.0 - rank], "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world_2():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        got = dict(out)
    assert got[0] == got[1] == [2.0, 10.0]


def test_job_value_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 128 units per step x 4 steps in 2 ms (the slower rank's time)
    assert bench.job_value(2, 128, 4, 2.0) == 2 * 128 * 4 / 2e-3
    assert bench.max_over_ranks([3.0, 4.0], "cpu") == [3.0, 4.0]   # no process group


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node",
           "2", "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "cfg1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_oracle_sample_stays_inside_the_reserved_capacity():
    """The CPU baseline appends one token per step: it stops at the workload's reserved
    capacity however much time budget is left."""
    sys.path.insert(0, ROOT)
    import bench
    from workloads import gen
    w = gen.scaled("cfg1", context_lens=(256,), extra_tokens=8)
    *_, n = bench.oracle_sample(w, budget_s=60.0)
    assert n == 8
    *_, n = bench.oracle_sample(w, 0.0, steps=20)
    assert n == 8


def _gather_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from block_sparse_linear_b200.sharded import dist_gather
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # this rank's two shards' candidate rows, marked with the global shard index
        local = torch.stack([torch.full((3, 2), 2 * rank + i, dtype=torch.int32) for i in range(2)])
        out[rank] = dist_gather(local).tolist()
    finally:
        dist.destroy_process_group()


def test_sharded_decode_gather_orders_shards_by_rank_gloo_world_2():
    """The all-gather between the sharded decode's phases stacks every rank's shards in
    global shard order (rank-major), as spla_shard_partials and spla_shard_merge expect."""
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_gather_main, args=(2, port, out), nprocs=2, join=True)
        got = dict(out)
    want = [[[s, s]] * 3 for s in range(4)]
    assert got[0] == got[1] == want
