"""The multi-rank plumbing of bench.py on CPU with gloo, world size 2: every
rank holds the same layer (the shards split one layer), the timed region is
the slowest rank's, only rank 0 prints the JSON line, and both arms print
the same config."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workloads.get("tiny")
        t = bench.max_over_ranks(1.5 + rank, world, "cpu")
        L = bench.make_layer(w, 0, 0, "cpu")          # the sharded run's inputs
        q0 = L["q"].float()
        gathered = [torch.zeros_like(q0) for _ in range(world)]
        dist.all_gather(gathered, q0)
        out.put((rank, t, bench.rank_seed(w, 0, rank),
                 bool(torch.equal(gathered[0], gathered[1]))))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_same_layer_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, t0, s0, same0), (r1, t1, s1, same1) = res
    assert t0 == t1 == 2.5               # both ranks see the slowest rank's time
    assert same0 and same1               # both ranks hold the layer the shards split


def test_reference_arm_prints_on_rank_zero_only():
    base = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
            "--workload", "tiny", "--steps", "1", "--warmup", "0", "--seq", "256",
            "--cpu-seconds", "1"]
    env1 = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r1 = subprocess.run(base, env=env1, capture_output=True, text=True, timeout=300)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    env0 = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r0 = subprocess.run(base, env=env0, capture_output=True, text=True, timeout=300)
    assert r0.returncode == 0, r0.stderr
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_both_arms_print_the_same_config():
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    base = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
            "--workload", "tiny", "--steps", "1", "--warmup", "0", "--cpu-seconds", "1"]
    for gpus in (1, 2):
        env0 = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
        r0 = subprocess.run(base + ["--gpus", str(gpus)], env=env0, capture_output=True,
                            text=True, timeout=300)
        assert r0.returncode == 0, r0.stderr
        line = json.loads(r0.stdout.strip().splitlines()[-1])
        # tiny routes heads 1 and 3 of 4 sparse: fraction 0.5
        assert line["config"] == bench.bench_config(workloads.get("tiny"), 0.5, gpus)
