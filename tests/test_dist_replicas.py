"""The N > 1 replica plumbing of bench.py on CPU (gloo, world size 2): every
rank takes the same collective steps (barriers, one max all-reduce of the
device-timed milliseconds), the result is the max over ranks on every rank,
and the environment parsing matches what torchrun sets."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    w, r, local = bench.dist_env()
    dist = bench.dist_init(w, backend="gloo")
    try:
        bench.dist_barrier(dist)
        mine = 1.5 + 2.0 * rank  # this rank's "elapsed ms"
        got = bench.dist_max(dist, mine, "cpu")
        bench.dist_barrier(dist)
        q.put((r, w, local, got))
    finally:
        dist.destroy_process_group()


def test_two_replicas_share_the_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    results = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[0] for r in results] == [0, 1]
    assert all(r[1] == 2 and r[2] == r[0] for r in results)
    assert all(abs(r[3] - 3.5) < 1e-12 for r in results)  # max(1.5, 3.5) on both ranks


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_init(1) is None
    assert bench.dist_max(None, 2.25, "cpu") == 2.25
    bench.dist_barrier(None)


def test_reference_arm_runs_on_rank_zero_only():
    import json
    import subprocess
    base = {**os.environ, "WORLD_SIZE": "2", "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(_free_port())}
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "2", "--warmup", "3", "--gpus", "2"]
    r1 = subprocess.run(cmd, env={**base, "RANK": "1", "LOCAL_RANK": "1"}, capture_output=True, text=True, timeout=300)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = subprocess.run(cmd, env={**base, "RANK": "0", "LOCAL_RANK": "0"}, capture_output=True, text=True, timeout=300)
    assert r0.returncode == 0, r0.stderr[-2000:]
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
