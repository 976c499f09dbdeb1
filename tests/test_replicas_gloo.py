"""The benchmark's multi-GPU layer (replicas, one process per GPU) on CPU:
two gloo ranks check the max-over-ranks timing, the whole-job throughput, the
per-rank rotation of hidden states, and that only rank 0 runs the reference
arm. No GPU is used."""
import argparse
import datetime
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, _ = bench.dist_setup()
        total = bench.max_over_ranks(10.0 * (r + 1), w, "cpu")  # rank r timed 10 (r+1) ms
        value = bench.job_throughput(total, 100, w)
        H = np.arange(1024 * 2).reshape(1024, 2)
        first = int(bench.rank_states(H, r)[0, 0])
        ref = "skipped"
        if r != 0:  # non-zero ranks leave the reference arm at once, without work
            ref = bench.run_reference(argparse.Namespace(steps=5, warmup=3, cpu_seconds=1.0))
        dist.barrier()
        q.put((r, w, total, value, first, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas():
    ctx = torch.multiprocessing.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    res = sorted(q.get(timeout=10) for _ in range(2))
    for r, w, total, value, first, ref in res:
        assert w == 2
        assert total == 20.0                      # the slowest rank's device time
        assert value == pytest.approx(2 * 100 / 0.020)  # both ranks' tokens over that time
    assert res[0][4] == 0 and res[1][4] == 37 * 2    # rank 1 starts 37 rows later
    assert res[1][5] is None                         # rank 1 returned from the reference arm


def test_bench_launches_its_own_ranks():
    # `bench.py --gpus 2` without an outside launcher starts two ranks itself;
    # the host self-test runs the replica layer on gloo and rank 0 alone prints
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--host-selftest",
                        "--steps", "20", "--warmup", "3"], capture_output=True, text=True, timeout=240, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["n_gpus"] == 2 and rec["host_selftest"] and rec["steps"] == 20
    assert rec["value"] == pytest.approx(2 * 20 / (rec["ms_per_step"] * 20 / 1e3))
