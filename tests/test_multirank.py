"""The benchmark's N > 1 plumbing on CPU: two gloo ranks (one process each, as torchrun runs
them), barrier, max over ranks of a device time, and the reference arm that only rank 0 runs.
Replicas: every rank runs the same per-GPU workload, so the job's value is the units of all
ranks over the max time; no collective touches the data path."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_init(backend="gloo")
    bench.barrier(w)
    # rank r "measured" (r + 1) ms; the job's time is the slowest rank's
    m = bench.max_over_ranks(w, float(r + 1))

    class Args:
        steps, warmup = 1, 3

    line = bench.run_reference(Args, w, r)
    out.put((r, w, m, None if line is None else (line["impl"], line["n_gpus"], line["unit"])))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, *_ in res] == [0, 1]
    assert all(w == 2 and m == 2.0 for _, w, m, _ in res)
    assert res[0][3] == ("reference", 2, "keys/s")   # rank 0 prints the reference line
    assert res[1][3] is None                          # the other ranks do no work


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1, 3.5) == 3.5
    bench.barrier(1)


def test_bench_launches_its_own_ranks():
    """`python bench.py --gpus 2` with no torchrun environment starts two ranks itself (one
    process per GPU) and rank 0 reports n_gpus = 2; here over gloo, with no GPU work."""
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR",
                                                            "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--plumbing-only",
                        "--steps", "3", "--warmup", "3"], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["plumbing_only"]
    assert lines[0]["ms_per_step"] >= 2.0      # the slower rank (2 ms per step) sets the time


def test_bench_refuses_a_mismatched_world_size():
    import subprocess
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--plumbing-only"],
                       capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode != 0 and "WORLD_SIZE" in r.stderr
