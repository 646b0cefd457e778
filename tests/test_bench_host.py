"""Host-side logic of bench.py, on CPU: the multi-rank timing reduction over a
world-size-2 gloo group, the reference arm's JSON line, and rank > 0 of the
reference arm exiting without output."""

import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        t = bench.reduce_max(10.0 + 5.0 * rank, world, torch.device("cpu"))
        q.put((rank, t))
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def test_launch_count_and_config_block():
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    assert bench.launches_per_step(32768, 4096) == 5 + 2 * 8
    assert bench.launches_per_step(300, 128) == 5 + 2 * 3
    assert bench.launches_per_step(0, 128) == 0
    assert bench.launches_per_step(32768, 4096, skip_rows=True) == 6 + 4 * 8
    blk = bench.config_block(workloads.get_config(3), 4)
    assert blk["global_batch"] == 4 * 32768 and blk["workload"].startswith("gptoss_head")


def _run_bench(args, env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True,
                          text=True, timeout=600, env=env, cwd=ROOT)


def test_reference_arm_line():
    out = _run_bench(["--impl", "reference", "--config", "0", "--steps", "2", "--warmup", "3"])
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"].startswith("small_parity")


def test_reference_arm_other_ranks_exit_quietly():
    out = _run_bench(["--impl", "reference", "--config", "0", "--steps", "1", "--warmup", "3"],
                     {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_warmup_below_three_rejected():
    out = _run_bench(["--impl", "reference", "--config", "0", "--steps", "1", "--warmup", "2"])
    assert out.returncode != 0


def test_teacher_topk_mode_host_logic():
    import bench
    assert bench.topk_launches_per_call(32768, 4096) == 16
    assert bench.topk_launches_per_call(4097, 4096) == 4
    assert bench.topk_launches_per_call(0, 4096) == 0
    # the cache writer has no reference arm of its own (its oracle is the cpu_baseline)
    out = _run_bench(["--op", "teacher-topk", "--impl", "reference", "--config", "0", "--steps", "1",
                      "--warmup", "3"])
    assert out.returncode != 0 and "teacher-topk" in out.stderr


def test_peak_memory_line_fit():
    """The secondary block's least-squares line through peak GiB against N:
    exact on points on a line, and the largest relative residual it reports
    is that of the point off the line."""
    sys.path.insert(0, ROOT)
    import bench
    ns = [4096, 16384, 32768, 65536, 131072, 262144]
    gib = [2.5 + n * 10000 / 2**30 for n in ns]
    fit = bench.line_fit(ns, gib)
    assert abs(fit["slope_bytes_per_token"] - 10000) < 1e-6
    assert abs(fit["intercept_gib"] - 2.5) < 1e-9
    assert fit["max_rel_residual"] < 1e-12
    gib[2] *= 1.01                                     # one point 1 % high
    fit = bench.line_fit(ns, gib)
    assert 0.005 < fit["max_rel_residual"] < 0.011
