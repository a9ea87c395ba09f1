"""Host logic of bench.py on the CPU: the multi-rank timing reduction over
world-size-2 gloo process groups, the weak-scaling job value, and the
reference arm's rank handling under a torchrun-style environment."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist)   # rank 1 is the slow one
        out.put((rank, ms, bench.job_value(world, 1000, ms)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo_world_2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the slowest rank's time; the value counts both replicas
    assert [r[1] for r in res] == [15.0, 15.0]
    assert res[0][2] == pytest.approx(2 * 1000 / 15e-3)


def test_job_value_single_rank():
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.job_value(1, 65536, 0.5) == pytest.approx(65536 / 0.5e-3)


def _run_reference(rank, workload=None):
    env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    extra = [] if workload is None else ["--workload", workload]
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--gpus", "2", "--steps", "1", "--warmup", "3"] + extra,
                          capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)


def test_reference_arm_rank0_prints_one_line():
    r = _run_reference(0)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "lact_causal_n32k"


def test_reference_arm_other_ranks_exit_without_work():
    r = _run_reference(1)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


@pytest.mark.parametrize("workload", ["ttt_linear_f32_n256", "lact_layer_causal_n32k"])
def test_reference_arm_other_workloads(workload):
    """The oracle arm also times the linear layer and the full language layer
    (memory + window attention) on a bounded sample."""
    r = _run_reference(0, workload)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["config"]["workload"] == workload and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_window_flop_count_matches_brute_force():
    """The window branch's algorithmic FLOPs (4 d per in-window (query, key)
    pair) against a direct count of the pairs."""
    import types
    import numpy as np
    for N, W in ((1000, 300), (300, 1000), (2048, 2048), (4097, 128)):
        i = np.arange(N)[:, None]
        j = np.arange(N)[None, :]
        pairs = int(((j <= i) & (j > i - W)).sum())
        b = types.SimpleNamespace(window=W, N=N, d=128, B=2, H=3)
        assert bench.LaCTBench.window_flops(b) == 4 * 128 * pairs * 6
    assert bench.LaCTBench.window_flops(types.SimpleNamespace(window=0, N=10, d=128, B=1, H=1)) == 0
