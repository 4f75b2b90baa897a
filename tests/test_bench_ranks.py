"""The multi-GPU path of bench.py, on CPU: two gloo ranks.

bench.py runs one independent replica per GPU; the only cross-rank step is taking
the slowest rank's timings and scaling the whole job's work by them. Those two pieces
are checked here with world size 2 on the gloo backend, plus the reference arm's
rank handling (only rank 0 prints) and its JSON line.
"""

import json
import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 5.0 - rank, 7.5]
        got = bench.max_over_ranks(mine, dist, "cpu")
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = 29500 + os.getpid() % 1000
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
    assert out[0] == out[1] == [11.0, 5.0, 7.5]


def test_job_throughput_is_whole_job_over_slowest_rank():
    # 2 ranks, 1e12 flop per rank-step, 10 steps, slowest rank 20 ms -> 1000 TFLOP/s
    assert bench.job_throughput(2, 1e12, 10, 20.0) == pytest.approx(1000.0)
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]


def test_reference_arm_prints_only_on_rank_0(capsys):
    class A:
        steps, warmup, gpus = 1, 0, 2
    bench.run_reference(A, bench.WORKLOADS["c1"], rank=1)
    assert capsys.readouterr().out == ""


def test_reference_arm_json_line():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "c1", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["metric"] == bench.METRIC


def test_linear_fit_recovers_slope_and_r2():
    slope, icpt, r2 = bench.linear_fit([1, 2, 4, 8], [13, 23, 43, 83])
    assert slope == pytest.approx(10.0) and icpt == pytest.approx(3.0) and r2 == pytest.approx(1.0)
    _, _, r2 = bench.linear_fit([1, 2, 3, 4], [1, 4, 9, 16])
    assert r2 < 1.0


def test_timing_inputs_have_the_workload_structure():
    """Seeded device-drawn inputs (timing runs): shape, dtype, and exactly floor(0.01 N)
    rows per head scaled x8 for the large-logit workload."""
    import torch
    w = type(bench.WORKLOADS["c4"])("t", 1, 2, 1000, 64, "bf16", True, 5, large_frac=0.01)
    q, k, v, do = bench.torch_inputs(w, "cpu", 5)
    assert q.shape == (1, 2, 1000, 64) and q.dtype == torch.bfloat16
    q2, _, _, _ = bench.torch_inputs(w, "cpu", 5)
    assert torch.equal(q, q2)
    norms = q.float().norm(dim=-1)[0]             # [H, N]
    assert ((norms > 40).sum(dim=1) == 10).all()  # ~8 * sqrt(64) vs ~sqrt(64)


@pytest.mark.parametrize("nq,nk", [(4, 4), (7, 30), (30, 7), (128, 1000)])
@pytest.mark.parametrize("window", [(-1, -1), (-1, 0), (3, 0), (0, 5), (10, -1), (0, 0)])
def test_visible_pairs_counts_the_window(nq, nk, window):
    import numpy as np
    i = np.arange(nq)[:, None]
    j = np.arange(nk)[None, :]
    off = nk - nq
    vis = np.ones((nq, nk), bool)
    if window[0] >= 0:
        vis &= j >= i + off - window[0]
    if window[1] >= 0:
        vis &= j <= i + off + window[1]
    assert bench.visible_pairs(nq, nk, window) == int(vis.sum())
