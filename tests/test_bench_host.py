"""Host logic of bench.py on CPU: the multi-rank timing reduction (gloo,
world size 2), the whole-job throughput, the reference arm's rank rule, and
the closed-form pair count the useful-FLOP figure rests on."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from oracle import ssa_oracle as orc  # noqa: E402


def _rank_main(rank, world, port, times, out):
    import torch.distributed as td
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    td.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(times[rank])
    finally:
        td.destroy_process_group()


def test_max_over_ranks_gloo_world_2():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    times = [3.25, 7.5]
    port = 29000 + os.getpid() % 2000
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 7.5


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(4.0) == 4.0


def test_job_throughput_counts_all_ranks_over_slowest_time():
    # 2 ranks x 10 steps x 1e9 units in 2000 ms (slowest rank) -> 1e10 units/s
    assert bench.job_throughput(2, 1e9, 10, 2000.0) == pytest.approx(1e10)
    assert bench.job_throughput(1, 5.0, 4, 1000.0) == pytest.approx(20.0)


def test_reference_arm_prints_only_on_rank_0():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3", "--config", "tiny"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_on_rank_0():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--config", "tiny",
                        "--ref-budget-s", "2"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


@pytest.mark.parametrize("L", [1, 127, 128, 1024, 1025, 5000])
def test_window_pairs_matches_oracle_row_counts(L):
    rows = np.arange(L)
    want = sum(orc.row_count(int(i), 128, 1, 7) for i in rows)
    assert bench.window_pairs(L) == want


def test_source_hash_ignores_comments_only():
    """The traffic records are keyed by a hash of the kernel code without its
    comments: an edit of comments keeps the hash, an edit of code changes it."""
    src = "int f(int a) { // add one\n  return a + 1; /* the\n result */ }\n"
    assert bench.code_only(src) == bench.code_only(
        "int f(int a) {\n  // a different comment\n  return a + 1;\n}\n")
    assert bench.code_only(src) != bench.code_only(src.replace("a + 1", "a + 2"))
