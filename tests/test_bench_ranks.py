"""bench.py's multi-rank plumbing on CPU (gloo, world size 2): the whole-job
rate counts every rank's units over the slowest rank's time, and the
reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.dist_barrier(world)
        ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        worst = bench.max_over_ranks(ms, world, torch.device("cpu"))
        out[rank] = (worst, bench.whole_job_rate(2e12, world, worst))
        bench.dist_barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][1] == pytest.approx(2 * 2e12 / 15e-3 / 1e12)


def test_single_rank_helpers_need_no_process_group():
    assert bench.max_over_ranks(3.0, 1, "cpu") == 3.0
    assert bench.whole_job_rate(1e12, 1, 1000.0) == pytest.approx(1.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_flop_and_byte_counts_match_closed_forms():
    # FA: T(T+1)/2 visible pairs; SA tiny case: 9 of 10 causal 64x64 tiles, diagonal halves.
    assert bench.causal_pairs_fa(256) == 256 * 257 // 2
    full, diag = 64 * 64, 64 * 65 // 2
    assert bench.pairs_sa(256, 64, 1, 2) == 5 * full + 4 * diag
    assert bench.sa_decode_tokens(131072, 128, 1, 16) == 128 + 16 * 128
    assert bench.sa_decode_tokens(131072 + 5, 128, 1, 16) == 128 + 15 * 128 + 5


def test_reference_arm_steps_and_config(monkeypatch):
    """The reference arm runs W untimed and K timed bounded samples and reports the same
    workload config as the library's arm; value = FLOPs of the timed steps / their time."""
    calls = []

    class FakeSample:
        class oracle:
            @staticmethod
            def num_threads():
                return 3

        def run(self, seconds):
            calls.append(seconds)
            return 1000, 0.5, 64          # visible pairs, seconds, rows

    monkeypatch.setattr(bench, "OracleSample", FakeSample)
    args = type("A", (), {"steps": 4, "warmup": 3, "gpus": 1})()
    line = bench.run_reference(args, 1)
    assert len(calls) == 7 and all(0.5 <= c <= 4.0 for c in calls)
    assert line["impl"] == "reference" and line["config"] == bench.bench_config(1)
    assert line["value"] == pytest.approx(4.0 * bench.D * 4000 / 2.0 / 1e12)
    assert line["ms_per_step"] == pytest.approx(500.0)
    assert line["cpu_baseline"]["cores"] == 3 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
