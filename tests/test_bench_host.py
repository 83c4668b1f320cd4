"""Host logic of bench.py: the replica aggregation over ranks (world size 2, gloo, on CPU),
the whole-job rate, and the JSON contract of the CPU reference arm."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        m = bench.max_over_ranks(ms)
        q.put((r, w, lr, m, bench.whole_job_rate(100.0, w, m / 1e3)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rate_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, (r, w, lr, m, rate) in enumerate(got):
        assert (r, w, lr) == (rank, 2, rank)
        assert m == 15.0                               # every rank sees the slowest rank
        assert rate == pytest.approx(100.0 * 2 / 0.015)


def test_single_process_aggregation_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.whole_job_rate(10.0, 1, 2.0) == 5.0


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                         env=env, timeout=600)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "TFLOP/s" and rec["value"] > 0
    assert rec["metric"] == bench.METRIC
    assert rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1"], capture_output=True, text=True, env=env, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_peaks_read_the_measured_file_and_fall_back_on_anything_else(tmp_path):
    good = tmp_path / "good.json"
    good.write_text(json.dumps({"hbm_gbs": 7100.5, "bf16_tflops": 1650, "bf16_tflops_sustained":
                                1420, "clocks": {"sm": 1965}}))
    p = bench._peaks(str(good))
    assert p["source"] == "measured" and p["hbm_gbs"] == 7100.5
    assert p["bf16_tflops"] == 1650.0 and p["bf16_tflops_sustained"] == 1420.0
    no_sustained = tmp_path / "burst_only.json"
    no_sustained.write_text(json.dumps({"hbm_gbs": 7000, "bf16_tflops": 1600}))
    assert bench._peaks(str(no_sustained))["bf16_tflops_sustained"] == 1600.0
    for i, bad in enumerate(['{"hbm_gbs": {"value": 7000}, "bf16_tflops": 1600}',
                             '{"hbm_gbs": "n/a", "bf16_tflops": 1600}',
                             '{"hbm_gbs": 0, "bf16_tflops": 1600}',
                             '{"bf16_tflops": 1600}', '[1, 2]', 'not json']):
        f = tmp_path / f"bad{i}.json"
        f.write_text(bad)
        p = bench._peaks(str(f))
        assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0, bad
    assert bench._peaks(str(tmp_path / "missing.json"))["source"] == "fallback"
