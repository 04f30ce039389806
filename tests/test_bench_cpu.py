"""Host logic of bench.py that needs no GPU: the multi-rank reduction (gloo,
world size 2, on CPU), the whole-job rate, and the reference arm's rank and
output contract."""
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


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (r + 1) * 1.5 ms: every rank must see the slowest rank's time
        ms = bench.max_over_ranks((rank + 1) * 1.5, "cpu")
        rate = bench.whole_job_rate(1e9, 10, ms, world)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"ms": ms, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["ms"] == pytest.approx(3.0)
        # 2 ranks x 1 GB x 10 steps over 3 ms
        assert r["rate"] == pytest.approx(2 * 1e9 * 10 / 3e-3 / 1e9)


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(2.5, "cpu") == 2.5
    assert bench.whole_job_rate(2e9, 4, 8.0, 1) == pytest.approx(1000.0)


def _run_bench(env_extra, *args):
    env = dict(os.environ)
    env.update(env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_only_rank0_reports():
    r1 = _run_bench({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, "--impl", "reference", "--steps", "3",
                    "--warmup", "3", "--ref-seconds", "2")
    assert r1.returncode == 0, r1.stderr
    assert r1.stdout.strip() == ""
    r0 = _run_bench({"RANK": "0", "WORLD_SIZE": "2", "LOCAL_RANK": "0"}, "--impl", "reference", "--steps", "3",
                    "--warmup", "3", "--ref-seconds", "2")
    assert r0.returncode == 0, r0.stderr
    lines = [ln for ln in r0.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 3 and d["warmup"] == 3
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "decode_hidden5120_m1"


def test_bench_refuses_short_warmup():
    r = _run_bench({}, "--impl", "reference", "--steps", "3", "--warmup", "2")
    assert r.returncode != 0
