"""Host logic of bench.py on CPU: the multi-rank aggregation (world size 2 over gloo), the
reference arm's rank handling, and the reference arm's JSON line."""
import json
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


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # rank r measured (r + 1) * 10 ms for 5 steps; the job's time is the slowest rank's
        ms = bench.max_over_ranks(10.0 * (rank + 1) * 5, world, "cpu")
        rate = bench.whole_job_rate(world, 128, ms / 5)
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
            json.dump({"ms": ms, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_world2_gloo(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(world)]
    for g in got:
        assert g["ms"] == 100.0                       # max of 50 and 100
        assert g["rate"] == pytest.approx(2 * 128 / 0.020)   # both ranks' queries over 20 ms/step


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_rate(1, 64, 2.0) == pytest.approx(32000.0)


def _run_bench(args, env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_on_a_nonzero_rank_exits_without_work():
    r = _run_bench(["--impl", "reference", "--gpus", "2"],
                   {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_line_with_the_contract_keys():
    r = _run_bench(["--impl", "reference", "--workload", "deep64k", "--steps", "1", "--warmup", "0"], {})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["unit"] == "queries/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "queries/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["config"]["workload"] == "deep_64k_C4L6"


def test_traffic_record_hash_ignores_comments_not_code():
    a = "int f(int x) {\n    return x + 1;   // one more\n}\n"
    b = "/* header\n   comment */\nint f(int x) {\n\n    return x + 1;\n}\n"
    c = "int f(int x) {\n    return x + 2;\n}\n"
    assert bench.source_code_sha256(a) == bench.source_code_sha256(b)
    assert bench.source_code_sha256(a) != bench.source_code_sha256(c)
