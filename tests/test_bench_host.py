"""Host-side logic of bench.py without a GPU: the multi-rank plumbing (2 gloo
ranks on 127.0.0.1), FLOP counting, the traffic table guard and the reference
arm's JSON line."""

import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    bench.barrier(world)
    # each replica reports its own step time; the job's time is the max
    got = bench.max_over_ranks(1.5 + rank, world)
    bench.barrier(world)
    dist.destroy_process_group()
    with open(out + f".{rank}", "w") as f:
        f.write(repr(got))


def test_max_over_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp

    port = _free_port()
    out = str(tmp_path / "r")
    mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True,
                       start_method="spawn")
    for r in range(2):
        assert float(open(out + f".{r}").read()) == 2.5


def test_causal_flop_count_closed_form():
    # causal L x L: L (L + 1) / 2 visible pairs
    assert bench.causal_pairs(4096, 4096, True) == 4096 * 4097 // 2
    assert bench.causal_pairs(100, 300, True) == sum(min(i + 201, 300) for i in range(100))
    assert bench.fwd_flops(bench.FWD) == 4.0 * 128 * (4096 * 4097 // 2) * 4 * 16
    assert bench.bwd_flops(bench.BWD) == 2.5 * 4.0 * 128 * (8192 * 8193 // 2) * 2 * 16


def test_traffic_table_guard(tmp_path, monkeypatch):
    src = tmp_path / "k.cuh"
    src.write_text("kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    table = tmp_path / "traffic.json"
    table.write_text(json.dumps({"k": {"sources": ["k.cuh"],
                                       "sources_sha256": bench.kernel_sources_sha(["k.cuh"]),
                                       "dram_bytes_per_launch": 100.0,
                                       "algorithmic_bytes_per_launch": 50.0}}))
    monkeypatch.setattr(bench, "TRAFFIC_TABLE", str(table))
    assert bench.traffic_per_launch("k") == 100.0
    assert bench.traffic_per_launch("k", 500.0) == 1000.0
    src.write_text("kernel v2")  # counters are stale once the kernel changed
    assert bench.traffic_per_launch("k") is None
    assert bench.traffic_per_launch("missing") is None


def test_reference_arm_json_line():
    env = dict(os.environ, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                       timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["value"] > 0 and line["cpu_baseline"]["cores"] >= 1
