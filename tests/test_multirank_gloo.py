"""The benchmark's multi-rank logic on CPU: two gloo ranks (no GPU).

Every rank scans its own batch (weak scaling, no data-path collective); the
job's time is the slowest rank's, and the value counts every rank's elements.
The reference arm prints one line from rank 0 only.
"""
import importlib.util
import json
import os
import socket
import subprocess
import sys
from pathlib import Path

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", ROOT / "bench.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _bench()
        bench._WORLD = world
        bench._REDUCE_DEVICE = "cpu"
        local_ms = 10.0 + 5.0 * rank                 # ranks finish at different times
        bench.barrier()
        worst = bench.max_over_ranks(local_ms)
        value = bench.job_gelem_per_s(world, elements_per_rank=1000, steps=4, max_ms=worst)
        Path(out_dir, f"rank{rank}.json").write_text(json.dumps(
            {"worst": worst, "value": value, "seed": bench.rank_seed(rank)}))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    for r in res:
        assert r["worst"] == 15.0                     # the slower rank's 15 ms
        assert r["value"] == pytest.approx(2 * 1000 * 4 / 15e-3 / 1e9)
    assert res[0]["seed"] != res[1]["seed"]           # each rank draws its own inputs


def test_single_rank_needs_no_process_group():
    bench = _bench()
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_gelem_per_s(1, 10**9, 1, 1000.0) == pytest.approx(1.0)


def test_reference_arm_prints_once_under_torchrun():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           str(ROOT / "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "2",
           "--warmup", "3", "--reference-seconds", "2"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
