"""The N > 1 path of bench.py on CPU: world size 2 over gloo.

The hot path does not shard (replicas only): the ranks share nothing but the
barrier and the max-over-ranks time reduction, and the reference arm runs on
rank 0 alone while the other ranks exit 0 without work."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world),
                       "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_setup()
    try:
        assert (w, r) == (world, rank)
        assert torch.distributed.get_backend() == "gloo"
        bench.barrier(w)
        out[rank] = bench.dist_max(1.5 + rank, w)
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="checks the host-only (gloo) launch")
def test_dist_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2,
                           join=True, start_method="spawn")
        assert dict(out) == {0: 2.5, 1: 2.5}


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="checks the host-only (gloo) launch")
def test_reference_arm_under_torchrun_world2():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
           "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "1",
           "--workload", "fmt_a_small", "--ref-seconds", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["unit"] == "GB/s"
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_default_workload_line():
    # the default workload's reference arm (the oracle as it stands, on host
    # cores) prints one JSON line with the keys of the bench contract
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
           "--warmup", "1", "--ref-seconds", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps",
                "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline",
                "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["n_gpus"] == 1
    assert line["config"]["workload"].startswith("decode_step")
    assert line["higher_is_better"] is True and line["unit"] == "GB/s"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
