"""Host-side logic of bench.py on CPU: max-over-ranks timing with world size 2
(gloo), whole-job aggregation, and the reference arm printing on rank 0 only."""

from __future__ import annotations

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
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    bench.init_dist(world, "gloo")
    local_ms = 100.0 + 50.0 * rank                     # rank 1 is the slow one
    ms = bench.max_over_ranks(local_ms, world)
    bench.barrier(world)
    out[rank] = (ms, bench.aggregate(1e12, ms / 1e3, world))
    import torch.distributed as dist

    dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo_world2():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        ms, val = out[r]
        assert ms == 150.0                              # every rank sees the slowest rank's time
        assert abs(val - 2e12 / 0.150) < 1.0           # all ranks' work over the slowest time


def test_aggregate_single_rank():
    assert bench.aggregate(3.0, 1.5, 1) == 2.0
    assert bench.aggregate(3.0, 0.0, 1) == 0.0


def test_reference_arm_is_silent_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_traffic_summary_is_tied_to_kernel_sources(tmp_path, monkeypatch):
    import hashlib

    srcs = [tmp_path / "a.cuh", tmp_path / "b.cuh"]
    srcs[0].write_text("kernel v1")
    srcs[1].write_text("helpers v1")
    sha = hashlib.sha256(b"kernel v1" + b"helpers v1").hexdigest()
    summ = tmp_path / "t.md"
    summ.write_text("traffic_bytes_per_launch: 1.5e6\nkernel_sources_sha256: %s\n" % sha)
    monkeypatch.setattr(bench, "KERNEL_SRCS", [str(x) for x in srcs])
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(summ))
    assert bench.traffic_per_launch()[0] == 1.5e6
    srcs[1].write_text("helpers v2")          # a change in any source voids the capture
    assert bench.traffic_per_launch()[0] is None

