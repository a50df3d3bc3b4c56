"""Host-side logic of bench.py, on CPU: the counted FLOPs, the traffic record, the argument checks
and the max-over-ranks timing reduction over 2 gloo processes."""
import os
import socket
import subprocess
import sys
import tempfile

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_counted_flops_per_token_head():
    # 4 B d + 4 d^2 per token and head: 196,608 at B = 256, d = 128 and 32,768 at B = 64, d = 64
    assert bench.flops_per_token_head(256, 128) == 196608
    assert bench.flops_per_token_head(64, 64) == 32768


def test_traffic_record_names_known_kernels():
    for line in open(bench.TRAFFIC_FILE):
        if line.startswith("#") or not line.strip():
            continue
        kernel, sha, nbytes = line.split()[:3]
        assert kernel in bench.KERNEL_SOURCES, kernel
        assert len(sha) == 16 and int(sha, 16) >= 0
        assert float(nbytes) > 0


def test_warmup_below_three_is_refused():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode != 0 and "warmup" in (r.stderr + r.stdout)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, outdir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    r, local, w, pg = bench.dist_setup(world, backend="gloo")
    try:
        assert (r, local, w) == (rank, rank, world)
        bench.barrier(pg, local)
        slowest = bench.max_over_ranks(pg, 1.5 + rank)
        with open(os.path.join(outdir, f"r{rank}"), "w") as f:
            f.write(repr(slowest))
    finally:
        pg.destroy_process_group()


def test_max_over_ranks_reports_the_slowest_rank():
    world = 2
    with tempfile.TemporaryDirectory() as outdir:
        mp.spawn(_rank, args=(world, _free_port(), outdir), nprocs=world, join=True)
        for r in range(world):
            assert float(open(os.path.join(outdir, f"r{r}")).read()) == 1.5 + (world - 1)


def test_gpu_count_must_match_world(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "0")
    with pytest.raises(SystemExit):
        bench.dist_setup(4, backend="gloo")
