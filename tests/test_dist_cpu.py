"""The multi-process paths of bench.py, on CPU with gloo (world size 2).

The layer shards by (sequence, head) with no data-path collective: each rank
runs its own replica and the only cross-rank steps are a barrier and the
max-over-ranks of the device time.  These tests exercise exactly those steps
and the reference arm's launch under torchrun.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, times, units, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup("gloo")
    assert (w, r) == (ws, rank)
    bench.barrier(w)
    ms = bench.reduce_max(times[rank], w, device="cpu")
    value = bench.aggregate(units, ms, w)
    bench.barrier(w)
    dist.destroy_process_group()
    q.put((rank, ms, value))


def test_replicas_report_the_slowest_rank_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    times = [12.5, 20.0]  # ms of device time per rank
    units = 131072        # tokens per rank
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, units, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, value in res:
        assert ms == max(times)
        assert value == pytest.approx(2 * units / (max(times) / 1e3))


def test_reference_arm_under_torchrun_prints_once():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--gpus", "2",
           "--impl", "reference", "--steps", "1", "--warmup", "0", "--ref-tokens", "256"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["value"] > 0
