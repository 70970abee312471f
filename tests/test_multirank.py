"""Host-side logic of the multi-rank benchmark, on CPU with the gloo backend.

Each (batch, head) is independent, so N GPUs run N copies of the workload
(weak scaling) with no data-path collective; the only cross-rank steps are the
barriers around the timed region and the max over ranks of the device time.
Those run here as two gloo ranks on 127.0.0.1; the reference arm is launched
the way the driver launches it (torchrun, two ranks) and must print one line.
"""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench
    import workloads as W

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        m = bench.max_over_ranks(1.5 + rank, world)
        w = W.WORKLOADS["sla_b1h2n1024d64"]
        v = bench.job_value(w, world, 2.0)
        bench.barrier(world)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_job_value():
    import torch.multiprocessing as mp

    sys.path.insert(0, ROOT)
    import bench
    import workloads as W

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    w = W.WORKLOADS["sla_b1h2n1024d64"]
    one = bench.job_value(w, 1, 2.0)
    for rank, m, v in res:
        assert m == 2.5  # the slower rank's time on both ranks
        assert v == pytest.approx(2 * one)  # two copies of the workload in one step


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "sla_b1h2n1024d64", "--steps", "1",
           "--warmup", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["n_gpus"] == 2
    assert res["value"] > 0 and res["cpu_baseline"]["kind"] == "oracle"
    assert res["e2e"]["h2d_bytes_per_step"] == 0
