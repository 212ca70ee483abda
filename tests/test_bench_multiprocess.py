"""The bench's multi-process host logic on CPU: two ranks over gloo.

On the GPU machine `bench.py --gpus N` runs one replica per GPU under torchrun
(NCCL); what is tested here without a GPU is the host side it relies on:
rank discovery from the torchrun environment, the max-over-ranks reduction
of the device-timed numbers, the whole-job (weak scaling) rate, and that the
reference arm works on rank 0 only while the other ranks exit quietly.
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w, r, l = bench.rank_info()
        # rank-dependent "timings": the reduction must return the slowest
        vals = bench.max_over_ranks([10.0 + r, 5.0 - r, 7.5], torch.device("cpu"), w)
        # the reference arm: rank 0 prints one line, the others nothing
        class A:
            workload = "llama3_prefill"; ref_rows = 1; warmup = 0; steps = 1; gpus = w
        buf = io.StringIO()
        with redirect_stdout(buf):
            rc = bench.run_reference(A) if r != 0 else 0
        q.put((r, (w, r, l), vals, rc, buf.getvalue()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_over_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        r, info, vals, rc, printed = q.get(timeout=120)
        out[r] = (info, vals, rc, printed)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        info, vals, rc, printed = out[r]
        assert info == (world, r, r)
        assert vals == [11.0, 5.0, 7.5]          # max over ranks, identical on every rank
    assert out[1][2] == 0 and out[1][3] == ""    # non-zero ranks do no reference work


def test_whole_job_rate_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_rate(1, 1e12, 10, 1000.0)
    assert one == pytest.approx(1e13)
    # N replicas each doing the same steps in the slowest rank's time
    assert bench.whole_job_rate(4, 1e12, 10, 1000.0) == pytest.approx(4e13)


def test_reference_arm_on_rank0_prints_one_json_line(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    # the line's contract does not depend on the size: a small linear keeps
    # the oracle's share of this test to well under a second
    import workloads as wl
    monkeypatch.setattr(bench, "workload_linears",
                        lambda name: [("small", wl.normal((16, 512), 1.0, 0, 3),
                                       wl.normal((256, 512), 0.02, 1, 3))])

    class A:
        workload = "llama3_prefill"; ref_rows = 1; warmup = 0; steps = 1; gpus = 1
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(A) == 0
    lines = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
