"""The multi-rank path of bench.py on CPU: two gloo ranks agree on the max
over ranks of their timed regions and on the whole-job value; the reference
arm prints only on rank 0."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        mine = [3.0, 5.0][rank]
        got = bench.max_over_ranks(mine, torch.device("cpu"))
        value = bench.whole_job_value(1000, world, got / 10)
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_sum_the_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [5.0, 5.0]
    # 2 ranks x 1000 token-heads per 0.5 ms step
    assert all(abs(r[2] - 2 * 1000 / 0.5e-3) < 1e-6 * r[2] for r in res)


def test_single_process_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, torch.device("cpu")) == 2.5
    assert bench.whole_job_value(10, 1, 1.0) == pytest.approx(10_000.0)


def test_reference_arm_is_silent_off_rank_zero():
    sys.path.insert(0, ROOT)
    import bench

    class A:
        steps, warmup, seq_len = 1, 0, 4096
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(A(), rank=1, world=2)
    assert buf.getvalue() == ""


def test_reference_arm_prints_the_contract_line_on_rank_zero():
    sys.path.insert(0, ROOT)
    import bench

    class A:
        steps, warmup, seq_len = 1, 0, 131072
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(A(), rank=0, world=1)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
