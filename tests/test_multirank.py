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


def test_gpus_flag_and_rank_count_cannot_disagree():
    """--gpus N is honoured: a torchrun rank whose WORLD_SIZE differs from N
    is an error, N > 1 without a launcher re-runs the command under
    torch.distributed.run with N processes, N = 1 runs in place."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.resolve_launch(1, {}, []) == ("run", 1, 0, 0)
    assert bench.resolve_launch(2, {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"},
                                []) == ("run", 2, 1, 1)
    how = bench.resolve_launch(8, {"WORLD_SIZE": "1"}, [])
    assert how[0] == "error" and "WORLD_SIZE=1" in how[1]
    how = bench.resolve_launch(1, {"WORLD_SIZE": "4", "RANK": "0"}, [])
    assert how[0] == "error"
    assert bench.resolve_launch(0, {}, [])[0] == "error"
    how = bench.resolve_launch(4, {}, ["--gpus", "4", "--steps", "10"])
    assert how[0] == "spawn"
    cmd = how[1]
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "10"]


def test_gpus_flag_mismatch_exits_nonzero_without_work():
    """`bench.py --gpus 8` inside a one-rank launch refuses to run instead of
    printing a line that says n_gpus 1."""
    import subprocess
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "8"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 2
    assert r.stdout == "" and "--gpus 8" in r.stderr
