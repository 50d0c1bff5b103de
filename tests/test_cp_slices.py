"""The host side of the context-parallel decode, on CPU: slice bounds, the
per-rank inputs, and the exchange over two gloo ranks.  Each rank's partial
is the oracle's decode of its slice (allocated from the slice's inputs);
gathered and merged (oracle.merge_partials) it must equal the oracle's
decode over all positions with the slices' tiers side by side."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from long_context_decode_ada_b200 import cp
from long_context_decode_ada_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("T,R,align", [(1000, 3, 16), (64, 8, 16), (131072, 8, 64), (5, 2, 1)])
def test_slice_bounds_partition_the_positions(T, R, align):
    b = [cp.slice_bounds(T, R, r, align) for r in range(R)]
    assert b[0][0] == 0 and b[-1][1] == T
    for (a0, a1), (c0, c1) in zip(b, b[1:]):
        assert a1 == c0 and a0 <= a1
    for a0, a1 in b[:-1]:
        assert a1 % align == 0 or a1 == T
    sizes = [a1 - a0 for a0, a1 in b]
    assert max(sizes) - min(sizes) <= align


def slice_partial(w, R, r):
    ws = cp.slice_workload(w, R, r)
    tier = oracle.allocate(ws.B, ws.Hkv, ws.Tmax, ws.d, ws.P, ws.seq_lens, ws.K, ws.utility,
                           ws.protect, ws.mode, ws.budget, ws.quota)
    out, lse = oracle.decode(ws.B, ws.Hq, ws.Hkv, ws.Tmax, ws.d, ws.seq_lens, ws.K, ws.V, tier,
                             ws.q, ws.q_dtype)
    return ws, tier, out, lse


def union_reference(w, R, tiers):
    full = np.full((w.B, w.Hkv, w.Tmax), 3, np.uint8)
    for r in range(R):
        t0, t1 = cp.slice_bounds(w.Tmax, R, r, w.P)
        full[:, :, t0:t1] = tiers[r][:, :, : t1 - t0]
    return full, oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, full, w.q,
                               w.q_dtype)


def budget_workload():
    lens = [600, 250, 31]
    return wl.custom(31, 3, 2, 4, 16, lens, wl.MODE_BUDGET, protect_sink=8, protect_recent=16,
                     zipf_alpha=1.1,
                     budget=[int(0.4 * T * 2 * 512) + 4 * 2 * 15 * 888 + 24 * 2 * 512
                             for T in lens])


@pytest.mark.parametrize("R", [1, 2, 3])
def test_sliced_decode_merges_to_the_union(R):
    w = budget_workload()
    parts = [slice_partial(w, R, r) for r in range(R)]
    for r, (ws, tier, out, lse) in enumerate(parts):
        t0, t1 = cp.slice_bounds(w.Tmax, R, r, w.P)
        assert ws.Tmax == max(t1 - t0, 1)
        assert np.array_equal(ws.seq_lens, np.clip(w.seq_lens - t0, 0, t1 - t0))
        assert torch.equal(ws.K[:, :, : t1 - t0], w.K[:, :, t0:t1])
        assert torch.equal(ws.q, w.q)
    # the slices' budgets beyond their page-rounding reserves add up to at
    # most the sequence's budget beyond one reserve
    reserve = w.Hkv * (w.P - 1) * (512 + 196 + 180)
    spent = sum(p[0].budget - reserve for p in parts)
    assert np.all(spent <= w.budget - reserve)
    assert np.all(spent >= w.budget - reserve - R)
    full, (ro, rl) = union_reference(w, R, [p[1] for p in parts])
    mo, ml = oracle.merge_partials([p[2] for p in parts], [p[3] for p in parts])
    np.testing.assert_allclose(mo, ro, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(ml, rl, rtol=1e-12, atol=1e-12)


def test_quota_slices_scale_the_tier_counts():
    lens = [320, 100]
    w = wl.custom(32, 2, 2, 2, 16, lens, wl.MODE_QUOTA,
                  quota=[[T // 4, T // 2, T // 8] for T in lens])
    for r in range(2):
        ws = cp.slice_workload(w, 2, r)
        frac = ws.seq_lens / w.seq_lens
        assert np.array_equal(ws.quota, np.floor(w.quota * frac[:, None]).astype(np.int32))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = budget_workload()
        ws, tier, out, lse = slice_partial(w, world, rank)
        n = w.B * w.Hq
        part = torch.cat([torch.from_numpy(out.reshape(-1)), torch.from_numpy(lse.reshape(-1))])
        g = cp.gather_partials(part, None).numpy()
        outs = g[:, : 128 * n].reshape(world, w.B, w.Hq, 128)
        lses = g[:, 128 * n:].reshape(world, w.B, w.Hq)
        mo, ml = oracle.merge_partials(outs, lses)
        q.put((rank, mo, ml, tier))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_and_merge():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = budget_workload()
    full, (ro, rl) = union_reference(w, world, [x[3] for x in res])
    for rank, mo, ml, _ in res:
        np.testing.assert_allclose(mo, ro, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(ml, rl, rtol=1e-12, atol=1e-12)
