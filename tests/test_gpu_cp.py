"""The context-parallel decode on one GPU: R ranks emulated one after
another in one process (their decodes wait on nothing, so nothing needs to
run at the same time), each with the store of its own slice; their packed
partials are stacked as the all-gather would leave them and merged by
skv_merge_partials.  Compared with the oracle: each slice's tiers bit for
bit (the oracle's allocate of the same slice inputs), and the merged out /
lse against the oracle's decode over all positions with the slices' tiers
side by side."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import cp, skv
from long_context_decode_ada_b200 import workloads as wl
from _gpu import assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("R,n", [(1, 32), (2, 7), (7, 64)])
def test_merge_kernel_against_oracle(R, n):
    rng = np.random.default_rng(R * 100 + n)
    out_p = rng.standard_normal((R, n, 128)).astype(np.float32)
    lse_p = (rng.standard_normal((R, n)) * 20).astype(np.float32)
    lse_p[rng.random((R, n)) < 0.2] = -np.inf        # empty partials
    lse_p[:, 0] = -np.inf                            # a row with nothing anywhere
    stride = cp.packed_len(n)
    g = np.full((R, stride), np.nan, np.float32)     # the pad is never read
    g[:, : 128 * n] = out_p.reshape(R, -1)
    g[:, 128 * n: 129 * n] = lse_p
    ctx = skv.Context(16)
    gathered = torch.from_numpy(g).cuda()
    out = torch.empty((n, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty(n, dtype=torch.float32, device="cuda")
    cp.merge_gathered(ctx, gathered, n, out, lse)
    ro, rl = oracle.merge_partials(out_p.astype(np.float64), lse_p.astype(np.float64))
    assert_close(out.cpu().numpy(), ro, "merged out")
    assert_close(lse.cpu().numpy(), rl, "merged lse")
    assert np.all(out.cpu().numpy()[0] == 0) and lse.cpu().numpy()[0] == -np.inf


def emulate_ranks(w, R):
    """Per rank: its slice, the store built from it, the local decode into
    the packed buffer; returns (stacked partials, per-rank oracle tiers)."""
    ctx = skv.Context(w.P)
    parts, tiers = [], []
    for r in range(R):
        ws = cp.slice_workload(w, R, r)
        dev = skv.workload_to_device(ws)
        cache = skv.build_cache(ctx, ws, dev)
        cache.check()
        tier = oracle.allocate(ws.B, ws.Hkv, ws.Tmax, ws.d, ws.P, ws.seq_lens, ws.K,
                               ws.utility, ws.protect, ws.mode, ws.budget, ws.quota)
        assert np.array_equal(cache.tier.cpu().numpy(), tier), f"slice {r}: tiers"
        dec = cp.ContextParallelDecoder(cache, w.Hq)
        cache.decode(dev["q"], dev["q_dtype"], w.Hq, out=dec.local_out, lse=dec.local_lse,
                     workspace=dec.workspace)
        cache.check()
        parts.append(dec.part.clone())
        tiers.append(tier)
        del cache, dev, dec
    return ctx, torch.stack(parts), tiers


def union_tiers(w, R, tiers):
    full = np.full((w.B, w.Hkv, w.Tmax), 3, np.uint8)
    for r in range(R):
        t0, t1 = cp.slice_bounds(w.Tmax, R, r, w.P)
        full[:, :, t0:t1] = tiers[r][:, :, : t1 - t0]
    return full


@pytest.mark.parametrize("R", [2, 4])
def test_context_parallel_small(R):
    lens = [900, 333, 47]
    w = wl.custom(41, 3, 2, 4, 16, lens, wl.MODE_BUDGET, protect_sink=8, protect_recent=16,
                  zipf_alpha=1.1,
                  budget=[int(0.35 * T * 2 * 512) + 4 * 2 * 15 * 888 + 24 * 2 * 512
                          for T in lens])
    ctx, g, tiers = emulate_ranks(w, R)
    n = w.B * w.Hq
    out = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    cp.merge_gathered(ctx, g, n, out, lse)
    full = union_tiers(w, R, tiers)
    ro, rl = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, full, w.q,
                           w.q_dtype)
    assert_close(out.cpu().numpy(), ro, "out")
    assert_close(lse.cpu().numpy(), rl, "lse")


def test_context_parallel_long_context_8_slices():
    """The 128K store cut into 8 slices of 16K positions (8 GPUs' worth),
    sampled rows against the oracle."""
    R = 8
    w = wl.long_context()
    ctx, g, tiers = emulate_ranks(w, R)
    n = w.B * w.Hq
    out = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    cp.merge_gathered(ctx, g, n, out, lse)
    full = union_tiers(w, R, tiers)
    rows = np.array([[0, 0], [0, 5], [0, 17], [0, 31]], np.int32)
    ro, rl = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, full, w.q,
                           w.q_dtype, units=rows)
    b, h = rows[:, 0], rows[:, 1]
    assert_close(out.cpu().numpy()[b, h], ro[b, h], "out (sampled rows)")
    assert_close(lse.cpu().numpy()[b, h], rl[b, h], "lse (sampled rows)")


def test_decoder_step_through_a_one_rank_nccl_group():
    """ContextParallelDecoder.step end to end (local decode, NCCL all-gather,
    merge) in a process group of one GPU: the result is the local decode."""
    import os
    import socket
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1)
    try:
        lens = [300, 120]
        w = wl.custom(42, 2, 2, 4, 16, lens, wl.MODE_QUOTA,
                      quota=[[T // 4, T // 2, T // 8] for T in lens])
        ctx = skv.Context(w.P)
        dev = skv.workload_to_device(w)
        cache = skv.build_cache(ctx, w, dev)
        dec = cp.ContextParallelDecoder(cache, w.Hq)
        out, lse = dec.step(dev["q"], dev["q_dtype"])
        torch.cuda.synchronize()
        cache.check()
        o2, l2 = cache.decode(dev["q"], dev["q_dtype"], w.Hq)
        assert torch.equal(out, o2) and torch.equal(lse, l2)
    finally:
        dist.destroy_process_group()
