"""skv_decode_attention_static (the library's fixed device scratch, nothing
allocated) against skv_decode_attention (caller workspace) on the same
store, two calls in a row; and its size limit.

This file sorts last so that the static scratch is first used after every
other GPU test has run in the same process (and also works alone)."""
import ctypes as C

import numpy as np
import pytest
import torch

from long_context_decode_ada_b200 import skv
from long_context_decode_ada_b200 import workloads as wl
from _gpu import ATOL, RTOL


def test_static_scratch_rejects_calls_beyond_its_size():
    ctx = skv.Context(16)
    L = skv.lib()
    pools = skv.SkvPools()
    # 200000 x 8 units need far more than the 4 MiB of static scratch; the
    # call is refused on the host before any pointer is used
    rc = L.skv_decode_attention_static(ctx.handle, None, skv.Q_BF16, 200000, 32, 8, None, None,
                                       None, C.byref(pools), None, None, None, 0, None)
    assert rc == skv.SKV_ERR_ARG
    assert b"static scratch" in L.skv_last_error()
    n = ctx.workspace_size(skv.WS_DECODE, 200000, 8, 32, 0, 0)
    assert n > 4 << 20


def _close(a, b, what):
    a = a.cpu().numpy().astype(np.float64)
    b = b.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isfinite(a), np.isfinite(b)), what
    fin = np.isfinite(b)
    assert np.array_equal(a[~fin], b[~fin]), what
    # the same kernel on the same store, within the parity tolerance of the
    # GPU tests: the unit-aligned split hands out its last chunks at run
    # time, so two launches may group rows differently (last-bit changes)
    assert np.all(np.abs(a[fin] - b[fin]) <= ATOL + RTOL * np.abs(b[fin])), what


@pytest.mark.gpu
@pytest.mark.parametrize("splits", [0, 7])
def test_static_scratch_matches_workspace_decode_twice(splits):
    lens = [900, 64, 2500, 17]
    w = wl.custom(64, 4, 2, 4, 64, lens, wl.MODE_QUOTA,
                  quota=[[T // 3, T // 3, T // 6] for T in lens], scatter=True)
    ctx = skv.Context(w.P)
    dev = skv.workload_to_device(w)
    cache = skv.build_cache(ctx, w, dev)
    cache.check()
    ref_out, ref_lse = cache.decode(dev["q"], dev["q_dtype"], w.Hq, num_splits=splits)
    cache.check()
    for call in range(2):
        out, lse = cache.decode_static(dev["q"], dev["q_dtype"], w.Hq, num_splits=splits)
        cache.check()
        _close(out, ref_out, f"out, call {call}")
        _close(lse, ref_lse, f"lse, call {call}")
    torch.cuda.synchronize()
