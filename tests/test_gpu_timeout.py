"""The decode's bounded-wait exit path (skv_set_wait_limit): with a wait
limit far shorter than a page copy takes, the call ends with SKV_ERR_TIMEOUT
in the error word instead of hanging, every CTA lets its page copies land
before it leaves, and the next call with the default limit on the same
context, store and workspace matches the oracle."""
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import skv
from long_context_decode_ada_b200 import workloads as wl
from _gpu import assert_close, run_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("deterministic", [False, True])
def test_short_wait_limit_times_out_and_the_next_call_is_exact(deterministic):
    lens = [3000, 700]
    quota = [[T // 10, T // 2, T // 4] for T in lens]
    w = wl.custom(66, 2, 2, 4, 64, lens, wl.MODE_QUOTA, quota=quota)
    ref = oracle.run_workload(w)
    ctx = skv.Context(w.P, deterministic=deterministic)
    g = run_gpu(w, ctx=ctx, decode=False)
    cache, dev = g["cache"], g["dev"]
    ws = cache.workspace(w.Hq)
    ctx.set_wait_limit(64)   # SM clocks: far below the microsecond a page copy takes
    cache.decode(dev["q"], dev["q_dtype"], w.Hq, workspace=ws)
    with pytest.raises(skv.SkvError) as e:
        cache.check()
    assert e.value.code == skv.SKV_ERR_TIMEOUT
    ctx.set_wait_limit(0)
    for _ in range(2):
        out, lse = cache.decode(dev["q"], dev["q_dtype"], w.Hq, workspace=ws)
        cache.check()
        assert_close(out.cpu().numpy(), ref["out"], "out after a timed-out call")
        assert_close(lse.cpu().numpy(), ref["lse"], "lse after a timed-out call")
    torch.cuda.synchronize()


def test_wait_limit_argument_check():
    ctx = skv.Context(64)
    with pytest.raises(skv.SkvError):
        ctx.set_wait_limit(-1)
    ctx.set_wait_limit(0)
