"""skv_decode_attention_host (one decode step from and to host memory)
against the device-buffer decode and the oracle, and its error path: a
device error reported by the step comes back as the call's status."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import skv
from long_context_decode_ada_b200 import workloads as wl
from _gpu import assert_close, run_gpu

pytestmark = pytest.mark.gpu


def host_buffers(w, dev, pinned=True, adjacent=False):
    """With adjacent=True lse follows out in one buffer on each side (the
    packed form, one result copy)."""
    pin = (lambda t: t.pin_memory()) if pinned else (lambda t: t)
    q_host = pin(dev["q"].cpu())
    n = w.B * w.Hq
    d = dev["q"].device
    if adjacent:   # packed: out then lse in one buffer on each side
        out_host = pin(torch.empty(n * 129, dtype=torch.float32))
        scratch = (torch.empty_like(dev["q"]), torch.empty(n * 129, dtype=torch.float32, device=d),
                   None)
        lse_host = None
    else:
        out_host = pin(torch.empty((w.B, w.Hq, 128), dtype=torch.float32))
        lse_host = pin(torch.empty((w.B, w.Hq), dtype=torch.float32))
        scratch = (torch.empty_like(dev["q"]),
                   torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device=d),
                   torch.empty((w.B, w.Hq), dtype=torch.float32, device=d))
    return q_host, out_host, lse_host, scratch


@pytest.mark.parametrize("q_dtype,pinned,adjacent", [("bf16", True, False), ("fp16", True, False),
                                                     ("bf16", False, False), ("bf16", True, True),
                                                     ("fp16", False, True)])
def test_host_step_equals_device_decode_and_oracle(q_dtype, pinned, adjacent):
    # pageable host buffers work too (the copies are then synchronous); out
    # and lse packed in one buffer come back in one copy
    lens = [600, 77, 1]
    w = wl.custom(95, 3, 2, 4, 16, lens, wl.MODE_QUOTA,
                  quota=[[100, 300, 150], [10, 30, 20], [1, 0, 0]], q_dtype=q_dtype)
    g = run_gpu(w)
    cache, dev = g["cache"], g["dev"]
    q_host, out_host, lse_host, scratch = host_buffers(w, dev, pinned, adjacent)
    cache.decode_host(q_host, dev["q_dtype"], w.Hq, out_host, lse_host, scratch)
    if adjacent:
        n = w.B * w.Hq
        out_host, lse_host = out_host[:n * 128].view(w.B, w.Hq, 128), out_host[n * 128:].view(w.B, w.Hq)
    assert np.array_equal(out_host.numpy(), g["out"])
    assert np.array_equal(lse_host.numpy(), g["lse"])
    ref = oracle.run_workload(w)
    assert_close(out_host.numpy(), ref["out"], "out")
    assert_close(lse_host.numpy(), ref["lse"], "lse")


def test_host_step_returns_the_device_error_and_resets_it():
    w = wl.custom(96, 1, 1, 4, 16, [100], wl.MODE_QUOTA, quota=[[10, 50, 40]])
    g = run_gpu(w, decode=False)
    cache, dev = g["cache"], g["dev"]
    q_host, out_host, lse_host, scratch = host_buffers(w, dev)
    good = int(cache.page_ids[2])
    cache.page_ids[2] = (1 << 30) | (cache.pool_slots[1] + 5)   # slot out of range
    with pytest.raises(skv.SkvError) as e:
        cache.decode_host(q_host, dev["q_dtype"], w.Hq, out_host, lse_host, scratch)
    assert e.value.code == skv.SKV_ERR_CORRUPT
    cache.page_ids[2] = good
    cache.decode_host(q_host, dev["q_dtype"], w.Hq, out_host, lse_host, scratch)
    cache.check()


def test_host_step_rejects_device_tensors_as_host_buffers():
    w = wl.custom(97, 1, 1, 4, 16, [40], wl.MODE_QUOTA, quota=[[10, 10, 10]])
    g = run_gpu(w, decode=False)
    cache, dev = g["cache"], g["dev"]
    q_host, out_host, lse_host, scratch = host_buffers(w, dev)
    with pytest.raises(skv.SkvError):
        cache.decode_host(dev["q"], dev["q_dtype"], w.Hq, out_host, lse_host, scratch)


def test_repeated_host_steps_on_a_side_stream_use_the_current_buffers():
    """Repeated calls with the same buffers on a stream of their own: every
    call decodes the q that is in the host buffer at that moment, and a
    device error comes back as the call's status (then the next call is
    clean again)."""
    lens = [700, 333]
    w = wl.custom(98, 2, 2, 4, 16, lens, wl.MODE_QUOTA,
                  quota=[[100, 300, 150], [30, 100, 60]])
    g = run_gpu(w)
    cache, dev = g["cache"], g["dev"]
    q_host, res_host, _, scratch = host_buffers(w, dev, True, adjacent=True)
    n = w.B * w.Hq
    qs = [dev["q"].cpu().clone(), (dev["q"].view(torch.bfloat16) * -0.5).view(torch.int16).cpu()]
    refs = []
    for q in qs:
        wq = wl.custom(98, 2, 2, 4, 16, lens, wl.MODE_QUOTA,
                       quota=[[100, 300, 150], [30, 100, 60]])
        wq.q = q
        refs.append(oracle.run_workload(wq))
    side = torch.cuda.Stream()
    for i in range(7):
        q_host.copy_(qs[i % 2])
        cache.decode_host(q_host, dev["q_dtype"], w.Hq, res_host, None, scratch, stream=side)
        out = res_host[:n * 128].view(w.B, w.Hq, 128).numpy()
        lse = res_host[n * 128:].view(w.B, w.Hq).numpy()
        assert_close(out, refs[i % 2]["out"], f"out, call {i}")
        assert_close(lse, refs[i % 2]["lse"], f"lse, call {i}")
    good = int(cache.page_ids[2])
    cache.page_ids[2] = (1 << 30) | (cache.pool_slots[1] + 5)   # slot out of range
    torch.cuda.synchronize()
    with pytest.raises(skv.SkvError) as e:
        cache.decode_host(q_host, dev["q_dtype"], w.Hq, res_host, None, scratch, stream=side)
    assert e.value.code == skv.SKV_ERR_CORRUPT
    cache.page_ids[2] = good
    torch.cuda.synchronize()
    cache.decode_host(q_host, dev["q_dtype"], w.Hq, res_host, None, scratch, stream=side)
    cache.check()


def test_pipelined_host_steps_return_each_previous_step():
    """skv_decode_attention_host_pipelined: call k issues step k and returns
    step k-1's results in the host buffers of call k-1 (two alternating
    sets; the copies run on the context's own streams, two device slots);
    the drain returns the last step.  A device error of one step is the
    status of the next call; after the drain the next steps are clean."""
    lens = [700, 333]
    quota = [[100, 300, 150], [30, 100, 60]]
    w = wl.custom(99, 2, 2, 4, 16, lens, wl.MODE_QUOTA, quota=quota)
    g = run_gpu(w)
    cache, dev, ctx = g["cache"], g["dev"], g["ctx"]
    n = w.B * w.Hq
    qs = [dev["q"].cpu().clone(), (dev["q"].view(torch.bfloat16) * -0.5).view(torch.int16).cpu()]
    refs = []
    for q in qs:
        wq = wl.custom(99, 2, 2, 4, 16, lens, wl.MODE_QUOTA, quota=quota)
        wq.q = q
        refs.append(oracle.run_workload(wq))
    sets = [(torch.empty_like(qs[0]).pin_memory(), torch.empty(n * 129).pin_memory())
            for _ in range(2)]
    q_dev = torch.empty(2 * n * 128, dtype=dev["q"].dtype, device=dev["q"].device)   # two slots
    res_dev = torch.empty(2 * n * 129, dtype=torch.float32, device=q_dev.device)
    side = torch.cuda.Stream()

    def check(k):
        res = sets[k % 2][1]
        assert_close(res[:n * 128].view(w.B, w.Hq, 128).numpy(), refs[k % 2]["out"], f"out {k}")
        assert_close(res[n * 128:].view(w.B, w.Hq).numpy(), refs[k % 2]["lse"], f"lse {k}")

    for k in range(6):
        qh, rh = sets[k % 2]
        qh.copy_(qs[k % 2])
        cache.decode_host_pipelined(qh, dev["q_dtype"], w.Hq, rh, q_dev, res_dev, stream=side)
        if k > 0:
            check(k - 1)
    ctx.drain_host_steps()
    check(5)
    # a corrupt page id: the first call's step fails, which the second call
    # reports; the drain reports the second step (it saw the same id)
    good = int(cache.page_ids[2])
    torch.cuda.synchronize()
    cache.page_ids[2] = (1 << 30) | (cache.pool_slots[1] + 5)   # slot out of range
    torch.cuda.synchronize()
    for k in range(2):
        qh, rh = sets[k % 2]
        qh.copy_(qs[k % 2])
        if k == 0:
            cache.decode_host_pipelined(qh, dev["q_dtype"], w.Hq, rh, q_dev, res_dev, stream=side)
        else:
            with pytest.raises(skv.SkvError) as e:
                cache.decode_host_pipelined(qh, dev["q_dtype"], w.Hq, rh, q_dev, res_dev,
                                            stream=side)
            assert e.value.code == skv.SKV_ERR_CORRUPT
    with pytest.raises(skv.SkvError) as e:
        ctx.drain_host_steps()
    assert e.value.code == skv.SKV_ERR_CORRUPT
    cache.page_ids[2] = good
    torch.cuda.synchronize()
    qh, rh = sets[0]
    qh.copy_(qs[0])
    cache.decode_host_pipelined(qh, dev["q_dtype"], w.Hq, rh, q_dev, res_dev, stream=side)
    ctx.drain_host_steps()
    check(0)
