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
