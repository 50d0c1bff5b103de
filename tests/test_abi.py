"""The C-ABI library loads and exports every symbol include/skv.h declares;
host-only calls (tables, page geometry, argument checks) work without a GPU.
The host tables are computed independently by the library and by the oracle
and must agree byte for byte."""
import ctypes as C
import os
import re

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import skv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(skv_\w+)\s*\(", src, re.M))
    return names


def test_library_exports_every_declared_symbol():
    L = skv.lib()
    names = declared_symbols()
    assert "skv_decode_attention" in names and "skv_allocate" in names and "skv_encode" in names
    for n in sorted(names):
        assert hasattr(L, n), n
    assert set(skv.EXPORTS) >= names - {n for n in names if n not in skv.EXPORTS}


def test_tables_match_oracle_bytes():
    ctx = skv.Context(64)
    bx6, by6 = oracle.boundaries(6)
    bx4, by4 = oracle.boundaries(4)
    assert ctx.table(skv.TABLE_BOUNDARY6_X, 64).tobytes() == bx6.tobytes()
    assert ctx.table(skv.TABLE_BOUNDARY6_Y, 64).tobytes() == by6.tobytes()
    assert ctx.table(skv.TABLE_BOUNDARY4_X, 16).tobytes() == bx4.tobytes()
    assert ctx.table(skv.TABLE_BOUNDARY4_Y, 16).tobytes() == by4.tobytes()
    assert ctx.table(skv.TABLE_KAPPA, 3).tobytes() == oracle.kappa(128).tobytes()
    lv = ctx.table(skv.TABLE_RHO_LEVELS, 4)
    assert list(lv) == [oracle.rho_level(c, 128) for c in range(4)]
    lm = skv.Context(64, share_grid=1).table(skv.TABLE_RHO_LEVELS, 4)
    with oracle.share_grid(1):
        np.testing.assert_allclose(lm, [oracle.rho_level(c, 128) for c in range(4)], rtol=1e-7)
    bx5, by5 = oracle.boundaries(5)
    assert ctx.table(skv.TABLE_BOUNDARY5_X, 32).tobytes() == bx5.tobytes()
    assert ctx.table(skv.TABLE_BOUNDARY5_Y, 32).tobytes() == by5.tobytes()


def test_t1_angle_bits_and_share_grid_are_checked():
    skv.Context(16, t1_angle_bits=5)
    skv.Context(16, t1_angle_bits=6)
    skv.Context(16, share_grid=1)
    with pytest.raises(skv.SkvError):
        skv.Context(16, t1_angle_bits=4)
    with pytest.raises(skv.SkvError):
        skv.Context(16, share_grid=2)


@pytest.mark.parametrize("P", [16, 32, 64])
def test_page_geometry_matches_oracle(P):
    ctx = skv.Context(P)
    for t in range(3):
        assert ctx.page_bytes(t) == (oracle.page_payload(t, P), oracle.page_stride(t, P))
    assert ctx.page_bytes(4) == ctx.page_bytes(0)


def test_argument_errors_without_gpu():
    L = skv.lib()
    cfg = skv.SkvConfig(head_dim=64, page_size=64)
    h = C.c_void_p()
    assert L.skv_create(C.byref(cfg), C.byref(h)) == skv.SKV_ERR_ARG
    assert b"head_dim" in L.skv_last_error()
    cfg = skv.SkvConfig(head_dim=128, page_size=48)
    assert L.skv_create(C.byref(cfg), C.byref(h)) == skv.SKV_ERR_ARG
    ctx = skv.Context(16)
    with pytest.raises(skv.SkvError) as e:
        ctx.workspace_size(skv.WS_DECODE, 2, 8, 12, 0, 0)   # Hq not a multiple of Hkv
    assert e.value.code == skv.SKV_ERR_ARG
    # decode with G = 8 is refused on the host
    pools = skv.SkvPools()
    rc = L.skv_decode_attention(ctx.handle, None, skv.Q_BF16, 1, 64, 8, None, None, None,
                                C.byref(pools), None, None, None, None, 0, 0, None)
    assert rc == skv.SKV_ERR_ARG
    # unaligned pool base is refused
    pools.base[0] = 64
    pools.slots[0] = 1
    rc = L.skv_decode_attention(ctx.handle, None, skv.Q_BF16, 1, 8, 8, None, None, None,
                                C.byref(pools), None, None, None, None, 0, 0, None)
    assert rc == skv.SKV_ERR_ARG


def test_workspace_sizes():
    ctx = skv.Context(64)
    sm, splits = ctx.device_info()
    def expect(S, U, G):
        # split partials, then each unit's range of runs (two int32), then
        # each unit's chunk counter (one 64-bit word)
        return (S + U) * G * 132 * 4 + 8 * U + 8 * U
    n = ctx.workspace_size(skv.WS_DECODE, 1, 8, 32, 0, 0)
    assert n == expect(splits, 8, 4)
    assert ctx.workspace_size(skv.WS_DECODE, 1, 8, 32, 0, 10) == expect(10, 8, 4)
    assert ctx.workspace_size(skv.WS_DECODE, 3, 3, 6, 0, 10) == expect(10, 9, 2)
    assert ctx.workspace_size(skv.WS_ALLOCATE, 2, 8, 0, 1000) > 2 * 8 * 1000 * 4
    # the utility decode: the decode's scratch rounded up to 256 bytes, then
    # page_cap * P rows x G fp32 logits
    for B, Hkv, Hq, cap in [(1, 8, 32, 1000), (3, 3, 6, 7), (2, 4, 4, 0)]:
        base = ctx.workspace_size(skv.WS_DECODE, B, Hkv, Hq, 0, 10)
        n = ctx.workspace_size(skv.WS_DECODE_UTILITY, B, Hkv, Hq, cap, 10)
        assert n == (base + 255) // 256 * 256 + cap * 64 * (Hq // Hkv) * 4


def test_decode_utility_argument_errors_without_gpu():
    ctx = skv.Context(16)
    pools = skv.SkvPools()
    L = skv.lib()
    # Hq not a multiple of Hkv; then a null utility (refused before any launch)
    rc = L.skv_decode_utility(ctx.handle, None, 0, 1, 6, 4, None, None, None, 10, C.byref(pools),
                              8, None, None, None, 1.0, None, None, None, None, None, 0, 0, None)
    assert rc == skv.SKV_ERR_ARG
    rc = L.skv_decode_utility(ctx.handle, None, 0, 1, 8, 4, None, None, None, 10, C.byref(pools),
                              8, None, None, None, 1.0, None, None, None, None, None, 0, 0, None)
    assert rc == skv.SKV_ERR_ARG
    # B = 0 is a no-op
    rc = L.skv_decode_utility(ctx.handle, None, 0, 0, 8, 4, None, None, None, 10, C.byref(pools),
                              8, None, None, None, 1.0, None, None, None, None, None, 0, 0, None)
    assert rc == skv.SKV_OK


def test_binding_checks_buffers_before_the_c_abi():
    # the C-ABI takes plain pointers; the binding checks what it can see
    q = torch.zeros((2, 8, 128), dtype=torch.float16)
    skv._expect(q, "q", 2 * 8 * 128, 2, cuda=False)
    with pytest.raises(skv.SkvError):
        skv._expect(q, "q", 2 * 8 * 128 + 1, 2, cuda=False)          # wrong count
    with pytest.raises(skv.SkvError):
        skv._expect(q.float(), "q", 2 * 8 * 128, 2, cuda=False)      # wrong element size
    with pytest.raises(skv.SkvError):
        skv._expect(q[:, :, ::2], "q", 2 * 8 * 64, 2, cuda=False)    # not contiguous
    with pytest.raises(skv.SkvError):
        skv._expect(q, "q", 2 * 8 * 128, 2, cuda=True)               # not on the device
    with pytest.raises(skv.SkvError):
        skv._expect(torch.zeros(4, dtype=torch.int32), "lse", 4, 4, torch.float32, cuda=False)


def test_ingest_checks_accept_the_test_workloads():
    # the inputs every GPU test builds (workload_to_device), here on the CPU
    from long_context_decode_ada_b200 import workloads as wl
    cases = [
        wl.custom(81, 1, 2, 4, 16, [200], wl.MODE_BUDGET, protect_sink=150, zipf_alpha=1.1,
                  budget=[150 * 2 * 512]),
        wl.custom(82, 1, 1, 4, 16, [200], wl.MODE_QUOTA, quota=[[0, 200, 0]]),
        wl.custom(93, 4, 2, 1, 16, [0, 40, 1, 77], wl.MODE_QUOTA,
                  quota=[[0, 0, 0], [0, 1, 0], [0, 1, 0], [3, 30, 40]], q_dtype="fp16",
                  utility=False),
    ]
    for w in cases:
        d = skv.workload_to_device(w, "cpu")
        skv._check_ingest(w.B, w.Hkv, w.Tmax, 128, K=d["K"], V=d["V"], seq_lens=d["seq_lens"],
                          utility=d["utility"], protect=d["protect"], budget=d["budget"],
                          quota=d["quota"], cuda=False)
        skv._expect(d["q"], "q", w.B * w.Hq * 128, 2, cuda=False)
        K_new = d["K"][:, :, 0].contiguous()
        skv._expect(K_new, "K_new", w.B * w.Hkv * 128, 2, cuda=False)
    with pytest.raises(skv.SkvError):
        skv._check_ingest(1, 1, 4, 128, seq_lens=torch.zeros(1, dtype=torch.int64), cuda=False)
    with pytest.raises(skv.SkvError):
        skv._check_ingest(1, 1, 4, 128, K=torch.zeros((1, 1, 3, 128), dtype=torch.float16),
                          cuda=False)


def test_retier_and_pipelined_host_step_argument_errors_without_gpu():
    ctx = skv.Context(16)
    pools = skv.SkvPools()
    free = skv.SkvFreeLists()
    L = skv.lib()
    # the re-tiering's workspace: the allocation's plus the old store's copies
    # (tiers, row map, both CSR tables, page ids) and the per-segment words
    n = C.c_size_t()
    assert L.skv_retier_workspace_size(ctx.handle, 2, 4, 1000, 500, C.byref(n)) == skv.SKV_OK
    assert n.value >= ctx.workspace_size(skv.WS_ALLOCATE, 2, 4, 0, 1000) + 8 * 1000 * 5 + 500 * 4
    assert L.skv_retier_workspace_size(ctx.handle, 2, 0, 1000, 500, C.byref(n)) == skv.SKV_ERR_ARG
    # null arguments are refused before any launch
    rc = L.skv_retier(ctx.handle, 1, 1, 16, None, None, None, None, C.byref(free), None,
                      C.byref(pools), None, None, None, None, None, 0, None, None, None, None, 0,
                      None)
    assert rc == skv.SKV_ERR_ARG
    # too many positions for the 32-bit row list
    rc = L.skv_retier(ctx.handle, 1024, 128, 1 << 23, None, None, None, None, C.byref(free), None,
                      C.byref(pools), None, None, None, None, None, 0, None, None, None, None, 0,
                      None)
    assert rc == skv.SKV_ERR_ARG
    # the pipelined host step: B = 0 and null buffers are refused; a drain
    # with nothing in flight is a no-op
    rc = L.skv_decode_attention_host_pipelined(ctx.handle, None, 0, 0, 8, 4, None, None, None,
                                               C.byref(pools), None, None, None, None, 0, 0, None)
    assert rc == skv.SKV_ERR_ARG
    rc = L.skv_decode_attention_host_pipelined(ctx.handle, None, 0, 1, 8, 4, None, None, None,
                                               C.byref(pools), None, None, None, None, 0, 0, None)
    assert rc == skv.SKV_ERR_ARG
    assert L.skv_decode_attention_host_drain(ctx.handle) == skv.SKV_OK
    assert L.skv_decode_attention_host_drain(None) == skv.SKV_ERR_ARG


def test_t0_bf16_refuses_the_code_variants_without_gpu():
    with pytest.raises(skv.SkvError) as e:
        skv.Context(16, t0_bf16=True, t1_angle_bits=5)
    assert e.value.code == skv.SKV_ERR_ARG
    with pytest.raises(skv.SkvError) as e:
        skv.Context(16, t0_bf16=True, share_grid=1)
    assert e.value.code == skv.SKV_ERR_ARG
    assert skv.Context(16, t0_bf16=True).t0_bf16
