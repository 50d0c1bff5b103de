"""Pins of the oracle's bf16 T0 storage (oracle.t0_bf16), the format of the
fused T0 / bf16 decode path: SPHERICAL KV technical summary 2.2 makes T0
the top precision tier; this variant keeps T0 keys and values in bf16 (the
dense baseline's element type) instead of fp16.

What fixes it independently of its own code: the fp16 -> bf16 rounding
equals torch's conversion on every finite fp16 bit pattern; the pack's T0
rows read back (documented layout) to torch's bf16 of K and V, and T1 / T2
pages do not change; on an all-T0 store the oracle's attention is the
textbook fp64 attention over torch-rounded bf16 K and V."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import workloads as wl
from test_oracle_rdr_pack import read_row, alloc


def test_rounding_matches_torch_on_every_finite_fp16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = ((bits >> 10) & 31) != 31
    h = torch.from_numpy(bits[finite].view(np.int16)).view(torch.float16)
    ref = h.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.lib().orc_h2bf(int(b)) for b in bits[finite]], np.uint16)
    assert np.array_equal(got, ref)


def test_rounding_ties_go_to_even():
    # 1 + 2^-8 lies halfway between the bf16 neighbours 1 and 1 + 2^-7
    half = np.float16(1.0 + 2.0 ** -8).view(np.uint16)
    assert oracle.lib().orc_h2bf(int(half)) == 0x3F80
    up = np.float16(1.0 + 3 * 2.0 ** -8).view(np.uint16)     # halfway, odd below
    assert oracle.lib().orc_h2bf(int(up)) == 0x3F82


def test_pack_t0_rows_hold_bf16_and_codes_do_not_change():
    P = 16
    w = wl.custom(31, 2, 2, 2, P, [45, 70], wl.MODE_QUOTA,
                  quota=[[7, 20, 11], [16, 33, 17]], scatter=True)
    tier = alloc(w)
    args = (w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.V, tier, w.free_lists, w.pool_slots)
    plain = oracle.pack(*args)
    with oracle.t0_bf16():
        bf = oracle.pack(*args)
    assert np.array_equal(plain["row_of"], bf["row_of"])
    assert np.array_equal(plain["page_ids"], bf["page_ids"])
    Kb = w.K.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    Vb = w.V.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    n_t0 = 0
    ids = np.asarray(bf["page_ids"], np.uint32)
    for b in range(w.B):
        for h in range(w.Hkv):
            u = b * w.Hkv + h
            for t in range(int(w.seq_lens[b])):
                tr = int(tier[b, h, t])
                if tr == 3:
                    continue
                loc = int(bf["row_of"][b, h, t])
                pid = int(ids[int(bf["page_indptr"][u]) + loc // P])
                slot = pid & ((1 << 30) - 1)
                st, pay = oracle.page_stride(tr, P), oracle.page_payload(tr, P)
                page_bf = bf["pools"][tr][slot * st: slot * st + pay]
                page_pl = plain["pools"][tr][slot * st: slot * st + pay]
                if tr == 0:
                    row = read_row(page_bf, 0, P, loc % P)
                    assert np.array_equal(row["K"], Kb[b, h, t]) and np.array_equal(row["V"], Vb[b, h, t])
                    n_t0 += 1
                else:
                    assert np.array_equal(page_bf, page_pl)
    assert n_t0 > 0


def test_all_t0_attention_is_the_textbook_over_bf16():
    lens = [90, 37]
    w = wl.custom(32, 2, 2, 4, 16, lens, wl.MODE_QUOTA, quota=[[90, 0, 0], [37, 0, 0]], k_scale=3.0)
    tier = np.zeros((w.B, w.Hkv, w.Tmax), np.uint8)
    for b in range(w.B):
        tier[b, :, lens[b]:] = 3
    with oracle.t0_bf16():
        out, lse = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q,
                                 w.q_dtype)
    plain_out, _ = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q,
                                 w.q_dtype)
    Kb = w.K.to(torch.bfloat16).double().numpy()
    Vb = w.V.to(torch.bfloat16).double().numpy()
    q = w.q.view(torch.int16).view(torch.bfloat16).double().numpy()
    G = w.Hq // w.Hkv
    for b in range(w.B):
        for hq in range(w.Hq):
            h = hq // G
            T = lens[b]
            l = Kb[b, h, :T] @ q[b, hq] / np.sqrt(128)
            m = l.max()
            e = np.exp(l - m)
            ref = (e[:, None] * Vb[b, h, :T]).sum(0) / e.sum()
            assert np.allclose(out[b, hq], ref, rtol=1e-12, atol=1e-12)
            assert abs(lse[b, hq] - (m + np.log(e.sum()))) < 1e-11
    # the bf16 store differs from the fp16 one (the switch is live)
    assert not np.allclose(out, plain_out, rtol=1e-6, atol=1e-6)
