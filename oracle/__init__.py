"""ctypes binding of the CPU oracle (oracle/skv_oracle.c).

TEST INFRASTRUCTURE.  Only tests/, ``__graft_entry__.smoke()`` and the
cpu_baseline / reference legs of ``bench.py`` may import this module.  The
product path never imports it and shares no code with it.

The shared library is built from ``skv_oracle.c`` with gcc (fp64, OpenMP,
``-ffp-contract=off``) on first use when it is missing or older than the
source; ``__graft_entry__.build()`` builds it too.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "skv_oracle.c")
_LIB = os.path.join(_HERE, "libskv_oracle.so")

TIER_T0, TIER_T1, TIER_T2, TIER_DROP = 0, 1, 2, 3
OK, ERR_ARG, ERR_BUDGET, ERR_POOL = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile the oracle library in place; returns its path."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
           "-shared", "-std=gnu11", _SRC, "-o", tmp, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None

_p = C.c_void_p
_i = C.c_int
_i64 = C.c_int64
_u16 = C.c_uint16
_d = C.c_double

_SIGS = {
    "orc_boundaries": (None, [_i, _p, _p]),
    "orc_rho_level": (_d, [_i, _i]),
    "orc_distortion": (None, [_p]),
    "orc_tier_bytes": (_i64, [_i, _i]),
    "orc_kappa": (None, [_i, _p]),
    "orc_norm2": (None, [_p, _i, _p]),
    "orc_rtilde_from_r2": (_u16, [_p]),
    "orc_rtilde": (_u16, [_p, _i]),
    "orc_angle_code": (_i, [_u16, _u16, _i]),
    "orc_rho_code": (_i, [_u16, _u16, _p, _i]),
    "orc_vquant": (None, [_p, _i, _p, _p]),
    "orc_reconstruct": (None, [_p, _i, _i, _p]),
    "orc_logit_codes": (_d, [_p, _p, _i, _i]),
    "orc_logit_recon": (_d, [_p, _p, _i, _i]),
    "orc_logit_variant": (_d, [_p, _p, _i, _i, _i]),
    "orc_allocate": (_i, [_i, _i, _i, _i, _i, _p, _p, _p, _p, _i, _p, _p, _p]),
    "orc_retier": (_i, [_i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p]),
    "orc_page_payload": (_i64, [_i, _i, _i]),
    "orc_page_stride": (_i64, [_i, _i, _i]),
    "orc_pack": (_i, [_i, _i, _i, _i, _i,                     # B Hkv Tmax d P
                      _p, _p, _p, _p,                         # seq_lens K V tier
                      _p, _p, _p, _p,                         # free0..2 free_len
                      _p, _p, _p, _i64,                       # row_of indptr ids cap
                      _p, _p, _p, _p]),                       # pool0..2 pool_slots
    "orc_decode": (_i, [_i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _i, _p, _p, _p, _i]),
    "orc_attention_mass": (_i, [_i, _i, _i, _i, _i, _p, _p, _p, _p, _i, _p]),
    "orc_outlier": (_i, [_p, _i]),
    "orc_set_t1_scheme": (None, [_i]),
    "orc_set_share_grid": (None, [_i]),
    "orc_share_grid": (_i, []),
    "orc_t1_scheme": (_i, []),
    "orc_rho_code3": (_i, [_u16, _u16, _p, _i]),
    "orc_rho_level3": (_d, [_i, _i]),
    "orc_reconstruct_tier": (None, [_p, _i, _i, _p]),
    "orc_logit_grid": (_d, [_p, _p, _i, _i, _i, _p, _p]),
    "orc_outlier_flags": (_i, [_i, _i, _i, _i, _p, _p, _p]),
    "orc_d2h": (_u16, [_d]),
    "orc_h2d": (_d, [_u16]),
    "orc_bf2d": (_d, [_u16]),
    "orc_h2bf": (_u16, [_u16]),
    "orc_set_t0_bf16": (None, [_i]),
    "orc_t0_bf16": (_i, []),
    "orc_threads": (_i, []),
}


def lib():
    global _lib
    if _lib is None:
        L = C.CDLL(build())
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def _u16(a) -> np.ndarray:
    """fp16/bf16 data as a contiguous uint16 numpy array (torch or numpy in)."""
    if hasattr(a, "numpy"):
        import torch
        if a.dtype == torch.float16 or a.dtype == torch.bfloat16:
            a = a.view(torch.int16)
        a = a.contiguous().numpy()
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    return a.view(np.uint16)


# ----------------------------------------------------------------------------
# primitives
# ----------------------------------------------------------------------------

def boundaries(b: int):
    bx = np.empty(1 << b, np.float32)
    by = np.empty(1 << b, np.float32)
    lib().orc_boundaries(b, _ptr(bx), _ptr(by))
    return bx, by


def rho_level(code: int, d: int = 128) -> float:
    return lib().orc_rho_level(code, d)


def distortion() -> np.ndarray:
    c = np.empty(4, np.float64)
    lib().orc_distortion(_ptr(c))
    return c


def tier_bytes(tier: int, d: int = 128) -> int:
    return lib().orc_tier_bytes(tier, d)


def kappa(d: int = 128) -> np.ndarray:
    k = np.empty(3, np.float32)
    lib().orc_kappa(d, _ptr(k))
    return k


def norm2(k16) -> int:
    k = _u16(k16)
    out = np.empty(2, np.uint64)
    lib().orc_norm2(_ptr(k), k.size, _ptr(out))
    return int(out[0]) + (int(out[1]) << 64)


def rtilde(k16) -> int:
    k = _u16(k16)
    return lib().orc_rtilde(_ptr(k), k.size)


def rtilde_from_r2(R2: int) -> int:
    a = np.array([R2 & (2**64 - 1), R2 >> 64], np.uint64)
    return lib().orc_rtilde_from_r2(_ptr(a))


def angle_code(x16: int, y16: int, b: int) -> int:
    return lib().orc_angle_code(int(x16), int(y16), b)


def rho_code(x16: int, y16: int, R2: int, d: int) -> int:
    a = np.array([R2 & (2**64 - 1), R2 >> 64], np.uint64)
    return lib().orc_rho_code(int(x16), int(y16), _ptr(a), d)


def vquant(v16):
    v = _u16(v16)
    codes = np.empty(v.size, np.int8)
    sc = np.empty(1, np.uint16)
    lib().orc_vquant(_ptr(v), v.size, _ptr(codes), _ptr(sc))
    return codes, int(sc[0])


def reconstruct(k16, b: int) -> np.ndarray:
    k = _u16(k16)
    out = np.empty(k.size, np.float64)
    lib().orc_reconstruct(_ptr(k), k.size, b, _ptr(out))
    return out


def logit_codes(q: np.ndarray, k16, b: int) -> float:
    k = _u16(k16)
    q = np.ascontiguousarray(q, np.float64)
    return lib().orc_logit_codes(_ptr(q), _ptr(k), k.size, b)


def logit_recon(q: np.ndarray, k16, b: int) -> float:
    k = _u16(k16)
    q = np.ascontiguousarray(q, np.float64)
    return lib().orc_logit_recon(_ptr(q), _ptr(k), k.size, b)


def logit_variant(q: np.ndarray, k16, b: int, share_mode: int) -> float:
    k = _u16(k16)
    q = np.ascontiguousarray(q, np.float64)
    return lib().orc_logit_variant(_ptr(q), _ptr(k), k.size, b, share_mode)


def d2h(x: float) -> int:
    return lib().orc_d2h(float(x))


def h2d(h: int) -> float:
    return lib().orc_h2d(int(h))


def threads() -> int:
    return lib().orc_threads()


def page_payload(tier: int, P: int, d: int = 128) -> int:
    return lib().orc_page_payload(tier, P, d)


def page_stride(tier: int, P: int, d: int = 128) -> int:
    return lib().orc_page_stride(tier, P, d)


# ----------------------------------------------------------------------------
# whole-workload calls
# ----------------------------------------------------------------------------

class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what} failed with status {code}")
        self.code = code


def allocate(B, Hkv, Tmax, d, P, seq_lens, K, utility, protect, mode, budget, quota,
             check: bool = True):
    """Tier per (seq, kv head, token): uint8 [B][Hkv][Tmax] (3 = dropped)."""
    seq = np.ascontiguousarray(seq_lens, np.int32)
    k = _u16(K)
    u = None if utility is None else np.ascontiguousarray(
        utility.numpy() if hasattr(utility, "numpy") else utility, np.float32)
    pr = None if protect is None else np.ascontiguousarray(
        protect.numpy() if hasattr(protect, "numpy") else protect, np.uint8)
    bud = np.ascontiguousarray(budget, np.int64)
    quo = np.ascontiguousarray(quota, np.int32)
    tier = np.empty((B, Hkv, Tmax), np.uint8)
    rc = lib().orc_allocate(B, Hkv, Tmax, d, P, _ptr(seq), _ptr(k), _ptr(u), _ptr(pr), mode,
                            _ptr(bud), _ptr(quo), _ptr(tier))
    if check and rc != OK:
        raise OracleError(rc, "allocate")
    return (tier, rc) if not check else tier


def retier(B, Hkv, Tmax, d, P, seq_lens, K, utility, tier_in, demote, budget,
           check: bool = True):
    """New tiers of a store whose rows flagged in `demote` (all T0) are
    re-decided under the budget, the other resident tokens keeping their
    tiers: uint8 [B][Hkv][Tmax] (3 = dropped); with check=False also the
    status (ERR_BUDGET: the kept tokens alone exceed the budget)."""
    seq = np.ascontiguousarray(seq_lens, np.int32)
    k = _u16(K)
    u = np.ascontiguousarray(utility.numpy() if hasattr(utility, "numpy") else utility, np.float32)
    tin = np.ascontiguousarray(tier_in, np.uint8)
    dm = np.ascontiguousarray(demote.numpy() if hasattr(demote, "numpy") else demote, np.uint8)
    bud = np.ascontiguousarray(budget, np.int64)
    tier = np.empty((B, Hkv, Tmax), np.uint8)
    rc = lib().orc_retier(B, Hkv, Tmax, d, P, _ptr(seq), _ptr(k), _ptr(u), _ptr(tin), _ptr(dm),
                          _ptr(bud), _ptr(tier))
    if check and rc != OK:
        raise OracleError(rc, "retier")
    return (tier, rc) if not check else tier


def pack(B, Hkv, Tmax, d, P, seq_lens, K, V, tier, free_lists: Sequence[np.ndarray],
         pool_slots: Sequence[int], page_cap: Optional[int] = None, check: bool = True):
    """Page table and page bytes; returns a dict of numpy arrays."""
    seq = np.ascontiguousarray(seq_lens, np.int32)
    k = _u16(K)
    v = _u16(V)
    tr = np.ascontiguousarray(tier, np.uint8)
    fl = [np.ascontiguousarray(f, np.uint32) for f in free_lists]
    flen = np.array([f.size for f in fl], np.int64)
    slots = np.array(pool_slots, np.int64)
    if page_cap is None:
        page_cap = int(sum(pool_slots))
    row_of = np.empty((B, Hkv, Tmax), np.int32)
    indptr = np.empty(B * Hkv + 1, np.int32)
    ids = np.zeros(max(page_cap, 1), np.uint32)
    pools = [np.zeros(int(slots[t]) * page_stride(t, P, d), np.uint8) for t in range(3)]
    rc = lib().orc_pack(B, Hkv, Tmax, d, P, _ptr(seq), _ptr(k), _ptr(v), _ptr(tr),
                        _ptr(fl[0]), _ptr(fl[1]), _ptr(fl[2]), _ptr(flen), _ptr(row_of),
                        _ptr(indptr), _ptr(ids), page_cap, _ptr(pools[0]), _ptr(pools[1]),
                        _ptr(pools[2]), _ptr(slots))
    if check and rc != OK:
        raise OracleError(rc, "pack")
    res = dict(row_of=row_of, page_indptr=indptr, page_ids=ids[: indptr[-1]] if rc == OK else ids,
               pools=pools, status=rc)
    return res


def decode(B, Hq, Hkv, Tmax, d, seq_lens, K, V, tier, q, q_dtype: str,
           units: Optional[np.ndarray] = None):
    """fp64 attention over the resident tokens: (out [B][Hq][d], lse [B][Hq]).
    With ``units`` (int32 [n][2] of (b, hq)), only those rows are computed;
    the others are NaN."""
    seq = np.ascontiguousarray(seq_lens, np.int32)
    k = _u16(K)
    v = _u16(V)
    tr = np.ascontiguousarray(tier, np.uint8)
    qq = _u16(q)
    out = np.full((B, Hq, d), np.nan, np.float64)
    lse = np.full((B, Hq), np.nan, np.float64)
    un = None if units is None else np.ascontiguousarray(units, np.int32)
    n = 0 if un is None else un.shape[0]
    rc = lib().orc_decode(B, Hq, Hkv, Tmax, d, _ptr(seq), _ptr(k), _ptr(v), _ptr(tr), _ptr(qq),
                          1 if q_dtype == "bf16" else 0, _ptr(out), _ptr(lse), _ptr(un), n)
    if rc != OK:
        raise OracleError(rc, "decode")
    return out, lse


def attention_mass(B, Hq, Hkv, Tmax, d, seq_lens, K, tier, q, q_dtype: str) -> np.ndarray:
    """fp64 softmax weight of every resident token, summed over the query
    heads of its kv group: [B][Hkv][Tmax] (0 where not resident)."""
    seq = np.ascontiguousarray(seq_lens, np.int32)
    k = _u16(K)
    tr = np.ascontiguousarray(tier, np.uint8)
    qq = _u16(q)
    mass = np.zeros((B, Hkv, Tmax), np.float64)
    rc = lib().orc_attention_mass(B, Hq, Hkv, Tmax, d, _ptr(seq), _ptr(k), _ptr(tr), _ptr(qq),
                                  1 if q_dtype == "bf16" else 0, _ptr(mass))
    if rc != OK:
        raise OracleError(rc, "attention_mass")
    return mass


def logit_grid(q: np.ndarray, k16, b: int, levels_u=None, thresh_u=None) -> float:
    """Logit of a tier variant: b-bit angles, shares quantised to the levels
    (u = (rho/r) sqrt(d/2) domain) by the ascending thresholds; exact shares
    when levels_u is None."""
    k = _u16(k16)
    q = np.ascontiguousarray(q, np.float64)
    if levels_u is None:
        return lib().orc_logit_grid(_ptr(q), _ptr(k), k.size, b, 0, None, None)
    lv = np.ascontiguousarray(levels_u, np.float64)
    th = np.ascontiguousarray(thresh_u if len(lv) > 1 else [0.0], np.float64)
    assert th.size >= lv.size - 1
    return lib().orc_logit_grid(_ptr(q), _ptr(k), k.size, b, lv.size, _ptr(lv), _ptr(th))


class t1_scheme:
    """Context manager: the oracle's T1 code scheme inside the block (0: 6-bit
    angle + 2-bit share, the pinned scheme; 1: 5-bit angle + 3-bit share)."""

    def __init__(self, scheme: int):
        self.scheme = scheme

    def __enter__(self):
        self.prev = lib().orc_t1_scheme()
        lib().orc_set_t1_scheme(self.scheme)
        return self

    def __exit__(self, *exc):
        lib().orc_set_t1_scheme(self.prev)
        return False


class t0_bf16:
    """Context manager: the oracle's T0 storage format inside the block
    (False: fp16 K and V as given; True: rounded to bf16, the fused T0 /
    bf16 decode path's pages)."""

    def __init__(self, on: bool = True):
        self.on = on

    def __enter__(self):
        self.prev = lib().orc_t0_bf16()
        lib().orc_set_t0_bf16(1 if self.on else 0)
        return self

    def __exit__(self, *exc):
        lib().orc_set_t0_bf16(self.prev)
        return False


class share_grid:
    """Context manager: the oracle's 2-bit share grid inside the block (0: the
    uniform levels 0.5 .. 2.0; 1: the exact Lloyd-Max grid)."""

    def __init__(self, grid: int):
        self.grid = grid

    def __enter__(self):
        self.prev = lib().orc_share_grid()
        lib().orc_set_share_grid(self.grid)
        return self

    def __exit__(self, *exc):
        lib().orc_set_share_grid(self.prev)
        return False


def rho_code3(x16: int, y16: int, R2: int, d: int) -> int:
    a = np.array([R2 & (2**64 - 1), R2 >> 64], np.uint64)
    return lib().orc_rho_code3(int(x16), int(y16), _ptr(a), d)


def rho_level3(code: int, d: int = 128) -> float:
    return lib().orc_rho_level3(code, d)


def reconstruct_tier(k16, tier: int) -> np.ndarray:
    """k^ of a key stored in tier 1 or 2 under the current T1 scheme."""
    k = _u16(k16)
    out = np.empty(k.size, np.float64)
    lib().orc_reconstruct_tier(_ptr(k), k.size, tier, _ptr(out))
    return out


def outlier(k16) -> bool:
    """Whether one pair of the key holds a share beyond twice the share
    grid's top level (u_i = (rho_i / r) sqrt(d/2) > 4)."""
    k = _u16(k16)
    return bool(lib().orc_outlier(_ptr(k), k.size))


def outlier_flags(B, Hkv, Tmax, d, seq_lens, K) -> np.ndarray:
    """uint8 [B][Hkv][Tmax]: outlier() of every resident position, else 0."""
    seq = np.ascontiguousarray(seq_lens, np.int32)
    k = _u16(K)
    flags = np.zeros((B, Hkv, Tmax), np.uint8)
    rc = lib().orc_outlier_flags(B, Hkv, Tmax, d, _ptr(seq), _ptr(k), _ptr(flags))
    if rc != OK:
        raise OracleError(rc, "outlier_flags")
    return flags


def accumulate_utility(utility, mass, seq_lens, gamma: float) -> np.ndarray:
    """The utility update of one decode step, in fp64: u <- gamma u + mass at
    every position t < seq_lens[b] (mass is 0 for dropped tokens), positions
    at or past seq_lens[b] unchanged.  READING: the pages only name an
    "estimated future utility"; accumulated attention mass with a geometric
    decay gamma (gamma = 1: the plain running sum) is the plainest estimator
    that the decode itself supplies."""
    u = np.array(utility, np.float64, copy=True)
    m = np.asarray(mass, np.float64)
    seq = np.asarray(seq_lens)
    for b in range(u.shape[0]):
        T = int(seq[b])
        u[b, :, :T] = gamma * u[b, :, :T] + m[b, :, :T]
    return u


def merge_partials(out_parts, lse_parts):
    """Log-sum-exp merge of R attention partials over disjoint token sets, in
    fp64: out_parts [R][...][d], lse_parts [R][...] -> (out [...][d], lse
    [...]).  With M = max_r lse_r and w_r = exp(lse_r - M):
        out = sum_r w_r out_r / sum_r w_r,   lse = M + log sum_r w_r.
    Softmax over the union of the token sets factors this way because each
    partial's out is its own normalised weighted sum and exp(lse_r) its
    denominator.  Partials with lse = -inf (no resident token) carry no
    weight; when every partial is empty the result is out 0, lse -inf, as the
    decode gives for an empty unit."""
    o = np.asarray(out_parts, np.float64)
    l = np.asarray(lse_parts, np.float64)
    M = l.max(axis=0)
    live = np.isfinite(M)
    Ms = np.where(live, M, 0.0)
    w = np.where(np.isfinite(l), np.exp(l - Ms[None]), 0.0)
    den = w.sum(axis=0)
    out = np.zeros(o.shape[1:], np.float64)
    num = (w[..., None] * np.where(np.isfinite(l)[..., None], o, 0.0)).sum(axis=0)
    out[live] = num[live] / den[live][..., None]
    lse = np.full(l.shape[1:], -np.inf)
    lse[live] = Ms[live] + np.log(den[live])
    return out, lse


def run_workload(w, units=None, do_decode=True):
    """allocate -> pack -> decode on a workloads.Workload; returns a dict."""
    tier = allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, w.protect,
                    w.mode, w.budget, w.quota)
    packed = pack(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.V, tier, w.free_lists,
                  w.pool_slots)
    res = dict(tier=tier, **packed)
    if do_decode:
        out, lse = decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q,
                          w.q_dtype, units)
        res.update(out=out, lse=lse)
    return res
