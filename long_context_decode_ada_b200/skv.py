"""ctypes binding of libskv (include/skv.h) for PyTorch callers.

Argument marshalling only: tensors become ``data_ptr()``s, the stream is
``torch.cuda.current_stream()``, status codes become ``SkvError``.  Every step
of the decode path runs in the CUDA kernels of ``libskv.so``; there is no
CPU or PyTorch fallback, and calling into this module without the library
raises.

``PagedCache`` owns the device buffers of one paged store (three tier pools,
page table, tiers, row map) and wraps the allocate -> encode -> decode calls.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import List, Optional, Sequence

import numpy as np
import torch

from . import build as _build

SKV_OK, SKV_ERR_ARG, SKV_ERR_BUDGET, SKV_ERR_POOL, SKV_ERR_CORRUPT, SKV_ERR_CUDA, \
    SKV_ERR_TIMEOUT = range(7)
TIER_T0, TIER_T1, TIER_T2, TIER_DROP = range(4)
MODE_QUOTA, MODE_BUDGET = 0, 1
Q_FP16, Q_BF16 = 0, 1
WS_ALLOCATE, WS_DECODE, WS_DENSE_DECODE, WS_APPEND, WS_DECODE_UTILITY = 0, 1, 2, 3, 4
TABLE_BOUNDARY6_X, TABLE_BOUNDARY6_Y, TABLE_BOUNDARY4_X, TABLE_BOUNDARY4_Y, TABLE_KAPPA, \
    TABLE_RHO_LEVELS, TABLE_BOUNDARY5_X, TABLE_BOUNDARY5_Y = range(8)

EXPORTS = [
    "skv_create", "skv_destroy", "skv_last_error", "skv_page_bytes", "skv_tables",
    "skv_device_info", "skv_workspace_size", "skv_allocate", "skv_encode", "skv_append",
    "skv_retier", "skv_retier_workspace_size",
    "skv_decode_attention", "skv_decode_attention_static", "skv_decode_attention_host",
    "skv_decode_attention_host_pipelined", "skv_decode_attention_host_drain",
    "skv_decode_utility", "skv_merge_partials",
    "skv_dense_pack_bf16",
    "skv_dense_decode_bf16",
    "skv_set_profile_event", "skv_set_wait_limit", "skv_check",
]


class SkvConfig(C.Structure):
    _fields_ = [("head_dim", C.c_int32), ("page_size", C.c_int32),
                ("outlier_protect", C.c_int32), ("t1_angle_bits", C.c_int32),
                ("share_grid", C.c_int32), ("deterministic", C.c_int32),
                ("t0_bf16", C.c_int32), ("reserved", C.c_int32 * 1)]


class SkvPools(C.Structure):
    _fields_ = [("base", C.c_void_p * 3), ("slots", C.c_int64 * 3)]


class SkvFreeLists(C.Structure):
    _fields_ = [("ids", C.c_void_p * 3), ("len", C.c_int64 * 3)]


_p, _i, _i64, _sz = C.c_void_p, C.c_int, C.c_int64, C.c_size_t
_SIGS = {
    "skv_create": (_i, [C.POINTER(SkvConfig), C.POINTER(_p)]),
    "skv_destroy": (_i, [_p]),
    "skv_last_error": (C.c_char_p, []),
    "skv_page_bytes": (_i, [_p, _i, C.POINTER(_i64), C.POINTER(_i64)]),
    "skv_tables": (_i, [_p, _i, _p, _i64]),
    "skv_device_info": (_i, [_p, C.POINTER(_i), C.POINTER(_i)]),
    "skv_workspace_size": (_i, [_p, _i, _i, _i, _i, _i64, _i, C.POINTER(_sz)]),
    "skv_allocate": (_i, [_p, _p, _i, _i, _i64, _p, _p, _p, _i, _p, _p, C.POINTER(SkvFreeLists),
                          C.POINTER(SkvPools), _p, _p, _p, _p, _p, _i64, _p, _p, _sz, _p]),
    "skv_encode": (_i, [_p, _p, _p, _i, _i, _i64, _p, _p, _p, _p, _p, C.POINTER(SkvPools), _p,
                        _p]),
    "skv_append": (_i, [_p, _p, _p, _i, _i, _i64, _p, _p, _p, _p, _p, _p, _i64, C.POINTER(SkvPools),
                        _p, _i64, _p, _p, _p, _sz, _p]),
    "skv_retier_workspace_size": (_i, [_p, _i, _i, _i64, _i64, C.POINTER(_sz)]),
    "skv_retier": (_i, [_p, _i, _i, _i64, _p, _p, _p, _p, C.POINTER(SkvFreeLists), _p,
                        C.POINTER(SkvPools), _p, _p, _p, _p, _p, _i64, _p, _p, _p, _p, _sz, _p]),
    "skv_decode_attention_host": (_i, [_p, _p, _i, _i, _i, _i, _p, _p, _p, C.POINTER(SkvPools),
                                       _p, _p, _p, _p, _p, _p, _p, _sz, _i, _p]),
    "skv_decode_attention_host_pipelined": (_i, [_p, _p, _i, _i, _i, _i, _p, _p, _p,
                                                 C.POINTER(SkvPools), _p, _p, _p, _p, _sz, _i,
                                                 _p]),
    "skv_decode_attention_host_drain": (_i, [_p]),
    "skv_merge_partials": (_i, [_p, _i, _i64, _p, _p, _i64, _p, _p, _p]),
    "skv_decode_utility": (_i, [_p, _p, _i, _i, _i, _i, _p, _p, _p, _i64, C.POINTER(SkvPools),
                                _i64, _p, _p, _p, C.c_float, _p, _p, _p, _p, _p, _sz, _i, _p]),
    "skv_decode_attention": (_i, [_p, _p, _i, _i, _i, _i, _p, _p, _p, C.POINTER(SkvPools), _p, _p,
                                  _p, _p, _sz, _i, _p]),
    "skv_decode_attention_static": (_i, [_p, _p, _i, _i, _i, _i, _p, _p, _p,
                                         C.POINTER(SkvPools), _p, _p, _p, _i, _p]),
    "skv_dense_pack_bf16": (_i, [_p, _p, _p, _i, _i, _i64, _p, _p, _i64, _p, _i64, _p, _p, _i64,
                                 _p, _p, _sz, _p]),
    "skv_dense_decode_bf16": (_i, [_p, _p, _i, _i, _i, _i, _p, _p, _p, _i64, _p, _p, _p, _p, _sz,
                                   _i, _p]),
    "skv_set_profile_event": (_i, [_p, _p]),
    "skv_set_wait_limit": (_i, [_p, _i64]),
    "skv_check": (_i, [_p, _p, _p]),
}

_lib = None


def lib_path() -> str:
    return _build.LIB


def lib():
    """Load libskv.so (building it with nvcc when it is missing or stale)."""
    global _lib
    if _lib is None:
        path = _build.LIB
        if not _build.up_to_date():
            path = _build.build()
        if not os.path.exists(path):
            raise RuntimeError("libskv.so is missing and could not be built")
        L = C.CDLL(path)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


class SkvError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libskv error {code}: {msg}")
        self.code = code


def _check(rc: int):
    if rc != SKV_OK:
        raise SkvError(rc, lib().skv_last_error().decode(errors="replace"))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return C.c_void_p(t.data_ptr())


def _expect(t: torch.Tensor, name: str, numel: int, elem_size: int,
            dtype: Optional[torch.dtype] = None, cuda: bool = True):
    """Argument check before a pointer crosses the C-ABI (which cannot see
    shapes): device, contiguity, element size or dtype, and element count."""
    if not isinstance(t, torch.Tensor):
        raise SkvError(SKV_ERR_ARG, f"{name}: a tensor is required")
    if cuda and not t.is_cuda:
        raise SkvError(SKV_ERR_ARG, f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise SkvError(SKV_ERR_ARG, f"{name}: must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise SkvError(SKV_ERR_ARG, f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.element_size() != elem_size:
        raise SkvError(SKV_ERR_ARG, f"{name}: {t.element_size()}-byte elements, expected {elem_size}")
    if t.numel() != numel:
        raise SkvError(SKV_ERR_ARG, f"{name}: {t.numel()} elements, expected {numel}")


def _decode_buffers(B: int, Hq: int, d: int, q, out, lse, device):
    """The decode's q check and its out / lse, allocated or checked."""
    _expect(q, "q", B * Hq * d, 2)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=device)
    _expect(out, "out", B * Hq * d, 4, torch.float32)
    _expect(lse, "lse", B * Hq, 4, torch.float32)
    return out, lse


def _check_ingest(B: int, Hkv: int, Tmax: int, d: int, K=None, V=None, seq_lens=None,
                  utility=None, protect=None, budget=None, quota=None, cuda: bool = True):
    """The allocate / encode inputs that are given: K, V fp16 [B][Hkv][Tmax][d],
    seq_lens int32 [B], utility fp32 and protect uint8 [B][Hkv][Tmax], budget
    int64 [B], quota int32 [B][3]."""
    n = B * Hkv * Tmax
    if K is not None:
        _expect(K, "K", n * d, 2, cuda=cuda)
    if V is not None:
        _expect(V, "V", n * d, 2, cuda=cuda)
    if seq_lens is not None:
        _expect(seq_lens, "seq_lens", B, 4, torch.int32, cuda=cuda)
    if utility is not None:
        _expect(utility, "utility", n, 4, torch.float32, cuda=cuda)
    if protect is not None:
        _expect(protect, "protect", n, 1, cuda=cuda)
    if budget is not None:
        _expect(budget, "budget", B, 8, torch.int64, cuda=cuda)
    if quota is not None:
        _expect(quota, "quota", 3 * B, 4, torch.int32, cuda=cuda)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


class Context:
    """An skv_ctx: head_dim 128, page size P; bound to the current device."""

    def __init__(self, page_size: int, head_dim: int = 128, outlier_protect: bool = False,
                 t1_angle_bits: int = 6, share_grid: int = 0, deterministic: bool = False,
                 t0_bf16: bool = False):
        cfg = SkvConfig(head_dim=head_dim, page_size=page_size,
                        outlier_protect=1 if outlier_protect else 0, t1_angle_bits=t1_angle_bits,
                        share_grid=share_grid, deterministic=1 if deterministic else 0,
                        t0_bf16=1 if t0_bf16 else 0)
        h = C.c_void_p()
        _check(lib().skv_create(C.byref(cfg), C.byref(h)))
        self._h = h
        self.P = page_size
        self.d = head_dim
        self.outlier_protect = bool(outlier_protect)
        self.t1_angle_bits = t1_angle_bits
        self.share_grid = share_grid
        self.deterministic = bool(deterministic)
        self.t0_bf16 = bool(t0_bf16)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and _lib is not None:
            _lib.skv_destroy(h)
            self._h = None

    @property
    def handle(self):
        return self._h

    def page_bytes(self, tier: int):
        pay, st = C.c_int64(), C.c_int64()
        _check(lib().skv_page_bytes(self._h, tier, C.byref(pay), C.byref(st)))
        return pay.value, st.value

    def table(self, which: int, n: int) -> np.ndarray:
        out = np.empty(n, np.float32)
        _check(lib().skv_tables(self._h, which, out.ctypes.data_as(C.c_void_p), n))
        return out

    def device_info(self):
        sm, sp = C.c_int(), C.c_int()
        _check(lib().skv_device_info(self._h, C.byref(sm), C.byref(sp)))
        return sm.value, sp.value

    def workspace_size(self, which, B, Hkv, Hq=0, Tmax=0, num_splits=0) -> int:
        n = C.c_size_t()
        _check(lib().skv_workspace_size(self._h, which, B, Hkv, Hq, Tmax, num_splits, C.byref(n)))
        return n.value

    def check(self, err: torch.Tensor, stream=None):
        _check(lib().skv_check(self._h, _ptr(err), _stream(stream)))

    def drain_host_steps(self):
        """Wait for the last pipelined host step and return its status as an
        exception (skv_decode_attention_host_drain)."""
        _check(lib().skv_decode_attention_host_drain(self._h))

    def set_wait_limit(self, cycles: int):
        """SM clocks a decode wait may take before the call ends with
        SKV_ERR_TIMEOUT (0: the default, about one second)."""
        _check(lib().skv_set_wait_limit(self._h, int(cycles)))

    def set_profile_event(self, event: Optional[torch.cuda.Event]):
        """Record `event` between the decode and merge kernels of later calls."""
        self._prof = event
        h = None if event is None else C.c_void_p(event.cuda_event)
        _check(lib().skv_set_profile_event(self._h, h))


def _pools_struct(pools: Sequence[Optional[torch.Tensor]], slots: Sequence[int]) -> SkvPools:
    s = SkvPools()
    for t in range(3):
        s.base[t] = pools[t].data_ptr() if pools[t] is not None and pools[t].numel() else None
        s.slots[t] = int(slots[t])
    return s


class PagedCache:
    """Device buffers of one paged store and the calls that fill and read it."""

    def __init__(self, ctx: Context, B: int, Hkv: int, Tmax: int, pool_slots: Sequence[int],
                 page_cap: Optional[int] = None, device="cuda"):
        self.ctx, self.B, self.Hkv, self.Tmax = ctx, B, Hkv, Tmax
        self.device = torch.device(device)
        self.pool_slots = [int(x) for x in pool_slots]
        self.stride = [ctx.page_bytes(t)[1] for t in range(3)]
        self.payload = [ctx.page_bytes(t)[0] for t in range(3)]
        self.pools = [torch.empty(max(1, self.pool_slots[t]) * self.stride[t], dtype=torch.uint8,
                                  device=self.device) for t in range(3)]
        self.page_cap = int(page_cap if page_cap is not None else sum(self.pool_slots))
        self.tier = torch.empty((B, Hkv, Tmax), dtype=torch.uint8, device=self.device)
        self.row_of = torch.empty((B, Hkv, Tmax), dtype=torch.int32, device=self.device)
        self.page_indptr = torch.zeros(B * Hkv + 1, dtype=torch.int32, device=self.device)
        self.page_tier_indptr = torch.zeros(3 * B * Hkv + 1, dtype=torch.int32, device=self.device)
        # the decode cuts its work by streamed bytes (False: by page count)
        self.split_by_bytes = True
        self.page_ids = torch.zeros(max(1, self.page_cap), dtype=torch.int32, device=self.device)
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self._ws_alloc = torch.empty(ctx.workspace_size(WS_ALLOCATE, B, Hkv, 0, Tmax),
                                     dtype=torch.uint8, device=self.device)
        self._pools_c = _pools_struct(self.pools, self.pool_slots)

    def allocate(self, K, seq_lens, utility, protect, mode, budget, quota, free_lists,
                 stream=None):
        _check_ingest(self.B, self.Hkv, self.Tmax, self.ctx.d, K=K, seq_lens=seq_lens,
                      utility=utility, protect=protect, budget=budget, quota=quota)
        self._cursor = None  # append() / retier() restart after the slots this call takes
        fl = SkvFreeLists()
        self._free = [f.to(self.device, dtype=torch.int32) if isinstance(f, torch.Tensor) else
                      torch.from_numpy(np.asarray(f, np.uint32).view(np.int32)).to(self.device)
                      for f in free_lists]
        for t in range(3):
            fl.ids[t] = self._free[t].data_ptr() if self._free[t].numel() else None
            fl.len[t] = self._free[t].numel()
        self._free_c = fl
        _check(lib().skv_allocate(
            self.ctx.handle, _ptr(K), self.B, self.Hkv, self.Tmax, _ptr(seq_lens), _ptr(utility),
            _ptr(protect), mode, _ptr(budget), _ptr(quota), C.byref(fl), C.byref(self._pools_c),
            _ptr(self.tier), _ptr(self.row_of), _ptr(self.page_indptr),
            _ptr(self.page_tier_indptr), _ptr(self.page_ids),
            self.page_cap, _ptr(self.err), _ptr(self._ws_alloc), self._ws_alloc.numel(),
            _stream(stream)))

    def append(self, K_new, V_new, seq_lens, stream=None):
        """Make the token at position seq_lens[b] of every kv head resident as
        T0 (skv_append) and advance seq_lens.  K_new, V_new: fp16
        [B][Hkv][128].  The T0 free list is the one given to allocate();
        its cursor starts after the slots allocate took."""
        _expect(K_new, "K_new", self.B * self.Hkv * self.ctx.d, 2)
        _expect(V_new, "V_new", self.B * self.Hkv * self.ctx.d, 2)
        _expect(seq_lens, "seq_lens", self.B, 4, torch.int32)
        cursor = self.free_cursor()
        if getattr(self, "_ws_append", None) is None:
            n = self.ctx.workspace_size(WS_APPEND, self.B, self.Hkv, 0, self.page_cap)
            self._ws_append = torch.empty(max(n, 1), dtype=torch.uint8, device=self.device)
        free0 = self._free[0]
        _check(lib().skv_append(
            self.ctx.handle, _ptr(K_new), _ptr(V_new), self.B, self.Hkv, self.Tmax, _ptr(seq_lens),
            _ptr(self.tier), _ptr(self.row_of), _ptr(self.page_indptr), _ptr(self.page_tier_indptr),
            _ptr(self.page_ids), self.page_cap, C.byref(self._pools_c),
            _ptr(free0) if free0.numel() else None, free0.numel(), _ptr(cursor),
            _ptr(self.err), _ptr(self._ws_append), self._ws_append.numel(), _stream(stream)))

    def free_cursor(self) -> torch.Tensor:
        """int32 [3] device: the first unused entry of each tier's free list
        (after the pages allocate() took; advanced by append and retier)."""
        if getattr(self, "_cursor", None) is None:
            tip = self.page_tier_indptr
            U = self.B * self.Hkv
            self._cursor = torch.stack(
                [(tip[t + 1:3 * U + 1:3] - tip[t:3 * U:3]).sum() for t in range(3)]
            ).to(torch.int32)
        return self._cursor

    def retier(self, utility, demote, budget, seq_lens, stream=None):
        """Re-decide the demoted T0 rows under the budget on the store itself
        (skv_retier).  utility fp32 and demote uint8 [B][Hkv][Tmax], budget
        int64 [B], all on the device.  New pages take slots from the free
        lists given to allocate(); returns (released, n_released): the ids
        of the old pages no longer referenced (device int32 [page_cap], the
        first n_released valid) -- valid until the next retier call."""
        _check_ingest(self.B, self.Hkv, self.Tmax, self.ctx.d, seq_lens=seq_lens,
                      utility=utility, budget=budget)
        _expect(demote, "demote", self.B * self.Hkv * self.Tmax, 1)
        cursor = self.free_cursor()
        if getattr(self, "_ws_retier", None) is None:
            n = C.c_size_t()
            _check(lib().skv_retier_workspace_size(self.ctx.handle, self.B, self.Hkv, self.Tmax,
                                                   self.page_cap, C.byref(n)))
            self._ws_retier = torch.empty(max(n.value, 1), dtype=torch.uint8, device=self.device)
            self.released = torch.zeros(max(1, self.page_cap), dtype=torch.int32,
                                         device=self.device)
            self.n_released = torch.zeros(1, dtype=torch.int32, device=self.device)
        _check(lib().skv_retier(
            self.ctx.handle, self.B, self.Hkv, self.Tmax, _ptr(seq_lens), _ptr(utility),
            _ptr(demote), _ptr(budget), C.byref(self._free_c), _ptr(cursor),
            C.byref(self._pools_c), _ptr(self.tier), _ptr(self.row_of), _ptr(self.page_indptr),
            _ptr(self.page_tier_indptr), _ptr(self.page_ids), self.page_cap, _ptr(self.released),
            _ptr(self.n_released), _ptr(self.err), _ptr(self._ws_retier), self._ws_retier.numel(),
            _stream(stream)))
        return self.released, self.n_released

    def encode(self, K, V, seq_lens, stream=None):
        _check_ingest(self.B, self.Hkv, self.Tmax, self.ctx.d, K=K, V=V, seq_lens=seq_lens)
        _check(lib().skv_encode(
            self.ctx.handle, _ptr(K), _ptr(V), self.B, self.Hkv, self.Tmax, _ptr(seq_lens),
            _ptr(self.tier), _ptr(self.row_of), _ptr(self.page_indptr), _ptr(self.page_ids),
            C.byref(self._pools_c), _ptr(self.err), _stream(stream)))

    def workspace(self, Hq: int, num_splits: int = 0) -> torch.Tensor:
        n = self.ctx.workspace_size(WS_DECODE, self.B, self.Hkv, Hq, 0, num_splits)
        return torch.empty(max(n, 1), dtype=torch.uint8, device=self.device)

    def decode(self, q: torch.Tensor, q_dtype: int, Hq: int, out=None, lse=None,
               workspace=None, num_splits: int = 0, stream=None):
        out, lse = _decode_buffers(self.B, Hq, self.ctx.d, q, out, lse, self.device)
        if workspace is None:
            workspace = self.workspace(Hq, num_splits)
        _check(lib().skv_decode_attention(
            self.ctx.handle, _ptr(q), q_dtype, self.B, Hq, self.Hkv, _ptr(self.page_indptr),
            _ptr(self.page_tier_indptr) if self.split_by_bytes else None,
            _ptr(self.page_ids), C.byref(self._pools_c), _ptr(out), _ptr(lse), _ptr(self.err),
            _ptr(workspace), workspace.numel(), num_splits, _stream(stream)))
        return out, lse

    def utility_workspace(self, Hq: int, num_splits: int = 0) -> torch.Tensor:
        n = self.ctx.workspace_size(WS_DECODE_UTILITY, self.B, self.Hkv, Hq, self.page_cap,
                                    num_splits)
        return torch.empty(max(n, 1), dtype=torch.uint8, device=self.device)

    def decode_utility(self, q: torch.Tensor, q_dtype: int, Hq: int, seq_lens: torch.Tensor,
                       utility: torch.Tensor, gamma: float = 1.0, out=None, lse=None,
                       workspace=None, num_splits: int = 0, stream=None):
        """decode() plus the utility update u <- gamma u + attention mass
        (skv_decode_utility); utility is fp32 [B][Hkv][Tmax] on the device."""
        if utility.dtype != torch.float32 or tuple(utility.shape) != (self.B, self.Hkv, self.Tmax) \
                or not utility.is_contiguous():
            raise SkvError(SKV_ERR_ARG, "utility must be contiguous fp32 [B][Hkv][Tmax]")
        out, lse = _decode_buffers(self.B, Hq, self.ctx.d, q, out, lse, self.device)
        if workspace is None:
            workspace = self.utility_workspace(Hq, num_splits)
        _check(lib().skv_decode_utility(
            self.ctx.handle, _ptr(q), q_dtype, self.B, Hq, self.Hkv, _ptr(self.page_indptr),
            _ptr(self.page_tier_indptr) if self.split_by_bytes else None,
            _ptr(self.page_ids), self.page_cap, C.byref(self._pools_c), self.Tmax,
            _ptr(seq_lens), _ptr(self.tier), _ptr(self.row_of), float(gamma), _ptr(utility),
            _ptr(out), _ptr(lse), _ptr(self.err), _ptr(workspace), workspace.numel(), num_splits,
            _stream(stream)))
        return out, lse

    def decode_host(self, q_host: torch.Tensor, q_dtype: int, Hq: int, out_host: torch.Tensor,
                    lse_host: torch.Tensor, scratch, workspace=None, num_splits: int = 0,
                    stream=None):
        """One decode step from host q to host out / lse (skv_decode_attention_host):
        the copies, the decode and the stream synchronisation in one call.
        scratch = (q_dev, out_dev, lse_dev) device tensors; host tensors
        should be pinned.  With lse_host and lse_dev None, out_host / out_dev
        hold B*Hq*129 floats, out then lse, and one copy returns both."""
        q_dev, out_dev, lse_dev = scratch
        packed = lse_host is None and lse_dev is None
        for t, dev_side in ((q_host, False), (out_host, False), (lse_host, False),
                            (q_dev, True), (out_dev, True), (lse_dev, True)):
            if t is None and packed:
                continue
            if t is None or t.is_cuda != dev_side or not t.is_contiguous():
                raise SkvError(SKV_ERR_ARG, "decode_host: host tensors on the host, scratch on "
                                            "the device, all contiguous")
        n = self.B * Hq * self.ctx.d
        for t, name in ((q_host, "q_host"), (q_dev, "q_dev")):
            _expect(t, name, n, 2, cuda=False)
        for t, name in ((out_host, "out_host"), (out_dev, "out_dev")):
            _expect(t, name, n + (self.B * Hq if packed else 0), 4, torch.float32, cuda=False)
        if not packed:
            for t, name in ((lse_host, "lse_host"), (lse_dev, "lse_dev")):
                _expect(t, name, self.B * Hq, 4, torch.float32, cuda=False)
        if workspace is None:
            workspace = self.workspace(Hq, num_splits)
        _check(lib().skv_decode_attention_host(
            self.ctx.handle, _ptr(q_host), q_dtype, self.B, Hq, self.Hkv, _ptr(self.page_indptr),
            _ptr(self.page_tier_indptr) if self.split_by_bytes else None,
            _ptr(self.page_ids), C.byref(self._pools_c), _ptr(q_dev), _ptr(out_dev),
            _ptr(lse_dev), _ptr(out_host), _ptr(lse_host), _ptr(self.err), _ptr(workspace),
            workspace.numel(), num_splits, _stream(stream)))
        return out_host, lse_host

    def decode_host_pipelined(self, q_host: torch.Tensor, q_dtype: int, Hq: int,
                              res_host: torch.Tensor, q_dev: torch.Tensor, res_dev: torch.Tensor,
                              workspace=None, num_splits: int = 0, stream=None):
        """Issue one host step (skv_decode_attention_host_pipelined) and wait
        for the previous one: on return the previous call's res_host holds
        that step's out (B*Hq*128 floats) then lse (B*Hq), and the previous
        step's device error, if any, is raised.  Alternate two (q_host,
        res_host) sets; ctx.drain_host_steps() waits for the last step.
        q_dev holds 2 x B*Hq*128 16-bit values and res_dev 2 x B*Hq*129
        floats (two slots)."""
        n = self.B * Hq * self.ctx.d
        for t, dev_side in ((q_host, False), (res_host, False), (q_dev, True), (res_dev, True)):
            if t.is_cuda != dev_side or not t.is_contiguous():
                raise SkvError(SKV_ERR_ARG, "decode_host_pipelined: host tensors on the host, "
                                            "scratch on the device, all contiguous")
        _expect(q_host, "q_host", n, 2, cuda=False)
        _expect(q_dev, "q_dev", 2 * n, 2, cuda=False)
        _expect(res_host, "res_host", n + self.B * Hq, 4, torch.float32, cuda=False)
        _expect(res_dev, "res_dev", 2 * (n + self.B * Hq), 4, torch.float32, cuda=False)
        if workspace is None:
            workspace = self.workspace(Hq, num_splits)
        _check(lib().skv_decode_attention_host_pipelined(
            self.ctx.handle, _ptr(q_host), q_dtype, self.B, Hq, self.Hkv, _ptr(self.page_indptr),
            _ptr(self.page_tier_indptr) if self.split_by_bytes else None, _ptr(self.page_ids),
            C.byref(self._pools_c), _ptr(q_dev), _ptr(res_dev), _ptr(res_host),
            _ptr(workspace), workspace.numel(), num_splits, _stream(stream)))

    def decode_static(self, q: torch.Tensor, q_dtype: int, Hq: int, out=None, lse=None,
                      num_splits: int = 0, stream=None):
        """decode() with the library's fixed scratch instead of a workspace
        (skv_decode_attention_static: calls must not overlap in time)."""
        out, lse = _decode_buffers(self.B, Hq, self.ctx.d, q, out, lse, self.device)
        _check(lib().skv_decode_attention_static(
            self.ctx.handle, _ptr(q), q_dtype, self.B, Hq, self.Hkv, _ptr(self.page_indptr),
            _ptr(self.page_tier_indptr) if self.split_by_bytes else None,
            _ptr(self.page_ids), C.byref(self._pools_c), _ptr(out), _ptr(lse), _ptr(self.err),
            num_splits, _stream(stream)))
        return out, lse

    def check(self, stream=None):
        self.ctx.check(self.err, stream)

    def page_bytes_of(self, page_id: int) -> torch.Tensor:
        """Payload bytes of one page (a device view)."""
        t, slot = page_id >> 30, page_id & ((1 << 30) - 1)
        return self.pools[t][slot * self.stride[t]: slot * self.stride[t] + self.payload[t]]


class DenseCache:
    """The dense bf16 baseline store: every token kept, bf16 K/V, T0 layout."""

    def __init__(self, ctx: Context, B: int, Hkv: int, Tmax: int, pool_slots: int,
                 device="cuda"):
        self.ctx, self.B, self.Hkv, self.Tmax = ctx, B, Hkv, Tmax
        self.device = torch.device(device)
        self.pool_slots = int(pool_slots)
        self.stride = ctx.page_bytes(4)[1]
        self.pool = torch.empty(max(1, pool_slots) * self.stride, dtype=torch.uint8,
                                device=self.device)
        self.page_cap = self.pool_slots
        self.page_indptr = torch.zeros(B * Hkv + 1, dtype=torch.int32, device=self.device)
        self.page_tier_indptr = torch.zeros(3 * B * Hkv + 1, dtype=torch.int32, device=self.device)
        # the decode cuts its work by streamed bytes (False: by page count)
        self.split_by_bytes = True
        self.page_ids = torch.zeros(max(1, self.page_cap), dtype=torch.int32, device=self.device)
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self._ws_alloc = torch.empty(ctx.workspace_size(WS_ALLOCATE, B, Hkv, 0, Tmax),
                                     dtype=torch.uint8, device=self.device)

    def pack(self, K, V, seq_lens, free_ids: torch.Tensor, stream=None):
        self._free = free_ids.to(self.device, dtype=torch.int32)
        _check(lib().skv_dense_pack_bf16(
            self.ctx.handle, _ptr(K), _ptr(V), self.B, self.Hkv, self.Tmax, _ptr(seq_lens),
            _ptr(self._free), self._free.numel(), _ptr(self.pool), self.pool_slots,
            _ptr(self.page_indptr), _ptr(self.page_ids), self.page_cap, _ptr(self.err),
            _ptr(self._ws_alloc), self._ws_alloc.numel(), _stream(stream)))

    def workspace(self, Hq: int, num_splits: int = 0) -> torch.Tensor:
        n = self.ctx.workspace_size(WS_DENSE_DECODE, self.B, self.Hkv, Hq, 0, num_splits)
        return torch.empty(max(n, 1), dtype=torch.uint8, device=self.device)

    def decode(self, q, q_dtype, Hq, out=None, lse=None, workspace=None, num_splits=0,
               stream=None):
        out, lse = _decode_buffers(self.B, Hq, self.ctx.d, q, out, lse, self.device)
        if workspace is None:
            workspace = self.workspace(Hq, num_splits)
        _check(lib().skv_dense_decode_bf16(
            self.ctx.handle, _ptr(q), q_dtype, self.B, Hq, self.Hkv, _ptr(self.page_indptr),
            _ptr(self.page_ids), _ptr(self.pool), self.pool_slots, _ptr(out), _ptr(lse),
            _ptr(self.err), _ptr(workspace), workspace.numel(), num_splits, _stream(stream)))
        return out, lse

    def check(self, stream=None):
        self.ctx.check(self.err, stream)


def workload_to_device(w, device="cuda"):
    """Host tensors of a workloads.Workload -> a dict of device tensors."""
    dev = torch.device(device)

    def t(x, dtype=None):
        if x is None:
            return None
        if isinstance(x, np.ndarray):
            x = torch.from_numpy(np.ascontiguousarray(x))
        return x.to(dev) if dtype is None else x.to(dev, dtype=dtype)

    q = w.q.view(torch.int16) if w.q.dtype == torch.uint16 else w.q.view(torch.int16)
    return dict(
        K=t(w.K), V=t(w.V), q=t(q), seq_lens=t(w.seq_lens), utility=t(w.utility),
        protect=t(w.protect), budget=t(w.budget), quota=t(w.quota),
        free_lists=[torch.from_numpy(f.view(np.int32)).to(dev) for f in w.free_lists],
        q_dtype=Q_BF16 if w.q_dtype == "bf16" else Q_FP16,
    )


def build_cache(ctx: Context, w, dev: dict, stream=None) -> PagedCache:
    """allocate + encode a workload's store on the device."""
    cache = PagedCache(ctx, w.B, w.Hkv, w.Tmax, w.pool_slots, device=dev["K"].device)
    cache.allocate(dev["K"], dev["seq_lens"], dev["utility"], dev["protect"], w.mode,
                   dev["budget"], dev["quota"], dev["free_lists"], stream=stream)
    cache.encode(dev["K"], dev["V"], dev["seq_lens"], stream=stream)
    return cache
