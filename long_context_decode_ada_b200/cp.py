"""Context-parallel decode over several GPUs (one process per GPU).

Every rank holds a contiguous slice of each sequence's token positions in a
paged store of its own, built by the same allocate + encode from that
slice's keys and values.  One decode step is:

1. the ordinary ADA decode over the local store (skv_decode_attention),
   written into a packed buffer {out [B*Hq][128], lse [B*Hq]};
2. one all-gather of those buffers (padded to an even length) over the
   process group (NCCL over
   NVLink / NVSwitch on GPUs; gloo in the CPU tests);
3. the log-sum-exp merge of the R partials (skv_merge_partials).

The pages fix attention over all resident tokens (SPHERICAL KV, Technical
Summary section 2.1); splitting it into slices and merging them is this
library's multi-GPU layout.  The retention budget is per sequence; under
slicing each rank keeps a page-rounding reserve, pays for its own protected
tokens and takes its unprotected tokens' share of the rest (budget mode), or
the share of the per-head tier counts that its tokens are of the sequence's
(quota mode).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import numpy as np
import torch
import torch.distributed as dist

from . import skv
from . import workloads as wl


def slice_bounds(Tmax: int, R: int, r: int, align: int = 1) -> Tuple[int, int]:
    """Positions [t0, t1) of rank r: R contiguous slices of [0, Tmax), cut
    at multiples of `align` (a page size keeps each slice's pages full)."""
    if not (0 <= r < R):
        raise ValueError("rank out of range")
    units = -(-Tmax // align)
    a, b = (units * r) // R, (units * (r + 1)) // R
    return min(Tmax, a * align), min(Tmax, b * align)


def slice_budget(w: wl.Workload, t0: int, t1: int, lens: np.ndarray) -> np.ndarray:
    """Budget of the slice [t0, t1) of every sequence.  The allocator spends a
    sequence's budget in three parts: a reserve for the partial last page of
    every (head, tier), the protected tokens (always T0) and the rest, which
    the rate-distortion walk fills.  A slice has pages of its own, so it
    keeps a full reserve; it pays for its own protected tokens; and it takes
    the share of the rest that its unprotected tokens are of the sequence's."""
    reserve = w.Hkv * (w.P - 1) * sum(wl._TIER_BYTES)
    budget = np.zeros(w.B, np.int64)
    for b in range(w.B):
        T = int(w.seq_lens[b])
        if w.protect is not None:
            prot_all = int(w.protect[b, :, :T].sum())
            prot = int(w.protect[b, :, t0:min(t1, T)].sum()) if T > t0 else 0
        else:
            prot_all = prot = 0
        unprot_all = w.Hkv * T - prot_all
        unprot = w.Hkv * int(lens[b]) - prot
        rest = int(w.budget[b]) - reserve - wl._TIER_BYTES[0] * prot_all
        share = (rest * unprot) // unprot_all if unprot_all > 0 and rest > 0 else 0
        budget[b] = reserve + wl._TIER_BYTES[0] * prot + share
    return budget


def slice_workload(w: wl.Workload, R: int, r: int, align: Optional[int] = None) -> wl.Workload:
    """The inputs of rank r: positions [t0, t1) of every sequence (K, V,
    utility and protection sliced along the token axis), the sequence
    lengths clipped to the slice, and the budget or quota scaled by the
    slice's share of each sequence.  q is every rank's (the full query)."""
    t0, t1 = slice_bounds(w.Tmax, R, r, align if align is not None else w.P)
    Tr = max(t1 - t0, 1)
    lens = np.clip(np.asarray(w.seq_lens, np.int64) - t0, 0, t1 - t0).astype(np.int32)
    full = np.maximum(np.asarray(w.seq_lens, np.int64), 1)
    frac = lens / full

    def cut(x):
        if x is None:
            return None
        y = torch.zeros((w.B, w.Hkv, Tr) + tuple(x.shape[3:]), dtype=x.dtype)
        y[:, :, : t1 - t0] = x[:, :, t0:t1]
        return y

    budget = slice_budget(w, t0, t1, lens)
    quota = np.floor(np.asarray(w.quota, np.float64) * frac[:, None]).astype(np.int32)
    slots = wl._pool_slots(w.B, w.Hkv, w.P, lens, budget, w.mode, quota)
    free = [np.arange(s, dtype=np.uint32) for s in slots]
    return dataclasses.replace(w, name=f"{w.name}[slice {r}/{R}]", Tmax=Tr, seq_lens=lens,
                               K=cut(w.K), V=cut(w.V), utility=cut(w.utility),
                               protect=cut(w.protect), budget=budget, quota=quota,
                               free_lists=free, pool_slots=slots)


def gather_partials(part: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of every rank's packed partial buffer: [R][len].  Without a
    process group (or with one rank) there is nothing to exchange."""
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return part.view(1, -1)
    R = dist.get_world_size(group)
    out = torch.empty((R, part.numel()), dtype=part.dtype, device=part.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, part, group=group)
    else:
        dist.all_gather(list(out.unbind(0)), part, group=group)
    return out


def packed_len(n: int) -> int:
    """Floats of one rank's packed partial {out [n][128], lse [n]}, rounded
    up to an even count (the merge reads out as float2)."""
    return 129 * n + (n & 1)


def merge_gathered(ctx: skv.Context, gathered: torch.Tensor, n: int, out: torch.Tensor,
                   lse: Optional[torch.Tensor], stream=None):
    """skv_merge_partials over a [R][packed_len(n)] buffer of packed partials."""
    R, stride = gathered.shape
    if stride != packed_len(n) or not gathered.is_contiguous():
        raise ValueError("gathered partials must be contiguous [R][packed_len(n)]")
    base = gathered.reshape(-1)
    skv._check(skv.lib().skv_merge_partials(
        ctx.handle, R, n, skv._ptr(base), skv._ptr(base[128 * n:]), stride, skv._ptr(out),
        skv._ptr(lse), skv._stream(stream)))
    return out, lse


class ContextParallelDecoder:
    """One rank's side of the context-parallel decode of a sliced store."""

    def __init__(self, cache: skv.PagedCache, Hq: int, group=None, num_splits: int = 0):
        self.cache, self.Hq, self.group, self.num_splits = cache, Hq, group, num_splits
        self.n = cache.B * Hq
        dev = cache.device
        self.part = torch.zeros(packed_len(self.n), dtype=torch.float32, device=dev)
        self.local_out = self.part[: 128 * self.n].view(cache.B, Hq, 128)
        self.local_lse = self.part[128 * self.n:].view(cache.B, Hq)
        self.workspace = cache.workspace(Hq, num_splits)
        self.out = torch.empty((cache.B, Hq, 128), dtype=torch.float32, device=dev)
        self.lse = torch.empty((cache.B, Hq), dtype=torch.float32, device=dev)

    def step(self, q: torch.Tensor, q_dtype: int, stream=None):
        self.cache.decode(q, q_dtype, self.Hq, out=self.local_out, lse=self.local_lse,
                          workspace=self.workspace, num_splits=self.num_splits, stream=stream)
        gathered = gather_partials(self.part, self.group)
        return merge_gathered(self.cache.ctx, gathered, self.n, self.out, self.lse, stream)
