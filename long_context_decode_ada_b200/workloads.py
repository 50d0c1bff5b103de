"""Seeded synthetic workloads for the ADA paged decode path.

This module only draws random inputs with the shapes, distributions and
structure of the five decode workloads (tiny all-T2, Llama-3-8B-shaped GQA
layer, 128K long context, ragged serving batch, 32-layer pipeline).  It holds
none of the method's arithmetic: no norms, no codes, no tiers, no attention.
Both the CUDA path and the CPU oracle take their inputs from here.

Every draw uses a ``torch.Generator`` on the CPU seeded from ``(seed, stream)``
so that each tensor is reproducible on its own, independent of draw order and
of thread count.  The recipe functions also take ``device="cuda"``: the same
distributions drawn by a CUDA generator on the GPU (a different random
stream, for timing runs at full size; parity runs draw on the CPU).  bf16 queries are carried as ``uint16`` bit patterns
(round-to-nearest-even from fp32), fp16 tensors as ``float16``.

The workloads stand in for the pages' evaluation (PG-19, LongBench, AgentBench,
ToolBench at 8K-128K contexts on Llama-3.1-8B-class models; SPHERICAL KV,
Technical Summary section 4): those datasets and trained weights are not used.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

D_HEAD = 128

# Tier sizes in bytes per (token, kv head) at d=128; used here only to size
# the page pools generously enough for any allocation under a budget.
_TIER_BYTES = (512, 196, 180)

MODE_QUOTA = 0
MODE_BUDGET = 1


@dataclasses.dataclass
class Workload:
    """One decode layer's worth of synthetic inputs (host tensors)."""

    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    P: int
    Tmax: int
    seq_lens: np.ndarray          # int32 [B]
    K: torch.Tensor               # float16 [B][Hkv][Tmax][d]
    V: torch.Tensor               # float16 [B][Hkv][Tmax][d]
    q: torch.Tensor               # uint16 bf16 bits or float16, [B][Hq][d]
    q_dtype: str                  # "bf16" | "fp16"
    mode: int                     # MODE_QUOTA | MODE_BUDGET
    utility: Optional[torch.Tensor]   # float32 [B][Hkv][Tmax] or None
    protect: Optional[torch.Tensor]   # uint8 [B][Hkv][Tmax] or None
    budget: np.ndarray            # int64 [B] bytes per sequence (budget mode)
    quota: np.ndarray             # int32 [B][3] tokens per head for T0,T1,T2 (quota mode)
    free_lists: List[np.ndarray]  # uint32 slot ids, one array per tier
    pool_slots: List[int]         # slots per tier pool

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


def _gen(seed: int, stream: int, device=None) -> torch.Generator:
    g = torch.Generator(device=device or "cpu")
    g.manual_seed((seed * 1_000_003 + stream * 7_919 + 12_345) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _normal(shape, seed, stream, device=None) -> torch.Tensor:
    return torch.randn(shape, generator=_gen(seed, stream, device), dtype=torch.float32,
                       device=device or "cpu")


def _uniform(shape, seed, stream, device=None) -> torch.Tensor:
    return torch.rand(shape, generator=_gen(seed, stream, device), dtype=torch.float32,
                      device=device or "cpu")


def _perm(n, seed, stream, device=None) -> torch.Tensor:
    return torch.randperm(n, generator=_gen(seed, stream, device), device=device or "cpu")


def to_bf16_bits(x: torch.Tensor) -> torch.Tensor:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even."""
    return x.to(torch.bfloat16).view(torch.int16).view(torch.uint16)


def _pool_slots(B, Hkv, P, seq_lens, budget, mode, quota, slack_pages=1):
    """Slots per tier that any allocation of these inputs can need."""
    slots = []
    for t in range(3):
        tot = 0
        for b in range(B):
            T = int(seq_lens[b])
            all_in_tier = Hkv * (-(-T // P))
            if mode == MODE_QUOTA:
                n = int(quota[b][t])
                need = Hkv * (-(-n // P))
            else:
                need = min(all_in_tier, int(budget[b]) // (P * _TIER_BYTES[t]) + Hkv)
            tot += need + slack_pages
        slots.append(max(tot, 1))
    return slots


def _finish(name, B, Hq, Hkv, P, Tmax, seq_lens, K, V, q, q_dtype, mode, utility,
            protect, budget, quota, seed, scatter):
    slots = _pool_slots(B, Hkv, P, seq_lens, budget, mode, quota)
    free = []
    for t in range(3):
        if scatter:
            free.append(_perm(slots[t], seed, 900 + t).numpy().astype(np.uint32))
        else:
            free.append(np.arange(slots[t], dtype=np.uint32))
    return Workload(name=name, B=B, Hq=Hq, Hkv=Hkv, d=D_HEAD, P=P, Tmax=Tmax,
                    seq_lens=np.asarray(seq_lens, dtype=np.int32), K=K, V=V, q=q,
                    q_dtype=q_dtype, mode=mode, utility=utility, protect=protect,
                    budget=np.asarray(budget, dtype=np.int64),
                    quota=np.asarray(quota, dtype=np.int32).reshape(B, 3),
                    free_lists=free, pool_slots=slots)


def tiny(seed: int = 0, T: int = 4096) -> Workload:
    """Tiny ADA decode: B=1, one KV head and one query head, d=128, P=16,
    every token in tier T2; q, k, v ~ N(0,1) drawn in fp32 then cast to fp16."""
    B, H, P = 1, 1, 16
    K = _normal((B, H, T, D_HEAD), seed, 1).to(torch.float16)
    V = _normal((B, H, T, D_HEAD), seed, 2).to(torch.float16)
    q = _normal((B, H, D_HEAD), seed, 3).to(torch.float16)
    quota = [[0, 0, T]]
    return _finish("tiny_all_t2", B, H, H, P, T, [T], K, V, q, "fp16", MODE_QUOTA,
                   None, None, [0], quota, seed, scatter=False)


def llama_layer(seed: int = 0, B: int = 8, T: int = 32768, Hkv: int = 8, G: int = 4,
                P: int = 64, device=None) -> Workload:
    """Llama-3-8B-shaped decode layer: 32 query / 8 KV heads, d=128, batch 8,
    T=32768, P=64, bf16 q.  K has per-(head, channel) LogNormal(0, 0.5) scales
    times N(0,1); V ~ N(0,1).  Tier quotas 10% T0 / 50% T1 / 25% T2 / 15%
    dropped, ranked by U(0,1) utilities."""
    Hq = Hkv * G
    scale = torch.exp(0.5 * _normal((1, Hkv, 1, D_HEAD), seed, 4, device))
    K = (_normal((B, Hkv, T, D_HEAD), seed, 1, device) * scale).to(torch.float16)
    V = _normal((B, Hkv, T, D_HEAD), seed, 2, device).to(torch.float16)
    q = to_bf16_bits(_normal((B, Hq, D_HEAD), seed, 3, device))
    u = _uniform((B, Hkv, T), seed, 5, device)
    quota = [[int(0.10 * T), int(0.50 * T), int(0.25 * T)] for _ in range(B)]
    return _finish("llama3_8b_layer", B, Hq, Hkv, P, T, [T] * B, K, V, q, "bf16",
                   MODE_QUOTA, u, None, [0] * B, quota, seed, scatter=False)


def zipf_utility(B, Hkv, T, alpha, seed, stream, device=None) -> torch.Tensor:
    """u_t = (1 + pi(t))^-alpha with pi a seeded permutation per (seq, head):
    a Zipf law over positions whose ranks are scattered through the context."""
    u = torch.empty((B, Hkv, T), dtype=torch.float32, device=device or "cpu")
    for b in range(B):
        for h in range(Hkv):
            rank = _perm(T, seed, stream + 1000 * b + h, device).to(torch.float64)
            u[b, h] = torch.pow(1.0 + rank, -alpha).to(torch.float32)
    return u


def long_context(seed: int = 0, T: int = 131072, B: int = 1, Hkv: int = 8, G: int = 4,
                 P: int = 64, budget_frac: float = 0.40, sink: int = 64,
                 recent: int = 1024, device=None) -> Workload:
    """Long-context decode: B=1, 32 query / 8 KV heads, T=131072, P=64.  The
    first 64 and last 1024 tokens are protected (kept dense); the rest are
    allocated under a budget of 40% of the dense fp16 KV bytes, with Zipf(1.1)
    utilities over positions.  K, V, q ~ N(0,1); q in bf16."""
    Hq = Hkv * G
    K = _normal((B, Hkv, T, D_HEAD), seed, 1, device).to(torch.float16)
    V = _normal((B, Hkv, T, D_HEAD), seed, 2, device).to(torch.float16)
    q = to_bf16_bits(_normal((B, Hq, D_HEAD), seed, 3, device))
    u = zipf_utility(B, Hkv, T, 1.1, seed, 10, device)
    prot = torch.zeros((B, Hkv, T), dtype=torch.uint8, device=device or "cpu")
    prot[:, :, :min(sink, T)] = 1
    prot[:, :, max(0, T - recent):] = 1
    budget = [int(math.floor(budget_frac * T * Hkv * 512))] * B
    return _finish("long_context_128k", B, Hq, Hkv, P, T, [T] * B, K, V, q, "bf16",
                   MODE_BUDGET, u, prot, budget, [[0, 0, 0]] * B, seed, scatter=False)


def ragged_batch(seed: int = 0, B: int = 64, Tlo: int = 1024, Thi: int = 8192,
                 Hkv: int = 8, G: int = 4, P: int = 16, device=None) -> Workload:
    """Ragged serving batch: 64 sequences with lengths uniform in [1024, 8192],
    32 query / 8 KV heads, P=16; every free list is a seeded permutation of a
    shared pool so pages are scattered; tiers 20% T0 / 40% T1 / 40% T2 (none
    dropped), ranked by U(0,1) utilities.  K, V, q ~ N(0,1); q in bf16."""
    Hq = Hkv * G
    g = _gen(seed, 6)
    lens = torch.randint(Tlo, Thi + 1, (B,), generator=g).numpy().astype(np.int32)
    Tmax = int(lens.max())
    K = _normal((B, Hkv, Tmax, D_HEAD), seed, 1, device).to(torch.float16)
    V = _normal((B, Hkv, Tmax, D_HEAD), seed, 2, device).to(torch.float16)
    q = to_bf16_bits(_normal((B, Hq, D_HEAD), seed, 3, device))
    u = _uniform((B, Hkv, Tmax), seed, 5, device)
    quota = []
    for b in range(B):
        T = int(lens[b])
        n0, n1 = int(0.2 * T), int(0.4 * T)
        quota.append([n0, n1, T - n0 - n1])
    return _finish("ragged_batch64", B, Hq, Hkv, P, Tmax, lens, K, V, q, "bf16",
                   MODE_QUOTA, u, None, [0] * B, quota, seed, scatter=True)


def pipeline_layer(layer: int, seed: int = 0, B: int = 4, T: int = 65536, Hkv: int = 8,
                   G: int = 4, P: int = 64, budget_frac: float = 0.30,
                   outlier_frac: float = 0.01, outlier_scale: float = 20.0,
                   device=None) -> Workload:
    """One layer of the 32-layer pipeline: B=4, T=65536, 32 query / 8 KV heads.
    K ~ N(0,1) with round(1% of Hkv*d) outlier channels of this layer scaled
    x20 (chosen without replacement, seeded per layer); V ~ N(0,1); a budget
    of 30% of the dense fp16 KV bytes per sequence; Zipf(1.2) utilities with
    an independent position permutation per (seq, head)."""
    Hq = Hkv * G
    s = seed * 97 + layer
    K = _normal((B, Hkv, T, D_HEAD), s, 1, device)
    n_out = int(round(outlier_frac * Hkv * D_HEAD))
    chans = _perm(Hkv * D_HEAD, s, 7)[:n_out]
    for c in chans.tolist():
        K[:, c // D_HEAD, :, c % D_HEAD] *= outlier_scale
    K = K.to(torch.float16)
    V = _normal((B, Hkv, T, D_HEAD), s, 2, device).to(torch.float16)
    q = to_bf16_bits(_normal((B, Hq, D_HEAD), s, 3, device))
    u = zipf_utility(B, Hkv, T, 1.2, s, 20, device)
    budget = [int(math.floor(budget_frac * T * Hkv * 512))] * B
    return _finish(f"pipeline_layer{layer}", B, Hq, Hkv, P, T, [T] * B, K, V, q, "bf16",
                   MODE_BUDGET, u, None, budget, [[0, 0, 0]] * B, s, scatter=False)


def custom(seed: int, B: int, Hkv: int, G: int, P: int, seq_lens, mode: int,
           quota=None, budget=None, protect_sink: int = 0, protect_recent: int = 0,
           q_dtype: str = "bf16", zipf_alpha: Optional[float] = None,
           k_scale: float = 1.0, scatter: bool = False,
           utility: bool = True) -> Workload:
    """Small workloads for tests: N(0,1) K, V, q of any shape and tier policy."""
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    Tmax = max(int(seq_lens.max()) if len(seq_lens) else 0, 1)
    Hq = Hkv * G
    K = (_normal((B, Hkv, Tmax, D_HEAD), seed, 1) * k_scale).to(torch.float16)
    V = _normal((B, Hkv, Tmax, D_HEAD), seed, 2).to(torch.float16)
    qf = _normal((B, Hq, D_HEAD), seed, 3)
    q = to_bf16_bits(qf) if q_dtype == "bf16" else qf.to(torch.float16)
    u = None
    if utility:
        u = (zipf_utility(B, Hkv, Tmax, zipf_alpha, seed, 10) if zipf_alpha
             else _uniform((B, Hkv, Tmax), seed, 5))
    prot = None
    if protect_sink or protect_recent:
        prot = torch.zeros((B, Hkv, Tmax), dtype=torch.uint8)
        for b in range(B):
            T = int(seq_lens[b])
            prot[b, :, :min(protect_sink, T)] = 1
            if protect_recent:
                prot[b, :, max(0, T - protect_recent):T] = 1
    if quota is None:
        quota = [[0, 0, 0]] * B
    if budget is None:
        budget = [0] * B
    return _finish("custom", B, Hq, Hkv, P, Tmax, seq_lens, K, V, q, q_dtype, mode,
                   u, prot, budget, quota, seed, scatter)


CONFIGS = {
    1: tiny,
    2: llama_layer,
    3: long_context,
    4: ragged_batch,
}
