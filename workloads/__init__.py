"""Seeded synthetic decode workloads for PRR (speculate-reuse-repair) DSA decoding.

This module is shared by the fp64 oracle's tests and by the CUDA path's tests and
bench.  It holds only input generation: no block scoring, no selection, no EMA and
no attention arithmetic.  Everything it returns is raw bf16 bit patterns (uint16)
or int32 block lists, so neither side can lean on a conversion made here.

Workload shapes follow the long-context decode settings the PRR pages describe
("Predict, Reuse, and Repair: Accelerating Dynamic Sparse Attention for
Long-Context LLM Decoding", method summary and key results): one attention layer,
grouped-query heads, a KV cache split into fixed-size blocks, one token appended
per decode step.  The pages print no sizes; the five configurations below are the
synthetic stand-ins for the long-context benchmarks the pages evaluate on.

Generator recipe
----------------
* q and k on the exact dyadic grid {-8..8}/8 (17 values, uniform), so that every
  product q*k is a multiple of 1/64 and every fp32 block score is exact.
* v ~ N(0, 1) rounded to bf16 (round to nearest even).
* Gaussian configuration: q, k and v all ~ N(0, 1) rounded to bf16.
* Query walk: at every decode step, each channel of each query head is kept with
  probability ``walk_p`` and otherwise redrawn from the same distribution.
* Each decode step appends one fresh k/v token per (sequence, KV head).
* Streams: numpy PCG64 seeded by SeedSequence([seed_of(b), tag, b, ...]) so any
  (sequence, KV head) slice can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "workload", "f32_to_bf16_bits", "bf16_bits_to_f32",
    "kv_prefix", "kv_appended", "queries", "forced_prediction", "forced_kept_count", "rep_offsets",
]

# stream tags (plain integers so SeedSequence accepts them)
_TAG_K0, _TAG_V0, _TAG_KNEW, _TAG_VNEW, _TAG_Q, _TAG_FORCED, _TAG_REP = 11, 12, 13, 14, 15, 16, 17


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int            # batch (sequences)
    Hq: int           # query heads
    Hkv: int          # KV heads
    d: int            # head dim
    N0: int           # context length before the first decode step
    bs: int           # tokens per KV block
    K: int            # top-K blocks selected per (sequence, KV head)
    P: int            # speculation budget (predicted blocks)
    steps: int        # decode steps
    alpha: float      # EMA decay
    qk: str           # "grid" or "gauss"
    walk_p: float     # query channel persistence
    per_seq_seed: bool = False
    seed: int = 0
    forced_overlaps: Optional[Sequence[float]] = None  # forced predictor overlap levels
    selector: str = "group_sum"  # block selector: "group_sum", "group_max" or "per_head"
    n_sink: int = 0              # forced first blocks
    n_local: int = 0             # forced newest blocks
    n0_seq: Optional[Sequence[int]] = None  # ragged batch: context of each sequence (each <= N0)
    n_rep: int = 0               # representative tokens per block (selector "representative")

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def sel_heads(self) -> int:
        """Selections per sequence: KV heads, or query heads under per-head selection."""
        return self.Hq if self.selector == "per_head" else self.Hkv

    @property
    def units(self) -> int:
        return self.B * self.sel_heads

    def n0(self, b: int) -> int:
        """Context length of sequence b before the first decode step."""
        return self.n0_seq[b] if self.n0_seq is not None else self.N0

    def seed_of(self, b: int) -> int:
        # per-sequence seeds are b (plus an offset that distinguishes replicas)
        return b + self.seed if self.per_seq_seed else self.seed

    def cap_tokens(self, extra_steps: int = 0) -> int:
        return self.N0 + self.steps + extra_steps

    def nb(self, n: int) -> int:
        return -(-n // self.bs)

    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    # batch 1, 1 KV head x 4 query heads, d 64, 4096 tokens in 64-token blocks
    "tiny": Workload("tiny", B=1, Hq=4, Hkv=1, d=64, N0=4096, bs=64, K=8, P=8, steps=16,
                     alpha=0.9, qk="grid", walk_p=0.9),
    # Llama-3.1-8B-shaped layer: 32 query / 8 KV heads, d 128, 32K context, 64-token blocks
    "llama8b_32k": Workload("llama8b_32k", B=1, Hq=32, Hkv=8, d=128, N0=32768, bs=64, K=64,
                            P=64, steps=128, alpha=0.9, qk="grid", walk_p=0.9),
    # batch 16 at 128K, 128-token blocks, top-32, per-sequence seeds
    "batched_128k": Workload("batched_128k", B=16, Hq=32, Hkv=8, d=128, N0=131072, bs=128,
                             K=32, P=32, steps=64, alpha=0.9, qk="grid", walk_p=0.9,
                             per_seq_seed=True),
    # Gaussian q/k/v, batch 8 at 64K, predicted set forced to a given overlap with top-K
    "repair_sweep_64k": Workload("repair_sweep_64k", B=8, Hq=32, Hkv=8, d=128, N0=65536,
                                 bs=64, K=64, P=64, steps=32, alpha=0.9, qk="gauss",
                                 walk_p=0.9,
                                 forced_overlaps=(1.0, 0.97, 0.9, 0.75, 0.5, 0.0)),
    # 512K context, batch 4, 64 query / 8 KV heads (8:1 GQA), 128-token blocks
    "long_512k": Workload("long_512k", B=4, Hq=64, Hkv=8, d=128, N0=524288, bs=128, K=64,
                          P=64, steps=32, alpha=0.9, qk="grid", walk_p=0.8),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


# ----------------------------------------------------------------------------- bf16 bits

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


_GRID_BITS = f32_to_bf16_bits(np.arange(-8, 9, dtype=np.float32) / np.float32(8.0))


def _rng(w: Workload, b: int, *tags: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed_of(b), *tags, b])))


def _draw_qk(w: Workload, rng: np.random.Generator, shape) -> np.ndarray:
    if w.qk == "grid":
        return _GRID_BITS[rng.integers(0, 17, size=shape, dtype=np.uint8)]
    return f32_to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


def _draw_v(rng: np.random.Generator, shape) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


# ----------------------------------------------------------------------------- KV cache

def kv_prefix(w: Workload, b: int, kvh: int, n: Optional[int] = None):
    """k, v bit patterns [n][d] for the first n (default N0) context tokens of one
    (sequence, KV head).  Tokens beyond N0 come from :func:`kv_appended`."""
    n = w.N0 if n is None else n
    assert n <= w.N0
    rk = _rng(w, b, _TAG_K0, kvh)
    rv = _rng(w, b, _TAG_V0, kvh)
    k = _draw_qk(w, rk, (w.N0, w.d))[:n]
    v = _draw_v(rv, (w.N0, w.d))[:n]
    return np.ascontiguousarray(k), np.ascontiguousarray(v)


def kv_appended(w: Workload, b: int, kvh: int, steps: Optional[int] = None):
    """k, v bit patterns [steps][d]: the token appended at decode step t is row t."""
    steps = w.steps if steps is None else steps
    rk = _rng(w, b, _TAG_KNEW, kvh)
    rv = _rng(w, b, _TAG_VNEW, kvh)
    return _draw_qk(w, rk, (steps, w.d)), _draw_v(rv, (steps, w.d))


def queries(w: Workload, steps: Optional[int] = None) -> np.ndarray:
    """q bit patterns [steps][B][Hq][d] following the channel-persistence walk."""
    steps = w.steps if steps is None else steps
    out = np.empty((steps, w.B, w.Hq, w.d), dtype=np.uint16)
    for b in range(w.B):
        rng = _rng(w, b, _TAG_Q)
        cur = _draw_qk(w, rng, (w.Hq, w.d))
        for t in range(steps):
            if t > 0:
                keep = rng.random((w.Hq, w.d)) < w.walk_p
                fresh = _draw_qk(w, rng, (w.Hq, w.d))
                cur = np.where(keep, cur, fresh)
            out[t, b] = cur
    return out


# ----------------------------------------------------------------------------- representatives

def rep_offsets(w: Workload, b: int, kvh: int, maxnb: int) -> np.ndarray:
    """Offsets [maxnb][n_rep] (uint8, uniform in [0, bs)) of each block's representative
    tokens for the representative-key selector: an input chosen when a block is built
    (here seeded per (sequence, KV head)), not part of the method's arithmetic."""
    rng = _rng(w, b, _TAG_REP, kvh)
    return rng.integers(0, w.bs, size=(maxnb, w.n_rep), dtype=np.uint8)


# ----------------------------------------------------------------------------- forced prediction

def forced_kept_count(overlap: float, K_eff: int) -> int:
    """Blocks of the true top-K kept in a forced predicted set: round half up of o*K."""
    return int(math.floor(overlap * K_eff + 0.5))


def forced_prediction(w: Workload, selected: Sequence[int], nb: int, overlap: float,
                      level: int, step: int, b: int, kvh: int) -> np.ndarray:
    """A predicted set of P = |selected| blocks with a forced overlap with `selected`.

    ``selected`` is the true top-K of this step.  round-half-up(overlap*K) of its blocks
    are kept (a seeded uniform subset) and the rest are seeded uniform picks among the
    blocks outside it.  Returned ascending, as int32.
    """
    sel = np.asarray(sorted(int(x) for x in selected), dtype=np.int64)
    K_eff = len(sel)
    kept = forced_kept_count(overlap, K_eff)
    rng = _rng(w, b, _TAG_FORCED, level, step, kvh)
    keep_part = rng.choice(sel, size=kept, replace=False) if kept else np.empty(0, np.int64)
    outside = np.setdiff1d(np.arange(nb, dtype=np.int64), sel, assume_unique=True)
    fill = K_eff - kept
    fill_part = rng.choice(outside, size=fill, replace=False) if fill else np.empty(0, np.int64)
    return np.sort(np.concatenate([keep_part, fill_part])).astype(np.int32)


def describe(w: Workload) -> List[str]:
    return [f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} d={w.d} N0={w.N0} bs={w.bs} K={w.K} "
            f"P={w.P} steps={w.steps} alpha={w.alpha} q/k={w.qk} walk_p={w.walk_p}"]
