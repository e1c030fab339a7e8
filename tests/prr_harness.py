"""Drive the CUDA decode path and the fp64 oracle over the same seeded workload and
compare them.  Inputs come only from ``workloads``; expected values come only from
``oracle``; nothing computed by the CUDA path is fed to the oracle.

Tolerances (fp32 attention on the GPU against fp64 on the CPU):
  selected sets, missed sets, keep masks, predicted sets, EMA state: bit-exact;
  out: max |gpu - oracle| <= 2e-3;  lse: |gpu - oracle| / |oracle| <= 1e-4.
For Gaussian workloads a differing selected set is accepted when it is a valid
selection (ascending, distinct, in range, of size min(K, nb)) and every differing
block's oracle score lies within 1e-5 * max(1, |s_K|) of the oracle's K-th score
(the score-gap reading of the repair-sweep workload).  Several sets are then correct;
the oracle continues from the GPU's accepted set, so the unit's missed set, keep
mask, out, lse, EMA state and next prediction are still compared, against the
oracle's values for that set.  Near ties must stay rare: at most
max(NEAR_TIE_MIN, NEAR_TIE_FRAC * unit-steps) per run.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np

import oracle as OR
import workloads as W

OUT_TOL = 2e-3
LSE_RTOL = 1e-4
GAP_RTOL = 1e-5
NEAR_TIE_FRAC = 0.01
NEAR_TIE_MIN = 2


def f64(bits):
    return W.bf16_bits_to_f32(bits).astype(np.float64)


@dataclass
class UnitOracle:
    """Oracle trajectory of one selection unit, driven step by step: a (sequence, KV
    head) pair scored with the group's query heads, or, under per-head selection, a
    (sequence, query head) pair scored with that head alone over its KV head's keys."""
    w: W.Workload
    b: int
    kvh: int           # selection head: a KV head, or a query head under per-head selection
    k: np.ndarray      # [N0+steps][d] bits
    v: np.ndarray
    smin: np.ndarray
    smax: np.ndarray
    ema: np.ndarray
    pred: np.ndarray   # Pred_t (ascending)
    o: OR.Oracle
    rep: Optional[np.ndarray] = None  # [maxnb][n_rep] representative offsets (representative selector)

    @property
    def kv_head(self) -> int:
        return self.kvh // self.w.G if self.w.selector == "per_head" else self.kvh

    @property
    def qrows(self) -> slice:
        if self.w.selector == "per_head":
            return slice(self.kvh, self.kvh + 1)
        return slice(self.kvh * self.w.G, (self.kvh + 1) * self.w.G)

    @classmethod
    def create(cls, w: W.Workload, b: int, kvh: int, steps: int, o: OR.Oracle):
        kv = kvh // w.G if w.selector == "per_head" else kvh
        n0 = w.n0(b)
        k0, v0 = W.kv_prefix(w, b, kv, n0)
        kn, vn = W.kv_appended(w, b, kv, steps)
        k = np.concatenate([k0, kn])
        v = np.concatenate([v0, vn])
        maxnb = w.nb(w.N0 + steps)
        smin = np.zeros((maxnb, w.d))
        smax = np.zeros((maxnb, w.d))
        lo, hi = o.build_summaries(k, n0, w.bs)
        smin[:lo.shape[0]], smax[:lo.shape[0]] = lo, hi
        ema = np.zeros(maxnb)
        pred = o.top_ranked(np.zeros(w.nb(n0)), w.P) if w.P > 0 else np.zeros(0, np.int32)
        rep = W.rep_offsets(w, b, kv, maxnb) if w.selector == "representative" else None
        return cls(w, b, kvh, k, v, smin, smax, ema, pred, o, rep)

    def select(self, t: int, q_bits: np.ndarray):
        """Summary update for token N0+t, scores, true top-K (all from the oracle)."""
        w, o = self.w, self.o
        n = w.n0(self.b) + t + 1
        nb = w.nb(n)
        tail = (n - 1) // w.bs
        lo, hi = o.block_summary(self.k, n, w.bs, tail)
        self.smin[tail], self.smax[tail] = lo, hi
        qg = f64(q_bits[self.b, self.qrows])
        if w.selector == "group_max":
            s = o.block_scores_max(qg, self.smin[:nb], self.smax[:nb])
        elif w.selector == "representative":
            s = o.block_scores_rep(qg, self.k, n, w.bs, self.rep[:nb].astype(np.int32))
        else:  # group sum, or one head's own bound under per-head selection
            s = o.block_scores(qg, self.smin[:nb], self.smax[:nb])
        if w.n_sink or w.n_local:
            sel = o.top_ranked_forced(s, w.K, w.n_sink, w.n_local)
        else:
            sel = o.top_ranked(s, w.K)
        return n, nb, qg, s, sel

    def finish(self, n, nb, qg, sel, pred):
        """Given S_t and the Pred_t actually used: missed/keep, attention, EMA update."""
        w, o = self.w, self.o
        missed, keep = o.missed_keep(sel, pred)
        outs, lses = [], []
        for g in range(qg.shape[0]):
            out, lse = o.attend_blocks(qg[g], self.k, self.v, n, w.bs, sel, w.scale())
            outs.append(out)
            lses.append(lse)
        self.ema[:] = o.ema_update(self.ema, nb, sel, w.alpha)
        pred_next = o.top_ranked(self.ema[:nb], w.P) if w.P > 0 else np.zeros(0, np.int32)
        return dict(sel=sel, missed=missed, keep=keep, out=np.stack(outs), lse=np.array(lses),
                    pred_next=pred_next)


def pad(x: Sequence[int], L: int) -> np.ndarray:
    a = np.full(L, -1, np.int32)
    a[:len(x)] = x
    return a


@dataclass
class Report:
    max_out_err: float = 0.0
    max_lse_rel: float = 0.0
    units_compared: int = 0
    unit_steps: int = 0
    near_tie_units: int = 0
    messages: List[str] = field(default_factory=list)

    def fail(self, msg: str):
        self.messages.append(msg)

    def near_tie_bound(self) -> int:
        return max(NEAR_TIE_MIN, int(NEAR_TIE_FRAC * self.unit_steps))

    def check_near_ties(self) -> None:
        if self.near_tie_units > self.near_tie_bound():
            self.fail(f"{self.near_tie_units} near-tie selections in {self.unit_steps} unit-steps "
                      f"(bound {self.near_tie_bound()})")


def accepted_selection(gpu_sel: np.ndarray, o_sel: np.ndarray, scores: np.ndarray,
                       gaussian: bool) -> Optional[np.ndarray]:
    """The set the comparison continues from, or None if the GPU's set is wrong.

    Exact grids: only the oracle's set.  Gaussian scores: the GPU's set is also
    accepted when it is a valid selection (strictly ascending, in range, as many blocks
    as the oracle's) whose differences from the oracle's set all lie within the score
    gap of the oracle's K-th score."""
    g = np.asarray([int(x) for x in gpu_sel if x >= 0], np.int32)
    r = np.asarray(o_sel, np.int32)
    if np.array_equal(g, r):
        return r
    if not gaussian or len(g) != len(r):
        return None
    if np.any(np.diff(g) <= 0) or (len(g) and (g[0] < 0 or g[-1] >= len(scores))):
        return None
    if any(int(x) != -1 for x in np.asarray(gpu_sel)[len(g):]):
        return None
    kth = np.sort(scores)[::-1][len(r) - 1]
    tol = GAP_RTOL * max(1.0, abs(kth))
    diff = set(g.tolist()) ^ set(r.tolist())
    if all(abs(scores[b] - kth) <= tol for b in diff):
        return g
    return None


def check_selection(rep: Report, tag: str, gpu_sel: np.ndarray, o_sel: np.ndarray,
                    scores: np.ndarray, K: int, gaussian: bool) -> Optional[np.ndarray]:
    """The selected set the oracle continues from for this unit: the oracle's set when
    the GPU's equals it, the GPU's set when a Gaussian near tie makes it another
    correct answer (counted in rep.near_tie_units), else None (a failure is recorded)."""
    rep.unit_steps += 1
    acc = accepted_selection(gpu_sel, o_sel, scores, gaussian)
    if acc is None:
        g = [int(x) for x in gpu_sel if x >= 0]
        rep.fail(f"{tag}: selected set differs: gpu={g} oracle={list(map(int, o_sel))}")
        return None
    if not np.array_equal(acc, np.asarray(o_sel, np.int32)):
        rep.near_tie_units += 1
    return acc


def compare_attention(rep: Report, tag: str, gpu_out: np.ndarray, gpu_lse: np.ndarray,
                      o_out: np.ndarray, o_lse: np.ndarray) -> None:
    err = float(np.max(np.abs(gpu_out.astype(np.float64) - o_out)))
    rel = float(np.max(np.abs(gpu_lse.astype(np.float64) - o_lse) / np.maximum(np.abs(o_lse), 1e-30)))
    rep.max_out_err = max(rep.max_out_err, err)
    rep.max_lse_rel = max(rep.max_lse_rel, rel)
    rep.units_compared += 1
    if not (err <= OUT_TOL) or not math.isfinite(err):
        rep.fail(f"{tag}: out max-abs error {err:.3e} > {OUT_TOL}")
    if not (rel <= LSE_RTOL) or not math.isfinite(rel):
        rep.fail(f"{tag}: lse relative error {rel:.3e} > {LSE_RTOL}")
