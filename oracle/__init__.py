"""fp64 CPU oracle for the PRR decode step (ctypes wrapper around prr_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the graft entry point's smoke check and the
bench's CPU-baseline / reference leg may import this package.  The product path
(``dynamic_sparse_attention_block_b200``) never does, and the two share no code.

Every function follows the plain definition of top-K dynamic sparse attention that
the PRR pages say the method reproduces exactly; see the header of prr_oracle.c for
the per-step definition and the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "prr_oracle.c")
LIBRARY = os.path.join(HERE, "libprr_oracle.so")

# -ffp-contract=off: no fused multiply-add, so the EMA recurrence rounds exactly as
# written (alpha*e rounded, beta*ind rounded, then the sum rounded).
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fopenmp"]


def build(source: str = SOURCE, output: str = LIBRARY, force: bool = False,
          extra_flags=()) -> str:
    """Compile the oracle with gcc (no GPU needed).  Returns the library path."""
    if (not force and os.path.exists(output)
            and os.path.getmtime(output) >= os.path.getmtime(source)):
        return output
    cmd = ["gcc", *CFLAGS, *extra_flags, "-o", output, source, "-lm"]
    subprocess.run(cmd, check=True)
    return output


_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_int = ctypes.c_int
_dbl = ctypes.c_double


class _Dims(ctypes.Structure):
    _fields_ = [("B", _int), ("Hq", _int), ("Hkv", _int), ("d", _int), ("bs", _int),
                ("cap", _int), ("K", _int), ("P", _int), ("alpha", _dbl), ("scale", _dbl)]


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class Oracle:
    """Thin typed view of one build of prr_oracle.c."""

    def __init__(self, path: Optional[str] = None):
        self.path = path or build()
        L = ctypes.CDLL(self.path)
        L.oracle_block_summary.argtypes = [_u16p, _int, _int, _int, _int, _f64p, _f64p]
        L.oracle_build_summaries.argtypes = [_u16p, _int, _int, _int, _f64p, _f64p]
        L.oracle_block_scores.argtypes = [_f64p, _int, _int, _f64p, _f64p, _int, _f64p]
        L.oracle_top_ranked.argtypes = [_f64p, _int, _int, _i32p]
        L.oracle_block_scores_max.argtypes = [_f64p, _int, _int, _f64p, _f64p, _int, _f64p]
        L.oracle_top_ranked_forced.argtypes = [_f64p, _int, _int, _int, _int, _i32p]
        L.oracle_gather_pages.argtypes = [_u16p, _i32p, _int, _int, _int, _int, _int, _u16p]
        L.oracle_block_scores_rep.argtypes = [_f64p, _int, _int, _u16p, _int, _int, _i32p, _int, _int, _f64p]
        L.oracle_top_ranked_forced.restype = _int
        L.oracle_top_ranked.restype = _int
        L.oracle_ema_update.argtypes = [_f64p, _int, _i32p, _int, _dbl]
        L.oracle_attend_blocks.argtypes = [_f64p, _u16p, _u16p, _int, _int, _int, _i32p, _int,
                                           _dbl, _f64p, _f64p]
        L.oracle_block_partial.argtypes = [_f64p, _u16p, _u16p, _int, _int, _int, _int, _dbl,
                                           _f64p, _f64p, _f64p]
        L.oracle_lse_merge.argtypes = [_int, _f64p, _f64p, _f64p, _int, _f64p, _f64p]
        L.oracle_missed_keep.argtypes = [_i32p, _int, _i32p, _int, _i32p, _u8p]
        L.oracle_missed_keep.restype = _int
        L.oracle_prr_attend.argtypes = [_f64p, _u16p, _u16p, _int, _int, _int, _i32p, _int,
                                        _i32p, _int, _dbl, _f64p, _f64p]
        L.oracle_decode_step.argtypes = [ctypes.POINTER(_Dims), _u16p, _u16p, _u16p, _i32p,
                                         _i32p, _f64p, _f64p, _f64p, _i32p, _i32p, _i32p,
                                         _u8p, _i32p, _f64p, _f64p, _int]
        L.oracle_decode_step.restype = _int
        L.oracle_max_threads.restype = _int
        self.L = L

    # -- 1. summaries
    def block_summary(self, k_bits, n, bs, blk) -> Tuple[np.ndarray, np.ndarray]:
        k_bits = _c(k_bits, np.uint16)
        d = k_bits.shape[1]
        lo, hi = np.empty(d), np.empty(d)
        self.L.oracle_block_summary(k_bits, n, d, bs, blk, lo, hi)
        return lo, hi

    def build_summaries(self, k_bits, n, bs) -> Tuple[np.ndarray, np.ndarray]:
        k_bits = _c(k_bits, np.uint16)
        d = k_bits.shape[1]
        nb = -(-n // bs)
        lo, hi = np.empty((nb, d)), np.empty((nb, d))
        self.L.oracle_build_summaries(k_bits, n, d, bs, lo, hi)
        return lo, hi

    # -- 2. scores
    def block_scores(self, q, smin, smax) -> np.ndarray:
        q = _c(q, np.float64)
        smin, smax = _c(smin, np.float64), _c(smax, np.float64)
        G, d = q.shape
        nb = smin.shape[0]
        s = np.empty(nb)
        self.L.oracle_block_scores(q, G, d, smin, smax, nb, s)
        return s

    # -- 3. / 5. ranking
    def top_ranked(self, values, K) -> np.ndarray:
        values = _c(values, np.float64)
        out = np.full(max(K, 1), -1, dtype=np.int32)
        cnt = self.L.oracle_top_ranked(values, len(values), K, out)
        return out[:cnt].copy()

    def block_scores_max(self, q, smin, smax) -> np.ndarray:
        """Selector variant: the largest per-head bound of the group (instead of the sum)."""
        q = _c(q, np.float64)
        G, d = q.shape
        nb = smin.shape[0]
        out = np.zeros(nb, np.float64)
        self.L.oracle_block_scores_max(q, G, d, _c(smin, np.float64), _c(smax, np.float64), nb, out)
        return out

    def top_ranked_forced(self, values, K, n_sink, n_local) -> np.ndarray:
        """Selector variant: first n_sink and last n_local blocks forced, best of the rest."""
        v = _c(values, np.float64)
        out = np.zeros(max(min(K, len(v)), 1), np.int32)
        cnt = self.L.oracle_top_ranked_forced(v, len(v), K, n_sink, n_local, out)
        return out[:cnt]

    def block_scores_rep(self, q, k_bits, n, bs, rep):
        """Selector variant (InfLLM-style): each block scored by r representative tokens
        of its own (rep [nb][r] offsets in the block), summed over heads and tokens."""
        q = _c(q, np.float64)
        G, d = q.shape
        rep = _c(rep, np.int32)
        nb, r = rep.shape
        out = np.zeros(nb, np.float64)
        self.L.oracle_block_scores_rep(q, G, d, _c(k_bits, np.uint16), n, bs, rep, r, nb, out)
        return out

    def gather_pages(self, pool_bits, table_row, h, n, bs):
        """Tokens [0, n) of KV head h of one sequence from a paged pool
        [pages][Hkv][bs][d] through the sequence's block-table row, as [n][d] bits."""
        pool_bits = _c(pool_bits, np.uint16)
        _, Hkv, bs_, d = pool_bits.shape
        assert bs_ == bs
        out = np.zeros((n, d), np.uint16)
        self.L.oracle_gather_pages(pool_bits, _c(table_row, np.int32), Hkv, h, n, bs, d, out)
        return out

    def select_per_head(self, q, smin, smax, K):
        """Selector variant: every query head selects with its own bound (no sharing)."""
        q = _c(q, np.float64)
        return [self.top_ranked(self.block_scores(q[h:h + 1], smin, smax), K) for h in range(q.shape[0])]

    def ema_update(self, e, nb, sel, alpha) -> np.ndarray:
        e = _c(e, np.float64).copy()
        sel = np.asarray(sel, np.int32)
        s1 = _c(sel, np.int32) if sel.size else np.zeros(1, np.int32)
        self.L.oracle_ema_update(e, nb, s1, int(sel.size), alpha)
        return e

    # -- 4. attention
    def attend_blocks(self, q, k_bits, v_bits, n, bs, blocks, scale):
        q = _c(q, np.float64)
        d = q.shape[0]
        blocks = np.asarray(blocks, np.int32)
        b1 = _c(blocks, np.int32) if blocks.size else np.zeros(1, np.int32)
        out, lse = np.empty(d), np.empty(1)
        self.L.oracle_attend_blocks(q, _c(k_bits, np.uint16), _c(v_bits, np.uint16), n, d, bs,
                                    b1, int(blocks.size), scale, out, lse)
        return out, float(lse[0])

    def block_partial(self, q, k_bits, v_bits, n, bs, blk, scale):
        q = _c(q, np.float64)
        d = q.shape[0]
        m, l, O = np.empty(1), np.empty(1), np.empty(d)
        self.L.oracle_block_partial(q, _c(k_bits, np.uint16), _c(v_bits, np.uint16), n, d, bs,
                                    blk, scale, m, l, O)
        return float(m[0]), float(l[0]), O

    def lse_merge(self, m, l, O):
        m, l, O = _c(m, np.float64), _c(l, np.float64), _c(O, np.float64)
        cnt = len(m)
        d = O.shape[1]
        if cnt == 0:
            m, l, O = np.zeros(1), np.zeros(1), np.zeros((1, d))
        out, lse = np.empty(d), np.empty(1)
        self.L.oracle_lse_merge(cnt, m, l, O, d, out, lse)
        return out, float(lse[0])

    def missed_keep(self, sel, pred):
        sel = np.asarray(sel, np.int32)
        pred = np.asarray(pred, np.int32)
        s1 = sel if sel.size else np.zeros(1, np.int32)
        p1 = pred if pred.size else np.zeros(1, np.int32)
        missed = np.full(max(len(sel), 1), -1, np.int32)
        keep = np.zeros(max(len(pred), 1), np.uint8)
        nm = self.L.oracle_missed_keep(_c(s1, np.int32), len(sel), _c(p1, np.int32), len(pred),
                                       missed, keep)
        return missed[:nm].copy(), keep[:len(pred)].copy()

    def prr_attend(self, q, k_bits, v_bits, n, bs, sel, pred, scale):
        q = _c(q, np.float64)
        d = q.shape[0]
        sel = np.asarray(sel, np.int32)
        pred = np.asarray(pred, np.int32)
        s1 = sel if sel.size else np.zeros(1, np.int32)
        p1 = pred if pred.size else np.zeros(1, np.int32)
        out, lse = np.empty(d), np.empty(1)
        self.L.oracle_prr_attend(q, _c(k_bits, np.uint16), _c(v_bits, np.uint16), n, d, bs,
                                 _c(s1, np.int32), len(sel), _c(p1, np.int32), len(pred), scale,
                                 out, lse)
        return out, float(lse[0])

    # -- one decode step over every unit
    def decode_step(self, dims: dict, q_bits, k_cache, v_cache, seq_lens, pred, state: dict,
                    nthreads: int = 1) -> dict:
        """Run one step.  ``state`` holds smin, smax, ema (updated in place)."""
        D = _Dims(dims["B"], dims["Hq"], dims["Hkv"], dims["d"], dims["bs"], dims["cap"],
                  dims["K"], dims["P"], float(dims["alpha"]), float(dims["scale"]))
        B, Hq, Hkv, K, P, d = D.B, D.Hq, D.Hkv, D.K, D.P, D.d
        units = B * Hkv
        res = {
            "sel": np.full((B, Hkv, K), -1, np.int32),
            "missed": np.full((B, Hkv, K), -1, np.int32),
            "n_missed": np.zeros((B, Hkv), np.int32),
            "keep": np.zeros((B, Hkv, P), np.uint8),
            "pred_next": np.full((B, Hkv, P), -1, np.int32),
            "out": np.zeros((B, Hq, d)),
            "lse": np.zeros((B, Hq)),
        }
        assert state["smin"].flags.c_contiguous and state["ema"].flags.c_contiguous
        used = self.L.oracle_decode_step(
            ctypes.byref(D), _c(q_bits, np.uint16), k_cache, v_cache, _c(seq_lens, np.int32),
            _c(pred, np.int32), state["smin"], state["smax"], state["ema"], res["sel"],
            res["missed"], res["n_missed"], res["keep"], res["pred_next"], res["out"],
            res["lse"], int(nthreads))
        res["threads"] = used
        assert units == B * Hkv
        return res

    def max_threads(self) -> int:
        return int(self.L.oracle_max_threads())


def new_state(B, Hkv, cap, bs, d) -> dict:
    maxnb = -(-cap // bs)
    return {"smin": np.zeros((B, Hkv, maxnb, d)), "smax": np.zeros((B, Hkv, maxnb, d)),
            "ema": np.zeros((B, Hkv, maxnb))}


_DEFAULT: Optional[Oracle] = None


def default() -> Oracle:
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT
