"""ctypes binding of the C ABI in include/prr.h (argument marshalling only).

Every function here has the name of the C entry point it calls and does nothing but
turn torch tensors into device pointers, streams into handles and non-zero statuses
into exceptions.  All arithmetic runs in the CUDA kernels of libprr_b200.so.  There
is no fallback: if the library is missing or no GPU is present, calls raise.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional

import torch

from . import build as _build

_c_void_p = ctypes.c_void_p
_i32 = ctypes.c_int32


class PrrDims(ctypes.Structure):
    _fields_ = [("B", _i32), ("Hq", _i32), ("Hkv", _i32), ("d", _i32), ("bs", _i32),
                ("cap_tokens", _i32), ("K", _i32), ("P", _i32), ("alpha", ctypes.c_double),
                ("scale", ctypes.c_float), ("selector", _i32), ("n_sink", _i32), ("n_local", _i32),
                ("pages", _i32), ("block_table", _c_void_p), ("n_rep", _i32), ("rep_offsets", _c_void_p)]


# block selectors (PRR_SELECT_* in include/prr.h)
SELECTORS = {"group_sum": 0, "group_max": 1, "per_head": 2, "representative": 3}


class PrrStepBuffers(ctypes.Structure):
    _fields_ = [(n, _c_void_p) for n in (
        "q", "k_cache", "v_cache", "seq_lens", "summ", "ema", "pred", "pred_next", "sel",
        "missed", "n_missed", "keep", "part_m", "part_l", "part_O", "out", "lse", "k_new", "v_new", "trace",
        "stats")]


STEP_EVENTS = ("fork", "sel_done", "spec_done", "join")
TIMING_MARKS = ("t_begin", "t_select_end", "t_repair_end", "t_combine_begin", "t_combine_end",
                "t_spec_begin", "t_spec_end", "t_ema_begin", "t_ema_end")


class PrrStepEvents(ctypes.Structure):
    _fields_ = [(n, _c_void_p) for n in STEP_EVENTS + TIMING_MARKS]


# exported C symbols, in header order
SYMBOLS = (
    "prr_version", "prr_status_string", "prr_workspace_bytes", "prr_workspace_init",
    "prr_get_device_status", "prr_append_kv", "prr_update_summaries", "prr_select_topk",
    "prr_ema_predict", "prr_speculate", "prr_repair_merge", "prr_decode_step",
    "prr_decode_step_fused", "prr_budget_fit", "prr_budget_choose", "prr_select_topk_static",
)

# mirrors PRR_WS_TEST_SKIP_SELECTION_OFFSET in include/prr.h
WS_TEST_SKIP_SELECTION_OFFSET = 4

# mirrors PRR_SELECT_STATIC_MAX_BLOCKS / PRR_SELECT_STATIC_SCRATCH_BYTES in include/prr.h
SELECT_STATIC_MAX_BLOCKS = 1 << 20
SELECT_STATIC_SCRATCH_BYTES = 256 + 65536 * 4 + SELECT_STATIC_MAX_BLOCKS * 4

STATUS = {0: "PRR_OK", 1: "PRR_ERR_INVALID_ARG", 2: "PRR_ERR_SHAPE", 3: "PRR_ERR_CAPACITY",
          4: "PRR_ERR_CUDA", 5: "PRR_ERR_DEVICE_STATUS", 6: "PRR_ERR_TIMEOUT"}
DEVICE_STATUS = {0: "ok", 1: "bad seq_len", 2: "bad predicted list", 3: "bad missed list",
                 4: "wait timed out", 5: "bad summary range"}


class PrrError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


_LIB: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return _build.LIBRARY


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libprr_b200.so (built in-tree).  Raises if it has not been built."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = path or _build.LIBRARY
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with dynamic_sparse_attention_block_b200.build.build()")
    L = ctypes.CDLL(p)
    vp, sz = _c_void_p, ctypes.c_size_t
    dims = ctypes.POINTER(PrrDims)
    L.prr_version.restype = ctypes.c_int
    L.prr_status_string.restype = ctypes.c_char_p
    L.prr_status_string.argtypes = [ctypes.c_int]
    L.prr_workspace_bytes.restype = sz
    L.prr_workspace_bytes.argtypes = [dims]
    L.prr_workspace_init.argtypes = [vp, sz, vp]
    L.prr_get_device_status.argtypes = [vp, ctypes.POINTER(_i32)]
    L.prr_append_kv.argtypes = [dims, vp, vp, vp, vp, vp, vp, vp]
    L.prr_update_summaries.argtypes = [dims, vp, vp, vp, vp, _i32, vp, vp, vp]
    L.prr_select_topk.argtypes = [dims, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.prr_ema_predict.argtypes = [dims, vp, vp, vp, vp, vp, vp]
    L.prr_speculate.argtypes = [dims, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.prr_repair_merge.argtypes = [dims, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.prr_decode_step.argtypes = [dims, ctypes.POINTER(PrrStepBuffers), vp, sz, vp, vp,
                                  ctypes.POINTER(PrrStepEvents)]
    L.prr_decode_step_fused.argtypes = [dims, ctypes.POINTER(PrrStepBuffers), vp, sz, _i32, vp]
    L.prr_select_topk_static.argtypes = [dims, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.prr_budget_fit.argtypes = [vp, vp, _i32, _i32, vp]
    L.prr_budget_choose.argtypes = [vp, vp, vp, _i32, _i32, _i32, ctypes.POINTER(_i32)]
    for name in SYMBOLS:
        if name not in ("prr_version", "prr_status_string", "prr_workspace_bytes"):
            getattr(L, name).restype = ctypes.c_int
    if path is None:
        _LIB = L
    return L


# ----------------------------------------------------------------------------- marshalling

@dataclasses.dataclass(frozen=True)
class Dims:
    B: int
    Hq: int
    Hkv: int
    d: int
    bs: int
    cap_tokens: int
    K: int
    P: int
    alpha: float = 0.9
    scale: Optional[float] = None
    selector: str = "group_sum"   # "group_sum", "group_max", "per_head" or "representative"
    n_sink: int = 0               # forced first blocks
    n_local: int = 0              # forced newest blocks
    pages: int = 0                # paged KV pool size (0: contiguous caches)
    block_table: Optional[int] = None  # device address of the int32 [B][maxnb] block table
    n_rep: int = 0                # representative tokens per block (representative selector)
    rep_offsets: Optional[int] = None  # device address of the uint8 [B][Hkv][maxnb][n_rep] offsets

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def sel_heads(self) -> int:
        """Selections per sequence: KV heads, or query heads under per-head selection."""
        return self.Hq if self.selector == "per_head" else self.Hkv

    @property
    def group(self) -> int:
        """Query heads one selection scores with (1 under per-head selection)."""
        return 1 if self.selector == "per_head" else self.G

    @property
    def units(self) -> int:
        return self.B * self.sel_heads

    @property
    def maxnb(self) -> int:
        return -(-self.cap_tokens // self.bs)

    def c(self) -> PrrDims:
        sc = self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)
        return PrrDims(self.B, self.Hq, self.Hkv, self.d, self.bs, self.cap_tokens, self.K,
                       self.P, float(self.alpha), float(sc), SELECTORS[self.selector], self.n_sink, self.n_local,
                       self.pages, self.block_table, self.n_rep, self.rep_offsets)


def _dims(d) -> PrrDims:
    return d.c() if isinstance(d, Dims) else d


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, where: str) -> None:
    if status != 0:
        raise PrrError(status, where)


def prr_version() -> int:
    return load().prr_version()


def prr_status_string(status: int) -> str:
    return load().prr_status_string(status).decode()


def prr_workspace_bytes(dims) -> int:
    return int(load().prr_workspace_bytes(ctypes.byref(_dims(dims))))


def prr_workspace_init(ws, stream=None) -> None:
    _check(load().prr_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "prr_workspace_init")


def prr_get_device_status(ws) -> int:
    code = _i32(0)
    st = load().prr_get_device_status(_ptr(ws), ctypes.byref(code))
    if st not in (0, 5):
        _check(st, "prr_get_device_status")
    return int(code.value)


def prr_append_kv(dims, k_new, v_new, seq_lens, k_cache, v_cache, ws, stream=None) -> None:
    _check(load().prr_append_kv(ctypes.byref(_dims(dims)), _ptr(k_new), _ptr(v_new), _ptr(seq_lens),
                                _ptr(k_cache), _ptr(v_cache), _ptr(ws), _stream(stream)),
           "prr_append_kv")


def prr_update_summaries(dims, k_cache, tok_begin, tok_end, seq_lens, max_range_tokens, summ, ws,
                         stream=None) -> None:
    _check(load().prr_update_summaries(ctypes.byref(_dims(dims)), _ptr(k_cache), _ptr(tok_begin),
                                       _ptr(tok_end), _ptr(seq_lens), int(max_range_tokens),
                                       _ptr(summ), _ptr(ws), _stream(stream)),
           "prr_update_summaries")


def prr_select_topk(dims, q, summ, seq_lens, pred, sel, missed, n_missed, keep, ws,
                    stream=None) -> None:
    _check(load().prr_select_topk(ctypes.byref(_dims(dims)), _ptr(q), _ptr(summ), _ptr(seq_lens),
                                  _ptr(pred), _ptr(sel), _ptr(missed), _ptr(n_missed), _ptr(keep),
                                  _ptr(ws), _stream(stream)),
           "prr_select_topk")


def prr_select_topk_static(dims, q, summ, seq_lens, pred, sel, missed, n_missed, keep,
                           status=None, stream=None) -> None:
    _check(load().prr_select_topk_static(ctypes.byref(_dims(dims)), _ptr(q), _ptr(summ), _ptr(seq_lens),
                                         _ptr(pred), _ptr(sel), _ptr(missed), _ptr(n_missed),
                                         _ptr(keep), _ptr(status), _stream(stream)),
           "prr_select_topk_static")


def prr_budget_fit(context_tokens, us, degree: int):
    """Least-squares polynomial (lowest order first) of us against context length."""
    import numpy as np
    x = np.ascontiguousarray(context_tokens, dtype=np.float64)
    y = np.ascontiguousarray(us, dtype=np.float64)
    if x.shape != y.shape or x.ndim != 1:
        raise ValueError("context_tokens and us must be 1-D and of one length")
    coef = np.zeros(degree + 1 if degree >= 0 else 1, dtype=np.float64)
    _check(load().prr_budget_fit(x.ctypes.data, y.ctypes.data, len(x), int(degree), coef.ctypes.data),
           "prr_budget_fit")
    return coef


def prr_budget_choose(sel_coef, spec_coef, p_grid, context_tokens: int) -> int:
    """Largest profiled budget whose predicted speculation time fits in selection's."""
    import numpy as np
    sc = np.ascontiguousarray(sel_coef, dtype=np.float64)
    pc = np.ascontiguousarray(spec_coef, dtype=np.float64)
    pg = np.ascontiguousarray(p_grid, dtype=np.int32)
    if pc.ndim != 2 or pc.shape != (len(pg), len(sc)):
        raise ValueError("spec_coef must be [len(p_grid)][degree+1]")
    out = _i32(0)
    _check(load().prr_budget_choose(sc.ctypes.data, pc.ctypes.data, pg.ctypes.data, len(pg), len(sc) - 1,
                                    int(context_tokens), ctypes.byref(out)), "prr_budget_choose")
    return int(out.value)


def prr_ema_predict(dims, ema, sel, seq_lens, pred_next, ws, stream=None) -> None:
    _check(load().prr_ema_predict(ctypes.byref(_dims(dims)), _ptr(ema), _ptr(sel), _ptr(seq_lens),
                                  _ptr(pred_next), _ptr(ws), _stream(stream)),
           "prr_ema_predict")


def prr_speculate(dims, q, k_cache, v_cache, seq_lens, pred, part_m, part_l, part_O, ws,
                  stream=None) -> None:
    _check(load().prr_speculate(ctypes.byref(_dims(dims)), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                _ptr(seq_lens), _ptr(pred), _ptr(part_m), _ptr(part_l),
                                _ptr(part_O), _ptr(ws), _stream(stream)),
           "prr_speculate")


def prr_repair_merge(dims, q, k_cache, v_cache, seq_lens, missed, n_missed, keep, pred, part_m,
                     part_l, part_O, out, lse, ws, stream=None) -> None:
    _check(load().prr_repair_merge(ctypes.byref(_dims(dims)), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                   _ptr(seq_lens), _ptr(missed), _ptr(n_missed), _ptr(keep),
                                   _ptr(pred), _ptr(part_m), _ptr(part_l), _ptr(part_O), _ptr(out),
                                   _ptr(lse), _ptr(ws), _stream(stream)),
           "prr_repair_merge")


def prr_decode_step(dims, buffers: PrrStepBuffers, ws, select_stream, spec_stream,
                    events: PrrStepEvents) -> None:
    _check(load().prr_decode_step(ctypes.byref(_dims(dims)), ctypes.byref(buffers), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(select_stream),
                                  _stream(spec_stream), ctypes.byref(events)),
           "prr_decode_step")


def prr_decode_step_fused(dims, buffers: PrrStepBuffers, ws, step_parity: int, stream=None) -> None:
    _check(load().prr_decode_step_fused(ctypes.byref(_dims(dims)), ctypes.byref(buffers), _ptr(ws),
                                        ws.numel() * ws.element_size(), int(step_parity),
                                        _stream(stream)),
           "prr_decode_step_fused")
