"""PRR decode state for one attention layer: device buffers, streams and the step call.

Torch is used for device memory, streams, events and CUDA graphs only; every step of
the path (summaries, selection, speculation, repair, merge, EMA prediction) runs in
libprr_b200.so through the C ABI.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _abi
from ._abi import Dims


class PRRDecoder:
    """Caller-owned state of the PRR decode step (PRR abstract / method summary: EMA
    predictor, speculative attention overlapped with selection, repair + LSE merge).

    Buffers (row-major):  k_cache/v_cache [B][Hkv][cap][d] bf16, seq_lens [B] int32,
    summ [B][Hkv][maxnb][2][d] bf16, ema [B][Hkv][maxnb] fp64, pred double buffer
    [2][B][Hkv][P] int32, sel/missed [B][Hkv][K], n_missed [B][Hkv], keep [B][Hkv][P],
    speculative partials [B][Hq][P](+[d]) fp32, out [B][Hq][d] fp32, lse [B][Hq] fp32.
    """

    def __init__(self, dims: Dims, device: Optional[torch.device] = None):
        if not torch.cuda.is_available():
            raise RuntimeError("PRRDecoder needs a CUDA device")
        _abi.load()
        self.dims = dims
        self.device = torch.device(device or "cuda")
        dev = self.device
        B, Hq, Hkv, d, cap, K, P = dims.B, dims.Hq, dims.Hkv, dims.d, dims.cap_tokens, dims.K, dims.P
        maxnb = dims.maxnb
        self.k_cache = torch.zeros((B, Hkv, cap, d), dtype=torch.bfloat16, device=dev)
        self.v_cache = torch.zeros((B, Hkv, cap, d), dtype=torch.bfloat16, device=dev)
        self.seq_lens = torch.zeros((B,), dtype=torch.int32, device=dev)
        self.summ = torch.zeros((B, Hkv, maxnb, 2, d), dtype=torch.bfloat16, device=dev)
        self.ema = torch.zeros((B, Hkv, maxnb), dtype=torch.float64, device=dev)
        self.pred_buf = torch.full((2, B, Hkv, max(P, 1)), -1, dtype=torch.int32, device=dev)
        self.sel = torch.full((B, Hkv, K), -1, dtype=torch.int32, device=dev)
        self.missed = torch.full((B, Hkv, K), -1, dtype=torch.int32, device=dev)
        self.n_missed = torch.zeros((B, Hkv), dtype=torch.int32, device=dev)
        self.keep = torch.zeros((B, Hkv, max(P, 1)), dtype=torch.uint8, device=dev)
        self.part_m = torch.zeros((B, Hq, max(P, 1)), dtype=torch.float32, device=dev)
        self.part_l = torch.zeros((B, Hq, max(P, 1)), dtype=torch.float32, device=dev)
        self.part_O = torch.zeros((B, Hq, max(P, 1), d), dtype=torch.float32, device=dev)
        # Per-step I/O in two contiguous buffers, so that a caller moves each direction
        # with one copy: io_in = [q | k_new | v_new] (bf16), io_out = [out | lse] (fp32).
        nq, nkv = B * Hq * d, B * Hkv * d
        self.io_in = torch.zeros((nq + 2 * nkv,), dtype=torch.bfloat16, device=dev)
        self.q = self.io_in[:nq].view(B, Hq, d)
        self.k_new = self.io_in[nq:nq + nkv].view(B, Hkv, d)
        self.v_new = self.io_in[nq + nkv:].view(B, Hkv, d)
        self.io_out = torch.zeros((B * Hq * (d + 1),), dtype=torch.float32, device=dev)
        self.out = self.io_out[:B * Hq * d].view(B, Hq, d)
        self.lse = self.io_out[B * Hq * d:].view(B, Hq)
        nbytes = _abi.prr_workspace_bytes(dims)
        if nbytes == 0:
            raise ValueError(f"unsupported dims {dims}")
        self.ws = torch.zeros((nbytes,), dtype=torch.uint8, device=dev)
        lo, hi = torch.cuda.Stream.priority_range()
        self.select_stream = torch.cuda.Stream(device=dev, priority=hi)
        self.spec_stream = torch.cuda.Stream(device=dev, priority=lo)
        # stream-ordering events of the step (torch creates a handle on first record)
        self.step_events = {name: torch.cuda.Event() for name in _abi.STEP_EVENTS}
        for ev in self.step_events.values():
            ev.record(self.select_stream)
        self.parity = 0  # which pred buffer holds Pred_t
        self.fused_parity = 0  # control-word copy of the next fused launch
        self.trace = None      # optional per-item timeline of fused launches (enable_trace)

    # ------------------------------------------------------------------ views
    @property
    def pred(self) -> torch.Tensor:
        return self.pred_buf[self.parity]

    @property
    def pred_next(self) -> torch.Tensor:
        return self.pred_buf[1 - self.parity]

    def buffers(self, parity: Optional[int] = None) -> _abi.PrrStepBuffers:
        par = self.parity if parity is None else parity
        b = _abi.PrrStepBuffers()
        b.q, b.k_cache, b.v_cache = self.q.data_ptr(), self.k_cache.data_ptr(), self.v_cache.data_ptr()
        b.seq_lens, b.summ, b.ema = self.seq_lens.data_ptr(), self.summ.data_ptr(), self.ema.data_ptr()
        b.pred, b.pred_next = self.pred_buf[par].data_ptr(), self.pred_buf[1 - par].data_ptr()
        b.sel, b.missed, b.n_missed = self.sel.data_ptr(), self.missed.data_ptr(), self.n_missed.data_ptr()
        b.keep = self.keep.data_ptr()
        b.part_m, b.part_l, b.part_O = self.part_m.data_ptr(), self.part_l.data_ptr(), self.part_O.data_ptr()
        b.out, b.lse = self.out.data_ptr(), self.lse.data_ptr()
        b.trace = self.trace.data_ptr() if self.trace is not None else None
        return b

    def events(self, timing: Optional[dict] = None) -> _abi.PrrStepEvents:
        """Step events; `timing` maps names of _abi.TIMING_MARKS to timing-enabled
        torch events that have been recorded once (so that their handles exist)."""
        e = _abi.PrrStepEvents()
        for name, ev in self.step_events.items():
            setattr(e, name, ev.cuda_event)
        for name, ev in (timing or {}).items():
            if name not in _abi.TIMING_MARKS:
                raise ValueError(f"unknown timing mark {name}")
            setattr(e, name, ev.cuda_event)
        return e

    def fused_items(self) -> dict:
        """Work-item counts of one fused launch, in queue order."""
        d = self.dims
        rep = min(d.K, max(4, -(-1024 // d.units)))
        chunk = min(128, max(32, -(-(-(-d.units * d.maxnb // 512)) // 32) * 32))
        return {"sel": d.units * -(-d.maxnb // chunk), "fin": d.units, "ema": d.units,
                "spec": d.units * d.P, "repair": d.units * rep, "combine": d.units * d.G}

    def enable_trace(self, on: bool = True) -> None:
        """Record start/end times of every work item of the fused launches."""
        self.trace = torch.zeros((sum(self.fused_items().values()), 4), dtype=torch.int64,
                                 device=self.device) if on else None

    def trace_summary(self) -> dict:
        """Timeline of the last traced fused launch, per item kind (see summarize_trace)."""
        if self.trace is None:
            raise RuntimeError("tracing is off: call enable_trace() before the step")
        return summarize_trace(self.trace.cpu().numpy(), self.fused_items())

    # ------------------------------------------------------------------ setup
    def prefill(self, k: torch.Tensor, v: torch.Tensor, n0: int) -> None:
        """Copy an initial context of n0 tokens ([B][Hkv][n0][d] bf16) into the cache,
        build all block summaries, reset the EMA and predict from the zero state."""
        d = self.dims
        with torch.cuda.stream(self.select_stream):
            self.k_cache[:, :, :n0].copy_(k)
            self.v_cache[:, :, :n0].copy_(v)
            self.seq_lens.fill_(n0)
            self.ema.zero_()
            self.pred_buf.fill_(-1)
            _abi.prr_workspace_init(self.ws, self.select_stream)
            zeros = torch.zeros((d.B,), dtype=torch.int32, device=self.device)
            ends = torch.full((d.B,), n0, dtype=torch.int32, device=self.device)
            _abi.prr_update_summaries(d, self.k_cache, zeros, ends, None, n0, self.summ, self.ws,
                                      self.select_stream)
            self.parity = 0
            if d.P > 0:
                _abi.prr_ema_predict(d, self.ema, None, self.seq_lens, self.pred_buf[0], self.ws,
                                     self.select_stream)
        self.select_stream.synchronize()

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> None:
        """Write the step's token (k_new/v_new [B][Hkv][d] bf16) and advance seq_lens."""
        _abi.prr_append_kv(self.dims, k_new, v_new, self.seq_lens, self.k_cache, self.v_cache,
                           self.ws, stream or self.select_stream)

    # ------------------------------------------------------------------ the step
    def step(self, q: Optional[torch.Tensor] = None, timing: Optional[dict] = None,
             swap: bool = True) -> None:
        """One decode step on the state's streams (q [B][Hq][d] bf16 is copied into the
        step's query buffer first when given).  Swaps Pred_t / Pred_{t+1} afterwards."""
        if q is not None:
            with torch.cuda.stream(self.select_stream):
                self.q.copy_(q)
        _abi.prr_decode_step(self.dims, self.buffers(), self.ws, self.select_stream,
                             self.spec_stream, self.events(timing))
        if swap and self.dims.P > 0:
            self.parity ^= 1

    def step_fused(self, q: Optional[torch.Tensor] = None, stream=None, swap: bool = True,
                   parity: Optional[int] = None) -> None:
        """The same step as one persistent launch on `stream` (default: select_stream)."""
        st = stream or self.select_stream
        if q is not None:
            with torch.cuda.stream(st):
                self.q.copy_(q)
        par = self.fused_parity if parity is None else parity
        _abi.prr_decode_step_fused(self.dims, self.buffers(), self.ws, par, st)
        if parity is None:
            self.fused_parity ^= 1
        if swap and self.dims.P > 0:
            self.parity ^= 1

    def device_status(self) -> int:
        return _abi.prr_get_device_status(self.ws)


def summarize_trace(trace, items: dict) -> dict:
    """Per item kind of one fused launch: how many items ran, when the first and last
    started and the last ended (microseconds after the earliest start), and the p50 /
    mean / max item duration.  `trace` is the [items][4] record of prr_step_buffers
    (start ns, end ns, SM << 32 | CTA, item), `items` the kind counts in queue order."""
    import numpy as np
    tr = np.asarray(trace, dtype=np.int64)
    ran = tr[:, 0] > 0
    if not ran.any():
        return {}
    t0 = tr[ran, 0].min()
    out, off = {}, 0
    for kind, cnt in items.items():
        seg = tr[off:off + cnt]
        off += cnt
        seg = seg[seg[:, 0] > 0]
        if len(seg) == 0:
            out[kind] = {"n": 0}
            continue
        st = (seg[:, 0] - t0) / 1e3
        en = (seg[:, 1] - t0) / 1e3
        dur = en - st
        out[kind] = {"n": int(len(seg)), "start_min_us": float(st.min()), "start_max_us": float(st.max()),
                     "end_max_us": float(en.max()), "dur_p50_us": float(np.median(dur)),
                     "dur_mean_us": float(dur.mean()), "dur_max_us": float(dur.max()),
                     "sms": int(len(np.unique(seg[:, 2] >> 32)))}
    return out
