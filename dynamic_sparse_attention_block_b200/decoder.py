"""PRR decode state for one attention layer: device buffers, streams and the step call.

Torch is used for device memory, streams, events and CUDA graphs only; every step of
the path (summaries, selection, speculation, repair, merge, EMA prediction) runs in
libprr_b200.so through the C ABI.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

from . import _abi
from ._abi import Dims


class PRRDecoder:
    """Caller-owned state of the PRR decode step (PRR abstract / method summary: EMA
    predictor, speculative attention overlapped with selection, repair + LSE merge).

    Buffers (row-major), with S = selections per sequence (Hkv; Hq under per-head
    selection):  k_cache/v_cache [B][Hkv][cap][d] bf16, seq_lens [B] int32,
    summ [B][Hkv][maxnb][2][d] bf16, ema [B][S][maxnb] fp64, pred double buffer
    [2][B][S][P] int32, sel/missed [B][S][K], n_missed [B][S], keep [B][S][P],
    speculative partials [B][Hq][P](+[d]) fp32, out [B][Hq][d] fp32, lse [B][Hq] fp32.
    """

    def __init__(self, dims: Dims, device: Optional[torch.device] = None,
                 block_table: Optional[torch.Tensor] = None, rep_offsets: Optional[torch.Tensor] = None):
        """dims.pages > 0 makes the KV cache a paged pool [pages][Hkv][bs][d];
        `block_table` (int32 [B][maxnb], page of block j of sequence b) then defaults to
        block j of sequence b in page b*maxnb + j.  The representative-key selector
        takes `rep_offsets` (uint8 [B][Hkv][maxnb][n_rep], offsets of each block's
        representative tokens inside the block)."""
        if not torch.cuda.is_available():
            raise RuntimeError("PRRDecoder needs a CUDA device")
        _abi.load()
        self.device = torch.device(device or "cuda")
        dev = self.device
        B, Hq, Hkv, d, cap, K, P = dims.B, dims.Hq, dims.Hkv, dims.d, dims.cap_tokens, dims.K, dims.P
        S = dims.sel_heads  # selections per sequence (per-unit arrays are [B][S][...])
        maxnb = dims.maxnb
        self.block_table = None
        if dims.pages > 0:
            if block_table is None:
                block_table = torch.arange(B * maxnb, dtype=torch.int32).view(B, maxnb)
            self.block_table = block_table.to(device=dev, dtype=torch.int32).contiguous()
            self.table_host = self.block_table.cpu().numpy()
            dims = dataclasses.replace(dims, block_table=self.block_table.data_ptr())
            self.k_cache = torch.zeros((dims.pages, Hkv, dims.bs, d), dtype=torch.bfloat16, device=dev)
        else:
            self.k_cache = torch.zeros((B, Hkv, cap, d), dtype=torch.bfloat16, device=dev)
        self.rep_offsets = None
        if dims.selector == "representative":
            if rep_offsets is None or tuple(rep_offsets.shape) != (B, Hkv, maxnb, dims.n_rep):
                raise ValueError("the representative selector needs rep_offsets [B][Hkv][maxnb][n_rep]")
            self.rep_offsets = rep_offsets.to(device=dev, dtype=torch.uint8).contiguous()
            dims = dataclasses.replace(dims, rep_offsets=self.rep_offsets.data_ptr())
        self.dims = dims
        self.v_cache = torch.zeros_like(self.k_cache)
        self.seq_lens = torch.zeros((B,), dtype=torch.int32, device=dev)
        self.summ = torch.zeros((B, Hkv, maxnb, 2, d), dtype=torch.bfloat16, device=dev)
        self.ema = torch.zeros((B, S, maxnb), dtype=torch.float64, device=dev)
        self.pred_buf = torch.full((2, B, S, max(P, 1)), -1, dtype=torch.int32, device=dev)
        self.sel = torch.full((B, S, K), -1, dtype=torch.int32, device=dev)
        self.missed = torch.full((B, S, K), -1, dtype=torch.int32, device=dev)
        self.n_missed = torch.zeros((B, S), dtype=torch.int32, device=dev)
        self.keep = torch.zeros((B, S, max(P, 1)), dtype=torch.uint8, device=dev)
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
        self.stats = None      # optional step counters (enable_stats)

    # ------------------------------------------------------------------ views
    @property
    def pred(self) -> torch.Tensor:
        return self.pred_buf[self.parity]

    @property
    def pred_next(self) -> torch.Tensor:
        return self.pred_buf[1 - self.parity]

    def buffers(self, parity: Optional[int] = None, append: bool = False) -> _abi.PrrStepBuffers:
        """Step buffers; with `append` the step also appends the token held in the
        decoder's k_new / v_new buffers (it then advances seq_lens itself)."""
        par = self.parity if parity is None else parity
        b = _abi.PrrStepBuffers()
        b.q, b.k_cache, b.v_cache = self.q.data_ptr(), self.k_cache.data_ptr(), self.v_cache.data_ptr()
        b.seq_lens, b.summ, b.ema = self.seq_lens.data_ptr(), self.summ.data_ptr(), self.ema.data_ptr()
        b.pred, b.pred_next = self.pred_buf[par].data_ptr(), self.pred_buf[1 - par].data_ptr()
        b.sel, b.missed, b.n_missed = self.sel.data_ptr(), self.missed.data_ptr(), self.n_missed.data_ptr()
        b.keep = self.keep.data_ptr()
        b.part_m, b.part_l, b.part_O = self.part_m.data_ptr(), self.part_l.data_ptr(), self.part_O.data_ptr()
        b.out, b.lse = self.out.data_ptr(), self.lse.data_ptr()
        if append:
            b.k_new, b.v_new = self.k_new.data_ptr(), self.v_new.data_ptr()
        b.trace = self.trace.data_ptr() if self.trace is not None else None
        b.stats = self.stats.data_ptr() if self.stats is not None else None
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

    def fused_items(self, sms: Optional[int] = None) -> dict:
        """Work items of one fused launch, in ticket (and trace record) order: selection
        chunks, finishers, predictor updates, speculative slots, repair items and merges."""
        d = self.dims
        chunk = min(128, max(32, -(-(-(-d.units * d.maxnb // 512)) // 32) * 32))
        rep = min(d.K, max(4, -(-1024 // d.units)))
        return {"sel": d.units * -(-d.maxnb // chunk), "finish": d.units, "ema": d.units, "spec": d.units * d.P,
                "repair": d.units * rep, "combine": d.units * d.group}

    def enable_trace(self, on: bool = True) -> None:
        """Record start/end times of every work item of the fused launches."""
        self.trace = torch.zeros((sum(self.fused_items().values()), 4), dtype=torch.int64,
                                 device=self.device) if on else None

    def trace_summary(self) -> dict:
        """Timeline of the last traced fused launch, per item kind (see summarize_trace)."""
        if self.trace is None:
            raise RuntimeError("tracing is off: call enable_trace() before the step")
        return summarize_trace(self.trace.cpu().numpy())

    STAT_NAMES = ("tie_mask_units", "key_search_units", "take_all_units", "spec_attended",
                  "spec_skipped", "repaired", "reserved6", "reserved7")

    def enable_stats(self, on: bool = True) -> None:
        """Count, over the following steps, which finisher path each unit took and how
        many speculative and repair blocks were attended or skipped (int64 [8] on the
        device, added to by the kernels; read it with stats_dict)."""
        self.stats = torch.zeros((8,), dtype=torch.int64, device=self.device) if on else None

    def stats_dict(self) -> dict:
        if self.stats is None:
            raise RuntimeError("counters are off: call enable_stats() before the steps")
        return dict(zip(self.STAT_NAMES, (int(x) for x in self.stats.cpu().tolist())))


    # ------------------------------------------------------------------ setup
    def load_context(self, b: int, h: int, k: torch.Tensor, v: torch.Tensor) -> None:
        """Write tokens [0, n) of sequence b, KV head h (k, v: [n][d] bf16 on the device)
        into the cache, through the block table when the cache is paged."""
        n, bs = k.shape[0], self.dims.bs
        if self.block_table is None:
            self.k_cache[b, h, :n].copy_(k)
            self.v_cache[b, h, :n].copy_(v)
            return
        nbk = -(-n // bs)
        pages = self.block_table[b, :nbk].long()
        pad = nbk * bs - n  # rows past n in the last page are never read
        kp = torch.nn.functional.pad(k, (0, 0, 0, pad)).view(nbk, bs, -1)
        vp = torch.nn.functional.pad(v, (0, 0, 0, pad)).view(nbk, bs, -1)
        self.k_cache[pages, h] = kp
        self.v_cache[pages, h] = vp

    def prefill(self, k: Optional[torch.Tensor], v: Optional[torch.Tensor], n0) -> None:
        """Start decoding after an initial context: optionally copy it in (k, v
        [B][Hkv][n][d] bf16 with n >= every length, contiguous caches only; else
        load_context wrote it), set the sequence lengths (n0: one length, or one per
        sequence), build all block summaries, reset the EMA and predict from the zero
        state."""
        d = self.dims
        lens = [int(n0)] * d.B if isinstance(n0, int) else [int(x) for x in n0]
        if len(lens) != d.B or min(lens) < 1 or max(lens) > d.cap_tokens:
            raise ValueError(f"need {d.B} lengths in [1, {d.cap_tokens}], got {lens}")
        if k is not None:
            if self.block_table is not None:
                raise ValueError("prefill copies k/v into a contiguous cache only: fill a paged one with load_context")
            if v is None or k.shape != v.shape or k.dim() != 4 or k.shape[2] < max(lens):
                raise ValueError("k and v must both be [B][Hkv][n][d] with n >= every sequence length")
        self._after_caller(self.select_stream)  # k/v (or load_context's writes) come from the caller's stream
        with torch.cuda.stream(self.select_stream):
            if k is not None:
                n = k.shape[2]
                self.k_cache[:, :, :n].copy_(k)
                self.v_cache[:, :, :n].copy_(v)
            self.seq_lens.copy_(torch.tensor(lens, dtype=torch.int32))
            self.ema.zero_()
            self.pred_buf.fill_(-1)
            _abi.prr_workspace_init(self.ws, self.select_stream)
            zeros = torch.zeros((d.B,), dtype=torch.int32, device=self.device)
            ends = torch.tensor(lens, dtype=torch.int32, device=self.device)
            _abi.prr_update_summaries(d, self.k_cache, zeros, ends, None, max(lens), self.summ, self.ws,
                                      self.select_stream)
            self.parity = 0
            if d.P > 0:
                _abi.prr_ema_predict(d, self.ema, None, self.seq_lens, self.pred_buf[0], self.ws,
                                     self.select_stream)
        self.select_stream.synchronize()

    # ------------------------------------------------------------------ checkpoint / resume
    def checkpoint(self) -> dict:
        """Host copies of the state a decode step carries to the next one: the caches,
        sequence lengths, block summaries, EMA state and the current prediction Pred_t
        (and the block table of a paged cache).  The workspace holds nothing that
        outlives a step, so it is not part of the state."""
        self.select_stream.synchronize()
        ck = {"k_cache": self.k_cache.cpu(), "v_cache": self.v_cache.cpu(), "seq_lens": self.seq_lens.cpu(),
              "summ": self.summ.cpu(), "ema": self.ema.cpu(), "pred": self.pred.cpu()}
        if self.block_table is not None:
            ck["block_table"] = self.block_table.cpu()
        return ck

    def restore(self, ck: dict) -> None:
        """Load a checkpoint() into this decoder (same dims): the next step continues
        exactly where the checkpointed decoder stopped."""
        self._after_caller(self.select_stream)
        with torch.cuda.stream(self.select_stream):
            for name in ("k_cache", "v_cache", "seq_lens", "summ", "ema"):
                getattr(self, name).copy_(ck[name])
            if self.block_table is not None:
                self.block_table.copy_(ck["block_table"])
                self.table_host = ck["block_table"].numpy().copy()
            self.parity, self.fused_parity = 0, 0
            self.pred_buf[0].copy_(ck["pred"])
            _abi.prr_workspace_init(self.ws, self.select_stream)
        self.select_stream.synchronize()

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> None:
        """Write the step's token (k_new/v_new [B][Hkv][d] bf16) and advance seq_lens, on
        `stream` (default: the step stream, ordered after the caller's current stream)."""
        st = stream or self.select_stream
        self._after_caller(st)
        _abi.prr_append_kv(self.dims, k_new, v_new, self.seq_lens, self.k_cache, self.v_cache, self.ws, st)

    # ------------------------------------------------------------------ the step
    def _after_caller(self, st) -> None:
        """Order `st` after the caller's current stream, on which the step's input
        tensors were produced (a no-op when the caller already runs on `st`)."""
        cur = torch.cuda.current_stream(self.device)
        if cur != st:
            st.wait_stream(cur)

    def step(self, q: Optional[torch.Tensor] = None, timing: Optional[dict] = None,
             swap: bool = True, append: bool = False) -> None:
        """One decode step on the state's streams (q [B][Hq][d] bf16 is copied into the
        step's query buffer first when given).  Swaps Pred_t / Pred_{t+1} afterwards."""
        if q is not None:
            self._after_caller(self.select_stream)
            with torch.cuda.stream(self.select_stream):
                self.q.copy_(q)
        _abi.prr_decode_step(self.dims, self.buffers(append=append), self.ws, self.select_stream,
                             self.spec_stream, self.events(timing))
        if swap and self.dims.P > 0:
            self.parity ^= 1

    def step_fused(self, q: Optional[torch.Tensor] = None, stream=None, swap: bool = True,
                   parity: Optional[int] = None, k_new: Optional[torch.Tensor] = None,
                   v_new: Optional[torch.Tensor] = None, append: bool = False) -> None:
        """The same step as one persistent launch on `stream` (default: select_stream).
        With k_new / v_new ([B][Hkv][d] bf16, copied into the decoder's token buffers)
        or `append`, the launch also appends the step's token (no separate append)."""
        st = stream or self.select_stream
        if q is not None or k_new is not None:
            self._after_caller(st)
        with torch.cuda.stream(st):
            if q is not None:
                self.q.copy_(q)
            if k_new is not None:
                self.k_new.copy_(k_new)
                self.v_new.copy_(v_new)
        par = self.fused_parity if parity is None else parity
        _abi.prr_decode_step_fused(self.dims, self.buffers(append=append or k_new is not None), self.ws, par, st)
        if parity is None:
            self.fused_parity ^= 1
        if swap and self.dims.P > 0:
            self.parity ^= 1

    def device_status(self) -> int:
        return _abi.prr_get_device_status(self.ws)


KINDS = {1: "sel", 2: "spec", 3: "repair", 4: "ema", 5: "combine", 6: "finish"}


def summarize_trace(trace) -> dict:
    """Per item kind of one fused launch: how many items ran, when the first and last
    started and the last ended (microseconds after the earliest start), and the p50 /
    mean / max item duration; "finisher" repeats the count and durations of the top-K
    finisher items.  `trace` is the [records][4] array of prr_step_buffers (start ns,
    end ns, SM << 32 | CTA index, kind)."""
    import numpy as np
    tr = np.asarray(trace, dtype=np.int64)
    ran = tr[:, 0] > 0
    if not ran.any():
        return {}
    t0 = tr[ran, 0].min()
    out = {"end_us": float((tr[ran, 1].max() - t0) / 1e3)}
    kinds = tr[:, 3] & 0xFFFFFFFF
    fin = ran & (kinds == 6)
    if fin.any():
        f = (tr[fin, 1] - tr[fin, 0]) / 1e3
        out["finisher"] = {"n": int(len(f)), "dur_p50_us": float(np.median(f)), "dur_max_us": float(f.max())}
    for code, kind in KINDS.items():
        seg = tr[ran & (kinds == code)]
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
