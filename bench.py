#!/usr/bin/env python
"""Benchmark of the PRR decode step (select + speculate + repair): one JSON line.

Metric: microseconds per decode step and KV-tokens/s (B * n per step, the context
served), with the fraction of the HBM roofline.  The headline workload is the
largest single-GPU configuration, batched long-context decode at 128K (B=16, 32
query / 8 KV heads, d 128, 128-token blocks, top-32, budget 32).  At N=1 the same line
also carries one record per other configuration ("records"): 512K context, the
Llama-3.1-8B-shaped 32K layer, and the 64K repair sweep at six forced predictor
overlaps.  Inputs are seeded synthetic data (workloads/).

Timing: W warm-up steps, then exactly K steps, each a CUDA-graph replay of the whole
step bracketed by CUDA events on the replay stream; a 256 MB write flushes L2 and the
next token's KV append runs between steps, outside the events.  Per-kernel durations
of the two-stream variant come from timing events recorded inside its graph.

Under torchrun (N > 1) every rank runs an independent replica on its own sequences
(weak scaling, no collective on the data path); value = tokens of all ranks / the max
over ranks of the summed step time.

--impl reference times the fp64 CPU oracle on the host cores on the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from concurrent.futures import ThreadPoolExecutor

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "µs/decode step & KV-tokens/s (select+speculate+repair), % of 8 TB/s HBM roofline"
UNIT = "KV-tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
HEADLINE = "batched_128k"
RECORDS = ("long_512k", "llama8b_32k", "repair_sweep_64k")


# ----------------------------------------------------------------------------- helpers

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def rank_workload(w: W.Workload, rank: int) -> W.Workload:
    return w if rank == 0 else w.with_(seed=w.seed + 7919 * rank)


def host_cache(w: W.Workload, cap: int, threads: int = 0):
    """KV bit patterns [B][Hkv][cap][d] with the first N0 tokens of every slice filled
    (one generator stream per slice, so slices are filled in parallel threads)."""
    kc = np.zeros((w.B, w.Hkv, cap, w.d), np.uint16)
    vc = np.zeros_like(kc)

    def fill(i):
        b, h = divmod(i, w.Hkv)
        k0, v0 = W.kv_prefix(w, b, h)
        kc[b, h, :w.N0], vc[b, h, :w.N0] = k0, v0

    with ThreadPoolExecutor(threads or min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, range(w.B * w.Hkv)))
    return kc, vc


def appended(w: W.Workload, steps: int):
    kn = np.empty((steps, w.B, w.Hkv, w.d), np.uint16)
    vn = np.empty_like(kn)
    for b in range(w.B):
        for h in range(w.Hkv):
            k, v = W.kv_appended(w, b, h, steps)
            kn[:, b, h], vn[:, b, h] = k, v
    return kn, vn


def algorithmic_bytes(w: W.Workload, n: int) -> dict:
    """Bytes a step must move: all block summaries + K and V of the true top-K blocks."""
    nb = w.nb(n)
    keff = min(w.K, nb)
    summ = w.units * nb * 4 * w.d
    kv = w.units * keff * w.bs * w.d * 2 * 2  # tail block counted whole (upper bound)
    return {"summaries": summ, "kv": kv, "total": summ + kv}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, period_ms: int = 50):
        self.lines = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(period_ms), "-i", gpu_id],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def wait_first(self, timeout=5.0):
        t0 = time.time()
        while self.proc and not self.lines and time.time() - t0 < timeout:
            time.sleep(0.01)

    def stop(self) -> dict:
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names[1:], parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def elapsed_ms(a, b) -> float:
    """cuEventElapsedTime on two events recorded by the library through their raw
    handles (torch's own elapsed_time only accepts events torch itself recorded)."""
    from cuda.bindings import driver
    err, ms = driver.cuEventElapsedTime(driver.CUevent(init_value=a.cuda_event),
                                        driver.CUevent(init_value=b.cuda_event))
    if err != driver.CUresult.CUDA_SUCCESS:
        raise RuntimeError(f"cuEventElapsedTime: {err}")
    return float(ms)


def kernel_spans(marks) -> dict:
    """Per-kernel device durations (ms) of the last step from its timing marks."""
    return {
        "select": elapsed_ms(marks["t_begin"], marks["t_select_end"]),
        "repair": elapsed_ms(marks["t_select_end"], marks["t_repair_end"]),
        "combine": elapsed_ms(marks["t_combine_begin"], marks["t_combine_end"]),
        "spec": elapsed_ms(marks["t_spec_begin"], marks["t_spec_end"]),
        "ema": elapsed_ms(marks["t_ema_begin"], marks["t_ema_end"]),
    }


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dynamic_sparse_attention_block_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it was taken
    on the current kernel sources (profiles/traffic.txt: kernel workload sha bytes)."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    sha = kernel_source_sha()
    with open(p) as fh:
        for ln in fh:
            parts = ln.split()
            if len(parts) >= 4 and not ln.startswith("#") and parts[0] == kernel \
                    and parts[1] == workload and parts[2] == sha:
                return float(parts[3])
    return None


def reduce_over_ranks(tokens: float, seconds: float, e2e_value, world: int, device: str):
    """Whole-job numbers of a replicas run: tokens summed over ranks, time = the max
    over ranks (the slowest replica bounds the job), end-to-end throughput summed.
    Every rank makes the same collective calls in the same order."""
    if world <= 1:
        return float(tokens), float(seconds), e2e_value
    import torch
    import torch.distributed as dist
    v = torch.tensor([float(tokens), float(e2e_value or 0.0)], dtype=torch.float64, device=device)
    m = torch.tensor([float(seconds)], dtype=torch.float64, device=device)
    dist.all_reduce(v, op=dist.ReduceOp.SUM)
    dist.all_reduce(m, op=dist.ReduceOp.MAX)
    return v[0].item(), m[0].item(), (v[1].item() if e2e_value is not None else None)


# ----------------------------------------------------------------------------- CPU oracle timing

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for ln in fh:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_run(w: W.Workload, warmup: int, steps: int, budget_s: float, nthreads: int, caches=None):
    """Time the fp64 oracle's decode step on the host.  Returns (tokens/s, seconds per
    step, steps timed, units per step, threads).  Each step runs every (sequence, KV
    head) unit; the number of timed steps is cut so the loop stays within budget_s.
    `caches` = (kc, vc) with room for warmup + steps tokens after N0 may be passed in."""
    import oracle as OR
    o = OR.default()
    total = warmup + steps
    if caches is None:
        kc, vc = host_cache(w, w.N0 + total)
    else:
        kc, vc = caches
        assert kc.shape[2] >= w.N0 + total
    cap = kc.shape[2]
    kn, vn = appended(w, total)
    qs = W.queries(w, total)
    st = OR.new_state(w.B, w.Hkv, cap, w.bs, w.d)

    def build(i):
        b, h = divmod(i, w.Hkv)
        lo, hi = o.build_summaries(kc[b, h], w.N0, w.bs)
        st["smin"][b, h, :lo.shape[0]], st["smax"][b, h, :lo.shape[0]] = lo, hi

    with ThreadPoolExecutor(min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(build, range(w.B * w.Hkv)))
    dims = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, bs=w.bs, cap=cap, K=w.K, P=w.P, alpha=w.alpha,
                scale=w.scale())
    pred = np.full((w.B, w.Hkv, max(w.P, 1)), -1, np.int32)
    pred[:, :, :min(w.P, w.nb(w.N0))] = np.arange(min(w.P, w.nb(w.N0)))
    times, tokens, used = [], 0, 1
    t_start = time.perf_counter()
    for t in range(total):
        n = w.N0 + t + 1
        kc[:, :, n - 1], vc[:, :, n - 1] = kn[t], vn[t]
        seq = np.full(w.B, n, np.int32)
        t0 = time.perf_counter()
        r = o.decode_step(dims, qs[t], kc, vc, seq, pred, st, nthreads=nthreads)
        dt = time.perf_counter() - t0
        used = r["threads"]
        pred = r["pred_next"]
        if t >= warmup:
            times.append(dt)
            tokens += w.B * n
        if t >= warmup and time.perf_counter() - t_start > budget_s:
            break
    secs = sum(times)
    return tokens / secs, secs / max(len(times), 1), len(times), w.units, used


def cpu_baseline(w: W.Workload, args, caches=None) -> dict:
    """The oracle's step on all host cores (OpenMP over units), timed on a bounded sample
    of the workload after 2 warm-up steps, and its rate on one thread (one cold step).
    `caches` needs room for 2 + args.cpu_max_steps tokens after N0."""
    threads = os.cpu_count() or 1
    value, sps, nsteps, units, used = oracle_run(w, 2, args.cpu_max_steps, args.cpu_budget_s, threads,
                                                 caches=caches)
    v1, sps1, _, _, used1 = oracle_run(w, 0, 1, 0.0, 1, caches=caches)
    return {"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"{nsteps} oracle decode steps of {w.name} after 2 warm-up steps "
                      f"({units} units per step, ~{args.cpu_budget_s:.0f} s budget)",
            "cpu_model": cpu_model(),
            "single_thread": {"value": v1, "unit": UNIT, "cores": used1, "ms_per_step": sps1 * 1e3,
                              "sample": f"1 oracle decode step of {w.name} on one thread"}}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    w = base_workload(args)
    threads = os.cpu_count() or 1
    value, sps, nsteps, units, used = oracle_run(w, args.warmup, args.steps, args.ref_budget_s, threads)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": nsteps, "warmup": args.warmup, "ms_per_step": sps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args),  # the GPU arm's config, key for key
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
                         "sample": f"{nsteps} full oracle decode steps ({units} (sequence, KV head) "
                                   f"units each) of {w.name}, OpenMP over units",
                         "cpu_model": cpu_model(),
                         "caches": "no flush between steps on the host; each step streams the "
                                   "whole KV cache, which is far larger than the host caches"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    if nsteps < args.steps:
        line["note"] = f"timed {nsteps} of {args.steps} requested steps (time budget {args.ref_budget_s}s)"
    print(json.dumps(line), flush=True)
    return 0


def base_workload(args) -> W.Workload:
    w = W.workload(args.workload)
    batch = getattr(args, "batch", 0)
    return w.with_(B=batch) if batch > 0 else w


def workload_config(w: W.Workload, args) -> dict:
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "context": w.N0,
            "block": w.bs, "top_k": w.K, "budget_P": w.P, "alpha": w.alpha, "qk": w.qk,
            "walk_p": w.walk_p, "l2": "256 MB write between timed steps",
            "parallelism": f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU"}


# ----------------------------------------------------------------------------- GPU arm

class Run:
    """One workload on the GPU: decoder, seeded inputs, graphs of both step variants."""

    def __init__(self, w: W.Workload, args, extra_steps: int, caches=None):
        import torch
        from dynamic_sparse_attention_block_b200 import Dims, PRRDecoder, _abi
        self.torch, self.abi = torch, _abi
        self.w = w
        self.total = extra_steps
        cap = w.N0 + extra_steps
        self.dims = Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, bs=w.bs, cap_tokens=cap, K=w.K, P=w.P,
                         alpha=w.alpha)
        self.dec = dec = PRRDecoder(self.dims)
        kc, vc = caches if caches is not None else host_cache(w, w.N0)
        for b in range(w.B):
            for h in range(w.Hkv):
                dec.k_cache[b, h, :w.N0].copy_(torch.from_numpy(kc[b, h, :w.N0].view(np.int16)).view(torch.bfloat16))
                dec.v_cache[b, h, :w.N0].copy_(torch.from_numpy(vc[b, h, :w.N0].view(np.int16)).view(torch.bfloat16))
        torch.cuda.synchronize()
        dec.prefill(dec.k_cache[:, :, :w.N0], dec.v_cache[:, :, :w.N0], w.N0)
        # step counters: on before the graphs are captured (their kernels keep the pointer)
        # and for the decoder's whole life
        dec.enable_stats()
        self.kn, self.vn = appended(w, extra_steps)
        self.qs = W.queries(w, extra_steps)
        self.kn_d = torch.from_numpy(self.kn.view(np.int16)).cuda().view(torch.bfloat16)
        self.vn_d = torch.from_numpy(self.vn.view(np.int16)).cuda().view(torch.bfloat16)
        self.qs_d = torch.from_numpy(self.qs.view(np.int16)).cuda().view(torch.bfloat16)
        self.flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        self.main = torch.cuda.current_stream()
        self.marks = {nm: torch.cuda.Event(enable_timing=True) for nm in _abi.TIMING_MARKS}
        for ev in self.marks.values():  # torch creates the CUDA event on its first record
            ev.record(self.main)
        self.t = 0
        self.graphs = {}

    def prepare(self, flush_l2=True):
        self.dec.append(self.kn_d[self.t], self.vn_d[self.t], stream=self.main)
        self.dec.q.copy_(self.qs_d[self.t])
        if flush_l2:
            self.flush.zero_()

    def force_prediction(self, overlap, level):
        """Replace Pred_t by a set with a forced overlap with this step's true top-K.
        S_t comes from the library (fold the appended key, then select); the forced set
        is built on the host from the seeded generator.  Runs before the L2 flush."""
        w, dec, dims, _abi = self.w, self.dec, self.dims, self.abi
        _abi.prr_update_summaries(dims, dec.k_cache, None, None, dec.seq_lens, 1, dec.summ, dec.ws, self.main)
        _abi.prr_select_topk(dims, dec.q, dec.summ, dec.seq_lens, dec.pred, dec.sel, dec.missed,
                             dec.n_missed, dec.keep, dec.ws, self.main)
        sel = dec.sel.cpu().numpy()
        nb = w.nb(w.N0 + self.t + 1)
        ph = np.full((w.B, w.Hkv, max(w.P, 1)), -1, np.int32)
        for b in range(w.B):
            for h in range(w.Hkv):
                fp = W.forced_prediction(w, sel[b, h][sel[b, h] >= 0], nb, overlap, level, self.t, b, h)
                ph[b, h, :len(fp)] = fp[:w.P]
        dec.pred.copy_(self.torch.from_numpy(ph))

    def capture(self, streams: bool, append_in_step: bool = False):
        """Eager warm-up of each step variant, then one graph per parity.  With
        `append_in_step` also the fused step that appends its own token from the
        decoder's k_new / v_new buffers (the end-to-end path)."""
        torch, dec = self.torch, self.dec
        for fused in ((True, False) if streams else (True,)):
            self.prepare()
            self.main.synchronize()
            if fused:
                dec.step_fused(stream=self.main)
            else:
                dec.step(timing=self.marks)
            torch.cuda.synchronize()
            self.t += 1
        saved = (dec.parity, dec.fused_parity)
        for par in (0, 1):
            dec.parity = par
            for cpar in (0, 1):  # control-word copy of the fused launch
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=dec.select_stream):
                    dec.step_fused(swap=False, parity=cpar)
                self.graphs[("fused", par, cpar)] = g
                if append_in_step:
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=dec.select_stream):
                        dec.step_fused(swap=False, parity=cpar, append=True)
                    self.graphs[("fused_app", par, cpar)] = g
            if streams:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=dec.select_stream):
                    dec.step(timing=self.marks, swap=False)
                self.graphs[("streams", par)] = g
        dec.parity, dec.fused_parity = saved
        torch.cuda.synchronize()

    def replay(self, kind):
        dec = self.dec
        if kind in ("fused", "fused_app"):
            self.graphs[(kind, dec.parity, dec.fused_parity)].replay()
            dec.fused_parity ^= 1  # consecutive fused launches alternate their control words
        else:
            self.graphs[("streams", dec.parity)].replay()
        if self.dims.P > 0:
            dec.parity ^= 1

    def release(self):
        for g in self.graphs.values():
            g.reset()
        self.graphs.clear()

    # ------------------------------------------------------------------ timed loops
    def timed_fused(self, steps, level=None, after=None):
        """`steps` fused steps, each bracketed by events; `after()` runs after each step
        is enqueued, outside the events.  Returns per-step ms and context lengths."""
        torch, dec = self.torch, self.dec
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ns = []
        for i in range(steps):
            if level is None:
                self.prepare()
            else:
                self.prepare(flush_l2=False)
                self.force_prediction(level[1], level[0])
                self.flush.zero_()
            starts[i].record(self.main)
            self.replay("fused")
            ends[i].record(self.main)
            if after is not None:
                after()
            ns.append(self.w.N0 + self.t + 1)
            self.t += 1
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in zip(starts, ends)], ns

    def timed_streams(self, steps, level=None):
        torch = self.torch
        sa = torch.cuda.Event(enable_timing=True)
        sb = torch.cuda.Event(enable_timing=True)
        s_ms, overlap_frac = [], []
        kern = {"select": [], "repair": [], "combine": [], "spec": [], "ema": []}
        for _ in range(steps):
            if level is None:
                self.prepare()
            else:
                self.prepare(flush_l2=False)
                self.force_prediction(level[1], level[0])
                self.flush.zero_()
            sa.record(self.main)
            self.replay("streams")
            sb.record(self.main)
            self.main.synchronize()
            s_ms.append(sa.elapsed_time(sb))
            for name, dur in kernel_spans(self.marks).items():
                kern[name].append(dur)
            m = self.marks
            a1 = elapsed_ms(m["t_begin"], m["t_select_end"])
            b0 = elapsed_ms(m["t_begin"], m["t_spec_begin"])
            b1 = elapsed_ms(m["t_begin"], m["t_spec_end"])
            if b1 > b0:
                overlap_frac.append(max(0.0, min(a1, b1) - max(0.0, b0)) / (b1 - b0))
            self.t += 1
        return {"us_per_step": statistics.mean(s_ms) * 1e3, "steps": steps,
                "kernels_us": {k: statistics.mean(v) * 1e3 for k, v in kern.items()},
                "spec_select_overlap": statistics.mean(overlap_frac) if overlap_frac else None,
                "gpu_launches_per_step": 4 + (1 if self.dims.P > 0 else 0)}


def step_record(run: Run, ms, ns, hbm_peak, stats: dict) -> dict:
    """Numbers of one set of timed fused steps."""
    w = run.w
    algo = statistics.mean(algorithmic_bytes(w, n)["total"] for n in ns)
    mean_ms = statistics.mean(ms)
    achieved = algo / (mean_ms * 1e-3) / 1e9
    units_steps = len(ms) * w.units
    keff = min(w.K, w.nb(w.N0))
    fin = stats["tie_mask_units"] + stats["key_search_units"] + stats["take_all_units"]
    block_bytes = w.bs * w.d * 2 * 2
    moved = statistics.mean(w.units * w.nb(n) * 4 * w.d for n in ns) + \
        (stats["spec_attended"] + stats["repaired"]) * block_bytes / len(ms)
    return {
        "us_per_step": mean_ms * 1e3, "us_per_step_p50": statistics.median(ms) * 1e3,
        "us_per_step_p90": float(np.percentile(ms, 90)) * 1e3, "steps": len(ms),
        "kv_tokens_per_s": sum(w.B * n for n in ns) / (sum(ms) * 1e-3),
        "attended_tokens_per_s": w.units * keff * w.bs / (mean_ms * 1e-3),
        "algorithmic_bytes_per_step": algo, "achieved_gbs": achieved,
        "frac_of_measured": achieved / hbm_peak, "frac_of_8tbs": achieved / NOMINAL_HBM_GBS,
        "moved_bytes_per_step": moved,
        "repaired_blocks_per_unit": stats["repaired"] / units_steps,
        "spec_blocks_attended_per_unit": stats["spec_attended"] / units_steps,
        "spec_blocks_skipped_per_unit": stats["spec_skipped"] / units_steps,
        "finisher_paths": {"tie_masks": stats["tie_mask_units"] / max(fin, 1),
                           "key_search": stats["key_search_units"] / max(fin, 1),
                           "take_all": stats["take_all_units"] / max(fin, 1)},
    }


def measure(w: W.Workload, args, hbm_peak, *, e2e=False, streams=False, caches=None) -> dict:
    """All timed numbers of one workload (and, for the repair sweep, of each forced
    overlap level).  Returns the record, the tokens and the seconds it timed."""
    import torch
    steps = args.steps
    levels = list(enumerate(w.forced_overlaps)) if w.forced_overlaps else [None]
    n_str = min(steps, 20) if streams else 0
    per_level_streams = 4 if (streams and w.forced_overlaps) else 0
    total = 2 + args.warmup + len(levels) * (steps + per_level_streams) + (steps if e2e else 0) + \
        (n_str if not w.forced_overlaps else 0) + 8
    run = Run(w, args, total, caches)
    dec = run.dec
    run.capture(streams, append_in_step=e2e)
    for _ in range(args.warmup):
        run.prepare()
        run.replay("fused")
        run.t += 1
    torch.cuda.synchronize()

    clocks = ClockSampler(f"GPU-{torch.cuda.get_device_properties(torch.cuda.current_device()).uuid}")
    clocks.wait_first()
    keff = min(w.K, w.nb(w.N0))
    all_ms, all_ns, rows = [], [], []
    for lvl in levels:
        dec.stats.zero_()
        keep_sum = torch.zeros((), dtype=torch.int64, device="cuda")

        def count_keep():  # kept predicted slots of each step, summed on the device
            keep_sum.add_(dec.keep.sum())

        ms, ns = run.timed_fused(steps, lvl, after=count_keep)
        st = dec.stats_dict()
        rec = step_record(run, ms, ns, hbm_peak, st)
        rec["predictor_overlap"] = keep_sum.item() / (steps * w.units * keff) if w.P > 0 else 0.0
        all_ms += ms
        all_ns += ns
        if lvl is not None:
            rec = {"overlap": lvl[1], "kept_blocks": W.forced_kept_count(lvl[1], keff), **rec}
            if per_level_streams:
                sp = run.timed_streams(per_level_streams, lvl)
                rec["streams_us_per_step"] = sp["us_per_step"]
                rec["streams_kernels_us"] = sp["kernels_us"]
        rows.append(rec)
    clk = clocks.stop()
    status = dec.device_status()
    if w.forced_overlaps:
        out = {"workload": w.name, "config": workload_config(w, args), "levels": rows,
               "us_per_step": statistics.mean(all_ms) * 1e3}
    else:
        out = {"workload": w.name, "config": workload_config(w, args), **rows[0]}
    out["clocks"] = clk
    if n_str and not w.forced_overlaps:
        out["streams_path"] = run.timed_streams(n_str)
        status = status or dec.device_status()

    if e2e:
        out["e2e"] = measure_e2e(run, steps)
        status = status or dec.device_status()
    out["device_status"] = status
    tokens = sum(w.B * n for n in all_ns)
    secs = sum(all_ms) / 1e3
    run.release()
    del run, dec
    torch.cuda.empty_cache()
    return out, tokens, secs, all_ms


def measure_e2e(run: Run, steps: int) -> dict:
    """The same step through the public API with host buffers: the step's inputs as the
    decoder lays them out, [q | k_new | v_new], one pinned host row per step; the
    outputs [out | lse] come back in one copy.  Copies are inside the timed region."""
    torch, dec = run.torch, run.dec
    total = run.total
    nq, nkv = dec.q.numel(), dec.k_new.numel()
    in_h = torch.empty((total, nq + 2 * nkv), dtype=torch.bfloat16).pin_memory()
    in_h[:, :nq] = torch.from_numpy(run.qs.reshape(total, -1).view(np.int16)).view(torch.bfloat16)
    in_h[:, nq:nq + nkv] = torch.from_numpy(run.kn.reshape(total, -1).view(np.int16)).view(torch.bfloat16)
    in_h[:, nq + nkv:] = torch.from_numpy(run.vn.reshape(total, -1).view(np.int16)).view(torch.bfloat16)
    out_h = torch.empty(dec.io_out.shape, dtype=torch.float32).pin_memory()
    e_tokens = 0
    es = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ee = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    finite = True
    for i in range(steps):
        run.flush.zero_()
        es[i].record(run.main)
        dec.io_in.copy_(in_h[run.t], non_blocking=True)
        run.replay("fused_app")  # appends the token inside the launch
        out_h.copy_(dec.io_out, non_blocking=True)
        ee[i].record(run.main)
        run.main.synchronize()
        finite = finite and bool(np.all(np.isfinite(out_h.numpy())))
        e_tokens += run.w.B * (run.w.N0 + run.t + 1)
        run.t += 1
    e_ms = [a.elapsed_time(b) for a, b in zip(es, ee)]
    return {"value": e_tokens / (sum(e_ms) / 1e3), "unit": UNIT, "h2d_bytes_per_step": in_h[0].numel() * 2,
            "d2h_bytes_per_step": out_h.numel() * 4, "ms_per_step": statistics.mean(e_ms),
            "finite": finite,
            "path": "one H2D of [q | k_new | v_new], the fused step graph (it appends the token "
                    "itself), one D2H of [out | lse]; pinned host buffers"}


def run_gpu(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    w = rank_workload(base_workload(args), rank)
    hbm_peak, peak_kind = measured_peaks()

    # host caches of the headline workload: shared by the CPU baseline and the GPU run
    cpu = None
    cpu_steps = 2 + args.cpu_max_steps
    caches = host_cache(w, w.N0 + (cpu_steps if rank == 0 and world == 1 and not args.no_cpu_baseline else 0))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args, caches)
        # the oracle appended its own tokens past N0; the GPU run reads only [0, N0)

    head, tokens, secs, step_ms = measure(w, args, hbm_peak, e2e=not args.no_e2e,
                                         streams=not args.no_streams, caches=caches)
    del caches
    records = []
    if world == 1 and not args.no_records:
        for name in args.records.split(","):
            if name and name != w.name:
                rec, _, _, _ = measure(W.workload(name), args, hbm_peak, streams=not args.no_streams)
                records.append(rec)

    status = head["device_status"] or max((r["device_status"] for r in records), default=0)
    if head.get("e2e") and not head["e2e"]["finite"]:
        status = status or -1

    e2e = head.get("e2e")
    tot_tokens, max_time, e2e_total = reduce_over_ranks(tokens, secs, e2e["value"] if e2e else None,
                                                        world, "cuda")
    if e2e is not None:
        e2e = {k: v for k, v in e2e.items() if k != "finite"}
        e2e["value"] = e2e_total
    value = tot_tokens / max_time
    traffic = recorded_traffic("fused_step_kernel", w.name)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": head["steps"],
        "warmup": args.warmup, "ms_per_step": head["us_per_step"] / 1e3, "us_per_step": head["us_per_step"],
        "us_per_step_p50": head["us_per_step_p50"], "us_per_step_p90": head["us_per_step_p90"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(w, args),
        "roofline": {"bound": "hbm", "kernel": "fused_step_kernel", "achieved": head["achieved_gbs"],
                     "peak": hbm_peak, "unit": "GB/s", "frac": head["frac_of_measured"], "traffic": traffic,
                     "peak_kind": f"{peak_kind} copy bandwidth (burst)",
                     "algorithmic_bytes_per_launch": head["algorithmic_bytes_per_step"],
                     "avg_launch_us": head["us_per_step"]},
        "step_roofline": {"algorithmic_bytes_per_step": head["algorithmic_bytes_per_step"],
                          "achieved_gbs": head["achieved_gbs"], "frac_of_8tbs": head["frac_of_8tbs"],
                          "frac_of_measured": head["frac_of_measured"],
                          "moved_bytes_per_step": head["moved_bytes_per_step"]},
        "predictor_overlap": head["predictor_overlap"],
        "repaired_blocks_per_unit": head["repaired_blocks_per_unit"],
        "finisher_paths": head["finisher_paths"],
        "streams_path": head.get("streams_path"),
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": head["steps"],
        "clocks": head["clocks"], "device_status": status,
        "records": records,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0 if status == 0 else 1


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("prr", "reference"), default="prr")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(W.WORKLOADS))
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (reduced cases for profiler captures)")
    ap.add_argument("--records", default=",".join(RECORDS),
                    help="comma-separated workloads measured after the headline (N=1 only)")
    ap.add_argument("--no-records", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-streams", action="store_true", help="skip the two-stream comparison run")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--cpu-max-steps", type=int, default=400)
    ap.add_argument("--ref-budget-s", type=float, default=150.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
