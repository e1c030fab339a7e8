"""Run a seeded workload through the CUDA decode path (C ABI via the Python binding)
and through the fp64 oracle, step by step, and collect a comparison report."""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Sequence, Tuple

import numpy as np
import torch

import oracle as OR
import workloads as W
from dynamic_sparse_attention_block_b200 import Dims, PRRDecoder
from tests.prr_harness import Report, UnitOracle, check_selection, compare_attention, pad


def to_dev_bits(a: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bit patterns -> device bf16 tensor (bit-for-bit)."""
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def shuffled_block_table(w: W.Workload, maxnb: int, spare: int, seed: int = 5):
    """A paged layout for the test: every block of every sequence gets its own page, the
    pages in a seeded random order inside a pool with `spare` pages left unused."""
    pages = w.B * maxnb + spare
    perm = np.random.default_rng(seed).permutation(pages)[:w.B * maxnb]
    return torch.from_numpy(perm.astype(np.int32).reshape(w.B, maxnb)), pages


def make_decoder(w: W.Workload, steps: int, cap_extra: int = 0, paged: bool = False) -> Tuple[PRRDecoder, Dims]:
    cap = w.N0 + steps + cap_extra
    dims = Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, bs=w.bs, cap_tokens=cap, K=w.K, P=w.P,
                alpha=w.alpha, selector=w.selector, n_sink=w.n_sink, n_local=w.n_local, n_rep=w.n_rep)
    table = None
    if paged:
        table, pages = shuffled_block_table(w, dims.maxnb, spare=7)
        dims = dataclasses.replace(dims, pages=pages)
    reps = None
    if w.selector == "representative":
        reps = torch.from_numpy(np.stack([np.stack([W.rep_offsets(w, b, h, dims.maxnb) for h in range(w.Hkv)])
                                          for b in range(w.B)]))
    dec = PRRDecoder(dims, block_table=table, rep_offsets=reps)
    for b in range(w.B):
        for h in range(w.Hkv):
            k0, v0 = W.kv_prefix(w, b, h, w.n0(b))
            dec.load_context(b, h, to_dev_bits(k0), to_dev_bits(v0))
    torch.cuda.synchronize()
    dec.prefill(None, None, [w.n0(b) for b in range(w.B)])
    return dec, dec.dims


def appended_tokens(w: W.Workload, steps: int):
    kn = np.empty((steps, w.B, w.Hkv, w.d), np.uint16)
    vn = np.empty_like(kn)
    for b in range(w.B):
        for h in range(w.Hkv):
            k, v = W.kv_appended(w, b, h, steps)
            kn[:, b, h], vn[:, b, h] = k, v
    return kn, vn


def run_parity(w: W.Workload, steps: int, units: Optional[Sequence[Tuple[int, int]]] = None,
               forced: Optional[Tuple[float, int]] = None, graph: bool = False,
               mode: str = "fused", append: str = "host", paged: bool = False) -> Report:
    """Compare `steps` decode steps.  `units` samples the (b, kvh) pairs the oracle
    follows (default: all).  `forced` = (overlap, level) replaces the predictor's output
    with a predicted set forced to that overlap with the oracle's true set (all units
    are then followed).  `mode` selects the step implementation: "fused" (one
    persistent launch) or "streams" (two streams, one launch per kernel).  `append`
    selects who appends each step's token: "host" (prr_append_kv before the step) or
    "step" (the step itself, from the decoder's k_new / v_new buffers).  `paged` puts
    the KV cache in a pool of pages in shuffled order behind a block table."""
    o = OR.default()
    all_units = [(b, h) for b in range(w.B) for h in range(w.sel_heads)]
    if units is None or forced is not None:
        units = all_units
    uo: Dict[Tuple[int, int], UnitOracle] = {u: UnitOracle.create(w, u[0], u[1], steps, o) for u in units}
    dec, dims = make_decoder(w, steps, paged=paged)
    kn, vn = appended_tokens(w, steps)
    qs = W.queries(w, steps)
    rep = Report()
    gaussian = w.qk == "gauss"
    graphs = {}
    in_step = append == "step"
    for t in range(steps):
        if in_step:  # on the step's stream, ahead of the launch that reads them
            with torch.cuda.stream(dec.select_stream):
                dec.k_new.copy_(to_dev_bits(kn[t]))
                dec.v_new.copy_(to_dev_bits(vn[t]))
        else:
            dec.append(to_dev_bits(kn[t]), to_dev_bits(vn[t]))
        q_dev = to_dev_bits(qs[t])
        sel_info = {u: uo[u].select(t, qs[t]) for u in units}
        if forced is not None:
            overlap, level = forced
            pred_host = np.full((w.B, w.sel_heads, w.P), -1, np.int32)
            for (b, h), (n, nb, qg, s, sel) in sel_info.items():
                fp = W.forced_prediction(w, sel, nb, overlap, level, t, b, h)
                pred_host[b, h, :len(fp)] = fp
                uo[(b, h)].pred = fp
            dec.pred.copy_(torch.from_numpy(pred_host))
        pred_used = dec.pred.clone()
        if graph and t >= 2:  # steps 0-1 run eagerly first (warm-up before capture)
            key = (dec.parity, dec.fused_parity)
            if key not in graphs:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=dec.select_stream):
                    if mode == "fused":
                        dec.step_fused(swap=False, parity=dec.fused_parity, append=in_step)
                    else:
                        dec.step(swap=False, append=in_step)
                graphs[key] = g
            dec.q.copy_(q_dev)
            torch.cuda.synchronize()
            graphs[key].replay()
            if mode == "fused":
                dec.fused_parity ^= 1
            if dims.P > 0:
                dec.parity ^= 1
        elif mode == "fused":
            dec.step_fused(q_dev, append=in_step)
        else:
            dec.step(q_dev, append=in_step)
        torch.cuda.synchronize()
        status = dec.device_status()
        if status != 0:
            rep.fail(f"step {t}: device status {status}")
            return rep
        g_sel = dec.sel.cpu().numpy()
        g_missed = dec.missed.cpu().numpy()
        g_nm = dec.n_missed.cpu().numpy()
        g_keep = dec.keep.cpu().numpy()
        g_pred_used = pred_used.cpu().numpy()
        g_pred_next = dec.pred.cpu().numpy() if dims.P > 0 else None  # swapped: now Pred_{t+1}
        g_out = dec.out.cpu().numpy()
        g_lse = dec.lse.cpu().numpy()
        g_ema = dec.ema.cpu().numpy()
        for (b, h) in units:
            u = uo[(b, h)]
            tag = f"step {t} unit ({b},{h})"
            n, nb, qg, s, sel = sel_info[(b, h)]
            pred = u.pred
            if w.P > 0 and not np.array_equal(g_pred_used[b, h], pad(pred, w.P)):
                rep.fail(f"{tag}: Pred_t differs gpu={g_pred_used[b, h].tolist()} oracle={list(pred)}")
            # a Gaussian near tie continues the oracle from the GPU's (equally correct) set
            acc = check_selection(rep, tag, g_sel[b, h], sel, s, w.K, gaussian)
            if acc is None:
                continue
            res = u.finish(n, nb, qg, acc, pred)
            if not np.array_equal(g_missed[b, h], pad(res["missed"], w.K)) or g_nm[b, h] != len(res["missed"]):
                rep.fail(f"{tag}: missed differs gpu={g_missed[b, h].tolist()} oracle={list(res['missed'])}")
            keep_ref = np.zeros(w.P, np.uint8)
            keep_ref[:len(res["keep"])] = res["keep"]
            if w.P > 0 and not np.array_equal(g_keep[b, h], keep_ref):
                rep.fail(f"{tag}: keep differs gpu={g_keep[b, h].tolist()} oracle={keep_ref.tolist()}")
            rows = u.qrows
            compare_attention(rep, tag, g_out[b, rows], g_lse[b, rows], res["out"], res["lse"])
            if not np.array_equal(g_ema[b, h, :nb], u.ema[:nb]):
                bad = np.nonzero(g_ema[b, h, :nb] != u.ema[:nb])[0][:5]
                rep.fail(f"{tag}: EMA state differs at blocks {bad.tolist()}")
            if w.P > 0 and not np.array_equal(g_pred_next[b, h], pad(res["pred_next"], w.P)):
                rep.fail(f"{tag}: Pred_(t+1) differs gpu={g_pred_next[b, h].tolist()} "
                         f"oracle={list(res['pred_next'])}")
            u.pred = res["pred_next"]
        if rep.messages:
            return rep
    rep.check_near_ties()
    got_lens = dec.seq_lens.cpu().numpy()
    want = [w.n0(b) + steps for b in range(w.B)]
    if got_lens.tolist() != want:
        rep.fail(f"seq_lens after {steps} steps: {got_lens.tolist()}, expected {want}")
    return rep
