"""Pins for the fp64 oracle: every check compares the oracle with something other than
itself -- a library routine it does not use (numpy min/max, torch SDPA / logsumexp),
brute-force enumeration, a closed form, or a hand-worked example under tests/golden.

Each check takes an ``oracle.Oracle`` so the mutation test can run the same checks
against deliberately broken builds of the oracle source and make sure one fails.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch

import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _grid_bits(rng, shape):
    return W.f32_to_bf16_bits(rng.integers(-8, 9, size=shape).astype(np.float32) / 8.0)


def _gauss_bits(rng, shape):
    return W.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def _f(bits):
    return W.bf16_bits_to_f32(bits).astype(np.float64)


# --------------------------------------------------------------------------- summaries

def check_summaries_vs_numpy(o):
    """Block summaries equal numpy's per-block min/max (ragged tail included)."""
    rng = np.random.default_rng(1)
    for n, bs, d in [(200, 64, 16), (64, 64, 8), (65, 64, 8), (1, 16, 4), (130, 1, 4)]:
        k = _gauss_bits(rng, (n, d))
        lo, hi = o.build_summaries(k, n, bs)
        kf = _f(k)
        for b in range(-(-n // bs)):
            blk = kf[b * bs:min(n, (b + 1) * bs)]
            assert np.array_equal(lo[b], blk.min(axis=0)), (n, bs, b)
            assert np.array_equal(hi[b], blk.max(axis=0)), (n, bs, b)


# --------------------------------------------------------------------------- Quest bound

def check_bound_dominates_and_is_tight(o):
    """Per head, U_h(b) >= max_{i in b} q_h.k_i; for the group, s_b >= max_i sum_h q_h.k_i;
    with one token per block the bound is exactly q.k (numpy dot)."""
    rng = np.random.default_rng(2)
    for G, d, n, bs in [(4, 16, 96, 16), (8, 32, 64, 8), (1, 8, 40, 5)]:
        q = _f(_grid_bits(rng, (G, d)))
        k = _grid_bits(rng, (n, d))
        kf = _f(k)
        lo, hi = o.build_summaries(k, n, bs)
        s_group = o.block_scores(q, lo, hi)
        per_head = np.stack([o.block_scores(q[h:h + 1], lo, hi) for h in range(G)])
        # the group score is the sum of the per-head bounds (GQA reading)
        assert np.allclose(s_group, per_head.sum(axis=0), rtol=0, atol=1e-12)
        for b in range(-(-n // bs)):
            toks = kf[b * bs:min(n, (b + 1) * bs)]
            qk = q @ toks.T  # [G][tokens]
            assert np.all(per_head[:, b] >= qk.max(axis=1) - 1e-12)
            assert s_group[b] >= qk.sum(axis=0).max() - 1e-12
        # bs = 1: min = max = k, so U_h = q_h.k exactly
        lo1, hi1 = o.build_summaries(k, n, 1)
        for h in range(G):
            u = o.block_scores(q[h:h + 1], lo1, hi1)
            assert np.allclose(u, kf @ q[h], rtol=0, atol=1e-12)
        assert np.allclose(o.block_scores(q, lo1, hi1), kf @ q.sum(axis=0), rtol=0, atol=1e-12)
        # sign closed forms: q >= 0 picks the max vector, q <= 0 the min vector
        qp = np.abs(q)
        assert np.allclose(o.block_scores(qp[:1], lo, hi), hi @ qp[0], rtol=0, atol=1e-12)
        assert np.allclose(o.block_scores(-qp[:1], lo, hi), lo @ (-qp[0]), rtol=0, atol=1e-12)


def check_grid_scores_exact(o):
    """On the dyadic grid every product is a multiple of 1/64 with |.| <= 1, so each
    score is a multiple of 1/64 bounded by G*d (what makes fp32 scores exact)."""
    rng = np.random.default_rng(3)
    G, d, n, bs = 8, 128, 512, 64
    q = _f(_grid_bits(rng, (G, d)))
    k = _grid_bits(rng, (n, d))
    lo, hi = o.build_summaries(k, n, bs)
    s = o.block_scores(q, lo, hi)
    assert np.all(np.abs(s) <= G * d)
    assert np.array_equal(s * 64, np.round(s * 64))


# --------------------------------------------------------------------------- top-K

def _brute_topk(vals, K):
    """The unique K-subset whose every member ranks before every non-member under
    (value desc, index asc), found by enumerating all subsets."""
    nb = len(vals)
    keff = min(K, nb)
    found = []
    for sub in itertools.combinations(range(nb), keff):
        inside = set(sub)
        ok = True
        for a in inside:
            for b in range(nb):
                if b in inside:
                    continue
                if not (vals[a] > vals[b] or (vals[a] == vals[b] and a < b)):
                    ok = False
                    break
            if not ok:
                break
        if ok:
            found.append(sub)
    assert len(found) == 1
    return list(found[0])


def check_topk_bruteforce(o):
    rng = np.random.default_rng(4)
    for trial in range(120):
        nb = int(rng.integers(1, 13))
        K = int(rng.integers(1, 5))
        vals = rng.integers(-3, 4, size=nb).astype(np.float64)  # many ties
        got = list(o.top_ranked(vals, K))
        assert got == _brute_topk(vals, K), (vals, K, got)


# --------------------------------------------------------------------------- EMA

def check_ema_closed_form(o):
    """e_t(b) = beta * sum_{s<=t} alpha^(t-s) [b in S_s] (e_0 = 0)."""
    rng = np.random.default_rng(5)
    for alpha in (0.9, 0.5, 0.75):
        nb, T = 20, 30
        beta = 1.0 - alpha
        hist = [np.sort(rng.choice(nb, size=int(rng.integers(0, 6)), replace=False))
                for _ in range(T)]
        e = np.zeros(nb)
        for t in range(T):
            e = o.ema_update(e, nb, hist[t].astype(np.int32), alpha)
            closed = np.zeros(nb)
            for s in range(t + 1):
                for b in hist[s]:
                    closed[b] += beta * alpha ** (t - s)
            assert np.allclose(e, closed, rtol=0, atol=1e-14), (alpha, t)


def check_ema_rounding_fixed(o):
    """The update rounds alpha*e and beta*ind separately, then their sum (no fused
    multiply-add): the oracle reproduces, bit for bit, a trajectory derived with exact
    rationals (tests/golden/ema_rounding.json, written by make_ema_rounding.py), which
    a contracted update leaves at the step the fixture names."""
    with open(os.path.join(GOLDEN, "ema_rounding.json")) as fh:
        ex = json.load(fh)
    e = np.zeros(ex["nb"])
    for t, sel in enumerate(ex["selections"]):
        e = o.ema_update(e, ex["nb"], np.array(sel, np.int32), ex["alpha"])
        assert e[0].hex() == ex["e_block0_hex"][t], (t, e[0].hex())
        assert e[1] == 0.0
    assert ex["e_block0_hex"] != ex["contracted_block0_hex"]


def check_predict_from_zero_state(o):
    """With no history all e = 0 and the tie rule predicts blocks 0..P-1."""
    for nb, P in [(65, 8), (5, 8), (513, 64)]:
        got = o.top_ranked(np.zeros(nb), P)
        assert list(got) == list(range(min(nb, P)))


# --------------------------------------------------------------------------- attention

def _sdpa_ref(q, kf, vf, mask, scale):
    """torch scaled_dot_product_attention (fp64, CPU) and torch.logsumexp."""
    qt = torch.from_numpy(q).view(1, 1, 1, -1)
    kt = torch.from_numpy(kf).view(1, 1, kf.shape[0], -1)
    vt = torch.from_numpy(vf).view(1, 1, vf.shape[0], -1)
    mt = torch.from_numpy(mask).view(1, 1, 1, -1)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mt, scale=scale)
    logits = (kt[0, 0] @ qt[0, 0, 0]) * scale
    lse = torch.logsumexp(logits[torch.from_numpy(mask)], dim=0)
    return out.view(-1).numpy(), float(lse)


def check_attention_vs_sdpa(o):
    """All blocks selected = dense attention; a block subset = SDPA with a block mask."""
    rng = np.random.default_rng(6)
    for d, n, bs in [(64, 300, 64), (128, 129, 64), (16, 40, 8)]:
        scale = 1.0 / math.sqrt(d)
        q = _f(_gauss_bits(rng, d))
        k, v = _gauss_bits(rng, (n, d)), _gauss_bits(rng, (n, d))
        kf, vf = _f(k), _f(v)
        nb = -(-n // bs)
        full = np.arange(nb, dtype=np.int32)
        out, lse = o.attend_blocks(q, k, v, n, bs, full, scale)
        ref, rlse = _sdpa_ref(q, kf, vf, np.ones(n, bool), scale)
        assert np.allclose(out, ref, rtol=0, atol=1e-12) and abs(lse - rlse) < 1e-12
        sub = np.sort(rng.choice(nb, size=max(1, nb // 2), replace=False)).astype(np.int32)
        mask = np.zeros(n, bool)
        for b in sub:
            mask[b * bs:min(n, (b + 1) * bs)] = True
        out, lse = o.attend_blocks(q, k, v, n, bs, sub, scale)
        ref, rlse = _sdpa_ref(q, kf, vf, mask, scale)
        assert np.allclose(out, ref, rtol=0, atol=1e-12) and abs(lse - rlse) < 1e-12


def check_prr_invariance(o):
    """Speculate-reuse-repair with any predicted set gives the direct top-K result:
    perfect, empty, random, adversarial (disjoint) and partially overlapping Pred."""
    rng = np.random.default_rng(7)
    d, n, bs = 64, 700, 64
    scale = 1.0 / math.sqrt(d)
    nb = -(-n // bs)
    q = _f(_gauss_bits(rng, d))
    k, v = _gauss_bits(rng, (n, d)), _gauss_bits(rng, (n, d))
    sel = np.sort(rng.choice(nb, size=5, replace=False)).astype(np.int32)
    ref, rlse = o.attend_blocks(q, k, v, n, bs, sel, scale)
    outside = np.setdiff1d(np.arange(nb), sel)
    preds = {
        "perfect": sel,
        "empty": np.zeros(0, np.int32),
        "random": np.sort(rng.choice(nb, size=5, replace=False)),
        "adversarial": np.sort(rng.choice(outside, size=5, replace=False)),
        "partial": np.sort(np.concatenate([sel[:3], outside[:2]])),
        "superset": np.sort(np.concatenate([sel, outside[:3]])),
    }
    for name, pred in preds.items():
        out, lse = o.prr_attend(q, k, v, n, bs, sel, pred.astype(np.int32), scale)
        assert np.allclose(out, ref, rtol=0, atol=1e-12), name
        assert abs(lse - rlse) < 1e-12, name
    # missed set / keep mask against python set algebra
    for pred in preds.values():
        missed, keep = o.missed_keep(sel, pred.astype(np.int32))
        assert list(missed) == sorted(set(sel.tolist()) - set(pred.tolist()))
        assert list(keep) == [int(p in set(sel.tolist())) for p in pred.tolist()]


def check_merge_of_two_token_sets(o):
    """Merging the statistics of two disjoint blocks equals attention over both."""
    rng = np.random.default_rng(8)
    d, n, bs = 32, 128, 64
    scale = 1.0 / math.sqrt(d)
    q = _f(_gauss_bits(rng, d)) * 3.0
    k, v = _gauss_bits(rng, (n, d)), _gauss_bits(rng, (n, d))
    parts = [o.block_partial(q, k, v, n, bs, b, scale) for b in (0, 1)]
    m = np.array([p[0] for p in parts])
    l = np.array([p[1] for p in parts])
    O = np.stack([p[2] for p in parts])
    out, lse = o.lse_merge(m, l, O)
    ref, rlse = _sdpa_ref(q, _f(k), _f(v), np.ones(n, bool), scale)
    assert np.allclose(out, ref, rtol=0, atol=1e-12) and abs(lse - rlse) < 1e-12


# --------------------------------------------------------------------------- hand-worked examples

def check_hand_examples(o):
    """Small examples worked by hand from the definitions (tests/golden)."""
    with open(os.path.join(GOLDEN, "hand_examples.json")) as fh:
        ex = json.load(fh)
    qb = ex["quest_bound"]
    lo, hi = o.build_summaries(W.f32_to_bf16_bits(np.array(qb["keys"], np.float32)),
                               len(qb["keys"]), len(qb["keys"]))
    s = o.block_scores(np.array([qb["q"]]), lo, hi)
    assert s[0] == qb["bound"]
    tk = ex["topk_ties"]
    assert list(o.top_ranked(np.array(tk["scores"], float), tk["K"])) == tk["selected"]
    em = ex["ema"]
    e = np.zeros(em["nb"])
    for sel in em["selections"]:
        e = o.ema_update(e, em["nb"], np.array(sel, np.int32), em["alpha"])
    assert np.array_equal(e, np.array(em["e_final"]))
    assert list(o.top_ranked(e, em["P"])) == em["pred"]
    at = ex["attention"]
    kb = W.f32_to_bf16_bits(np.array(at["k"], np.float32))
    vb = W.f32_to_bf16_bits(np.array(at["v"], np.float32))
    out, lse = o.attend_blocks(np.array(at["q"], float), kb, vb, len(at["k"]), at["bs"],
                               np.array(at["blocks"], np.int32), at["scale"])
    e1 = math.e
    assert np.allclose(out, [1 / (1 + e1), e1 / (1 + e1), 0.0, 0.0], rtol=0, atol=1e-15)
    assert abs(lse - math.log(1 + e1)) < 1e-15
    mg = ex["merge"]
    out, lse = o.lse_merge(np.array(mg["m"], float), np.array(mg["l"], float),
                           np.array(mg["O"], float))
    ei = math.exp(-1.0)
    assert abs(out[0] - (ei * 1.0 + 2.0) / (ei + 1.0)) < 1e-15
    assert abs(lse - (1.0 + math.log(1.0 + ei))) < 1e-15


# --------------------------------------------------------------------------- step driver

def check_decode_step_driver(o):
    """The all-units step driver against independent recomputation: numpy summaries of
    the cache, brute-force-free ranking of its own scores (cross-checked by the top-K
    pin), SDPA restricted to the selected tokens, EMA closed form over the history."""
    w = W.workload("tiny").with_(B=2, Hq=8, Hkv=2, N0=300, bs=32, K=3, P=4, steps=5)
    cap = w.N0 + w.steps
    d, G = w.d, w.G
    kc = np.zeros((w.B, w.Hkv, cap, d), np.uint16)
    vc = np.zeros_like(kc)
    for b in range(w.B):
        for h in range(w.Hkv):
            k0, v0 = W.kv_prefix(w, b, h)
            kn, vn = W.kv_appended(w, b, h)
            kc[b, h, :w.N0], vc[b, h, :w.N0] = k0, v0
            kc[b, h, w.N0:], vc[b, h, w.N0:] = kn, vn
    import oracle as OR
    st = OR.new_state(w.B, w.Hkv, cap, w.bs, d)
    for b in range(w.B):
        for h in range(w.Hkv):
            lo, hi = o.build_summaries(kc[b, h], w.N0, w.bs)
            st["smin"][b, h, :lo.shape[0]], st["smax"][b, h, :lo.shape[0]] = lo, hi
    qs = W.queries(w)
    dims = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=d, bs=w.bs, cap=cap, K=w.K, P=w.P,
                alpha=w.alpha, scale=w.scale())
    pred = np.full((w.B, w.Hkv, w.P), -1, np.int32)
    pred[:, :, :w.P] = np.arange(w.P)
    hist = {(b, h): [] for b in range(w.B) for h in range(w.Hkv)}
    for t in range(w.steps):
        n = w.N0 + t + 1
        seq = np.full(w.B, n, np.int32)
        r = o.decode_step(dims, qs[t], kc, vc, seq, pred, st, nthreads=2)
        nb = -(-n // w.bs)
        for b in range(w.B):
            for h in range(w.Hkv):
                kf = _f(kc[b, h, :n])
                for blk in range(nb):
                    toks = kf[blk * w.bs:min(n, (blk + 1) * w.bs)]
                    assert np.array_equal(st["smin"][b, h, blk], toks.min(axis=0))
                    assert np.array_equal(st["smax"][b, h, blk], toks.max(axis=0))
                qg = _f(qs[t, b, h * G:(h + 1) * G])
                s = o.block_scores(qg, st["smin"][b, h, :nb], st["smax"][b, h, :nb])
                sel = r["sel"][b, h][r["sel"][b, h] >= 0]
                assert list(sel) == _brute_topk(s, w.K) if nb <= 12 else True
                assert list(sel) == list(o.top_ranked(s, w.K))
                mask = np.zeros(n, bool)
                for blk in sel:
                    mask[blk * w.bs:min(n, (blk + 1) * w.bs)] = True
                for g in range(G):
                    ref, rlse = _sdpa_ref(qg[g], kf, _f(vc[b, h, :n]), mask, w.scale())
                    assert np.allclose(r["out"][b, h * G + g], ref, rtol=0, atol=1e-12)
                    assert abs(r["lse"][b, h * G + g] - rlse) < 1e-12
                hist[(b, h)].append(set(sel.tolist()))
                closed = np.zeros(nb)
                for s_i, S in enumerate(hist[(b, h)]):
                    for blk in S:
                        closed[blk] += (1 - w.alpha) * w.alpha ** (t - s_i)
                assert np.allclose(st["ema"][b, h, :nb], closed, rtol=0, atol=1e-14)
                pn = r["pred_next"][b, h][r["pred_next"][b, h] >= 0]
                order = sorted(range(nb), key=lambda i: (-st["ema"][b, h, i], i))
                assert list(pn) == sorted(order[:min(w.P, nb)])
                pr = pred[b, h][pred[b, h] >= 0]
                assert r["n_missed"][b, h] == len(set(sel.tolist()) - set(pr.tolist()))
        pred = r["pred_next"]


def _brute_forced(v, K, n_sink, n_local):
    """Forced sink/local blocks (sinks first, then newest local, within min(K, nb)), then
    the unique completion whose members all rank before every non-member."""
    nb = len(v)
    keff = min(K, nb)
    forced = [b for b in range(min(n_sink, nb))][:keff]
    for i in range(n_local):
        b = nb - 1 - i
        if b < 0 or len(forced) >= keff:
            break
        if b not in forced:
            forced.append(b)
    rest = [b for b in range(nb) if b not in forced]
    key = lambda b: (-v[b], b)
    wins = [sub for sub in itertools.combinations(rest, keff - len(forced))
            if all(key(a) < key(b) for a in sub for b in rest if b not in sub)]
    assert len(wins) == 1
    return sorted(forced + list(wins[0]))


def check_selector_variants(o):
    """Max-over-heads scores reduce to the sum for one head, bound every head's best
    q.k and are exact with one token per block; forced sink/local selection matches
    brute force and reduces to top-K with nothing forced."""
    rng = np.random.default_rng(21)
    k = _f(_grid_bits(rng, (512, 32)))
    lo = np.stack([k[b * 64:(b + 1) * 64].min(0) for b in range(8)])
    hi = np.stack([k[b * 64:(b + 1) * 64].max(0) for b in range(8)])
    q1 = _f(_grid_bits(rng, (1, 32)))
    assert np.array_equal(o.block_scores_max(q1, lo, hi), o.block_scores(q1, lo, hi))
    q = _f(_grid_bits(rng, (4, 32)))
    s = o.block_scores_max(q, lo, hi)
    best = np.array([(q @ k[b * 64:(b + 1) * 64].T).max() for b in range(8)])
    assert np.all(s >= best - 1e-12)
    assert np.allclose(o.block_scores_max(q, k[:20], k[:20]), (q @ k[:20].T).max(0), atol=1e-12)
    for seed in range(8):
        r = np.random.default_rng(300 + seed)
        nb, K = int(r.integers(1, 10)), int(r.integers(1, 5))
        ns, nl = int(r.integers(0, 3)), int(r.integers(0, 3))
        v = r.integers(0, 4, size=nb).astype(np.float64)
        assert list(o.top_ranked_forced(v, K, ns, nl)) == _brute_forced(v, K, ns, nl)
        assert np.array_equal(o.top_ranked_forced(v, K, 0, 0), o.top_ranked(v, K))


def check_rep_scores(o):
    """Representative-key scores: with every token of full blocks as a representative
    they equal the sum of the group's queries dotted with the block's key sum (numpy);
    with one token per block they are r times that token's dot product; a
    representative past a ragged tail stands for the block's last valid token; top-K
    over them matches brute-force enumeration."""
    rng = np.random.default_rng(41)
    G, d, bs = 3, 16, 8
    n = 8 * bs
    q = _f(_grid_bits(rng, (G, d)))
    k = _grid_bits(rng, (n, d))
    kf = _f(k)
    rep = np.tile(np.arange(bs, dtype=np.int32), (n // bs, 1))
    s = o.block_scores_rep(q, k, n, bs, rep)
    ref = np.array([q.sum(0) @ kf[b * bs:(b + 1) * bs].sum(0) for b in range(n // bs)])
    assert np.allclose(s, ref, rtol=0, atol=1e-12)
    r = 3
    s1 = o.block_scores_rep(q, k, n, 1, np.zeros((n, r), np.int32))
    assert np.allclose(s1, r * (kf @ q.sum(0)), rtol=0, atol=1e-12)
    # ragged tail: n = 5*bs + 3, block 5 holds 3 tokens; offsets 6 and 7 mean token 2
    n2 = 5 * bs + 3
    rep2 = np.array([[0, 6], [1, 7], [2, 2], [3, 0], [4, 5], [1, 7]], np.int32)
    s2 = o.block_scores_rep(q, k[:n2], n2, bs, rep2)
    qs = q.sum(0)
    assert abs(s2[5] - qs @ (kf[5 * bs + 1] + kf[5 * bs + 2])) < 1e-12
    assert abs(s2[1] - qs @ (kf[bs + 1] + kf[bs + 7])) < 1e-12
    for trial in range(20):
        nbt = int(rng.integers(1, 9))
        rep3 = rng.integers(0, bs, size=(nbt, 2)).astype(np.int32)
        v = o.block_scores_rep(q, k[:nbt * bs], nbt * bs, bs, rep3)
        K = int(rng.integers(1, 4))
        assert list(o.top_ranked(v, K)) == _brute_topk(v, K)


def check_paged_gather(o):
    """Gathering a sequence through its block table from a pool whose pages hold the
    blocks in a shuffled order gives back the contiguous slice (numpy scatter), so
    summaries, scores and attention on the gathered slice are the contiguous ones."""
    rng = np.random.default_rng(43)
    Hkv, bs, d = 3, 8, 16
    for n in (5 * bs, 5 * bs - 3, 1):
        nbk = -(-n // bs)
        pages = nbk * 2 + 3
        k = _grid_bits(rng, (Hkv, nbk * bs, d))
        table = rng.permutation(pages)[:nbk].astype(np.int32)
        pool = np.zeros((pages, Hkv, bs, d), np.uint16)
        for j in range(nbk):
            pool[table[j]] = k[:, j * bs:(j + 1) * bs]
        for h in range(Hkv):
            g = o.gather_pages(pool, table, h, n, bs)
            assert np.array_equal(g, k[h, :n]), (n, h)
            lo, hi = o.build_summaries(g, n, bs)
            lo2, hi2 = o.build_summaries(k[h, :n], n, bs)
            assert np.array_equal(lo, lo2) and np.array_equal(hi, hi2)


ALL_CHECKS = [
    check_summaries_vs_numpy, check_bound_dominates_and_is_tight, check_grid_scores_exact,
    check_topk_bruteforce, check_ema_closed_form, check_ema_rounding_fixed, check_predict_from_zero_state,
    check_attention_vs_sdpa, check_prr_invariance, check_merge_of_two_token_sets,
    check_hand_examples, check_decode_step_driver, check_selector_variants, check_rep_scores,
    check_paged_gather,
]
