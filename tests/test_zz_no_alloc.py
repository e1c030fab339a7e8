"""prr_select_topk_static (fixed in-library scratch, no workspace) against
prr_select_topk (caller workspace) and against the fp64 oracle, through the C ABI.
Needs a B200; marked gpu.

Some callers cannot allocate device memory for a workspace (code inside another
runtime's memory pool, hosts that forbid cudaMalloc once serving has started); the
static entry point serves them from an array inside the library.  Both entry points
run the same selection kernel, so the selected, missed and keep outputs must agree
exactly, and on exact-grid inputs they must equal the oracle's top-K bit for bit.
Two calls in a row with fresh inputs check that the shared scratch array, which keeps
the previous call's contents, is re-armed correctly, also after a call that stopped
early on a bad sequence length.  The file name sorts last so that pytest runs it
after every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest

import oracle as OR
import workloads as W
from tests.prr_harness import f64, pad

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU-only machines, never run there
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import dynamic_sparse_attention_block_b200 as prr  # noqa: E402


def _bits(rng, shape, gauss):
    x = rng.standard_normal(shape) if gauss else rng.integers(-8, 9, size=shape) / 8
    return torch.from_numpy(W.f32_to_bf16_bits(np.asarray(x, np.float32)).view(np.int16)).cuda()


def _summaries(rng, B, Hkv, maxnb, d, gauss):
    """Valid block summaries: per channel a min row not above the max row (the scorer's
    bound equals the oracle's only for such pairs)."""
    x = rng.standard_normal((B, Hkv, maxnb, 2, d)) if gauss else rng.integers(-8, 9, size=(B, Hkv, maxnb, 2, d)) / 8
    x = np.sort(x, axis=3)
    return torch.from_numpy(W.f32_to_bf16_bits(np.asarray(x, np.float32)).view(np.int16)).cuda()


def _outputs(B, Hkv, K, P):
    sel = torch.full((B, Hkv, K), -7, dtype=torch.int32, device="cuda")
    return (sel, torch.full_like(sel, -7), torch.full((B, Hkv), -7, dtype=torch.int32, device="cuda"),
            torch.full((B, Hkv, max(P, 1)), 9, dtype=torch.uint8, device="cuda"))


@pytest.mark.parametrize("d,bs,G,K,P,n,gauss", [
    (128, 64, 4, 64, 64, 32769, False),  # Llama-8B-shaped at 32K, ragged tail
    (64, 128, 2, 32, 16, 9000, True),    # Gaussian keys, P < K
    (128, 64, 1, 7, 0, 500, False),      # no speculation
])
def test_static_scratch_matches_workspace_entry(d, bs, G, K, P, n, gauss):
    rng = np.random.default_rng(2024)
    B, Hkv = 2, 2
    cap = n + 3
    dims = prr.Dims(B=B, Hq=G * Hkv, Hkv=Hkv, d=d, bs=bs, cap_tokens=cap, K=K, P=P)
    nb = -(-n // bs)
    ws = torch.zeros(prr.prr_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    seq = torch.full((B,), n, dtype=torch.int32, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call in range(2):  # fresh inputs each call: the shared array keeps the last call's contents
        summ = _summaries(rng, B, Hkv, dims.maxnb, d, gauss)
        q = _bits(rng, (B, G * Hkv, d), gauss)
        pred_h = np.full((B, Hkv, max(P, 1)), -1, np.int32)
        for b in range(B):
            for h in range(Hkv):
                c = min(P, nb)
                pred_h[b, h, :c] = np.sort(rng.choice(nb, size=c, replace=False))
        pred = torch.from_numpy(pred_h).cuda()
        ref = _outputs(B, Hkv, K, P)
        got = _outputs(B, Hkv, K, P)
        prr.prr_select_topk(dims, q, summ, seq, pred, *ref, ws)
        prr.prr_select_topk_static(dims, q, summ, seq, pred, *got, status)
        torch.cuda.synchronize()
        assert prr.prr_get_device_status(ws) == 0
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        for name, r, g in zip(("sel", "missed", "n_missed", "keep"), ref, got):
            r, g = r.cpu().numpy(), g.cpu().numpy()
            if name == "keep":  # only the predicted slots are defined
                r, g = r[..., :P], g[..., :P]
            assert np.array_equal(r, g), f"call {call}: {name} differs"
        assert (ref[0] >= 0).sum().item() == B * Hkv * min(K, nb)
        if not gauss:  # exact grid: the oracle's top-K, missed set and keep mask
            _check_against_oracle(got, q, summ, pred_h, G, K, P, nb)


def _check_against_oracle(got, q, summ, pred_h, G, K, P, nb):
    o = OR.default()
    qh = q.cpu().numpy().view(np.uint16)
    sh = summ.cpu().numpy().view(np.uint16)
    g_sel, g_missed, g_nm, g_keep = (x.cpu().numpy() for x in got)
    B, Hkv = g_sel.shape[:2]
    for b in range(B):
        for h in range(Hkv):
            s = o.block_scores(f64(qh[b, h * G:(h + 1) * G]), f64(sh[b, h, :nb, 0]), f64(sh[b, h, :nb, 1]))
            ref = o.top_ranked(s, K)
            assert np.array_equal(g_sel[b, h], pad(ref, K)), (b, h)
            pr = pred_h[b, h][pred_h[b, h] >= 0]
            ref_missed, ref_keep = o.missed_keep(ref, pr)
            assert np.array_equal(g_missed[b, h], pad(ref_missed, K)) and g_nm[b, h] == len(ref_missed)
            if P > 0:
                assert np.array_equal(g_keep[b, h][:len(pr)], ref_keep)


def test_static_scratch_recovers_after_bad_seq_len():
    """A call whose sequence length is out of range reports status 1 (bad seq_len)
    through the status word, with no fault, and leaves its units unfinished; the next
    good call re-arms the shared array and matches prr_select_topk and the oracle."""
    rng = np.random.default_rng(77)
    B, Hkv, G, d, bs, K, P, n = 2, 2, 4, 128, 64, 16, 16, 5000
    cap = n + 3
    dims = prr.Dims(B=B, Hq=G * Hkv, Hkv=Hkv, d=d, bs=bs, cap_tokens=cap, K=K, P=P)
    nb = -(-n // bs)
    summ = _summaries(rng, B, Hkv, dims.maxnb, d, False)
    q = _bits(rng, (B, G * Hkv, d), False)
    pred_h = np.full((B, Hkv, P), -1, np.int32)
    for b in range(B):
        for h in range(Hkv):
            pred_h[b, h] = np.sort(rng.choice(nb, size=P, replace=False))
    pred = torch.from_numpy(pred_h).cuda()
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    bad = torch.tensor([n, cap + 9], dtype=torch.int32, device="cuda")  # sequence 1 beyond the cache
    prr.prr_select_topk_static(dims, q, summ, bad, pred, *_outputs(B, Hkv, K, P), status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1  # PRR_DEV_BAD_SEQ_LEN
    seq = torch.full((B,), n, dtype=torch.int32, device="cuda")
    ws = torch.zeros(prr.prr_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    ref, got = _outputs(B, Hkv, K, P), _outputs(B, Hkv, K, P)
    prr.prr_select_topk(dims, q, summ, seq, pred, *ref, ws)
    prr.prr_select_topk_static(dims, q, summ, seq, pred, *got, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and prr.prr_get_device_status(ws) == 0
    for r, g in zip(ref, got):
        assert np.array_equal(r.cpu().numpy(), g.cpu().numpy())
    _check_against_oracle(got, q, summ, pred_h, G, K, P, nb)


def test_static_scratch_rejects_oversized_shapes():
    # B*Hkv*ceil(cap/bs) one block above the limit: refused before anything is enqueued
    bs, Hkv = 64, 8
    per_unit = 8192
    B = prr.SELECT_STATIC_MAX_BLOCKS // (Hkv * per_unit)
    dims = prr.Dims(B=B, Hq=4 * Hkv, Hkv=Hkv, d=128, bs=bs, cap_tokens=per_unit * bs + 1, K=64, P=64)
    t = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(prr.PrrError) as ei:
        prr.prr_select_topk_static(dims, t, t, t, t, t, t, t, t, t)
    assert ei.value.status == 3  # PRR_ERR_CAPACITY
    ok = prr.Dims(B=B, Hq=4 * Hkv, Hkv=Hkv, d=128, bs=bs, cap_tokens=per_unit * bs, K=64, P=64)
    assert B * Hkv * ok.maxnb == prr.SELECT_STATIC_MAX_BLOCKS  # the limit itself is accepted
