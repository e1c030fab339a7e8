"""prr_select_topk_static (fixed in-library scratch, no workspace) against
prr_select_topk (caller workspace), through the C ABI.  Needs a B200; marked gpu.

Both run the same selection kernel, so the selected, missed and keep outputs must
agree exactly, as the selection parity tests require against the oracle.  Two calls
in a row with fresh inputs check that the shared scratch array, which keeps the
previous call's contents, is re-armed correctly.  The file name sorts last so that
pytest runs it after every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest

import workloads as W

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU-only machines, never run there
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import dynamic_sparse_attention_block_b200 as prr  # noqa: E402


def _bits(rng, shape, gauss):
    x = rng.standard_normal(shape) if gauss else rng.integers(-8, 9, size=shape) / 8
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
        summ = _bits(rng, (B, Hkv, dims.maxnb, 2, d), gauss)
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
