"""Host-side argument checks of PRRDecoder that answer before any device work (run
without a GPU on an instance that holds only its dims)."""
import pytest
import torch

from dynamic_sparse_attention_block_b200 import Dims
from dynamic_sparse_attention_block_b200.decoder import PRRDecoder


def _bare(dims, paged=False):
    dec = PRRDecoder.__new__(PRRDecoder)  # no buffers: every case below must fail first
    dec.dims = dims
    dec.block_table = torch.zeros((dims.B, dims.maxnb), dtype=torch.int32) if paged else None
    return dec


DIMS = Dims(B=2, Hq=4, Hkv=1, d=64, bs=64, cap_tokens=1000, K=8, P=8)


@pytest.mark.parametrize("n0", [[500], [500, 0], [500, 1001], 0, 1001])
def test_prefill_refuses_lengths_outside_the_cache(n0):
    with pytest.raises(ValueError):
        _bare(DIMS).prefill(None, None, n0)


def test_prefill_refuses_short_or_mismatched_context():
    k = torch.zeros((2, 1, 400, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        _bare(DIMS).prefill(k, k, [400, 401])  # k shorter than a sequence
    with pytest.raises(ValueError):
        _bare(DIMS).prefill(k, None, 400)
    with pytest.raises(ValueError):
        _bare(DIMS).prefill(k, k[:, :, :300], 300)


def test_prefill_copies_into_contiguous_caches_only():
    k = torch.zeros((2, 1, 400, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="paged"):
        _bare(DIMS, paged=True).prefill(k, k, 400)
