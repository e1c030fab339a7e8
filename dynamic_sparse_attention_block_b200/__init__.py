"""PRR speculate-reuse-repair decode step for dynamic sparse attention on B200 (sm_100a).

The hot path is the C-ABI library libprr_b200.so (include/prr.h); this package is its
thin Python binding (``_abi``, same names as the C entry points) plus ``PRRDecoder``,
which owns the caller-side device buffers and streams.  Nothing here computes the
method's arithmetic on the host and there is no CPU fallback.
"""
from ._abi import (  # noqa: F401
    Dims, PrrError, PrrDims, PrrStepBuffers, PrrStepEvents, SELECT_STATIC_MAX_BLOCKS, SELECT_STATIC_SCRATCH_BYTES,
    SELECTORS, WS_TEST_SKIP_SELECTION_OFFSET,
    SYMBOLS, load, library_path,
    prr_append_kv, prr_budget_choose, prr_budget_fit, prr_decode_step, prr_decode_step_fused, prr_ema_predict, prr_get_device_status, prr_repair_merge,
    prr_select_topk, prr_select_topk_static, prr_speculate, prr_status_string, prr_update_summaries, prr_version,
    prr_workspace_bytes, prr_workspace_init,
)
from .decoder import PRRDecoder  # noqa: F401
