"""Profiling-guided speculation budget.

PRR (abstract) sizes its speculative work from profiling so that it stays off the
critical path; its limitations list says the overheads at context lengths off the
profiled grid (between or beyond its points) come from polynomial regressions.  This
module:

- profiles, on the GPU, the selection time and the speculation time over a grid of
  context lengths and speculation budgets: of the two-stream decode step
  (``prr_decode_step`` with its per-kernel timing marks, ``profile``) or of the fused
  single-launch step, from the launch's per-item trace (``profile_fused``: selection
  ends when the last top-K finisher does, speculation when the last speculative block
  does, both measured from the launch's first item);
- fits one polynomial in the context length to the selection times and one per
  budget to the speculation times (``SpecBudget.fit``, through ``prr_budget_fit``);
- answers, for any context length, the largest profiled budget whose speculation is
  predicted to finish before selection does (``SpecBudget.choose``, through
  ``prr_budget_choose``).

The fit and the choice are host functions of the C library; the timing runs the
library's kernels.  A decoder is then built with that budget as its ``P``.
"""
from __future__ import annotations

import dataclasses
import statistics
from typing import Dict, List, Sequence, Tuple

import numpy as np

from . import _abi


@dataclasses.dataclass
class Profile:
    """Mean per-kernel times (microseconds) of the two-stream step."""
    contexts: List[int]
    p_grid: List[int]
    select_us: Dict[Tuple[int, int], float]  # (context, P) -> selection time
    spec_us: Dict[Tuple[int, int], float]    # (context, P) -> speculation time


def profile(base: _abi.Dims, contexts: Sequence[int], p_grid: Sequence[int], steps: int = 8,
            warmup: int = 3, seed: int = 0) -> Profile:
    """Time selection and speculation of the two-stream step for every (context, P).

    ``base`` fixes B, heads, d, bs, K and alpha; each grid point gets its own decoder
    with cap_tokens = context + warmup + steps and P from the grid.  The cache holds
    seeded N(0,1) bf16 keys and values (timing does not depend on their values beyond
    the predicted set, which starts at blocks 0..P-1 and then follows the EMA).
    """
    import torch

    from .decoder import PRRDecoder

    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    sel_us, spec_us = {}, {}
    for n0 in contexts:
        for p in p_grid:
            dims = dataclasses.replace(base, cap_tokens=n0 + warmup + steps + 1, P=p)
            dec = PRRDecoder(dims)
            shape = (dims.B, dims.Hkv, n0, dims.d)
            dec.k_cache[:, :, :n0].copy_(torch.randn(shape, generator=gen, device="cuda").to(torch.bfloat16))
            dec.v_cache[:, :, :n0].copy_(torch.randn(shape, generator=gen, device="cuda").to(torch.bfloat16))
            dec.prefill(dec.k_cache[:, :, :n0], dec.v_cache[:, :, :n0], n0)
            marks = {name: torch.cuda.Event(enable_timing=True) for name in _abi.TIMING_MARKS}
            for ev in marks.values():
                ev.record(dec.select_stream)
            s_list, p_list = [], []
            kv = (dims.B, dims.Hkv, dims.d)
            for t in range(warmup + steps):
                dec.append(torch.randn(kv, generator=gen, device="cuda").to(torch.bfloat16),
                           torch.randn(kv, generator=gen, device="cuda").to(torch.bfloat16))
                q = torch.randn((dims.B, dims.Hq, dims.d), generator=gen, device="cuda").to(torch.bfloat16)
                dec.step(q, timing=marks)
                torch.cuda.synchronize()
                if t >= warmup:
                    s_list.append(_elapsed_us(marks["t_begin"], marks["t_select_end"]))
                    p_list.append(_elapsed_us(marks["t_spec_begin"], marks["t_spec_end"]))
            status = dec.device_status()
            if status != 0:
                raise RuntimeError(f"device status {status} while profiling context {n0}, P {p}")
            sel_us[(n0, p)] = statistics.median(s_list)
            spec_us[(n0, p)] = statistics.median(p_list)
            del dec
    return Profile(list(contexts), list(p_grid), sel_us, spec_us)


def profile_fused(base: _abi.Dims, contexts: Sequence[int], p_grid: Sequence[int], steps: int = 8,
                  warmup: int = 3, seed: int = 0) -> Profile:
    """Time selection and speculation inside the fused step for every (context, P).

    The same decoders and inputs as ``profile``; each step runs ``step_fused`` with the
    trace on.  From the trace (microseconds after the launch's first item starts):
    selection time = when the last selection chunk or top-K finisher ends, speculation
    time = when the last speculative block ends.  Speculation is off the critical path
    when it ends no later than selection."""
    import torch

    from .decoder import PRRDecoder, summarize_trace

    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    sel_us, spec_us = {}, {}
    for n0 in contexts:
        for p in p_grid:
            dims = dataclasses.replace(base, cap_tokens=n0 + warmup + steps + 1, P=p)
            dec = PRRDecoder(dims)
            shape = (dims.B, dims.Hkv, n0, dims.d)
            dec.k_cache[:, :, :n0].copy_(torch.randn(shape, generator=gen, device="cuda").to(torch.bfloat16))
            dec.v_cache[:, :, :n0].copy_(torch.randn(shape, generator=gen, device="cuda").to(torch.bfloat16))
            dec.prefill(dec.k_cache[:, :, :n0], dec.v_cache[:, :, :n0], n0)
            dec.enable_trace(True)
            s_list, p_list = [], []
            kv = (dims.B, dims.Hkv, dims.d)
            for t in range(warmup + steps):
                q = torch.randn((dims.B, dims.Hq, dims.d), generator=gen, device="cuda").to(torch.bfloat16)
                kn = torch.randn(kv, generator=gen, device="cuda").to(torch.bfloat16)
                vn = torch.randn(kv, generator=gen, device="cuda").to(torch.bfloat16)
                dec.trace.zero_()
                dec.step_fused(q, k_new=kn, v_new=vn)
                torch.cuda.synchronize()
                if t >= warmup:
                    tr = summarize_trace(dec.trace.cpu().numpy())
                    s_list.append(max(tr["sel"].get("end_max_us", 0.0), tr["finish"].get("end_max_us", 0.0)))
                    p_list.append(tr["spec"].get("end_max_us", 0.0))
            status = dec.device_status()
            if status != 0:
                raise RuntimeError(f"device status {status} while profiling context {n0}, P {p}")
            sel_us[(n0, p)] = statistics.median(s_list)
            spec_us[(n0, p)] = statistics.median(p_list)
            del dec
    return Profile(list(contexts), list(p_grid), sel_us, spec_us)


def _elapsed_us(a, b) -> float:
    """Microseconds between two events the library recorded (torch's elapsed_time
    only accepts events torch recorded itself)."""
    from cuda.bindings import driver
    err, ms = driver.cuEventElapsedTime(driver.CUevent(init_value=a.cuda_event),
                                        driver.CUevent(init_value=b.cuda_event))
    if err != driver.CUresult.CUDA_SUCCESS:
        raise RuntimeError(f"cuEventElapsedTime: {err}")
    return float(ms) * 1e3


@dataclasses.dataclass
class SpecBudget:
    """Polynomial models of selection and speculation time against context length."""
    p_grid: List[int]
    sel_coef: np.ndarray   # [degree+1]
    spec_coef: np.ndarray  # [len(p_grid)][degree+1]

    @classmethod
    def fit(cls, prof: Profile, degree: int = 2) -> "SpecBudget":
        """Selection time is fitted over every profiled (context, P) point (it does not
        depend on P); speculation time per budget P over the profiled contexts."""
        ctx = [n for (n, _) in prof.select_us]
        sel = _abi.prr_budget_fit(ctx, [prof.select_us[k] for k in prof.select_us], degree)
        spec = np.stack([_abi.prr_budget_fit(prof.contexts, [prof.spec_us[(n, p)] for n in prof.contexts], degree)
                         for p in prof.p_grid])
        return cls(list(prof.p_grid), sel, spec)

    def choose(self, context_tokens: int) -> int:
        return _abi.prr_budget_choose(self.sel_coef, self.spec_coef, self.p_grid, context_tokens)
