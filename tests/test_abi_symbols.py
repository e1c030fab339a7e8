"""The C-ABI library loads without a GPU and exports every entry point that
include/prr.h declares; host-side validation answers before any device work.

No call here reaches a kernel: only the version, status strings, workspace sizing and
argument/shape checks that return before anything is enqueued.  The ceiling test also
makes accepted calls, which stop at the CUDA runtime, so it runs only where no GPU is
reachable.
"""
import ctypes
import os
import re

import pytest
import torch

from dynamic_sparse_attention_block_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "prr.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^[A-Za-z_][\w \t\*]*?\b(prr_\w+)\s*\(", text, flags=re.M)


@pytest.fixture(scope="module")
def lib():
    build.build(verbose=False)
    return _abi.load()


def test_header_lists_the_binding_symbols():
    decl = _declared()
    assert len(decl) == len(set(decl))
    assert set(decl) == set(_abi.SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_host_side_calls(lib):
    assert _abi.prr_version() >= 100
    for s in range(7):
        assert _abi.prr_status_string(s) != "unknown status"
    d = _abi.Dims(B=1, Hq=32, Hkv=8, d=128, bs=64, cap_tokens=32768, K=64, P=64)
    assert _abi.prr_workspace_bytes(d) > 0
    bad = _abi.Dims(B=1, Hq=32, Hkv=8, d=96, bs=64, cap_tokens=32768, K=64, P=64)
    assert _abi.prr_workspace_bytes(bad) == 0  # unsupported head dim


@pytest.mark.parametrize("kw,ok", [
    (dict(cap_tokens=1 << 30), True), (dict(cap_tokens=(1 << 30) + 1), False), (dict(cap_tokens=2**31 - 1), False),
    (dict(B=8191, Hkv=8, Hq=32), True), (dict(B=8192, Hkv=8, Hq=32), False),  # 65,535 selection units
    (dict(B=2047, Hkv=8, Hq=32, selector="per_head"), True), (dict(B=2048, Hkv=8, Hq=32, selector="per_head"), False),
    (dict(K=128, P=128), True), (dict(K=129), False), (dict(P=129), False), (dict(P=-1), False),
    (dict(Hq=64, Hkv=8), True), (dict(Hq=72, Hkv=8), False), (dict(Hq=12, Hkv=8), False),  # 1 <= G <= 8
    (dict(bs=32), False), (dict(d=256), False),
    (dict(selector="representative", n_rep=1, rep_offsets=1 << 20), True),
    (dict(selector="representative", n_rep=16, rep_offsets=1 << 20), True),
    (dict(selector="representative", n_rep=17, rep_offsets=1 << 20), False),
    (dict(selector="representative", n_rep=0, rep_offsets=1 << 20), False),
    (dict(selector="representative", n_rep=4), False),  # no offsets
    (dict(n_sink=1 << 22, n_local=1 << 22), True), (dict(n_sink=(1 << 22) + 1), False),
    (dict(n_local=-1), False), (dict(alpha=1.0), True), (dict(alpha=1.5), False), (dict(alpha=-0.1), False),
    (dict(pages=64, block_table=1 << 20), True), (dict(pages=64), False),  # a pool needs its table
    (dict(block_table=1 << 20), False),                                     # and a table its pool
    (dict(pages=(1 << 28), Hkv=8, Hq=32, block_table=1 << 20), False),      # pages*Hkv reaches 2^31
])
def test_shape_rules(lib, kw, ok):
    """The documented shape rules, at and just past each bound: a refused shape sizes no
    workspace (0 bytes)."""
    base = dict(B=1, Hq=32, Hkv=8, d=128, bs=64, cap_tokens=4096, K=64, P=64)
    base.update(kw)
    assert (_abi.prr_workspace_bytes(_abi.Dims(**base)) > 0) == ok, kw


def test_argument_checks_return_before_any_launch(lib):
    d = _abi.Dims(B=1, Hq=4, Hkv=1, d=64, bs=64, cap_tokens=4096, K=8, P=8).c()
    null = ctypes.c_void_p(0)
    # null buffers: invalid argument
    st = lib.prr_select_topk(ctypes.byref(d), null, null, null, null, null, null, null, null, null, null)
    assert st == 1
    bad = _abi.Dims(B=1, Hq=4, Hkv=1, d=64, bs=64, cap_tokens=4096, K=0, P=8).c()
    st = lib.prr_select_topk(ctypes.byref(bad), null, null, null, null, null, null, null, null, null, null)
    assert st == 2  # K = 0: shape error
    # the no-workspace selection refuses shapes above its fixed scratch
    big = _abi.Dims(B=16, Hq=32, Hkv=8, d=128, bs=64, cap_tokens=8192 * 64 + 1, K=64, P=64).c()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    st = lib.prr_select_topk_static(ctypes.byref(big), fake, fake, fake, fake, fake, fake, fake, fake,
                                    null, null)
    assert st == 3


@pytest.mark.parametrize("lang,std", [("c", "c99"), ("c++", "c++17")])
def test_header_compiles_standalone(tmp_path, lang, std):
    """include/prr.h is a plain C header: it compiles on its own as C99 and as C++."""
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    src = tmp_path / ("t.c" if lang == "c" else "t.cpp")
    src.write_text('#include "prr.h"\nint main(void) { prr_dims d = {0}; (void)d; return PRR_OK; }\n')
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    r = subprocess.run([cc, "-fsyntax-only", "-Wall", "-Werror", f"-std={std}", "-I", os.path.join(ROOT, "include"),
                        "-I", cuda_inc, str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


@pytest.mark.parametrize("struct,cls", [("prr_dims", "PrrDims"), ("prr_step_buffers", "PrrStepBuffers"),
                                        ("prr_step_events", "PrrStepEvents")])
def test_binding_structs_match_the_header_layout(tmp_path, struct, cls):
    """The ctypes mirrors of the header's structs have the C compiler's layout: every
    field at the same offset, and the same size."""
    import shutil
    import subprocess
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no host compiler")
    mirror = getattr(_abi, cls)
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "prr.h"', 'int main(void) {',
             f'  printf("size %zu\\n", sizeof({struct}));']
    for name, _ in mirror._fields_:
        lines.append(f'  printf("{name} %zu\\n", offsetof({struct}, {name}));')
    lines += ['  return 0;', '}']
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    r = subprocess.run([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = dict(ln.split() for ln in subprocess.run([str(exe)], capture_output=True, text=True).stdout.splitlines())
    assert int(out["size"]) == ctypes.sizeof(mirror)
    for name, _ in mirror._fields_:
        assert int(out[name]) == getattr(mirror, name).offset, name


def test_readme_c_example_compiles(tmp_path):
    """The C example in README.md names only entry points, fields and constants that the
    header declares, with the right argument counts (it compiles as C99 inside a
    function that declares the buffers it uses)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no host compiler")
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```c\n(.*?)```", text, flags=re.S)
    assert len(blocks) == 1, "expected one C example"
    body = [ln for ln in blocks[0].splitlines() if not ln.startswith("#include")]
    decls = ("  uint16_t *k_cache = 0, *summ = 0; const int32_t *tok_begin = 0, *tok_end = 0;\n"
             "  int32_t *seq_lens = 0, *pred = 0; int32_t n0 = 0; double *ema = 0; void *ws = 0;\n"
             "  cudaStream_t stream = 0; int steps = 1; prr_step_buffers buf = {0};\n")
    src = tmp_path / "example.c"
    src.write_text('#include "prr.h"\nint example(void) {\n' + decls + "\n".join("  " + ln for ln in body)
                   + "\n  return 0;\n}\n")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    r = subprocess.run([cc, "-fsyntax-only", "-Wall", "-Werror", "-Wno-unused-variable", "-std=c99",
                        "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr + src.read_text()


def _ceiling_call(lib, call, d, maxnb):
    """Status of `call` with maxnb blocks and never-dereferenced buffer addresses."""
    dims = _abi.Dims(B=1, Hq=4, Hkv=1, d=d, bs=64, cap_tokens=maxnb * 64, K=8, P=8).c()
    fake, null = ctypes.c_void_p(1 << 20), ctypes.c_void_p(0)
    if call == "select":
        return lib.prr_select_topk(ctypes.byref(dims), fake, fake, fake, fake, fake, fake, fake, fake, fake, null)
    if call == "static":
        return lib.prr_select_topk_static(ctypes.byref(dims), fake, fake, fake, fake, fake, fake, fake, fake,
                                          null, null)
    if call == "ema":
        return lib.prr_ema_predict(ctypes.byref(dims), fake, fake, fake, fake, fake, null)
    buf = _abi.PrrStepBuffers()
    for i, (name, _) in enumerate(buf._fields_):  # distinct 16-byte-aligned addresses
        if name not in ("k_new", "v_new", "trace", "stats"):
            setattr(buf, name, (1 << 20) * (i + 1))
    big = ctypes.c_size_t(1 << 60)  # workspace size: never the limiting check here
    if call == "fused":
        return lib.prr_decode_step_fused(ctypes.byref(dims), ctypes.byref(buf), fake, big, 0, null)
    ev = _abi.PrrStepEvents()
    for i, name in enumerate(_abi.STEP_EVENTS):
        setattr(ev, name, (1 << 20) * (i + 1))
    return lib.prr_decode_step(ctypes.byref(dims), ctypes.byref(buf), fake, big, null, null, ctypes.byref(ev))


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="at a ceiling the call goes on to launch, which needs real buffers")
@pytest.mark.parametrize("call,d,limit", [
    ("select", 128, 19715), ("select", 64, 34800), ("static", 128, 19715), ("static", 64, 34800),
    ("ema", 128, 26890), ("ema", 64, 26890), ("streams", 128, 19715), ("streams", 64, 26890),
    ("fused", 128, 26760), ("fused", 64, 26760),
])
def test_shared_memory_ceilings_are_the_documented_ones(lib, call, d, limit):
    """The ceilings include/prr.h states, to the block: one block more is refused with
    PRR_ERR_SHAPE before anything is enqueued; at the ceiling the call passes every
    check and only fails on reaching the CUDA runtime (PRR_ERR_CUDA: no GPU here)."""
    assert f"{limit:,}" in open(HEADER).read()
    assert _ceiling_call(lib, call, d, limit + 1) == 2
    assert _ceiling_call(lib, call, d, limit) == 4


# (entry point, argument position, name) of every buffer a call needs 16-byte aligned.
_ALIGNED = {
    "prr_append_kv": (8, [(1, "k_new"), (2, "v_new"), (4, "k_cache"), (5, "v_cache")]),
    "prr_update_summaries": (9, [(1, "k_cache"), (6, "summ")]),
    "prr_select_topk": (11, [(2, "summ")]),
    "prr_select_topk_static": (11, [(2, "summ")]),
    "prr_speculate": (11, [(1, "q"), (2, "k_cache"), (3, "v_cache"), (8, "part_O")]),
    "prr_repair_merge": (16, [(1, "q"), (2, "k_cache"), (3, "v_cache"), (11, "part_O"), (12, "out")]),
}


@pytest.mark.parametrize("fn", sorted(_ALIGNED))
def test_misaligned_buffers_are_refused_before_anything_is_enqueued(lib, fn):
    """Every buffer that include/prr.h requires on a 16-byte boundary, moved 2 bytes off
    it, makes the call return PRR_ERR_INVALID_ARG (never-dereferenced addresses; the
    refusal comes before any CUDA call, so this runs with or without a GPU)."""
    nargs, aligned = _ALIGNED[fn]
    dims = _abi.Dims(B=1, Hq=4, Hkv=1, d=64, bs=64, cap_tokens=4096, K=8, P=8).c()
    for pos, name in aligned:
        args = [ctypes.byref(dims)] + [ctypes.c_void_p((1 << 20) * (i + 1)) for i in range(1, nargs - 1)]
        args.append(ctypes.c_void_p(0))  # stream
        if fn == "prr_update_summaries":
            args[5] = ctypes.c_int32(1)  # max_range_tokens
        if fn == "prr_select_topk_static":
            args[9] = ctypes.c_void_p(0)  # optional status
        args[pos] = ctypes.c_void_p(args[pos].value + 2)
        assert getattr(lib, fn)(*args) == 1, (fn, name)


def test_misaligned_step_buffers_are_refused(lib):
    dims = _abi.Dims(B=1, Hq=4, Hkv=1, d=64, bs=64, cap_tokens=4096, K=8, P=8).c()
    fake = ctypes.c_void_p(1 << 20)
    big = ctypes.c_size_t(1 << 60)
    ev = _abi.PrrStepEvents()
    for i, name in enumerate(_abi.STEP_EVENTS):
        setattr(ev, name, (1 << 20) * (i + 1))
    for name in ("q", "k_cache", "v_cache", "summ", "part_O", "out", "k_new", "v_new"):
        buf = _abi.PrrStepBuffers()
        for i, (field, _) in enumerate(buf._fields_):
            if field not in ("trace", "stats"):
                setattr(buf, field, (1 << 20) * (i + 1))
        setattr(buf, name, getattr(buf, name) + 2)
        assert lib.prr_decode_step_fused(ctypes.byref(dims), ctypes.byref(buf), fake, big, 0, None) == 1, name
        assert lib.prr_decode_step(ctypes.byref(dims), ctypes.byref(buf), fake, big, None, None,
                                   ctypes.byref(ev)) == 1, name


# (entry point, argument count, positions that must not be NULL, positions needed only
# when P > 0).  Positions count from 0 = dims; the last argument is the stream.
_REQUIRED = {
    "prr_append_kv": (8, [1, 2, 3, 4, 5, 6], []),
    "prr_update_summaries": (9, [1, 6, 7], []),
    "prr_select_topk": (11, [1, 2, 3, 5, 6, 7, 9], [4, 8]),
    "prr_select_topk_static": (11, [1, 2, 3, 5, 6, 7], [4, 8]),
    "prr_ema_predict": (7, [1, 3, 5], [4]),
    "prr_speculate": (11, [1, 2, 3, 4, 5, 6, 7, 8, 9], []),
    "prr_repair_merge": (16, [1, 2, 3, 4, 5, 6, 12, 13, 14], [7, 8, 9, 10, 11]),
}


def _args(fn, nargs, dims):
    args = [ctypes.byref(dims)] + [ctypes.c_void_p((1 << 20) * (i + 1)) for i in range(1, nargs - 1)]
    args.append(ctypes.c_void_p(0))
    if fn == "prr_update_summaries":
        args[5] = ctypes.c_int32(1)
    if fn == "prr_select_topk_static":
        args[9] = ctypes.c_void_p(0)
    return args


@pytest.mark.parametrize("fn", sorted(_REQUIRED))
def test_null_required_buffers_are_refused(lib, fn):
    """A NULL where include/prr.h needs a buffer returns PRR_ERR_INVALID_ARG before
    anything is enqueued; buffers of the speculative slots are needed only when P > 0."""
    nargs, always, with_p = _REQUIRED[fn]
    for P in (8, 0):
        dims = _abi.Dims(B=1, Hq=4, Hkv=1, d=64, bs=64, cap_tokens=4096, K=8, P=P).c()
        needed = always + (with_p if P > 0 else [])
        if fn == "prr_speculate" and P == 0:
            needed = []  # nothing to speculate: the call returns PRR_OK at once
            args = [ctypes.byref(dims)] + [ctypes.c_void_p(0)] * (nargs - 1)
            assert getattr(lib, fn)(*args) == 0
        for pos in needed:
            args = _args(fn, nargs, dims)
            args[pos] = ctypes.c_void_p(0)
            assert getattr(lib, fn)(*args) == 1, (fn, P, pos)


def test_summary_range_arguments(lib):
    """prr_update_summaries: tok_begin and tok_end come together; without them the call
    covers the token just appended, so it needs seq_lens and max_range_tokens = 1; the
    range bound lies in [1, cap_tokens]."""
    dims = _abi.Dims(B=1, Hq=4, Hkv=1, d=64, bs=64, cap_tokens=4096, K=8, P=8).c()

    def call(tb, te, sl, mr):
        args = _args("prr_update_summaries", 9, dims)
        args[2], args[3], args[4], args[5] = tb, te, sl, ctypes.c_int32(mr)
        return lib.prr_update_summaries(*args)

    a, null = ctypes.c_void_p(1 << 24), ctypes.c_void_p(0)
    assert call(a, null, a, 1) == 1 and call(null, a, a, 1) == 1  # one without the other
    assert call(null, null, null, 1) == 1                          # appended token needs seq_lens
    assert call(null, null, a, 2) == 2                             # appended token is one token
    assert call(a, a, null, 0) == 2 and call(a, a, null, 4097) == 2


def test_step_argument_rules(lib):
    """The decode steps: pred and pred_next must differ, the workspace must be at least
    prr_workspace_bytes, k_new and v_new come together, step_parity is 0 or 1, and the
    two-stream step needs its four ordering events."""
    d = _abi.Dims(B=1, Hq=4, Hkv=1, d=64, bs=64, cap_tokens=4096, K=8, P=8)
    dims = d.c()
    need = _abi.prr_workspace_bytes(d)
    ws = ctypes.c_void_p(1 << 20)

    def buffers(**change):
        buf = _abi.PrrStepBuffers()
        for i, (field, _) in enumerate(buf._fields_):
            if field not in ("k_new", "v_new", "trace", "stats"):
                setattr(buf, field, (1 << 24) * (i + 1))
        for k, v in change.items():
            setattr(buf, k, v)
        return buf

    def events(drop=None):
        ev = _abi.PrrStepEvents()
        for i, name in enumerate(_abi.STEP_EVENTS):
            setattr(ev, name, None if name == drop else (1 << 20) * (i + 1))
        return ev

    def fused(buf, nbytes=1 << 60, parity=0):
        return lib.prr_decode_step_fused(ctypes.byref(dims), ctypes.byref(buf), ws, ctypes.c_size_t(nbytes),
                                         parity, None)

    def streams(buf, nbytes=1 << 60, ev=None):
        return lib.prr_decode_step(ctypes.byref(dims), ctypes.byref(buf), ws, ctypes.c_size_t(nbytes), None, None,
                                   ctypes.byref(ev or events()))

    same = buffers()
    same.pred_next = same.pred
    assert fused(same) == 1 and streams(same) == 1
    assert fused(buffers(), nbytes=need - 1) == 3 and streams(buffers(), nbytes=need - 1) == 3
    half = buffers(k_new=1 << 30)
    assert fused(half) == 1 and streams(half) == 1
    assert fused(buffers(), parity=2) == 1 and fused(buffers(), parity=-1) == 1
    for name in _abi.STEP_EVENTS:
        assert streams(buffers(), ev=events(drop=name)) == 1, name
    for field in ("q", "k_cache", "v_cache", "seq_lens", "summ", "ema", "sel", "missed", "n_missed", "out", "lse",
                  "pred", "pred_next", "keep", "part_m", "part_l", "part_O"):
        assert fused(buffers(**{field: None})) == 1, field
