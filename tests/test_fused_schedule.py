"""The fused decode step's work-item order, checked on the host.

`fused_schedule_check.cpp` enumerates the tickets of one launch through the header the
kernel includes (csrc/prr_schedule.h) for 8,400 shapes and grid sizes: every item is
handed out once, every item comes after the items it waits for (the property that
keeps the persistent grid free of deadlock), the dependent tickets trail their unit's
speculative tickets by two grid rounds, and a simulated grid that takes tickets the
way the kernel does always finishes.  Planted mistakes in copies of the header must
each fail it, and the Python mirror of the item counts (PRRDecoder.fused_items, which
sizes the trace buffer) must agree with the header.
"""
import os
import shutil
import subprocess
from types import SimpleNamespace

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "dynamic_sparse_attention_block_b200", "csrc")
HEADER = os.path.join(CSRC, "prr_schedule.h")
CHECK = os.path.join(ROOT, "tests", "fused_schedule_check.cpp")

GXX = shutil.which("g++")
pytestmark = pytest.mark.skipif(GXX is None, reason="needs the host C++ compiler")


def _build(tmp_path, header_text=None, defines=()):
    inc = CSRC
    if header_text is not None:
        inc = str(tmp_path / "inc")
        os.makedirs(inc, exist_ok=True)
        with open(os.path.join(inc, "prr_schedule.h"), "w") as f:
            f.write(header_text)
    exe = str(tmp_path / "fused_schedule_check")
    r = subprocess.run([GXX, "-std=c++17", "-O2", "-Wall", "-Werror", *defines, "-I", inc, CHECK, "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_ticket_order_is_complete_dependency_ordered_and_deadlock_free(tmp_path):
    r = subprocess.run([_build(tmp_path)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout
    assert "shapes 8400" in r.stdout and "failures 0" in r.stdout, r.stdout


# Each mutant: (replacements in the header, what it breaks).
MUTANTS = {
    # dependents right behind their own unit's SPEC tickets: order valid, no lag
    "no_lag": [("const int Lc = dep_lag < U ? dep_lag : U;", "const int Lc = 0;")],
    # a lag of one grid round instead of two
    "one_round_lag": [("(2 * grid + P - 1) / P", "(grid + P - 1) / P")],
    # the merge tickets indexed by the repair count
    "combine_index": [("*idx = v * G + (r - R);", "*idx = v * R + (r - R);")],
    # the launch's item count without the predictor updates
    "total_drops_ema": [("(fchunks + 1 + 1 + P + R + G)", "(fchunks + 1 + P + R + G)")],
    # a unit's dependents placed before its own SPEC tickets (a bijection that breaks
    # the dependency order, so the simulated grid deadlocks too)
    "dependents_first": [
        ("if (q < P) {\n      *idx = (Lc + k) * P + q;", "if (q >= M) {\n      *idx = (Lc + k) * P + (q - M);"),
        ("    v = k;\n    r = q - P;", "    v = Lc + k;\n    r = q;"),
        ("    v = U - Lc + t / M;", "    v = t / M;"),
    ],
    # the interleaved section sized without the merge tickets
    "mid_stride": [("const int mid = (U - Lc) * (P + M);", "const int mid = (U - Lc) * (P + R);")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_schedule_mistake_is_caught(tmp_path, name):
    text = open(HEADER).read()
    for old, new in MUTANTS[name]:
        assert old in text, f"mutant {name}: pattern not found in the header"
        text = text.replace(old, new)
    r = subprocess.run([_build(tmp_path, text)], capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "FAIL" in r.stdout, f"mutant {name} survived:\n{r.stdout}"


def test_simulated_grid_alone_catches_dependents_before_their_inputs(tmp_path):
    text = open(HEADER).read()
    for old, new in MUTANTS["dependents_first"]:
        text = text.replace(old, new)
    r = subprocess.run([_build(tmp_path, text, defines=("-DSIMULATION_ONLY",))], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode != 0 and "deadlocked" in r.stdout, r.stdout


def test_python_item_counts_match_the_header(tmp_path):
    from dynamic_sparse_attention_block_b200.decoder import PRRDecoder

    shapes = [(1, 1, 0, 1, 1), (8, 513, 64, 64, 4), (128, 1026, 32, 32, 4), (32, 4098, 64, 64, 8),
              (64, 1025, 64, 64, 4), (3, 33, 5, 3, 2), (300, 4100, 64, 128, 8), (1, 70000, 1, 1, 1)]
    r = subprocess.run([_build(tmp_path), "items"], input="".join("%d %d %d %d %d\n" % s for s in shapes),
                       capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    lines = r.stdout.splitlines()
    assert len(lines) == len(shapes)
    for (U, maxnb, P, K, G), line in zip(shapes, lines):
        dims = SimpleNamespace(units=U, maxnb=maxnb, P=P, K=K, group=G)
        got = PRRDecoder.fused_items(SimpleNamespace(dims=dims))
        order = ("sel", "finish", "ema", "spec", "repair", "combine")
        assert [got[k] for k in order] == [int(x) for x in line.split()], (U, maxnb, P, K, G)
