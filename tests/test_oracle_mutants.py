"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that every
one of them fails at least one pin.  This is the evidence that the pins constrain each
part of the oracle: a dropped term, a wrong sign or index, a transposed operand."""
import os
import subprocess

import pytest

import oracle
from oracle import build as obuild
from oracle_pins import ALL_PINS

MUTANTS = [
    ("drop (1-f) weight", "(1.0 - (double)f) * x_at(x, S, b, ci, i0)", "x_at(x, S, b, ci, i0)"),
    ("swap lerp weights", "double v = (1.0 - (double)f) * x_at(x, S, b, ci, i0) + (double)f * x_at(x, S, b, ci, i0 + 1);",
     "double v = (double)f * x_at(x, S, b, ci, i0) + (1.0 - (double)f) * x_at(x, S, b, ci, i0 + 1);"),
    ("wrong right neighbour", "x_at(x, S, b, ci, i0 + 1)", "x_at(x, S, b, ci, i0 - 1)"),
    ("offset sign", "float pos = (float)base + off;", "float pos = (float)base - off;"),
    ("dilation dropped", "int64_t base = start + k * S->dilation;", "int64_t base = start + k;"),
    ("padding sign", "int64_t start = l * S->stride - S->padding;",
     "int64_t start = l * S->stride + S->padding;"),
    ("stride dropped", "int64_t start = l * S->stride - S->padding;",
     "int64_t start = l - S->padding;"),
    ("offset group strided", "int64_t og = ci / cin_per_og;", "int64_t og = ci % S->offset_groups;"),
    ("kernel flipped (convolution)", "acc += (double)w[(co * cin_g + c) * S->K + k] * v;",
     "acc += (double)w[(co * cin_g + c) * S->K + (S->K - 1 - k)] * v;"),
    ("bias dropped", "double acc = bias ? (double)bias[co] : 0.0;", "double acc = 0.0;"),
    ("mask ignored", "v *= (double)mask[oidx];", "v *= 1.0;"),
    ("edge replicated, not zero", "    if (i < 0 || i >= S->L_in)\n        return 0.0;",
     "    if (i < 0) i = 0;\n    if (i >= S->L_in) i = S->L_in - 1;"),
    ("upper clamp missing", "        if (pos > hi) pos = hi;\n", ""),
    ("lower clamp missing", "        if (pos < lo) pos = lo;\n", ""),
    ("clamp to a per-tap cell", "float hi = (float)(start + S->dilation * (S->K - 1));",
     "float hi = (float)(base + S->dilation);"),
    ("trunc instead of floor", "float fl = floorf(pos);", "float fl = truncf(pos);"),
    ("fraction from the offset", "*f = pos - (float)(*i0);", "*f = off - floorf(off);"),
    ("L_out off by one", "return num / s + 1;", "return num / s;"),
    ("groups ignored in channel base", "int64_t ci = g * cin_g + c;", "int64_t ci = c;"),
]


def _build_mutant(tmp_path, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    path = os.path.join(tmp_path, "mut.c")
    with open(path, "w") as fh:
        fh.write(src.replace(old, new))
    lib = os.path.join(tmp_path, "libmut.so")
    subprocess.run(["gcc", *obuild.CFLAGS, "-w", "-o", lib, path, "-lm"], check=True)
    return oracle.Oracle(lib)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    o = _build_mutant(str(tmp_path), old, new)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake: {name}"
