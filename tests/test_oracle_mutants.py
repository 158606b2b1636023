"""The oracle's pins must catch plausible mistakes.  Each case below plants
one mistake in a copy of the oracle's C source (on the CPU), builds it, loads
it in place of the real oracle and runs the pin suite; at least one pin must
fail.  The real oracle is restored afterwards."""
import inspect
import os
import shutil

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "hata_oracle.c")

MUTANTS = {
    "W_H transposed": ("fmaf(x[i], W[(int64_t)i * r + j], acc[j])",
                       "fmaf(x[i], W[(int64_t)j * d + i], acc[j])"),
    "sign test >= 0": ("if (acc[j] > 0.0f)", "if (acc[j] >= 0.0f)"),
    "bits packed MSB first": ("code[j / 32] |= 1u << (j % 32);",
                              "code[j / 32] |= 1u << (31 - j % 32);"),
    "projection in descending order": (
        "for (int i = 0; i < d; ++i)\n        for (int j = 0; j < r; ++j)",
        "for (int i = d - 1; i >= 0; --i)\n        for (int j = 0; j < r; ++j)"),
    "hamming counts equal bits": ("uint32_t x = a[j / 32] ^ b[j / 32];",
                                  "uint32_t x = ~(a[j / 32] ^ b[j / 32]);"),
    "ties go to the higher index": ("return a->i < b->i ? -1 : 1;",
                                    "return a->i > b->i ? -1 : 1;"),
    "largest distances selected": ("return a->d < b->d ? -1 : 1;",
                                   "return a->d > b->d ? -1 : 1;"),
    "one key too few when k >= n": ("int64_t m = k < n ? k : n;",
                                    "int64_t m = k < n ? k : n - 1;"),
    "softmax scale dropped": ("s[t] = scale * acc;", "s[t] = acc;"),
    "softmax not normalised": ("out[i] /= l;", "out[i] /= 1.0;"),
    "bf16 widened from the low half": ("uint32_t u = ((uint32_t)h) << 16;",
                                       "uint32_t u = ((uint32_t)h);"),
    "bf16 cache rows strided as 4-byte elements": (
        "row * d * (dtype == ORACLE_DT_BF16 ? 2 : 4);",
        "row * d * (dtype == ORACLE_DT_BF16 ? 4 : 4);"),
    "hamming stops at 128 bits": (
        "for (int j = 0; j < r; ++j) {\n        uint32_t x",
        "for (int j = 0; j < (r < 128 ? r : 128); ++j) {\n        uint32_t x"),
    "distance 256 counted as 255": (
        "dist += (int)((x >> (j % 32)) & 1u);\n    }\n    return dist;",
        "dist += (int)((x >> (j % 32)) & 1u);\n    }\n    return dist > 255 ? 255 : dist;"),
}


def _argsets(fn) -> list[dict]:
    """The keyword sets pytest would call a pin with (from its parametrize
    marks; a pin without marks runs once with no arguments)."""
    sets = [dict()]
    for mark in getattr(fn, "pytestmark", []):
        if mark.name != "parametrize":
            continue
        names = [n.strip() for n in mark.args[0].split(",")] if isinstance(mark.args[0], str) \
            else list(mark.args[0])
        combos = []
        for values in mark.args[1]:
            values = values if len(names) > 1 else (values,)
            combos.append(dict(zip(names, values)))
        sets = [dict(a, **b) for a in sets for b in combos]
    return sets


def _run_pins() -> int:
    failures = 0
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        for kw in _argsets(fn):
            try:
                fn(**kw)
            except Exception:
                failures += 1
    return failures


def test_pins_pass_on_the_real_oracle():
    """Without this, a pin that cannot run at all would 'catch' every mutant."""
    assert _run_pins() == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor not unique: {old!r}"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    lib = oracle.build(force=True, src=str(src), out=str(tmp_path / "libmutant.so"))
    oracle.use_library(lib)
    try:
        assert _run_pins() >= 1, f"no pin caught the mutant: {name}"
    finally:
        oracle.use_library(None)
    shutil.rmtree(tmp_path, ignore_errors=True)
