"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in a temporary copy of oracle/dsa_oracle.c --
a dropped term, a wrong operand or index, an off-by-one, a reversed
tie-break, a bad decoder -- builds it with the oracle's own compiler flags,
and runs tests/test_oracle_pins.py against that library.  At least one pin
must fail for every mistake.  The committed oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dsa_oracle.c")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# (name, text in the oracle, replacement, which occurrence)
MUTANTS = [
    ("ReLU dropped from the indexer", "double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;", 0),
    ("ReLU dropped from the key-range indexer", "double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;", 1),
    ("head weight applied inside the ReLU",
     "double relu = dot > 0.0 ? dot : 0.0;\n            score += (double)w[(int64_t)t * H_I + h] * relu;",
     "double wd = (double)w[(int64_t)t * H_I + h] * dot;\n            score += wd > 0.0 ? wd : 0.0;", 0),
    ("query's own position not visible", "for (int s = 0; s <= p_t; ++s) {",
     "for (int s = 0; s <= p_t; ++s) { if (s == p_t) { out[s] = 0.0; continue; }", 0),
    ("indexer query heads and dims transposed", "((int64_t)t * H_I + h) * D_I + d)",
     "((int64_t)t * D_I + d) * H_I + h)", 0),
    ("ties go to the larger key index", "return (a->i > b->i) - (a->i < b->i);",
     "return (a->i < b->i) - (a->i > b->i);", 0),
    ("blocked fold keeps one key too few", "if (n > topk) n = topk;", "if (n > topk - 1) n = topk - 1;", 0),
    ("rope term dropped from the logits", "z[j] = scale * (lat + rope);", "z[j] = scale * lat;", 0),
    ("softmax scale not applied", "z[j] = scale * (lat + rope);", "z[j] = lat + rope;", 0),
    ("value read from the wrong columns", "out[d] += p * oracle_bf16_value(kr[d]);",
     "out[d] += p * oracle_bf16_value(kr[d + 64]);", 0),
    ("log-sum-exp without the running max", "*lse = m + log(Z);", "*lse = log(Z);", 0),
    ("bf16 decoded with a one-bit shift", "(uint32_t)bits << 16", "(uint32_t)bits << 15", 0),
    ("e4m3 exponent bias off by one", "ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)", 0),
]


def _build(c_source, tmp_path, stem):
    c = tmp_path / f"{stem}.c"
    c.write_text(c_source)
    lib = tmp_path / f"{stem}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
                           str(c), "-o", str(lib), "-lm"])
    return lib


def _run_pins(lib):
    env = dict(os.environ, DSA_ORACLE_LIB=str(lib))
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", PINS],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)


def test_pins_pass_on_an_unmodified_copy(tmp_path):
    """Control: the same build and run with the oracle as committed passes every pin."""
    with open(SRC) as f:
        r = _run_pins(_build(f.read(), tmp_path, "dsa_oracle_copy"))
    assert r.returncode == 0, r.stdout[-2000:]


def _mutate(src, old, new, occurrence):
    start = -1
    for _ in range(occurrence + 1):
        start = src.find(old, start + 1)
        assert start >= 0, f"the oracle no longer contains {old!r} (occurrence {occurrence})"
    return src[:start] + new + src[start + len(old):]


@pytest.mark.parametrize("name,old,new,occurrence", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, old, new, occurrence, tmp_path):
    with open(SRC) as f:
        src = f.read()
    r = _run_pins(_build(_mutate(src, old, new, occurrence), tmp_path, "dsa_oracle_mutant"))
    # exit status 1 = some test failed (not a collection error or a crash)
    assert r.returncode == 1, f"no pin fails when the oracle has this mistake: {name}\n{r.stdout[-2000:]}"
