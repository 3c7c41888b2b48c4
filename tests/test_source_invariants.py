"""Static checks on the CUDA sources that the launch path relies on (CPU only).

Every kernel of the library is launched with programmatic stream serialisation
(it may be scheduled while the previous kernel in the stream is still running),
so each one must wait for its prerequisite grids before it touches memory.  The
launcher helper is the only way kernels are started.
"""
import os
import re

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "deepseek_sparse_attention_relu_b200", "csrc")
SOURCES = sorted(f for f in os.listdir(CSRC) if f.endswith(".cu"))


def _close(text, i):
    """Index of the parenthesis that closes the one at text[i]."""
    depth = 0
    for j in range(i, len(text)):
        if text[j] == "(":
            depth += 1
        elif text[j] == ")":
            depth -= 1
            if depth == 0:
                return j
    raise AssertionError("unbalanced parentheses")


def kernel_bodies(text):
    """(name, first statement of the body) of every __global__ function in a source file."""
    out = []
    for m in re.finditer(r"__global__\s+void\s+", text):
        i = m.end()
        if text.startswith("__launch_bounds__", i):
            i = _close(text, text.index("(", i)) + 1
        paren = text.index("(", i)
        name = text[i:paren].strip()
        assert re.fullmatch(r"\w+", name), f"cannot parse the kernel name near {text[m.start():paren + 1]!r}"
        j = _close(text, paren)
        brace = text.index("{", j)
        assert text[j + 1:brace].strip() == "", f"unexpected text between the parameters and body of {name}"
        first = text[brace + 1:].lstrip().split(";", 1)[0].strip()
        out.append((name, first))
    return out


def test_sources_found():
    assert {"api.cu", "indexer.cu", "mla.cu", "select.cu"} <= set(SOURCES)


@pytest.mark.parametrize("fname", SOURCES)
def test_every_kernel_waits_for_its_predecessor_first(fname):
    with open(os.path.join(CSRC, fname)) as f:
        text = f.read()
    for name, first in kernel_bodies(text):
        assert first == "pdl_wait_and_release()", f"{fname}: kernel {name} starts with {first!r}"


@pytest.mark.parametrize("fname", SOURCES)
def test_kernels_are_started_only_through_the_launcher(fname):
    with open(os.path.join(CSRC, fname)) as f:
        text = f.read()
    assert "<<<" not in text, f"{fname}: a triple-chevron launch bypasses launch_kernel()"
