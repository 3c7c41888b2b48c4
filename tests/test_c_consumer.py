"""include/dsa.h is a plain C interface: a C99 program compiles against it with every warning as an
error, links libdsa.so and calls the entry points that need no GPU (CPU only)."""
import os
import subprocess

import pytest

from deepseek_sparse_attention_relu_b200 import build as dsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "dsa.h"

int main(void) {
  size_t ws;
  float scale = 0.0625f;
  int32_t idx[4] = {0, 1, 2, -1};
  if (dsa_version() != 1) return 1;
  if (strncmp(dsa_status_string(DSA_ERR_WORKSPACE), "DSA_ERR_WORKSPACE", 17) != 0) return 2;
  ws = dsa_prefill_chunk_workspace(1024, 131072, 32, 128, 64, 2048, 0, DSA_BF16, 1);
  if (ws == 0) return 3;
  if (dsa_indexer_topk_workspace(0, 10, 32, 128, 8, DSA_BF16) != 0) return 4;
  /* a host-side argument error comes back before anything reaches a device */
  if (dsa_sparse_mla_prefill(NULL, NULL, 0, idx, 1, 4, 64, 4, scale, NULL, NULL, NULL, 0, NULL)
      != DSA_ERR_INVALID_ARG) return 5;
  printf("ok %zu\n", ws);
  return 0;
}
"""


def test_c99_program_builds_links_and_runs(tmp_path):
    lib = dsa_build.build()
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(lib)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                           "-L", libdir, "-ldsa", f"-Wl,-rpath,{libdir}"])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.startswith("ok ")


def test_header_is_also_valid_cxx(tmp_path):
    src = tmp_path / "consumer.cc"
    src.write_text('#include "dsa.h"\nint main() { return dsa_version() == 1 ? 0 : 1; }\n')
    subprocess.check_call(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-fsyntax-only",
                           "-I", os.path.join(ROOT, "include"), str(src)])


if __name__ == "__main__":
    pytest.main([__file__])
