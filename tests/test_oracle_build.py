"""The oracle's lazy build is safe when many worker threads ask for a stale library at once (CPU only)."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import os, sys
sys.path.insert(0, sys.argv[1])
import oracle
oracle.build()
os.utime(oracle._LIB, (0, 0))          # older than dsa_oracle.c: the next lib() rebuilds it
vals = oracle.map_rows(lambda i: oracle.lib().oracle_bf16_value(0x3F80 + (i % 4)), list(range(64)), threads=16)
assert len(vals) == 64 and all(v >= 1.0 for v in vals), vals
assert os.path.getmtime(oracle._LIB) > 0
print("ok")
"""


def test_concurrent_rebuild_of_a_stale_oracle():
    env = {k: v for k, v in os.environ.items() if k != "DSA_ORACLE_LIB"}
    r = subprocess.run([sys.executable, "-c", SCRIPT, ROOT], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr[-2000:]
    leftovers = [f for f in os.listdir(os.path.join(ROOT, "oracle")) if f.endswith(".tmp")]
    assert leftovers == []
