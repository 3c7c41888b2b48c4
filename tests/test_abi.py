"""The C-ABI library loads, exports every declared entry point and rejects bad arguments on the host (CPU only)."""
import ctypes
import os
import re

import pytest

import deepseek_sparse_attention_relu_b200 as dsa
from deepseek_sparse_attention_relu_b200 import build as dsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    dsa_build.build()
    return dsa.lib()


def _declared_functions():
    with open(os.path.join(ROOT, "include", "dsa.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 9
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(dsa.EXPORTED)


def test_version_and_status_strings(lib):
    assert lib.dsa_version() == 1
    for code in range(6):
        assert lib.dsa_status_string(code).decode().startswith(dsa.STATUS_NAMES[code])


def test_workspace_sizes(lib):
    a = lib.dsa_indexer_topk_workspace(1024, 131072, 32, 128, 2048, 0)
    b = lib.dsa_indexer_topk_workspace(4096, 131072, 32, 128, 2048, 0)
    assert a > 1024 * 8192 * 8 and a == b  # query blocks of 1,024 bound the workspace
    assert lib.dsa_indexer_topk_workspace(0, 10, 32, 128, 8, 0) == 0
    # one query (decode): one exact-fallback score row and one candidate list, however many fallback CTAs run
    assert lib.dsa_indexer_topk_workspace(1, 131072, 32, 128, 2048, 0) < (1 << 20)
    # a 1,024-query block holds at least 16 fallback score rows of N floats
    assert a > 16 * 131072 * 4 + 1024 * 8192 * 8
    c = lib.dsa_prefill_chunk_workspace(1024, 131072, 32, 128, 64, 2048, 0, 0, 0)
    d = lib.dsa_prefill_chunk_workspace(1024, 131072, 32, 128, 64, 2048, 0, 0, 1)
    assert c - d >= 1024 * 2048 * 4
    assert lib.dsa_sparse_mla_workspace(8, 64, 2048) >= 4


def _P(x):
    return ctypes.c_void_p(x)


def test_argument_errors_before_any_launch(lib):
    """Shape / pointer errors come back synchronously, before any launch or copy.

    Every call here fails a host-side check, so the fake pointers are never
    handed to the device (valid strides are exercised with real buffers by
    the GPU tests)."""
    fake = 1 << 20  # a 16-byte-aligned non-null address that is never dereferenced
    ws = 1 << 24
    call = lambda **kw: lib.dsa_indexer_topk(  # noqa: E731
        _P(kw.get("q", fake)), _P(kw.get("k", fake)), kw.get("ldk", 0), _P(kw.get("w", fake)), kw.get("dt", 0),
        kw.get("L", 4),
        kw.get("N", 100), kw.get("H_I", 32), kw.get("D_I", 128), kw.get("q_pos0", 96), kw.get("topk", 8),
        _P(kw.get("idx", fake)), None, _P(ws), 1 << 30, None)
    assert call(q=0) == 1                 # null pointer
    assert call(q=fake + 4) == 1          # misaligned
    assert call(q_pos0=97) == 1           # q_pos0 + L > N
    assert call(q_pos0=-1) == 1
    assert call(L=0) == 1
    assert call(topk=0) == 1
    assert call(dt=7) == 1
    assert call(topk=5000) == 2           # beyond the supported top-k
    assert call(H_I=3) == 2               # unsupported head count
    assert call(D_I=96) == 2
    assert call(ldk=100) == 1             # row stride shorter than a row
    assert call(ldk=132) == 1             # rows not 16-byte aligned (132 bf16 = 264 B)
    st = lib.dsa_sparse_mla_prefill(_P(fake), _P(fake), 0, _P(0), 4, 100, 8, 16, ctypes.c_float(0.1), _P(fake),
                                    None, _P(ws), 256, None)
    assert st == 1
    st = lib.dsa_sparse_mla_prefill(_P(fake), _P(fake), 580, _P(fake), 4, 100, 8, 16, ctypes.c_float(0.1),
                                    _P(fake), None, _P(ws), 256, None)
    assert st == 1                        # kv rows not 16-byte aligned
    st = lib.dsa_sparse_mla_prefill(_P(fake), _P(fake), 0, _P(fake), 4, 100, 8, 16, ctypes.c_float(0.1), _P(fake),
                                    None, None, 0, None)
    assert st == 3                        # no workspace


def test_argument_errors_other_entry_points(lib):
    """The chunk, per-query-range, profiled and self-test entry points also refuse bad arguments up front."""
    fake = 1 << 20
    ws = 1 << 24
    scale = ctypes.c_float(0.1)
    # per-query key ranges without the range arrays
    assert lib.dsa_indexer_topk_ranges(_P(fake), _P(fake), 0, _P(fake), 0, 4, 100, 32, 128, None, None, 8,
                                       _P(fake), None, _P(ws), 1 << 30, None) == 1
    assert lib.dsa_prefill_chunk_ranges(_P(fake), _P(fake), 0, _P(fake), 0, _P(fake), _P(fake), 0, 4, 100, 32, 128,
                                        64, None, None, 8, scale, 0, _P(fake), _P(fake), None, _P(ws), 1 << 30,
                                        None) == 1

    def chunk(dt=0, ldkv=0, q_pos0=96, H=64):
        return lib.dsa_prefill_chunk(_P(fake), _P(fake), 0, _P(fake), dt, _P(fake), _P(fake), ldkv, 4, 100, 32, 128,
                                     H, q_pos0, 8, scale, 0, _P(fake), _P(fake), None, _P(ws), 1 << 30, None)
    assert chunk(q_pos0=97) == 1          # q_pos0 + L > N
    assert chunk(dt=5) == 1               # unknown indexer dtype
    assert chunk(ldkv=580) == 1           # kv rows not 16-byte aligned
    assert chunk(H=0) == 1                # no attention heads
    # the profiled entry point needs its events
    assert lib.dsa_prefill_chunk_profiled(_P(fake), _P(fake), 0, _P(fake), 0, _P(fake), _P(fake), 0, 4, 100, 32,
                                          128, 64, 96, 8, scale, 0, _P(fake), _P(fake), None, _P(ws), 1 << 30,
                                          None, None, 0) == 1
    # the bounded-wait self-test checks its workspace and limit before anything runs
    assert lib.dsa_selftest_wait_timeout(None, 0, 50, None) == 3
    assert lib.dsa_selftest_wait_timeout(_P(ws), 4096, 0, None) == 1
    assert lib.dsa_selftest_wait_timeout(_P(ws), 4096, 5000, None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(2, 32, 128, dtype=torch.bfloat16)
    k = torch.zeros(16, 128, dtype=torch.bfloat16)
    w = torch.zeros(2, 32)
    idx = torch.zeros(2, 4, dtype=torch.int32)
    with pytest.raises(ValueError):
        dsa.dsa_indexer_topk(q, k, w, 14, 4, idx, workspace=torch.zeros(256, dtype=torch.uint8))
