"""CPU oracle for the DSA sparse-prefill path -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / ``--impl reference`` legs may import this package.  The
product library never loads it and shares no code with it.

The arithmetic lives in ``dsa_oracle.c`` (plain C, fp64, single-threaded,
fixed loop order).  This module only builds that file with gcc, loads it with
ctypes and marshals numpy / torch CPU buffers into it.  ctypes releases the GIL
during each call, so callers may run disjoint rows on several threads.

Sources: mlx-lm PR #1997 "GLM prefill now attends only to the keys its indexer
picks" (section "How it works"), LiteTopK/LiteDSA (arXiv 2607.11976, Abstract),
llama.cpp PR #25917 (discussion: int32 index mask, -1 = masked).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
# Tests of the pins themselves point this at a prebuilt, deliberately mutated copy of the oracle.
_OVERRIDE = os.environ.get("DSA_ORACLE_LIB")
_LIB = _OVERRIDE or os.path.join(_HERE, "liboracle.so")

IDX_BF16 = 0
IDX_E4M3 = 1
MLA_LAT = 512
MLA_DIM = 576

_lib = None
_lock = threading.RLock()  # the worker threads of map_rows may all ask for the library at once


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c into liboracle.so (gcc -O2, strict IEEE: no fast-math)."""
    if _OVERRIDE:
        return _LIB
    with _lock:
        if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            fd, tmp = tempfile.mkstemp(prefix="liboracle.", suffix=".so.tmp", dir=_HERE)
            os.close(fd)
            try:
                subprocess.check_call(
                    ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
                     _SRC, "-o", tmp, "-lm"])
                os.replace(tmp, _LIB)
            finally:
                if os.path.exists(tmp):
                    os.remove(tmp)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        return _lib if _lib is not None else _load()


def _load() -> ctypes.CDLL:
    """Build (if stale) and load liboracle.so, declaring every entry point; called under _lock."""
    global _lib
    build()
    L = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    i32 = ctypes.c_int
    d = ctypes.c_double
    L.oracle_bf16_value.restype = d
    L.oracle_bf16_value.argtypes = [ctypes.c_uint16]
    L.oracle_e4m3_value.restype = d
    L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    L.oracle_indexer_scores.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, P]
    L.oracle_indexer_scores_range.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, i32, P]
    L.oracle_topk_fullsort.argtypes = [P, i32, i32, P, P]
    L.oracle_topk_blocked_fold.argtypes = [P, i32, i32, i32, P]
    L.oracle_sparse_mla.argtypes = [P, P, P, i32, i32, i32, i32, d, i32, P, P]
    L.oracle_dense_causal_mla.argtypes = [P, P, i32, i32, i32, i32, d, i32, P, P]
    L.oracle_prefill_row.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, P, P, i32, d, i32,
                                     P, P, P, P]
    for name in ("oracle_indexer_scores", "oracle_indexer_scores_range", "oracle_topk_fullsort",
                 "oracle_topk_blocked_fold", "oracle_sparse_mla", "oracle_dense_causal_mla", "oracle_prefill_row",
                 "oracle_version"):
        getattr(L, name).restype = i32
    _lib = L
    return _lib


def _ptr(a) -> int:
    """Address of a contiguous numpy array or torch CPU tensor."""
    if isinstance(a, np.ndarray):
        assert a.flags["C_CONTIGUOUS"]
        return a.ctypes.data
    assert a.device.type == "cpu" and a.is_contiguous()
    return a.data_ptr()


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


class Problem:
    """Raw buffers of one DSA prefill chunk, as the oracle reads them.

    q_idx [L,H_I,D_I] (bf16 or e4m3 bits), k_idx [N,D_I], w [L,H_I] fp32,
    q [L,H,576] bf16 bits, kv [N,576] bf16 bits.  Any of the MLA buffers may be
    None when only the indexer is checked.
    """

    def __init__(self, q_idx, k_idx, w, idx_dtype: int, L: int, N: int, H_I: int, D_I: int, q_pos0: int,
                 topk: int, q=None, kv=None, H: int = 0, scale: float = 0.0):
        self.q_idx, self.k_idx, self.w = q_idx, k_idx, w
        self.idx_dtype, self.L, self.N, self.H_I, self.D_I = idx_dtype, L, N, H_I, D_I
        self.q_pos0, self.topk, self.q, self.kv, self.H, self.scale = q_pos0, topk, q, kv, H, scale

    def nvis(self, t: int) -> int:
        return self.q_pos0 + t + 1


def indexer_scores(pb: Problem, t: int) -> np.ndarray:
    out = np.empty(pb.nvis(t), dtype=np.float64)
    _check(lib().oracle_indexer_scores(_ptr(pb.q_idx), _ptr(pb.k_idx), _ptr(pb.w), pb.idx_dtype, pb.L, pb.N,
                                       pb.H_I, pb.D_I, pb.q_pos0, t, _ptr(out)), "indexer_scores")
    return out


def indexer_scores_range(pb: Problem, t: int, lo: int, hi: int) -> np.ndarray:
    """Scores of query t over keys [lo, hi) (general causality through an index mask)."""
    out = np.empty(max(0, hi - lo), dtype=np.float64)
    _check(lib().oracle_indexer_scores_range(_ptr(pb.q_idx), _ptr(pb.k_idx), _ptr(pb.w), pb.idx_dtype, pb.L,
                                             pb.N, pb.H_I, pb.D_I, lo, hi, t, _ptr(out)), "indexer_scores_range")
    return out


def topk_row_range(pb: Problem, t: int, lo: int, hi: int):
    """(selected keys ascending with -1 padding, k-th score, score row of [lo, hi)) of query t over its range."""
    s = indexer_scores_range(pb, t, lo, hi)
    idx, kth = topk_fullsort(s, pb.topk)
    idx = np.where(idx >= 0, idx + lo, -1).astype(np.int32)
    return idx, kth, s


def topk_fullsort(scores: np.ndarray, topk: int):
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    idx = np.empty(topk, dtype=np.int32)
    kth = ctypes.c_double(0.0)
    _check(lib().oracle_topk_fullsort(_ptr(scores), scores.shape[0], topk, _ptr(idx), ctypes.addressof(kth)),
           "topk_fullsort")
    return idx, kth.value


def topk_blocked_fold(scores: np.ndarray, topk: int, block: int = 4096) -> np.ndarray:
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    idx = np.empty(topk, dtype=np.int32)
    _check(lib().oracle_topk_blocked_fold(_ptr(scores), scores.shape[0], topk, block, _ptr(idx)),
           "topk_blocked_fold")
    return idx


def sparse_mla(pb: Problem, t: int, idx_row) -> tuple[np.ndarray, np.ndarray]:
    idx_row = np.ascontiguousarray(np.asarray(idx_row, dtype=np.int32))
    out = np.empty((pb.H, MLA_LAT), dtype=np.float64)
    lse = np.empty(pb.H, dtype=np.float64)
    _check(lib().oracle_sparse_mla(_ptr(pb.q), _ptr(pb.kv), _ptr(idx_row), pb.L, pb.N, pb.H, idx_row.shape[0],
                                   pb.scale, t, _ptr(out), _ptr(lse)), "sparse_mla")
    return out, lse


def dense_causal_mla(pb: Problem, t: int) -> tuple[np.ndarray, np.ndarray]:
    out = np.empty((pb.H, MLA_LAT), dtype=np.float64)
    lse = np.empty(pb.H, dtype=np.float64)
    _check(lib().oracle_dense_causal_mla(_ptr(pb.q), _ptr(pb.kv), pb.L, pb.N, pb.H, pb.q_pos0, pb.scale, t,
                                         _ptr(out), _ptr(lse)), "dense_causal_mla")
    return out, lse


def topk_row(pb: Problem, t: int):
    """(selected keys ascending with -1 padding, k-th score, full score row) of query t."""
    s = indexer_scores(pb, t)
    idx, kth = topk_fullsort(s, pb.topk)
    return idx, kth, s


def prefill_row(pb: Problem, t: int):
    """Whole path for query t in one oracle call: (idx [topk], out [H,512], lse [H])."""
    scratch = np.empty(pb.nvis(t), dtype=np.float64)
    idx = np.empty(pb.topk, dtype=np.int32)
    out = np.empty((pb.H, MLA_LAT), dtype=np.float64)
    lse = np.empty(pb.H, dtype=np.float64)
    _check(lib().oracle_prefill_row(_ptr(pb.q_idx), _ptr(pb.k_idx), _ptr(pb.w), pb.idx_dtype, pb.L, pb.N, pb.H_I,
                                    pb.D_I, pb.q_pos0, pb.topk, _ptr(pb.q), _ptr(pb.kv), pb.H, pb.scale, t,
                                    _ptr(scratch), _ptr(idx), _ptr(out), _ptr(lse)), "prefill_row")
    return idx, out, lse


def map_rows(fn, rows, threads: int | None = None):
    """Run fn(row) over rows on a thread pool (the C calls release the GIL)."""
    rows = list(rows)
    threads = threads or os.cpu_count() or 1
    if threads <= 1 or len(rows) <= 1:
        return [fn(r) for r in rows]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, rows))
