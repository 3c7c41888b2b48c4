"""Python binding of libdsa.so, the B200 (sm_100a) DeepSeek Sparse Attention prefill path.

Argument marshalling only: every function here checks tensor placement and
layout, turns torch CUDA tensors into raw device pointers plus the current CUDA
stream, and calls the C entry point of the same name declared in
include/dsa.h.  All arithmetic runs in the library's CUDA kernels; there is no
CPU fallback.  If libdsa.so is missing the first call raises.

PyTorch is used only for device memory and streams.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

DSA_OK = 0
DSA_BF16 = 0
DSA_FP8_E4M3 = 1
STATUS_NAMES = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_WORKSPACE",
                4: "DSA_ERR_CUDA", 5: "DSA_ERR_INTERNAL"}

EXPORTED = ("dsa_version", "dsa_status_string", "dsa_last_error_string", "dsa_indexer_topk_workspace", "dsa_indexer_topk",
            "dsa_sparse_mla_workspace", "dsa_sparse_mla_prefill", "dsa_prefill_chunk_workspace",
            "dsa_prefill_chunk", "dsa_prefill_chunk_profiled", "dsa_workspace_status",
            "dsa_indexer_topk_noalloc", "dsa_indexer_topk_ranges", "dsa_prefill_chunk_ranges",
            "dsa_selftest_wait_timeout", "dsa_indexer_topk_noalloc_status", "dsa_workspace_selection_stats")

_lib = None


class SelectionStats(ctypes.Structure):
    """dsa_selection_stats_t (include/dsa.h)."""
    _fields_ = [("candidates", ctypes.c_ulonglong), ("queries", ctypes.c_uint), ("fallback_queries", ctypes.c_uint),
                ("max_candidates", ctypes.c_uint), ("reserved", ctypes.c_uint)]


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().dsa_status_string(status).decode()
        if status == 4:
            msg += f" ({lib().dsa_last_error_string().decode()})"
        super().__init__(f"{where}: {msg}")


def lib() -> ctypes.CDLL:
    """Load libdsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdsa.so not found at {LIB_PATH}; build it with "
                               "`python -m deepseek_sparse_attention_relu_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        L.dsa_version.restype = I
        L.dsa_version.argtypes = []
        L.dsa_status_string.restype = ctypes.c_char_p
        L.dsa_status_string.argtypes = [I]
        L.dsa_last_error_string.restype = ctypes.c_char_p
        L.dsa_last_error_string.argtypes = []
        L.dsa_indexer_topk_workspace.restype = Z
        L.dsa_indexer_topk_workspace.argtypes = [I, I, I, I, I, I]
        L.dsa_indexer_topk.restype = I
        LL = ctypes.c_longlong
        L.dsa_indexer_topk.argtypes = [P, P, LL, P, I, I, I, I, I, I, I, P, P, P, Z, P]
        L.dsa_sparse_mla_workspace.restype = Z
        L.dsa_sparse_mla_workspace.argtypes = [I, I, I]
        L.dsa_sparse_mla_prefill.restype = I
        L.dsa_sparse_mla_prefill.argtypes = [P, P, LL, P, I, I, I, I, F, P, P, P, Z, P]
        L.dsa_prefill_chunk_workspace.restype = Z
        L.dsa_prefill_chunk_workspace.argtypes = [I, I, I, I, I, I, I, I, I]
        L.dsa_prefill_chunk.restype = I
        L.dsa_prefill_chunk.argtypes = [P, P, LL, P, I, P, P, LL, I, I, I, I, I, I, I, F, I, P, P, P, P, Z, P]
        L.dsa_prefill_chunk_profiled.restype = I
        L.dsa_prefill_chunk_profiled.argtypes = [P, P, LL, P, I, P, P, LL, I, I, I, I, I, I, I, F, I, P, P, P, P, Z,
                                                 P, P, I]
        L.dsa_indexer_topk_noalloc.restype = I
        L.dsa_indexer_topk_noalloc.argtypes = [P, P, LL, P, I, I, I, I, I, I, I, P, P, P]
        L.dsa_indexer_topk_ranges.restype = I
        L.dsa_indexer_topk_ranges.argtypes = [P, P, LL, P, I, I, I, I, I, P, P, I, P, P, P, Z, P]
        L.dsa_prefill_chunk_ranges.restype = I
        L.dsa_prefill_chunk_ranges.argtypes = [P, P, LL, P, I, P, P, LL, I, I, I, I, I, P, P, I, F, I, P, P, P, P, Z,
                                               P]
        L.dsa_selftest_wait_timeout.restype = I
        L.dsa_selftest_wait_timeout.argtypes = [P, Z, ctypes.c_uint, P]
        L.dsa_workspace_status.restype = I
        L.dsa_workspace_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint)]
        L.dsa_indexer_topk_noalloc_status.restype = I
        L.dsa_workspace_selection_stats.restype = I
        L.dsa_workspace_selection_stats.argtypes = [P, P, ctypes.POINTER(SelectionStats)]
        L.dsa_indexer_topk_noalloc_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint)]
        _lib = L
    return _lib


def _dev(t: torch.Tensor | None, name: str, dtypes=None) -> int | None:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    return t.data_ptr()


def _rows(t: torch.Tensor, name: str, dtypes=None) -> tuple[int, int]:
    """(pointer, row stride in elements) of a 2-D CUDA tensor whose rows are contiguous (a padded cache or
    a view of the leading columns of a wider buffer)."""
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 2 or t.stride(1) != 1 or t.stride(0) < t.shape[1]:
        raise ValueError(f"{name} must be 2-D with contiguous rows")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    return t.data_ptr(), t.stride(0)


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DSA_BF16
    if t.dtype == torch.float8_e4m3fn:
        return DSA_FP8_E4M3
    raise ValueError(f"indexer operands must be bfloat16 or float8_e4m3fn, got {t.dtype}")


def _check(status: int, where: str) -> None:
    if status != DSA_OK:
        raise DSAError(status, where)


def dsa_version() -> int:
    return lib().dsa_version()


def dsa_indexer_topk_workspace(L: int, N: int, H_I: int, D_I: int, topk: int, dtype: int = DSA_BF16) -> int:
    return lib().dsa_indexer_topk_workspace(L, N, H_I, D_I, topk, dtype)


def dsa_sparse_mla_workspace(L: int, H: int, topk: int) -> int:
    return lib().dsa_sparse_mla_workspace(L, H, topk)


def dsa_prefill_chunk_workspace(L: int, N: int, H_I: int, D_I: int, H: int, topk: int, query_block: int = 0,
                                dtype: int = DSA_BF16, want_topk_out: bool = True) -> int:
    return lib().dsa_prefill_chunk_workspace(L, N, H_I, D_I, H, topk, query_block, dtype, int(want_topk_out))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A device byte buffer of at least nbytes (the caller owns it)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def dsa_indexer_topk(q_idx: torch.Tensor, k_idx: torch.Tensor, w: torch.Tensor, q_pos0: int, topk: int,
                     topk_idx: torch.Tensor, topk_score: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, stream=None) -> None:
    """Stages 1+2: indexer scores and exact top-k.  Shapes: q_idx [L,H_I,D_I], k_idx [N,D_I], w [L,H_I] fp32,
    topk_idx [L,topk] int32 (out), topk_score [L,topk] fp32 (optional out)."""
    L, H_I, D_I = q_idx.shape
    N = k_idx.shape[0]
    dt = _dtype_code(q_idx)
    if k_idx.dtype != q_idx.dtype or k_idx.shape[1] != D_I or tuple(w.shape) != (L, H_I):
        raise ValueError("inconsistent indexer operand shapes or dtypes")
    if tuple(topk_idx.shape) != (L, topk):
        raise ValueError("topk_idx must be [L, topk]")
    if workspace is None:
        workspace = alloc_workspace(dsa_indexer_topk_workspace(L, N, H_I, D_I, topk, dt), q_idx.device)
    _check(lib().dsa_indexer_topk(
        _dev(q_idx, "q_idx"), *_rows(k_idx, "k_idx"), _dev(w, "w", (torch.float32,)), dt, L, N, H_I, D_I, q_pos0,
        topk, _dev(topk_idx, "topk_idx", (torch.int32,)), _dev(topk_score, "topk_score", (torch.float32,)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)),
        "dsa_indexer_topk")


def dsa_indexer_topk_ranges(q_idx: torch.Tensor, k_idx: torch.Tensor, w: torch.Tensor, key_lo: torch.Tensor,
                            key_hi: torch.Tensor, topk: int, topk_idx: torch.Tensor,
                            topk_score: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                            stream=None) -> None:
    """dsa_indexer_topk with general visibility: query t sees keys key_lo[t] <= s < key_hi[t] (int32 CUDA
    tensors [L]) instead of the causal prefix."""
    L, H_I, D_I = q_idx.shape
    N = k_idx.shape[0]
    dt = _dtype_code(q_idx)
    if k_idx.dtype != q_idx.dtype or k_idx.shape[1] != D_I or tuple(w.shape) != (L, H_I):
        raise ValueError("inconsistent indexer operand shapes or dtypes")
    if tuple(topk_idx.shape) != (L, topk) or key_lo.numel() != L or key_hi.numel() != L:
        raise ValueError("topk_idx must be [L, topk] and key_lo / key_hi [L]")
    if workspace is None:
        workspace = alloc_workspace(dsa_indexer_topk_workspace(L, N, H_I, D_I, topk, dt), q_idx.device)
    _check(lib().dsa_indexer_topk_ranges(
        _dev(q_idx, "q_idx"), *_rows(k_idx, "k_idx"), _dev(w, "w", (torch.float32,)), dt, L, N, H_I, D_I,
        _dev(key_lo, "key_lo", (torch.int32,)), _dev(key_hi, "key_hi", (torch.int32,)), topk,
        _dev(topk_idx, "topk_idx", (torch.int32,)), _dev(topk_score, "topk_score", (torch.float32,)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)),
        "dsa_indexer_topk_ranges")


def dsa_indexer_topk_noalloc(q_idx: torch.Tensor, k_idx: torch.Tensor, w: torch.Tensor, q_pos0: int, topk: int,
                             topk_idx: torch.Tensor, topk_score: torch.Tensor | None = None, stream=None) -> None:
    """dsa_indexer_topk without a workspace, for callers that cannot allocate device memory (a runtime that
    plans all memory up front and hands kernels only their inputs and outputs, or a device fully reserved by
    others).  The scratch is a fixed 16 MiB array inside libdsa.so shared by every call on the device: calls
    that overlap on the GPU race, and problems too large for it raise DSAError(DSA_ERR_WORKSPACE).  The first
    call on a device looks up the array's address, so make it before any stream capture.  Device-side
    conditions are read with dsa_indexer_topk_noalloc_status()."""
    L, H_I, D_I = q_idx.shape
    N = k_idx.shape[0]
    dt = _dtype_code(q_idx)
    if k_idx.dtype != q_idx.dtype or k_idx.shape[1] != D_I or tuple(w.shape) != (L, H_I):
        raise ValueError("inconsistent indexer operand shapes or dtypes")
    if tuple(topk_idx.shape) != (L, topk):
        raise ValueError("topk_idx must be [L, topk]")
    _check(lib().dsa_indexer_topk_noalloc(
        _dev(q_idx, "q_idx"), *_rows(k_idx, "k_idx"), _dev(w, "w", (torch.float32,)), dt, L, N, H_I, D_I, q_pos0,
        topk, _dev(topk_idx, "topk_idx", (torch.int32,)), _dev(topk_score, "topk_score", (torch.float32,)),
        _stream(stream)), "dsa_indexer_topk_noalloc")


def dsa_sparse_mla_prefill(q: torch.Tensor, kv: torch.Tensor, topk_idx: torch.Tensor, scale: float,
                           out: torch.Tensor, lse: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None, stream=None) -> None:
    """Stage 3: sparse absorbed-MLA attention.  q [L,H,576] bf16, kv [N,576] bf16, topk_idx [L,topk] int32,
    out [L,H,512] bf16 (out), lse [L,H] fp32 (optional out)."""
    L, H, D = q.shape
    N = kv.shape[0]
    topk = topk_idx.shape[1]
    if D != 576 or kv.shape[1] != 576 or tuple(out.shape) != (L, H, 512) or topk_idx.shape[0] != L:
        raise ValueError("inconsistent MLA operand shapes")
    if workspace is None:
        workspace = alloc_workspace(dsa_sparse_mla_workspace(L, H, topk), q.device)
    _check(lib().dsa_sparse_mla_prefill(
        _dev(q, "q", (torch.bfloat16,)), *_rows(kv, "kv", (torch.bfloat16,)), _dev(topk_idx, "topk_idx", (torch.int32,)),
        L, N, H, topk, float(scale), _dev(out, "out", (torch.bfloat16,)), _dev(lse, "lse", (torch.float32,)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)),
        "dsa_sparse_mla_prefill")


def dsa_prefill_chunk(q_idx: torch.Tensor, k_idx: torch.Tensor, w: torch.Tensor, q: torch.Tensor, kv: torch.Tensor,
                      q_pos0: int, topk: int, scale: float, out: torch.Tensor, topk_idx: torch.Tensor | None = None,
                      lse: torch.Tensor | None = None, query_block: int = 0,
                      workspace: torch.Tensor | None = None, stream=None) -> None:
    """All three stages for one prefill chunk, per query block (query_block <= 0: 1,024)."""
    L, H_I, D_I = q_idx.shape
    N = k_idx.shape[0]
    H = q.shape[1]
    dt = _dtype_code(q_idx)
    if workspace is None:
        workspace = alloc_workspace(dsa_prefill_chunk_workspace(L, N, H_I, D_I, H, topk, query_block, dt,
                                                                topk_idx is not None), q.device)
    _check(lib().dsa_prefill_chunk(
        _dev(q_idx, "q_idx"), *_rows(k_idx, "k_idx"), _dev(w, "w", (torch.float32,)), dt,
        _dev(q, "q", (torch.bfloat16,)), *_rows(kv, "kv", (torch.bfloat16,)), L, N, H_I, D_I, H, q_pos0, topk,
        float(scale), query_block, _dev(topk_idx, "topk_idx", (torch.int32,)), _dev(out, "out", (torch.bfloat16,)),
        _dev(lse, "lse", (torch.float32,)), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)), "dsa_prefill_chunk")


def dsa_prefill_chunk_ranges(q_idx: torch.Tensor, k_idx: torch.Tensor, w: torch.Tensor, q: torch.Tensor,
                             kv: torch.Tensor, key_lo: torch.Tensor, key_hi: torch.Tensor, topk: int, scale: float,
                             out: torch.Tensor, topk_idx: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                             query_block: int = 0, workspace: torch.Tensor | None = None, stream=None) -> None:
    """dsa_prefill_chunk with general visibility: query t sees keys key_lo[t] <= s < key_hi[t]."""
    L, H_I, D_I = q_idx.shape
    N = k_idx.shape[0]
    H = q.shape[1]
    dt = _dtype_code(q_idx)
    if key_lo.numel() != L or key_hi.numel() != L:
        raise ValueError("key_lo / key_hi must have one entry per query")
    if workspace is None:
        workspace = alloc_workspace(dsa_prefill_chunk_workspace(L, N, H_I, D_I, H, topk, query_block, dt,
                                                                topk_idx is not None), q.device)
    _check(lib().dsa_prefill_chunk_ranges(
        _dev(q_idx, "q_idx"), *_rows(k_idx, "k_idx"), _dev(w, "w", (torch.float32,)), dt,
        _dev(q, "q", (torch.bfloat16,)), *_rows(kv, "kv", (torch.bfloat16,)), L, N, H_I, D_I, H,
        _dev(key_lo, "key_lo", (torch.int32,)), _dev(key_hi, "key_hi", (torch.int32,)), topk, float(scale),
        query_block, _dev(topk_idx, "topk_idx", (torch.int32,)), _dev(out, "out", (torch.bfloat16,)),
        _dev(lse, "lse", (torch.float32,)), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)), "dsa_prefill_chunk_ranges")


def dsa_prefill_chunk_profiled(q_idx: torch.Tensor, k_idx: torch.Tensor, w: torch.Tensor, q: torch.Tensor,
                               kv: torch.Tensor, q_pos0: int, topk: int, scale: float, out: torch.Tensor,
                               events: list, topk_idx: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                               query_block: int = 0, workspace: torch.Tensor | None = None, stream=None) -> None:
    """dsa_prefill_chunk recording 7 CUDA events per query block between its stages (see include/dsa.h).

    events: torch.cuda.Event objects that have been recorded at least once (so their handles exist), or None
    for a boundary that should not be marked."""
    L, H_I, D_I = q_idx.shape
    N = k_idx.shape[0]
    H = q.shape[1]
    dt = _dtype_code(q_idx)
    if workspace is None:
        workspace = alloc_workspace(dsa_prefill_chunk_workspace(L, N, H_I, D_I, H, topk, query_block, dt,
                                                                topk_idx is not None), q.device)
    handles = (ctypes.c_void_p * len(events))(*[None if e is None else e.cuda_event for e in events])
    _check(lib().dsa_prefill_chunk_profiled(
        _dev(q_idx, "q_idx"), *_rows(k_idx, "k_idx"), _dev(w, "w", (torch.float32,)), dt,
        _dev(q, "q", (torch.bfloat16,)), *_rows(kv, "kv", (torch.bfloat16,)), L, N, H_I, D_I, H, q_pos0, topk,
        float(scale), query_block, _dev(topk_idx, "topk_idx", (torch.int32,)), _dev(out, "out", (torch.bfloat16,)),
        _dev(lse, "lse", (torch.float32,)), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream), handles, len(events)),
        "dsa_prefill_chunk_profiled")


def dsa_selftest_wait_timeout(workspace: torch.Tensor, limit_ms: int = 50, stream=None) -> None:
    """Run the bounded-wait self-test into `workspace` (see include/dsa.h); read it with dsa_workspace_status."""
    _check(lib().dsa_selftest_wait_timeout(_dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                           int(limit_ms), _stream(stream)), "dsa_selftest_wait_timeout")


def dsa_indexer_topk_noalloc_status(stream=None) -> int:
    """Synchronise the stream and return the status word of dsa_indexer_topk_noalloc's fixed scratch on the
    current device (0 = clean; it describes the most recent call)."""
    flags = ctypes.c_uint(0)
    st = lib().dsa_indexer_topk_noalloc_status(_stream(stream), ctypes.byref(flags))
    if st not in (DSA_OK, 5):
        raise DSAError(st, "dsa_indexer_topk_noalloc_status")
    return flags.value


def dsa_workspace_selection_stats(workspace: torch.Tensor, stream=None) -> dict:
    """Synchronise the stream and return the selection totals of the most recent call on `workspace`:
    candidates (all queries), queries, fallback_queries, max_candidates."""
    s = SelectionStats()
    _check(lib().dsa_workspace_selection_stats(_dev(workspace, "workspace"), _stream(stream), ctypes.byref(s)),
           "dsa_workspace_selection_stats")
    return {"candidates": s.candidates, "queries": s.queries, "fallback_queries": s.fallback_queries,
            "max_candidates": s.max_candidates}


def dsa_workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and return the device status word of a workspace (0 = clean)."""
    flags = ctypes.c_uint(0)
    st = lib().dsa_workspace_status(_dev(workspace, "workspace"), _stream(stream), ctypes.byref(flags))
    if st not in (DSA_OK, 5):
        raise DSAError(st, "dsa_workspace_status")
    return flags.value
