"""General visibility (per-query key ranges) against the oracle: dsa_indexer_topk_ranges and
dsa_prefill_chunk_ranges (llama.cpp PR #25917, discussion: causality carried by the index mask)."""
import numpy as np
import pytest
import torch

import dsa_inputs
import oracle
import deepseek_sparse_attention_relu_b200 as dsa
from tests._helpers import oracle_problem, topk_set_check

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_ABS = 3e-2


def run_ranges(cfg, inp, lo, hi, ws_bytes=None, with_scores=False):
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in inp.items()}
    idx = torch.full((cfg.L, cfg.topk), -7, dtype=torch.int32, device=dev)
    sc = torch.full((cfg.L, cfg.topk), float("nan"), dtype=torch.float32, device=dev) if with_scores else None
    full = dsa.dsa_indexer_topk_workspace(cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.topk, dsa._dtype_code(g["q_idx"]))
    ws = dsa.alloc_workspace(ws_bytes or full, dev)
    dsa.dsa_indexer_topk_ranges(g["q_idx"], g["k_idx"], g["w"], torch.tensor(lo, dtype=torch.int32, device=dev),
                                torch.tensor(hi, dtype=torch.int32, device=dev), cfg.topk, idx, sc, workspace=ws)
    if with_scores:
        return idx.cpu().numpy(), ws, sc.cpu().numpy()
    return idx.cpu().numpy(), ws


def check_range_row(pb, gpu_row, t, lo, hi, exact):
    ref, kth, s = oracle.topk_row_range(pb, t, lo, hi)
    if exact:
        assert np.array_equal(gpu_row, ref), f"query {t} [{lo},{hi}): selection differs"
        return 0
    rel = lambda r: np.where(r >= 0, r - lo, -1)
    return topk_set_check(rel(gpu_row), rel(ref), s, kth)


def test_ranges_equal_causal_path():
    """The causal prefix given as ranges selects exactly what the causal entry point selects."""
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=20000, L=300, topk=512)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in inp.items()}
    causal = torch.full((cfg.L, cfg.topk), -7, dtype=torch.int32, device=dev)
    dsa.dsa_indexer_topk(g["q_idx"], g["k_idx"], g["w"], cfg.q_pos0, cfg.topk, causal)
    lo = [0] * cfg.L
    hi = [cfg.q_pos0 + t + 1 for t in range(cfg.L)]
    ranged, ws = run_ranges(cfg, inp, lo, hi)
    assert dsa.dsa_workspace_status(ws) == 0
    assert np.array_equal(ranged, causal.cpu().numpy())


def test_packed_sequences_batched_prefill():
    """Three sequences stored back to back in one cache; each query sees its own sequence up to itself."""
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=20000, L=300, topk=512, H=64)
    inp = dsa_inputs.generate(cfg)
    starts, lens = [0, 6000, 15000], [6000, 9000, 5000]
    lo, hi = [], []
    for b, n in zip(starts, lens):
        for j in range(100):  # the last 100 positions of each sequence
            lo.append(b)
            hi.append(b + n - 100 + j + 1)
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in inp.items()}
    idx = torch.full((cfg.L, cfg.topk), -7, dtype=torch.int32, device=dev)
    out = torch.full((cfg.L, cfg.H, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.empty(cfg.L, cfg.H, dtype=torch.float32, device=dev)
    ws = dsa.alloc_workspace(dsa.dsa_prefill_chunk_workspace(cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.H, cfg.topk, 0,
                                                             dsa.DSA_BF16, 1), dev)
    dsa.dsa_prefill_chunk_ranges(g["q_idx"], g["k_idx"], g["w"], g["q"], g["kv"],
                                 torch.tensor(lo, dtype=torch.int32, device=dev),
                                 torch.tensor(hi, dtype=torch.int32, device=dev), cfg.topk, cfg.scale, out,
                                 topk_idx=idx, lse=lse, workspace=ws)
    assert dsa.dsa_workspace_status(ws) == 0
    idx = idx.cpu().numpy()
    pb = oracle_problem(cfg, inp)
    rows = [0, 57, 99, 100, 150, 199, 200, 250, 299]
    out_rows = out[torch.tensor(rows, device=dev)].float().cpu().numpy()
    for i, t in enumerate(rows):
        check_range_row(pb, idx[t], t, lo[t], hi[t], exact=False)
        ro, _ = oracle.sparse_mla(pb, t, idx[t])
        err = np.linalg.norm(out_rows[i] - ro) / np.linalg.norm(ro)
        assert err <= REL_L2 and np.max(np.abs(out_rows[i] - ro)) <= MAX_ABS
    for t in range(cfg.L):  # every selection stays inside its own sequence
        sel = idx[t][idx[t] >= 0]
        assert len(sel) == min(cfg.topk, hi[t] - lo[t]) and sel.min() >= lo[t] and sel.max() < hi[t]


def test_ranges_edges_exact():
    """Integer inputs (exact scores): empty ranges, ranges shorter than k, the last key alone, windows."""
    cfg = dsa_inputs.small_variant(dsa_inputs.TIES, N=16384, L=40, topk=256)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    rng = np.random.default_rng(8)
    lo, hi = [], []
    for t in range(cfg.L):
        kind = t % 5
        if kind == 0:
            a = b = int(rng.integers(0, cfg.N))                 # empty
        elif kind == 1:
            a = int(rng.integers(0, cfg.N - 200)); b = a + int(rng.integers(1, 200))  # shorter than k
        elif kind == 2:
            a, b = cfg.N - 1, cfg.N                              # the last key alone
        elif kind == 3:
            a = int(rng.integers(0, 4000)); b = a + 12000        # long window (pilot + threshold)
        else:
            a = 0; b = int(rng.integers(9000, cfg.N + 1))        # prefix
        lo.append(a); hi.append(b)
    idx, ws = run_ranges(cfg, inp, lo, hi)
    assert dsa.dsa_workspace_status(ws) == 0
    pb = oracle_problem(cfg, inp)
    for t in range(cfg.L):
        check_range_row(pb, idx[t], t, lo[t], hi[t], exact=True)


def test_invalid_range_is_flagged_and_empty():
    cfg = dsa_inputs.small_variant(dsa_inputs.TIES, N=4096, L=8, topk=64)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    lo = [0, 10, 500, 0, 4000, 3, 0, 100]
    hi = [4096, 5, 700, 4097, 4096, 3, 64, 2000]  # query 1: lo > hi; query 3: hi > N
    idx, ws = run_ranges(cfg, inp, lo, hi)
    flags = dsa.dsa_workspace_status(ws)
    assert flags & 2  # bad range flagged
    assert np.all(idx[1] == -1) and np.all(idx[3] == -1)
    pb = oracle_problem(cfg, inp)
    for t in (0, 2, 4, 5, 6, 7):
        check_range_row(pb, idx[t], t, lo[t], hi[t], exact=True)


def test_ranges_forced_fallback_is_bit_identical():
    """Windows of several lengths with a candidate capacity below top-k: every query whose window needs the pilot
    threshold is rescored by the exact fallback, which scores with the main pass's arithmetic, so indices and
    scores equal those of the run without a fallback bit for bit."""
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=30000, L=200, topk=512)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    lo = [max(0, cfg.q_pos0 + t + 1 - (9000 + 97 * t)) for t in range(cfg.L)]
    hi = [cfg.q_pos0 + t + 1 for t in range(cfg.L)]
    idx_a, ws_a, sc_a = run_ranges(cfg, inp, lo, hi, with_scores=True)
    assert dsa.dsa_workspace_status(ws_a) == 0
    assert dsa.dsa_workspace_selection_stats(ws_a)["fallback_queries"] == 0
    full = dsa.dsa_indexer_topk_workspace(cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.topk)
    small = full - cfg.L * (8192 - 256) * 8  # candidate capacity 256 < top-k
    idx_b, ws_b, sc_b = run_ranges(cfg, inp, lo, hi, ws_bytes=small, with_scores=True)
    assert dsa.dsa_workspace_status(ws_b) == 0
    assert dsa.dsa_workspace_selection_stats(ws_b)["fallback_queries"] == cfg.L
    assert np.array_equal(idx_a, idx_b) and np.array_equal(sc_a, sc_b)
    pb = oracle_problem(cfg, inp)
    for t in (0, 99, 199):
        check_range_row(pb, idx_b[t], t, lo[t], hi[t], exact=False)
