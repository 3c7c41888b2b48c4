"""End-to-end parity of dsa_prefill_chunk (indexer -> exact top-k -> sparse MLA) with the CPU oracle.

Small cases are checked on every query.  The five workloads run at full size in
the launch configuration the benchmark times; the tiny, tie, 64K and 128K
workloads are checked on every query and the 256K workload on 64 seeded queries
of each of its eight 1,024-query blocks (first and last included).  The
attention output is scored on the GPU's own selection (a swap of near-equal
keys may carry a very different attention weight), and the selection itself
against the oracle's; the attention error against the oracle's own selection
(the end-to-end result) and the number of swapped keys are reported.
"""
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


def run_chunk(cfg, inp, query_block=0, ws_bytes=None):
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in inp.items()}
    out = torch.full((cfg.L, cfg.H, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.empty(cfg.L, cfg.H, dtype=torch.float32, device=dev)
    idx = torch.full((cfg.L, cfg.topk), -7, dtype=torch.int32, device=dev)
    dt = dsa.DSA_BF16 if cfg.idx_dtype == "bf16" else dsa.DSA_FP8_E4M3
    full = dsa.dsa_prefill_chunk_workspace(cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.H, cfg.topk, query_block, dt)
    ws = dsa.alloc_workspace(full if ws_bytes is None else ws_bytes, dev)
    dsa.dsa_prefill_chunk(g["q_idx"], g["k_idx"], g["w"], g["q"], g["kv"], cfg.q_pos0, cfg.topk, cfg.scale, out,
                          topk_idx=idx, lse=lse, query_block=query_block, workspace=ws)
    assert dsa.dsa_workspace_status(ws) == 0
    stats = dsa.dsa_workspace_selection_stats(ws)
    assert stats["queries"] == cfg.L
    return idx.cpu().numpy(), out, lse, stats


def check_chunk(cfg, inp, idx, out, rows, exact=False):
    """Selection against the oracle's (bit-exact or within the swap band) and attention on the GPU's selection
    within the stated bounds, for the given rows.  Returns (swapped keys, worst rel-L2 against the oracle's own
    selection)."""
    pb = oracle_problem(cfg, inp)
    rows = list(rows)
    out_rows = out[torch.tensor(rows, device=out.device)].float().cpu().numpy()

    def one(i_t):
        i, t = i_t
        ref, kth, s = oracle.topk_row(pb, t)
        ro, _ = oracle.sparse_mla(pb, t, idx[t])
        own = ro if np.array_equal(idx[t], ref) else oracle.sparse_mla(pb, t, ref)[0]
        return i, t, ref, kth, s, ro, own

    swaps, worst_own = 0, 0.0
    for i, t, ref, kth, s, ro, own in oracle.map_rows(one, list(enumerate(rows))):
        if exact:
            assert np.array_equal(idx[t], ref), f"query {t}: selection differs"
        else:
            swaps += topk_set_check(idx[t], ref, s, kth)
        o = out_rows[i]
        err = np.linalg.norm(o - ro) / np.linalg.norm(ro)
        assert err <= REL_L2, f"query {t}: rel-L2 {err}"
        assert np.max(np.abs(o - ro)) <= MAX_ABS
        worst_own = max(worst_own, float(np.linalg.norm(o - own) / np.linalg.norm(own)))
    return swaps, worst_own


def test_small_chunk_every_query():
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=9000, L=130, topk=512, H=64)
    inp = dsa_inputs.generate(cfg)
    idx, out, _, _ = run_chunk(cfg, inp)
    check_chunk(cfg, inp, idx, out, range(cfg.L))


def _fixed_bytes(cfg, query_block):
    """Workspace of dsa_prefill_chunk minus its candidate lists (the part a smaller workspace must still hold);
    the lists take QB x max(8192, 4 topk) x 8 bytes (include/dsa.h: a smaller workspace shrinks the per-query
    candidate capacity)."""
    dt = dsa.DSA_BF16 if cfg.idx_dtype == "bf16" else dsa.DSA_FP8_E4M3
    qb = min(cfg.L, (query_block + 7) // 8 * 8 if query_block > 0 else 1024)
    full = dsa.dsa_prefill_chunk_workspace(cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.H, cfg.topk, query_block, dt)
    return full - qb * max(8192, 4 * cfg.topk) * 8, qb


@pytest.mark.parametrize("base", [dsa_inputs.CTX64K, dsa_inputs.CTX128K], ids=["fp8", "bf16"])
def test_query_block_invariance(base):
    """Selections and outputs do not depend on the query blocking (mlx-lm PR #1997, "Evidence": query blocks
    match), bit for bit, including when some queries go through the exact fallback in one blocking only."""
    cfg = dsa_inputs.small_variant(base, N=20000, L=300, topk=1024, H=64)
    inp = dsa_inputs.generate(cfg)
    idx_a, out_a, lse_a, st_a = run_chunk(cfg, inp, query_block=0)
    assert st_a["fallback_queries"] == 0
    for qb in (64, 7):
        idx_b, out_b, lse_b, _ = run_chunk(cfg, inp, query_block=qb)
        assert np.array_equal(idx_a, idx_b), f"query_block={qb}: selection differs"
        assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b), f"query_block={qb}: output differs"
    # A candidate capacity near the typical candidate count: about half the queries overflow their list and
    # are rescored by the fallback in the 64-query blocking only.
    fixed, qb = _fixed_bytes(cfg, 64)
    mean_cands = st_a["candidates"] / st_a["queries"]
    cap = int(mean_cands)
    assert cap >= cfg.topk
    idx_c, out_c, lse_c, st_c = run_chunk(cfg, inp, query_block=64, ws_bytes=fixed + qb * cap * 8)
    assert 0 < st_c["fallback_queries"] < cfg.L
    assert np.array_equal(idx_a, idx_c)
    assert torch.equal(out_a, out_c) and torch.equal(lse_a, lse_c)
    # Capacity below top-k: every query that needs the pilot threshold goes through the fallback.
    idx_d, out_d, lse_d, st_d = run_chunk(cfg, inp, query_block=0, ws_bytes=_fixed_bytes(cfg, 0)[0] + 300 * 512 * 8)
    assert st_d["fallback_queries"] == cfg.L
    assert np.array_equal(idx_a, idx_d)
    assert torch.equal(out_a, out_d) and torch.equal(lse_a, lse_d)
    check_chunk(cfg, inp, idx_c, out_c, [0, 63, 64, 65, 200, 299])


def _sampled_rows(cfg, per_block=64, block=1024):
    g = np.random.default_rng(4321)
    rows = []
    for b0 in range(0, cfg.L, block):
        n = min(block, cfg.L - b0)
        pick = set(g.choice(n, size=min(per_block, n) - 2, replace=False).tolist()) | {0, n - 1}
        rows += sorted(b0 + r for r in pick)
    return rows


# The five workloads at full size: every query, except 64 per 1,024-query block at 256K.
FULL = [dsa_inputs.TINY, dsa_inputs.TIES, dsa_inputs.CTX64K, dsa_inputs.CTX128K, dsa_inputs.CTX256K]


@pytest.mark.parametrize("cfg", FULL, ids=[c.name for c in FULL])
def test_full_size_workloads(cfg):
    inp = dsa_inputs.generate(cfg)
    idx, out, lse, stats = run_chunk(cfg, inp)
    assert np.isfinite(lse.cpu().numpy()).all()
    rows = _sampled_rows(cfg) if cfg.L > 4096 else range(cfg.L)
    swaps, worst_own = check_chunk(cfg, inp, idx, out, rows, exact=cfg.idx_dist == "int3")
    print(f"\n[parity] {cfg.name}: {len(rows)} queries checked, {swaps} swapped key pairs (1e-6 band), "
          f"worst rel-L2 against the oracle's own selection {worst_own:.2e}, "
          f"candidates/query {stats['candidates'] / stats['queries']:.0f}, fallback queries "
          f"{stats['fallback_queries']}")
    # every query: a well-formed selection (ascending, in range, no padding since all see > topk keys)
    assert np.all(np.diff(idx, axis=1) > 0)
    assert idx.min() >= 0 and np.all(idx.max(axis=1) <= cfg.q_pos0 + np.arange(cfg.L))


def test_small_head_chunk_uses_packing_path():
    """H = 8 MLA heads over 2,400 queries: the attention stage packs queries per CTA."""
    cfg = dsa_inputs.small_variant(dsa_inputs.TINY, N=8192, L=2400, topk=256, H=8)
    inp = dsa_inputs.generate(cfg)
    idx, out, _, _ = run_chunk(cfg, inp)
    check_chunk(cfg, inp, idx, out, list(range(0, cfg.L, 61)) + [1023, 1024, cfg.L - 1])
    # packs start at block boundaries and never straddle one: any blocking gives the same bits
    idx_b, out_b, _, _ = run_chunk(cfg, inp, query_block=64)
    assert np.array_equal(idx, idx_b) and torch.equal(out, out_b)


def test_decode_chunk_split_key():
    """One query over the 128K cache (decode): the attention stage runs split-key."""
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=131072, L=1, topk=2048, H=64)
    inp = dsa_inputs.generate(cfg)
    idx, out, lse, _ = run_chunk(cfg, inp)
    assert np.isfinite(lse.cpu().numpy()).all()
    check_chunk(cfg, inp, idx, out, [0])


def test_status_word_describes_the_latest_call():
    """Each call clears the workspace's status word when it starts (dsa_workspace_status is the explicit check
    of the most recent call): a timed-out self-test leaves bit 0 set, the next chunk on the same workspace
    clears it."""
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=9000, L=64, topk=512, H=64)
    inp = dsa_inputs.generate(cfg)
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in inp.items()}
    out = torch.empty(cfg.L, cfg.H, 512, dtype=torch.bfloat16, device=dev)
    ws = dsa.alloc_workspace(dsa.dsa_prefill_chunk_workspace(cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.H, cfg.topk,
                                                             0, dsa.DSA_BF16, False), dev)
    dsa.dsa_selftest_wait_timeout(ws, limit_ms=20)
    assert dsa.dsa_workspace_status(ws) & 1
    dsa.dsa_prefill_chunk(g["q_idx"], g["k_idx"], g["w"], g["q"], g["kv"], cfg.q_pos0, cfg.topk, cfg.scale, out,
                          workspace=ws)
    assert dsa.dsa_workspace_status(ws) == 0


def test_correlated_queries_stress():
    """The overlap stress input (neighbouring queries' indexer rows and weights are random walks, so their
    selections share most keys) at 64 heads: every query against the oracle."""
    cfg = dsa_inputs.small_variant(dsa_inputs.CORRELATED, N=20000, L=300, topk=1024, H=64)
    inp = dsa_inputs.generate(cfg)
    idx, out, _, _ = run_chunk(cfg, inp)
    shared = [np.intersect1d(idx[t], idx[t + 1]).size for t in range(cfg.L - 1)]
    assert np.mean(shared) > 0.5 * cfg.topk  # the input does what it is for
    check_chunk(cfg, inp, idx, out, range(cfg.L))
