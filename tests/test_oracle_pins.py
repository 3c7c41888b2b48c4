"""Pins of the CPU oracle to things other than itself (CPU only).

Each test ties one oracle function to a hand-derived closed form (fixtures
under tests/golden/), a library routine that the special case reduces to, an
exact invariant, or brute force on tiny inputs.  A dropped term, a wrong sign,
a transposed operand, an off-by-one in causality or a reversed tie-break each
fail at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import dsa_inputs
import oracle
from tests._helpers import oracle_problem, to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- decoding

def test_bf16_decode_all_codes(oracle_lib):
    codes = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(codes.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    L = oracle_lib.lib()
    got = np.array([L.oracle_bf16_value(int(c)) for c in codes[::7]])
    r = ref[::7]
    finite = np.isfinite(r)
    assert np.array_equal(got[finite], r[finite])
    assert np.all(np.isnan(got[np.isnan(r)]))


def test_e4m3_decode_all_codes(oracle_lib):
    codes = torch.arange(256, dtype=torch.int16).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    L = oracle_lib.lib()
    got = np.array([L.oracle_e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ---------------------------------------------------------------- indexer

def _hand_problem(ex, topk):
    q = to_bf16_bits(ex["q_idx"], (ex["L"], ex["H_I"], ex["D_I"]))
    k = to_bf16_bits(ex["k_idx"], (ex["N"], ex["D_I"]))
    w = torch.tensor(ex["w"], dtype=torch.float32)
    return oracle.Problem(q.view(torch.uint16), k.view(torch.uint16), w, oracle.IDX_BF16, ex["L"], ex["N"],
                          ex["H_I"], ex["D_I"], ex["q_pos0"], topk)


def test_indexer_hand_example(oracle_lib):
    ex = _load("indexer_hand_example.json")
    for k, want in ex["topk"].items():
        pb = _hand_problem(ex, int(k))
        s = oracle.indexer_scores(pb, 0)
        assert s.tolist() == ex["scores"]
        idx, kth = oracle.topk_fullsort(s, int(k))
        assert idx.tolist() == want["idx"]
        if want["kth"] is None:
            assert kth == -math.inf
        else:
            assert kth == want["kth"]
        assert oracle.topk_blocked_fold(s, int(k), block=2).tolist() == want["idx"]


def test_topk_ties_example(oracle_lib):
    ex = _load("topk_ties_example.json")
    k = to_bf16_bits(ex["k"], (ex["N"], 1))
    q = to_bf16_bits([1.0], (1, 1, 1))
    w = torch.ones(1, 1, dtype=torch.float32)
    for kk, want in ex["topk"].items():
        pb = oracle.Problem(q.view(torch.uint16), k.view(torch.uint16), w, oracle.IDX_BF16, 1, ex["N"], 1, 1,
                            ex["q_pos0"], int(kk))
        s = oracle.indexer_scores(pb, 0)
        assert s.tolist() == ex["scores"]
        assert oracle.topk_fullsort(s, int(kk))[0].tolist() == want
        for block in (1, 2, 3, 4096):
            assert oracle.topk_blocked_fold(s, int(kk), block).tolist() == want


def test_single_head_top1_is_argmax(oracle_lib):
    """H_I=1, w=1: I[s] = max(0, q.k_s); top-1 is numpy's argmax (first index on ties)."""
    rng = np.random.default_rng(5)
    for trial in range(6):
        N, D = 300, 64
        k = torch.from_numpy(rng.integers(-2, 3, size=(N, D)).astype(np.float32)).to(torch.bfloat16)
        q = torch.from_numpy(rng.integers(-2, 3, size=(1, 1, D)).astype(np.float32)).to(torch.bfloat16)
        if trial == 0:
            q = -q.abs()
            k = k.abs()  # every dot <= 0: all scores 0, winner is key 0
        w = torch.ones(1, 1)
        q_pos0 = N - 1 - trial
        pb = oracle.Problem(q.view(torch.uint16), k.view(torch.uint16), w, oracle.IDX_BF16, 1, N, 1, D, q_pos0, 1)
        s = oracle.indexer_scores(pb, 0)
        dots = k.to(torch.float64).numpy()[: q_pos0 + 1] @ q.to(torch.float64).numpy()[0, 0]
        assert oracle.topk_fullsort(s, 1)[0][0] == int(np.argmax(np.maximum(dots, 0.0)))


def test_head_permutation_and_weight_scaling(oracle_lib):
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=640, L=4, topk=32)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    pb = oracle_problem(cfg, inp)
    base = [oracle.indexer_scores(pb, t) for t in range(cfg.L)]
    perm = torch.randperm(cfg.H_I, generator=torch.Generator().manual_seed(1))
    inp2 = dict(inp, q_idx=inp["q_idx"][:, perm].contiguous(), w=inp["w"][:, perm].contiguous())
    pb2 = oracle_problem(cfg, inp2)
    inp3 = dict(inp, w=(inp["w"] * 4.0).contiguous())
    pb3 = oracle_problem(cfg, inp3)
    for t in range(cfg.L):
        np.testing.assert_allclose(oracle.indexer_scores(pb2, t), base[t], rtol=1e-12, atol=1e-12)
        assert np.array_equal(oracle.indexer_scores(pb3, t), 4.0 * base[t])  # power of two: exact


def test_relu_gates_negative_dots(oracle_lib):
    """q = -k for every key direction: all dots <= 0 so every score is 0 for any w."""
    D, N = 16, 40
    k = torch.zeros(N, D)
    for s in range(N):
        k[s, s % D] = 1.0 + s % 3
    q = torch.full((1, 3, D), -1.0)
    w = torch.tensor([[1.5, -2.0, 0.25]])
    pb = oracle.Problem(q.to(torch.bfloat16).view(torch.uint16), k.to(torch.bfloat16).view(torch.uint16), w,
                        oracle.IDX_BF16, 1, N, 3, D, N - 1, 4)
    s = oracle.indexer_scores(pb, 0)
    assert np.all(s == 0.0)
    assert oracle.topk_fullsort(s, 4)[0].tolist() == [0, 1, 2, 3]


def test_integer_inputs_scores_exact(oracle_lib):
    """Integer-valued inputs: fp64 sums are exact, so the scores equal an int64 matmul's."""
    cfg = dsa_inputs.small_variant(dsa_inputs.TIES, N=2048, L=8, topk=256)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    pb = oracle_problem(cfg, inp)
    k = inp["k_idx"].to(torch.int64)
    for t in (0, 5, 7):
        q = inp["q_idx"][t].to(torch.int64)
        dots = torch.clamp(k[: cfg.q_pos0 + t + 1] @ q.T, min=0)
        want = (dots * inp["w"][t].to(torch.int64)).sum(1).numpy().astype(np.float64)
        assert np.array_equal(oracle.indexer_scores(pb, t), want)


def test_range_scores_integer_exact(oracle_lib):
    """Per-query key ranges (general causality): on integer inputs the scores of keys [lo, hi) equal an
    int64 matmul over exactly those key rows, whatever the query's position (a shifted or clipped range
    fails)."""
    cfg = dsa_inputs.small_variant(dsa_inputs.TIES, N=2048, L=8, topk=256)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    pb = oracle_problem(cfg, inp)
    k = inp["k_idx"].to(torch.int64)
    for t, lo, hi in [(0, 0, 2048), (3, 100, 101), (5, 1500, 2048), (7, 700, 1300), (2, 40, 40)]:
        q = inp["q_idx"][t].to(torch.int64)
        dots = torch.clamp(k[lo:hi] @ q.T, min=0)
        want = (dots * inp["w"][t].to(torch.int64)).sum(1).numpy().astype(np.float64)
        got = oracle.indexer_scores_range(pb, t, lo, hi)
        assert got.shape == (hi - lo,) and np.array_equal(got, want)
    # the causal row is the range [0, q_pos0 + t + 1)
    assert np.array_equal(oracle.indexer_scores_range(pb, 4, 0, cfg.q_pos0 + 5), oracle.indexer_scores(pb, 4))


def test_range_topk_is_lexsort_of_the_slice(oracle_lib):
    """Top-k over a range = the (score desc, key asc) sort of that slice, reported as absolute keys;
    -1 padding when the range holds fewer than k keys; an empty range selects nothing."""
    cfg = dsa_inputs.small_variant(dsa_inputs.TIES, N=2048, L=4, topk=64)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    pb = oracle_problem(cfg, inp)
    for t, lo, hi in [(0, 300, 1800), (1, 1000, 1040), (2, 7, 7), (3, 0, 2048)]:
        idx, kth, s = oracle.topk_row_range(pb, t, lo, hi)
        want = _lexsort_topk(s, cfg.topk)
        want = np.where(want >= 0, want + lo, -1)
        assert np.array_equal(idx, want)
        assert np.all((idx == -1) | ((idx >= lo) & (idx < hi)))
        if hi - lo <= cfg.topk:
            assert kth == -math.inf and np.count_nonzero(idx >= 0) == hi - lo


# ---------------------------------------------------------------- top-k

def _lexsort_topk(scores, k):
    order = np.lexsort((np.arange(len(scores)), -scores))  # by score desc, then index asc
    sel = np.sort(order[:k]).astype(np.int32)
    return np.concatenate([sel, -np.ones(max(0, k - len(sel)), dtype=np.int32)])


@pytest.mark.parametrize("seed", range(4))
def test_topk_fullsort_vs_fold_vs_lexsort(oracle_lib, seed):
    rng = np.random.default_rng(seed)
    for n, k in [(1, 1), (5, 8), (100, 7), (5000, 64), (20000, 2048)]:
        scores = rng.integers(-20, 20, size=n).astype(np.float64)  # heavy ties
        if seed % 2:
            scores = rng.normal(size=n)
        full, _ = oracle.topk_fullsort(scores, k)
        assert np.array_equal(full, _lexsort_topk(scores, k))
        for block in (1, 3, 4096):
            if n > 5000 and block < 100:
                continue
            assert np.array_equal(oracle.topk_blocked_fold(scores, k, block), full)


def test_topk_bruteforce_property(oracle_lib):
    """Every selected key beats every unselected visible key under (score desc, index asc)."""
    rng = np.random.default_rng(11)
    for _ in range(50):
        n = int(rng.integers(1, 40))
        k = int(rng.integers(1, 12))
        scores = rng.integers(-3, 4, size=n).astype(np.float64)
        idx, kth = oracle.topk_fullsort(scores, k)
        sel = set(int(i) for i in idx if i >= 0)
        assert len(sel) == min(n, k)
        for a in sel:
            for b in set(range(n)) - sel:
                assert (scores[a] > scores[b]) or (scores[a] == scores[b] and a < b)
        if n > k:
            assert kth == min(scores[list(sel)])


# ---------------------------------------------------------------- attention

def _hand_mla():
    ex = _load("attention_hand_example.json")
    q = torch.zeros(1, 1, 576)
    for c, v in ex["q_sparse"].items():
        q[0, 0, int(c)] = v
    kv = torch.zeros(2, 576)
    for r, row in enumerate(ex["kv_sparse"]):
        for c, v in row.items():
            kv[r, int(c)] = v
    return ex, q.to(torch.bfloat16), kv.to(torch.bfloat16)


def test_attention_hand_example(oracle_lib):
    ex, q, kv = _hand_mla()
    pb = oracle.Problem(None, None, None, 0, 1, 2, 1, 1, 1, 2, q=q.view(torch.uint16), kv=kv.view(torch.uint16),
                        H=1, scale=ex["scale"])
    out, lse = oracle.sparse_mla(pb, 0, [0, 1])
    want = np.zeros(512)
    for c, v in ex["out_nonzero"].items():
        want[int(c)] = v
    np.testing.assert_allclose(out[0], want, rtol=1e-15, atol=1e-15)
    assert abs(lse[0] - ex["lse"]) < 1e-15
    out2, lse2 = oracle.sparse_mla(pb, 0, [1, -1, 0, -1])  # order and padding do not matter here
    np.testing.assert_allclose(out2, out, rtol=1e-15, atol=1e-16)
    out3, lse3 = oracle.sparse_mla(pb, 0, [1])  # a single key: its latent row exactly
    assert np.array_equal(out3[0], kv[1, :512].to(torch.float64).numpy())
    assert lse3[0] == 1.0


def _mla_problem(N, L, H, topk, seed, q_pos0=None):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(L, H, 576, generator=g) * 0.5).to(torch.bfloat16)
    kv = (torch.randn(N, 576, generator=g) * 0.5).to(torch.bfloat16)
    q_pos0 = N - L if q_pos0 is None else q_pos0
    return oracle.Problem(None, None, None, 0, L, N, 1, 1, q_pos0, topk, q=q.view(torch.uint16),
                          kv=kv.view(torch.uint16), H=H, scale=1 / math.sqrt(192)), q, kv


def test_attention_full_selection_equals_dense_and_sdpa(oracle_lib):
    """top-k >= visible keys: sparse == dense causal (same arithmetic) == torch SDPA in fp64."""
    N = L = 64
    pb, q, kv = _mla_problem(N, L, H=4, topk=64, seed=3, q_pos0=0)
    qd = q.to(torch.float64).permute(1, 0, 2)  # [H, L, 576]
    kd = kv.to(torch.float64)
    mask = torch.ones(L, N, dtype=torch.bool).tril()
    ref = torch.nn.functional.scaled_dot_product_attention(
        qd, kd.expand(4, N, 576), kd[:, :512].expand(4, N, 512), attn_mask=mask, scale=pb.scale)
    for t in (0, 1, 17, 63):
        idx = np.concatenate([np.arange(t + 1), -np.ones(64 - t - 1)]).astype(np.int32)
        o_s, l_s = oracle.sparse_mla(pb, t, idx)
        o_d, l_d = oracle.dense_causal_mla(pb, t)
        assert np.array_equal(o_s, o_d) and np.array_equal(l_s, l_d)
        np.testing.assert_allclose(o_s, ref[:, t].numpy(), rtol=1e-11, atol=1e-13)
        # lse against the library logsumexp of the same logits
        z = (qd[:, t] @ kd[: t + 1].T) * pb.scale
        np.testing.assert_allclose(l_s, torch.logsumexp(z, dim=-1).numpy(), rtol=1e-13)


def test_attention_constant_values(oracle_lib):
    """All latent rows equal: softmax weights sum to one so the output is that row."""
    pb, q, kv = _mla_problem(256, 4, H=3, topk=100, seed=8)
    kv2 = kv.clone()
    kv2[:, :512] = kv[7, :512]
    pb.kv = kv2.view(torch.uint16)
    idx = np.sort(np.random.default_rng(0).choice(253, 100, replace=False)).astype(np.int32)
    out, _ = oracle.sparse_mla(pb, 1, idx)
    np.testing.assert_allclose(out, np.broadcast_to(kv2[7, :512].to(torch.float64).numpy(), out.shape),
                               rtol=1e-14, atol=1e-15)


def test_prefill_row_composes_stages(oracle_lib):
    cfg = dsa_inputs.small_variant(dsa_inputs.TINY, N=600, L=8, topk=64)
    inp = dsa_inputs.generate(cfg)
    pb = oracle_problem(cfg, inp)
    for t in (0, 7):
        idx, out, lse = oracle.prefill_row(pb, t)
        idx2, _, _ = oracle.topk_row(pb, t)
        assert np.array_equal(idx, idx2)
        o2, l2 = oracle.sparse_mla(pb, t, idx)
        assert np.array_equal(out, o2) and np.array_equal(lse, l2)


def test_generator_is_deterministic():
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX64K, N=1024, L=16, topk=64)
    a = dsa_inputs.generate(cfg)
    b = dsa_inputs.generate(cfg)
    for k in a:
        assert torch.equal(dsa_inputs.raw_bits(a[k]), dsa_inputs.raw_bits(b[k]))
    assert a["q_idx"].dtype == torch.float8_e4m3fn and a["q"].shape == (16, 64, 576)
