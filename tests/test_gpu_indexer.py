"""Parity of the CUDA indexer + exact top-k (dsa_indexer_topk) with the CPU oracle."""
import numpy as np
import pytest
import torch

import dsa_inputs
import oracle
import deepseek_sparse_attention_relu_b200 as dsa
from tests._helpers import oracle_problem, topk_set_check

pytestmark = pytest.mark.gpu


def run_indexer(cfg, inp, ws_bytes=None, with_scores=False):
    dev = torch.device("cuda")
    q_idx, k_idx, w = inp["q_idx"].to(dev), inp["k_idx"].to(dev), inp["w"].to(dev)
    idx = torch.full((cfg.L, cfg.topk), -7, dtype=torch.int32, device=dev)
    score = torch.full((cfg.L, cfg.topk), float("nan"), dtype=torch.float32, device=dev) if with_scores else None
    dt = dsa.DSA_BF16 if cfg.idx_dtype == "bf16" else dsa.DSA_FP8_E4M3
    nbytes = ws_bytes or dsa.dsa_indexer_topk_workspace(cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.topk, dt)
    ws = dsa.alloc_workspace(nbytes, dev)
    dsa.dsa_indexer_topk(q_idx, k_idx, w, cfg.q_pos0, cfg.topk, idx, score, workspace=ws)
    flags = dsa.dsa_workspace_status(ws)
    assert flags == 0, f"device status word {flags:#x}"
    return idx.cpu().numpy(), (score.cpu().numpy() if with_scores else None)


def check_rows(cfg, inp, gpu_idx, rows, exact=False, gpu_scores=None):
    pb = oracle_problem(cfg, inp)
    swaps = 0

    def one(t):
        ref, kth, s = oracle.topk_row(pb, t)
        return t, ref, kth, s

    for t, ref, kth, s in oracle.map_rows(one, rows):
        if exact:
            assert np.array_equal(gpu_idx[t], ref), f"query {t}: selection differs from the oracle"
        else:
            swaps += topk_set_check(gpu_idx[t], ref, s, kth)
        if gpu_scores is not None:
            sel = gpu_idx[t] >= 0
            np.testing.assert_allclose(gpu_scores[t][sel], s[gpu_idx[t][sel]], rtol=2e-6, atol=1e-4 * max(1.0, abs(kth)))
            assert np.all(np.isneginf(gpu_scores[t][~sel]))
    return swaps


def test_tiny_all_rows():
    cfg = dsa_inputs.TINY
    inp = dsa_inputs.generate(cfg, with_mla=False)
    idx, sc = run_indexer(cfg, inp, with_scores=True)
    check_rows(cfg, inp, idx, range(cfg.L), gpu_scores=sc)


def test_exact_ties_bit_exact_full_size():
    """Integer inputs: every fp32 sum is exact, so the selection must equal the oracle's bit for bit."""
    cfg = dsa_inputs.TIES
    inp = dsa_inputs.generate(cfg, with_mla=False)
    idx, _ = run_indexer(cfg, inp)
    check_rows(cfg, inp, idx, range(cfg.L), exact=True)


def test_bf16_pilot_path_ragged():
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=40000, L=203, topk=2048)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    idx, sc = run_indexer(cfg, inp, with_scores=True)
    check_rows(cfg, inp, idx, list(range(0, cfg.L, 13)) + [cfg.L - 1], gpu_scores=sc)


def test_fp8_concentrated_pilot_path():
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX64K, N=30000, L=300, topk=2048)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    idx, _ = run_indexer(cfg, inp)
    check_rows(cfg, inp, idx, list(range(0, cfg.L, 17)) + [cfg.L - 1])


def test_forced_fallback_is_exact():
    """A workspace with room for only 64 candidates per query: every query goes to the exact fallback."""
    cfg = dsa_inputs.small_variant(dsa_inputs.TIES, N=6000, L=40, topk=256)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    full = dsa.dsa_indexer_topk_workspace(cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.topk)
    small = full - cfg.L * (8192 - 64) * 8
    idx, _ = run_indexer(cfg, inp, ws_bytes=small)
    check_rows(cfg, inp, idx, range(cfg.L), exact=True)


def test_prefill_from_empty_cache_pads():
    """q_pos0 = 0: early queries see fewer than top-k keys and get -1 padding."""
    cfg = dsa_inputs.small_variant(dsa_inputs.TINY, N=700, L=700, topk=100)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    assert cfg.q_pos0 == 0
    idx, _ = run_indexer(cfg, inp)
    check_rows(cfg, inp, idx, range(cfg.L))
    assert np.all(idx[0, 1:] == -1) and idx[0, 0] == 0


def test_multiple_query_blocks():
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=12000, L=2100, topk=512)
    inp = dsa_inputs.generate(cfg, with_mla=False)
    idx, _ = run_indexer(cfg, inp)
    check_rows(cfg, inp, idx, [0, 1, 511, 1023, 1024, 1025, 2047, 2048, 2099])


def test_topk_one_and_topk_equals_visible():
    for topk in (1, 4096):
        cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=4096, L=16, topk=topk)
        inp = dsa_inputs.generate(cfg, with_mla=False)
        idx, _ = run_indexer(cfg, inp)
        check_rows(cfg, inp, idx, range(cfg.L))


# Every indexer shape the header declares supported, on the pilot path with a ragged query count:
# (D_I, H_I, fp8).  The five workloads only reach (128, 32, *) and (64, 4, bf16).
OTHER_SHAPES = [(128, 16, False), (128, 16, True), (128, 8, False), (128, 8, True), (64, 32, False)]


@pytest.mark.parametrize("D_I,H_I,fp8", OTHER_SHAPES, ids=[f"D{d}-H{h}-{'fp8' if f else 'bf16'}"
                                                          for d, h, f in OTHER_SHAPES])
def test_supported_indexer_shapes(D_I, H_I, fp8):
    from dataclasses import replace
    base = dsa_inputs.CTX64K if fp8 else dsa_inputs.CTX128K
    cfg = replace(dsa_inputs.small_variant(base, N=20000, L=141, topk=512), H_I=H_I, D_I=D_I,
                  name=f"shape-D{D_I}-H{H_I}-{'fp8' if fp8 else 'bf16'}")
    inp = dsa_inputs.generate(cfg, with_mla=False)
    assert tuple(inp["q_idx"].shape) == (cfg.L, H_I, D_I)
    idx, sc = run_indexer(cfg, inp, with_scores=True)
    check_rows(cfg, inp, idx, list(range(0, cfg.L, 7)) + [cfg.L - 1], gpu_scores=sc)
    # the exact fallback (candidate capacity 64 < top-k: every query) scores with the same arithmetic
    full = dsa.dsa_indexer_topk_workspace(cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.topk)
    idx_f, sc_f = run_indexer(cfg, inp, ws_bytes=full - cfg.L * (8192 - 64) * 8, with_scores=True)
    assert np.array_equal(idx, idx_f) and np.array_equal(sc, sc_f)
