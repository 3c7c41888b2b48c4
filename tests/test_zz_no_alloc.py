"""dsa_indexer_topk_noalloc: the workspace-free indexer top-k for callers that cannot allocate device memory.

Such callers (a runtime that plans every byte up front and hands kernels only
their inputs and outputs, or a device fully reserved by others) get their
scratch from a fixed device array inside the library instead of a
caller-provided workspace.  The selection does not depend on the query blocking
or on which queries go through the exact fallback, so the entry point's output
must equal the workspace entry point's bit for bit.  This file is collected
last on purpose; it must pass both alone and after the other tests.
"""
import numpy as np
import pytest
import torch

import dsa_inputs
import deepseek_sparse_attention_relu_b200 as dsa

pytestmark = pytest.mark.gpu


def _selections(cfg):
    inp = dsa_inputs.generate(cfg, with_mla=False)
    dev = torch.device("cuda")
    q_idx, k_idx, w = inp["q_idx"].to(dev), inp["k_idx"].to(dev), inp["w"].to(dev)
    ref_idx = torch.empty(cfg.L, cfg.topk, dtype=torch.int32, device=dev)
    ref_sc = torch.empty(cfg.L, cfg.topk, dtype=torch.float32, device=dev)
    dsa.dsa_indexer_topk(q_idx, k_idx, w, cfg.q_pos0, cfg.topk, ref_idx, ref_sc)
    runs = []
    for _ in range(2):  # two calls in a row: the shared scratch keeps the previous call's contents
        idx = torch.full((cfg.L, cfg.topk), -7, dtype=torch.int32, device=dev)
        sc = torch.full((cfg.L, cfg.topk), float("nan"), dtype=torch.float32, device=dev)
        dsa.dsa_indexer_topk_noalloc(q_idx, k_idx, w, cfg.q_pos0, cfg.topk, idx, sc)
        assert dsa.dsa_indexer_topk_noalloc_status() == 0  # no device-side condition in the fixed scratch
        runs.append((idx.cpu().numpy(), sc.cpu().numpy()))
    return ref_idx.cpu().numpy(), ref_sc.cpu().numpy(), runs


@pytest.mark.parametrize("cfg", [
    dsa_inputs.small_variant(dsa_inputs.CTX128K, N=40000, L=300, topk=2048),
    dsa_inputs.small_variant(dsa_inputs.TIES, N=16384, L=130, topk=2048),
    dsa_inputs.small_variant(dsa_inputs.CTX64K, N=30000, L=200, topk=2048),
    dsa_inputs.CTX128K,
], ids=["bf16-N40000-L300", "ties-N16384-L130", "fp8-N30000-L200", "bf16-N131072-L1024"])
def test_noalloc_matches_workspace_entry_point(cfg):
    ref_idx, ref_sc, runs = _selections(cfg)
    for idx, sc in runs:
        assert np.array_equal(idx, ref_idx)
        assert np.array_equal(sc, ref_sc)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 64 queries: a full 64-query block, whose 16 fallback score rows of N floats alone fill the fixed scratch
    dev = torch.device("cuda")
    N, L = 262144, 64
    q = torch.zeros(L, 32, 128, dtype=torch.bfloat16, device=dev)
    k = torch.zeros(N, 128, dtype=torch.bfloat16, device=dev)
    w = torch.zeros(L, 32, dtype=torch.float32, device=dev)
    idx = torch.empty(L, 2048, dtype=torch.int32, device=dev)
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_indexer_topk_noalloc(q, k, w, N - L, 2048, idx)
    assert e.value.status == 3  # DSA_ERR_WORKSPACE
