"""Failure detection without a GPU fault: a wait that never completes runs out after its limit, the kernel
records a timeout in the status word, and the CUDA context stays usable for the real path."""
import time

import numpy as np
import pytest
import torch

import dsa_inputs
import deepseek_sparse_attention_relu_b200 as dsa

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    dev = torch.device("cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    dsa.dsa_selftest_wait_timeout(ws, limit_ms=50)
    flags = dsa.dsa_workspace_status(ws)
    elapsed = time.perf_counter() - t0
    assert flags & 1, f"status word {flags:#x}: the timeout bit is not set"
    assert 0.04 < elapsed < 1.5  # the wait gave up at its limit, not at the kernels' 2 s default
    # the same context then runs the whole path cleanly
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=4096, L=64, topk=256, H=64)
    g = {k: v.to(dev) for k, v in dsa_inputs.generate(cfg).items()}
    out = torch.empty(cfg.L, cfg.H, 512, dtype=torch.bfloat16, device=dev)
    ws2 = dsa.alloc_workspace(dsa.dsa_prefill_chunk_workspace(cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.H, cfg.topk, 0,
                                                              dsa.DSA_BF16, False), dev)
    dsa.dsa_prefill_chunk(g["q_idx"], g["k_idx"], g["w"], g["q"], g["kv"], cfg.q_pos0, cfg.topk, cfg.scale, out,
                          workspace=ws2)
    assert dsa.dsa_workspace_status(ws2) == 0
    assert np.isfinite(out.float().cpu().numpy()).all()


def test_selftest_rejects_bad_arguments():
    dev = torch.device("cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device=dev)
    with pytest.raises(dsa.DSAError):
        dsa.dsa_selftest_wait_timeout(ws, limit_ms=0)
    with pytest.raises(dsa.DSAError):
        dsa.dsa_selftest_wait_timeout(ws[:100], limit_ms=10)
