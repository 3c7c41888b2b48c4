"""Shared test plumbing: turn generated inputs into oracle problems and compare results."""
from __future__ import annotations

import numpy as np
import torch

import dsa_inputs
import oracle


def oracle_problem(cfg: dsa_inputs.ChunkConfig, inp: dict) -> oracle.Problem:
    return oracle.Problem(
        q_idx=dsa_inputs.raw_bits(inp["q_idx"]), k_idx=dsa_inputs.raw_bits(inp["k_idx"]), w=inp["w"],
        idx_dtype=cfg.idx_code, L=cfg.L, N=cfg.N, H_I=cfg.H_I, D_I=cfg.D_I, q_pos0=cfg.q_pos0, topk=cfg.topk,
        q=dsa_inputs.raw_bits(inp["q"]) if "q" in inp else None,
        kv=dsa_inputs.raw_bits(inp["kv"]) if "kv" in inp else None, H=cfg.H, scale=cfg.scale)


def topk_set_check(gpu_idx: np.ndarray, ora_idx: np.ndarray, scores: np.ndarray, kth: float, rel: float = 1e-6):
    """Compare one query's selection with the oracle's.

    Both are ascending key lists with -1 padding.  Passes when the sets are
    equal, or when every key in the symmetric difference has an oracle score
    within rel*|kth| of the oracle's k-th score (a swap of near-equal keys).
    Returns the number of swapped keys.  Raises AssertionError otherwise.
    """
    g = gpu_idx[gpu_idx >= 0]
    o = ora_idx[ora_idx >= 0]
    assert np.all(np.diff(g) > 0), "selection not strictly ascending"
    assert np.all(gpu_idx[len(g):] == -1), "padding not at the end"
    assert len(g) == len(o), f"selected {len(g)} keys, oracle {len(o)}"
    if len(g) and (g.min() < 0 or g.max() >= len(scores)):
        raise AssertionError("selected a key outside the visible range")
    diff = np.setxor1d(g, o)
    if len(diff) == 0:
        return 0
    bad = diff[np.abs(scores[diff] - kth) > rel * abs(kth)]
    assert len(bad) == 0, (f"{len(diff)} keys differ; {len(bad)} beyond the swap band, e.g. key {bad[0]} "
                           f"score {scores[bad[0]]!r} vs kth {kth!r}")
    return len(diff) // 2


def to_bf16_bits(values, shape) -> torch.Tensor:
    return torch.tensor(values, dtype=torch.float32).reshape(shape).to(torch.bfloat16).contiguous()
