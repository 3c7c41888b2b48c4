"""The seeded input generator draws what the workload recipe states (CPU only).

The five workloads (and the decode case) are checked for their sizes, dtypes,
seeds and positions, and small variants of each are checked for the stated
distributions: N(0,1) indexer operands, exact integers in [-3, 3] with weights
in {1, 2}, the shared mean direction of norm 2 of the concentrated fp8
workloads, the weight scales and the MLA latent / rope standard deviations.
"""
import math

import pytest
import torch

import dsa_inputs as di


def test_workload_table():
    got = {c.name: (c.N, c.L, c.H_I, c.D_I, c.idx_dtype, c.idx_dist, c.w_dist, c.topk, c.H, c.seed)
           for c in di.WORKLOADS}
    assert got == {
        "dsa-tiny-N4096-L256": (4096, 256, 4, 64, "bf16", "normal", "normal_half", 256, 8, 0),
        "dsa-ties-N16384-L512": (16384, 512, 32, 128, "bf16", "int3", "int12", 2048, 64, 1),
        "dsa-64k-fp8-N65536-L2048": (65536, 2048, 32, 128, "e4m3", "concentrated", "normal_rsqrt", 2048, 64, 2),
        "dsa-128k-N131072-L1024": (131072, 1024, 32, 128, "bf16", "normal", "normal_rsqrt", 2048, 64, 3),
        "dsa-256k-fp8-N262144-L8192": (262144, 8192, 32, 128, "e4m3", "concentrated", "normal_rsqrt", 2048, 128, 4),
    }
    for c in di.WORKLOADS + [di.DECODE128K]:
        assert c.q_pos0 == c.N - c.L
        assert c.scale == pytest.approx(1.0 / math.sqrt(192.0))
    assert di.DECODE128K.L == 1 and di.DECODE128K.seed == di.CTX128K.seed


@pytest.mark.parametrize("N,L", [(10, 1), (300, 7), (4096, 256)])
def test_visible_pairs_closed_form(N, L):
    c = di.small_variant(di.TINY, N=N, L=L)
    assert c.visible_pairs() == sum(c.q_pos0 + t + 1 for t in range(L))


def _std(x):
    return x.float().std().item()


def test_exact_integer_workload():
    inp = di.generate(di.small_variant(di.TIES, N=2048, L=64, H=8), with_mla=False)
    for name in ("q_idx", "k_idx"):
        v = inp[name].float()
        assert torch.equal(v, v.round()) and v.min() == -3 and v.max() == 3
        assert set(v.unique().tolist()) == set(range(-3, 4))
    assert set(inp["w"].unique().tolist()) == {1.0, 2.0}


@pytest.mark.parametrize("base", [di.CTX64K, di.CTX256K], ids=["64k", "256k"])
def test_concentrated_fp8_operands(base):
    cfg = di.small_variant(base, N=16384, L=64, H=8)
    inp = di.generate(cfg, with_mla=False)
    assert inp["k_idx"].dtype == torch.float8_e4m3fn and inp["q_idx"].dtype == torch.float8_e4m3fn
    k = inp["k_idx"].float()
    q = inp["q_idx"].float().reshape(-1, cfg.D_I)
    mk, mq = k.mean(0), q.mean(0)
    assert mk.norm().item() == pytest.approx(2.0, abs=0.05)          # shared mean direction of norm 2
    assert torch.nn.functional.cosine_similarity(mk, mq, dim=0).item() > 0.98  # the same direction for queries
    assert _std(k - mk) == pytest.approx(1.0, rel=0.03)
    assert k.abs().max().item() <= 448.0
    assert _std(inp["w"]) == pytest.approx(1.0 / math.sqrt(cfg.H_I), rel=0.1)


def test_normal_bf16_operands_and_mla_scales():
    cfg = di.small_variant(di.CTX128K, N=16384, L=64, H=8)
    inp = di.generate(cfg)
    assert inp["k_idx"].dtype == torch.bfloat16
    assert abs(inp["k_idx"].float().mean().item()) < 0.01
    assert _std(inp["k_idx"]) == pytest.approx(1.0, rel=0.02)
    assert _std(inp["q_idx"]) == pytest.approx(1.0, rel=0.03)
    assert _std(inp["w"]) == pytest.approx(1.0 / math.sqrt(32), rel=0.1)
    kv, q = inp["kv"].float(), inp["q"].float()
    assert kv.shape == (cfg.N, 576) and q.shape == (cfg.L, cfg.H, 576)
    assert _std(kv[:, :512]) == pytest.approx(0.5, rel=0.02) and _std(kv[:, 512:]) == pytest.approx(0.5, rel=0.03)
    assert _std(q[..., :512]) == pytest.approx(0.5, rel=0.03)


def test_tiny_workload_scales():
    inp = di.generate(di.TINY)
    assert _std(inp["w"]) == pytest.approx(0.5, rel=0.1)
    assert _std(inp["kv"][:, :512]) == pytest.approx(0.5, rel=0.03)
    assert _std(inp["kv"][:, 512:]) == pytest.approx(1.0, rel=0.05)


def test_correlated_stress_input_is_a_random_walk_over_queries():
    """The overlap stress input: neighbouring queries' indexer rows and weights differ by 0.05 N(0, 1) steps."""
    cfg = di.small_variant(di.CORRELATED, N=4096, L=200, H=8)
    assert cfg.name.startswith("dsa-correlated") and di.CORRELATED not in di.WORKLOADS
    inp = di.generate(cfg, with_mla=False)
    q = inp["q_idx"].float()
    step = q[1:] - q[:-1]
    assert _std(step) == pytest.approx(di.WALK_STEP, rel=0.1)   # bf16 rounding adds a little
    assert _std(q[0]) == pytest.approx(1.0, rel=0.15)
    assert _std(inp["k_idx"]) == pytest.approx(1.0, rel=0.02)
    w = inp["w"]
    assert _std(w[1:] - w[:-1]) == pytest.approx(di.WALK_STEP / math.sqrt(cfg.H_I), rel=0.1)
