"""Parity of the CUDA sparse absorbed-MLA attention (dsa_sparse_mla_prefill) with the CPU oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import deepseek_sparse_attention_relu_b200 as dsa

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_ABS = 3e-2


def make(N, L, H, seed, lat_std=0.5, rope_std=0.5):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(L, H, 576, generator=g)
    q[..., :512] *= lat_std
    q[..., 512:] *= rope_std
    kv = torch.randn(N, 576, generator=g)
    kv[:, :512] *= lat_std
    kv[:, 512:] *= rope_std
    return q.to(torch.bfloat16).contiguous(), kv.to(torch.bfloat16).contiguous()


def random_selection(N, L, topk, seed, pad=0, q_pos0=None):
    rng = np.random.default_rng(seed)
    q_pos0 = N - L if q_pos0 is None else q_pos0
    idx = np.full((L, topk), -1, dtype=np.int32)
    for t in range(L):
        nvis = q_pos0 + t + 1
        k = min(topk - pad, nvis)
        idx[t, :k] = np.sort(rng.choice(nvis, k, replace=False))
    return idx


def run_mla(q, kv, idx, scale):
    dev = torch.device("cuda")
    L, H, _ = q.shape
    out = torch.full((L, H, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((L, H), float("nan"), dtype=torch.float32, device=dev)
    ws = dsa.alloc_workspace(dsa.dsa_sparse_mla_workspace(L, H, idx.shape[1]), dev)
    dsa.dsa_sparse_mla_prefill(q.to(dev), kv.to(dev), torch.from_numpy(idx).to(dev), scale, out, lse, workspace=ws)
    assert dsa.dsa_workspace_status(ws) == 0
    return out.float().cpu().numpy(), lse.cpu().numpy()


def check(q, kv, idx, scale, rows=None):
    out, lse = run_mla(q, kv, idx, scale)
    L, H, _ = q.shape
    pb = oracle.Problem(None, None, None, 0, L, kv.shape[0], 1, 1, 0, idx.shape[1], q=q.view(torch.uint16),
                        kv=kv.view(torch.uint16), H=H, scale=scale)
    rows = range(L) if rows is None else rows
    res = oracle.map_rows(lambda t: (t, *oracle.sparse_mla(pb, t, idx[t])), rows)
    for t, ro, rl in res:
        err = np.linalg.norm(out[t] - ro) / max(np.linalg.norm(ro), 1e-30)
        assert err <= REL_L2, f"query {t}: rel-L2 {err}"
        assert np.max(np.abs(out[t] - ro)) <= MAX_ABS, f"query {t}: max-abs {np.max(np.abs(out[t] - ro))}"
        np.testing.assert_allclose(lse[t], rl, rtol=1e-4, atol=1e-3)
    return out, lse


@pytest.mark.parametrize("H", [64, 8, 128, 100])
def test_heads(H):
    N, L, topk = 3000, 12, 256
    q, kv = make(N, L, H, seed=H)
    idx = random_selection(N, L, topk, seed=H)
    check(q, kv, idx, 1 / math.sqrt(192))


def test_ragged_topk_and_padding():
    N, L, topk = 5000, 10, 100  # not a multiple of the 64-key tile
    q, kv = make(N, L, 64, seed=3)
    idx = random_selection(N, L, topk, seed=3, pad=37)
    check(q, kv, idx, 1 / math.sqrt(192))


@pytest.mark.parametrize("topk,pad", [(32, 0), (33, 0), (95, 0), (96, 0), (97, 0), (160, 31), (192, 0), (193, 64),
                                      (288, 1), (2047, 0)])
def test_tile_and_group_boundaries(topk, pad):
    """Selections ending at, just before and just after a 32-key release group and a 96-key tile, with and
    without -1 padding: every key lands in the right row group of the right stage."""
    N, L, H = 4096, 4, 64
    q, kv = make(N, L, H, seed=topk)
    idx = random_selection(N, L, topk, seed=topk + 1, pad=pad)
    check(q, kv, idx, 1 / math.sqrt(192))


def test_unsorted_indices_and_large_scale():
    N, L, topk = 4096, 6, 512
    q, kv = make(N, L, 64, seed=5, lat_std=1.0, rope_std=1.0)
    idx = random_selection(N, L, topk, seed=5)
    rng = np.random.default_rng(1)
    for t in range(L):
        rng.shuffle(idx[t])
    check(q, kv, idx, 0.25)  # large logits: exercises the running-max rescale


def test_single_key_is_exact_and_no_key_is_zero():
    N, L, topk = 1000, 3, 64
    q, kv = make(N, L, 64, seed=9)
    idx = np.full((L, topk), -1, dtype=np.int32)
    idx[0, 17] = 123
    idx[1, 0] = 999
    out, lse = run_mla(q, kv, idx, 1 / math.sqrt(192))
    assert np.array_equal(out[0], np.broadcast_to(kv[123, :512].float().numpy(), (64, 512)))
    assert np.array_equal(out[1], np.broadcast_to(kv[999, :512].float().numpy(), (64, 512)))
    assert np.all(out[2] == 0.0) and np.all(np.isneginf(lse[2]))


def test_output_alignment_16_and_32_bytes():
    """Output rows go out as 32-byte stores when the output is 32-byte aligned and as 16-byte stores when it is
    only 16-byte aligned: the bits must not depend on which."""
    N, L, H, topk = 3000, 5, 64, 256
    q, kv = make(N, L, H, seed=13)
    idx = torch.from_numpy(random_selection(N, L, topk, seed=13)).cuda()
    q, kv = q.cuda(), kv.cuda()
    ws = dsa.alloc_workspace(dsa.dsa_sparse_mla_workspace(L, H, topk), torch.device("cuda"))
    ref = torch.empty((L, H, 512), dtype=torch.bfloat16, device="cuda")
    assert ref.data_ptr() % 32 == 0
    dsa.dsa_sparse_mla_prefill(q, kv, idx, 1 / math.sqrt(192), ref, workspace=ws)
    buf = torch.full((L * H * 512 + 8,), float("nan"), dtype=torch.bfloat16, device="cuda")
    shifted = buf[8:].view(L, H, 512)  # 16 bytes past a 32-byte boundary
    assert shifted.data_ptr() % 32 == 16
    dsa.dsa_sparse_mla_prefill(q, kv, idx, 1 / math.sqrt(192), shifted, workspace=ws)
    assert dsa.dsa_workspace_status(ws) == 0
    assert torch.equal(ref, shifted)
    assert torch.isnan(buf[:8]).all()  # nothing written before the output


def test_full_selection_matches_dense_causal():
    """top-k covering every visible key: the sparse path equals dense causal attention (mlx-lm PR #1997 tests)."""
    N = L = 300
    q, kv = make(N, L, 64, seed=11)
    idx = random_selection(N, L, 320, seed=0, q_pos0=0)  # pads every row
    out, _ = run_mla(q, kv, idx, 1 / math.sqrt(192))
    pb = oracle.Problem(None, None, None, 0, L, N, 1, 1, 0, 320, q=q.view(torch.uint16), kv=kv.view(torch.uint16),
                        H=64, scale=1 / math.sqrt(192))
    for t in (0, 1, 150, 299):
        ro, _ = oracle.dense_causal_mla(pb, t)
        assert np.linalg.norm(out[t] - ro) / np.linalg.norm(ro) <= REL_L2


# ---- packed attention: queries with H <= 32 heads share a 64-row tile over the union of their selections
@pytest.mark.parametrize("H,topk,L", [(8, 256, 2400), (16, 512, 1200), (32, 2048, 600)])
def test_packed_small_head_counts(H, topk, L):
    """Enough queries that the library packs 64 / H of them per CTA (capped to keep two waves)."""
    N = 8192
    q, kv = make(N, L, H, seed=H + 100)
    idx = random_selection(N, L, topk, seed=H)
    rows = list(range(0, L, max(1, L // 40))) + [L - 1]
    check(q, kv, idx, 1 / math.sqrt(192), rows=rows)


def test_packed_high_overlap_and_padding():
    """Neighbouring queries share most keys (the case packing is for); some rows padded with -1."""
    N, L, H, topk = 6000, 1600, 16, 256
    q, kv = make(N, L, H, seed=21)
    rng = np.random.default_rng(4)
    base = np.sort(rng.choice(N - L, topk, replace=False))
    idx = np.empty((L, topk), dtype=np.int32)
    for t in range(L):
        row = base.copy()
        swap = rng.choice(topk, 16, replace=False)
        row[swap] = rng.choice(np.arange(N - L, N - L + t + 1), 16)
        row = np.unique(row)
        idx[t, : len(row)] = row
        idx[t, len(row):] = -1
    idx[7, 100:] = -1
    rows = list(range(0, L, 53)) + [7, L - 1]
    check(q, kv, idx, 1 / math.sqrt(192), rows=rows)


# ---- split-key attention: blocks with too few queries to fill the GPU (decode) divide each
# ---- query's selection among several CTAs and merge the shares by their log-sum-exp
@pytest.mark.parametrize("N,L,H,topk,pad", [(131072, 1, 64, 2048, 0), (131072, 1, 128, 2048, 0),
                                            (5000, 3, 64, 300, 0), (9000, 2, 64, 1000, 400)])
def test_decode_split_key(N, L, H, topk, pad):
    q, kv = make(N, L, H, seed=N % 97 + H)
    idx = random_selection(N, L, topk, seed=L + H, pad=pad)
    check(q, kv, idx, 1 / math.sqrt(192))


def test_decode_split_key_empty_shares():
    """Shares left with no valid key (all -1) contribute nothing; an all-padding row is zero with LSE -inf."""
    N, L, H, topk = 4000, 2, 64, 1024
    q, kv = make(N, L, H, seed=31)
    idx = np.full((L, topk), -1, dtype=np.int32)
    idx[0, :100] = np.sort(np.random.default_rng(2).choice(N, 100, replace=False))  # only the first share has keys
    out, lse = run_mla(q, kv, idx, 1 / math.sqrt(192))
    assert np.all(out[1] == 0.0) and np.all(np.isneginf(lse[1]))
    check(q, kv, idx, 1 / math.sqrt(192), rows=[0])
