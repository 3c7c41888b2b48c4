"""Padded key caches: k_idx and kv given as row-strided views (rows wider than the data, as a cache with
padding or a view of the leading columns of a wider buffer) select and attend exactly as contiguous ones."""
import pytest
import torch

import dsa_inputs
import deepseek_sparse_attention_relu_b200 as dsa

pytestmark = pytest.mark.gpu


def padded_view(x: torch.Tensor, extra: int) -> torch.Tensor:
    buf = torch.full((x.shape[0], x.shape[1] + extra), 0, dtype=x.dtype, device=x.device)
    if x.dtype == torch.float8_e4m3fn:
        buf.view(torch.uint8).fill_(0x7F)  # fill the padding with a large value: it must never be read
    else:
        buf.fill_(float("nan"))
    buf[:, : x.shape[1]] = x
    v = buf[:, : x.shape[1]]
    assert v.stride(0) == x.shape[1] + extra and not v.is_contiguous()
    return v


@pytest.mark.parametrize("base,k_extra", [(dsa_inputs.CTX128K, 64), (dsa_inputs.CTX64K, 16)], ids=["bf16", "fp8"])
def test_strided_caches_match_contiguous(base, k_extra):
    cfg = dsa_inputs.small_variant(base, N=20000, L=130, topk=512, H=64)
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in dsa_inputs.generate(cfg).items()}
    dt = dsa.DSA_BF16 if cfg.idx_dtype == "bf16" else dsa.DSA_FP8_E4M3
    ws = dsa.alloc_workspace(dsa.dsa_prefill_chunk_workspace(cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.H, cfg.topk, 0, dt,
                                                             True), dev)

    def run(k_idx, kv):
        out = torch.empty(cfg.L, cfg.H, 512, dtype=torch.bfloat16, device=dev)
        idx = torch.empty(cfg.L, cfg.topk, dtype=torch.int32, device=dev)
        lse = torch.empty(cfg.L, cfg.H, dtype=torch.float32, device=dev)
        dsa.dsa_prefill_chunk(g["q_idx"], k_idx, g["w"], g["q"], kv, cfg.q_pos0, cfg.topk, cfg.scale, out,
                              topk_idx=idx, lse=lse, workspace=ws)
        assert dsa.dsa_workspace_status(ws) == 0
        return idx, out, lse

    ref = run(g["k_idx"], g["kv"])
    got = run(padded_view(g["k_idx"], k_extra), padded_view(g["kv"], 64))
    for a, b in zip(ref, got):
        assert torch.equal(a, b)


def test_strided_kv_attention_only_and_bad_strides():
    dev = torch.device("cuda")
    N, L, H, topk = 3000, 6, 64, 256
    gen = torch.Generator().manual_seed(5)
    q = (torch.randn(L, H, 576, generator=gen) * 0.5).to(torch.bfloat16).to(dev)
    kv = (torch.randn(N, 576, generator=gen) * 0.5).to(torch.bfloat16).to(dev)
    idx = torch.stack([torch.randperm(N, generator=gen)[:topk].sort().values for _ in range(L)]).to(torch.int32).to(dev)
    ws = dsa.alloc_workspace(dsa.dsa_sparse_mla_workspace(L, H, topk), dev)
    outs = []
    for kvv in (kv, padded_view(kv, 64)):
        out = torch.empty(L, H, 512, dtype=torch.bfloat16, device=dev)
        dsa.dsa_sparse_mla_prefill(q, kvv, idx, 0.07, out, workspace=ws)
        assert dsa.dsa_workspace_status(ws) == 0
        outs.append(out)
    assert torch.equal(outs[0], outs[1])
    with pytest.raises(ValueError):  # rows must be contiguous
        dsa.dsa_sparse_mla_prefill(q, kv.t().contiguous().t(), idx, 0.07, outs[0], workspace=ws)
    with pytest.raises(dsa.DSAError):  # rows not 16-byte aligned
        dsa.dsa_sparse_mla_prefill(q, padded_view(kv, 4), idx, 0.07, outs[0], workspace=ws)
