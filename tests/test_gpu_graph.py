"""The whole path is capturable in a CUDA graph (no host synchronisation or allocation inside a call):
a captured dsa_prefill_chunk replays to the same bytes as the eager call."""
import pytest
import torch

import dsa_inputs
import deepseek_sparse_attention_relu_b200 as dsa

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,L,topk", [(8192, 1, 512), (12000, 130, 1024)], ids=["decode", "prefill"])
def test_prefill_chunk_replays_from_a_cuda_graph(N, L, topk):
    cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=N, L=L, topk=topk, H=64)
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in dsa_inputs.generate(cfg).items()}
    ws = dsa.alloc_workspace(dsa.dsa_prefill_chunk_workspace(L, N, cfg.H_I, cfg.D_I, cfg.H, topk, 0,
                                                             dsa.DSA_BF16, True), dev)

    def call(out, idx, lse, stream):
        dsa.dsa_prefill_chunk(g["q_idx"], g["k_idx"], g["w"], g["q"], g["kv"], cfg.q_pos0, topk, cfg.scale, out,
                              topk_idx=idx, lse=lse, workspace=ws, stream=stream)

    ref_out = torch.empty(L, cfg.H, 512, dtype=torch.bfloat16, device=dev)
    ref_idx = torch.empty(L, topk, dtype=torch.int32, device=dev)
    ref_lse = torch.empty(L, cfg.H, dtype=torch.float32, device=dev)
    call(ref_out, ref_idx, ref_lse, torch.cuda.current_stream())
    assert dsa.dsa_workspace_status(ws) == 0

    out = torch.full_like(ref_out, float("nan"))
    idx = torch.full_like(ref_idx, -7)
    lse = torch.full_like(ref_lse, float("nan"))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            call(out, idx, lse, side)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(3):
        out.fill_(float("nan"))
        idx.fill_(-7)
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert torch.equal(out, ref_out)
        assert torch.equal(lse, ref_lse)
    assert dsa.dsa_workspace_status(ws) == 0
