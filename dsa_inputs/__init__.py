"""Seeded synthetic inputs for DSA prefill chunks.

This module only draws random numbers and rounds them to the storage types;
it holds none of the method's arithmetic.  Both the CUDA library's tests and
benchmark and the CPU oracle read the buffers it produces, so the two sides see
the same bytes.

Every workload is a single prefill chunk of L queries at the end of a cache of
N keys (query t sits at position q_pos0 + t, q_pos0 = N - L):

* indexer operands q_idx [L, H_I, D_I] and k_idx [N, D_I] in bf16 or fp8 e4m3,
  head weights w [L, H_I] fp32;
* MLA operands q [L, H, 576] and the joined cache kv [N, 576] in bf16, each row
  512 latent columns then 64 rope columns.

Draw recipe (torch CPU generator seeded with ``seed``; fixed draw order
direction -> k_idx -> q_idx -> w -> kv -> q; kv drawn in blocks of 8192 rows and
q in blocks of 64 query rows so that peak host memory stays bounded):

* ``normal``: N(0, 1), rounded to nearest-even into bf16;
* ``int3``: integers uniform in [-3, 3], exact in bf16;
* ``concentrated``: N(0, 1) plus a shared mean direction mu = 2 * u, u a
  seeded uniform unit vector in R^D_I, added to every q_idx head row and every
  k_idx row, then rounded to e4m3 (RNE, saturated to +-448);
* ``walk`` (a stress input with correlated neighbouring queries, not one of
  the five workloads): k_idx N(0, 1); q_idx[0] N(0, 1) and q_idx[t] =
  q_idx[t-1] + 0.05 N(0, 1) elementwise, so neighbouring queries select
  mostly the same keys; rounded to bf16;
* weights ``normal_half`` N(0,1)/2, ``int12`` integers in {1, 2},
  ``normal_rsqrt`` N(0,1)/sqrt(H_I), ``walk_rsqrt``: w[0] N(0,1)/sqrt(H_I) and
  w[t] = w[t-1] + 0.05 N(0,1)/sqrt(H_I);
* MLA latent and rope columns N(0, std^2) with the stated standard deviations.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

IDX_BF16 = 0
IDX_E4M3 = 1
MLA_LAT = 512
MLA_ROPE = 64
MLA_DIM = MLA_LAT + MLA_ROPE


@dataclass(frozen=True)
class ChunkConfig:
    name: str
    N: int
    L: int
    H_I: int
    D_I: int
    idx_dtype: str  # "bf16" | "e4m3"
    idx_dist: str  # "normal" | "int3" | "concentrated" | "walk"
    w_dist: str  # "normal_half" | "int12" | "normal_rsqrt" | "walk_rsqrt"
    topk: int
    H: int
    lat_std: float
    rope_std: float
    seed: int
    query_block: int = 1024
    scale: float = 1.0 / math.sqrt(192.0)

    @property
    def q_pos0(self) -> int:
        return self.N - self.L

    @property
    def idx_code(self) -> int:
        return IDX_BF16 if self.idx_dtype == "bf16" else IDX_E4M3

    def visible_pairs(self) -> int:
        """Number of (query, visible key) pairs: sum over t of (q_pos0 + t + 1)."""
        return self.L * (self.q_pos0 + 1) + self.L * (self.L - 1) // 2


# The five workloads, smallest first.  Seeds are fixed per workload.
TINY = ChunkConfig("dsa-tiny-N4096-L256", N=4096, L=256, H_I=4, D_I=64, idx_dtype="bf16", idx_dist="normal",
                   w_dist="normal_half", topk=256, H=8, lat_std=0.5, rope_std=1.0, seed=0)
TIES = ChunkConfig("dsa-ties-N16384-L512", N=16384, L=512, H_I=32, D_I=128, idx_dtype="bf16", idx_dist="int3",
                   w_dist="int12", topk=2048, H=64, lat_std=0.5, rope_std=0.5, seed=1)
CTX64K = ChunkConfig("dsa-64k-fp8-N65536-L2048", N=65536, L=2048, H_I=32, D_I=128, idx_dtype="e4m3",
                     idx_dist="concentrated", w_dist="normal_rsqrt", topk=2048, H=64, lat_std=0.5, rope_std=0.5,
                     seed=2)
CTX128K = ChunkConfig("dsa-128k-N131072-L1024", N=131072, L=1024, H_I=32, D_I=128, idx_dtype="bf16",
                      idx_dist="normal", w_dist="normal_rsqrt", topk=2048, H=64, lat_std=0.5, rope_std=0.5, seed=3)
CTX256K = ChunkConfig("dsa-256k-fp8-N262144-L8192", N=262144, L=8192, H_I=32, D_I=128, idx_dtype="e4m3",
                      idx_dist="concentrated", w_dist="normal_rsqrt", topk=2048, H=128, lat_std=0.5, rope_std=0.5,
                      seed=4)

WORKLOADS = [TINY, TIES, CTX64K, CTX128K, CTX256K]
# Decode: one new query over the 128K cache (the same distributions as the 128K
# workload).  Not one of the five benchmark workloads; a latency case.
DECODE128K = ChunkConfig("dsa-decode-128k-N131072-L1", N=131072, L=1, H_I=32, D_I=128, idx_dtype="bf16",
                         idx_dist="normal", w_dist="normal_rsqrt", topk=2048, H=64, lat_std=0.5, rope_std=0.5,
                         seed=3)
# Stress input for candidate-overlap reuse: queries whose selections overlap
# heavily (q_idx and w random walks over the queries).  Not a benchmark workload.
CORRELATED = ChunkConfig("dsa-correlated-N65536-L1024", N=65536, L=1024, H_I=32, D_I=128, idx_dtype="bf16",
                         idx_dist="walk", w_dist="walk_rsqrt", topk=2048, H=64, lat_std=0.5, rope_std=0.5, seed=5)
WALK_STEP = 0.05
BY_NAME = {c.name: c for c in WORKLOADS + [DECODE128K, CORRELATED]}


def small_variant(cfg: ChunkConfig, N: int, L: int, topk: int | None = None, H: int | None = None,
                  seed: int | None = None) -> ChunkConfig:
    """The same distributions at a smaller size (for parity runs the oracle finishes quickly)."""
    return replace(cfg, name=f"{cfg.name}@N{N}-L{L}", N=N, L=L, topk=topk if topk is not None else cfg.topk,
                   H=H if H is not None else cfg.H, seed=cfg.seed if seed is None else seed)


def _to_idx_storage(x: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return x.to(torch.bfloat16)
    return x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn)


def _draw_idx(g: torch.Generator, shape, dist: str, mu: torch.Tensor | None, walk: bool = False) -> torch.Tensor:
    if dist == "int3":
        return torch.randint(-3, 4, shape, generator=g).to(torch.float32)
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if dist == "concentrated":
        x += mu
    if dist == "walk" and walk:  # along the first axis: x[t] = x[t-1] + WALK_STEP * N(0, 1)
        x[1:] *= WALK_STEP
        x = torch.cumsum(x, dim=0)
    return x


def _draw_mla(g: torch.Generator, rows: int, lat_std: float, rope_std: float) -> torch.Tensor:
    x = torch.randn(rows, MLA_DIM, generator=g, dtype=torch.float32)
    x[:, :MLA_LAT] *= lat_std
    x[:, MLA_LAT:] *= rope_std
    return x.to(torch.bfloat16)


def generate(cfg: ChunkConfig, with_mla: bool = True) -> dict:
    """All input buffers of one chunk as contiguous torch CPU tensors.

    Returns q_idx (bfloat16 or float8_e4m3fn), k_idx, w (float32) and, when
    with_mla, q [L,H,576] and kv [N,576] (bfloat16).
    """
    g = torch.Generator().manual_seed(cfg.seed)
    mu = None
    if cfg.idx_dist == "concentrated":
        u = torch.randn(cfg.D_I, generator=g, dtype=torch.float64)
        mu = (2.0 * u / u.norm()).to(torch.float32)
    k_idx = _to_idx_storage(_draw_idx(g, (cfg.N, cfg.D_I), cfg.idx_dist, mu), cfg.idx_dtype)
    q_idx = _to_idx_storage(_draw_idx(g, (cfg.L, cfg.H_I, cfg.D_I), cfg.idx_dist, mu, walk=True), cfg.idx_dtype)
    if cfg.w_dist == "int12":
        w = torch.randint(1, 3, (cfg.L, cfg.H_I), generator=g).to(torch.float32)
    elif cfg.w_dist == "normal_half":
        w = torch.randn(cfg.L, cfg.H_I, generator=g, dtype=torch.float32) / 2.0
    elif cfg.w_dist == "normal_rsqrt":
        w = torch.randn(cfg.L, cfg.H_I, generator=g, dtype=torch.float32) / math.sqrt(cfg.H_I)
    elif cfg.w_dist == "walk_rsqrt":
        w = torch.randn(cfg.L, cfg.H_I, generator=g, dtype=torch.float32)
        w[1:] *= WALK_STEP
        w = torch.cumsum(w, dim=0) / math.sqrt(cfg.H_I)
    else:
        raise ValueError(cfg.w_dist)
    out = {"q_idx": q_idx.contiguous(), "k_idx": k_idx.contiguous(), "w": w.contiguous()}
    if with_mla:
        kv = torch.empty(cfg.N, MLA_DIM, dtype=torch.bfloat16)
        for r0 in range(0, cfg.N, 8192):
            r1 = min(cfg.N, r0 + 8192)
            kv[r0:r1] = _draw_mla(g, r1 - r0, cfg.lat_std, cfg.rope_std)
        q = torch.empty(cfg.L, cfg.H, MLA_DIM, dtype=torch.bfloat16)
        for t0 in range(0, cfg.L, 64):
            t1 = min(cfg.L, t0 + 64)
            q[t0:t1] = _draw_mla(g, (t1 - t0) * cfg.H, cfg.lat_std, cfg.rope_std).view(t1 - t0, cfg.H, MLA_DIM)
        out["kv"] = kv
        out["q"] = q
    return out


def raw_bits(t: torch.Tensor) -> torch.Tensor:
    """The storage bits of a bf16 / e4m3 tensor (uint16 / uint8 view), for byte-level consumers."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8)
    return t
