"""Seeded synthetic inputs shared by the CUDA path's tests, the bench and the oracle checks.

This module holds no attention or quantization arithmetic: it only draws
i.i.d. N(0, 1) values with torch's CPU generator and rounds them to bf16, the
activations' dtype, and draws uniform random NF4 weight storage.  Seeds 0, 1,
2, 3 draw q, k, v and dO respectively (an offset shifts all four).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Shape:
    """One attention problem: batch B, query heads H, kv heads Hkv, head dim D,
    sequence length N, group size G (G == N means dense causal)."""
    name: str
    B: int
    H: int
    Hkv: int
    D: int
    N: int
    G: int

    def dense(self) -> "Shape":
        return Shape(self.name + "-dense", self.B, self.H, self.Hkv, self.D, self.N, self.N)


# The five workload shapes: group size a quarter of the sequence, half the
# (query) heads shifted by half a group.
TINY = Shape("tiny", 1, 4, 4, 64, 1024, 256)
LLAMA2_7B_8K = Shape("llama2-7b-n8192", 1, 32, 32, 128, 8192, 2048)
QWEN3_8B_16K = Shape("qwen3-8b-gqa-n16384", 1, 32, 8, 128, 16384, 4096)
LLAMA2_70B_32K = Shape("llama2-70b-gqa-n32768", 1, 64, 8, 128, 32768, 8192)
LLAMA2_7B_100K = Shape("llama2-7b-n102400", 1, 32, 32, 128, 102400, 25600)
WORKLOADS = [TINY, LLAMA2_7B_8K, QWEN3_8B_16K, LLAMA2_70B_32K, LLAMA2_7B_100K]


def randn_bf16(shape, seed: int) -> torch.Tensor:
    """fp32 N(0,1) from a seeded CPU generator, rounded to bf16 (RNE)."""
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def make_inputs(s: Shape, seed_offset: int = 0):
    """(q, k, v, dO) as CPU bf16 tensors: q, dO [B,N,H,D]; k, v [B,N,Hkv,D]."""
    q = randn_bf16((s.B, s.N, s.H, s.D), 0 + seed_offset)
    k = randn_bf16((s.B, s.N, s.Hkv, s.D), 1 + seed_offset)
    v = randn_bf16((s.B, s.N, s.Hkv, s.D), 2 + seed_offset)
    do = randn_bf16((s.B, s.N, s.H, s.D), 3 + seed_offset)
    return q, k, v, do


# The QKV projection of the LLaMA2-7B layer at 8192 tokens: model width 4096,
# 32 heads of 128 (q, k and v each 4096 features).
NF4_LLAMA2_7B_8K = dict(name="llama2-7b-qkv-n8192", M=8192, K=4096, H=32, Hkv=32, D=128)


def make_nf4_weights(rows: int, K: int, seed: int):
    """Random NF4 weight storage for a [rows, K] weight (CPU tensors).  Codes
    of quantized normal weights are close to uniform (the levels are normal
    quantiles), so the codes are uniform 4-bit values: uint8 [rows, K/2], two
    a byte; first-level scale codes int8 [rows K/64] uniform in [64, 127];
    second-level scales fp32 [ceil(rows K/64 / 256)] uniform in [0.05, 0.08]
    (absmax of 64 weights of a layer with std 0.02)."""
    g = torch.Generator().manual_seed(seed)
    codes = torch.randint(0, 256, (rows, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    nblk = rows * (K // 64)
    sq = torch.randint(64, 128, (nblk,), generator=g, dtype=torch.int32).to(torch.int8)
    c2 = 0.05 + 0.03 * torch.rand(((nblk + 255) // 256,), generator=g, dtype=torch.float32)
    return codes, sq, c2


def make_hga_selection(B: int, N: int, G: int, S: int, seed: int):
    """int32 [B, N/256, S] historical tile lists for HGA-style attention:
    for every 256-row query block, min(S, earlier tiles) distinct 128-row key
    tiles drawn uniformly from the segments before its own (ascending), the
    unused slots -1.  Random stand-ins for a model's chunk-summary choice."""
    import numpy as np
    rng = np.random.default_rng(seed)
    sel = -np.ones((B, N // 256, S), dtype=np.int32)
    for b in range(B):
        for qb in range(N // 256):
            prev = (qb * 256 // G) * G // 128
            n = min(S, prev)
            if n:
                sel[b, qb, :n] = np.sort(rng.choice(prev, size=n, replace=False))
    return torch.from_numpy(sel)
