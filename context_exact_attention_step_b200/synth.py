"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds no attention arithmetic: it only draws tensors and document
lengths from fixed seeds so that the CUDA path and the fp64 oracle see the same
bits.  Recipe (the pages' model: 32 heads, hidden 4096, bf16; "Context
Parallelism" write-up (pwwt.cn) §4.1):

* Q, K, V: float32 N(0, 1) from ``torch.Generator('cpu').manual_seed(seed)``
  (seeds Q=1, K=2, V=3 unless overridden), multiplied by ``std`` (0.5 for the
  bf16 workloads, 1.0 for the tiny fp32 one), then rounded to bf16 with
  round-to-nearest-even when ``dtype`` is bf16.
* Upstream gradient dO for the backward: same recipe as Q (seed 5).
* Packed documents: integer lengths uniform on [lo, hi] inclusive drawn from
  seed 4 until their sum reaches the total; the last one is truncated so the
  lengths add up to exactly the total.  ``cu_seqlens`` are their int32 prefix
  sums starting at 0.
"""
from __future__ import annotations

import torch

SEED_Q, SEED_K, SEED_V, SEED_DOCS, SEED_DO = 1, 2, 3, 4, 5


def normal(shape, seed, std=1.0, dtype=torch.bfloat16):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(dtype) if dtype != torch.float32 else x


def qkv(S, hq, hkv, dh, std=0.5, dtype=torch.bfloat16, seeds=(SEED_Q, SEED_K, SEED_V)):
    """Q [S, hq, dh], K and V [S, hkv, dh] on the CPU."""
    q = normal((S, hq, dh), seeds[0], std, dtype)
    k = normal((S, hkv, dh), seeds[1], std, dtype)
    v = normal((S, hkv, dh), seeds[2], std, dtype)
    return q, k, v


def doc_lengths(total, lo=1024, hi=32768, seed=SEED_DOCS):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    lens = []
    acc = 0
    while acc < total:
        L = int(torch.randint(lo, hi + 1, (1,), generator=g).item())
        L = min(L, total - acc)
        lens.append(L)
        acc += L
    return lens


def cu_seqlens_from_lengths(lens):
    cu = [0]
    for L in lens:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32)


# The workloads the library is tested and measured on.
CONFIGS = {
    "tiny_ring_fp32": dict(S=1024, hq=4, hkv=4, dh=64, P=4, layout="contiguous",
                           causal=True, varlen=False, std=1.0, dtype="fp32"),
    "ring_contig_32k": dict(S=32768, hq=32, hkv=32, dh=128, P=4, layout="contiguous",
                            causal=True, varlen=False, std=0.5, dtype="bf16"),
    "ring_zigzag_64k": dict(S=65536, hq=32, hkv=32, dh=128, P=8, layout="zigzag",
                            causal=True, varlen=False, std=0.5, dtype="bf16"),
    "ring_striped_64k": dict(S=65536, hq=32, hkv=32, dh=128, P=8, layout="striped",
                             causal=True, varlen=False, std=0.5, dtype="bf16"),
    "ulysses_gqa_128k": dict(S=131072, hq=32, hkv=8, dh=128, P=8, layout="ulysses",
                             causal=True, varlen=False, std=0.5, dtype="bf16"),
    # Ulysses over Pu = 4 ranks inside each of Pr = 2 zigzag ring groups: 8
    # ranks against 4 KV heads, which Ulysses alone cannot shard.
    "usp_gqa_128k": dict(S=131072, hq=32, hkv=4, dh=128, P=8, Pr=2, Pu=4, layout="usp", ring_layout="zigzag",
                         causal=True, varlen=False, std=0.5, dtype="bf16"),
    "varlen_zigzag_128k": dict(S=131072, hq=32, hkv=32, dh=128, P=8, layout="zigzag",
                               causal=True, varlen=True, std=0.5, dtype="bf16",
                               doc_lo=1024, doc_hi=32768),
}
