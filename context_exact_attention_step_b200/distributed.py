"""Ring Attention and DeepSpeed-Ulysses across the GPUs of a process group.

One process per GPU, ``torch.distributed`` (NCCL over NVLink / NVSwitch) for
the exchanges, the library's kernels for every computation.  Rank r holds
shard r of the sequence in the same order the single-GPU entry points use
(contiguous, zigzag or striped), so a run on P GPUs computes exactly what
``ring_attn_fwd`` computes with P virtual ranks on one GPU.

* Ring ("序列並行（Sequence Parallelism）" concept page (compassingai),
  "Ring Attention 的不同思路" steps 1-4; "Context Parallelism" write-up
  (pwwt.cn) §2.2): rank r keeps Q_r; the K/V shard it holds moves one rank
  forward per step, so at step t it holds shard j = (r - t) mod P.  The
  exchange for step t+1 is posted before step t's block attention is launched,
  so the transfer overlaps the computation; every live step leaves a partial
  (O, LSE) and the LSE merge folds them once at the end.  Steps whose block
  pair admits no (q, k) pair (the host schedule decides) skip the computation
  but still forward the shard, so every rank posts the same exchanges in the
  same order.
* Ulysses (compassingai §三 "Ulysses 的 AllToAll 轉置"; pwwt.cn §2.3): each
  rank regroups its rows by head block, one all-to-all gives it every position
  of its own heads, it attends over the whole sequence, and a second
  all-to-all plus the inverse regrouping bring O back to sequence shards.

``kernels`` is the object whose ``block_attn_fwd``, ``lse_merge``,
``head_block_split`` and ``ring_schedule`` are called: the library's API by
default.  The multi-process CPU tests pass stand-ins with the same signatures
to exercise the communication on ``gloo``; there is no fallback here.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import api as _api


def query_chunks(S: int, P: int, layout: str, r: int) -> List[Tuple[int, int]]:
    """(position, length) chunks of rank r's query rows, in storage order.
    Striped shards use local row indices as positions."""
    if layout == "contiguous":
        n = S // P
        return [(r * n, n)]
    if layout == "zigzag":
        c = S // (2 * P)
        return [(r * c, c), ((2 * P - 1 - r) * c, c)]
    if layout == "striped":
        return [(0, S // P)]
    raise ValueError(f"unknown layout {layout}")


def key_chunks(S: int, P: int, layout: str, r: int, j: int) -> List[Tuple[int, int]]:
    """Chunks of key shard j as seen from query rank r: its own positions,
    except in the striped layout, where position j + P*b is at or before
    r + P*a exactly when b <= a (j <= r) or b < a (j > r), i.e. the local index
    shifted by one key when j > r."""
    if layout == "striped":
        return [(1 if j > r else 0, S // P)]
    return query_chunks(S, P, layout, j)


def _peer(group, rank: int) -> int:
    return rank if group is None else dist.get_global_rank(group, rank)


def ring_attn_fwd_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, layout: str = "contiguous",
                       causal: bool = True, cu_seqlens: Optional[Sequence[int]] = None, group=None,
                       softmax_scale: float = 0.0, kernels=_api):
    """Ring attention forward over the ranks of ``group``.  q [n, hq, dh],
    k, v [n, hkv, dh]: this rank's shard (S = n * P tokens in all).
    cu_seqlens: host document table of the whole sequence, or None.
    Returns this rank's (O [n, hq, dh] fp32, LSE [hq, n] fp32)."""
    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    n = q.shape[0]
    S = n * P
    if k.shape != v.shape:
        raise ValueError("k and v must have the same shape")
    sched = kernels.ring_schedule(S, P, layout, causal, cu_seqlens)
    cu_dev = None
    if cu_seqlens is not None:
        cu_dev = torch.as_tensor(list(cu_seqlens), dtype=torch.int32, device=q.device)
    kv = torch.cat([k, v], dim=0).contiguous()
    nxt = torch.empty_like(kv)
    send_to, recv_from = _peer(group, (r + 1) % P), _peer(group, (r - 1) % P)
    q_chunks = query_chunks(S, P, layout, r)
    parts_o, parts_l = [], []
    for t in range(P):
        j = (r - t) % P
        reqs = None
        if t < P - 1:
            reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, kv, send_to, group),
                                           dist.P2POp(dist.irecv, nxt, recv_from, group)])
        if sched["launched"][r * P + t]:
            o_t, l_t = kernels.block_attn_fwd(q, kv[:n], kv[n:], q_chunks, key_chunks(S, P, layout, r, j), causal,
                                              cu_dev, softmax_scale)
            parts_o.append(o_t)
            parts_l.append(l_t)
        if reqs is not None:
            for req in reqs:
                req.wait()
            kv, nxt = nxt, kv
    return kernels.lse_merge(parts_o, parts_l)


def ulysses_attn_fwd_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True, group=None,
                          softmax_scale: float = 0.0, kernels=_api):
    """DeepSpeed-Ulysses forward over the ranks of ``group``.  q [n, hq, dh],
    k, v [n, hkv, dh]: this rank's contiguous sequence shard (positions
    r*n .. r*n + n - 1).  P must divide hkv (no KV replication).
    Returns this rank's (O [n, hq, dh] fp32, LSE [hq, n] fp32)."""
    P = dist.get_world_size(group)
    n, hq, dh = q.shape
    hkv = k.shape[1]
    if hkv % P != 0:
        raise ValueError(f"P = {P} must divide the KV head count {hkv}")
    S = n * P
    hg = hq // P

    def to_heads(x):
        blocks = kernels.head_block_split(x, P)           # [P, n, h/P, dh]: block p goes to rank p
        got = torch.empty_like(blocks)
        dist.all_to_all_single(got, blocks, group=group)  # got[p] = rank p's rows of my heads
        return got.view(S, x.shape[1] // P, dh)

    qh, kh, vh = to_heads(q), to_heads(k), to_heads(v)
    o_h, lse_h = kernels.block_attn_fwd(qh, kh, vh, [(0, S)], [(0, S)], causal, None, softmax_scale)
    # O back to sequence shards: block p of my heads' output holds rank p's rows
    o_blocks = torch.empty_like(o_h).view(P, n, hg, dh)
    dist.all_to_all_single(o_blocks, o_h.view(P, n, hg, dh).contiguous(), group=group)
    o = kernels.head_block_split(o_blocks, P, inverse=True)  # [n, hq, dh]
    # LSE [hg, S] -> per destination rank p the [hg, n] slab of its rows
    lse_send = kernels.head_block_split(lse_h.view(hg, P, n), P).view(P, hg, n)
    lse_recv = torch.empty_like(lse_send)
    dist.all_to_all_single(lse_recv, lse_send.contiguous(), group=group)
    return o, lse_recv.view(hq, n)
