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

* Backward (the gradient of the same exact attention; the pages define the
  forward only): the ring form keeps each rank's merged O and LSE, so at step
  t rank r adds the contribution of block pair (r, j) to its dQ_r and to the
  dK_j, dV_j that travel with shard j: K/V move one rank forward per step as
  in the forward, and the fp32 dK/dV of the shard follow them, so after P
  moves every shard's gradient is back at its owner.  Ulysses: Q, K, V, dO, O
  and LSE go to head layout, the backward runs over the whole sequence, and
  dQ, dK, dV come back by the inverse all-to-all.

``kernels`` is the object whose ``block_attn_fwd``, ``lse_merge``,
``head_block_split``, ``ring_schedule``, ``attn_bwd_prep``,
``block_attn_bwd`` and ``ring_attn_bwd`` are called: the library's API by
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


def ring_attn_bwd_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                       do: torch.Tensor, layout: str = "contiguous", causal: bool = True,
                       cu_seqlens: Optional[Sequence[int]] = None, group=None, softmax_scale: float = 0.0,
                       kernels=_api):
    """Ring attention backward over the ranks of ``group``.  q, do [n, hq, dh]
    and k, v [n, hkv, dh]: this rank's shard as given to ``ring_attn_fwd_dist``;
    o [n, hq, dh], lse [hq, n]: what it returned.  Returns this rank's
    (dQ [n, hq, dh], dK [n, hkv, dh], dV [n, hkv, dh]) fp32.

    Per step: the K/V exchange for the next step is posted first; the dK/dV
    kernel adds this pair's share to the gradient of the shard held; that
    gradient is posted to the next rank; the dQ kernel runs while it travels."""
    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    n = q.shape[0]
    S = n * P
    if k.shape != v.shape:
        raise ValueError("k and v must have the same shape")
    hkv, dh = k.shape[1], k.shape[2]
    sched = kernels.ring_schedule(S, P, layout, causal, cu_seqlens)
    cu_dev = None
    if cu_seqlens is not None:
        cu_dev = torch.as_tensor(list(cu_seqlens), dtype=torch.int32, device=q.device)
    lg, dd = kernels.attn_bwd_prep(o, lse, do)
    kv = torch.cat([k, v], dim=0).contiguous()
    kv_next = torch.empty_like(kv)
    gdt = torch.promote_types(q.dtype, torch.float32)  # gradients in fp32 (or the inputs' wider type)
    dq = torch.empty(q.shape, dtype=gdt, device=q.device)
    dkv = torch.empty((2 * n, hkv, dh), dtype=gdt, device=q.device)  # gradient of the shard held
    dkv_next = torch.empty_like(dkv)
    send_to, recv_from = _peer(group, (r + 1) % P), _peer(group, (r - 1) % P)
    q_chunks = query_chunks(S, P, layout, r)
    for t in range(P):
        j = (r - t) % P
        reqs = []
        if t < P - 1:
            reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, kv, send_to, group),
                                           dist.P2POp(dist.irecv, kv_next, recv_from, group)])
        live = sched["launched"][r * P + t]
        k_chunks = key_chunks(S, P, layout, r, j)
        if live:
            kernels.block_attn_bwd(q, kv[:n], kv[n:], do, lg, dd, q_chunks, k_chunks, causal, cu_dev, softmax_scale,
                                   dk=dkv[:n], dv=dkv[n:], parts=2, accumulate=t > 0)
        elif t == 0:
            dkv.zero_()
        # the shard's gradient moves on with it; the last move brings it home
        # (with one rank it is home already)
        if P > 1:
            reqs += dist.batch_isend_irecv([dist.P2POp(dist.isend, dkv, send_to, group),
                                            dist.P2POp(dist.irecv, dkv_next, recv_from, group)])
        if live:
            kernels.block_attn_bwd(q, kv[:n], kv[n:], do, lg, dd, q_chunks, k_chunks, causal, cu_dev, softmax_scale,
                                   dq=dq, parts=1, accumulate=t > 0)
        elif t == 0:
            dq.zero_()
        for req in reqs:
            req.wait()
        if t < P - 1:
            kv, kv_next = kv_next, kv
        if P > 1:
            dkv, dkv_next = dkv_next, dkv
    return dq, dkv[:n], dkv[n:]


def ulysses_attn_bwd_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                          do: torch.Tensor, causal: bool = True, group=None, softmax_scale: float = 0.0,
                          kernels=_api):
    """DeepSpeed-Ulysses backward over the ranks of ``group``: inputs as
    ``ulysses_attn_fwd_dist`` plus its o [n, hq, dh], lse [hq, n] and the
    upstream do [n, hq, dh].  Returns this rank's (dQ [n, hq, dh], dK, dV
    [n, hkv, dh]) fp32."""
    P = dist.get_world_size(group)
    n, hq, dh = q.shape
    hkv = k.shape[1]
    if hkv % P != 0:
        raise ValueError(f"P = {P} must divide the KV head count {hkv}")
    S = n * P
    hg = hq // P

    def to_heads(x):
        blocks = kernels.head_block_split(x, P)
        got = torch.empty_like(blocks)
        dist.all_to_all_single(got, blocks, group=group)
        return got.view(S, x.shape[1] // P, x.shape[2])

    def to_seq(x_h):
        h = x_h.shape[1]
        blocks = torch.empty_like(x_h).view(P, n, h, dh)
        dist.all_to_all_single(blocks, x_h.view(P, n, h, dh).contiguous(), group=group)
        return kernels.head_block_split(blocks, P, inverse=True)

    qh, kh, vh, doh, oh = (to_heads(x) for x in (q, k, v, do, o))
    # LSE [hq, n]: head block p goes to rank p; the [P][hg][n] slabs received
    # become [hg][P][n] = [hg, S]
    lse_recv = torch.empty_like(lse)
    dist.all_to_all_single(lse_recv, lse.contiguous(), group=group)
    lse_h = kernels.head_block_split(lse_recv.view(P, hg, 1, n), P, inverse=True).view(hg, S)
    dqh, dkh, dvh = kernels.ring_attn_bwd(qh, kh, vh, oh, lse_h, doh, 1, "contiguous", causal,
                                          softmax_scale=softmax_scale)
    return to_seq(dqh), to_seq(dkh), to_seq(dvh)
