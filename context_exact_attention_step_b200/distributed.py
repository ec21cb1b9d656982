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

* USP (compassingai, closing section: Ulysses inside the NVLink domain, Ring
  across it; pwwt.cn §6): a Pr x Pu grid of ranks, Ulysses inside each group
  of Pu ranks, then a ring over the Pr groups for every head block, each on
  its own process group (``usp_groups``).
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


def _seq_to_heads(x: torch.Tensor, P: int, group, kernels) -> torch.Tensor:
    """[n, h, dh] rows of this rank -> [P*n, h/P, dh]: every rank's rows of
    this rank's head block (block p of the heads goes to rank p)."""
    n, h, dh = x.shape
    blocks = kernels.head_block_split(x, P)           # [P, n, h/P, dh]: block p goes to rank p
    got = torch.empty_like(blocks)
    dist.all_to_all_single(got, blocks, group=group)  # got[p] = rank p's rows of my heads
    return got.view(P * n, h // P, dh)


def _heads_to_seq(x_h: torch.Tensor, P: int, group, kernels) -> torch.Tensor:
    """Inverse of _seq_to_heads: [P*n, hb, dh] -> [n, P*hb, dh]."""
    rows, hb, dh = x_h.shape
    n = rows // P
    blocks = torch.empty((P, n, hb, dh), dtype=x_h.dtype, device=x_h.device)
    dist.all_to_all_single(blocks, x_h.view(P, n, hb, dh).contiguous(), group=group)
    return kernels.head_block_split(blocks, P, inverse=True)


def _lse_seq_to_heads(lse: torch.Tensor, P: int, group, kernels) -> torch.Tensor:
    """LSE [h, n] of this rank's rows -> [h/P, P*n] of its head block: head
    block p goes to rank p, and the [P][h/P][n] slabs received become
    [h/P][P][n]."""
    h, n = lse.shape
    got = torch.empty((h, n), dtype=lse.dtype, device=lse.device)
    dist.all_to_all_single(got, lse.contiguous(), group=group)
    return kernels.head_block_split(got.view(P, h // P, 1, n), P, inverse=True).view(h // P, P * n)


def _lse_heads_to_seq(lse_h: torch.Tensor, P: int, group, kernels) -> torch.Tensor:
    """Inverse of _lse_seq_to_heads: [hb, P*n] -> [P*hb, n]."""
    hb, rows = lse_h.shape
    n = rows // P
    send = kernels.head_block_split(lse_h.view(hb, P, n), P).view(P, hb, n)  # slab p: rank p's rows
    got = torch.empty_like(send)
    dist.all_to_all_single(got, send.contiguous(), group=group)
    return got.view(P * hb, n)


def ulysses_attn_fwd_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True, group=None,
                          softmax_scale: float = 0.0, kernels=_api):
    """DeepSpeed-Ulysses forward over the ranks of ``group``.  q [n, hq, dh],
    k, v [n, hkv, dh]: this rank's contiguous sequence shard (positions
    r*n .. r*n + n - 1).  P must divide hkv (no KV replication).
    Returns this rank's (O [n, hq, dh] fp32, LSE [hq, n] fp32)."""
    P = dist.get_world_size(group)
    n = q.shape[0]
    if k.shape[1] % P != 0:
        raise ValueError(f"P = {P} must divide the KV head count {k.shape[1]}")
    S = n * P
    qh, kh, vh = (_seq_to_heads(x, P, group, kernels) for x in (q, k, v))
    o_h, lse_h = kernels.block_attn_fwd(qh, kh, vh, [(0, S)], [(0, S)], causal, None, softmax_scale)
    return _heads_to_seq(o_h, P, group, kernels), _lse_heads_to_seq(lse_h, P, group, kernels)


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
                                   dk=dkv[:n], dv=dkv[n:], parts=_api.BWD_DKDV, accumulate=t > 0)
        elif t == 0:
            dkv.zero_()
        # the shard's gradient moves on with it; the last move brings it home
        # (with one rank it is home already)
        if P > 1:
            reqs += dist.batch_isend_irecv([dist.P2POp(dist.isend, dkv, send_to, group),
                                            dist.P2POp(dist.irecv, dkv_next, recv_from, group)])
        if live:
            kernels.block_attn_bwd(q, kv[:n], kv[n:], do, lg, dd, q_chunks, k_chunks, causal, cu_dev, softmax_scale,
                                   dq=dq, parts=_api.BWD_DQ, accumulate=t > 0)
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
    if k.shape[1] % P != 0:
        raise ValueError(f"P = {P} must divide the KV head count {k.shape[1]}")
    qh, kh, vh, doh, oh = (_seq_to_heads(x, P, group, kernels) for x in (q, k, v, do, o))
    lse_h = _lse_seq_to_heads(lse, P, group, kernels)
    dqh, dkh, dvh = kernels.ring_attn_bwd(qh, kh, vh, oh, lse_h, doh, 1, "contiguous", causal,
                                          softmax_scale=softmax_scale)
    return tuple(_heads_to_seq(g, P, group, kernels) for g in (dqh, dkh, dvh))


# ------------------------------------------------------------------ USP hybrid
def usp_groups(Pr: int, Pu: int):
    """The two process groups of the calling rank in a Pr x Pu grid of the
    default group's P = Pr * Pu ranks, rank R = g * Pu + u: its Ulysses group
    (the Pu ranks of ring group g, in order of u) and its ring group (the Pr
    ranks with the same u, in order of g).  Every rank must call this, in the
    same order, because creating a group is collective."""
    P = dist.get_world_size()
    if Pr * Pu != P:
        raise ValueError(f"Pr * Pu = {Pr * Pu} != world size {P}")
    R = dist.get_rank()
    mine_u = mine_r = None
    for g in range(Pr):
        grp = dist.new_group([g * Pu + u for u in range(Pu)])
        if R // Pu == g:
            mine_u = grp
    for u in range(Pu):
        grp = dist.new_group([g * Pu + u for g in range(Pr)])
        if R % Pu == u:
            mine_r = grp
    return mine_u, mine_r


def usp_attn_fwd_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, layout: str = "contiguous",
                      causal: bool = True, cu_seqlens: Optional[Sequence[int]] = None, groups=None,
                      softmax_scale: float = 0.0, kernels=_api):
    """The Ulysses-inside / Ring-across hybrid over a Pr x Pu rank grid
    (compassingai, closing section; pwwt.cn §6).  ``groups`` = (Ulysses
    group, ring group) from ``usp_groups``.  Rank (g, u) holds rows
    [u*n, (u+1)*n) of ring shard g of ``layout`` over Pr (q [n, hq, dh], k, v
    [n, hkv, dh]); Pu must divide hkv.  Steps: Ulysses seq->head inside the
    group (the group's m = Pu*n rows of head block u), the ring over the Pr
    groups for that head block, Ulysses head->seq.  Returns this rank's
    (O [n, hq, dh] fp32, LSE [hq, n] fp32)."""
    ug, rg = groups
    Pu = dist.get_world_size(ug)
    if k.shape[1] % Pu != 0:
        raise ValueError(f"Pu = {Pu} must divide the KV head count {k.shape[1]}")
    qh, kh, vh = (_seq_to_heads(x, Pu, ug, kernels) for x in (q, k, v))
    o_h, lse_h = ring_attn_fwd_dist(qh, kh, vh, layout, causal, cu_seqlens, rg, softmax_scale, kernels)
    return _heads_to_seq(o_h, Pu, ug, kernels), _lse_heads_to_seq(lse_h, Pu, ug, kernels)


def usp_attn_bwd_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                      do: torch.Tensor, layout: str = "contiguous", causal: bool = True,
                      cu_seqlens: Optional[Sequence[int]] = None, groups=None, softmax_scale: float = 0.0,
                      kernels=_api):
    """Backward of ``usp_attn_fwd_dist``: Q, K, V, dO, O and LSE to head
    layout inside the Ulysses group, the ring backward over the ring group
    for this head block, dQ, dK, dV back.  Returns this rank's (dQ [n, hq, dh],
    dK, dV [n, hkv, dh]) fp32."""
    ug, rg = groups
    Pu = dist.get_world_size(ug)
    if k.shape[1] % Pu != 0:
        raise ValueError(f"Pu = {Pu} must divide the KV head count {k.shape[1]}")
    qh, kh, vh, doh, oh = (_seq_to_heads(x, Pu, ug, kernels) for x in (q, k, v, do, o))
    lse_h = _lse_seq_to_heads(lse, Pu, ug, kernels)
    grads = ring_attn_bwd_dist(qh, kh, vh, oh, lse_h, doh, layout, causal, cu_seqlens, rg, softmax_scale, kernels)
    return tuple(_heads_to_seq(g, Pu, ug, kernels) for g in grads)
