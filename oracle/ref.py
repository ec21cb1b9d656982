"""fp64 CPU oracle for context-parallel exact attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
it is used by ``tests/``, by ``__graft_entry__.smoke()`` and by the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``.  It shares no code
with the CUDA library and does not import it.

Every function is the plain definition of what the method computes, written in
numpy float64 on the host, with no blocking, fusion or reordering beyond the
definition itself:

* ``attention``          -- full-matrix masked softmax attention with an
  explicit boolean mask (causal and/or same-document), natural log LSE of the
  scaled scores.  Sources: "序列並行（Sequence Parallelism）" concept page
  (compassingai), 技術原理 §二 "Ring Attention 的塊級線上 Softmax" (scores
  S = Q K^T / sqrt(d_k); the recurrence there is exact, so the unsplit softmax
  is the definition); "Context Parallelism" write-up (pwwt.cn) §3.3 and §5.2
  (the mask must follow the global positions of each KV block).
* ``ring_pair_partial``  -- one ring step: a shard's Q rows against one KV
  shard, same definition restricted to those rows/columns (compassingai page,
  "Ring Attention 的不同思路", steps 1-4; pwwt.cn §2.2).
* ``lse_merge``          -- folds partial (O, LSE) pairs, the block-granular
  form of the same recurrence (compassingai §二).
* ``zigzag_order`` / ``zigzag_reorder`` / ``zigzag_restore`` -- shard i holds
  chunks i and 2P-1-i of the 2P equal chunks ("长上下文序列并行训练深度解析"
  (mooersco) timeline: Striped / zigzag load-balancing reorder; the exact chunk
  pairing is the plainest balanced reading).  ``striped_order``: token t on
  rank t mod P (same timeline, Striped Attention).
* ``ulysses_seq_to_head`` / ``ulysses_head_to_seq`` -- the all-to-all
  transpose [S/P, H, d_h] -> [S, H/P, d_h] (compassingai §三 "Ulysses 的
  AllToAll 轉置"; pwwt.cn §2.3), device i taking head block i.
* ``usp_attention``      -- the Ulysses-inside / Ring-across hybrid, composed
  from the functions above (compassingai, closing section; pwwt.cn §6).
* ``attention_bwd`` / ``ring_attention_bwd`` -- the gradient of the exact
  attention for an upstream dO: by definition over the whole score matrix, and
  the ring form (per block pair with the merged LSE, KV gradients travelling
  with their shard).
* ``live_pair_count``    -- number of (q, k) pairs the explicit mask admits
  (brute force), the unit of the causal-effective FLOP count.
"""
from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf


# --------------------------------------------------------------------------
# masks
# --------------------------------------------------------------------------
def doc_of(pos, cu_seqlens):
    """Document index of each global position (cu_seqlens = prefix sums of
    document lengths, first entry 0, last entry S; XTuner tutorial ch09 §9.5,
    flash-attn ``cu_seqlens`` convention)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    return np.searchsorted(cu, np.asarray(pos, dtype=np.int64), side="right") - 1


def explicit_mask(qpos, kpos, causal, cu_seqlens=None):
    """Boolean [len(qpos), len(kpos)] mask, True where key k may be attended by
    query q.  causal: k <= q by global position; varlen: same document."""
    qpos = np.asarray(qpos, dtype=np.int64)
    kpos = np.asarray(kpos, dtype=np.int64)
    m = np.ones((qpos.size, kpos.size), dtype=bool)
    if causal:
        m &= kpos[None, :] <= qpos[:, None]
    if cu_seqlens is not None:
        m &= doc_of(qpos, cu_seqlens)[:, None] == doc_of(kpos, cu_seqlens)[None, :]
    return m


# --------------------------------------------------------------------------
# attention (the definition)
# --------------------------------------------------------------------------
def attention(q, k, v, causal=True, cu_seqlens=None, scale=None, qpos=None,
              kpos=None, row_block=256):
    """Masked softmax attention in float64.

    q: [Sq, Hq, dh]; k, v: [Sk, Hkv, dh] (Hq a multiple of Hkv; query head h
    reads KV head h // (Hq // Hkv)).  qpos / kpos are the global token
    positions of the rows (default 0..S-1).  Returns O [Sq, Hq, dh] and
    LSE [Hq, Sq] with LSE = ln sum_j exp(s_j) over the admitted keys of the
    scaled scores s_j = scale * q.k_j.  A row that admits no key gets O = 0 and
    LSE = -inf.  Rows are processed in blocks of ``row_block`` queries against
    ALL keys; no key blocking and no online softmax.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    sq, hq, dh = q.shape
    sk, hkv, _ = k.shape
    assert hq % hkv == 0
    group = hq // hkv
    if scale is None:
        scale = 1.0 / math.sqrt(dh)
    qpos = np.arange(sq) if qpos is None else np.asarray(qpos)
    kpos = np.arange(sk) if kpos is None else np.asarray(kpos)
    o = np.zeros((sq, hq, dh), dtype=np.float64)
    lse = np.full((hq, sq), NEG_INF, dtype=np.float64)
    for r0 in range(0, sq, row_block):
        r1 = min(sq, r0 + row_block)
        mask = explicit_mask(qpos[r0:r1], kpos, causal, cu_seqlens)
        live = mask.any(axis=1)
        for h in range(hq):
            g = h // group
            s = (q[r0:r1, h, :] @ k[:, g, :].T) * scale
            s = np.where(mask, s, NEG_INF)
            m = np.max(s, axis=1, initial=NEG_INF)
            m_safe = np.where(live, m, 0.0)
            e = np.where(mask, np.exp(s - m_safe[:, None]), 0.0)
            l = e.sum(axis=1)
            l_safe = np.where(live, l, 1.0)
            o[r0:r1, h, :] = np.where(live[:, None], (e @ v[:, g, :]) / l_safe[:, None], 0.0)
            lse[h, r0:r1] = np.where(live, m_safe + np.log(l_safe), NEG_INF)
    return o, lse


# --------------------------------------------------------------------------
# sharding layouts
# --------------------------------------------------------------------------
def shard_positions(S, P, layout, r):
    """Global positions held by virtual rank r, in the order the rank stores
    them.  contiguous: [r*S/P, (r+1)*S/P).  zigzag: chunk r then chunk 2P-1-r
    of the 2P chunks of S/(2P) tokens.  striped: r, r+P, r+2P, ... (token t
    on rank t mod P)."""
    if layout == "striped":
        return np.arange(r, S, P)
    if layout == "contiguous":
        n = S // P
        return np.arange(r * n, (r + 1) * n)
    if layout == "zigzag":
        c = S // (2 * P)
        return np.concatenate([np.arange(r * c, (r + 1) * c),
                               np.arange((2 * P - 1 - r) * c, (2 * P - r) * c)])
    raise ValueError(layout)


def zigzag_order(S, P):
    """order[i] = natural position of the token stored at row i of the
    rank-major zigzag layout."""
    return np.concatenate([shard_positions(S, P, "zigzag", r) for r in range(P)])


def zigzag_reorder(x, P, axis=0):
    """Natural order -> rank-major zigzag order (gather along ``axis``)."""
    x = np.asarray(x)
    return np.take(x, zigzag_order(x.shape[axis], P), axis=axis)


def striped_order(S, P):
    """order[i] = natural position of the token stored at row i of the
    rank-major striped layout."""
    return np.concatenate([shard_positions(S, P, "striped", r) for r in range(P)])


def zigzag_restore(y, P, axis=0):
    """Inverse of ``zigzag_reorder`` (scatter along ``axis``)."""
    y = np.asarray(y)
    order = zigzag_order(y.shape[axis], P)
    out = np.empty_like(y)
    idx = [slice(None)] * y.ndim
    idx[axis] = order
    out[tuple(idx)] = y
    return out


def ulysses_seq_to_head(x, P):
    """[P, n, H, dh] (rank p holds tokens p*n..p*n+n-1, all heads) ->
    [P, S, H/P, dh] (rank r holds all S tokens of heads r*H/P..(r+1)*H/P-1):
    out[r, p*n + s, h', d] = x[p, s, r*H/P + h', d]."""
    x = np.asarray(x)
    p_, n, h, dh = x.shape
    assert p_ == P and h % P == 0
    hg = h // P
    return x.reshape(P, n, P, hg, dh).transpose(2, 0, 1, 3, 4).reshape(P, P * n, hg, dh)


def ulysses_head_to_seq(y, P):
    """Inverse transpose: [P, S, H/P, dh] -> [P, S/P, H, dh]:
    out[p, s, r*H/P + h', d] = y[r, p*n + s, h', d]."""
    y = np.asarray(y)
    p_, s_total, hg, dh = y.shape
    assert p_ == P and s_total % P == 0
    n = s_total // P
    return y.reshape(P, P, n, hg, dh).transpose(1, 2, 0, 3, 4).reshape(P, n, P * hg, dh)


# --------------------------------------------------------------------------
# ring steps and the merge
# --------------------------------------------------------------------------
def ring_source(r, t, P):
    """KV shard that virtual rank r holds at ring step t: blocks move one rank
    forward per step, so rank r sees shard (r - t) mod P."""
    return (r - t) % P


def ring_pair_partial(q, k, v, S, P, layout, r, j, causal=True, cu_seqlens=None,
                      scale=None):
    """Partial (O, LSE) of rank r's queries against shard j's keys/values.
    q, k, v are in NATURAL order [S, H, dh]; the result rows follow rank r's
    storage order."""
    qp = shard_positions(S, P, layout, r)
    kp = shard_positions(S, P, layout, j)
    return attention(q[qp], k[kp], v[kp], causal=causal, cu_seqlens=cu_seqlens,
                     scale=scale, qpos=qp, kpos=kp)


def lse_merge(o_parts, lse_parts):
    """Fold partials: LSE = ln sum_i exp(LSE_i); O = sum_i exp(LSE_i - LSE) O_i.
    o_parts: [n, rows, H, dh]; lse_parts: [n, H, rows].  Partials with
    LSE_i = -inf contribute nothing; rows where every LSE_i is -inf give
    O = 0, LSE = -inf."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = np.max(lse_parts, axis=0)                      # [H, rows]
    live = np.isfinite(m)
    m_safe = np.where(live, m, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - m_safe[None]), 0.0)
    tot = w.sum(axis=0)
    tot_safe = np.where(live, tot, 1.0)
    lse = np.where(live, m_safe + np.log(tot_safe), NEG_INF)
    wn = w / tot_safe[None]                            # [n, H, rows]
    o = np.zeros(o_parts.shape[1:], dtype=np.float64)
    for i in range(o_parts.shape[0]):
        wi = np.transpose(wn[i])[:, :, None]           # [rows, H, 1]
        o += np.where(wi > 0, wi * o_parts[i], 0.0)
    return o, lse


def ring_attention(q, k, v, S, P, layout, causal=True, cu_seqlens=None, scale=None):
    """All P virtual ranks, all P ring steps, merged per rank.  Inputs in
    natural order; outputs in rank-major storage order:
    O [S, Hq, dh], LSE [Hq, S]."""
    outs, lses = [], []
    for r in range(P):
        parts_o, parts_l = [], []
        for t in range(P):
            j = ring_source(r, t, P)
            o_rj, l_rj = ring_pair_partial(q, k, v, S, P, layout, r, j, causal,
                                           cu_seqlens, scale)
            parts_o.append(o_rj)
            parts_l.append(l_rj)
        o_r, l_r = lse_merge(np.stack(parts_o), np.stack(parts_l))
        outs.append(o_r)
        lses.append(l_r)
    return np.concatenate(outs, axis=0), np.concatenate(lses, axis=1)


def usp_attention(q, k, v, S, Pr, Pu, layout, causal=True, cu_seqlens=None, scale=None):
    """USP, the two-dimensional hybrid: P = Pr * Pu ranks, Ulysses inside each
    group of Pu ranks and Ring across the Pr groups ("序列並行（Sequence
    Parallelism）" concept page (compassingai), closing section on mixing the
    two: Ulysses all-to-all inside the NVLink domain, Ring P2P across it;
    "Context Parallelism" write-up (pwwt.cn) §2 comparison and §6: first the
    Ulysses head regrouping inside the CP group, then the Ring passes the
    sequence).

    Reading taken: group g is ring shard g of ``layout`` over Pr ranks; its
    m = S/Pr tokens are split into Pu consecutive sub-shards of n = m/Pu tokens,
    sub-rank u of group g being global rank g*Pu + u.  Steps:
      1. Ulysses seq->head inside each group: sub-rank u gathers all m tokens of
         its group for query heads [u*Hq/Pu, ...) and KV heads [u*Hkv/Pu, ...);
      2. for each head block u, a ring over the Pr groups: group g holds KV
         shard j = (g - t) mod Pr at step t, the partials are folded by
         ``lse_merge``;
      3. Ulysses head->seq inside each group.
    Inputs in natural order [S, H, dh]; outputs in the storage order of the
    ranks (the ring layout over Pr, rank-major): O [S, Hq, dh], LSE [Hq, S]."""
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    hq, hkv, dh = q.shape[1], k.shape[1], q.shape[2]
    assert hq % Pu == 0 and hkv % Pu == 0 and S % (Pr * Pu) == 0
    m = S // Pr
    n = m // Pu
    hg = hq // Pu
    pos = [shard_positions(S, Pr, layout, g) for g in range(Pr)]
    # step 1: per group, [Pu, n, H, dh] -> [Pu, m, H/Pu, dh]
    qh = [ulysses_seq_to_head(q[pos[g]].reshape(Pu, n, hq, dh), Pu) for g in range(Pr)]
    kh = [ulysses_seq_to_head(k[pos[g]].reshape(Pu, n, hkv, dh), Pu) for g in range(Pr)]
    vh = [ulysses_seq_to_head(v[pos[g]].reshape(Pu, n, hkv, dh), Pu) for g in range(Pr)]
    # step 2: ring across groups, one per head block
    o_grp = [np.zeros((Pu, m, hg, dh)) for _ in range(Pr)]
    lse_grp = [np.zeros((Pu, hg, m)) for _ in range(Pr)]
    for u in range(Pu):
        for g in range(Pr):
            parts_o, parts_l = [], []
            for t in range(Pr):
                j = ring_source(g, t, Pr)
                o_p, l_p = attention(qh[g][u], kh[j][u], vh[j][u], causal=causal, cu_seqlens=cu_seqlens,
                                     scale=scale, qpos=pos[g], kpos=pos[j])
                parts_o.append(o_p)
                parts_l.append(l_p)
            o_grp[g][u], lse_grp[g][u] = lse_merge(np.stack(parts_o), np.stack(parts_l))
    # step 3: per group, [Pu, m, H/Pu, dh] -> [Pu, n, H, dh]; LSE head block u
    # of group g covers heads [u*hg, (u+1)*hg) and the group's m rows
    o = np.concatenate([ulysses_head_to_seq(o_grp[g], Pu).reshape(m, hq, dh) for g in range(Pr)], axis=0)
    lse = np.concatenate([lse_grp[g].reshape(hq, m) for g in range(Pr)], axis=1)
    return o, lse


# --------------------------------------------------------------------------
# backward
# --------------------------------------------------------------------------
def attention_bwd(q, k, v, do, causal=True, cu_seqlens=None, scale=None, qpos=None, kpos=None,
                  row_block=256):
    """Gradients of ``attention``'s O with respect to q, k, v for an upstream
    gradient ``do`` [Sq, Hq, dh], in float64, from the definition of the
    masked softmax: with P the attention probabilities (explicit mask, every
    key at once),
        dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(P * dP)),
        dQ = scale * dS K,  dK = scale * dS^T Q,
    where GQA sums dK, dV over the query heads that share a KV head.  The
    pages state no backward; this is the gradient of the exact attention they
    define (training runs both passes: the DeepSpeed-Ulysses / ring-flash-
    attention how-to (2kiu.com), §4 "启动命令与显存吞吐验证", checks memory
    after the forward and after the backward).  Returns dQ [Sq, Hq, dh],
    dK, dV [Sk, Hkv, dh]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    sq, hq, dh = q.shape
    sk, hkv, _ = k.shape
    group = hq // hkv
    if scale is None:
        scale = 1.0 / math.sqrt(dh)
    qpos = np.arange(sq) if qpos is None else np.asarray(qpos)
    kpos = np.arange(sk) if kpos is None else np.asarray(kpos)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for r0 in range(0, sq, row_block):
        r1 = min(sq, r0 + row_block)
        mask = explicit_mask(qpos[r0:r1], kpos, causal, cu_seqlens)
        live = mask.any(axis=1)
        for h in range(hq):
            g = h // group
            s = np.where(mask, (q[r0:r1, h, :] @ k[:, g, :].T) * scale, NEG_INF)
            m = np.where(live, np.max(s, axis=1, initial=NEG_INF), 0.0)
            e = np.where(mask, np.exp(s - m[:, None]), 0.0)
            l = np.where(live, e.sum(axis=1), 1.0)
            p = e / l[:, None]
            dp = do[r0:r1, h, :] @ v[:, g, :].T
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            dv[:, g, :] += p.T @ do[r0:r1, h, :]
            dq[r0:r1, h, :] = scale * (ds @ k[:, g, :])
            dk[:, g, :] += scale * (ds.T @ q[r0:r1, h, :])
    return dq, dk, dv


def ring_attention_bwd(q, k, v, do, S, P, layout, causal=True, cu_seqlens=None, scale=None):
    """Ring backward over P virtual ranks: the forward's merged O and LSE of
    each rank are kept; at ring step t rank r holds KV shard j = (r - t) mod P
    and, with P_rj = exp(scale Q_r K_j^T - LSE_r) (the merged LSE, so P_rj is
    the true slice of the global probabilities) and D_r = rowsum(dO_r * O_r),
        dS_rj = P_rj * (dO_r V_j^T - D_r),
        dQ_r += scale dS_rj K_j,  dK_j += scale dS_rj^T Q_r,  dV_j += P_rj^T dO_r,
    the KV gradients travelling with their shard.  Inputs q, k, v, do in
    natural order; outputs in rank-major storage order (dQ [S, Hq, dh],
    dK, dV [S, Hkv, dh])."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    hq, dh = q.shape[1], q.shape[2]
    hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(dh)
    o_all, lse_all = ring_attention(q, k, v, S, P, layout, causal, cu_seqlens, scale)
    pos = [shard_positions(S, P, layout, r) for r in range(P)]
    n = pos[0].size
    dq = [np.zeros((n, hq, dh)) for _ in range(P)]
    dk = [np.zeros((n, hkv, dh)) for _ in range(P)]
    dv = [np.zeros((n, hkv, dh)) for _ in range(P)]
    for t in range(P):
        for r in range(P):
            j = ring_source(r, t, P)
            qp, kp = pos[r], pos[j]
            o_r = o_all[r * n:(r + 1) * n]
            lse_r = lse_all[:, r * n:(r + 1) * n]
            gq, gk, gv = ring_pair_bwd(q[qp], k[kp], v[kp], do[qp], o_r, lse_r, qp, kp, causal, cu_seqlens, scale)
            dq[r] += gq
            dk[j] += gk
            dv[j] += gv
    return np.concatenate(dq), np.concatenate(dk), np.concatenate(dv)


def ring_pair_bwd(q_r, k_j, v_j, do_r, o_r, lse_r, qpos, kpos, causal=True, cu_seqlens=None, scale=None,
                  d_r=None):
    """One ring step of the backward: the contributions of block pair (r, j)
    to dQ_r, dK_j and dV_j, from rank r's rows q_r, do_r [n_q, Hq, dh], its
    merged forward o_r [n_q, Hq, dh] and lse_r [Hq, n_q], and shard j's k_j,
    v_j [n_k, Hkv, dh]; qpos, kpos are the rows' global positions.  With
    P_rj = exp(scale Q_r K_j^T - LSE_r) on the admitted pairs and
    D_r = rowsum(dO_r * O_r):  dS = P_rj * (dO_r V_j^T - D_r),
    dQ = scale dS K_j, dK = scale dS^T Q_r, dV = P_rj^T dO_r (GQA: summed over
    the query heads of each KV head).  d_r [Hq, n_q], when given, is D_r
    itself and o_r is not read."""
    q_r, k_j, v_j, do_r, lse_r = (np.asarray(a, dtype=np.float64) for a in (q_r, k_j, v_j, do_r, lse_r))
    if d_r is None:
        d_r = (do_r * np.asarray(o_r, dtype=np.float64)).sum(axis=2).T
    d_r = np.asarray(d_r, dtype=np.float64)
    hq, dh = q_r.shape[1], q_r.shape[2]
    group = hq // k_j.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(dh)
    mask = explicit_mask(np.asarray(qpos), np.asarray(kpos), causal, cu_seqlens)
    dq = np.zeros(q_r.shape)
    dk = np.zeros(k_j.shape)
    dv = np.zeros(v_j.shape)
    for h in range(hq):
        g = h // group
        s = (q_r[:, h, :] @ k_j[:, g, :].T) * scale
        lse_h = np.where(np.isfinite(lse_r[h]), lse_r[h], 0.0)
        p = np.where(mask, np.exp(s - lse_h[:, None]), 0.0)
        ds = p * (do_r[:, h, :] @ v_j[:, g, :].T - d_r[h][:, None])
        dq[:, h, :] += scale * (ds @ k_j[:, g, :])
        dk[:, g, :] += scale * (ds.T @ q_r[:, h, :])
        dv[:, g, :] += p.T @ do_r[:, h, :]
    return dq, dk, dv


def live_pair_count(S, causal=True, cu_seqlens=None, qpos=None, kpos=None):
    """Brute-force count of admitted (q, k) pairs (explicit mask summed)."""
    qpos = np.arange(S) if qpos is None else np.asarray(qpos)
    kpos = np.arange(S) if kpos is None else np.asarray(kpos)
    total = 0
    for r0 in range(0, qpos.size, 1024):
        total += int(explicit_mask(qpos[r0:r0 + 1024], kpos, causal, cu_seqlens).sum())
    return total


def pair_classes(S, P, layout, causal=True, cu_seqlens=None):
    """For every (rank r, step t): (j, live count, total count) of the block
    pair, by brute force over the explicit mask."""
    out = {}
    for r in range(P):
        for t in range(P):
            j = ring_source(r, t, P)
            qp = shard_positions(S, P, layout, r)
            kp = shard_positions(S, P, layout, j)
            live = live_pair_count(S, causal, cu_seqlens, qp, kp)
            out[(r, t)] = (j, live, qp.size * kp.size)
    return out
