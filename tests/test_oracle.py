"""Pins for the fp64 oracle: closed forms, invariants, brute force and a library
special case.  None of these re-types the oracle's own formula; each is chosen
so that a dropped term, a wrong sign, a wrong scale or a transposed index fails
at least one of them.  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


def randn(*shape):
    return rng.standard_normal(shape)


# ---------------------------------------------------------------- closed forms
def test_golden_identical_keys_causal():
    with open(os.path.join(GOLDEN, "identical_keys_causal.json")) as f:
        g = json.load(f)
    o, lse = ref.attention(np.array(g["q"], float), np.array(g["k"], float),
                           np.array(g["v"], float), causal=g["causal"])
    np.testing.assert_allclose(o, np.array(g["expected_o"], float), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, np.array(g["expected_lse"], float), rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [True, False])
def test_identical_keys_give_mean_of_v(causal):
    S, H, dh = 37, 3, 8
    q = randn(S, H, dh)
    kvec = randn(1, H, dh)
    k = np.repeat(kvec, S, axis=0)
    v = randn(S, H, dh)
    o, lse = ref.attention(q, k, v, causal=causal)
    scale = 1 / math.sqrt(dh)
    for i in range(S):
        n = i + 1 if causal else S
        for h in range(H):
            np.testing.assert_allclose(o[i, h], v[:n, h].mean(axis=0), atol=1e-12)
            s = scale * float(q[i, h] @ kvec[0, h])
            assert abs(lse[h, i] - (s + math.log(n))) < 1e-12


def test_causal_row_zero_is_v0():
    S, H, dh = 16, 2, 16
    q, k, v = randn(S, H, dh), randn(S, H, dh), randn(S, H, dh)
    o, lse = ref.attention(q, k, v, causal=True)
    np.testing.assert_allclose(o[0], v[0], atol=1e-14)
    for h in range(H):
        assert abs(lse[h, 0] - float(q[0, h] @ k[0, h]) / 4.0) < 1e-14


def test_zero_queries_give_uniform_mean():
    S, H, dh = 20, 2, 8
    q = np.zeros((S, H, dh))
    k, v = randn(S, H, dh), randn(S, H, dh)
    o, lse = ref.attention(q, k, v, causal=True)
    for i in range(S):
        np.testing.assert_allclose(o[i], v[:i + 1].mean(axis=0), atol=1e-13)
        np.testing.assert_allclose(lse[:, i], math.log(i + 1), atol=1e-14)


def test_onehot_values_give_probabilities():
    # V_j = e_j: O[i] is the probability row of query i: non-negative, sums to
    # one, zero on keys the causal mask excludes.
    S, dh = 32, 32
    q, k = randn(S, 1, dh), randn(S, 1, dh)
    v = np.eye(S).reshape(S, 1, dh)
    o, _ = ref.attention(q, k, v, causal=True)
    p = o[:, 0, :]
    assert np.all(p >= 0)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)
    assert np.all(np.triu(p, 1) == 0)


def test_lse_bounds():
    S, H, dh = 64, 2, 16
    q, k, v = randn(S, H, dh), randn(S, H, dh), randn(S, H, dh)
    _, lse = ref.attention(q, k, v, causal=True)
    for h in range(H):
        s = q[:, h] @ k[:, h].T / 4.0
        for i in range(S):
            mx = s[i, :i + 1].max()
            assert mx - 1e-12 <= lse[h, i] <= mx + math.log(i + 1) + 1e-12


# ------------------------------------------------------------- brute force
def _scalar_attention(q, k, v, causal, scale, docs=None):
    """Triple loop with math.exp, no numpy linear algebra."""
    S, Hq, dh = q.shape
    Hkv = k.shape[1]
    o = [[[0.0] * dh for _ in range(Hq)] for _ in range(S)]
    lse = [[-math.inf] * S for _ in range(Hq)]
    for h in range(Hq):
        g = h // (Hq // Hkv)
        for i in range(S):
            scores = []
            for j in range(S):
                if causal and j > i:
                    continue
                if docs is not None and docs[i] != docs[j]:
                    continue
                s = 0.0
                for d in range(dh):
                    s += float(q[i, h, d]) * float(k[j, g, d])
                scores.append((j, s * scale))
            if not scores:
                continue
            m = max(s for _, s in scores)
            den = sum(math.exp(s - m) for _, s in scores)
            for d in range(dh):
                o[i][h][d] = sum(math.exp(s - m) * float(v[j, g, d]) for j, s in scores) / den
            lse[h][i] = m + math.log(den)
    return np.array(o), np.array(lse)


@pytest.mark.parametrize("causal", [True, False])
def test_bruteforce_gqa(causal):
    S, Hq, Hkv, dh = 19, 4, 2, 5
    q, k, v = randn(S, Hq, dh), randn(S, Hkv, dh), randn(S, Hkv, dh)
    o, lse = ref.attention(q, k, v, causal=causal, row_block=7)
    o2, lse2 = _scalar_attention(q, k, v, causal, 1 / math.sqrt(dh))
    np.testing.assert_allclose(o, o2, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, atol=1e-12)


def test_bruteforce_varlen():
    S, H, dh = 24, 2, 4
    cu = [0, 5, 6, 17, 24]
    docs = [int(np.searchsorted(cu, i, side="right") - 1) for i in range(S)]
    q, k, v = randn(S, H, dh), randn(S, H, dh), randn(S, H, dh)
    o, lse = ref.attention(q, k, v, causal=True, cu_seqlens=cu)
    o2, lse2 = _scalar_attention(q, k, v, True, 0.5, docs)
    np.testing.assert_allclose(o, o2, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, atol=1e-12)


def test_seq_equals_cp_size_one_token_per_rank():
    # pwwt.cn Context Parallelism write-up §5.2: sequence length = CP size, one
    # token per rank, checked element by element against a hand computation.
    P = 4
    dh = 3
    q, k, v = randn(P, 1, dh), randn(P, 1, dh), randn(P, 1, dh)
    o, lse = ref.ring_attention(q, k, v, P, P, "contiguous", causal=True)
    o2, lse2 = _scalar_attention(q, k, v, True, 1 / math.sqrt(dh))
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, atol=1e-13)


# ------------------------------------------------------ library special case
def test_matches_torch_sdpa_fp64_with_bool_mask():
    S, Hq, Hkv, dh = 300, 4, 2, 32
    q, k, v = randn(S, Hq, dh), randn(S, Hkv, dh), randn(S, Hkv, dh)
    cu = [0, 40, 41, 200, 300]
    o, lse = ref.attention(q, k, v, causal=True, cu_seqlens=cu)
    docs = np.searchsorted(cu, np.arange(S), side="right") - 1
    mask = (np.arange(S)[None, :] <= np.arange(S)[:, None]) & (docs[:, None] == docs[None, :])
    tq = torch.from_numpy(q).permute(1, 0, 2)
    tk = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
    tv = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
    ot = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(mask))
    np.testing.assert_allclose(o, ot.permute(1, 0, 2).numpy(), atol=1e-12)
    s = torch.einsum("hqd,hkd->hqk", tq, tk) / math.sqrt(dh)
    lt = torch.logsumexp(s.masked_fill(~torch.from_numpy(mask), -math.inf), dim=-1)
    np.testing.assert_allclose(lse, lt.numpy(), atol=1e-12)


# ------------------------------------------------------------- invariants
@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "striped"])
@pytest.mark.parametrize("P", [1, 2, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_split_then_merge_equals_unsplit(layout, P, causal):
    # compassingai §二: the block recurrence is exact, so merging the P ring
    # steps of every rank reproduces unsplit attention.
    S, Hq, Hkv, dh = 48, 4, 2, 8
    q, k, v = randn(S, Hq, dh), randn(S, Hkv, dh), randn(S, Hkv, dh)
    o, lse = ref.attention(q, k, v, causal=causal)
    o_r, lse_r = ref.ring_attention(q, k, v, S, P, layout, causal=causal)
    order = np.concatenate([ref.shard_positions(S, P, layout, r) for r in range(P)])
    np.testing.assert_allclose(o_r, o[order], atol=1e-12)
    np.testing.assert_allclose(lse_r, lse[:, order], atol=1e-12)


def test_split_invariance_varlen_zigzag():
    S, H, dh, P = 64, 2, 8, 4
    cu = [0, 3, 30, 31, 64]
    q, k, v = randn(S, H, dh), randn(S, H, dh), randn(S, H, dh)
    o, lse = ref.attention(q, k, v, causal=True, cu_seqlens=cu)
    o_r, lse_r = ref.ring_attention(q, k, v, S, P, "zigzag", causal=True, cu_seqlens=cu)
    order = ref.zigzag_order(S, P)
    np.testing.assert_allclose(o_r, o[order], atol=1e-12)
    np.testing.assert_allclose(lse_r, lse[:, order], atol=1e-12)


def test_varlen_equals_separate_documents():
    S, H, dh = 50, 2, 8
    cu = [0, 7, 8, 33, 50]
    q, k, v = randn(S, H, dh), randn(S, H, dh), randn(S, H, dh)
    o, lse = ref.attention(q, k, v, causal=True, cu_seqlens=cu)
    for a, b in zip(cu[:-1], cu[1:]):
        od, ld = ref.attention(q[a:b], k[a:b], v[a:b], causal=True)
        np.testing.assert_allclose(o[a:b], od, atol=1e-12)
        np.testing.assert_allclose(lse[:, a:b], ld, atol=1e-12)


def test_varlen_single_document_is_plain_causal():
    S, H, dh = 40, 2, 8
    q, k, v = randn(S, H, dh), randn(S, H, dh), randn(S, H, dh)
    o1, l1 = ref.attention(q, k, v, causal=True)
    o2, l2 = ref.attention(q, k, v, causal=True, cu_seqlens=[0, S])
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_merge_edge_cases():
    rows, H, dh = 5, 2, 3
    o1, l1 = randn(rows, H, dh), randn(H, rows)
    o, l = ref.lse_merge(o1[None], l1[None])
    np.testing.assert_allclose(o, o1, atol=1e-15)
    np.testing.assert_allclose(l, l1, atol=1e-15)
    # a -inf partial with garbage O contributes nothing
    bad = np.full_like(o1, np.nan)
    o, l = ref.lse_merge(np.stack([o1, bad]), np.stack([l1, np.full_like(l1, -np.inf)]))
    np.testing.assert_allclose(o, o1, atol=1e-15)
    np.testing.assert_allclose(l, l1, atol=1e-15)
    # two equal partials: same O, LSE + ln 2
    o, l = ref.lse_merge(np.stack([o1, o1]), np.stack([l1, l1]))
    np.testing.assert_allclose(o, o1, atol=1e-14)
    np.testing.assert_allclose(l, l1 + math.log(2), atol=1e-14)
    # all -inf: zero output
    o, l = ref.lse_merge(np.stack([o1, o1]), np.full((2, H, rows), -np.inf))
    assert np.all(o == 0) and np.all(np.isneginf(l))


# ------------------------------------------------------------- layouts
def test_zigzag_order_by_hand():
    # S=16, P=2: chunks of 4; rank 0 = chunks 0, 3; rank 1 = chunks 1, 2
    assert list(ref.zigzag_order(16, 2)) == [0, 1, 2, 3, 12, 13, 14, 15, 4, 5, 6, 7, 8, 9, 10, 11]


def test_striped_order_by_hand():
    # S=8, P=2: rank 0 holds even positions, rank 1 odd ones
    assert list(ref.striped_order(8, 2)) == [0, 2, 4, 6, 1, 3, 5, 7]
    assert sorted(ref.striped_order(48, 4)) == list(range(48))


def test_striped_pairs_are_balanced_local_causal_blocks():
    # every striped block pair is a local causal block: n(n+1)/2 admitted
    # pairs for j <= r and n(n-1)/2 for j > r
    S, P = 64, 4
    n = S // P
    for (r, t), (j, live, tot) in ref.pair_classes(S, P, "striped").items():
        assert live == (n * (n + 1) // 2 if j <= r else n * (n - 1) // 2)


def test_zigzag_round_trip_and_permutation():
    x = randn(64, 3, 2)
    y = ref.zigzag_reorder(x, 4)
    assert sorted(ref.zigzag_order(64, 4)) == list(range(64))
    np.testing.assert_array_equal(ref.zigzag_restore(y, 4), x)
    lse = randn(3, 64)
    np.testing.assert_array_equal(ref.zigzag_restore(ref.zigzag_reorder(lse, 4, axis=1), 4, axis=1), lse)


def test_ulysses_index_formula_by_loops():
    P, n, H, dh = 3, 4, 6, 2
    x = randn(P, n, H, dh)
    y = ref.ulysses_seq_to_head(x, P)
    hg = H // P
    assert y.shape == (P, P * n, hg, dh)
    for r in range(P):
        for p in range(P):
            for s in range(n):
                for hh in range(hg):
                    for d in range(dh):
                        assert y[r, p * n + s, hh, d] == x[p, s, r * hg + hh, d]
    np.testing.assert_array_equal(ref.ulysses_head_to_seq(y, P), x)
    np.testing.assert_array_equal(ref.ulysses_seq_to_head(x[:1], 1)[0], x[0])


def test_ulysses_composite_equals_attention():
    # compassingai §三: permute seq->head, full-sequence attention per head
    # block, permute back == attention on the unsplit sequence (GQA 4:2, P=2).
    P, S, Hq, Hkv, dh = 2, 24, 4, 2, 4
    q, k, v = randn(S, Hq, dh), randn(S, Hkv, dh), randn(S, Hkv, dh)
    o, lse = ref.attention(q, k, v, causal=True)
    n = S // P
    qh = ref.ulysses_seq_to_head(q.reshape(P, n, Hq, dh), P)
    kh = ref.ulysses_seq_to_head(k.reshape(P, n, Hkv, dh), P)
    vh = ref.ulysses_seq_to_head(v.reshape(P, n, Hkv, dh), P)
    oh = np.stack([ref.attention(qh[r], kh[r], vh[r], causal=True)[0] for r in range(P)])
    back = ref.ulysses_head_to_seq(oh, P).reshape(S, Hq, dh)
    np.testing.assert_allclose(back, o, atol=1e-12)


def _storage_order(S, P, layout):
    return np.concatenate([ref.shard_positions(S, P, layout, r) for r in range(P)])


@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "striped"])
@pytest.mark.parametrize("Pr,Pu", [(2, 2), (4, 2), (2, 4), (1, 4), (3, 2)])
@pytest.mark.parametrize("causal", [True, False])
def test_usp_equals_unsplit_attention(layout, Pr, Pu, causal):
    # The hybrid is exact (compassingai §二: the block recurrence loses
    # nothing), so in storage order it must equal attention of the whole
    # sequence.  GQA 8:4, so each Ulysses head block has its own KV heads.
    S, Hq, Hkv, dh = 48, 8, 4, 8
    q, k, v = randn(S, Hq, dh), randn(S, Hkv, dh), randn(S, Hkv, dh)
    o, lse = ref.attention(q, k, v, causal=causal)
    o_u, lse_u = ref.usp_attention(q, k, v, S, Pr, Pu, layout, causal=causal)
    order = _storage_order(S, Pr, layout)
    np.testing.assert_allclose(o_u, o[order], atol=1e-12)
    np.testing.assert_allclose(lse_u, lse[:, order], atol=1e-12)


def test_usp_with_documents_equals_unsplit():
    S, Hq, Hkv, dh, Pr, Pu = 64, 4, 2, 8, 2, 2
    cu = [0, 5, 6, 41, 64]
    q, k, v = randn(S, Hq, dh), randn(S, Hkv, dh), randn(S, Hkv, dh)
    o, lse = ref.attention(q, k, v, causal=True, cu_seqlens=cu)
    o_u, lse_u = ref.usp_attention(q, k, v, S, Pr, Pu, "zigzag", causal=True, cu_seqlens=cu)
    order = _storage_order(S, Pr, "zigzag")
    np.testing.assert_allclose(o_u, o[order], atol=1e-12)
    np.testing.assert_allclose(lse_u, lse[:, order], atol=1e-12)


def test_usp_special_cases_reduce_to_ring_and_ulysses():
    S, Hq, Hkv, dh = 32, 4, 2, 8
    q, k, v = randn(S, Hq, dh), randn(S, Hkv, dh), randn(S, Hkv, dh)
    # Pu = 1: no Ulysses dimension, the hybrid is the plain ring over Pr ranks
    o_u, l_u = ref.usp_attention(q, k, v, S, 4, 1, "zigzag")
    o_r, l_r = ref.ring_attention(q, k, v, S, 4, "zigzag")
    np.testing.assert_allclose(o_u, o_r, atol=1e-12)
    np.testing.assert_allclose(l_u, l_r, atol=1e-12)
    # Pr = 1: no ring dimension, the hybrid is Ulysses over Pu ranks
    P = 2
    n = S // P
    qh = ref.ulysses_seq_to_head(q.reshape(P, n, Hq, dh), P)
    kh = ref.ulysses_seq_to_head(k.reshape(P, n, Hkv, dh), P)
    vh = ref.ulysses_seq_to_head(v.reshape(P, n, Hkv, dh), P)
    oh = np.stack([ref.attention(qh[r], kh[r], vh[r], causal=True)[0] for r in range(P)])
    o_u, _ = ref.usp_attention(q, k, v, S, 1, P, "contiguous")
    np.testing.assert_allclose(o_u, ref.ulysses_head_to_seq(oh, P).reshape(S, Hq, dh), atol=1e-12)


# ------------------------------------------------------ backward
def _torch_grads(q, k, v, do, causal, cu=None, scale=None):
    """Gradients by torch autograd (fp64, CPU) of masked softmax attention
    written with plain torch ops and an explicit boolean mask."""
    S, hq, dh = q.shape
    hkv = k.shape[1]
    scale = 1.0 / math.sqrt(dh) if scale is None else scale
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    mask = torch.from_numpy(ref.explicit_mask(np.arange(S), np.arange(k.shape[0]), causal, cu))
    kk = tk.repeat_interleave(hq // hkv, dim=1)
    vv = tv.repeat_interleave(hq // hkv, dim=1)
    s = torch.einsum("qhd,khd->hqk", tq, kk) * scale
    s = s.masked_fill(~mask[None], float("-inf"))
    o = torch.einsum("hqk,khd->qhd", torch.softmax(s, dim=-1), vv)
    o.backward(torch.tensor(do, dtype=torch.float64))
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("causal", [True, False])
def test_bwd_matches_torch_autograd(causal):
    S, hq, hkv, dh = 40, 4, 2, 8
    q, k, v, do = randn(S, hq, dh), randn(S, hkv, dh), randn(S, hkv, dh), randn(S, hq, dh)
    cu = [0, 9, 10, 40]
    for docs in (None, cu):
        got = ref.attention_bwd(q, k, v, do, causal=causal, cu_seqlens=docs)
        want = _torch_grads(q, k, v, do, causal, docs)
        for g, w in zip(got, want):
            np.testing.assert_allclose(g, w, atol=1e-12)


def test_bwd_matches_finite_differences():
    # central differences of L = sum(dO * O) on a tiny causal GQA case
    S, hq, hkv, dh = 6, 2, 1, 3
    q, k, v, do = randn(S, hq, dh), randn(S, hkv, dh), randn(S, hkv, dh), randn(S, hq, dh)
    dq, dk, dv = ref.attention_bwd(q, k, v, do, causal=True)
    loss = lambda a, b, c: float((ref.attention(a, b, c, causal=True)[0] * do).sum())
    eps = 1e-6
    for x, g, idx in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        for i in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[i] += eps
            xm[i] -= eps
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[idx], args_m[idx] = xp, xm
            num[i] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-7)


def test_bwd_closed_forms_and_invariants():
    S, hq, hkv, dh = 32, 4, 2, 8
    q, k, v, do = randn(S, hq, dh), randn(S, hkv, dh), randn(S, hkv, dh), randn(S, hq, dh)
    dq, dk, dv = ref.attention_bwd(q, k, v, do, causal=True)
    # every row of dS sums to zero, so the key gradients of a KV head sum to 0
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-10)
    # every row of P sums to one, so the value gradients of a KV head sum to
    # the upstream gradients of its query heads
    want = do.reshape(S, hkv, hq // hkv, dh).sum(axis=(0, 2))
    np.testing.assert_allclose(dv.sum(axis=0), want, atol=1e-10)
    # causal row 0 sees only key 0: its softmax is constant, so dQ_0 = 0
    np.testing.assert_allclose(dq[0], 0.0, atol=1e-12)
    # identical keys: P is uniform over the live keys whatever q is, so dQ = 0
    k1 = np.repeat(randn(1, hkv, dh), S, axis=0)
    dq1, _, _ = ref.attention_bwd(q, k1, v, do, causal=True)
    np.testing.assert_allclose(dq1, 0.0, atol=1e-12)


@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "striped"])
@pytest.mark.parametrize("P", [1, 2, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_bwd_equals_unsplit(layout, P, causal):
    # the ring form with the merged LSE is exact: it equals the gradient of
    # the unsplit attention, in storage order
    S, hq, hkv, dh = 32, 4, 2, 8
    q, k, v, do = randn(S, hq, dh), randn(S, hkv, dh), randn(S, hkv, dh), randn(S, hq, dh)
    dq, dk, dv = ref.attention_bwd(q, k, v, do, causal=causal)
    rq, rk, rv = ref.ring_attention_bwd(q, k, v, do, S, P, layout, causal=causal)
    order = _storage_order(S, P, layout)
    np.testing.assert_allclose(rq, dq[order], atol=1e-12)
    np.testing.assert_allclose(rk, dk[order], atol=1e-12)
    np.testing.assert_allclose(rv, dv[order], atol=1e-12)


def test_ring_bwd_with_documents_equals_unsplit():
    S, hq, hkv, dh, P = 64, 2, 2, 8, 4
    cu = [0, 3, 30, 31, 64]
    q, k, v, do = randn(S, hq, dh), randn(S, hkv, dh), randn(S, hkv, dh), randn(S, hq, dh)
    dq, dk, dv = ref.attention_bwd(q, k, v, do, causal=True, cu_seqlens=cu)
    rq, rk, rv = ref.ring_attention_bwd(q, k, v, do, S, P, "zigzag", causal=True, cu_seqlens=cu)
    order = _storage_order(S, P, "zigzag")
    for a, b in ((rq, dq), (rk, dk), (rv, dv)):
        np.testing.assert_allclose(a, b[order], atol=1e-12)


def test_ring_pair_bwd_single_pair_is_whole_gradient_and_takes_d():
    # one pair covering every row and key is the whole gradient (pinned
    # against autograd above); passing D = rowsum(dO * O) directly changes
    # nothing; a pair that admits no (q, k) gives exactly zero
    S, hq, hkv, dh = 24, 4, 2, 8
    q, k, v, do = randn(S, hq, dh), randn(S, hkv, dh), randn(S, hkv, dh), randn(S, hq, dh)
    o, lse = ref.attention(q, k, v, causal=True)
    pos = np.arange(S)
    want = ref.attention_bwd(q, k, v, do, causal=True)
    got = ref.ring_pair_bwd(q, k, v, do, o, lse, pos, pos, causal=True)
    d = np.einsum("shc,shc->hs", do, o)
    got_d = ref.ring_pair_bwd(q, k, v, do, None, lse, pos, pos, causal=True, d_r=d)
    for a, b, c in zip(got, got_d, want):
        np.testing.assert_allclose(a, c, atol=1e-12)
        np.testing.assert_allclose(a, b, atol=1e-13)  # D summed in another order
    # queries 0..7 against keys 16..23 under causal: nothing admitted
    zero = ref.ring_pair_bwd(q[:8], k[16:], v[16:], do[:8], o[:8], lse[:, :8], pos[:8], pos[16:], causal=True)
    assert all(not np.any(z) for z in zero)


# ------------------------------------------------------ work counts
def test_live_pair_counts_closed_forms():
    S = 96
    assert ref.live_pair_count(S, causal=True) == S * (S + 1) // 2
    assert ref.live_pair_count(S, causal=False) == S * S
    cu = [0, 10, 11, 60, 96]
    lens = np.diff(cu)
    assert ref.live_pair_count(S, True, cu) == int(sum(L * (L + 1) // 2 for L in lens))


def test_pair_classes_contiguous_and_zigzag():
    S, P = 64, 4
    n = S // P
    cls = ref.pair_classes(S, P, "contiguous")
    for (r, t), (j, live, tot) in cls.items():
        assert j == (r - t) % P
        assert live == (n * n if j < r else (n * (n + 1) // 2 if j == r else 0))
    c = S // (2 * P)
    cls = ref.pair_classes(S, P, "zigzag")
    for (r, t), (j, live, tot) in cls.items():
        assert live == (2 * c * c + c if j == r else 2 * c * c)


def test_ring_source_hand_table_p3():
    """The rotation of "序列並行" concept page (compassingai), "Ring Attention 的
    不同思路" steps 1-4: every rank starts with its own K/V block and at each
    step passes the block it holds to the next rank and takes the previous
    rank's.  For three ranks, written out by hand (rows: step t, columns: rank
    r, entry: the shard rank r holds)."""
    table = [[0, 1, 2],
             [2, 0, 1],
             [1, 2, 0]]
    for t in range(3):
        for r in range(3):
            assert ref.ring_source(r, t, 3) == table[t][r], (r, t)


def test_ring_source_matches_simulated_message_passing():
    """Pass the blocks around explicitly (rank r sends what it holds to rank
    r + 1 each step) and check that the oracle's schedule names the block each
    rank holds, and that over P steps every rank meets every shard once."""
    for P in range(1, 10):
        held = list(range(P))            # step 0: every rank holds its own shard
        seen = [set() for _ in range(P)]
        for t in range(P):
            for r in range(P):
                assert ref.ring_source(r, t, P) == held[r], (P, r, t)
                seen[r].add(held[r])
            nxt = [None] * P
            for r in range(P):
                nxt[(r + 1) % P] = held[r]   # send to the next rank
            held = nxt
        assert all(sv == set(range(P)) for sv in seen)


# ------------------------------------------------- planted mistakes are caught
def test_pins_catch_planted_mistakes(monkeypatch):
    """Plant plausible mistakes in the oracle (on the CPU) and check that the
    pins above fail for each."""
    S, H, dh = 12, 1, 4
    q = np.zeros((S, H, dh))
    k, v = randn(S, H, dh), randn(S, H, dh)
    good_o, _ = ref.attention(q, k, v, causal=True)

    orig = ref.explicit_mask

    def off_by_one(qpos, kpos, causal, cu_seqlens=None):
        m = orig(qpos, kpos, causal, cu_seqlens)
        if causal:
            m &= np.asarray(kpos)[None, :] < np.asarray(qpos)[:, None] + 0  # drops the diagonal
            m[:, 0] = True
        return m

    monkeypatch.setattr(ref, "explicit_mask", off_by_one)
    bad_o, _ = ref.attention(q, k, v, causal=True)
    monkeypatch.setattr(ref, "explicit_mask", orig)
    # the zero-query closed form (uniform mean over keys 0..i) rejects it
    assert not np.allclose(bad_o[3], v[:4].mean(axis=0), atol=1e-9)
    np.testing.assert_allclose(good_o[3], v[:4].mean(axis=0), atol=1e-13)

    # wrong scale (1/dh instead of 1/sqrt(dh)) is caught by causal row 0
    q2, k2 = randn(S, H, dh), randn(S, H, dh)
    _, lse_bad = ref.attention(q2, k2, v, causal=True, scale=1.0 / dh)
    assert abs(lse_bad[0, 0] - float(q2[0, 0] @ k2[0, 0]) / 2.0) > 1e-6


def test_bwd_pins_catch_planted_mistakes(monkeypatch):
    """A dropped D term (dS = P * dP) and a transposed GQA sum in the ring
    backward are each caught by a pin above."""
    S, hq, hkv, dh = 16, 2, 1, 4
    q, k, v, do = randn(S, hq, dh), randn(S, hkv, dh), randn(S, hkv, dh), randn(S, hq, dh)
    # (1) without the rowsum term the key gradients no longer sum to zero
    orig_exp = np.exp

    def bwd_no_d(q, k, v, do, causal=True):
        sc = 1.0 / math.sqrt(dh)
        mask = ref.explicit_mask(np.arange(S), np.arange(S), causal)
        dk = np.zeros_like(k)
        for h in range(hq):
            s = np.where(mask, (q[:, h] @ k[:, 0].T) * sc, -np.inf)
            p = orig_exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            ds = p * (do[:, h] @ v[:, 0].T)          # planted: D dropped
            dk[:, 0] += sc * ds.T @ q[:, h]
        return dk

    assert np.abs(bwd_no_d(q, k, v, do).sum(axis=0)).max() > 1e-6
    assert np.abs(ref.attention_bwd(q, k, v, do)[1].sum(axis=0)).max() < 1e-10
    # (2) a ring backward whose P uses a wrong normaliser (LSE off by ln 2)
    # no longer equals the unsplit gradient
    o_all, lse_all = ref.ring_attention(q, k, v, S, 2, "contiguous")
    monkeypatch.setattr(ref, "ring_attention",
                        lambda *a, **kw: (o_all, lse_all - np.log(2.0)))  # planted: wrong normaliser
    bad = ref.ring_attention_bwd(q, k, v, do, S, 2, "contiguous")
    monkeypatch.undo()
    good = ref.attention_bwd(q, k, v, do)
    assert not np.allclose(bad[0], good[0], atol=1e-6)
