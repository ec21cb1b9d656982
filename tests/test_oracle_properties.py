"""Randomised (hypothesis) checks of the oracle's exactness claims: for random
shard counts, layouts, masks, GQA ratios and document tables, the ring form
(partials per ring step folded by the LSE merge), its backward with the merged
LSE, and the Ulysses-inside / Ring-across hybrid all equal the unsplit
attention (or its gradient) in the ranks' storage order, to fp64 rounding.
The unsplit attention and gradient are themselves pinned against closed forms,
brute force and torch autograd in test_oracle.py."""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import ref


def _order(S, P, layout):
    return np.concatenate([ref.shard_positions(S, P, layout, r) for r in range(P)])


@st.composite
def problems(draw, hybrid=False):
    layout = draw(st.sampled_from(["contiguous", "zigzag", "striped"]))
    if hybrid:
        Pr = draw(st.integers(1, 3))
        Pu = draw(st.sampled_from([1, 2]))
        P = Pr
    else:
        P = draw(st.integers(1, 5))
        Pr = Pu = None
    unit = (2 * P if layout == "zigzag" else P) * (Pu or 1)
    S = unit * draw(st.integers(1, max(1, 48 // unit)))
    hkv = draw(st.sampled_from([1, 2]))
    if hybrid and hkv % Pu:
        hkv = Pu
    group = draw(st.sampled_from([1, 2]))
    causal = draw(st.booleans())
    cu = None
    if layout != "striped" and draw(st.booleans()):
        cuts = sorted(set(draw(st.lists(st.integers(1, S - 1), max_size=4)))) if S > 1 else []
        cu = [0] + cuts + [S]
    seed = draw(st.integers(0, 2**31 - 1))
    return dict(layout=layout, P=P, Pr=Pr, Pu=Pu, S=S, hq=hkv * group, hkv=hkv, causal=causal, cu=cu, seed=seed)


def _qkv(p, dh=4):
    g = np.random.default_rng(p["seed"])
    S = p["S"]
    return (g.standard_normal((S, p["hq"], dh)), g.standard_normal((S, p["hkv"], dh)),
            g.standard_normal((S, p["hkv"], dh)), g.standard_normal((S, p["hq"], dh)))


@settings(max_examples=40, deadline=None)
@given(problems())
def test_ring_forward_is_exact(p):
    q, k, v, _ = _qkv(p)
    o, lse = ref.attention(q, k, v, causal=p["causal"], cu_seqlens=p["cu"])
    ro, rl = ref.ring_attention(q, k, v, p["S"], p["P"], p["layout"], p["causal"], p["cu"])
    order = _order(p["S"], p["P"], p["layout"])
    np.testing.assert_allclose(ro, o[order], atol=1e-12)
    fin = np.isfinite(lse[:, order])
    assert np.array_equal(np.isfinite(rl), fin)
    np.testing.assert_allclose(rl[fin], lse[:, order][fin], atol=1e-12)


@settings(max_examples=30, deadline=None)
@given(problems())
def test_ring_backward_is_exact(p):
    q, k, v, do = _qkv(p)
    want = ref.attention_bwd(q, k, v, do, causal=p["causal"], cu_seqlens=p["cu"])
    got = ref.ring_attention_bwd(q, k, v, do, p["S"], p["P"], p["layout"], p["causal"], p["cu"])
    order = _order(p["S"], p["P"], p["layout"])
    for a, b in zip(got, want):
        np.testing.assert_allclose(a, b[order], atol=1e-11)


@settings(max_examples=30, deadline=None)
@given(problems(hybrid=True))
def test_hybrid_forward_is_exact(p):
    q, k, v, _ = _qkv(p)
    o, lse = ref.attention(q, k, v, causal=p["causal"], cu_seqlens=p["cu"])
    uo, ul = ref.usp_attention(q, k, v, p["S"], p["Pr"], p["Pu"], p["layout"], p["causal"], p["cu"])
    order = _order(p["S"], p["Pr"], p["layout"])
    np.testing.assert_allclose(uo, o[order], atol=1e-12)
    fin = np.isfinite(lse[:, order])
    np.testing.assert_allclose(ul[fin], lse[:, order][fin], atol=1e-12)
