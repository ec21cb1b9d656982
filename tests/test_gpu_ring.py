"""GPU parity of the whole ring forward (schedule -> block attention ->
merge) and of the Ulysses path against the fp64 oracle: exhaustively at
sizes the oracle finishes in seconds, and on sampled rows at the full
workload sizes."""
import numpy as np
import pytest
import torch

from context_exact_attention_step_b200 import api, synth
from oracle import ref

from _util import compare, f64

pytestmark = pytest.mark.gpu


def natural_order(S, P, layout):
    return np.concatenate([ref.shard_positions(S, P, layout, r) for r in range(P)])


def ring_case(S, hq, hkv, dh, P, layout, causal=True, cu=None, std=0.5, dtype=torch.bfloat16):
    q, k, v = synth.qkv(S, hq, hkv, dh, std=std, dtype=dtype)
    order = natural_order(S, P, layout)
    qs, ks, vs = (t[torch.from_numpy(order)].contiguous().cuda() for t in (q, k, v))
    o, lse = api.ring_attn_fwd(qs, ks, vs, P, layout, causal, cu)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    # the kernel consumes bf16-rounded values; so does the oracle
    r16 = lambda t: f64(t.to(torch.bfloat16))
    want_o, want_l = ref.attention(r16(q), r16(k), r16(v), causal=causal, cu_seqlens=cu)
    return compare(o, lse, want_o[order], want_l[:, order], what=f"S={S} P={P} {layout}")


def test_tiny_fp32_contiguous_full():
    # B=1, H=4, dh=64, S=1024, P=4 contiguous, causal, fp32 N(0,1) inputs
    ring_case(1024, 4, 4, 64, 4, "contiguous", std=1.0, dtype=torch.float32)


@pytest.mark.parametrize("P", [1, 2, 4, 8])
def test_contiguous_small(P):
    ring_case(2048, 2, 2, 128, P, "contiguous")


@pytest.mark.parametrize("P", [2, 4, 8])
def test_zigzag_small(P):
    ring_case(2048, 2, 1, 128, P, "zigzag")


def test_zigzag_ragged_chunks():
    # chunk of 100 rows: tiles straddle nothing but every tile is partial
    ring_case(800, 2, 2, 64, 4, "zigzag")


def test_noncausal_ring():
    ring_case(1536, 2, 2, 128, 3, "contiguous", causal=False)


def test_varlen_zigzag_small():
    S, P = 4096, 4
    lens = synth.doc_lengths(S, 64, 1024, seed=4)
    cu = synth.cu_seqlens_from_lengths(lens).tolist()
    ring_case(S, 2, 2, 128, P, "zigzag", cu=cu)


@pytest.mark.parametrize("n_docs", [300, 1100])
def test_varlen_many_short_documents(n_docs):
    """Many short documents (random cuts): most block pairs admit nothing
    and the live ones are trimmed to a few rows at shard edges, every key
    tile holds several documents, and with 1100 documents the document table
    is too long for the attention kernel's shared-memory copy, so the kernel
    reads it from global memory."""
    S, P = 8192, 4
    rng = np.random.default_rng(n_docs)
    cuts = np.sort(rng.choice(np.arange(1, S), size=n_docs - 1, replace=False))
    cu = [0] + cuts.tolist() + [S]
    ring_case(S, 2, 2, 64, P, "zigzag", cu=cu)
    ring_case(S, 2, 2, 64, P, "contiguous", cu=cu)


def test_varlen_sixteen_ranks_many_documents():
    """Sixteen zigzag ranks over 1100 short documents: 43 of the 256 block
    pairs are live, each trimmed to the few rows whose documents cross a
    chunk edge, so every rank's rows are cut into many merge tasks with
    different sets of partials."""
    S, P, n_docs = 16384, 16, 1100
    rng = np.random.default_rng(7)
    cuts = np.sort(rng.choice(np.arange(1, S), size=n_docs - 1, replace=False))
    ring_case(S, 2, 2, 64, P, "zigzag", cu=[0] + cuts.tolist() + [S])


def test_seq_equals_cp_size():
    # the pages' mask check: one token per rank
    ring_case(8, 2, 2, 64, 8, "contiguous")
    ring_case(16, 2, 2, 64, 8, "zigzag")


def test_ulysses_small_gqa():
    S, hq, hkv, dh, P = 2048, 8, 4, 128, 4
    q, k, v = synth.qkv(S, hq, hkv, dh)
    o, lse = api.ulysses_attn_fwd(q.cuda(), k.cuda(), v.cuda(), P)
    torch.cuda.synchronize()
    want_o, want_l = ref.attention(f64(q), f64(k), f64(v), causal=True)
    compare(o, lse, want_o, want_l, what="ulysses")


def test_ring_and_ulysses_agree_at_fixed_length():
    """The pages' A/B of Ring and Ulysses at one sequence length: both are
    exact, so on the same inputs they give the same O and LSE (to the
    kernels' rounding) and each matches the oracle."""
    S, hq, hkv, dh, P = 4096, 8, 8, 128, 4
    q, k, v = synth.qkv(S, hq, hkv, dh, seeds=(41, 42, 43))
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o_r, l_r = api.ring_attn_fwd(qd, kd, vd, P, "contiguous", True)
    o_u, l_u = api.ulysses_attn_fwd(qd, kd, vd, P)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    want_o, want_l = ref.attention(f64(q), f64(k), f64(v), causal=True)
    compare(o_r, l_r, want_o, want_l, what="ring")
    compare(o_u, l_u, want_o, want_l, what="ulysses")
    compare(o_r, l_r, f64(o_u), f64(l_u), what="ring vs ulysses")


@pytest.mark.parametrize("P,hkv", [(16, 16), (32, 32)])
def test_ulysses_many_head_groups(P, hkv):
    # every head group is its own block of the attention launch: 16 blocks
    # fill one launch, 32 need two (the plan is split at the block limit),
    # CTAs head-major inside each block
    S, hq, dh = 2048, 32, 64
    q, k, v = synth.qkv(S, hq, hkv, dh, seeds=(31, 32, 33))
    o, lse = api.ulysses_attn_fwd(q.cuda(), k.cuda(), v.cuda(), P)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    want_o, want_l = ref.attention(f64(q), f64(k), f64(v), causal=True)
    compare(o, lse, want_o, want_l, what=f"ulysses P={P}")


# ----------------------------------------------------------- full sizes
def sample_rows(S, P, layout, cu=None, n=192, seed=7):
    """Row 0, the last row, every shard / chunk / document boundary +-1, and
    random rows (natural positions)."""
    rng = np.random.default_rng(seed)
    rows = {0, S - 1}
    bounds = [r * S // P for r in range(P + 1)] + [c * S // (2 * P) for c in range(2 * P + 1)]
    if cu is not None:
        bounds += list(cu)
    for b in bounds:
        for d in (-1, 0, 1):
            if 0 <= b + d < S:
                rows.add(b + d)
    rows |= set(rng.integers(0, S, n).tolist())
    return np.array(sorted(rows))


def full_size_ring(S, hq, hkv, dh, P, layout, cu=None):
    q, k, v = synth.qkv(S, hq, hkv, dh)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    if layout == "zigzag":
        qs, ks, vs = (api.zigzag_reorder(t, P) for t in (qg, kg, vg))
    else:
        qs, ks, vs = qg, kg, vg
    del qg, kg, vg
    o, lse = api.ring_attn_fwd(qs, ks, vs, P, layout, True, cu)
    if layout == "zigzag":
        o = api.zigzag_reorder(o, P, inverse=True)
        lse = api.zigzag_reorder(lse, P, inverse=True, seq_dim=1)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    rows = sample_rows(S, P, layout, cu)
    want_o, want_l = ref.attention(f64(q[torch.from_numpy(rows)]), f64(k), f64(v), causal=True,
                                   cu_seqlens=cu, qpos=rows)
    idx = torch.from_numpy(rows).cuda()
    return compare(o[idx], lse[:, idx], want_o, want_l, what=f"full {layout} S={S}")


def test_full_size_contiguous_32k():
    full_size_ring(32768, 32, 32, 128, 4, "contiguous")


def test_full_size_zigzag_64k():
    full_size_ring(65536, 32, 32, 128, 8, "zigzag")


def test_full_size_varlen_zigzag_128k():
    lens = synth.doc_lengths(131072)
    cu = synth.cu_seqlens_from_lengths(lens).tolist()
    full_size_ring(131072, 32, 32, 128, 8, "zigzag", cu=cu)


def test_full_size_ulysses_gqa_128k():
    S, hq, hkv, dh, P = 131072, 32, 8, 128, 8
    q, k, v = synth.qkv(S, hq, hkv, dh)
    o, lse = api.ulysses_attn_fwd(q.cuda(), k.cuda(), v.cuda(), P)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    rows = sample_rows(S, P, "contiguous", n=96)
    want_o, want_l = ref.attention(f64(q[torch.from_numpy(rows)]), f64(k), f64(v), causal=True, qpos=rows)
    idx = torch.from_numpy(rows).cuda()
    compare(o[idx], lse[:, idx], want_o, want_l, what="full ulysses")


# ----------------------------------------------------------- striped layout
@pytest.mark.parametrize("P", [2, 4, 8])
def test_striped_small(P):
    ring_case(2048, 2, 1, 128, P, "striped")


def test_striped_noncausal_dh64():
    ring_case(1536, 4, 4, 64, 3, "striped", causal=False)


def test_full_size_striped_64k():
    S, P = 65536, 8
    q, k, v = synth.qkv(S, 32, 32, 128)
    qs, ks, vs = (api.striped_reorder(t.cuda(), P) for t in (q, k, v))
    o, lse = api.ring_attn_fwd(qs, ks, vs, P, "striped", True)
    o = api.striped_reorder(o, P, inverse=True)
    lse = api.striped_reorder(lse, P, inverse=True, seq_dim=1)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    rows = sample_rows(S, P, "contiguous", n=128)
    want_o, want_l = ref.attention(f64(q[torch.from_numpy(rows)]), f64(k), f64(v), causal=True, qpos=rows)
    idx = torch.from_numpy(rows).cuda()
    compare(o[idx], lse[:, idx], want_o, want_l, what="full striped")


# ----------------------------------------------------------- more shapes
@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
def test_sixteen_ranks_split_launches(layout):
    # P = 16: up to 256 block pairs, more than one attention launch
    ring_case(4096, 2, 2, 64, 16, layout)


def test_gqa_inside_the_ring():
    ring_case(2048, 8, 2, 128, 4, "zigzag")


def test_varlen_gqa_contiguous():
    S = 3072
    lens = synth.doc_lengths(S, 100, 900, seed=9)
    ring_case(S, 4, 2, 64, 4, "contiguous", cu=synth.cu_seqlens_from_lengths(lens).tolist())


@pytest.mark.parametrize("causal", [True, False])
def test_ulysses_dh64(causal):
    S, hq, hkv, dh, P = 1024, 8, 8, 64, 4
    q, k, v = synth.qkv(S, hq, hkv, dh)
    o, lse = api.ulysses_attn_fwd(q.cuda(), k.cuda(), v.cuda(), P, causal=causal)
    torch.cuda.synchronize()
    want_o, want_l = ref.attention(f64(q), f64(k), f64(v), causal=causal)
    compare(o, lse, want_o, want_l, what=f"ulysses dh64 causal={causal}")
