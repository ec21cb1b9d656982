"""GPU parity of the backward (prep, dQ kernel, dK/dV kernel; ring, Ulysses
and the hybrid) against the fp64 oracle's gradient of the exact attention.

Tolerance, derived from the arithmetic: the kernels round P and dS to bf16
(unit roundoff u = 2^-8) before the tensor-core products and accumulate in
fp32, so each term of a gradient carries a relative error of at most about
2u and the sums of such terms stay within a few u of the largest entry.  A
gradient tensor passes when max |gpu - oracle| <= 2e-2 * max |oracle| (about
5u), the same 2e-2 as the forward's O bound, scaled by the tensor's size
because gradients, unlike O, are not bounded by 1."""
import numpy as np
import pytest
import torch

from context_exact_attention_step_b200 import api, synth
from oracle import ref

from _util import f64

pytestmark = pytest.mark.gpu

REL_TOL = 2e-2


def storage_order(S, P, layout):
    return np.concatenate([ref.shard_positions(S, P, layout, r) for r in range(P)])


def check_grad(got, want, what):
    got = f64(got)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    scale = float(np.max(np.abs(want)))
    err = float(np.max(np.abs(got - want)))
    assert err <= REL_TOL * max(scale, 1e-6), f"{what}: max-abs error {err:.3e} vs max |ref| {scale:.3e}"
    return err / max(scale, 1e-30)


def bwd_case(S, hq, hkv, dh, P, layout, causal=True, cu=None):
    q, k, v = synth.qkv(S, hq, hkv, dh)
    do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5)
    order = storage_order(S, P, layout)
    idx = torch.from_numpy(order)
    qs, ks, vs, dos = (t[idx].contiguous().cuda() for t in (q, k, v, do))
    o, lse = api.ring_attn_fwd(qs, ks, vs, P, layout, causal, cu)
    dq, dk, dv = api.ring_attn_bwd(qs, ks, vs, o, lse, dos, P, layout, causal, cu)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    wq, wk, wv = ref.attention_bwd(f64(q), f64(k), f64(v), f64(do), causal=causal, cu_seqlens=cu)
    what = f"S={S} P={P} {layout} causal={causal}"
    return (check_grad(dq, wq[order], "dQ " + what), check_grad(dk, wk[order], "dK " + what),
            check_grad(dv, wv[order], "dV " + what))


def test_bwd_single_block():
    bwd_case(256, 2, 2, 128, 1, "contiguous")


@pytest.mark.parametrize("P", [1, 2, 4])
def test_bwd_contiguous(P):
    bwd_case(1024, 2, 2, 128, P, "contiguous")


@pytest.mark.parametrize("P", [2, 4, 8])
def test_bwd_zigzag(P):
    bwd_case(2048, 2, 1, 128, P, "zigzag")


@pytest.mark.parametrize("P", [2, 4])
def test_bwd_striped(P):
    bwd_case(1024, 2, 2, 128, P, "striped")


def test_bwd_noncausal_dh64():
    bwd_case(768, 4, 2, 64, 3, "contiguous", causal=False)


def test_bwd_ragged_tiles():
    # zigzag chunks of 100 rows: every tile is partial
    bwd_case(800, 2, 2, 64, 4, "zigzag")


def test_bwd_gqa():
    bwd_case(1024, 8, 2, 128, 4, "zigzag")


def test_bwd_documents():
    S = 2048
    lens = synth.doc_lengths(S, 64, 700, seed=6)
    bwd_case(S, 2, 2, 128, 4, "zigzag", cu=synth.cu_seqlens_from_lengths(lens).tolist())


def test_bwd_documents_noncausal():
    S = 1536
    lens = synth.doc_lengths(S, 100, 600, seed=8)
    bwd_case(S, 2, 2, 64, 2, "contiguous", causal=False, cu=synth.cu_seqlens_from_lengths(lens).tolist())


def test_bwd_one_token_per_rank():
    bwd_case(8, 2, 2, 64, 8, "contiguous")


def test_bwd_from_oracle_forward():
    # the backward kernels alone: O and LSE taken from the oracle instead of
    # the library's forward
    S, hq, hkv, dh, P = 1024, 2, 2, 128, 4
    q, k, v = synth.qkv(S, hq, hkv, dh)
    do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5)
    order = storage_order(S, P, "zigzag")
    idx = torch.from_numpy(order)
    o_ref, lse_ref = ref.attention(f64(q), f64(k), f64(v), causal=True)
    o = torch.from_numpy(o_ref[order]).float().cuda()
    lse = torch.from_numpy(lse_ref[:, order]).float().contiguous().cuda()
    qs, ks, vs, dos = (t[idx].contiguous().cuda() for t in (q, k, v, do))
    dq, dk, dv = api.ring_attn_bwd(qs, ks, vs, o, lse, dos, P, "zigzag")
    torch.cuda.synchronize()
    wq, wk, wv = ref.attention_bwd(f64(q), f64(k), f64(v), f64(do), causal=True)
    check_grad(dq, wq[order], "dQ")
    check_grad(dk, wk[order], "dK")
    check_grad(dv, wv[order], "dV")


def test_bwd_many_tiles_8k():
    # 8192 tokens, 4 heads, P = 4 zigzag: 64 query and 64 key tiles per head
    bwd_case(8192, 4, 4, 128, 4, "zigzag")


def test_bwd_full_size_32k():
    # the bench workload (32768 tokens, 32 heads, P = 4 contiguous): dQ on
    # sampled rows against the oracle row by row; dK and dV through the
    # identities every row of dS summing to 0 and every row of P to 1
    S, hq, hkv, dh, P = 32768, 32, 32, 128, 4
    q, k, v = synth.qkv(S, hq, hkv, dh)
    do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = api.ring_attn_fwd(qd, kd, vd, P, "contiguous")
    dq, dk, dv = api.ring_attn_bwd(qd, kd, vd, o, lse, dod, P, "contiguous")
    torch.cuda.synchronize()
    assert api.device_error() == 0
    rng = np.random.default_rng(3)
    rows = {0, S - 1} | {b + d for b in range(0, S + 1, S // P) for d in (-1, 0, 1) if 0 <= b + d < S}
    rows = np.array(sorted(rows | set(rng.integers(0, S, 40).tolist())))
    wq, _, _ = ref.attention_bwd(f64(q[torch.from_numpy(rows)]), f64(k), f64(v), f64(do[torch.from_numpy(rows)]),
                                 causal=True, qpos=rows)
    check_grad(dq[torch.from_numpy(rows).cuda()], wq, "full dQ")
    sum_dk = f64(dk.sum(dim=0))
    abs_dk = f64(dk.abs().sum(dim=0))
    assert np.all(np.abs(sum_dk) <= 1e-2 * abs_dk + 1e-6), "sum over keys of dK is not ~0"
    sum_dv = f64(dv.sum(dim=0))
    want_dv = f64(do.float().sum(dim=0))
    assert np.max(np.abs(sum_dv - want_dv)) <= 2e-2 * np.max(np.abs(want_dv)), "sum over keys of dV != sum of dO"


# ----------------------------------------------------------- Ulysses and the hybrid
def usp_bwd_case(S, hq, hkv, dh, Pr, Pu, layout, causal=True, cu=None):
    q, k, v = synth.qkv(S, hq, hkv, dh)
    do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5)
    order = storage_order(S, Pr, layout)
    idx = torch.from_numpy(order)
    qs, ks, vs, dos = (t[idx].contiguous().cuda() for t in (q, k, v, do))
    o, lse = api.usp_attn_fwd(qs, ks, vs, Pr, Pu, layout, causal, cu)
    dq, dk, dv = api.usp_attn_bwd(qs, ks, vs, o, lse, dos, Pr, Pu, layout, causal, cu)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    wq, wk, wv = ref.attention_bwd(f64(q), f64(k), f64(v), f64(do), causal=causal, cu_seqlens=cu)
    what = f"usp S={S} Pr={Pr} Pu={Pu} {layout}"
    check_grad(dq, wq[order], "dQ " + what)
    check_grad(dk, wk[order], "dK " + what)
    check_grad(dv, wv[order], "dV " + what)


@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "striped"])
@pytest.mark.parametrize("Pr,Pu", [(2, 2), (1, 4), (4, 2)])
def test_usp_bwd(layout, Pr, Pu):
    usp_bwd_case(1024, 8, 4, 128, Pr, Pu, layout)


def test_usp_bwd_documents_noncausal_dh64():
    S = 2048
    lens = synth.doc_lengths(S, 64, 700, seed=6)
    usp_bwd_case(S, 4, 2, 64, 2, 2, "zigzag", causal=False, cu=synth.cu_seqlens_from_lengths(lens).tolist())


def test_usp_bwd_many_items():
    # 8 zigzag ring ranks x 4 head blocks: 256 own tiles of four head blocks
    # interleaved in one launch per kernel
    usp_bwd_case(8192, 8, 4, 64, 8, 4, "zigzag")


@pytest.mark.parametrize("causal", [True, False])
def test_ulysses_bwd(causal):
    S, hq, hkv, dh, P = 1024, 8, 4, 128, 4
    q, k, v = synth.qkv(S, hq, hkv, dh)
    do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = api.ulysses_attn_fwd(qd, kd, vd, P, causal=causal)
    dq, dk, dv = api.ulysses_attn_bwd(qd, kd, vd, o, lse, dod, P, causal=causal)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    wq, wk, wv = ref.attention_bwd(f64(q), f64(k), f64(v), f64(do), causal=causal)
    check_grad(dq, wq, "ulysses dQ")
    check_grad(dk, wk, "ulysses dK")
    check_grad(dv, wv, "ulysses dV")


def test_bwd_sixteen_ranks():
    # the backward's rank limit: 16 zigzag shards of 128 rows
    bwd_case(4096, 2, 2, 64, 16, "zigzag")


def test_bwd_ragged_shards():
    # 3 ranks of 500 rows: every shard ends in a 116-row tile
    bwd_case(1500, 2, 2, 128, 3, "contiguous")


def test_bwd_gqa_documents():
    S = 2048
    lens = synth.doc_lengths(S, 50, 600, seed=10)
    bwd_case(S, 8, 2, 64, 4, "zigzag", cu=synth.cu_seqlens_from_lengths(lens).tolist())
