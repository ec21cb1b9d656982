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
from context_exact_attention_step_b200 import distributed as D
from oracle import ref

from _util import GRAD_REL_TOL, check_grad, f64

pytestmark = pytest.mark.gpu

assert GRAD_REL_TOL == 2e-2


def storage_order(S, P, layout):
    return np.concatenate([ref.shard_positions(S, P, layout, r) for r in range(P)])


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


# ------------------------------------------- block pairs: one step of the ring across GPUs
def _pair_setup(S, hq, hkv, dh, P, layout, causal, cu):
    q, k, v = synth.qkv(S, hq, hkv, dh)
    do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5)
    o_ref, lse_ref = ref.attention(f64(q), f64(k), f64(v), causal=causal, cu_seqlens=cu)
    return q, k, v, do, o_ref, lse_ref


@pytest.mark.parametrize("layout,r,j", [("zigzag", 1, 3), ("zigzag", 3, 0), ("contiguous", 2, 2),
                                        ("striped", 1, 2), ("striped", 2, 1)])
def test_block_bwd_pair(layout, r, j):
    # the rows of rank r against shard j, with the merged O and LSE of the
    # whole attention: equal to the oracle's contribution of that pair
    S, hq, hkv, dh, P = 2048, 4, 2, 128, 4
    q, k, v, do, o_ref, lse_ref = _pair_setup(S, hq, hkv, dh, P, layout, True, None)
    qp, kp = ref.shard_positions(S, P, layout, r), ref.shard_positions(S, P, layout, j)
    qi, ki = torch.from_numpy(qp), torch.from_numpy(kp)
    o_r = torch.from_numpy(o_ref[qp]).float().cuda()
    lse_r = torch.from_numpy(np.ascontiguousarray(lse_ref[:, qp])).float().cuda()
    q_r, do_r = q[qi].contiguous().cuda(), do[qi].contiguous().cuda()
    k_j, v_j = k[ki].contiguous().cuda(), v[ki].contiguous().cuda()
    lg, dd = api.attn_bwd_prep(o_r, lse_r, do_r)
    qc, kc = D.query_chunks(S, P, layout, r), D.key_chunks(S, P, layout, r, j)
    dq, dk, dv = api.block_attn_bwd(q_r, k_j, v_j, do_r, lg, dd, qc, kc, True)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    want = ref.ring_pair_bwd(f64(q)[qp], f64(k)[kp], f64(v)[kp], f64(do)[qp], o_ref[qp], lse_ref[:, qp], qp, kp,
                             causal=True)
    for got, w, what in zip((dq, dk, dv), want, ("dQ", "dK", "dV")):
        if np.max(np.abs(w)) == 0.0:
            assert float(got.abs().max()) == 0.0, f"{what}: a pair with no admitted keys must give 0"
        else:
            check_grad(got, w, f"{what} {layout} r={r} j={j}")


def test_block_bwd_parts_and_accumulate():
    # parts picks the kernels; accumulate adds to what the buffers hold
    S, hq, hkv, dh = 640, 2, 2, 64
    q, k, v, do, o_ref, lse_ref = _pair_setup(S, hq, hkv, dh, 1, "contiguous", False, None)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o = torch.from_numpy(o_ref).float().cuda()
    lse = torch.from_numpy(lse_ref).float().cuda()
    lg, dd = api.attn_bwd_prep(o, lse, dod)
    base_q = torch.randn(S, hq, dh, device="cuda")
    base_k = torch.randn(S, hkv, dh, device="cuda")
    dq = base_q.clone()
    dk, dv = base_k.clone(), base_k.clone()
    api.block_attn_bwd(qd, kd, vd, dod, lg, dd, causal=False, dq=dq, parts=api.BWD_DQ, accumulate=True)
    torch.cuda.synchronize()
    assert torch.equal(dk, base_k) and torch.equal(dv, base_k), "the dQ part alone must leave dK, dV alone"
    api.block_attn_bwd(qd, kd, vd, dod, lg, dd, causal=False, dk=dk, dv=dv, parts=api.BWD_DKDV, accumulate=True)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    wq, wk, wv = ref.attention_bwd(f64(q), f64(k), f64(v), f64(do), causal=False)
    check_grad(f64(dq) - f64(base_q), wq, "accumulated dQ")
    check_grad(f64(dk) - f64(base_k), wk, "accumulated dK")
    check_grad(f64(dv) - f64(base_k), wv, "accumulated dV")


@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "striped"])
def test_block_bwd_ring_emulated(layout):
    # the multi-GPU ring backward's arithmetic on one GPU: for every ring step
    # and rank, one block-pair call adding to dQ_r and to the dK_j, dV_j the
    # shard carries; the sums must equal the gradient of the whole attention
    S, hq, hkv, dh, P = 2048, 4, 2, 64, 4
    lens = synth.doc_lengths(S, 64, 900, seed=12)
    cu = synth.cu_seqlens_from_lengths(lens).tolist()
    if layout == "striped":
        cu = None  # the striped layout has no document mask
    q, k, v, do, o_ref, lse_ref = _pair_setup(S, hq, hkv, dh, P, layout, True, cu)
    sched = api.ring_schedule(S, P, layout, True, cu)
    cu_dev = None if cu is None else torch.tensor(cu, dtype=torch.int32, device="cuda")
    pos = [ref.shard_positions(S, P, layout, r) for r in range(P)]
    take = lambda t, r: t[torch.from_numpy(pos[r])].contiguous().cuda()
    qs, ks, vs, dos = ([take(t, r) for r in range(P)] for t in (q, k, v, do))
    preps = [api.attn_bwd_prep(torch.from_numpy(o_ref[pos[r]]).float().cuda(),
                               torch.from_numpy(np.ascontiguousarray(lse_ref[:, pos[r]])).float().cuda(), dos[r])
             for r in range(P)]
    n = S // P
    dq = [torch.empty(n, hq, dh, device="cuda") for _ in range(P)]
    dk = [torch.empty(n, hkv, dh, device="cuda") for _ in range(P)]
    dv = [torch.empty(n, hkv, dh, device="cuda") for _ in range(P)]
    for t in range(P):
        for r in range(P):
            j = (r - t) % P
            assert sched["launched"][r * P + t] or t > 0
            if sched["launched"][r * P + t]:
                api.block_attn_bwd(qs[r], ks[j], vs[j], dos[r], *preps[r], D.query_chunks(S, P, layout, r),
                                   D.key_chunks(S, P, layout, r, j), True, cu_dev, dq=dq[r], dk=dk[j], dv=dv[j],
                                   accumulate=t > 0)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    wq, wk, wv = ref.attention_bwd(f64(q), f64(k), f64(v), f64(do), causal=True, cu_seqlens=cu)
    order = storage_order(S, P, layout)
    check_grad(torch.cat(dq), wq[order], f"emulated ring dQ {layout}")
    check_grad(torch.cat(dk), wk[order], f"emulated ring dK {layout}")
    check_grad(torch.cat(dv), wv[order], f"emulated ring dV {layout}")
