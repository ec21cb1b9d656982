"""The distributed entry points with the library's CUDA kernels, in a
one-rank NCCL process group (a single GPU: no peer to wait on).  The
exchanges themselves are covered by the multi-rank gloo tests."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

from context_exact_attention_step_b200 import distributed as D, synth
from oracle import ref

from _util import check_grad, compare, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def one_rank_group():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"))
    yield
    dist.destroy_process_group()


def test_ring_dist_one_rank(one_rank_group):
    S, hq, hkv, dh = 1024, 4, 2, 128
    q, k, v = synth.qkv(S, hq, hkv, dh)
    o, lse = D.ring_attn_fwd_dist(q.cuda(), k.cuda(), v.cuda(), "contiguous", True)
    torch.cuda.synchronize()
    want_o, want_l = ref.attention(f64(q), f64(k), f64(v), causal=True)
    compare(o, lse, want_o, want_l, what="ring over one rank")


def test_ulysses_dist_one_rank(one_rank_group):
    S, hq, hkv, dh = 1024, 4, 2, 64
    q, k, v = synth.qkv(S, hq, hkv, dh)
    o, lse = D.ulysses_attn_fwd_dist(q.cuda(), k.cuda(), v.cuda(), False)
    torch.cuda.synchronize()
    want_o, want_l = ref.attention(f64(q), f64(k), f64(v), causal=False)
    compare(o, lse, want_o, want_l, what="ulysses over one rank")


def test_ring_bwd_dist_one_rank(one_rank_group):
    S, hq, hkv, dh = 1024, 4, 2, 128
    q, k, v = synth.qkv(S, hq, hkv, dh)
    do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = D.ring_attn_fwd_dist(qd, kd, vd, "contiguous", True)
    dq, dk, dv = D.ring_attn_bwd_dist(qd, kd, vd, o, lse, dod, "contiguous", True)
    torch.cuda.synchronize()
    want = ref.attention_bwd(f64(q), f64(k), f64(v), f64(do), causal=True)
    for got, w, what in zip((dq, dk, dv), want, ("dQ", "dK", "dV")):
        check_grad(got, w, f"ring backward over one rank: {what}")


def test_ulysses_bwd_dist_one_rank(one_rank_group):
    S, hq, hkv, dh = 1024, 4, 2, 64
    q, k, v = synth.qkv(S, hq, hkv, dh)
    do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = D.ulysses_attn_fwd_dist(qd, kd, vd, False)
    dq, dk, dv = D.ulysses_attn_bwd_dist(qd, kd, vd, o, lse, dod, False)
    torch.cuda.synchronize()
    want = ref.attention_bwd(f64(q), f64(k), f64(v), f64(do), causal=False)
    for got, w, what in zip((dq, dk, dv), want, ("dQ", "dK", "dV")):
        check_grad(got, w, f"ulysses backward over one rank: {what}")


def test_usp_dist_one_rank(one_rank_group):
    # the hybrid's two process groups on a 1 x 1 grid: forward and backward
    S, hq, hkv, dh = 768, 4, 2, 64
    q, k, v = synth.qkv(S, hq, hkv, dh)
    do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    groups = D.usp_groups(1, 1)
    o, lse = D.usp_attn_fwd_dist(qd, kd, vd, "zigzag", True, None, groups)
    dq, dk, dv = D.usp_attn_bwd_dist(qd, kd, vd, o, lse, dod, "zigzag", True, None, groups)
    torch.cuda.synchronize()
    want_o, want_l = ref.attention(f64(q), f64(k), f64(v), causal=True)
    compare(o, lse, want_o, want_l, what="usp over one rank")
    want = ref.attention_bwd(f64(q), f64(k), f64(v), f64(do), causal=True)
    for got, w, what in zip((dq, dk, dv), want, ("dQ", "dK", "dV")):
        check_grad(got, w, f"usp backward over one rank: {what}")
