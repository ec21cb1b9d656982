"""Multi-process (gloo, CPU) tests of the communication in
``context_exact_attention_step_b200.distributed``: the ring's K/V rotation
with live-step skipping and the two Ulysses all-to-alls, on 2 and 4 ranks.

The library's CUDA kernels cannot run here, so each rank passes stand-ins
with the same signatures: the fp64 oracle for block attention and the LSE
merge, a reshape for the head-block split, and the library's own host
scheduler for the skip decisions.  Every rank's result must equal the oracle's
attention over the whole sequence for that rank's rows."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleKernels:
    """CPU stand-ins for the kernels ``distributed`` calls (test only)."""

    @staticmethod
    def ring_schedule(S, P, layout, causal, cu):
        from context_exact_attention_step_b200 import api
        return api.ring_schedule(S, P, layout, causal, cu)

    @staticmethod
    def block_attn_fwd(q, k, v, q_chunks, k_chunks, causal, cu_dev, scale):
        from oracle import ref
        qpos = np.concatenate([np.arange(a, a + n) for a, n in q_chunks])
        kpos = np.concatenate([np.arange(a, a + n) for a, n in k_chunks])
        cu = None if cu_dev is None else cu_dev.tolist()
        o, lse = ref.attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), causal=causal,
                               cu_seqlens=cu, scale=scale or None, qpos=qpos, kpos=kpos)
        return torch.from_numpy(o), torch.from_numpy(lse)

    @staticmethod
    def lse_merge(parts_o, parts_l):
        from oracle import ref
        o, lse = ref.lse_merge(np.stack([t.numpy() for t in parts_o]), np.stack([t.numpy() for t in parts_l]))
        return torch.from_numpy(o), torch.from_numpy(lse)

    @staticmethod
    def head_block_split(x, P, inverse=False):
        if not inverse:
            n, h, dh = x.shape
            return x.reshape(n, P, h // P, dh).permute(1, 0, 2, 3).contiguous()
        p_, n, hg, dh = x.shape
        return x.permute(1, 0, 2, 3).reshape(n, p_ * hg, dh).contiguous()


def _worker(rank, world, port, kind, cfg, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from context_exact_attention_step_b200 import distributed as D, synth
        from oracle import ref
        S, hq, hkv, dh = cfg["S"], cfg["hq"], cfg["hkv"], cfg["dh"]
        q, k, v = (t.double() for t in synth.qkv(S, hq, hkv, dh))
        layout = cfg.get("layout", "contiguous")
        rows = ref.shard_positions(S, world, layout, rank)
        idx = torch.from_numpy(rows)
        if kind == "ring":
            o, lse = D.ring_attn_fwd_dist(q[idx], k[idx], v[idx], layout, cfg["causal"], cfg.get("cu"),
                                          kernels=OracleKernels)
        else:
            o, lse = D.ulysses_attn_fwd_dist(q[idx], k[idx], v[idx], cfg["causal"], kernels=OracleKernels)
        results[rank] = (o.numpy(), lse.numpy())
    finally:
        dist.destroy_process_group()


def _run(kind, world, cfg):
    from oracle import ref
    from context_exact_attention_step_b200 import synth
    manager = mp.Manager()
    results = manager.dict()
    mp.spawn(_worker, args=(world, _free_port(), kind, cfg, results), nprocs=world, join=True)
    S, hq, hkv, dh = cfg["S"], cfg["hq"], cfg["hkv"], cfg["dh"]
    q, k, v = (t.double().numpy() for t in synth.qkv(S, hq, hkv, dh))
    want_o, want_l = ref.attention(q, k, v, causal=cfg["causal"], cu_seqlens=cfg.get("cu"))
    for r in range(world):
        rows = ref.shard_positions(S, world, cfg.get("layout", "contiguous"), r)
        o, lse = results[r]
        np.testing.assert_allclose(o, want_o[rows], atol=1e-10)
        np.testing.assert_allclose(lse, want_l[:, rows], atol=1e-10)


@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "striped"])
@pytest.mark.parametrize("world", [2, 4])
def test_ring_over_ranks(layout, world):
    _run("ring", world, dict(S=64, hq=4, hkv=2, dh=8, layout=layout, causal=True))


def test_ring_over_three_ranks():
    # an odd ring: every rank's shard visits the others in the same order
    _run("ring", 3, dict(S=48, hq=2, hkv=1, dh=8, layout="zigzag", causal=True))


def test_ring_over_ranks_noncausal_documents():
    _run("ring", 4, dict(S=64, hq=2, hkv=2, dh=8, layout="zigzag", causal=False, cu=[0, 5, 6, 40, 64]))
    _run("ring", 2, dict(S=64, hq=2, hkv=2, dh=8, layout="contiguous", causal=True, cu=[0, 5, 6, 40, 64]))


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_over_ranks(world):
    _run("ulysses", world, dict(S=32, hq=8, hkv=4, dh=8, causal=True))


def test_ulysses_over_ranks_noncausal():
    _run("ulysses", 2, dict(S=32, hq=4, hkv=2, dh=8, causal=False))
