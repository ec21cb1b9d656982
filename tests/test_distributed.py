"""Multi-process (gloo, CPU) tests of the communication in
``context_exact_attention_step_b200.distributed``: the ring's K/V rotation
with live-step skipping and the two Ulysses all-to-alls, forward and
backward (where the shard's dK/dV travel with it), on 2, 3 and 4 ranks.

The library's CUDA kernels cannot run here, so each rank passes stand-ins
with the same signatures: the fp64 oracle for block attention, the block
pair's backward and the LSE merge, a reshape for the head-block split, and
the library's own host scheduler for the skip decisions.  Every rank's result
must equal the oracle's attention (or its gradient) over the whole sequence
for that rank's rows."""
import datetime
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
    def attn_bwd_prep(o, lse, do):
        # the stand-in's per-row state: the merged LSE itself and D = rowsum(dO * O)
        return lse.clone(), (do * o).sum(dim=2).T.contiguous()

    @staticmethod
    def block_attn_bwd(q, k, v, do, lg, dd, q_chunks, k_chunks, causal, cu_dev, scale, dq=None, dk=None, dv=None,
                       parts=3, accumulate=False):
        from context_exact_attention_step_b200 import api
        from oracle import ref
        qpos = np.concatenate([np.arange(a, a + n) for a, n in q_chunks])
        kpos = np.concatenate([np.arange(a, a + n) for a, n in k_chunks])
        cu = None if cu_dev is None else cu_dev.tolist()
        grads = ref.ring_pair_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), None, lg.numpy(), qpos, kpos, causal,
                                  cu, scale or None, d_r=dd.numpy())
        for g, out, bit in zip(grads, (dq, dk, dv), (api.BWD_DQ, api.BWD_DKDV, api.BWD_DKDV)):
            if parts & bit:
                t = torch.from_numpy(g).to(out.dtype)
                if accumulate:
                    out += t
                else:
                    out.copy_(t)
        return dq, dk, dv

    @staticmethod
    def ring_attn_bwd(q, k, v, o, lse, do, P, layout, causal, softmax_scale=0.0):
        # the head-layout backward over the whole sequence, from the O and LSE
        # it is given (so their transposes are checked too)
        from oracle import ref
        assert P == 1 and layout == "contiguous"
        pos = np.arange(q.shape[0])
        grads = ref.ring_pair_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), o.numpy(), lse.numpy(), pos, pos,
                                  causal, None, softmax_scale or None)
        return tuple(torch.from_numpy(g) for g in grads)

    @staticmethod
    def head_block_split(x, P, inverse=False):
        if not inverse:
            n, h, dh = x.shape
            return x.reshape(n, P, h // P, dh).permute(1, 0, 2, 3).contiguous()
        p_, n, hg, dh = x.shape
        return x.permute(1, 0, 2, 3).reshape(n, p_ * hg, dh).contiguous()


def _run_case(rank, world, kind, cfg):
    """One case on this rank: the distributed entry point with the stand-ins."""
    from context_exact_attention_step_b200 import distributed as D, synth
    from oracle import ref
    S, hq, hkv, dh = cfg["S"], cfg["hq"], cfg["hkv"], cfg["dh"]
    q, k, v = (t.double() for t in synth.qkv(S, hq, hkv, dh))
    layout = cfg.get("layout", "contiguous")
    rows = _rows(S, world, kind, cfg, rank)
    idx = torch.from_numpy(rows)
    groups = D.usp_groups(cfg["Pr"], cfg["Pu"]) if kind.startswith("usp") else None
    if kind == "usp":
        o, lse = D.usp_attn_fwd_dist(q[idx], k[idx], v[idx], layout, cfg["causal"], cfg.get("cu"), groups,
                                     kernels=OracleKernels)
        return o.numpy(), lse.numpy()
    if kind == "ring":
        o, lse = D.ring_attn_fwd_dist(q[idx], k[idx], v[idx], layout, cfg["causal"], cfg.get("cu"),
                                      kernels=OracleKernels)
        return o.numpy(), lse.numpy()
    if kind == "ulysses":
        o, lse = D.ulysses_attn_fwd_dist(q[idx], k[idx], v[idx], cfg["causal"], kernels=OracleKernels)
        return o.numpy(), lse.numpy()
    # the backward: the forward's merged O and LSE of this rank's rows, from the oracle
    do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5).double()
    o_all, lse_all = ref.attention(q.numpy(), k.numpy(), v.numpy(), causal=cfg["causal"], cu_seqlens=cfg.get("cu"))
    o, lse = torch.from_numpy(o_all[rows]), torch.from_numpy(np.ascontiguousarray(lse_all[:, rows]))
    if cfg.get("lse_transposed"):  # same values, column-major storage
        lse = lse.T.contiguous().T
    if kind == "usp_bwd":
        grads = D.usp_attn_bwd_dist(q[idx], k[idx], v[idx], o, lse, do[idx], layout, cfg["causal"], cfg.get("cu"),
                                    groups, kernels=OracleKernels)
    elif kind == "ring_bwd":
        grads = D.ring_attn_bwd_dist(q[idx], k[idx], v[idx], o, lse, do[idx], layout, cfg["causal"], cfg.get("cu"),
                                     kernels=OracleKernels)
    else:
        grads = D.ulysses_attn_bwd_dist(q[idx], k[idx], v[idx], o, lse, do[idx], cfg["causal"],
                                        kernels=OracleKernels)
    return tuple(g.numpy() for g in grads)


def _worker(rank, world, port, cases, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    # a short timeout: ranks that fall out of step end with an error, not a hang
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    # log every point-to-point exchange the distributed code posts:
    # (op, peer, elements) per batch, in posting order
    from context_exact_attention_step_b200 import distributed as D
    post = D.dist.batch_isend_irecv
    log = []

    def logged(ops):
        log.append(tuple(("send" if op.op is dist.isend else "recv", op.peer, op.tensor.numel()) for op in ops))
        return post(ops)

    D.dist.batch_isend_irecv = logged
    try:
        for name, kind, cfg in cases:
            log.clear()
            results[(name, rank)] = _run_case(rank, world, kind, cfg)
            results[("exchanges", name, rank)] = list(log)
    finally:
        D.dist.batch_isend_irecv = post
        dist.destroy_process_group()


def _rows(S, world, kind, cfg, r):
    """Global positions of rank r's rows, in its storage order."""
    from oracle import ref
    layout = cfg.get("layout", "contiguous")
    if kind.startswith("usp"):
        Pr, Pu = cfg["Pr"], cfg["Pu"]
        n = S // world
        return ref.shard_positions(S, Pr, layout, r // Pu)[(r % Pu) * n:(r % Pu + 1) * n]
    return ref.shard_positions(S, world, layout, r)


# every case: (name, kind, world, cfg); the cases of one world size run in one
# set of spawned ranks, one after another in the same process group
CASES = []
for _layout in ("contiguous", "zigzag", "striped"):
    for _world in (2, 4):
        CASES.append((f"ring-{_layout}-{_world}", "ring", _world,
                      dict(S=64, hq=4, hkv=2, dh=8, layout=_layout, causal=True)))
CASES += [
    ("ring-zigzag-3", "ring", 3, dict(S=48, hq=2, hkv=1, dh=8, layout="zigzag", causal=True)),
    ("ring-docs-noncausal-4", "ring", 4, dict(S=64, hq=2, hkv=2, dh=8, layout="zigzag", causal=False,
                                              cu=[0, 5, 6, 40, 64])),
    ("ring-docs-2", "ring", 2, dict(S=64, hq=2, hkv=2, dh=8, layout="contiguous", causal=True, cu=[0, 5, 6, 40, 64])),
    ("ulysses-2", "ulysses", 2, dict(S=32, hq=8, hkv=4, dh=8, causal=True)),
    ("ulysses-4", "ulysses", 4, dict(S=32, hq=8, hkv=4, dh=8, causal=True)),
    ("ulysses-noncausal-2", "ulysses", 2, dict(S=32, hq=4, hkv=2, dh=8, causal=False)),
    ("ring_bwd-contiguous-2", "ring_bwd", 2, dict(S=64, hq=4, hkv=2, dh=8, layout="contiguous", causal=True)),
    ("ring_bwd-zigzag-4", "ring_bwd", 4, dict(S=64, hq=4, hkv=2, dh=8, layout="zigzag", causal=True)),
    ("ring_bwd-striped-2", "ring_bwd", 2, dict(S=64, hq=4, hkv=2, dh=8, layout="striped", causal=True)),
    ("ring_bwd-striped-4", "ring_bwd", 4, dict(S=64, hq=4, hkv=2, dh=8, layout="striped", causal=True)),
    ("ring_bwd-docs-3", "ring_bwd", 3, dict(S=48, hq=2, hkv=1, dh=8, layout="zigzag", causal=True,
                                            cu=[0, 7, 8, 30, 48])),
    ("ring_bwd-noncausal-2", "ring_bwd", 2, dict(S=32, hq=2, hkv=2, dh=8, layout="contiguous", causal=False)),
    ("ulysses_bwd-2", "ulysses_bwd", 2, dict(S=32, hq=8, hkv=4, dh=8, causal=True)),
    ("ulysses_bwd-4", "ulysses_bwd", 4, dict(S=32, hq=8, hkv=4, dh=8, causal=True)),
    ("ulysses_bwd-noncausal-2", "ulysses_bwd", 2, dict(S=32, hq=4, hkv=2, dh=8, causal=False)),
    ("ulysses_bwd-lse-transposed-2", "ulysses_bwd", 2, dict(S=32, hq=4, hkv=2, dh=8, causal=True,
                                                            lse_transposed=True)),
]
for _layout in ("contiguous", "zigzag", "striped"):
    CASES.append((f"usp-{_layout}-2x2", "usp", 4,
                  dict(S=64, hq=4, hkv=2, dh=8, layout=_layout, causal=True, Pr=2, Pu=2)))
CASES += [
    ("usp-docs-1x4", "usp", 4, dict(S=64, hq=8, hkv=4, dh=8, layout="zigzag", causal=True, Pr=1, Pu=4,
                                    cu=[0, 9, 40, 64])),
    ("usp-docs-noncausal-4x1", "usp", 4, dict(S=64, hq=4, hkv=4, dh=8, layout="zigzag", causal=False, Pr=4, Pu=1,
                                              cu=[0, 9, 40, 64])),
    ("usp_bwd-zigzag-2x2", "usp_bwd", 4, dict(S=64, hq=4, hkv=2, dh=8, layout="zigzag", causal=True, Pr=2, Pu=2)),
    ("usp_bwd-striped-2x2", "usp_bwd", 4, dict(S=64, hq=4, hkv=2, dh=8, layout="striped", causal=True, Pr=2, Pu=2)),
    ("usp_bwd-docs-2x2", "usp_bwd", 4, dict(S=64, hq=4, hkv=2, dh=8, layout="contiguous", causal=True, Pr=2, Pu=2,
                                            cu=[0, 5, 6, 40, 64])),
]
_RESULTS = {}


def _results(world):
    if world not in _RESULTS:
        cases = [(name, kind, cfg) for name, kind, w, cfg in CASES if w == world]
        manager = mp.Manager()
        results = manager.dict()
        mp.spawn(_worker, args=(world, _free_port(), cases, results), nprocs=world, join=True)
        _RESULTS[world] = dict(results)
    return _RESULTS[world]


@pytest.mark.parametrize("name", [c[0] for c in CASES])
def test_distributed_case(name):
    """Every rank's rows equal the oracle's attention (or its gradient) over
    the whole sequence."""
    from oracle import ref
    from context_exact_attention_step_b200 import synth
    _, kind, world, cfg = next(c for c in CASES if c[0] == name)
    results = _results(world)
    S, hq, hkv, dh = cfg["S"], cfg["hq"], cfg["hkv"], cfg["dh"]
    q, k, v = (t.double().numpy() for t in synth.qkv(S, hq, hkv, dh))
    if kind.endswith("_bwd"):
        do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5).double().numpy()
        want = ref.attention_bwd(q, k, v, do, causal=cfg["causal"], cu_seqlens=cfg.get("cu"))
        for r in range(world):
            rows = _rows(S, world, kind, cfg, r)
            for got, w, what in zip(results[(name, r)], want, ("dQ", "dK", "dV")):
                np.testing.assert_allclose(got, w[rows], atol=1e-10, err_msg=f"{what} of rank {r}")
        return
    want_o, want_l = ref.attention(q, k, v, causal=cfg["causal"], cu_seqlens=cfg.get("cu"))
    for r in range(world):
        rows = _rows(S, world, kind, cfg, r)
        o, lse = results[(name, r)]
        np.testing.assert_allclose(o, want_o[rows], atol=1e-10)
        np.testing.assert_allclose(lse, want_l[:, rows], atol=1e-10)


@pytest.mark.parametrize("name", ["ring_bwd-docs-3", "ring_bwd-zigzag-4", "ring-docs-noncausal-4", "ring-zigzag-3"])
def test_ring_exchanges_are_the_same_on_every_rank(name):
    """Every rank posts the same exchanges in the same order, skipped steps
    included: the ring forward moves K/V P - 1 times; the backward also moves
    the shard's dK/dV P times (the last move brings it home).  Each batch sends
    to rank r + 1 and receives from rank r - 1."""
    _, kind, world, cfg = next(c for c in CASES if c[0] == name)
    results = _results(world)
    n = cfg["S"] // world
    kv = 2 * n * cfg["hkv"] * cfg["dh"]
    logs = [results[("exchanges", name, r)] for r in range(world)]
    want = [kv] * (world - 1)
    if kind == "ring_bwd":  # per step: K/V (except the last step), then dK/dV
        want = [x for t in range(world) for x in ([kv] if t < world - 1 else []) + [kv]]
    for r, log in enumerate(logs):
        assert [batch[0][2] for batch in log] == want, f"rank {r}: {log}"
        for batch in log:
            assert batch == (("send", (r + 1) % world, batch[0][2]), ("recv", (r - 1) % world, batch[0][2]))
