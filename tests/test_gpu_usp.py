"""GPU parity of the Ulysses-inside / Ring-across hybrid (USP) against the
fp64 oracle: the library's path (seq->head transpose over Pu, one attention
launch for every head block's ring pairs over Pr, one merge that writes the
head blocks back into [S, hq, dh]) must equal plain attention of the whole
sequence, in the ring layout's storage order."""
import numpy as np
import pytest
import torch

from context_exact_attention_step_b200 import api, synth
from oracle import ref

from _util import compare, f64

pytestmark = pytest.mark.gpu


def storage_order(S, Pr, layout):
    return np.concatenate([ref.shard_positions(S, Pr, layout, g) for g in range(Pr)])


def usp_case(S, hq, hkv, dh, Pr, Pu, layout, causal=True, cu=None):
    q, k, v = synth.qkv(S, hq, hkv, dh)
    order = storage_order(S, Pr, layout)
    qs, ks, vs = (t[torch.from_numpy(order)].contiguous().cuda() for t in (q, k, v))
    o, lse = api.usp_attn_fwd(qs, ks, vs, Pr, Pu, layout, causal, cu)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    want_o, want_l = ref.attention(f64(q), f64(k), f64(v), causal=causal, cu_seqlens=cu)
    return compare(o, lse, want_o[order], want_l[:, order], what=f"usp Pr={Pr} Pu={Pu} {layout}")


@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "striped"])
@pytest.mark.parametrize("Pr,Pu", [(2, 2), (4, 2), (2, 4), (1, 4), (4, 1)])
def test_usp_small(layout, Pr, Pu):
    usp_case(2048, 8, 4, 128, Pr, Pu, layout)


def test_usp_noncausal_dh64():
    usp_case(1536, 4, 2, 64, 3, 2, "contiguous", causal=False)


def test_usp_varlen_zigzag():
    S = 4096
    lens = synth.doc_lengths(S, 64, 1024, seed=4)
    usp_case(S, 4, 2, 128, 2, 2, "zigzag", cu=synth.cu_seqlens_from_lengths(lens).tolist())


def test_usp_matches_the_oracle_composite():
    # the same case through the oracle's own USP steps (permute, per-head-block
    # ring, merge, permute back) instead of the unsplit definition
    S, hq, hkv, dh, Pr, Pu = 1024, 4, 4, 64, 2, 2
    q, k, v = synth.qkv(S, hq, hkv, dh)
    order = storage_order(S, Pr, "zigzag")
    qs, ks, vs = (t[torch.from_numpy(order)].contiguous().cuda() for t in (q, k, v))
    o, lse = api.usp_attn_fwd(qs, ks, vs, Pr, Pu, "zigzag")
    torch.cuda.synchronize()
    want_o, want_l = ref.usp_attention(f64(q), f64(k), f64(v), S, Pr, Pu, "zigzag")
    compare(o, lse, want_o, want_l, what="usp vs oracle composite")


def test_usp_many_pairs_split_launches():
    # Pr = 8 zigzag, Pu = 4: 64 ring pairs x 4 head blocks = 256 block pairs,
    # four attention launches; 8 ranks x 2 tasks x 4 head blocks merge tasks
    usp_case(4096, 8, 4, 64, 8, 4, "zigzag")


def test_full_size_usp_gqa_128k():
    # 131072 tokens, 32 query / 4 KV heads: eight ranks exceed the KV head
    # count, so Ulysses alone cannot shard it; Pu = 4 x Pr = 2 zigzag can.
    S, hq, hkv, dh, Pr, Pu = 131072, 32, 4, 128, 2, 4
    q, k, v = synth.qkv(S, hq, hkv, dh)
    qs, ks, vs = (api.zigzag_reorder(t.cuda(), Pr) for t in (q, k, v))
    o, lse = api.usp_attn_fwd(qs, ks, vs, Pr, Pu, "zigzag")
    o = api.zigzag_reorder(o, Pr, inverse=True)
    lse = api.zigzag_reorder(lse, Pr, inverse=True, seq_dim=1)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    rng = np.random.default_rng(11)
    bounds = [c * S // (2 * Pr) for c in range(2 * Pr + 1)] + [x * S // (Pr * Pu) for x in range(Pr * Pu + 1)]
    rows = {0, S - 1} | {b + d for b in bounds for d in (-1, 0, 1) if 0 <= b + d < S}
    rows = np.array(sorted(rows | set(rng.integers(0, S, 96).tolist())))
    want_o, want_l = ref.attention(f64(q[torch.from_numpy(rows)]), f64(k), f64(v), causal=True, qpos=rows)
    idx = torch.from_numpy(rows).cuda()
    compare(o[idx], lse[:, idx], want_o, want_l, what="full usp")
