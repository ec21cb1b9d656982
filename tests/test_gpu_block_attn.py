"""GPU parity of one ring step (cp_block_attn_fwd) against the fp64 oracle on
every kind of block pair: full, causal diagonal, zigzag halves, partial query
and key tiles (ragged tails), rows with no admitted key, documents, GQA,
dh 64 and 128, non-causal."""
import numpy as np
import pytest
import torch

from context_exact_attention_step_b200 import api, synth
from oracle import ref

from _util import compare, f64

pytestmark = pytest.mark.gpu


def positions(chunks):
    return np.concatenate([np.arange(s, s + n) for s, n in chunks])


def run_case(q_chunks, k_chunks, hq=2, hkv=2, dh=128, causal=True, cu=None, seed=0):
    n_q = sum(n for _, n in q_chunks)
    n_k = sum(n for _, n in k_chunks)
    q = synth.normal((n_q, hq, dh), 100 + seed, 0.5)
    k = synth.normal((n_k, hkv, dh), 200 + seed, 0.5)
    v = synth.normal((n_k, hkv, dh), 300 + seed, 0.5)
    cu_dev = torch.tensor(cu, dtype=torch.int32, device="cuda") if cu is not None else None
    o, lse = api.block_attn_fwd(q.cuda(), k.cuda(), v.cuda(), q_chunks, k_chunks, causal, cu_dev)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    want_o, want_l = ref.attention(f64(q), f64(k), f64(v), causal=causal, cu_seqlens=cu,
                                   qpos=positions(q_chunks), kpos=positions(k_chunks))
    return compare(o, lse, want_o, want_l, what=f"q={q_chunks} k={k_chunks}")


def test_full_pair_noncausal():
    run_case([(1024, 256)], [(0, 256)], causal=False)


def test_full_pair_causal_all_visible():
    run_case([(1024, 512)], [(0, 512)])


def test_causal_diagonal():
    run_case([(0, 512)], [(0, 512)])


def test_causal_diagonal_dh64():
    run_case([(0, 384)], [(0, 384)], dh=64, hq=4, hkv=4)


def test_gqa_4_to_1():
    run_case([(0, 256)], [(0, 256)], hq=8, hkv=2)


def test_ragged_tiles():
    # query tile of 200 rows (second sub-tile partial), keys 300 (last tile partial)
    run_case([(300, 200)], [(0, 300)])
    run_case([(17, 333)], [(5, 345)], causal=False)


def test_rows_without_keys_are_empty():
    # queries before every key: causal admits nothing -> O = 0, LSE = -inf
    run_case([(0, 128)], [(500, 256)])
    # half of the rows see keys
    run_case([(0, 256)], [(128, 256)])


def test_zigzag_diagonal_pair():
    S, P, r = 2048, 4, 1
    c = S // (2 * P)
    ch = [(r * c, c), ((2 * P - 1 - r) * c, c)]
    run_case(ch, ch)


def test_zigzag_off_diagonal_pairs():
    S, P = 2048, 4
    c = S // (2 * P)
    sh = lambda r: [(r * c, c), ((2 * P - 1 - r) * c, c)]
    run_case(sh(2), sh(0))   # j < r: all queries vs the first key chunk
    run_case(sh(0), sh(3))   # j > r: second query chunk vs all keys


def test_documents():
    cu = [0, 100, 101, 700, 1024]
    run_case([(0, 1024)], [(0, 1024)], cu=cu)
    run_case([(512, 512)], [(0, 512)], cu=cu)


def test_documents_noncausal():
    cu = [0, 300, 1024]
    run_case([(0, 512)], [(256, 512)], causal=False, cu=cu)


def test_long_pair_many_tiles():
    err_o, err_l = run_case([(0, 2048)], [(0, 2048)], hq=2, hkv=1)
    assert err_o < 5e-3 and err_l < 1e-4


def test_four_chunks_per_side():
    # up to CP_MAX_CHUNKS segments on each side, out of position order
    qc = [(900, 100), (0, 50), (300, 130), (2000, 40)]
    kc = [(0, 200), (250, 300), (880, 77), (1990, 60)]
    run_case(qc, kc, hq=2, hkv=1)
    run_case(qc, kc, hq=2, hkv=1, causal=False)
