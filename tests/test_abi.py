"""CPU checks of the C ABI: the library loads, exports every entry point the
header declares, validates arguments before launching anything, and its host
ring-step scheduler agrees with the oracle's brute-force mask counts."""
import ctypes
import os
import re

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from context_exact_attention_step_b200 import _lib, api
from context_exact_attention_step_b200._lib import cp_chunk, lib
from oracle import ref

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from context_exact_attention_step_b200 import build
    build.build()


def header_functions():
    with open(os.path.join(ROOT, "include", "cp_attn.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const char\*|cp_status)\s+(cp_\w+)\s*\(", text, re.M)))


def test_library_exports_every_declared_symbol():
    names = header_functions()
    assert len(names) >= 13
    L = lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(_lib.EXPORTS)
    assert b"sm_100a" in L.cp_version()


FAKE = ctypes.c_void_p(1 << 20)        # aligned, never dereferenced on error paths
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)


def _block(q=FAKE, k=FAKE, v=FAKE, dtype=_lib.CP_BF16, n_q=256, n_k=256, hq=4, hkv=4, dh=128, nqc=1, nkc=1,
           mask=_lib.CP_MASK_CAUSAL, cu=None, n_docs=0, o=FAKE, lse=FAKE, qchunks=None):
    qc = qchunks or (cp_chunk * 1)(cp_chunk(0, n_q))
    kc = (cp_chunk * 1)(cp_chunk(0, n_k))
    return lib().cp_block_attn_fwd(q, k, v, dtype, n_q, n_k, hq, hkv, dh, qc, nqc, kc, nkc, mask,
                                   cu or ctypes.c_void_p(0), n_docs, 0.0, o, lse, ctypes.c_void_p(0))


@pytest.mark.parametrize("kw,status", [
    (dict(dh=96), _lib.CP_ERR_UNSUPPORTED),
    (dict(hq=6, hkv=4), _lib.CP_ERR_INVALID_ARG),
    (dict(dtype=_lib.CP_FP32), _lib.CP_ERR_UNSUPPORTED),
    (dict(q=ctypes.c_void_p(0)), _lib.CP_ERR_INVALID_ARG),
    (dict(k=MISALIGNED), _lib.CP_ERR_ALIGNMENT),
    (dict(o=MISALIGNED), _lib.CP_ERR_ALIGNMENT),
    (dict(n_q=0), _lib.CP_ERR_INVALID_ARG),
    (dict(nqc=5), _lib.CP_ERR_UNSUPPORTED),
    (dict(n_docs=3), _lib.CP_ERR_INVALID_ARG),
    (dict(mask=7), _lib.CP_ERR_INVALID_ARG),
    (dict(qchunks=(cp_chunk * 1)(cp_chunk(0, 100))), _lib.CP_ERR_INVALID_ARG),
])
def test_block_attn_rejects_bad_arguments(kw, status):
    assert _block(**kw) == status
    assert len(lib().cp_last_error_string()) > 0


def _ring(S=1024, hq=4, hkv=4, dh=64, P=4, layout=_lib.CP_LAYOUT_CONTIGUOUS, cu=None, n_docs=0, ws=FAKE, wsb=1 << 40,
          o=FAKE):
    return lib().cp_ring_attn_fwd(FAKE, FAKE, FAKE, _lib.CP_BF16, S, hq, hkv, dh, P, layout, _lib.CP_MASK_CAUSAL,
                                  cu, ctypes.c_void_p(0) if not n_docs else FAKE, n_docs, 0.0, o, FAKE, ws, wsb,
                                  ctypes.c_void_p(0))


def test_ring_rejects_bad_arguments():
    assert _ring(S=1000, P=3) == _lib.CP_ERR_INVALID_ARG            # P does not divide S
    assert _ring(S=1028, P=4, layout=_lib.CP_LAYOUT_ZIGZAG) == _lib.CP_ERR_INVALID_ARG  # 2P does not divide S
    assert _ring(P=17) == _lib.CP_ERR_UNSUPPORTED
    assert _ring(ws=ctypes.c_void_p(0), wsb=0) == _lib.CP_ERR_WORKSPACE
    assert _ring(wsb=16) == _lib.CP_ERR_WORKSPACE
    assert _ring(o=MISALIGNED) == _lib.CP_ERR_ALIGNMENT
    bad = (ctypes.c_int32 * 3)(0, 600, 500)
    assert _ring(cu=bad, n_docs=2) == _lib.CP_ERR_INVALID_ARG       # not increasing
    short = (ctypes.c_int32 * 3)(0, 600, 1000)
    assert _ring(cu=short, n_docs=2) == _lib.CP_ERR_INVALID_ARG     # does not end at S


def test_striped_rejects_documents():
    cu = (ctypes.c_int32 * 3)(0, 600, 1024)
    assert _ring(layout=_lib.CP_LAYOUT_STRIPED, cu=cu, n_docs=2) == _lib.CP_ERR_UNSUPPORTED


def _usp(S=1024, hq=8, hkv=4, dh=128, Pr=2, Pu=2, layout=_lib.CP_LAYOUT_ZIGZAG, cu=None, n_docs=0, ws=FAKE,
         wsb=1 << 40):
    return lib().cp_usp_attn_fwd(FAKE, FAKE, FAKE, S, hq, hkv, dh, Pr, Pu, layout, _lib.CP_MASK_CAUSAL, cu,
                                 ctypes.c_void_p(0) if not n_docs else FAKE, n_docs, 0.0, FAKE, FAKE, ws, wsb,
                                 ctypes.c_void_p(0))


def test_usp_rejects_bad_arguments():
    assert _usp(hkv=4, Pu=8, hq=8) == _lib.CP_ERR_UNSUPPORTED        # Pu does not divide the KV heads
    assert _usp(S=1026, Pr=2, Pu=2, layout=_lib.CP_LAYOUT_CONTIGUOUS) == _lib.CP_ERR_INVALID_ARG  # Pr*Pu
    assert _usp(S=1026, Pr=2, Pu=1) == _lib.CP_ERR_INVALID_ARG        # 2*Pr does not divide S (zigzag)
    assert _usp(Pr=17) == _lib.CP_ERR_UNSUPPORTED
    assert _usp(dh=96) == _lib.CP_ERR_UNSUPPORTED
    assert _usp(ws=ctypes.c_void_p(0), wsb=0) == _lib.CP_ERR_WORKSPACE
    assert _usp(wsb=1024) == _lib.CP_ERR_WORKSPACE
    cu = (ctypes.c_int32 * 3)(0, 600, 1024)
    assert _usp(layout=_lib.CP_LAYOUT_STRIPED, cu=cu, n_docs=2) == _lib.CP_ERR_UNSUPPORTED
    assert len(lib().cp_last_error_string()) > 0


@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "striped"])
def test_usp_workspace_is_copies_plus_pu_rings(layout):
    # head-major bf16 Q, K, V, then one set of ring partials (P = Pr, hq/Pu
    # heads) per Ulysses head block
    S, hq, hkv, dh, Pr, Pu = 4096, 32, 4, 128, 2, 4
    ring = api.ring_attn_workspace_size(S, hq // Pu, hkv // Pu, dh, Pr, layout)
    a = lambda x: (x + 255) // 256 * 256
    want = a(S * hq * dh * 2) + 2 * a(S * hkv * dh * 2) + Pu * a(ring)
    assert api.usp_attn_workspace_size(S, hq, hkv, dh, Pr, Pu, layout) == want


def _bwd(S=1024, hq=4, hkv=4, dh=128, P=4, layout=_lib.CP_LAYOUT_ZIGZAG, ws=FAKE, wsb=1 << 40, dq=FAKE,
         dout=FAKE, cu=None, n_docs=0):
    return lib().cp_ring_attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, dout, S, hq, hkv, dh, P, layout, _lib.CP_MASK_CAUSAL,
                                  cu, ctypes.c_void_p(0) if not n_docs else FAKE, n_docs, 0.0, dq, FAKE, FAKE, ws,
                                  wsb, ctypes.c_void_p(0))


def test_ring_bwd_rejects_bad_arguments():
    assert _bwd(dh=96) == _lib.CP_ERR_UNSUPPORTED
    assert _bwd(hq=6, hkv=4) == _lib.CP_ERR_INVALID_ARG
    assert _bwd(S=1028) == _lib.CP_ERR_INVALID_ARG                   # 2P does not divide S (zigzag)
    assert _bwd(P=17) == _lib.CP_ERR_UNSUPPORTED
    assert _bwd(dq=ctypes.c_void_p(0)) == _lib.CP_ERR_INVALID_ARG
    assert _bwd(dout=MISALIGNED) == _lib.CP_ERR_ALIGNMENT
    assert _bwd(ws=ctypes.c_void_p(0), wsb=0) == _lib.CP_ERR_WORKSPACE
    assert _bwd(wsb=1024) == _lib.CP_ERR_WORKSPACE
    cu = (ctypes.c_int32 * 3)(0, 600, 1024)
    assert _bwd(layout=_lib.CP_LAYOUT_STRIPED, cu=cu, n_docs=2) == _lib.CP_ERR_UNSUPPORTED
    assert len(lib().cp_last_error_string()) > 0


def test_ring_bwd_workspace_is_two_vectors_per_head():
    # D and LSE*log2(e), fp32 [hq][S] each, 256-byte aligned
    a = lambda x: (x + 255) // 256 * 256
    assert api.ring_attn_bwd_workspace_size(4096, 32, 8, 128, 4, "zigzag") == 2 * a(4096 * 32 * 4)


def _pair_bwd(n_q=256, n_k=256, hq=4, hkv=2, dh=128, qc=((0, 256),), kc=((0, 256),), parts=3, acc=0, dq=FAKE,
              dk=FAKE, lg=FAKE, mask=_lib.CP_MASK_CAUSAL, n_docs=0):
    qa = (_lib.cp_chunk * len(qc))(*[_lib.cp_chunk(a, b) for a, b in qc])
    ka = (_lib.cp_chunk * len(kc))(*[_lib.cp_chunk(a, b) for a, b in kc])
    return lib().cp_block_attn_bwd(FAKE, FAKE, FAKE, FAKE, lg, FAKE, n_q, n_k, hq, hkv, dh, qa, len(qc), ka, len(kc),
                                   mask, ctypes.c_void_p(0), n_docs, 0.0, dq, dk, FAKE, parts, acc,
                                   ctypes.c_void_p(0))


def test_block_bwd_rejects_bad_arguments():
    assert _pair_bwd(dh=96) == _lib.CP_ERR_UNSUPPORTED
    assert _pair_bwd(hq=3) == _lib.CP_ERR_INVALID_ARG
    assert _pair_bwd(n_q=0) == _lib.CP_ERR_INVALID_ARG
    assert _pair_bwd(parts=0) == _lib.CP_ERR_INVALID_ARG
    assert _pair_bwd(parts=4) == _lib.CP_ERR_INVALID_ARG
    assert _pair_bwd(acc=2) == _lib.CP_ERR_INVALID_ARG
    assert _pair_bwd(dq=ctypes.c_void_p(0)) == _lib.CP_ERR_INVALID_ARG          # dQ asked for, no buffer
    assert _pair_bwd(dk=ctypes.c_void_p(0)) == _lib.CP_ERR_INVALID_ARG          # dK/dV asked for, no buffer
    assert _pair_bwd(lg=MISALIGNED) == _lib.CP_ERR_ALIGNMENT
    assert _pair_bwd(mask=7) == _lib.CP_ERR_INVALID_ARG
    assert _pair_bwd(qc=((0, 100), (200, 100), (400, 56))) == _lib.CP_ERR_UNSUPPORTED  # three chunks
    assert _pair_bwd(qc=((0, 100),)) == _lib.CP_ERR_INVALID_ARG                 # chunks miss rows
    assert _pair_bwd(kc=((-1, 256),)) == _lib.CP_ERR_INVALID_ARG
    assert _pair_bwd(n_docs=2) == _lib.CP_ERR_INVALID_ARG                       # documents without the table
    L = lib()
    assert L.cp_attn_bwd_prep(FAKE, FAKE, FAKE, 128, 4, 96, FAKE, FAKE, None) == _lib.CP_ERR_UNSUPPORTED
    assert L.cp_attn_bwd_prep(FAKE, FAKE, FAKE, 0, 4, 128, FAKE, FAKE, None) == _lib.CP_ERR_INVALID_ARG
    assert L.cp_attn_bwd_prep(FAKE, FAKE, FAKE, 128, 4, 128, FAKE, ctypes.c_void_p(0), None) == _lib.CP_ERR_INVALID_ARG


def test_permute_and_merge_reject_bad_arguments():
    L = lib()
    # Ulysses head limit: P must divide the head count
    assert L.cp_ulysses_permute(FAKE, ctypes.c_void_p(1 << 30), 8, 1024, 4, 128, 2, 0, None) == _lib.CP_ERR_UNSUPPORTED
    assert L.cp_ulysses_permute(FAKE, ctypes.c_void_p(1 << 30), 4, 1022, 8, 128, 2, 0, None) == _lib.CP_ERR_INVALID_ARG
    assert L.cp_ulysses_permute(FAKE, FAKE, 4, 1024, 8, 128, 2, 0, None) == _lib.CP_ERR_INVALID_ARG  # overlap
    assert L.cp_zigzag_reorder(FAKE, ctypes.c_void_p(1 << 30), 4, 1020, 1, 16, 0, None) == _lib.CP_ERR_INVALID_ARG
    sz = ctypes.c_size_t(0)
    assert L.cp_ulysses_attn_workspace_size(1024, 32, 4, 128, 8, ctypes.byref(sz)) == _lib.CP_ERR_UNSUPPORTED
    parts = (ctypes.c_void_p * 1)(1 << 20)
    assert L.cp_lse_merge(0, parts, parts, 16, 2, 128, FAKE, FAKE, None, None) == _lib.CP_ERR_UNSUPPORTED
    assert L.cp_lse_merge(1, parts, parts, 16, 2, 96, FAKE, FAKE, None, None) == _lib.CP_ERR_UNSUPPORTED
    assert L.cp_lse_merge(1, parts, parts, 16, 2, 128, FAKE, FAKE, None, None) == _lib.CP_ERR_INVALID_ARG  # alias


# ------------------------------------------------------------ scheduler
@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "striped"])
@pytest.mark.parametrize("P", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("causal", [True, False])
def test_schedule_matches_bruteforce(layout, P, causal):
    S = 16 * P * 2
    sch = api.ring_schedule(S, P, layout, causal)
    cls = ref.pair_classes(S, P, layout, causal)
    for r in range(P):
        for t in range(P):
            j, live, tot = cls[(r, t)]
            i = r * P + t
            assert sch["src"][i] == j
            assert sch["live_pairs"][i] == live
            assert sch["launched"][i] == (1 if live > 0 else 0)


@pytest.mark.parametrize("layout,P,causal", [("zigzag", 4, True), ("contiguous", 4, True), ("zigzag", 16, True),
                                             ("zigzag", 4, False), ("contiguous", 8, False)])
def test_schedule_varlen_matches_bruteforce(layout, P, causal):
    S = 256 * (2 if P == 16 else 1)
    cu = [0, 3, 70, 71, 200, S]
    sch = api.ring_schedule(S, P, layout, causal, cu)
    cls = ref.pair_classes(S, P, layout, causal, cu)
    for (r, t), (j, live, _) in cls.items():
        assert sch["live_pairs"][r * P + t] == live
        assert sch["launched"][r * P + t] == (1 if live else 0)
        if live:
            # every query row that admits a key of the pair is computed
            qp = ref.shard_positions(S, P, layout, r)
            kp = ref.shard_positions(S, P, layout, j)
            rows_live = ref.explicit_mask(qp, kp, causal, cu).any(axis=1).sum()
            assert sch["q_rows"][r * P + t] >= rows_live


def test_schedule_skip_counts_for_the_workloads():
    # contiguous causal P=4: P(P+1)/2 live pairs; zigzag P=8: all P^2 live
    assert api.ring_schedule(32768, 4, "contiguous")["launched"].sum() == 10
    z = api.ring_schedule(65536, 8, "zigzag")
    assert z["launched"].sum() == 64
    c = 65536 // 16
    # off-diagonal zigzag pairs compute half the query rows (or all rows vs half the keys)
    assert set(np.unique(z["live_pairs"])) == {2 * c * c, 2 * c * c + c}


def test_live_pair_count_against_oracle():
    cu = [0, 5, 6, 40, 64]
    assert api.count_live_pairs(64, True, cu) == ref.live_pair_count(64, True, cu)
    assert api.count_live_pairs(64, True) == 64 * 65 // 2
    assert api.count_live_pairs(64, False) == 64 * 64
    assert api.count_live_pairs(131072, True) == 131072 * 131073 // 2


@settings(max_examples=60, deadline=None)
@given(st.data())
def test_schedule_random_problems_match_bruteforce(data):
    # random shard counts, layouts, masks and document tables: the host
    # scheduler's source shard, admitted-pair count and launch decision of
    # every (rank, step) equal the brute-force mask's
    layout = data.draw(st.sampled_from(["contiguous", "zigzag", "striped"]))
    P = data.draw(st.integers(1, 9))
    unit = 2 * P if layout == "zigzag" else P
    S = unit * data.draw(st.integers(1, max(1, 160 // unit)))
    causal = data.draw(st.booleans())
    cu = None
    if layout != "striped" and S > 1 and data.draw(st.booleans()):
        cu = [0] + sorted(set(data.draw(st.lists(st.integers(1, S - 1), max_size=5)))) + [S]
    sch = api.ring_schedule(S, P, layout, causal, cu)
    for (r, t), (j, live, _) in ref.pair_classes(S, P, layout, causal, cu).items():
        i = r * P + t
        assert sch["src"][i] == j
        assert sch["live_pairs"][i] == live
        assert sch["launched"][i] == (1 if live else 0)
