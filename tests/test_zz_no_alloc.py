"""The no-allocation ring entry point against the workspace entry point.

cp_ring_attn_fwd_noalloc exists for callers that may not allocate device
memory while they run (a plugin inside an application that owns the device
memory budget, a latency-critical loop where an allocation would stall the
GPU).  It keeps the ring steps' partial results in a fixed scratch array
inside the library instead of a caller workspace.  These tests call it
through the C ABI twice in a row, on different problems, and check each
result against cp_ring_attn_fwd on the same inputs; the second call shows
that what the first call left in the shared scratch does not leak into the
next result.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from context_exact_attention_step_b200 import _lib, api, synth

from _util import compare

pytestmark = pytest.mark.gpu


def _inputs(S, hq, hkv, dh, P, layout, dtype, seeds):
    q, k, v = synth.qkv(S, hq, hkv, dh, std=0.5 if dtype == torch.bfloat16 else 1.0, dtype=dtype, seeds=seeds)
    return tuple(t.cuda() for t in (q, k, v))


@pytest.fixture(scope="module", autouse=True)
def built():
    import __graft_entry__
    __graft_entry__.build()


def test_noalloc_matches_workspace_path_two_calls_in_a_row():
    cases = [
        # (S, hq, hkv, dh, P, layout, dtype, cu_seqlens, seeds)
        (4096, 8, 4, 128, 4, "zigzag", torch.bfloat16, None, (11, 12, 13)),
        (1024, 4, 4, 64, 4, "contiguous", torch.float32, [0, 300, 301, 1024], (21, 22, 23)),
    ]
    for S, hq, hkv, dh, P, layout, dtype, cu, seeds in cases:
        need = api.ring_attn_workspace_size(S, hq, hkv, dh, P, layout, True, dtype, cu)
        assert need <= _lib_scratch_bytes()
        q, k, v = _inputs(S, hq, hkv, dh, P, layout, dtype, seeds)
        o_ref, lse_ref = api.ring_attn_fwd(q, k, v, P, layout, True, cu)
        o_na, lse_na = api.ring_attn_fwd_noalloc(q, k, v, P, layout, True, cu)
        torch.cuda.synchronize()
        assert api.device_error() == 0
        compare(o_na, lse_na, o_ref.double().cpu().numpy(), lse_ref.double().cpu().numpy(),
                what=f"noalloc {layout} S={S}")


def _lib_scratch_bytes():
    return 64 << 20


def test_noalloc_rejects_problems_larger_than_its_scratch():
    # the 32K-token workload needs ~1.3 GB of partials: far above the scratch
    L = _lib.lib()
    fake = ctypes.c_void_p(1 << 20)
    st = L.cp_ring_attn_fwd_noalloc(fake, fake, fake, _lib.CP_BF16, 32768, 32, 32, 128, 4,
                                    _lib.CP_LAYOUT_CONTIGUOUS, _lib.CP_MASK_CAUSAL, None, None, 0, 0.0, fake, fake,
                                    None)
    assert st == _lib.CP_ERR_WORKSPACE
    msg = L.cp_last_error_string().decode()
    assert "scratch" in msg and str(64 << 20) in msg
