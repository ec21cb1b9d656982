"""The no-allocation ring entry point against the workspace entry point.

cp_ring_attn_fwd_noalloc exists for callers that may not allocate device
memory while they run (a plugin inside an application that owns the device
memory budget, a latency-critical loop where an allocation would stall the
GPU).  It keeps the ring steps' partial results in a fixed scratch array
inside the library instead of a caller workspace.  These tests call it
through the C ABI twice in a row, on different problems (the larger one
first, so that its leftovers sit under the smaller one), and check each
result against cp_ring_attn_fwd on the same inputs bit for bit: both run the
same deterministic kernels, so any difference would be stale scratch leaking
into the result.  Each result is also compared with the oracle.  This file
is collected last on purpose.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from context_exact_attention_step_b200 import _lib, api, synth
from oracle import ref

from _util import compare

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _scratch_bytes_from_header():
    """CP_NOALLOC_SCRATCH_BYTES as include/cp_attn.h defines it."""
    with open(os.path.join(ROOT, "include", "cp_attn.h")) as f:
        m = re.search(r"#define\s+CP_NOALLOC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", f.read())
    assert m, "CP_NOALLOC_SCRATCH_BYTES not found in include/cp_attn.h"
    return int(m.group(1)) << int(m.group(2))


@pytest.fixture(scope="module", autouse=True)
def built():
    import __graft_entry__
    __graft_entry__.build()


def _case(S, hq, hkv, dh, P, layout, dtype, cu, seeds):
    """Natural-order inputs, their storage order for `layout`, and the
    oracle's result in storage order."""
    std = 0.5 if dtype == torch.bfloat16 else 1.0
    q, k, v = synth.qkv(S, hq, hkv, dh, std=std, dtype=dtype, seeds=seeds)
    # the kernels round fp32 inputs to bf16: the oracle takes the same values
    qn, kn, vn = (t.to(torch.bfloat16).double().numpy() for t in (q, k, v))
    o_nat, lse_nat = ref.attention(qn, kn, vn, causal=True, cu_seqlens=cu)
    if layout == "zigzag":
        order = ref.zigzag_order(S, P)
        q, k, v = (t[torch.from_numpy(order)] for t in (q, k, v))
        o_ref, lse_ref = o_nat[order], lse_nat[:, order]
    else:
        o_ref, lse_ref = o_nat, lse_nat
    return tuple(t.contiguous().cuda() for t in (q, k, v)), o_ref, lse_ref


def test_noalloc_matches_workspace_path_two_calls_in_a_row():
    scratch = _scratch_bytes_from_header()
    cases = [
        # (S, hq, hkv, dh, P, layout, dtype, cu_seqlens, seeds): larger scratch need first
        (4096, 8, 4, 128, 4, "zigzag", torch.bfloat16, None, (11, 12, 13)),
        (1024, 4, 4, 64, 4, "contiguous", torch.float32, [0, 300, 301, 1024], (21, 22, 23)),
    ]
    needs = [api.ring_attn_workspace_size(S, hq, hkv, dh, P, layout, True, dtype, cu)
             for S, hq, hkv, dh, P, layout, dtype, cu, _ in cases]
    assert needs[0] > needs[1] and needs[0] <= scratch
    for S, hq, hkv, dh, P, layout, dtype, cu, seeds in cases:
        (q, k, v), o_ora, lse_ora = _case(S, hq, hkv, dh, P, layout, dtype, cu, seeds)
        o_ref, lse_ref = api.ring_attn_fwd(q, k, v, P, layout, True, cu)
        o_na, lse_na = api.ring_attn_fwd_noalloc(q, k, v, P, layout, True, cu)
        torch.cuda.synchronize()
        assert api.device_error() == 0
        assert torch.equal(o_na, o_ref), f"noalloc {layout} S={S}: O differs from the workspace path"
        assert torch.equal(lse_na, lse_ref), f"noalloc {layout} S={S}: LSE differs from the workspace path"
        compare(o_na, lse_na, o_ora, lse_ora, what=f"noalloc {layout} S={S} vs oracle")


def test_noalloc_rejects_problems_larger_than_its_scratch():
    # the 32K-token workload needs ~1.3 GB of partials: far above the scratch
    scratch = _scratch_bytes_from_header()
    L = _lib.lib()
    fake = ctypes.c_void_p(1 << 20)
    st = L.cp_ring_attn_fwd_noalloc(fake, fake, fake, _lib.CP_BF16, 32768, 32, 32, 128, 4,
                                    _lib.CP_LAYOUT_CONTIGUOUS, _lib.CP_MASK_CAUSAL, None, None, 0, 0.0, fake, fake,
                                    None)
    assert st == _lib.CP_ERR_WORKSPACE
    msg = L.cp_last_error_string().decode()
    assert "scratch" in msg and str(scratch) in msg
