"""Failure detection on the GPU without faulting it: a kernel whose barrier
wait can never complete must give up after its bounded time, report through
the device error word, and leave the context usable for the next launch."""
import numpy as np
import pytest
import torch

from context_exact_attention_step_b200 import api, synth
from oracle import ref

from _util import compare, f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    api.device_error(clear=True)
    api.selftest_wait_timeout(2_000_000)  # 2 ms
    torch.cuda.synchronize()
    assert api.device_error(clear=True) & 1
    assert api.device_error(clear=False) == 0
    # the context is still usable: a block pair runs and matches the oracle
    q = synth.normal((256, 2, 128), 1, 0.5)
    k = synth.normal((256, 2, 128), 2, 0.5)
    v = synth.normal((256, 2, 128), 3, 0.5)
    o, lse = api.block_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    want_o, want_l = ref.attention(f64(q), f64(k), f64(v), causal=True)
    compare(o, lse, want_o, want_l, what="after timeout")
