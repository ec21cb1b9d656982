"""GPU parity of the LSE merge against the oracle's fp64 fold."""
import numpy as np
import pytest
import torch

from context_exact_attention_step_b200 import api
from oracle import ref

from _util import compare, f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,rows,h,dh", [(1, 37, 3, 128), (4, 300, 8, 128), (7, 129, 4, 64), (10, 1024, 32, 128),
                                         (18, 100, 13, 64)])  # more partials than the kernel stages in shared memory
def test_merge_matches_oracle(n, rows, h, dh):
    g = torch.Generator().manual_seed(n * 1000 + rows)
    o = [torch.randn(rows, h, dh, generator=g) for _ in range(n)]
    l = [torch.randn(h, rows, generator=g) * 3 for _ in range(n)]
    # some partials see no key for some rows: LSE = -inf, O is garbage
    if n > 1:
        l[1][:, ::3] = -float("inf")
        o[1][::3] = float("nan")
    if n > 2:
        l[2][0, :] = -float("inf")
    og = [t.cuda() for t in o]
    lg = [t.cuda() for t in l]
    out, lse, o16 = api.lse_merge(og, lg, bf16_out=True)
    ow = np.stack([np.nan_to_num(t.double().numpy()) for t in o])
    want_o, want_l = ref.lse_merge(ow, np.stack([t.double().numpy() for t in l]))
    compare(out, lse, want_o, want_l, o_tol=1e-5, lse_tol=1e-5, what="merge")
    assert torch.equal(o16.cpu(), out.cpu().to(torch.bfloat16))


def test_merge_all_empty_rows():
    rows, h, dh = 64, 2, 128
    o = [torch.full((rows, h, dh), float("nan"), device="cuda") for _ in range(2)]
    l = [torch.full((h, rows), -float("inf"), device="cuda") for _ in range(2)]
    out, lse = api.lse_merge(o, l)
    assert torch.all(out == 0)
    assert torch.all(torch.isneginf(lse))
