"""GPU parity of the layout kernels: bit-exact against the oracle's numpy
index formulas (Ulysses transpose, zigzag reorder), through the C ABI."""
import numpy as np
import pytest
import torch

from context_exact_attention_step_b200 import api, synth
from oracle import ref

pytestmark = pytest.mark.gpu


def bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy()
    return t.view(torch.int32).numpy() if t.element_size() == 4 else t.numpy()


@pytest.mark.parametrize("P,S,h,dh,dtype", [
    (4, 64, 8, 128, torch.bfloat16),
    (8, 1024, 32, 128, torch.bfloat16),
    (8, 1024, 8, 128, torch.bfloat16),      # GQA K/V: one head per rank
    (2, 96, 4, 64, torch.float32),
    (4, 40, 4, 3, torch.bfloat16),          # odd row size: narrow copy units
    (1, 32, 4, 16, torch.bfloat16),         # P = 1 is the identity
])
def test_ulysses_permute_bit_exact(P, S, h, dh, dtype):
    x = synth.normal((S, h, dh), 11, 1.0, dtype).cuda()
    y = api.ulysses_permute(x, P, "seq_to_head")
    want = ref.ulysses_seq_to_head(bits(x).reshape(P, S // P, h, dh), P)
    assert np.array_equal(bits(y), want)
    back = api.ulysses_permute(y, P, "head_to_seq")
    assert np.array_equal(bits(back), bits(x))


def test_ulysses_permute_full_size_q():
    # the 128K-token GQA workload's Q (32 heads) and K (8 heads), P = 8
    P, S, dh = 8, 131072, 128
    for h, seed in ((32, 1), (8, 2)):
        x = synth.normal((S, h, dh), seed, 0.5, torch.bfloat16).cuda()
        y = api.ulysses_permute(x, P, "seq_to_head")
        # spot-check whole rows of every (r, p) block against the formula
        xb = x.view(P, S // P, h, dh)
        for r in range(P):
            for p in range(P):
                for s in (0, 1, S // P - 1, 777 % (S // P)):
                    got = y[r, p * (S // P) + s]
                    exp = xb[p, s, r * (h // P):(r + 1) * (h // P)]
                    assert torch.equal(got.view(torch.int16), exp.view(torch.int16))
        back = api.ulysses_permute(y, P, "head_to_seq")
        assert torch.equal(back.view(torch.int16), x.view(torch.int16))


def test_ulysses_permute_full_size_bit_exact():
    """The whole 128K-token GQA workload (32 query / 8 KV heads, dh 128, P = 8):
    seq->head of Q, K and V and head->seq of an fp32 O, every element against
    the oracle's index formula."""
    P, S, dh = 8, 131072, 128
    n = S // P
    for h, seed in ((32, 1), (8, 2), (8, 3)):
        x = synth.normal((S, h, dh), seed, 0.5, torch.bfloat16).cuda()
        y = api.ulysses_permute(x, P, "seq_to_head")
        assert np.array_equal(bits(y), ref.ulysses_seq_to_head(bits(x).reshape(P, n, h, dh), P)), (h, seed)
        del x, y
    o = synth.normal((P, S, 32 // P, dh), 4, 1.0, torch.float32).cuda()
    back = api.ulysses_permute(o, P, "head_to_seq")
    assert np.array_equal(bits(back).reshape(P, n, 32, dh), ref.ulysses_head_to_seq(bits(o), P))


def test_zigzag_full_size_bit_exact():
    """The 64K-token zigzag workload (32 heads, dh 128, P = 8): the forward
    reorder of a bf16 Q and the inverse of an fp32 O and LSE, every element
    against the oracle's chunk order."""
    P, S, h, dh = 8, 65536, 32, 128
    q = synth.normal((S, h, dh), 1, 0.5, torch.bfloat16).cuda()
    assert np.array_equal(bits(api.zigzag_reorder(q, P)), ref.zigzag_reorder(bits(q), P))
    del q
    o = synth.normal((S, h, dh), 5, 1.0, torch.float32).cuda()
    assert np.array_equal(bits(api.zigzag_reorder(o, P, inverse=True)), ref.zigzag_restore(bits(o), P))
    del o
    lse = synth.normal((h, S), 6, 1.0, torch.float32).cuda()
    got = api.zigzag_reorder(lse, P, inverse=True, seq_dim=1)
    assert np.array_equal(bits(got), ref.zigzag_restore(bits(lse), P, axis=1))


@pytest.mark.parametrize("P,S,shape,dtype", [
    (4, 64, (8, 128), torch.bfloat16),
    (8, 4096, (32, 128), torch.bfloat16),
    (2, 40, (3,), torch.float32),
    (3, 36, (2, 5), torch.bfloat16),
])
def test_zigzag_bit_exact(P, S, shape, dtype):
    x = synth.normal((S,) + shape, 5, 1.0, dtype).cuda()
    y = api.zigzag_reorder(x, P)
    assert np.array_equal(bits(y), ref.zigzag_reorder(bits(x), P))
    z = api.zigzag_reorder(y, P, inverse=True)
    assert np.array_equal(bits(z), bits(x))


@pytest.mark.parametrize("P,S,shape,dtype", [
    (4, 64, (8, 128), torch.bfloat16),
    (8, 4096, (32, 128), torch.bfloat16),
    (3, 36, (2, 5), torch.bfloat16),
])
def test_striped_bit_exact(P, S, shape, dtype):
    x = synth.normal((S,) + shape, 6, 1.0, dtype).cuda()
    y = api.striped_reorder(x, P)
    assert np.array_equal(bits(y), np.take(bits(x), ref.striped_order(S, P), axis=0))
    assert np.array_equal(bits(api.striped_reorder(y, P, inverse=True)), bits(x))
    lse = synth.normal((4, S), 7, 1.0, torch.float32).cuda()
    yl = api.striped_reorder(lse, P, seq_dim=1)
    assert np.array_equal(bits(yl), np.take(bits(lse), ref.striped_order(S, P), axis=1))
    assert torch.equal(api.striped_reorder(yl, P, inverse=True, seq_dim=1), lse)


def test_zigzag_lse_rows():
    P, S, h = 8, 4096, 32
    lse = synth.normal((h, S), 9, 1.0, torch.float32).cuda()
    y = api.zigzag_reorder(lse, P, seq_dim=1)
    assert np.array_equal(bits(y), ref.zigzag_reorder(bits(lse), P, axis=1))
    assert torch.equal(api.zigzag_reorder(y, P, inverse=True, seq_dim=1), lse)


@pytest.mark.parametrize("P,elem", [(2, torch.bfloat16), (4, torch.float32), (8, torch.bfloat16)])
def test_head_block_split_bit_exact(P, elem):
    n, h, dh = 300, 16, 64
    x = synth.normal((n, h, dh), 9, 1.0, dtype=torch.float32).to(elem)
    y = api.head_block_split(x.cuda(), P)
    want = x.reshape(n, P, h // P, dh).permute(1, 0, 2, 3).contiguous()
    assert torch.equal(y.cpu(), want)
    back = api.head_block_split(y, P, inverse=True)
    assert torch.equal(back.cpu(), x)
