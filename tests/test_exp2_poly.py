"""The softmax kernel's software 2^x (FMA-pipe path), emulated in float32 on
the CPU step by step, against the exact 2^x: relative error within the bound
printed by csrc/gen_exp2_poly.py over the whole input range the kernel feeds
it, and the bit-level range reduction exact for every integer part."""
import numpy as np

C = [np.float32(9.999280572e-01), np.float32(6.932609677e-01), np.float32(2.426111251e-01),
     np.float32(5.517166853e-02)]


def fma32(a, b, c):
    return (a.astype(np.float64) * b + c).astype(np.float32)


def exp2_poly(x):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = fma32(n, np.float32(-1.0), x)
    p = fma32(f, C[3], C[2])
    p = fma32(p, f, C[1])
    p = fma32(p, f, C[0])
    bits = p.view(np.int32).astype(np.int64) + ((t.view(np.int32).astype(np.int64) << 23) & 0xFFFFFFFF)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_bound_over_kernel_range():
    x = np.concatenate([np.linspace(-125, 64, 2_000_001, dtype=np.float32),
                        np.float32(np.random.default_rng(0).uniform(-125, 64, 200_000))])
    got = exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1)
    assert rel.max() < 8e-5, rel.max()


def test_integer_inputs_are_nearly_exact_powers_of_two():
    x = np.arange(-125, 65, dtype=np.float32)
    got = exp2_poly(x).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1) < 8e-5)
    assert np.all(got > 0)


def test_below_range_is_tiny_and_positive():
    got = exp2_poly(np.array([-126.0, -500.0, -1e30], dtype=np.float32)).astype(np.float64)
    assert np.all(got > 0) and np.all(got < 3e-38)
