"""Helpers shared by the GPU parity tests."""
import numpy as np
import torch

# tolerances of the forward for bf16 inputs with fp32 accumulation: O max-abs
# 2e-2 and LSE max-abs 1e-3
O_TOL = 2e-2
LSE_TOL = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def compare(o_gpu, lse_gpu, o_ref, lse_ref, o_tol=O_TOL, lse_tol=LSE_TOL, what=""):
    """Element-by-element comparison; -inf LSE must match exactly."""
    o = f64(o_gpu) if isinstance(o_gpu, torch.Tensor) else o_gpu
    l = f64(lse_gpu) if isinstance(lse_gpu, torch.Tensor) else lse_gpu
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert l.shape == lse_ref.shape, (l.shape, lse_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite O"
    ninf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(l), ninf_ref), f"{what}: -inf LSE pattern differs"
    fin = ~ninf_ref
    err_o = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    err_l = float(np.max(np.abs(l[fin] - lse_ref[fin]))) if fin.any() else 0.0
    assert err_o <= o_tol, f"{what}: O max-abs error {err_o:.3e} > {o_tol}"
    assert err_l <= lse_tol, f"{what}: LSE max-abs error {err_l:.3e} > {lse_tol}"
    return err_o, err_l


# gradients: relative to the largest entry of the reference tensor (the
# derivation of 2e-2 sits with the backward parity tests)
GRAD_REL_TOL = 2e-2


def check_grad(got, want, what, rel_tol=GRAD_REL_TOL):
    got = f64(got) if isinstance(got, torch.Tensor) else got
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    scale = float(np.max(np.abs(want))) if want.size else 0.0
    err = float(np.max(np.abs(got - want))) if want.size else 0.0
    assert err <= rel_tol * max(scale, 1e-6), f"{what}: max-abs error {err:.3e} vs max |ref| {scale:.3e}"
    return err / max(scale, 1e-30)
