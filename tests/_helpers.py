"""Shared test helpers (no method arithmetic here)."""

import numpy as np
import pytest
import torch

gpu = pytest.mark.gpu

BF16_O_TOL = 2e-2      # max-abs on O for bf16 inputs
BF16_LSE_TOL = 1e-3    # max-abs on LSE for bf16 inputs
F32_TOL = 1e-5         # max-abs for fp32 inputs
# Gradient tolerance for bf16 (not stated by the method's pages): the bf16 O
# tolerance, max-abs, relative to the largest reference magnitude when that
# exceeds 1 (dK / dV sums grow with the number of visible queries).
BF16_GRAD_TOL = 2e-2


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def max_abs(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):
        d = np.where(both_inf, 0.0, np.abs(a - b))
    return float(np.nanmax(np.where(np.isnan(d), np.inf, d))) if d.size else 0.0


def assert_max_abs(got, ref, tol, what=""):
    err = max_abs(got, ref)
    assert err <= tol, f"{what}: max-abs error {err:.3e} > {tol:.1e}"


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.linalg.norm(ref))
    return float(np.linalg.norm(got - ref)) / den if den > 0 else float(np.linalg.norm(got))


def assert_grad_close(got, ref, tol=BF16_GRAD_TOL, what=""):
    """Max-abs within tol x max(1, max|ref|); prints the scale and the
    relative L2 error beside it (shown with pytest -s or on failure)."""
    ref = np.asarray(ref, dtype=np.float64)
    scale = max(1.0, float(np.abs(ref).max()) if ref.size else 1.0)
    err = max_abs(got, ref)
    rl2 = rel_l2(got, ref) if ref.size else 0.0
    print(f"{what}: max-abs {err:.3e} (bound {tol:.1e} x scale {scale:.3f}), rel-L2 {rl2:.3e}")
    assert err <= tol * scale, \
        f"{what}: max-abs error {err:.3e} > {tol:.1e} x {scale:.2f} (rel-L2 {rl2:.3e})"


def assert_f32_close(got, ref, what=""):
    """fp32 inputs: max-abs within 1e-5 x max(1, max|ref|)."""
    assert_grad_close(got, ref, tol=F32_TOL, what=what)


def requires_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
