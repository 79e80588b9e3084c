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


def assert_grad_close(got, ref, tol=BF16_GRAD_TOL, what=""):
    ref = np.asarray(ref, dtype=np.float64)
    scale = max(1.0, float(np.abs(ref).max()) if ref.size else 1.0)
    err = max_abs(got, ref)
    assert err <= tol * scale, f"{what}: max-abs error {err:.3e} > {tol:.1e} x {scale:.2f}"


def requires_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
