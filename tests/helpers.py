"""Shared helpers for the parity tests: conversions and the tolerance checks
(max abs error 1e-2 and mean abs error 1e-3 on outputs with unit-variance V,
relative error 1e-3 on rho, bit-exact block index)."""

import numpy as np
import torch

O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
RHO_REL = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a (bf16/fp32) tensor to a float64 NumPy array on the host."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def check_out(got: np.ndarray, want: np.ndarray, what: str, max_abs=O_MAX_ABS, mean_abs=O_MEAN_ABS, rel=0.0):
    """Element-wise |got - want| <= max_abs + rel * |want| and mean |got - want| <=
    mean_abs + rel * mean |want|.  rel = 0 is the plain bound; rel > 0 adds the
    bf16 rounding of outputs whose magnitude is beyond where half a bf16 ulp
    alone exceeds max_abs."""
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - want)
    over = err - (max_abs + rel * np.abs(want))
    assert over.max() <= 0.0, f"{what}: max abs err {err.max():.3e} > {max_abs} + {rel} |want|"
    mean_bound = mean_abs + rel * float(np.abs(want).mean())
    assert err.mean() <= mean_bound, f"{what}: mean abs err {err.mean():.3e} > {mean_bound:.3e}"
    return float(err.max()), float(err.mean())


def check_rho(got: np.ndarray, want: np.ndarray, what="rho", rel=RHO_REL):
    assert got.shape == want.shape
    assert np.all(np.isfinite(got))
    err = np.abs(got - want) / np.maximum(np.abs(want), 1e-30)
    assert err.max() <= rel, f"{what}: max rel err {err.max():.3e} > {rel}"
    return float(err.max())
