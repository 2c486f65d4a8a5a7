"""Parity helpers: tolerance policy and sub-problem extraction for sampled checks.

Tolerances ("Results must match the oracle ... max |err| <= 1e-5 in fp32 and <= 2e-2
relative (fp32 accumulate) in bf16"):
  * bf16: per tensor, max_i |g_i - r_i| / max(|r_i|, rms(r)) <= 2e-2 (the rms floor
    keeps near-zero outputs from dividing by ~0);
  * fp32: max_i |g_i - r_i| <= 1e-5 for y and dx; for the fp32 reductions dz, dU and
    dw the bound is scaled by max(1, max|r|), since their magnitude grows with the
    number of summed terms.
"""
from __future__ import annotations

import numpy as np
import torch

BF16_REL = 2e-2
F32_ABS = 1e-5


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref)))
    den = np.maximum(np.abs(ref), max(rms, 1e-30))
    return float(np.max(np.abs(got - ref) / den))


def abs_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref))) if ref.size else 0.0


def assert_close(got, ref, dtype: str, what: str, reduction: bool = False):
    got = f64(got) if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, "%s: shape %s vs %s" % (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "%s: non-finite output" % what
    if dtype == "f32":
        tol = F32_ABS * (max(1.0, float(np.max(np.abs(ref)))) if reduction else 1.0)
        e = abs_err(got, ref)
        assert e <= tol, "%s: max|err| %.3e > %.1e" % (what, e, tol)
    else:
        e = rel_err(got, ref)
        assert e <= BF16_REL, "%s: rel err %.3e > %.0e" % (what, e, BF16_REL)
    return e


def window(T: int, t: int, W: int):
    """Token range [t0, t+1) that determines y_t (and dz_t)."""
    return max(0, t - W + 1), t + 1


def future(T: int, s: int, W: int):
    """Token range [s, e) that determines dx_s."""
    return s, min(s + W, T)
