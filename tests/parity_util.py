"""Shared helpers of the GPU parity tests: error metrics and tolerances.

Tolerances (fixed before any kernel was measured):
  * float32 I/O:  max relative error <= 1e-4, relative error of element i
    being |d_i| / max(|ref_i|, 1e-3 * max|ref|) -- the floor keeps near-zero
    outputs from dominating;
  * bf16 I/O (float32 accumulation and state): normalised max-abs error
    max|d| / max|ref| <= 2e-2;
  * decode state (float32, in place): max|d| / max|ref| <= 1e-5;
  * conv-cache columns are copies of inputs: bit-exact.
Final states and gradients are sums of many terms with cancellation: an
element far below its tensor's scale carries the float32 rounding of terms at
that scale.  For float32 I/O they are therefore held to 1e-4 normalised
max-abs (the implementation's accuracy relative to the tensor's scale) and,
so that small elements are still watched, to 1e-3 floored relative error
(TOL_F32_REL_SUMS; measured up to 2e-4 on float32 summation).  For bf16 I/O
they take the bf16 bound, 2e-2 normalised max-abs.
"""
from __future__ import annotations

import numpy as np
import torch

TOL_F32_REL = 1e-4
TOL_BF16_NMA = 2e-2
TOL_STATE_F32 = 1e-5
TOL_F32_NMA_SUMS = 1e-4
TOL_F32_REL_SUMS = 1e-3


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def norm_max_abs(got, ref) -> float:
    got, ref = f64(got), f64(ref)
    den = float(np.max(np.abs(ref))) if ref.size else 1.0
    return float(np.max(np.abs(got - ref))) / max(den, 1e-300) if ref.size else 0.0


def rel_err_floored(got, ref) -> float:
    got, ref = f64(got), f64(ref)
    if not ref.size:
        return 0.0
    floor = 1e-3 * float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), max(floor, 1e-300))))


def assert_output(got, ref, dtype: str, what: str):
    """y-style outputs: fp32 relative bound or bf16 normalised max-abs bound."""
    if dtype == "f32":
        e = rel_err_floored(got, ref)
        assert e <= TOL_F32_REL, f"{what}: relative error {e:.3e} > {TOL_F32_REL:.0e}"
    else:
        e = norm_max_abs(got, ref)
        assert e <= TOL_BF16_NMA, f"{what}: normalised max-abs error {e:.3e} > {TOL_BF16_NMA:.0e}"
    assert np.all(np.isfinite(f64(got))), f"{what}: non-finite values"
    return e


def assert_state(got, ref, dtype: str, what: str):
    """A final state or a gradient (sums with cancellation): for float32 I/O
    1e-4 normalised max-abs and 1e-3 floored relative error; for bf16 I/O the
    bf16 normalised max-abs bound."""
    if dtype == "f32":
        e = norm_max_abs(got, ref)
        r = rel_err_floored(got, ref)
        assert e <= TOL_F32_NMA_SUMS and r <= TOL_F32_REL_SUMS, \
            f"{what}: normalised error {e:.3e} (bound {TOL_F32_NMA_SUMS:.0e}), " \
            f"floored relative {r:.3e} (bound {TOL_F32_REL_SUMS:.0e})"
    else:
        e = norm_max_abs(got, ref)
        assert e <= TOL_BF16_NMA, f"{what}: normalised max-abs error {e:.3e} > {TOL_BF16_NMA:.0e}"
    assert np.all(np.isfinite(f64(got))), f"{what}: non-finite values"
    return e


def cuda(t):
    return None if t is None else t.to("cuda", non_blocking=False)
