"""Tolerance checks used to compare a result with the oracle -- TEST INFRASTRUCTURE ONLY.

Two bars:

* float32 workloads: relative error at most 1e-5, measured element by element against
  max(|ref_i|, rms(ref)) so that entries near zero do not make the ratio unbounded;
* bfloat16 workloads: absolute error at most 2e-2 on outputs of unit scale. Outputs here are
  not of unit scale (diffuse attention over thousands of rows shrinks them to ~0.02 RMS), so
  the error is divided by rms(ref) first -- otherwise a zero output would pass -- and the
  literal unscaled bound is checked as well.
"""
from __future__ import annotations

import numpy as np

F32_REL_TOL = 1e-5
BF16_SCALED_TOL = 2e-2


def rms(x: np.ndarray) -> float:
    x = np.asarray(x, dtype=np.float64)
    return float(np.sqrt(np.mean(x * x)))


def normwise_rel_error(got: np.ndarray, ref: np.ndarray) -> float:
    """max_i |got_i - ref_i| / max(|ref_i|, rms(ref))."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    denom = np.maximum(np.abs(ref), rms(ref))
    return float(np.max(np.abs(got - ref) / denom))


def scaled_max_error(got: np.ndarray, ref: np.ndarray) -> float:
    """max |got - ref| / rms(ref)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref)) / rms(ref))


def max_abs_error(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.max(np.abs(np.asarray(got, dtype=np.float64) - np.asarray(ref, dtype=np.float64))))


def per_vector_scaled_error(got: np.ndarray, ref: np.ndarray) -> float:
    """max over output vectors (last axis) of max |got - ref| / rms(ref vector): every head's
    output brought to unit scale on its own."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    r = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    return float(np.max(np.abs(got - ref) / np.maximum(r, 1e-30)))


def within(got: np.ndarray, ref: np.ndarray, dtype: str, per_vector: bool = True):
    """(ok, metric) for the workload's storage type ("f32" or "bf16").

    bf16: the error scaled by the rms of the whole output, the literal unscaled bound, and
    (``per_vector``) the error of every output vector scaled by its own rms, all <= 2e-2.
    """
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if got.shape != ref.shape or not np.all(np.isfinite(got)):
        return False, float("inf")
    if dtype == "f32":
        e = normwise_rel_error(got, ref)
        return e <= F32_REL_TOL, e
    e = scaled_max_error(got, ref)
    ok = e <= BF16_SCALED_TOL and max_abs_error(got, ref) <= BF16_SCALED_TOL
    if per_vector:
        ev = per_vector_scaled_error(got, ref)
        ok = ok and ev <= BF16_SCALED_TOL
        e = max(e, ev)
    return ok, e
