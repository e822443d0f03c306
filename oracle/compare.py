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


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bfloat16 numbers at |x| (8 significant bits): 2^(floor(log2|x|) - 7)."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    out = np.zeros_like(x)
    nz = x > 0
    out[nz] = 2.0 ** (np.floor(np.log2(np.maximum(x[nz], 2.0 ** -126))) - 7)
    return out


def peaky_tolerance(Q: np.ndarray, rows: np.ndarray, w_uv: np.ndarray, kv_rank: int,
                    scale: float, j: int, ref_o: np.ndarray, ref_lat: np.ndarray):
    """Elementwise tolerance for outputs dominated by one cached row j (a planted needle).

    Two correct bf16 implementations may round the packed query Q or row j differently by one
    bfloat16 ulp. Through row j's score that moves the output to first order by
    d o / d s_j = p_j (V_j - o) times the score change, at most
        delta = scale * sum_k (ulp(Q_k) |row_jk| + |Q_k| ulp(row_jk)).
    The tolerance is 2e-2 of every output vector's rms plus twice that first-order change
    (the factor covers second-order terms and the other rows' far smaller shifts).
    Q (T, H, r + d_r) exact, rows (L, r + d_r); ref_o (T, H, d_v) and ref_lat (T, H, r) are the
    oracle's outputs for the same inputs. Returns (tol_o, tol_lat).
    """
    from .mla_ref import _causal_lengths, softmax

    Q = np.asarray(Q, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    T, H, _ = Q.shape
    L = rows.shape[0]
    keep = np.arange(L)[None, :] < _causal_lengths(L, T)[:, None]
    s = np.where(keep[:, None, :], np.einsum("thd,ld->thl", Q, rows) * scale, -np.inf)
    pj = softmax(s)[:, :, j]                                                   # (T, H)
    rj = rows[j]
    delta = scale * (bf16_ulp(Q) @ np.abs(rj) + np.abs(Q) @ bf16_ulp(rj))      # (T, H)
    cj = rj[:kv_rank]
    Vj = np.einsum("hij,j->hi", np.asarray(w_uv, dtype=np.float64), cj)        # (H, d_v)
    sens_o = (delta * pj)[..., None] * np.abs(Vj[None] - ref_o)
    sens_lat = (delta * pj)[..., None] * np.abs(cj[None, None] - ref_lat)
    rms_o = np.sqrt(np.mean(ref_o ** 2, axis=-1, keepdims=True))
    rms_lat = np.sqrt(np.mean(ref_lat ** 2, axis=-1, keepdims=True))
    return (BF16_SCALED_TOL * rms_o + 2.0 * sens_o,
            BF16_SCALED_TOL * rms_lat + 2.0 * sens_lat)
