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


def within(got: np.ndarray, ref: np.ndarray, dtype: str, per_vector: bool = True,
           out_ulps: float = 0.0):
    """(ok, metric) for the workload's storage type ("f32" or "bf16").

    bf16: the error scaled by the rms of the whole output, the literal unscaled bound, and
    (``per_vector``) the error of every output vector scaled by its own rms, all <= 2e-2.
    ``out_ulps``: every element's error is first reduced by that many bfloat16 ulps of the
    expected value (the output format's own granularity; see PROMPT_OUTPUT_ULPS).
    """
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if got.shape != ref.shape or not np.all(np.isfinite(got)):
        return False, float("inf")
    if dtype == "f32":
        e = normwise_rel_error(got, ref)
        return e <= F32_REL_TOL, e
    if out_ulps:
        # the part of each error within out_ulps ulps of the expected value is not counted:
        # compare the expected value with got moved toward it by that much
        slack = out_ulps * bf16_ulp(ref)
        got = ref + np.sign(got - ref) * np.maximum(np.abs(got - ref) - slack, 0.0)
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


# A bf16 prompt (prefill) output: one query token's (H, d_v) output averages few keys in its
# first rows and many later, so its elements can reach several times the rms of the whole
# output or of one head's vector, where half an ulp of the bf16 result alone (0.39 % of the
# element at the top of a binade) exceeds 2e-2 of the rms. The tensor-core pipeline also holds
# P, K and V as bf16 MMA operands, once each. One ulp of the expected element is granted for
# those roundings together; everything beyond it must meet the 2e-2 bar.
PROMPT_OUTPUT_ULPS = 1.0

FP32_UNIT_ROUNDOFF = 2.0 ** -24


def bf16_rounding_ambiguous(x: np.ndarray, err: np.ndarray) -> np.ndarray:
    """True where a value computed as x with an error of at most err may round to another
    bfloat16 number than x itself: rounding is monotone, so that happens exactly when x - err
    and x + err round to different numbers."""
    from .mla_ref import round_bf16

    x = np.asarray(x, dtype=np.float64)
    err = np.broadcast_to(np.abs(np.asarray(err, dtype=np.float64)), x.shape)
    return round_bf16(x - err) != round_bf16(x + err)


def peaky_tolerance(Q: np.ndarray, rows: np.ndarray, w_uv: np.ndarray, kv_rank: int,
                    scale: float, j: int, ref_o: np.ndarray, ref_lat: np.ndarray,
                    amb_q: np.ndarray, amb_row: np.ndarray):
    """Elementwise tolerance for outputs dominated by one cached row j (a planted needle),
    against the oracle's bf16-query form (the exact arithmetic on the query rounded once to
    bfloat16, which is what a bf16 boundary stores).

    An implementation computes Q and row j in fp32 before rounding them to bfloat16. Where the
    exact value lies within that computation's error bound of a rounding boundary (amb_q,
    amb_row: see bf16_rounding_ambiguous), it may round to the neighbouring bfloat16 number.
    Through row j's score that moves the output to first order by d o / d s_j = p_j (V_j - o)
    times the score change, at most
        delta = scale * (sum over ambiguous k of ulp(Q_k) |row_jk| + |Q_k| ulp(row_jk)).
    The tolerance is 2e-2 of every output vector's rms plus twice that first-order change (the
    factor covers second-order terms and the other rows' far smaller shifts). With no
    ambiguous element it is the plain bf16 bar.
    Q (T, H, r + d_r) bf16-rounded query, rows (L, r + d_r); amb_q like Q, amb_row (r + d_r);
    ref_o (T, H, d_v) and ref_lat (T, H, r) the oracle's outputs for the same inputs.
    Returns (tol_o, tol_lat).
    """
    from .mla_ref import _causal_lengths, softmax

    Q = np.asarray(Q, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    T, H, _ = Q.shape
    L = rows.shape[0]
    keep = np.arange(L)[None, :] < _causal_lengths(L, T)[:, None]
    s = np.where(keep[:, None, :], (Q @ rows.T) * scale, -np.inf)
    pj = softmax(s)[:, :, j]                                                   # (T, H)
    rj = rows[j]
    uq = np.where(amb_q, bf16_ulp(Q), 0.0)
    ur = np.where(amb_row, bf16_ulp(rj), 0.0)
    delta = scale * (uq @ np.abs(rj) + np.abs(Q) @ ur)                         # (T, H)
    cj = rj[:kv_rank]
    Vj = np.einsum("hij,j->hi", np.asarray(w_uv, dtype=np.float64), cj)        # (H, d_v)
    sens_o = (delta * pj)[..., None] * np.abs(Vj[None] - ref_o)
    sens_lat = (delta * pj)[..., None] * np.abs(cj[None, None] - ref_lat)
    rms_o = np.sqrt(np.mean(ref_o ** 2, axis=-1, keepdims=True))
    rms_lat = np.sqrt(np.mean(ref_lat ** 2, axis=-1, keepdims=True))
    return (BF16_SCALED_TOL * rms_o + 2.0 * sens_o,
            BF16_SCALED_TOL * rms_lat + 2.0 * sens_lat)


def needle_ambiguity(q_nope: np.ndarray, w_uk: np.ndarray, Q_exact: np.ndarray,
                     row_j: np.ndarray, kv_rank: int):
    """Masks of the query and needle-row elements whose bfloat16 rounding an fp32
    implementation may do the other way.

    Q's latent part is a d_h-term fp32 sum of exact products of bf16 operands: its error is at
    most gamma_n sum |q_i w_i| with gamma_n = n u / (1 - n u), the textbook bound of recursive
    summation in any order, taken with u = 2^-23 (twice the fp32 unit roundoff, in case the
    tensor core truncates its partial sums). Its RoPE part and the row's RoPE part are rotated
    in double and rounded once (error below 2^-40 relative). The row's latent part is RMSNorm(x) * gamma in fp32: at most (r/2 + 8)
    units in the last fp32 place of the result (the mean of r squares, a reciprocal square root
    and two products).
    q_nope (T, H, d_h), w_uk (H, d_h, r), Q_exact (T, H, r + d_r) unrounded, row_j (r + d_r).
    """
    q_nope = np.asarray(q_nope, dtype=np.float64)
    w = np.asarray(w_uk, dtype=np.float64)
    Q_exact = np.asarray(Q_exact, dtype=np.float64)
    err_q = np.abs(Q_exact) * 2.0 ** -40
    # sum_i |q_nope[t, h, i]| |w_uk[h, i, c]| for every latent column c
    lat_err = np.einsum("thi,hic->thc", np.abs(q_nope), np.abs(w))
    d_h = q_nope.shape[-1]
    u = 2.0 * FP32_UNIT_ROUNDOFF
    g = d_h * u / (1.0 - d_h * u)
    err_q[..., :kv_rank] = g * lat_err
    row_j = np.asarray(row_j, dtype=np.float64)
    err_r = np.abs(row_j) * 2.0 ** -40
    err_r[:kv_rank] = (kv_rank / 2 + 8) * FP32_UNIT_ROUNDOFF * np.abs(row_j[:kv_rank])
    return bf16_rounding_ambiguous(Q_exact, err_q), bf16_rounding_ambiguous(row_j, err_r)
