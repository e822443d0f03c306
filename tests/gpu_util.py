"""Helpers for the GPU parity tests: expected values come only from the CPU oracle."""
import numpy as np
import torch

import mla_inputs as mi
from oracle import compare, mla_ref as ref


def oracle_sequence(state, b: int, form: str = "naive"):
    """The oracle's result for sequence b of a DecodeState, from the same host inputs."""
    w = state.w
    ckv, kr, qn, qr = state.host_draws[b]
    return ref.decode_sequence_from_raw(ckv, kr, qn, qr, state.w_uk_host, state.w_uv_host,
                                        state.gamma_host, w.softmax_scale, w.rms_eps, w.rope_base,
                                        store_bf16=(w.dtype == "bf16"), form=form)


def check_sequence(state, b: int, form: str = "naive", lse_tol=None, peaky: bool = False):
    """Compare o, out_latent and lse of sequence b with the oracle; returns the error metrics.

    Tolerance: fp32 1e-5 relative; bf16 2e-2 on unit-scaled outputs (oracle.compare.within).
    peaky: one planted row takes most of the attention weight, which amplifies one-ulp
    rounding differences of the bf16 query; the elementwise tolerance of
    oracle.compare.peaky_tolerance applies instead.
    """
    exp = oracle_sequence(state, b, form)
    sl = state.tokens_of(b)
    o = state.o[sl].float().cpu().numpy()
    lat = state.out_latent[sl].cpu().numpy()
    lse = state.lse[sl].cpu().numpy()
    dt = state.w.dtype
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lat)), f"seq {b}: non-finite output"
    if peaky:
        # one needle row dominates: compare with the oracle's bf16-query form (the exact
        # arithmetic on the query rounded once to bfloat16, as the boundary stores it) under
        # the plain bar plus the first-order effect of the query and needle-row elements whose
        # rounding an fp32 computation may do the other way (oracle.compare.peaky_tolerance)
        w = state.w
        ckv, kr, qn, qr = state.host_draws[b]
        n = ckv.shape[0]
        j = state.needle_rows[b]
        exp = ref.decode_sequence_bf16_query(ckv, kr, qn, qr, state.w_uk_host, state.w_uv_host,
                                             state.gamma_host, w.softmax_scale, w.rms_eps,
                                             w.rope_base)
        rows = ref.cache_rows(ckv, kr, state.gamma_host, np.arange(n), w.rms_eps, w.rope_base,
                              True)
        Qx = ref.absorb_ref(qn, qr, np.arange(n - w.new_tokens, n), state.w_uk_host, w.rope_base)
        amb_q, amb_r = compare.needle_ambiguity(qn, state.w_uk_host, Qx, rows[j], w.kv_rank)
        tol_o, tol_l = compare.peaky_tolerance(ref.round_bf16(Qx), rows, state.w_uv_host,
                                               w.kv_rank, w.softmax_scale, j, exp.o, exp.o_lat,
                                               amb_q, amb_r)
        widen = needle_widening(tol_o, exp.o)
        assert widen <= NEEDLE_MAX_WIDENING, f"seq {b}: needle tolerance {widen:.2f}x the plain bar"
        assert np.all(np.abs(o - exp.o) <= tol_o), f"seq {b}: output outside the needle tolerance"
        assert np.all(np.abs(lat - exp.o_lat) <= tol_l), f"seq {b}: latent outside the needle tolerance"
        e_o = float(np.max(np.abs(o - exp.o) / (compare.BF16_SCALED_TOL * _vec_rms(exp.o))))
        e_l = float(np.max(np.abs(lat - exp.o_lat) / (compare.BF16_SCALED_TOL * _vec_rms(exp.o_lat))))
    else:
        ok_o, e_o = compare.within(o, exp.o, dt)
        ok_l, e_l = compare.within(lat, exp.o_lat, dt)
        assert ok_o, f"seq {b}: output error {e_o}"
        assert ok_l, f"seq {b}: latent output error {e_l}"
    e_lse = float(np.max(np.abs(lse - exp.lse)))
    tol = lse_tol if lse_tol is not None else (2e-2 if dt == "bf16" else 1e-5 * max(1.0, float(np.max(np.abs(exp.lse)))))
    if not peaky:
        assert e_lse <= tol, f"seq {b}: lse error {e_lse}"
    return e_o, e_l, e_lse


# The needle tolerance may exceed the plain 2e-2 bar only by the first-order effect of
# ambiguous roundings; on the needle inputs of the tests that is at most about 2.2x the bar.
NEEDLE_MAX_WIDENING = 4.0


def _vec_rms(x):
    return np.sqrt(np.mean(np.asarray(x, dtype=np.float64) ** 2, axis=-1, keepdims=True))


def needle_widening(tol, ref_out) -> float:
    """max over elements of the needle tolerance over the plain bar (2e-2 of its vector's rms)."""
    return float(np.max(tol / (compare.BF16_SCALED_TOL * _vec_rms(ref_out))))


def dev_err(state) -> int:
    torch.cuda.synchronize()
    return int(state.dev_err.item())


def layer_raw(w: mi.Workload, seed: int = 0):
    """Projections of seeded hidden states by the oracle's front end (small workloads)."""
    d = mi.layer_draw(w, seed)
    p = ref.project_layer(d.x, w.num_heads, w.head_dim, w.rope_dim, d.w_dkv, d.w_kr, d.w_qr,
                          w_q=d.w_q, w_dq=d.w_dq, w_uq=d.w_uq, gamma_q=d.gamma_q, eps=w.rms_eps)
    rows = mi.total_rows(w, seed)
    T = w.new_tokens
    H = w.num_heads
    raw = dict(w_uk=d.w_uk.reshape(H, w.head_dim, w.kv_rank).astype(np.float32),
               w_uv=d.w_uv.reshape(H, w.head_dim_v, w.kv_rank).astype(np.float32),
               gamma=d.gamma_kv.astype(np.float32), ckv_raw=[], krope_raw=[], q_nope=[],
               q_rope_raw=[])
    for b in range(w.batch):
        n = int(rows[b])
        raw["ckv_raw"].append(p.ckv_raw[b, :n].astype(np.float32))
        raw["krope_raw"].append(p.krope_raw[b, :n].astype(np.float32))
        raw["q_nope"].append(p.q_nope[b, n - T:n].astype(np.float32))
        raw["q_rope_raw"].append(p.q_rope_raw[b, n - T:n].astype(np.float32))
    return raw
