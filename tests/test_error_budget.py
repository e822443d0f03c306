"""Error budget of a bf16 decode step at the DeepSeek-V2 shape (CPU, float64).

The smoke's check (2 sequences of 700 cached rows, one query token each) measures the device
step against the naive form in float64 (oracle.mla_ref.decode_sequence_from_raw, the cache
rows rounded to bf16 as stored). Three roundings separate a correct bf16 step from that
reference: the absorbed query [W_UK^T q_nope ‖ RoPE(q_rope)] is a bf16 tensor at the library's
boundary; the kernel's attention weights P are bf16 MMA operands; the step's output o is
bf16. Each is emulated here, alone and together, on the smoke's own inputs (the same seeded
draws as mla_latent_kv_44_b200.step.DecodeState), in the bf16 scaled-error metric of
oracle.compare.within, so that the smoke's figure can be read against its parts.
"""
import numpy as np
import pytest

import mla_inputs as mi
from oracle import compare
from oracle import mla_ref as ref


def _budget(b: int):
    w = mi.scaled(mi.WORKLOADS["dsv2"], batch=2, cached=700)
    seed = 0
    n = int(mi.total_rows(w, seed)[b])
    wuk, wuv = (mi.storage_round(w, x) for x in mi.up_projection_weights(w, seed))
    gamma = np.asarray(mi.rms_gain(w, seed, False), dtype=np.float32)
    d = mi.sequence_draw(w, b, n, seed)
    ckv, kr = mi.storage_round(w, d.ckv_raw), mi.storage_round(w, d.krope_raw)
    q1, q2 = mi.storage_round(w, d.q_nope), mi.storage_round(w, d.q_rope_raw)
    exp = ref.decode_sequence_from_raw(ckv, kr, q1, q2, wuk, wuv, gamma, w.softmax_scale,
                                       w.rms_eps, w.rope_base, store_bf16=True)
    rows = ref.cache_rows(ckv, kr, gamma, np.arange(n), w.rms_eps, w.rope_base, True)
    T, r = w.new_tokens, w.kv_rank
    Q = ref.absorb_ref(q1, q2, np.arange(n - T, n), wuk, w.rope_base)

    def step(q_bf16, p_bf16, out_bf16):
        Qx = ref.round_bf16(Q) if q_bf16 else Q
        s = np.einsum("thc,lc->thl", Qx, rows) * w.softmax_scale
        p = np.exp(s - s.max(-1, keepdims=True))
        if p_bf16:  # the MMA's operand; l sums the same rounded values
            p = ref.round_bf16(p)
        o_lat = np.einsum("thl,lc->thc", p, rows[:, :r]) / p.sum(-1, keepdims=True)
        o = ref.output_ref(o_lat, wuv)
        return ref.round_bf16(o) if out_bf16 else o

    parts = {"none": (0, 0, 0), "query": (1, 0, 0), "P": (0, 1, 0), "output": (0, 0, 1),
             "all": (1, 1, 1)}
    return {k: compare.within(step(*f), exp.o, "bf16")[1] for k, f in parts.items()}


@pytest.mark.parametrize("b", [0, 1])
def test_bf16_step_error_budget(b):
    e = _budget(b)
    print(f"sequence {b}: " + ", ".join(f"{k} {v:.2e}" for k, v in e.items()))
    # the absorbed form with no rounding is the naive form (float64 round-off only)
    assert e["none"] < 1e-12
    # each rounding alone is a visible part of the 2e-2 bar, and none fills it
    for k in ("query", "P", "output"):
        assert 1e-3 < e[k] < 2e-2, k
    # a step that rounds exactly where the kernel does stays within the bar
    assert e["all"] <= compare.BF16_SCALED_TOL
