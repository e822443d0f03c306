"""mla_decode_step: one call for the whole step gives the same bits as the four calls.

Two DecodeStates built from the same seeded inputs run one step each, one through the four
calls (absorb, append, decode, output), the other through mla_decode_step. On the
DeepSeek-V2-shaped bf16 workloads the step takes its fused launches (absorb, append and
planner in one grid, then attention, combine and output); on the small shapes it runs the four
calls' own kernels. Every output must be identical, bit for bit, and
agree with the oracle.
"""
import numpy as np
import pytest
import torch

import mla_inputs as mi
from tests.gpu_util import check_sequence, dev_err


@pytest.fixture(scope="module")
def mla():
    import mla_latent_kv_44_b200 as m

    return m


def _bits(t):
    """A tensor's bytes as integers (NaN sentinels compare equal to themselves)."""
    t = t.contiguous()
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


CASES = [
    ("dsv2", dict(batch=8, cached=2000)),    # fused; split row groups
    ("ragged", dict(batch=24)),               # fused; ragged lengths up to 32k
    ("mtp", dict(batch=6, cached=1500)),      # fused; four causal query tokens per sequence
    ("dsv2", dict(batch=1, cached=300)),      # fused; one short sequence split across ranges
    ("small_bf16", dict()),                   # the four calls' kernels (no tensor-core decode)
    ("tiny_fp32", dict()),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,kw", CASES)
def test_fused_step_matches_the_four_calls(mla, name, kw):
    from mla_latent_kv_44_b200.step import DecodeState

    w = mi.scaled(mi.WORKLOADS[name], **kw)
    a = DecodeState(w, sequences=[0, w.batch - 1])
    b = DecodeState(w, sequences=[0, w.batch - 1])
    a.step()
    b.step_fused()
    assert dev_err(a) == 0 and dev_err(b) == 0
    for field in ("q", "out_latent", "lse", "o", "pool"):
        assert torch.equal(_bits(getattr(a, field)), _bits(getattr(b, field))), field
    for s in (0, w.batch - 1):
        check_sequence(b, s, "absorbed")


@pytest.mark.gpu
def test_fused_step_rejects_what_the_calls_reject(mla):
    from mla_latent_kv_44_b200.step import DecodeState

    w = mi.scaled(mi.WORKLOADS["dsv2"], batch=2, cached=200)
    st = DecodeState(w, sequences=[0])
    small_ws = st.workspace[:-256]
    with pytest.raises(mla.MlaError) as e:
        mla.decode_step(st.cfg, st.q_nope, st.q_rope, st.w_uk, st.ckv_new, st.krope_new, st.gamma,
                        st.seq_new, st.pos_new, st.block_table, st.pool, st.seq_lens,
                        w.new_tokens, st.q, small_ws, st.out_latent, st.lse, st.w_uv, st.o,
                        st.dev_err)
    assert e.value.status == mla.MLA_ERR_WORKSPACE
    # nothing was enqueued: the outputs still hold what they held
    torch.cuda.synchronize()
    assert int(st.dev_err.item()) == 0
