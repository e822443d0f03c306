"""mla_prefill: causal attention of packed prompts, against the oracle.

The prompt's forward with the causal mask ("MLA from scratch in PyTorch", The MLAAttention
module: K and V rebuilt from every cached latent, query t attends rows 0 .. t) is the oracle's
attention over the expanded operands (oracle.mla_ref.expanded_attention, pinned to torch's
causal attention and to the naive form). The cache rows are the oracle's (RMSNorm and RoPE,
rounded to the storage type once) and go to the device as its input. A bf16 prefill holds the
expanded K and V and the rotated query as bf16 MMA operands, so for bf16 the oracle rounds
them at the same points before the attention (round-to-nearest-even of the exact values),
and the bar applies to every query token's (H, d_v) output, with one bf16 ulp of each
expected element granted for the output format's rounding (oracle.compare.PROMPT_OUTPUT_ULPS). GPU cases: the DeepSeek-V2 head shape on the tensor
cores with prompts that end inside a 128-row tile, fill one exactly, or hold a single token;
C2's head shape in bf16 and fp32 on CUDA cores. CPU: argument validation.
"""
import ctypes

import numpy as np
import pytest
import torch

import mla_inputs as mi
from oracle import compare
from oracle import mla_ref as ref


@pytest.fixture(scope="module")
def mla():
    from mla_latent_kv_44_b200 import build

    build.build()
    import mla_latent_kv_44_b200 as m

    return m


def _cfg(mla, w):
    return mla.Config(num_heads=w.num_heads, head_dim=w.head_dim, kv_rank=w.kv_rank,
                      rope_dim=w.rope_dim, block_size=64, dtype=w.dtype)


def test_prefill_validates_arguments(mla):
    c = _cfg(mla, mi.WORKLOADS["dsv2"]).c()
    size = mla.lib.mla_prefill_workspace_size
    ws = size(ctypes.byref(c), 1000)
    assert ws >= 1000 * 128 * (64 + 128 + 128) * 2  # rotated RoPE query, K_nope, V (bf16)
    assert size(ctypes.byref(c), 0) == 0 and size(None, 10) == 0
    f = mla.lib.mla_prefill
    p = [256] * 7   # q_nope, q_rope, pos, rows, w_uk, w_uv, cu_seqlens

    def call(ptrs, batch=2, maxlen=600, n=1000, o=256, wsp=256, wsz=ws):
        return f(ctypes.byref(c), *ptrs, batch, maxlen, n, o, wsp, wsz, None, None)

    assert call(p, batch=0) == mla.MLA_OK and call(p, n=0) == mla.MLA_OK
    for i in range(7):
        q = list(p)
        q[i] = None
        assert call(q) == mla.MLA_ERR_INVALID_ARG, i
    assert call(p, o=None) == mla.MLA_ERR_INVALID_ARG
    assert call(p, maxlen=0) == mla.MLA_ERR_INVALID_ARG
    assert call(p, wsz=ws - 1) == mla.MLA_ERR_WORKSPACE
    assert call(p, wsp=128) == mla.MLA_ERR_WORKSPACE
    q = list(p)
    q[3] = 264                                   # rows misaligned
    assert call(q) == mla.MLA_ERR_INVALID_ARG


def test_prefill_workspace_layout(mla):
    """The tensor-core path's workspace is the rotated RoPE query, K_nope and V in bf16 (80 KB
    per token at the DeepSeek-V2 heads), each region 256-byte aligned; the CUDA-core path
    also holds the packed query and the front end's partial sums."""
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    w = mi.WORKLOADS["dsv2"]
    c = _cfg(mla, w).c()
    H, dh, dr, dv = w.num_heads, w.head_dim, w.rope_dim, w.head_dim_v
    for n in (1, 7, 1000, 16384):
        want = up(n * H * dr * 2) + up(n * H * dh * 2) + up(n * H * dv * 2)
        assert mla.lib.mla_prefill_workspace_size(ctypes.byref(c), n) == want, n
    assert mla.lib.mla_prefill_workspace_size(ctypes.byref(c), 16384) == 1280 * 2 ** 20
    w = mi.WORKLOADS["small_fp32"]
    c = _cfg(mla, w).c()
    H, dh, dr, dv = w.num_heads, w.head_dim, w.rope_dim, w.head_dim_v
    n = 1000
    assert mla.lib.mla_prefill_workspace_size(ctypes.byref(c), n) >= n * H * (dh + dr + dh + dv) * 4


def _run(mla, w, lens, seed=5, sample=None):
    """Device prefill of sequences of the given lengths, and the oracle's outputs (for the
    query tokens sample[b] of sequence b when a sample is given, else for every token)."""
    H, dh, dr, dv, r = w.num_heads, w.head_dim, w.rope_dim, w.head_dim_v, w.kv_rank
    wuk, wuv = (mi.storage_round(w, x) for x in mi.up_projection_weights(w, seed))
    gamma = mi.rms_gain(w, seed, perturbed=True)
    qn, qr, rows, pos, exp = [], [], [], [], []
    for b, L in enumerate(lens):
        d = mi.sequence_draw(mi.scaled(w, new_tokens=L), b, L, seed)
        ckv, kr = mi.storage_round(w, d.ckv_raw), mi.storage_round(w, d.krope_raw)
        q1, q2 = mi.storage_round(w, d.q_nope), mi.storage_round(w, d.q_rope_raw)
        p = np.arange(L)
        rw = ref.cache_rows(ckv, kr, gamma, p, w.rms_eps, w.rope_base, w.dtype == "bf16")
        # the operands as the device holds them: bf16 for a bf16 prefill
        stored = ref.round_bf16 if w.dtype == "bf16" else (lambda x: x)
        Q = stored(np.concatenate([q1, ref.rope_rotate(q2, p[:, None], w.rope_base)], -1))
        K = np.concatenate([stored(np.einsum("lr,hdr->lhd", rw[:, :r], wuk, optimize=True)),
                            np.repeat(rw[:, None, r:], H, axis=1)], -1)
        V = stored(np.einsum("lr,hdr->lhd", rw[:, :r], wuv, optimize=True))
        if sample is None:
            e = ref.expanded_attention(Q, K, V, w.softmax_scale)
        else:  # token t attends rows 0 .. t: the last query of the prefix t + 1
            e = np.concatenate([ref.expanded_attention(Q[t:t + 1], K[:t + 1], V[:t + 1],
                                                       w.softmax_scale) for t in sample[b]])
        qn.append(q1), qr.append(q2), rows.append(rw), pos.append(p), exp.append(e)
    cfg = _cfg(mla, w)
    tdt = cfg.torch_dtype
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(np.concatenate(a), np.float32)).cuda().to(tdt)  # noqa: E731,E501
    n = int(sum(lens))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)).cuda()
    o = torch.full((n, H, dv), float("nan"), dtype=tdt, device="cuda")
    ws = torch.empty(mla.prefill_workspace_size(cfg, n), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    w_uk = torch.from_numpy(wuk).cuda().to(tdt)
    w_uv = torch.from_numpy(wuv).cuda().to(tdt)
    mla.prefill(cfg, dev(qn), dev(qr), torch.from_numpy(np.concatenate(pos).astype(np.int32)).cuda(),
                dev(rows), w_uk, w_uv, cu, max(lens), o, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = o.float().cpu().numpy()
    offs = np.concatenate([[0], np.cumsum(lens)])
    return [got[offs[b]:offs[b + 1]] for b in range(len(lens))], exp


@pytest.mark.gpu
@pytest.mark.parametrize("name,lens", [
    ("dsv2", [300, 129, 1, 640]),
    ("dsv2", [128]),
    ("dsv2", [1000]),
    ("small_bf16", [200, 33, 1]),
    ("small_fp32", [150, 64]),
])
def test_prefill_matches_the_oracle(mla, name, lens):
    w = mi.WORKLOADS[name]
    got, exp = _run(mla, w, lens)
    # each query token is one attention problem (as one decode step's token is): the bar
    # applies to its (H, d_v) output, whose scale shrinks as the token averages more keys
    worst = 0.0
    for b, (g, e) in enumerate(zip(got, exp)):
        assert np.all(np.isfinite(g)), f"sequence {b}: non-finite output"
        for t in range(lens[b]):
            ok, err = compare.within(g[t], e[t], w.dtype, out_ulps=compare.PROMPT_OUTPUT_ULPS)
            worst = max(worst, err)
            assert ok, f"sequence {b} (length {lens[b]}), token {t}: error {err:.3g}"
    print(f"{name} {lens}: worst scaled error {worst:.3g}")


@pytest.mark.gpu
def test_prefill_long_prompts_sampled(mla):
    """Prompts of 2300 and 200 tokens (20 token tiles: the expansion's weight tiles walk two
    token chunks; nine query-tile pairs): query tokens at tile and chunk boundaries, the
    first and the last, against the oracle's attention over each token's prefix."""
    w = mi.WORKLOADS["dsv2"]
    lens = [2300, 200]
    sample = [[0, 1, 127, 128, 255, 256, 1000, 2047, 2048, 2049, 2175, 2299],
              [0, 63, 127, 128, 199]]
    got, exp = _run(mla, w, lens, sample=sample)
    worst = 0.0
    for b in range(len(lens)):
        assert np.all(np.isfinite(got[b])), f"sequence {b}: non-finite output"
        for i, t in enumerate(sample[b]):
            ok, err = compare.within(got[b][t], exp[b][i], w.dtype,
                                     out_ulps=compare.PROMPT_OUTPUT_ULPS)
            worst = max(worst, err)
            assert ok, f"sequence {b}, token {t}: error {err:.3g}"
    print(f"long prompts {lens}: worst scaled error {worst:.3g}")
