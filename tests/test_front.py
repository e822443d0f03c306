"""mla_project: hidden states -> q_nope, q_rope, ckv_raw, krope_raw, against the oracle.

The oracle's front end (oracle.mla_ref.project_layer, pinned to torch.nn.functional.linear) is
computed in float64 from the same storage-rounded inputs. GPU cases: the scaled DeepSeek-V2
shape of C2 in bf16 (query rank 96: a ragged last 64-wide K slab) and fp32 (CUDA cores), C1's
full-rank fp32 query, and the DeepSeek-V2 shape (d_model 5120, query rank 1536) at 1, 64 and
130 tokens (two token tiles). CPU cases: argument validation.
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


# ------------------------------------------------------------------------------------ CPU
def test_project_validates_arguments(mla):
    w = mi.WORKLOADS["dsv2"]
    c = _cfg(mla, w).c()
    good = mla.front_config(5120, 1536)
    size = mla.lib.mla_project_workspace_size
    assert size(ctypes.byref(c), ctypes.byref(good), 64) > 64 * 1536 * 2
    assert size(ctypes.byref(c), ctypes.byref(good), 0) == 0
    for bad in (mla.front_config(0, 1536), mla.front_config(5120, -1),
                mla.front_config(5120, 1536, float("nan")), mla.front_config(5120, 20000)):
        assert size(ctypes.byref(c), ctypes.byref(bad), 64) == 0
    ws = size(ctypes.byref(c), ctypes.byref(good), 64)
    f = mla.lib.mla_project
    ptrs = [256] * 11
    call = lambda front, p, n=64, wsz=ws, wsp=256: f(  # noqa: E731
        ctypes.byref(c), ctypes.byref(front), *p, n, wsp, wsz, None, None)
    assert call(good, ptrs, n=0) == mla.MLA_OK                              # no tokens
    assert call(mla.front_config(0, 1536), ptrs) == mla.MLA_ERR_INVALID_ARG
    for i in range(11):                                                      # every pointer
        p = list(ptrs)
        p[i] = None
        assert call(good, p) == mla.MLA_ERR_INVALID_ARG, i
    assert call(good, ptrs, wsz=ws - 1) == mla.MLA_ERR_WORKSPACE
    assert call(good, ptrs, wsp=128) == mla.MLA_ERR_WORKSPACE
    # a bf16 width the tensor-core kernel cannot stride over (every call here returns before
    # any launch)
    assert call(mla.front_config(5124, 1536), ptrs, wsz=4 * ws) == mla.MLA_ERR_UNSUPPORTED
    p = list(ptrs)
    p[0] = 264                                                               # x misaligned
    assert call(good, p) == mla.MLA_ERR_INVALID_ARG


# ------------------------------------------------------------------------------------ GPU
def _run(mla, w, n, seed=3):
    """The device front end and the oracle's on the same storage-rounded inputs."""
    d = mi.layer_draw(w, seed, x_rows=n)
    rnd = lambda a: None if a is None else mi.storage_round(w, a)  # noqa: E731
    x, w_dq, w_uq, w_qr, w_dkv, w_kr = map(rnd, (d.x, d.w_dq if w.q_rank else d.w_q, d.w_uq,
                                                 d.w_qr, d.w_dkv, d.w_kr))
    gq = None if d.gamma_q is None else d.gamma_q.astype(np.float32)
    cfg = _cfg(mla, w)
    tdt = cfg.torch_dtype
    dev = lambda a: None if a is None else torch.from_numpy(  # noqa: E731
        np.ascontiguousarray(a, dtype=np.float32)).cuda().to(tdt)
    H, dh, dr, r = w.num_heads, w.head_dim, w.rope_dim, w.kv_rank
    out = dict(q_nope=torch.empty((n, H, dh), dtype=tdt, device="cuda"),
               q_rope=torch.empty((n, H, dr), dtype=tdt, device="cuda"),
               ckv_raw=torch.empty((n, r), dtype=tdt, device="cuda"),
               krope_raw=torch.empty((n, dr), dtype=tdt, device="cuda"))
    front = mla.front_config(w.d_model, w.q_rank or 0, w.rms_eps)
    ws = torch.empty(mla.project_workspace_size(cfg, front, n), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.project(cfg, front, dev(x), dev(w_dq), None if gq is None else torch.from_numpy(gq).cuda(),
                dev(w_uq), dev(w_qr), dev(w_dkv), dev(w_kr), out["q_nope"], out["q_rope"],
                out["ckv_raw"], out["krope_raw"], ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    kw = dict(w_q=w_dq) if not w.q_rank else dict(w_dq=w_dq, w_uq=w_uq, gamma_q=gq)
    exp = ref.project_layer(x[None], H, dh, dr, w_dkv, w_kr, w_qr, eps=w.rms_eps, **kw)
    exp = dict(q_nope=exp.q_nope[0], q_rope=exp.q_rope_raw[0], ckv_raw=exp.ckv_raw[0],
               krope_raw=exp.krope_raw[0])
    return {k: v.float().cpu().numpy() for k, v in out.items()}, exp


@pytest.mark.gpu
@pytest.mark.parametrize("name,n", [("small_bf16", 16), ("small_bf16", 1), ("small_fp32", 9),
                                    ("tiny_fp32", 3), ("dsv2", 64), ("dsv2", 1), ("dsv2", 130)])
def test_project_matches_the_oracle(mla, name, n):
    w = mi.WORKLOADS[name]
    got, exp = _run(mla, w, n)
    for k in got:
        assert got[k].shape == exp[k].shape, k
        ok, e = compare.within(got[k], exp[k], w.dtype)
        assert ok, f"{k}: error {e:.3g}"


@pytest.mark.gpu
def test_project_is_deterministic(mla):
    w = mi.WORKLOADS["dsv2"]
    a, _ = _run(mla, w, 64)
    b, _ = _run(mla, w, 64)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
