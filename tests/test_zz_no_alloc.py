"""mla_decode_static_workspace: the decode entry point that allocates nothing.

It exists for callers that cannot allocate device memory themselves (a host program with no
device allocator, or a decode loop that must not call cudaMalloc because it synchronises the
device). It must give the same results as mla_decode with a caller-owned workspace, call after
call, although every call reuses the library's one fixed device array. This file is named to
be collected last; it also passes on its own in a fresh process, where its first call performs
the per-device set-up.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import mla_inputs as mi
from oracle import compare, mla_ref as ref

pytestmark = pytest.mark.gpu


def _case(mla, H, dh, r, dr, lengths, T, seed):
    g = np.random.default_rng([seed, 9])
    bs, D, B = 64, r + dr, len(lengths)
    rows = [mi.round_to_bf16(np.concatenate([g.standard_normal((L, r)),
                                             2 * g.standard_normal((L, dr))], 1))
            for L in lengths]
    nblk = [(L + bs - 1) // bs for L in lengths]
    nb = sum(nblk) + 1
    ids = g.permutation(nb)
    table = np.full((B, max(nblk)), -1, np.int32)
    pool = np.zeros((nb, bs, D), np.float32)
    off = 0
    for b, L in enumerate(lengths):
        table[b, :nblk[b]] = ids[off:off + nblk[b]]
        off += nblk[b]
        for j in range(L):
            pool[table[b, j // bs], j % bs] = rows[b][j]
    Q = mi.round_to_bf16(0.25 * g.standard_normal((B * T, H, D)))
    cfg = mla.Config(num_heads=H, head_dim=dh, kv_rank=r, rope_dim=dr, block_size=bs,
                     dtype="bf16")
    dev = "cuda"
    t = dict(q=torch.from_numpy(Q).to(dev, torch.bfloat16),
             pool=torch.from_numpy(pool).to(dev, torch.bfloat16),
             table=torch.from_numpy(table).to(dev),
             lens=torch.tensor(lengths, dtype=torch.int32, device=dev))
    return cfg, t, Q, rows


def _outputs(B, T, H, r):
    return (torch.full((B * T, H, r), float("nan"), device="cuda"),
            torch.full((B * T, H), float("nan"), device="cuda"),
            torch.zeros(1, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("shape,lengths,T", [
    ((128, 128, 512, 64), [1, 130, 2000, 64 * 74 + 9], 1),   # tensor-core attention kernel
    ((128, 128, 512, 64), [5, 700, 3000], 4),
    ((16, 64, 64, 32), [3, 200, 1500], 1),                    # CUDA-core attention kernel
])
def test_static_workspace_matches_caller_workspace(shape, lengths, T):
    import mla_latent_kv_44_b200 as mla

    H, dh, r, dr = shape
    cfg, t, Q, rows = _case(mla, H, dh, r, dr, lengths, T, seed=len(lengths) + T)
    B = len(lengths)
    assert mla.decode_workspace_size(cfg, B, T) <= mla.STATIC_WORKSPACE_BYTES

    ws = torch.empty(mla.decode_workspace_size(cfg, B, T), dtype=torch.uint8, device="cuda")
    out_ref, lse_ref, err_ref = _outputs(B, T, H, r)
    mla.decode(cfg, t["q"], t["pool"], t["table"], t["lens"], T, ws, out_ref, lse_ref, err_ref)
    torch.cuda.synchronize()
    assert int(err_ref.item()) == 0

    scale = 1 / math.sqrt(dh + dr)
    for _ in range(2):  # two calls in a row reuse the same device array
        out, lse, err = _outputs(B, T, H, r)
        mla.decode_static_workspace(cfg, t["q"], t["pool"], t["table"], t["lens"], T, out, lse,
                                    err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        got, want = out.cpu().numpy(), out_ref.cpu().numpy()
        ok, e = compare.within(got, want, "bf16")
        assert ok, f"static-workspace result differs from mla_decode: {e}"
        assert np.max(np.abs(lse.cpu().numpy() - lse_ref.cpu().numpy())) <= 2e-2
        # both follow the oracle too
        for b in range(B):
            exp = ref.latent_attention(Q[b * T:(b + 1) * T], rows[b], r, scale, T)
            assert compare.within(got[b * T:(b + 1) * T], exp.o_lat, "bf16")[0]


def test_static_workspace_rejects_oversized_work():
    import mla_latent_kv_44_b200 as mla

    cfg = mla.Config(num_heads=1024, head_dim=64, kv_rank=1024, rope_dim=64, block_size=64,
                     dtype="bf16")
    assert mla.decode_workspace_size(cfg, 4, 1) > mla.STATIC_WORKSPACE_BYTES
    c = cfg.c()
    st = mla.lib.mla_decode_static_workspace(ctypes.byref(c), 256, 256, 256, 4, 4, 256, 4, 1,
                                             256, None, 256, None)
    assert st == mla.MLA_ERR_WORKSPACE
