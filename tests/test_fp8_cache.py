"""FP8 latent cache: mla_append_latent_fp8 codes and scales, and mla_decode_fp8, against the oracle.

The oracle's row is [RMSNorm(c_kv) * gamma ‖ RoPE(k_rope)] in float64; its scale is
max |row| / 448 and its codes E4M3(row / scale) (oracle.mla_ref.quantize_rows_fp8, E4M3
rounding pinned to torch's float8_e4m3fn). The device computes the row in fp32, so a code may
come out as the other neighbour only where row / scale lies within the fp32 arithmetic's
relative error (1e-5 here, from r-term sums of squares) of a rounding midpoint; every other
code must be equal, bit for bit. The decode over the fp8 pool is compared with the oracle's
attention over its own dequantised rows (codes * scale; rounded to bf16 where the tensor-core
path consumes them as bf16 operands), within the bar of the 8-bit storage type's nearest one
(2e-2, as bf16). CPU: argument validation.
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


def _cfg(mla, w, bs):
    return mla.Config(num_heads=w.num_heads, head_dim=w.head_dim, kv_rank=w.kv_rank,
                      rope_dim=w.rope_dim, block_size=bs, dtype=w.dtype)


def test_fp8_calls_validate_arguments(mla):
    c = _cfg(mla, mi.WORKLOADS["dsv2"], 64).c()
    app = mla.lib.mla_append_latent_fp8
    args = [256] * 6  # ckv, krope, gamma, seq, pos, table
    assert app(ctypes.byref(c), *args, 2, 4, 256, 256, 8, 0, 256, None) == mla.MLA_OK
    for i in range(6):
        a = list(args)
        a[i] = None
        assert app(ctypes.byref(c), *a, 2, 4, 256, 256, 8, 4, 256, None) == mla.MLA_ERR_INVALID_ARG
    assert app(ctypes.byref(c), *args, 2, 4, 256, None, 8, 4, 256, None) == mla.MLA_ERR_INVALID_ARG
    dec = mla.lib.mla_decode_fp8
    ws = mla.lib.mla_decode_fp8_workspace_size(ctypes.byref(c), 2, 1, 4)
    # the tensor-core path's scratch: 2 sequences x 4 blocks of bf16 rows
    assert ws >= mla.lib.mla_decode_workspace_size(ctypes.byref(c), 2, 1) + 8 * 64 * 576 * 2
    call = lambda scale, wsz, wsp=256, pool=256: dec(  # noqa: E731
        ctypes.byref(c), 256, pool, scale, 256, 4, 8, 256, 2, 1, wsp, wsz, 256, None, 256, None)
    assert call(None, ws) == mla.MLA_ERR_INVALID_ARG
    assert call(256, ws - 1) == mla.MLA_ERR_WORKSPACE
    assert call(256, ws, wsp=128) == mla.MLA_ERR_WORKSPACE
    assert call(256, ws, pool=264) == mla.MLA_ERR_INVALID_ARG


def _setup(mla, w, lens, T=1, seed=7, bs=64):
    """fp8 pool filled by mla_append_latent_fp8 (every row, contiguous blocks per sequence),
    and the oracle's rows, codes and scales."""
    H, r, dr = w.num_heads, w.kv_rank, w.rope_dim
    D = r + dr
    cfg = _cfg(mla, w, bs)
    tdt = cfg.torch_dtype
    nblk = [-(-L // bs) for L in lens]
    table = np.zeros((len(lens), max(nblk)), dtype=np.int32)
    first = np.concatenate([[0], np.cumsum(nblk)])
    for b in range(len(lens)):
        table[b, :nblk[b]] = first[b] + np.arange(nblk[b])
    gamma = mi.rms_gain(w, seed, perturbed=True)
    ckv, kr, seq, pos, draws = [], [], [], [], []
    for b, L in enumerate(lens):
        d = mi.sequence_draw(mi.scaled(w, new_tokens=T), b, L, seed)
        c1, k1 = mi.storage_round(w, d.ckv_raw), mi.storage_round(w, d.krope_raw)
        draws.append((c1, k1, mi.storage_round(w, d.q_nope), mi.storage_round(w, d.q_rope_raw)))
        ckv.append(c1), kr.append(k1)
        seq.append(np.full(L, b, np.int32)), pos.append(np.arange(L, dtype=np.int32))
    dev = lambda a, dt=tdt: torch.from_numpy(np.ascontiguousarray(np.concatenate(a))).cuda().to(dt)  # noqa: E731,E501
    pool = torch.zeros((int(first[-1]), bs, D), dtype=torch.uint8, device="cuda")
    scale = torch.zeros((int(first[-1]), bs), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tab = torch.from_numpy(table).cuda()
    mla.append_latent_fp8(cfg, dev(ckv), dev(kr), torch.from_numpy(gamma).cuda(),
                          dev(seq, torch.int32), dev(pos, torch.int32), tab, pool, scale, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows, codes, scales = [], [], []
    for b, L in enumerate(lens):
        rw = ref.cache_rows(draws[b][0], draws[b][1], gamma, np.arange(L), w.rms_eps,
                            w.rope_base, False)
        cd, sc = ref.quantize_rows_fp8(rw)
        rows.append(rw), codes.append(cd), scales.append(sc)
    return cfg, pool, scale, tab, err, table, draws, rows, codes, scales


def _device_rows(pool, scale, table, b, L, bs):
    ids = torch.from_numpy(table[b, :-(-L // bs)].astype(np.int64)).cuda()
    codes = pool[ids].reshape(-1, pool.shape[-1])[:L].view(torch.float8_e4m3fn).float()
    return codes.cpu().numpy(), scale[ids].reshape(-1)[:L].cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("name,lens", [("small_bf16", [130, 64, 7]), ("dsv2", [300, 65])])
def test_append_fp8_codes_and_scales(mla, name, lens):
    w = mi.WORKLOADS[name]
    bs = 64
    cfg, pool, scale, tab, err, table, draws, rows, codes, scales = _setup(mla, w, lens, bs=bs)
    flips = 0
    for b, L in enumerate(lens):
        got_c, got_s = _device_rows(pool, scale, table, b, L, bs)
        assert np.max(np.abs(got_s / scales[b] - 1.0)) < 1e-5, f"sequence {b}: scales"
        v = rows[b] / scales[b][:, None]
        amb = ref.round_fp8_e4m3(v * (1 - 1e-5)) != ref.round_fp8_e4m3(v * (1 + 1e-5))
        same = got_c == codes[b]
        assert np.all(same | amb), f"sequence {b}: a code differs away from a midpoint"
        flips += int(np.count_nonzero(~same))
    print(f"{name}: {flips} codes on the other side of a midpoint")


@pytest.mark.gpu
@pytest.mark.parametrize("name,lens,T", [("small_bf16", [300, 90, 1], 1), ("dsv2", [700, 129], 1),
                                         ("dsv2", [400, 70], 4)])
def test_decode_fp8_matches_the_oracle(mla, name, lens, T):
    w = mi.scaled(mi.WORKLOADS[name], new_tokens=T)
    bs = 64
    cfg, pool, scale, tab, err, table, draws, rows, codes, scales = _setup(mla, w, lens, T=T,
                                                                         bs=bs)
    H, r = w.num_heads, w.kv_rank
    wuk, _ = (mi.storage_round(w, x) for x in mi.up_projection_weights(w, 7))
    # where the tensor-core attention runs (bf16, H = 128, r = 512, d_r = 64, 64-row blocks),
    # the rows are expanded to bf16 operands first, as a bf16 cache's rows are bf16 on both
    # sides; the CUDA-core path reads codes * scale in fp32
    tc = (w.dtype == "bf16" and H == 128 and r == 512 and w.rope_dim == 64 and bs == 64)
    Qs, exp = [], []
    for b, L in enumerate(lens):
        c1, k1, qn, qr = draws[b]
        Q = ref.absorb_ref(qn, qr, np.arange(L - T, L), wuk, w.rope_base)
        Qb = mi.storage_round(w, Q)
        Qs.append(Qb)
        deq = codes[b] * scales[b][:, None]
        if tc:
            deq = ref.round_bf16(deq)
        exp.append(ref.latent_attention(Qb, deq, r, w.softmax_scale, T))
    tdt = cfg.torch_dtype
    q = torch.from_numpy(np.ascontiguousarray(np.concatenate(Qs), np.float32)).cuda().to(tdt)
    lens_t = torch.tensor(lens, dtype=torch.int32).cuda()
    ws = torch.empty(mla.decode_fp8_workspace_size(cfg, len(lens), T, table.shape[1]),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty((len(lens) * T, H, r), device="cuda")
    lse = torch.empty((len(lens) * T, H), device="cuda")
    mla.decode_fp8(cfg, q, pool, scale, tab, lens_t, T, ws, out, lse, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for b in range(len(lens)):
        got = out[b * T:(b + 1) * T].cpu().numpy()
        ok, e = compare.within(got, exp[b].o_lat, "bf16")
        assert ok, f"sequence {b}: latent error {e:.3g}"
        assert np.max(np.abs(lse[b * T:(b + 1) * T].cpu().numpy() - exp[b].lse)) < 1e-3
