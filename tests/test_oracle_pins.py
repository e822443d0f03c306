"""Pins of the CPU oracle against what the pages and the mathematics fix (no GPU).

Each test below would fail for a plausible mistake in the oracle: a dropped term, a wrong
sign or index, a transposed operand, a wrong scale or an off-by-one in the causal mask.
"""
import math

import numpy as np
import pytest
import torch

import mla_inputs as mi
from oracle import compare, kv_accounting as acc, mla_ref as ref
from tests.conftest import read_golden, read_table


# ----------------------------------------------------------------------------------------
# Cache arithmetic against the pages' printed values
# ----------------------------------------------------------------------------------------

def test_cache_table_printed_on_page():
    for n_heads, kv_heads, mha, gqa, mla in read_table("cache_per_token_table.txt"):
        assert acc.cache_values_mha(n_heads, 64) == mha
        assert acc.cache_values_gqa(kv_heads, 64) == gqa
        assert acc.cache_values_mla(64, 16) == mla
        assert n_heads == 4 * kv_heads


def test_arithmetic_printed_on_pages():
    g = read_golden("arithmetic_pins.txt")
    iv = lambda k: int(g[k])  # noqa: E731
    assert acc.cache_values_mla(iv("glm_kv_rank"), iv("glm_rope_dim")) == iv("glm_cache_values")
    mha = acc.cache_values_mha(iv("mha_heads"), iv("mha_head_dim"))
    assert mha == 32768
    assert round(mha / iv("glm_cache_values")) == iv("glm_saving_x")
    assert round(100 * acc.reduction_fraction(iv("glm_cache_values"), mha), 1) == float(
        g["reduction_vs_same_shape_mha_pct"])
    assert iv("hbm_mha_values") // iv("hbm_latent_values") == iv("hbm_ratio_x")
    assert acc.cache_values_mha(iv("mha_heads"), iv("mha_head_dim")) == iv("hbm_mha_values")
    gqa2 = acc.cache_values_gqa(iv("gqa2_kv_heads"), iv("gqa2_head_dim"))
    assert gqa2 == iv("gqa2_values")
    mla = acc.cache_values_mla(iv("mla_rank"), iv("mla_rope"))
    assert mla == iv("mla_values")
    assert round(gqa2 / mla, 1) == float(g["gqa2_over_mla"])
    assert acc.gqa_crossover_rank(iv("gqa2_kv_heads"), iv("gqa2_head_dim"), iv("mla_rope")) == iv(
        "crossover_rank")
    # at the crossover rank MLA is no longer smaller, one rank below it still is
    r = iv("crossover_rank")
    assert acc.cache_values_mla(r, iv("mla_rope")) == gqa2
    assert acc.cache_values_mla(r - 1, iv("mla_rope")) < gqa2
    assert acc.cache_values_mha(8, iv("wide_width") // 8) == iv("wide_mha_values")
    assert iv("train_mha_values") / iv("train_mla_values") == float(g["train_ratio_x"])


def test_cache_bytes_formula_matches_code_on_page():
    # "MLA from scratch in PyTorch", Memory comparison: the page's own function gives
    # elements * 2 bytes; for MLA at 60 layers, B=1, 4K context, d_c=512 that is 0.25 GB.
    b = acc.cache_bytes(512, n_layers=60, batch=1, seq=4096)
    assert b == 512 * 60 * 4096 * 2
    assert round(b / 1e9, 2) == 0.25


def test_decode_work_per_row():
    # 576-wide bf16 row = 1152 B; 128 heads x 2 x (576 + 512) FLOPs.
    nbytes, flops = acc.absorbed_decode_work(1, 128, 512, 64)
    assert nbytes == 1152 and flops == 278528


class _CountingFloat:
    """A float that counts the multiplications and additions performed on it."""
    mul = 0
    add = 0

    def __init__(self, v):
        self.v = float(v)

    def __mul__(self, o):
        _CountingFloat.mul += 1
        return _CountingFloat(self.v * (o.v if isinstance(o, _CountingFloat) else o))

    def __add__(self, o):
        _CountingFloat.add += 1
        return _CountingFloat(self.v + (o.v if isinstance(o, _CountingFloat) else o))


def test_naive_decode_flops_counts_the_contractions_of_the_expanded_form():
    # "MLA from scratch in PyTorch", The up-projection cost at decode time: the expanded form
    # rebuilds K and V from every cached latent, then scores the query against K. Count the
    # multiply-adds a scalar-loop version of exactly those contractions executes at a tiny
    # shape (one multiply and one add per term, 2 FLOPs per multiply-add, as the page counts),
    # check that the loops compute the oracle's K, V and scores, and compare the count.
    S, H, dh, r = 5, 3, 2, 4
    g = np.random.default_rng([5, 1])
    c = g.standard_normal((S, r))
    wuk = g.standard_normal((H, dh, r))
    wuv = g.standard_normal((H, dh, r))
    q = g.standard_normal((H, dh))
    C = _CountingFloat
    C.mul = C.add = 0

    def dot(a, b):
        acc_ = C(0.0)
        for x, y in zip(a, b):
            acc_ = acc_ + C(x) * y
        return acc_.v

    K = np.array([[[dot(wuk[h, i], c[j]) for i in range(dh)] for j in range(S)] for h in range(H)])
    V = np.array([[[dot(wuv[h, i], c[j]) for i in range(dh)] for j in range(S)] for h in range(H)])
    s = np.array([[dot(q[h], K[h, j]) for j in range(S)] for h in range(H)])
    assert C.mul == C.add
    counted = 2 * C.mul
    assert counted == acc.naive_decode_flops(S, H, dh, r)
    # the loops are the expanded form's own contractions
    np.testing.assert_allclose(K, np.einsum("hir,jr->hji", wuk, c), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(V, np.einsum("hir,jr->hji", wuv, c), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s, np.einsum("hi,hji->hj", q, K), rtol=1e-12, atol=1e-12)
    # and an asymmetric shape cannot pass with d_h and r exchanged in only one of the terms
    assert acc.naive_decode_flops(S, H, dh, r) != 4 * S * r * H * dh + 2 * H * r * S


# ----------------------------------------------------------------------------------------
# Absorption identity, its negative control, and the RoPE counterexample
# ----------------------------------------------------------------------------------------

def _tiny_inputs(seed=0, L=65, T=1, H=8, dh=32, r=64, dr=16, dtype=np.float64):
    g = np.random.default_rng([seed, 77])
    c = g.standard_normal((L, r))
    kr = g.standard_normal((L, dr))
    qn = g.standard_normal((T, H, dh))
    qr = g.standard_normal((T, H, dr))
    wuk = g.standard_normal((H, dh, r)) / math.sqrt(r)
    wuv = g.standard_normal((H, dh, r)) / math.sqrt(r)
    return [x.astype(dtype) for x in (c, kr, qn, qr, wuk, wuv)], 1.0 / math.sqrt(dh + dr)


def test_absorption_identity_float64():
    args, scale = _tiny_inputs()
    a = ref.naive_decode(*args, scale)
    b = ref.absorbed_decode(*args, scale)
    for x, y in zip(a, b):
        assert np.max(np.abs(x - y)) < 1e-12


def test_absorption_identity_float32_at_page_scale():
    printed = float(read_golden("absorption_identity.txt")["max_abs_diff_printed"])
    args, scale = _tiny_inputs(dtype=np.float32)
    a = ref.naive_decode(*args, scale, dtype=np.float32)
    b = ref.absorbed_decode(*args, scale, dtype=np.float32)
    d = float(np.max(np.abs(a.o - b.o)))
    # same order as the page: float32 rounding only, well under 1e-6, not exactly zero
    assert 0.0 < d < 1e-6
    assert d < 20 * printed


def test_absorption_negative_control_detects_perturbed_wuk():
    args, scale = _tiny_inputs()
    c, kr, qn, qr, wuk, wuv = args
    bad = wuk.copy()
    bad[3, 5, 7] += 1e-3
    a = ref.naive_decode(c, kr, qn, qr, bad, wuv, scale)
    b = ref.absorbed_decode(c, kr, qn, qr, wuk, wuv, scale)
    assert np.max(np.abs(a.o - b.o)) > 1e-6          # the comparison can fail
    assert np.max(np.abs(a.o[:, 3] - b.o[:, 3])) > 1e-6
    others = [h for h in range(8) if h != 3]
    assert np.max(np.abs(a.o[:, others] - b.o[:, others])) < 1e-12


def test_rope_on_reconstructed_key_breaks_absorption():
    """RoPE applied to the up-projected key makes the score depend on the key's position,
    so no position-free absorbed matrix can reproduce it; the decoupled key keeps it exact."""
    g = np.random.default_rng([0, 78])
    dh, r, base = 16, 32, 10000.0
    wuk = g.standard_normal((dh, r)) / math.sqrt(r)
    q = g.standard_normal(dh)
    c = g.standard_normal(r)
    pq = 40
    # same latent c cached at two different positions
    s_at = [ref.rope_rotate(q, pq, base) @ ref.rope_rotate(wuk @ c, p, base) for p in (3, 17)]
    assert abs(s_at[0] - s_at[1]) > 1e-3
    # an absorbed score (A^T q) . c is the same for the two copies of c, whatever A is
    a = (wuk.T @ ref.rope_rotate(q, pq, base)) @ c
    assert abs(a - s_at[0]) > 1e-3 or abs(a - s_at[1]) > 1e-3
    # decoupled: content part unrotated, RoPE only on a separate key -> absorption exact
    kr = g.standard_normal(8)
    qr = g.standard_normal(8)
    for p in (3, 17):
        naive = q @ (wuk @ c) + ref.rope_rotate(qr, pq, base) @ ref.rope_rotate(kr, p, base)
        absorbed = (wuk.T @ q) @ c + ref.rope_rotate(qr, pq, base) @ ref.rope_rotate(kr, p, base)
        assert abs(naive - absorbed) < 1e-12


# ----------------------------------------------------------------------------------------
# Brute force on tiny inputs (pure Python loops, no array arithmetic)
# ----------------------------------------------------------------------------------------

def _brute_force(c, kr, qn, qr, wuk, wuv, scale):
    L, r = len(c), len(c[0])
    T, H, dh = len(qn), len(qn[0]), len(qn[0][0])
    dr = len(kr[0])
    dv = len(wuv[0])
    o = [[[0.0] * dv for _ in range(H)] for _ in range(T)]
    for t in range(T):
        n = L - T + 1 + t
        for h in range(H):
            s = []
            for l in range(n):
                k = [sum(wuk[h][i][j] * c[l][j] for j in range(r)) for i in range(dh)]
                dot = sum(qn[t][h][i] * k[i] for i in range(dh))
                dot += sum(qr[t][h][i] * kr[l][i] for i in range(dr))
                s.append(dot * scale)
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = sum(e)
            for i in range(dv):
                v = [sum(wuv[h][i][j] * c[l][j] for j in range(r)) for l in range(n)]
                o[t][h][i] = sum(e[l] / z * v[l] for l in range(n))
    return np.array(o)


@pytest.mark.parametrize("T", [1, 3])
def test_bruteforce_small(T):
    args, scale = _tiny_inputs(L=7, T=T, H=3, dh=4, r=6, dr=4)
    bf = _brute_force(*[a.tolist() for a in args], scale)
    a = ref.naive_decode(*args, scale)
    b = ref.absorbed_decode(*args, scale)
    assert np.max(np.abs(a.o - bf)) < 1e-12
    assert np.max(np.abs(b.o - bf)) < 1e-12


def test_expanded_attention_equals_library_causal_sdpa_and_the_naive_form():
    # a prompt (every token new): torch's causal scaled-dot-product attention, float64
    g = np.random.default_rng([0, 90])
    L, H, D, dv = 11, 3, 6, 5
    Q = g.standard_normal((L, H, D))
    K = g.standard_normal((L, H, D))
    V = g.standard_normal((L, H, dv))
    o = ref.expanded_attention(Q, K, V, 0.4)
    t = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q.transpose(1, 0, 2)), torch.from_numpy(K.transpose(1, 0, 2)),
        torch.from_numpy(V.transpose(1, 0, 2)), is_causal=True, scale=0.4)
    assert np.max(np.abs(o - t.numpy().transpose(1, 0, 2))) < 1e-12
    # keys and values expanded from the latent: the naive form (pinned by brute force above),
    # for a decode step of 3 tokens and for a whole prompt
    for L_, T in ((9, 3), (7, 7)):
        args, scale = _tiny_inputs(L=L_, T=T, H=2, dh=4, r=6, dr=4)
        c, kr, qn, qr, wuk, wuv = args
        Kx = np.concatenate([np.einsum("lr,hdr->lhd", c, wuk),
                             np.repeat(kr[:, None, :], wuk.shape[0], axis=1)], axis=-1)
        Vx = np.einsum("lr,hdr->lhd", c, wuv)
        Qx = np.concatenate([qn, qr], axis=-1)
        want = ref.naive_decode(*args, scale).o
        assert np.max(np.abs(ref.expanded_attention(Qx, Kx, Vx, scale) - want)) < 1e-12
        # negative control: the heads' keys swapped
        assert np.max(np.abs(ref.expanded_attention(Qx, Kx[:, ::-1], Vx, scale) - want)) > 1e-3


def test_causal_mask_is_not_off_by_one():
    args, scale = _tiny_inputs(L=9, T=3, H=2, dh=4, r=6, dr=4)
    c, kr, qn, qr, wuk, wuv = args
    full = ref.naive_decode(*args, scale)
    # query t of a T-token step equals a 1-token step over the first L - T + t + 1 rows
    for t in range(3):
        n = 9 - 3 + t + 1
        one = ref.naive_decode(c[:n], kr[:n], qn[t:t + 1], qr[t:t + 1], wuk, wuv, scale)
        assert np.max(np.abs(one.o[0] - full.o[t])) < 1e-12
        assert np.max(np.abs(one.lse[0] - full.lse[t])) < 1e-12


# ----------------------------------------------------------------------------------------
# Special cases that reduce to a closed form or a library routine
# ----------------------------------------------------------------------------------------

def test_single_row_returns_value_of_that_row():
    args, scale = _tiny_inputs(L=1)
    c, kr, qn, qr, wuk, wuv = args
    out = ref.naive_decode(*args, scale)
    for h in range(wuv.shape[0]):
        assert np.max(np.abs(out.o[0, h] - wuv[h] @ c[0])) < 1e-14
    assert np.max(np.abs(out.o_lat[0] - c[0])) < 1e-14


def test_identical_rows_make_output_query_independent():
    args, scale = _tiny_inputs(L=10)
    c, kr, qn, qr, wuk, wuv = args
    c[:] = c[0]
    kr[:] = kr[0]
    out = ref.naive_decode(c, kr, qn, qr, wuk, wuv, scale)
    out2 = ref.naive_decode(c, kr, -3.0 * qn, qr + 1.0, wuk, wuv, scale)
    for h in range(wuv.shape[0]):
        assert np.max(np.abs(out.o[0, h] - wuv[h] @ c[0])) < 1e-12
    assert np.max(np.abs(out.o - out2.o)) < 1e-12


def test_identity_weights_reduce_to_library_sdpa():
    g = np.random.default_rng([0, 79])
    L, r = 12, 16
    c = g.standard_normal((L, r))
    q = g.standard_normal((1, 1, r))
    eye = np.eye(r)[None]
    out = ref.naive_decode(c, np.zeros((L, 0)), q, np.zeros((1, 1, 0)), eye, eye, 1.0 / math.sqrt(r))
    t = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[0][None]), torch.from_numpy(c[None]), torch.from_numpy(c[None]))
    assert np.max(np.abs(out.o[0, 0] - t.numpy()[0, 0])) < 1e-12


def test_softmax_rows_sum_to_one_and_masked_entries_are_zero():
    g = np.random.default_rng([0, 80])
    s = g.standard_normal((5, 17)) * 10
    s[:, 11:] = -np.inf
    p = ref.softmax(s)
    assert np.max(np.abs(p.sum(-1) - 1.0)) < 1e-12
    assert np.all(p[:, 11:] == 0.0)
    assert np.max(np.abs(ref.logsumexp(s) - np.log(np.exp(s).sum(-1)))) < 1e-12


def test_latent_outputs_and_lse_consistent():
    args, scale = _tiny_inputs(L=20, T=2)
    out = ref.naive_decode(*args, scale)
    c, kr, qn, qr, wuk, wuv = args
    Q = np.concatenate([ref.absorb_query(qn, wuk), qr], axis=-1)
    lat = ref.latent_attention(Q, np.concatenate([c, kr], axis=1), c.shape[1], scale, T=2)
    assert np.max(np.abs(lat.o_lat - out.o_lat)) < 1e-12
    assert np.max(np.abs(lat.lse - out.lse)) < 1e-12
    assert np.max(np.abs(ref.output_ref(lat.o_lat, wuv) - out.o)) < 1e-12


def test_combine_of_disjoint_ranges_equals_whole():
    g = np.random.default_rng([0, 81])
    L, H, r, dr = 50, 4, 8, 4
    rows = g.standard_normal((L, r + dr))
    Q = g.standard_normal((1, H, r + dr)) * 2
    whole = ref.latent_attention(Q, rows, r, 0.3, T=1)
    cuts = [0, 7, 8, 31, 50]
    parts = [ref.latent_attention(Q, rows[a:b], r, 0.3, T=1) for a, b in zip(cuts[:-1], cuts[1:])]
    o, L_ = ref.combine_ref([p.o_lat for p in parts], [p.lse for p in parts])
    assert np.max(np.abs(o - whole.o_lat)) < 1e-12
    assert np.max(np.abs(L_ - whole.lse)) < 1e-12
    # one part: the combine is the identity
    o1, l1 = ref.combine_ref([whole.o_lat], [whole.lse])
    assert np.max(np.abs(o1 - whole.o_lat)) == 0 and np.max(np.abs(l1 - whole.lse)) == 0


# ----------------------------------------------------------------------------------------
# RoPE, RMSNorm, bf16 rounding, projections
# ----------------------------------------------------------------------------------------

def test_rope_matches_complex_rotation_and_properties():
    g = np.random.default_rng([0, 82])
    d, base = 16, 10000.0
    x = g.standard_normal((5, d))
    pos = np.array([0, 1, 7, 100, 32767])
    y = ref.rope_rotate(x, pos, base)
    # complex form: (x0 + i x1) * exp(i * pos * base^(-2k/d))
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(
        1j * pos[:, None] * base ** (-2.0 * np.arange(d // 2) / d))
    assert np.max(np.abs(y[:, 0::2] - z.real)) < 1e-12
    assert np.max(np.abs(y[:, 1::2] - z.imag)) < 1e-12
    assert np.max(np.abs(np.linalg.norm(y, axis=1) - np.linalg.norm(x, axis=1))) < 1e-12
    assert np.max(np.abs(y[0] - x[0])) == 0.0                 # position 0 is the identity
    q, k = x[1], x[2]
    # relative position: (R_p q).(R_p' k) depends only on p - p'
    a = ref.rope_rotate(q, 50, base) @ ref.rope_rotate(k, 20, base)
    b = ref.rope_rotate(q, 1030, base) @ ref.rope_rotate(k, 1000, base)
    assert abs(a - b) < 1e-10
    assert abs(a - ref.rope_rotate(q, 30, base) @ k) < 1e-10
    # the first pair turns fastest: theta_0 = 1, theta_last = base^(-(d-2)/d)
    th = ref.rope_inv_freq(d, base)
    assert th[0] == 1.0 and abs(th[-1] - base ** (-(d - 2) / d)) < 1e-18


def test_rmsnorm_closed_form_and_library():
    g = np.random.default_rng([0, 83])
    x = g.standard_normal((6, 64)) * 3
    eps = 1e-6
    y = ref.rms_norm(x, np.ones(64), eps)
    ms = np.mean(x * x, axis=1)
    assert np.max(np.abs(np.mean(y * y, axis=1) - ms / (ms + eps))) < 1e-12
    gam = 1 + 0.1 * g.standard_normal(64)
    lib = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(gam), eps)
    assert np.max(np.abs(ref.rms_norm(x, gam, eps) - lib.numpy())) < 1e-12


def test_round_bf16_matches_library_conversion():
    g = np.random.default_rng([0, 84])
    vals = [g.standard_normal(20000).astype(np.float32),
            (g.standard_normal(2000) * 1e-39).astype(np.float32),      # subnormals
            (g.standard_normal(2000) * 1e38).astype(np.float32),       # near overflow
            np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.3895314e38, -3.3961814e38],
                     dtype=np.float32)]
    # exact ties: 1 + 2^-8 (tie, rounds to 1) and 1 + 3*2^-8 (tie, rounds up to 1 + 2^-6)
    ties = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8)], dtype=np.float32)
    for v in vals + [ties]:
        lib = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
        mine = ref.round_bf16(v.astype(np.float64))
        assert np.array_equal(mine, lib, equal_nan=True), v[mine != lib][:5]
    assert ref.round_bf16(np.array([1 + 2 ** -8]))[0] == 1.0
    assert ref.round_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6


def test_round_fp8_e4m3_matches_library_conversion():
    # every E4M3 value, the midpoints between neighbours (ties to even), points just off the
    # midpoints, subnormals, and random values; torch's float8_e4m3fn conversion bit for bit
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    vals = np.unique(codes[np.isfinite(codes)])
    mids = (vals[1:] + vals[:-1]) / 2
    g = np.random.default_rng([0, 92])
    x = np.concatenate([vals, mids, mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20),
                        g.uniform(-448, 448, 2000), g.uniform(-0.02, 0.02, 500),
                        [0.0, -0.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11, 447.9, -447.9]])
    x = x.astype(np.float32)   # the library converts from float32
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).float().numpy()
    got = ref.round_fp8_e4m3(x.astype(np.float64))
    assert np.array_equal(got.astype(np.float32), want)
    # the grid: 1 + k/8 between 1 and 2, spacing 2^-9 among the subnormals, 448 the largest
    assert ref.round_fp8_e4m3(np.array([1.0 + 1 / 16]))[0] == 1.0      # tie -> even mantissa
    assert ref.round_fp8_e4m3(np.array([1.0 + 3 / 16]))[0] == 1.25
    assert ref.round_fp8_e4m3(np.array([1000.0]))[0] == 448.0          # saturation
    codes_, scale = ref.quantize_rows_fp8(np.array([[0.5, -2.0, 1.0], [0.0, 0.0, 0.0]]))
    assert scale[0] == 2.0 / 448 and scale[1] == 1.0
    assert np.array_equal(codes_[0], [112.0, -448.0, 224.0]) and not codes_[1].any()


def test_project_layer_matches_library_linear():
    w = mi.WORKLOADS["small_fp32"]
    d = mi.layer_draw(mi.scaled(w, batch=2, cached=5))
    p = ref.project_layer(d.x, w.num_heads, w.head_dim, w.rope_dim, d.w_dkv, d.w_kr, d.w_qr,
                          w_dq=d.w_dq, w_uq=d.w_uq, gamma_q=d.gamma_q, eps=w.rms_eps)
    F = torch.nn.functional
    x = torch.from_numpy(d.x)
    cq = F.rms_norm(F.linear(x, torch.from_numpy(d.w_dq)), (w.q_rank,), eps=w.rms_eps)
    q = F.linear(cq, torch.from_numpy(d.w_uq)).reshape(2, -1, w.num_heads, w.head_dim)
    assert np.max(np.abs(p.q_nope - q.numpy())) < 1e-12
    assert np.max(np.abs(p.ckv_raw - F.linear(x, torch.from_numpy(d.w_dkv)).numpy())) < 1e-12
    assert np.max(np.abs(p.krope_raw - F.linear(x, torch.from_numpy(d.w_kr)).numpy())) < 1e-12


# ----------------------------------------------------------------------------------------
# Paged placement (integer work: exact)
# ----------------------------------------------------------------------------------------

def test_paged_placement_bruteforce_and_invalid_entries():
    g = np.random.default_rng([0, 85])
    B, maxb, bs, nb = 3, 4, 5, 9
    table = g.permutation(nb)[: B * maxb - 3].tolist() + [-1, 99, 4]
    table = np.array(table, dtype=np.int32).reshape(B, maxb)
    seq = g.integers(0, B, 200)
    pos = g.integers(-2, maxb * bs + 3, 200)
    pl = ref.paged_placement(seq, pos, table, bs, nb)
    for i in range(200):
        b, p = int(seq[i]), int(pos[i])
        ok = 0 <= p < maxb * bs and 0 <= table[b][p // bs] < nb
        assert bool(pl.valid[i]) == ok
        if ok:
            assert pl.block[i] == table[b][p // bs] and pl.slot[i] == p % bs


def test_append_grows_cache_like_the_shape_trace():
    g = read_golden("shape_trace.txt")
    B, S, r = int(g["batch"]), int(g["prefill"]), int(g["latent"])
    bs = 4
    nblk = (S + 1 + bs - 1) // bs
    table = np.arange(B * nblk, dtype=np.int32).reshape(B, nblk)
    pool = np.full((B * nblk, bs, r + 2), np.nan)
    rng = np.random.default_rng([0, 86])
    seq = np.repeat(np.arange(B), S)
    pos = np.tile(np.arange(S), B)
    ref.append_ref(pool, rng.standard_normal((B * S, r)), rng.standard_normal((B * S, 2)),
                   np.ones(r), seq, pos, table, bs, 1e-6, 1e4, False)
    filled = lambda b: sum(np.isfinite(pool[table[b], :, 0]).ravel())  # noqa: E731
    assert [B, filled(0), r] == [int(v) for v in g["after_prefill"]]
    ref.append_ref(pool, rng.standard_normal((B, r)), rng.standard_normal((B, 2)), np.ones(r),
                   np.arange(B), np.full(B, S), table, bs, 1e-6, 1e4, False)
    assert [B, filled(0), r] == [int(v) for v in g["after_one_step"]]
    assert filled(1) == S + 1


# ----------------------------------------------------------------------------------------
# The tolerance harness itself must be able to fail
# ----------------------------------------------------------------------------------------

def _small_decode(dtype="bf16"):
    w = mi.scaled(mi.WORKLOADS["small_bf16"], batch=1, cached=200)
    rows = int(mi.total_rows(w)[0])
    d = mi.sequence_draw(w, 0, rows)
    wuk, wuv = mi.up_projection_weights(w)
    return w, d, wuk, wuv, ref.decode_sequence_from_raw(
        d.ckv_raw, d.krope_raw, d.q_nope, d.q_rope_raw, wuk, wuv, np.ones(w.kv_rank),
        w.softmax_scale, w.rms_eps, w.rope_base, store_bf16=True)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_tolerance_negative_controls(dtype):
    w, d, wuk, wuv, out = _small_decode()
    o = out.o[0]
    ok, _ = compare.within(o, o, dtype)
    assert ok
    assert not compare.within(np.zeros_like(o), o, dtype)[0]
    swapped = o.copy()
    swapped[[0, 1]] = swapped[[1, 0]]
    assert not compare.within(swapped, o, dtype)[0]
    # a one-token shift of the query position changes the output beyond tolerance
    rows = d.ckv_raw.shape[0]
    c = ref.cache_rows(d.ckv_raw, d.krope_raw, np.ones(w.kv_rank), np.arange(rows), w.rms_eps,
                       w.rope_base, True)
    qr = ref.rope_rotate(d.q_rope_raw.astype(np.float64), np.array([[rows - 2]]), w.rope_base)
    shifted = ref.naive_decode(c[:, :w.kv_rank], c[:, w.kv_rank:], d.q_nope, qr, wuk, wuv,
                               w.softmax_scale)
    assert not compare.within(shifted.o[0], o, dtype)[0]


def test_output_ulp_allowance_admits_the_formats_rounding_only():
    g = np.random.default_rng([0, 91])
    exp = 0.1 * g.standard_normal((4, 64))
    exp[2, 5] = 1.0585                        # > 5x the rms, just above a power of two
    got = ref.round_bf16(exp)                 # the exact values, rounded to bf16 once
    ok, e = compare.within(got, exp, "bf16")
    assert not ok and e > 2e-2                # the format alone misses the plain bar ...
    ok, e = compare.within(got, exp, "bf16", out_ulps=compare.PROMPT_OUTPUT_ULPS)
    assert ok, e                              # ... and meets it with one ulp granted
    bad = got.copy()
    bad[2, 5] += 3 * compare.bf16_ulp(np.array(1.0585))
    assert not compare.within(bad, exp, "bf16", out_ulps=compare.PROMPT_OUTPUT_ULPS)[0]
    bad = got + 0.03 * np.sqrt(np.mean(exp ** 2))   # a real error on every element
    assert not compare.within(bad, exp, "bf16", out_ulps=compare.PROMPT_OUTPUT_ULPS)[0]
    assert not compare.within(np.zeros_like(exp), exp, "bf16",
                              out_ulps=compare.PROMPT_OUTPUT_ULPS)[0]


def test_needle_makes_attention_peaky():
    w = mi.scaled(mi.WORKLOADS["small_bf16"], batch=1, cached=300)
    rows = int(mi.total_rows(w)[0])
    d = mi.sequence_draw(w, 0, rows)
    j = mi.plant_needle(w, d, factor=8.0)
    wuk, wuv = mi.up_projection_weights(w)
    c = ref.cache_rows(d.ckv_raw, d.krope_raw, np.ones(w.kv_rank), np.arange(rows), w.rms_eps,
                       w.rope_base, True)
    qr = ref.rope_rotate(d.q_rope_raw.astype(np.float64), np.array([[rows - 1]]), w.rope_base)
    Q = np.concatenate([ref.absorb_query(d.q_nope, wuk), qr], axis=-1)
    s = np.einsum("thd,ld->thl", Q, c) * w.softmax_scale
    p = ref.softmax(s)
    assert p[0, :, j].max() > 0.5
    assert np.argmax(p[0].max(axis=1)) is not None


# ----------------------------------------------------------------------------------------
# The bf16-query form: only the query's storage differs from the absorbed form
# ----------------------------------------------------------------------------------------

def _emulate_bf16_path(Q, rows, r, scale, wuv):
    """bf16 query, weights rounded to bf16 before the weighted sum, bf16 output."""
    Qb = ref.round_bf16(Q)
    s = np.einsum("thd,ld->thl", Qb, rows) * scale
    pe = np.exp(s - s.max(-1, keepdims=True))
    lat = np.einsum("thl,lj->thj", ref.round_bf16(pe), rows[:, :r]) / pe.sum(-1, keepdims=True)
    return ref.round_bf16(ref.output_ref(lat, wuv)), lat


@pytest.mark.parametrize("factor", [0.0, 4.0, 16.0])
def test_bf16_query_form(factor):
    w = mi.scaled(mi.WORKLOADS["small_bf16"], batch=1, cached=400)
    rows_n = int(mi.total_rows(w)[0])
    d = mi.sequence_draw(w, 0, rows_n)
    if factor:
        mi.plant_needle(w, d, factor=factor)
    wuk, wuv = (mi.storage_round(w, x) for x in mi.up_projection_weights(w))
    ckv, kr, qn, qr = (mi.storage_round(w, x) for x in (d.ckv_raw, d.krope_raw, d.q_nope,
                                                         d.q_rope_raw))
    g = np.ones(w.kv_rank)
    args = (ckv, kr, qn, qr, wuk, wuv, g, w.softmax_scale, w.rms_eps, w.rope_base)
    exact = ref.decode_sequence_from_raw(*args, True, "absorbed")
    qb = ref.decode_sequence_bf16_query(*args)
    # identical to the absorbed form when the query is already bf16-representable
    Q = ref.absorb_ref(qn, qr, np.array([rows_n - 1]), wuk, w.rope_base)
    rows = ref.cache_rows(ckv, kr, g, np.arange(rows_n), w.rms_eps, w.rope_base, True)
    direct = ref.latent_attention(ref.round_bf16(Q), rows, w.kv_rank, w.softmax_scale, 1)
    assert np.max(np.abs(direct.o_lat - qb.o_lat)) < 1e-12
    # an emulation of the bf16 path's own roundings stays within 2e-2 of the bf16-query form
    o, lat = _emulate_bf16_path(Q, rows, w.kv_rank, w.softmax_scale, wuv)
    assert compare.within(o, qb.o, "bf16")[0] and compare.within(lat, qb.o_lat, "bf16")[0]
    # and a head swap does not
    sw = o.copy()
    sw[:, [0, 1]] = sw[:, [1, 0]]
    assert not compare.within(sw, qb.o, "bf16")[0]
    # the query's storage is the whole difference from the exact form (small when diffuse)
    if not factor:
        assert compare.within(qb.o, exact.o, "bf16")[0]


def _fp32_absorbed_query(qn, qr, pos, wuk, base):
    """An fp32 implementation of the absorbed query: each latent element summed in float32,
    in reverse order, before it is rounded to bfloat16 (the RoPE part as the oracle's)."""
    qn32 = np.asarray(qn, dtype=np.float32)
    w32 = np.asarray(wuk, dtype=np.float32)
    T, H, dh = qn32.shape
    acc = np.zeros((T, H, w32.shape[2]), dtype=np.float32)
    for i in reversed(range(dh)):
        acc = (acc + qn32[:, :, i, None] * w32[None, :, i, :]).astype(np.float32)
    q = ref.absorb_ref(qn, qr, pos, wuk, base)
    q[..., :w32.shape[2]] = acc
    return ref.round_bf16(q)


@pytest.mark.parametrize("factor", [4.0, 8.0, 16.0])
def test_needle_tolerance_admits_only_ambiguous_roundings(factor):
    w = mi.scaled(mi.WORKLOADS["small_bf16"], batch=1, cached=400)
    n = int(mi.total_rows(w)[0])
    d = mi.sequence_draw(w, 0, n)
    j = mi.plant_needle(w, d, factor=factor)
    wuk, wuv = (mi.storage_round(w, x) for x in mi.up_projection_weights(w))
    ckv, kr, qn, qr = (mi.storage_round(w, x) for x in (d.ckv_raw, d.krope_raw, d.q_nope,
                                                         d.q_rope_raw))
    g = np.ones(w.kv_rank)
    args = (ckv, kr, qn, qr, wuk, wuv, g, w.softmax_scale, w.rms_eps, w.rope_base)
    qb = ref.decode_sequence_bf16_query(*args)
    rows = ref.cache_rows(ckv, kr, g, np.arange(n), w.rms_eps, w.rope_base, True)
    pos = np.array([n - 1])
    Qx = ref.absorb_ref(qn, qr, pos, wuk, w.rope_base)
    amb_q, amb_r = compare.needle_ambiguity(qn, wuk, Qx, rows[j], w.kv_rank)
    Qb = ref.round_bf16(Qx)
    tol_o, tol_l = compare.peaky_tolerance(Qb, rows, wuv, w.kv_rank, w.softmax_scale, j, qb.o,
                                           qb.o_lat, amb_q, amb_r)
    # the allowance is a small multiple of the plain bar, and only ambiguous elements count
    rms_o = np.sqrt(np.mean(qb.o ** 2, axis=-1, keepdims=True))
    assert np.max(tol_o / (compare.BF16_SCALED_TOL * rms_o)) < 4.0
    assert 0 < amb_q.sum() < 0.2 * amb_q.size
    # an fp32 implementation with another summation order lands inside
    Q32 = _fp32_absorbed_query(qn, qr, pos, wuk, w.rope_base)
    assert np.all((Q32 == Qb) | amb_q)  # it rounds differently only where the mask allows
    lat = ref.latent_attention(Q32, rows, w.kv_rank, w.softmax_scale, 1)
    assert np.all(np.abs(ref.output_ref(lat.o_lat, wuv) - qb.o) <= tol_o)
    assert np.all(np.abs(lat.o_lat - qb.o_lat) <= tol_l)
    # so does every ambiguous element rounded the other way at once
    flip = Qb + np.where(amb_q, np.sign(Qx - Qb + 1e-300) * compare.bf16_ulp(Qb), 0.0)
    lat = ref.latent_attention(flip, rows, w.kv_rank, w.softmax_scale, 1)
    assert np.all(np.abs(lat.o_lat - qb.o_lat) <= tol_l)
    # with the sharpest needle, one-ulp changes of a random tenth of the elements that are
    # not ambiguous already fall outside (at the milder factors they stay within the plain bar)
    if factor >= 16.0:
        rng = np.random.default_rng(5)
        other = (rng.random(Qb.shape) < 0.1) & ~amb_q
        bad = Qb + np.where(other, np.sign(Qx - Qb + 1e-300) * compare.bf16_ulp(Qb), 0.0)
        lat = ref.latent_attention(bad, rows, w.kv_rank, w.softmax_scale, 1)
        assert not np.all(np.abs(lat.o_lat - qb.o_lat) <= tol_l)
    # nor a head swap, nor a zero output
    sw = qb.o.copy()
    sw[:, [0, 1]] = sw[:, [1, 0]]
    assert not np.all(np.abs(sw - qb.o) <= tol_o)
    assert not np.all(np.abs(qb.o) <= tol_o)
