"""CUDA path vs. the CPU oracle, through the C ABI (needs a B200)."""
import math

import numpy as np
import pytest
import torch

import mla_inputs as mi
from oracle import compare, mla_ref as ref
from tests.gpu_util import check_sequence, dev_err, layer_raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mla():
    import mla_latent_kv_44_b200 as m

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _tdt(dtype):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def _store(x, dtype):
    return mi.round_to_bf16(x) if dtype == "bf16" else np.asarray(x, np.float32)


def _cfg(mla, H, dh, r, dr, bs, dtype, kernel=0):
    return mla.Config(num_heads=H, head_dim=dh, kv_rank=r, rope_dim=dr, block_size=bs,
                      dtype=dtype, decode_kernel=kernel)


def _bf16_ulp_ok(got, exp):
    """|got - exp| <= one bf16 ulp of exp (exp already a bf16 value)."""
    got = np.asarray(got, np.float64)
    exp = np.asarray(exp, np.float64)
    e = np.maximum(np.abs(exp), 2.0 ** -126)
    ulp = 2.0 ** (np.floor(np.log2(e)) - 7)
    return np.abs(got - exp) <= ulp


# ----------------------------------------------------------------------------------------
# Whole step, small workloads: hidden states -> oracle projections -> the four calls
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny_fp32", "small_fp32", "small_bf16"])
def test_full_step_small(mla, name):
    from mla_latent_kv_44_b200.step import DecodeState

    w = mi.WORKLOADS[name]
    st = DecodeState(w, raw=layer_raw(w))
    st.step()
    assert dev_err(st) == 0
    for b in range(w.batch):
        check_sequence(st, b, "naive")


@pytest.mark.parametrize("name", ["small_bf16", "dsv2"])
def test_needle_peaky_attention(mla, name):
    from mla_latent_kv_44_b200.step import DecodeState

    w = mi.WORKLOADS[name]
    if name == "dsv2":
        w = mi.scaled(w, batch=2, cached=1000)
    st = DecodeState(w, needle=8.0, gamma_perturbed=True)
    st.step()
    assert dev_err(st) == 0
    for b in range(w.batch):
        check_sequence(st, b, "naive", peaky=True)


# ----------------------------------------------------------------------------------------
# Whole step, full-size workloads: every sequence decoded, sampled sequences checked
# ----------------------------------------------------------------------------------------

def _split_sequences(rows, T):
    """Sequences with a row group that the planner splits across work ranges (from the split
    rule restated on the host in tests/test_plan.py)."""
    from tests.test_plan import expected_plan

    plan = expected_plan([int(x) for x in rows], T, int(max(rows)))
    return sorted({bt // T for bt, n in enumerate(plan["bt_nseg"]) if n >= 2})


@pytest.mark.parametrize("name", ["dsv2", "ragged", "mtp"])
def test_full_step_large(mla, name):
    """Full-size DeepSeek-V2-shaped steps. C3 (64 sequences) and C5 (32): every sequence is
    checked; C4 (128 ragged sequences): every sequence with a split row group (each of the
    planner's range boundaries inside a sequence) and a fixed sample of 16 others. The two
    shortest checked sequences go against the naive form, the rest against the absorbed
    float64 cross-form (the naive form costs about 0.3 TFLOP per 8k-row sequence)."""
    from mla_latent_kv_44_b200.step import DecodeState

    w = mi.WORKLOADS[name]
    rows = mi.total_rows(w, 0)
    if name == "ragged":
        seqs = sorted(set(_split_sequences(rows, w.new_tokens)) | set(mi.sample_sequences(w, 16)))
        assert len(seqs) >= 16
    else:
        seqs = list(range(w.batch))
    st = DecodeState(w, sequences=seqs)
    st.step()
    assert dev_err(st) == 0
    naive = sorted(seqs, key=lambda b: rows[b])[:2]
    for b in seqs:
        check_sequence(st, b, "naive" if b in naive else "absorbed")
    # every output row is finite (no sentinel rows leaked into any sequence)
    assert torch.isfinite(st.out_latent).all() and torch.isfinite(st.o.float()).all()


# ----------------------------------------------------------------------------------------
# Stage: absorbed query
# ----------------------------------------------------------------------------------------

_SIMT, _TC = 1, 2  # mla_config.decode_kernel: CUDA-core or tensor-core kernels


@pytest.mark.parametrize("dtype,shape,N,kernel", [
    ("f32", (16, 64, 64, 32), 37, 0),
    ("f32", (8, 32, 64, 16), 1, 0),
    ("bf16", (16, 64, 64, 32), 37, _SIMT),
    ("bf16", (16, 64, 64, 32), 37, _TC),
    ("bf16", (128, 128, 512, 64), 37, _SIMT),
    ("bf16", (128, 128, 512, 64), 1, _TC),
    ("bf16", (128, 128, 512, 64), 64, _TC),
    ("bf16", (128, 128, 512, 64), 200, _TC),
    ("bf16", (4, 256, 192, 0), 300, _TC),
    ("bf16", (8, 64, 128, 8), 5, _TC),
])
def test_absorb_stage(mla, dtype, shape, N, kernel):
    H, dh, r, dr = shape
    g = np.random.default_rng([1, 1, N])
    qn = _store(g.standard_normal((N, H, dh)), dtype)
    qr = _store(g.standard_normal((N, H, dr)), dtype)
    wuk = _store(g.standard_normal((H, dh, r)) / math.sqrt(r), dtype)
    pos = g.integers(0, 32768, N).astype(np.int32)
    pos[:min(N, 3)] = [0, 1, 32767][:min(N, 3)]
    dev = "cuda"
    t = _tdt(dtype)
    out = torch.empty((N, H, r + dr), dtype=t, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    cfg = _cfg(mla, H, dh, r, dr, 64, dtype, kernel)
    mla.absorb_query(cfg, torch.from_numpy(qn).to(dev, t), torch.from_numpy(qr).to(dev, t),
                     torch.from_numpy(pos).to(dev), torch.from_numpy(wuk).to(dev, t), out,
                     dev_err=err)
    got = out.float().cpu().numpy()
    assert int(err.item()) == 0
    exp = ref.absorb_ref(qn, qr, pos, wuk, 10000.0)
    if dtype == "f32":
        assert compare.normwise_rel_error(got, exp) <= 1e-5
    else:
        # one bf16 rounding (relative u = 2^-8) of an fp32 sum of d_h products, whose own error
        # is at most d_h * 2^-24 * sum |q_i w_ij|, whatever order the kernel sums in
        u = 2.0 ** -8
        mag = ref.absorb_ref(np.abs(qn), np.abs(qr), np.zeros(N, np.int64), np.abs(wuk), 10000.0)
        bound = u * np.abs(exp) + 1.01 * dh * 2.0 ** -24 * mag + 1e-30
        ok = np.abs(got - exp) <= bound
        assert ok.all(), f"{(~ok).sum()} of {ok.size} values outside one rounding"


# ----------------------------------------------------------------------------------------
# Stage: append (integer placement bit-exact, values within one rounding)
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,r,dr", [("f32", 64, 16), ("bf16", 64, 32), ("bf16", 512, 64),
                                       ("bf16", 1024, 0), ("bf16", 256, 8)])
def test_append_stage(mla, dtype, r, dr):
    g = np.random.default_rng([1, 2])
    B, maxb, bs, nb = 3, 4, 16, 14
    table = g.permutation(nb)[: B * maxb].astype(np.int32).reshape(B, maxb)
    table[1, 3] = -1          # missing block
    table[2, 2] = nb + 5      # block id outside the pool
    n = 90
    seq = g.integers(0, B, n).astype(np.int32)
    pos = g.integers(0, maxb * bs, n).astype(np.int32)
    pos[:3] = [maxb * bs, maxb * bs + 7, 0]   # past the table
    seq[3] = B                                  # sequence index outside the table
    # distinct (seq, pos) so each slot is written once
    key = seq.astype(np.int64) * 10000 + pos
    _, first = np.unique(key, return_index=True)
    keep = np.sort(first)
    seq, pos = seq[keep], pos[keep]
    n = len(seq)
    ckv = _store(g.standard_normal((n, r)) * 3, dtype)
    kr = _store(g.standard_normal((n, dr)), dtype)
    gamma = (1 + 0.1 * g.standard_normal(r)).astype(np.float32)
    D = r + dr
    t = _tdt(dtype)
    pool = torch.empty((nb, bs, D), dtype=t, device="cuda")
    ibits = torch.int16 if dtype == "bf16" else torch.int32
    pool.view(ibits).fill_(-1)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cfg = _cfg(mla, 8, 16, r, dr, bs, dtype)
    dev = "cuda"
    mla.append_latent(cfg, torch.from_numpy(ckv).to(dev, t), torch.from_numpy(kr).to(dev, t),
                      torch.from_numpy(gamma).to(dev), torch.from_numpy(seq).to(dev),
                      torch.from_numpy(pos).to(dev), torch.from_numpy(table).to(dev), pool, err)
    torch.cuda.synchronize()
    assert int(err.item()) == (mla.DEV_OOB_POS | mla.DEV_OOB_BLOCK)

    exp = np.full((nb, bs, D), np.nan)
    pl = ref.append_ref(exp, ckv, kr, gamma, seq, pos, table, bs, 1e-6, 10000.0,
                        store_bf16=(dtype == "bf16"))
    assert (~pl.valid).sum() >= 4
    bits = pool.view(ibits).cpu().numpy()
    written_gpu = ~np.all(bits == -1, axis=2)
    written_exp = np.isfinite(exp[:, :, 0])
    assert np.array_equal(written_gpu, written_exp)      # placement: bit-exact
    got = pool.float().cpu().numpy()[written_exp]
    want = exp[written_exp]
    if dtype == "bf16":
        ok = _bf16_ulp_ok(got, want)
        assert ok.all(), f"{(~ok).sum()} values off by more than one bf16 ulp"
    else:
        assert compare.normwise_rel_error(got, want) <= 1e-6


# ----------------------------------------------------------------------------------------
# Stage: decode (plan + attention + combine) on oracle-built cache rows
# ----------------------------------------------------------------------------------------

def _decode_case(mla, dtype, H, dh, r, dr, lengths, T, bs=64, kernel=0, permute=True, seed=3,
                 table_override=None, needle=0.0):
    g = np.random.default_rng([seed, 4])
    D = r + dr
    B = len(lengths)
    rows = [_store(np.concatenate([g.standard_normal((L, r)), g.standard_normal((L, dr)) * 2], 1),
                   dtype) for L in lengths]
    Q = _store(g.standard_normal((B * T, H, D)) * 0.25, dtype)
    if needle:
        # one earlier row per sequence made parallel to head 0's query: peaky attention
        for b in range(B):
            j = (lengths[b] - T) // 2
            rows[b][j] = _store(needle * Q[b * T, 0] / np.sqrt(np.mean(Q[b * T, 0] ** 2)), dtype)
    nblk = [(L + bs - 1) // bs for L in lengths]
    nb = sum(nblk) + 3
    ids = np.random.default_rng([seed, 5]).permutation(nb) if permute else np.arange(nb)
    maxb = max(nblk)
    table = np.full((B, maxb), -1, np.int32)
    off = 0
    pool_h = np.full((nb, bs, D), np.nan, np.float32)
    for b in range(B):
        table[b, :nblk[b]] = ids[off:off + nblk[b]]
        off += nblk[b]
        for j in range(lengths[b]):
            pool_h[table[b, j // bs], j % bs] = rows[b][j]
    if table_override is not None:
        table = table_override(table)
    t = _tdt(dtype)
    dev = "cuda"
    pool = torch.from_numpy(pool_h).to(dev, t)
    cfg = _cfg(mla, H, dh, r, dr, bs, dtype, kernel)
    ws = torch.empty(mla.decode_workspace_size(cfg, B, T), dtype=torch.uint8, device=dev)
    out = torch.full((B * T, H, r), float("nan"), device=dev)
    lse = torch.full((B * T, H), float("nan"), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    seq_lens = torch.tensor(lengths, dtype=torch.int32, device=dev)
    mla.decode(cfg, torch.from_numpy(Q).to(dev, t), pool, torch.from_numpy(table).to(dev),
               seq_lens, T, ws, out, lse, err)
    torch.cuda.synchronize()
    return dict(Q=Q, rows=rows, out=out.cpu().numpy(), lse=lse.cpu().numpy(),
                err=int(err.item()), T=T, H=H, r=r, dh=dh, dr=dr)


def _check_decode(c, dtype, scale):
    T = c["T"]
    for b, rows in enumerate(c["rows"]):
        exp = ref.latent_attention(c["Q"][b * T:(b + 1) * T], rows, c["r"], scale, T)
        got = c["out"][b * T:(b + 1) * T]
        ok, e = compare.within(got, exp.o_lat, dtype)
        assert ok, f"seq {b} (len {len(rows)}): error {e}"
        tol = 1e-5 * max(1.0, np.abs(exp.lse).max()) if dtype == "f32" else 2e-2
        assert np.max(np.abs(c["lse"][b * T:(b + 1) * T] - exp.lse)) <= tol


LENGTHS = [1, 2, 63, 64, 65, 127, 200, 1000, 64 * 74 * 2 + 5]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 4])
def test_decode_stage_small_heads(mla, dtype, T):
    lengths = [L + T - 1 for L in LENGTHS]
    c = _decode_case(mla, dtype, 16, 64, 64, 32, lengths, T)
    assert c["err"] == 0
    _check_decode(c, dtype, 1 / math.sqrt(96))


@pytest.mark.parametrize("T", [1, 4])
def test_decode_stage_dsv2_shape(mla, T):
    lengths = [L + T - 1 for L in [1, 65, 129, 1000, 64 * 74 + 3]]
    c = _decode_case(mla, "bf16", 128, 128, 512, 64, lengths, T)
    assert c["err"] == 0
    _check_decode(c, "bf16", 1 / math.sqrt(192))


@pytest.mark.parametrize("shape", [(16, 64, 64, 32), (128, 128, 512, 64)])
def test_decode_stage_needle(mla, shape):
    # Q given in bf16 (the same bits for both sides): only the kernel's own roundings remain,
    # so the 2e-2 bound holds on unit-scaled outputs even when one row takes most of the weight
    H, dh, r, dr = shape
    lengths = [70, 300, 1000]
    c = _decode_case(mla, "bf16", H, dh, r, dr, lengths, 1, needle=3.0)
    assert c["err"] == 0
    scale = 1 / math.sqrt(dh + dr)
    p = ref.softmax(np.einsum("d,ld->l", c["Q"][0, 0], c["rows"][0]) * scale)
    assert p.max() > 0.5
    _check_decode(c, "bf16", scale)


def test_decode_many_short_sequences(mla):
    # more row groups than work ranges: segments outnumber ranges
    g = np.random.default_rng([5, 5])
    lengths = g.integers(1, 150, 300).tolist()
    c = _decode_case(mla, "f32", 4, 32, 32, 8, lengths, 1)
    assert c["err"] == 0
    _check_decode(c, "f32", 1 / math.sqrt(40))


def test_decode_block_size_not_multiple_of_chunk(mla):
    lengths = [5, 99, 300, 1001]
    c = _decode_case(mla, "f32", 8, 32, 64, 16, lengths, 1, bs=24)
    assert c["err"] == 0
    _check_decode(c, "f32", 1 / math.sqrt(48))


def test_decode_is_deterministic_and_paging_invariant(mla):
    lengths = [70, 1000, 64 * 80 + 1]
    a = _decode_case(mla, "bf16", 16, 64, 64, 32, lengths, 1, permute=True)
    b = _decode_case(mla, "bf16", 16, 64, 64, 32, lengths, 1, permute=True)
    c = _decode_case(mla, "bf16", 16, 64, 64, 32, lengths, 1, permute=False)
    assert np.array_equal(a["out"], b["out"]) and np.array_equal(a["lse"], b["lse"])
    assert np.array_equal(a["out"], c["out"]) and np.array_equal(a["lse"], c["lse"])


def test_decode_flags_bad_lengths_and_blocks(mla):
    # sequence 3 meets a block id outside the pool: no fault, the bit is set, and the other
    # sequences are still correct.
    lengths = [100, 1, 130, 200]

    def corrupt(table):
        table = table.copy()
        table[3, 1] = 10_000
        return table

    c = _decode_case(mla, "f32", 8, 32, 64, 16, lengths, 1, table_override=corrupt)
    assert c["err"] == mla.DEV_OOB_BLOCK
    c["rows"] = c["rows"][:3]
    _check_decode(c, "f32", 1 / math.sqrt(48))
    # now impossible lengths through seq_lens directly
    g = np.random.default_rng(0)
    H, r, dr, bs = 4, 32, 8, 16
    cfg = _cfg(mla, H, 8, r, dr, bs, "f32")
    dev = "cuda"
    pool = torch.zeros((4, bs, r + dr), device=dev)
    table = torch.tensor([[0, 1], [2, 3]], dtype=torch.int32, device=dev)
    seq_lens = torch.tensor([0, 2 * bs + 1], dtype=torch.int32, device=dev)
    ws = torch.empty(mla.decode_workspace_size(cfg, 2, 1), dtype=torch.uint8, device=dev)
    out = torch.full((2, H, r), float("nan"), device=dev)
    lse = torch.zeros((2, H), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    Q = torch.from_numpy(g.standard_normal((2, H, r + dr)).astype(np.float32)).to(dev)
    mla.decode(cfg, Q, pool, table, seq_lens, 1, ws, out, lse, err)
    torch.cuda.synchronize()
    assert int(err.item()) & mla.DEV_BAD_LENGTH
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


# ----------------------------------------------------------------------------------------
# Stage: output projection
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,shape,N,kernel", [
    ("f32", (8, 32, 64), 21, 0),
    ("bf16", (128, 128, 512), 21, _SIMT),
    ("bf16", (128, 128, 512), 1, _TC),
    ("bf16", (128, 128, 512), 64, _TC),
    ("bf16", (128, 128, 512), 200, _TC),
    ("bf16", (16, 64, 64), 8, _TC),
    ("bf16", (8, 32, 64), 21, _TC),
    ("bf16", (2, 200, 320), 150, _TC),
])
def test_output_stage(mla, dtype, shape, N, kernel):
    H, dv, r = shape
    g = np.random.default_rng([1, 6, N])
    lat = g.standard_normal((N, H, r)).astype(np.float32) * 0.05
    wuv = _store(g.standard_normal((H, dv, r)) / math.sqrt(r), dtype)
    t = _tdt(dtype)
    o = torch.empty((N, H, dv), dtype=t, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cfg = _cfg(mla, H, dv, r, 0, 64, dtype, kernel)
    mla.output(cfg, torch.from_numpy(lat).cuda(), torch.from_numpy(wuv).to("cuda", t), o,
               dev_err=err)
    got = o.float().cpu().numpy()
    assert int(err.item()) == 0
    exp = ref.output_ref(lat, wuv)
    if dtype == "f32":
        assert compare.normwise_rel_error(got, exp) <= 1e-5
        return
    # bf16: an fp32 sum of r products (error <= r * 2^-24 * sum |w_ij lat_j|) rounded once to
    # bf16 (relative u = 2^-8). The tensor-core kernel feeds the latent to its bf16 MMA as
    # hi + lo (hi = bf16(x), lo = bf16(x - hi)), which misses x by at most 2^-16 |x| and sums
    # 2r products instead of r.
    u = 2.0 ** -8
    mag = ref.output_ref(np.abs(lat), np.abs(wuv))
    operand, terms = (2.0 ** -16, 2 * r) if kernel == _TC else (0.0, r)
    bound = u * np.abs(exp) + (1 + u) * (operand + 1.02 * terms * 2.0 ** -24) * mag + 1e-30
    ok = np.abs(got - exp) <= bound
    assert ok.all(), f"{(~ok).sum()} of {ok.size} values outside the bound"


def test_empty_calls_launch_nothing(mla):
    cfg = _cfg(mla, 8, 32, 64, 16, 64, "f32")
    x = torch.empty((0, 8, 32), device="cuda")
    mla.absorb_query(cfg, x, x, torch.empty(0, dtype=torch.int32, device="cuda"), x, x)
    mla.output(cfg, torch.empty((0, 8, 64), device="cuda"), x, x)
    torch.cuda.synchronize()
