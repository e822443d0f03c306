"""Plain CPU reference of MLA decode in float64 -- TEST INFRASTRUCTURE ONLY.

Nothing on the product path may import, call or execute this module: only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use it. It shares no code,
table or constant generator with the CUDA library.

Every routine below is the textbook definition written out with NumPy, in the order and
notation of the pages it cites:

* "DeepSeek MLA, Built From the Paper" (sections 1 "The problem MLA solves", 2 "Decoupled RoPE",
  3 "Matrix absorption"),
* "MLA from scratch in PyTorch" (sections "Module structure", "The MLAAttention module",
  "KV cache management during decode", "Absorbing projections (inference optimisation)"),
* "Build a DeepSeek Model from Scratch", chapter 3 (figure captions on the score and output
  rearrangements, the latent-cache update, and RoPE's pairwise rotation),
* "Multi-head latent attention" (section "Compress keys and values into one latent").

Readings where the pages are silent (each is listed in the design notes):

* RoPE rotates adjacent pairs (2i, 2i+1) by the angle pos * base^(-2i/d_r), computed in
  float64 here (RoFormer's convention, which the course page on DeepSeek-V2 cites).
* The softmax scale with the decoupled RoPE key is 1/sqrt(d_h + d_r): the query is the
  concatenation [q_nope, q_rope] of width d_h + d_r ("Multi-head latent attention",
  ``_project_mla``), and scaled dot-product attention divides by the root of the query width.
* The RoPE key is one d_r-wide row per token shared by all heads (sections above of the
  first and last page); it is broadcast to every head in the naive form.
* The new token's latent row is appended before attention and the token attends to itself;
  with T new tokens, query t attends rows 0 .. S + t (causal among the new tokens).
* The cache stores bfloat16 for the bf16 workloads ("KV cache management during decode"
  allocates the latent cache in torch.bfloat16); the rounding is round-to-nearest-even.
* RMSNorm uses eps = 1e-6 and a gain gamma (the page's ``nn.RMSNorm(d_c)`` gives neither).

Parity of every function here is pinned by tests under ``tests/test_oracle_*.py`` against the
pages' printed values, closed forms, brute force and library routines.
"""
from __future__ import annotations

from typing import NamedTuple, Optional, Sequence

import numpy as np

F64 = np.float64


# --------------------------------------------------------------------------------------
# Elementary pieces
# --------------------------------------------------------------------------------------

def rms_norm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * gamma.

    "MLA from scratch in PyTorch", The MLAAttention module: ``norm_kv`` is applied to the KV
    latent before it is cached (and ``norm_q`` to the query latent).
    """
    x = np.asarray(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * gamma


def rope_inv_freq(d_r: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/d_r) for i < d_r/2, in float64 (RoFormer; pairs share one theta)."""
    i = np.arange(d_r // 2, dtype=F64)
    return np.power(F64(base), -2.0 * i / d_r)


def rope_rotate(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate adjacent pairs (x[2i], x[2i+1]) of the last axis by the angle pos * theta_i.

    "Build a DeepSeek Model from Scratch" ch. 3, the two RoPE figures (a query or key vector's
    dimensions taken two at a time, each pair turned as a 2-D vector through an angle that
    grows with the position). ``pos`` broadcasts against x.shape[:-1].
    """
    x = np.asarray(x)
    d_r = x.shape[-1]
    if d_r == 0:
        return x.copy()
    theta = rope_inv_freq(d_r, base)
    ang = np.asarray(pos, dtype=F64)[..., None] * theta          # (..., d_r/2)
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (d_r,)), dtype=np.result_type(x, F64))
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even), returned as float64.

    bfloat16 keeps 8 significant bits and float32's exponent range: a value in
    [2^(e-1), 2^e) is rounded to a multiple of 2^(e-8); below the smallest normal 2^-126 the
    spacing stays 2^-133; magnitudes that round to 2^128 or beyond become infinite.
    """
    x = np.asarray(x, dtype=F64)
    out = x.copy()
    fin = np.isfinite(x)
    v = x[fin]
    _, e = np.frexp(v)
    q = np.maximum(e - 8, -133)
    y = np.ldexp(np.rint(np.ldexp(v, -q)), q)
    y = np.where(np.abs(y) >= 2.0 ** 128, np.copysign(np.inf, y), y)
    out[fin] = y
    return out


def round_fp8_e4m3(x: np.ndarray) -> np.ndarray:
    """Round to the nearest FP8 E4M3 value, ties to even, saturating at +-448.

    E4M3 ("MLA from scratch in PyTorch", What's not in this implementation: the latent cache
    can be quantised to FP8): a sign, 4 exponent bits with bias 7 and 3 mantissa bits, so the
    values in [2^e, 2^(e+1)) are spaced 2^(e-3) for e >= -6, and below 2^-6 the subnormals are
    spaced 2^-9; the largest finite value is 1.75 * 2^8 = 448.
    """
    x = np.asarray(x, dtype=F64)
    a = np.abs(x)
    e = np.maximum(np.floor(np.log2(np.maximum(a, 2.0 ** -30))), -6.0)
    step = 2.0 ** (e - 3.0)
    y = np.minimum(np.round(a / step) * step, 448.0)   # np.round: half to even
    return np.copysign(y, x)


def quantize_rows_fp8(rows: np.ndarray):
    """(codes, scale) of cache rows stored as E4M3 with one scale per row: scale =
    max |row| / 448 (1 for an all-zero row), codes = E4M3(row / scale); a row reads back as
    codes * scale. rows (..., D) -> codes (..., D) as float values, scale (...,)."""
    rows = np.asarray(rows, dtype=F64)
    amax = np.max(np.abs(rows), axis=-1)
    scale = np.where(amax > 0, amax / 448.0, 1.0)
    return round_fp8_e4m3(rows / scale[..., None]), scale


def softmax(s: np.ndarray, axis: int = -1) -> np.ndarray:
    """exp(s - max) / sum(exp(s - max)); entries equal to -inf get exactly 0."""
    m = np.max(s, axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def logsumexp(s: np.ndarray, axis: int = -1) -> np.ndarray:
    m = np.max(s, axis=axis, keepdims=True)
    return (m + np.log(np.sum(np.exp(s - m), axis=axis, keepdims=True))).squeeze(axis)


# --------------------------------------------------------------------------------------
# Upstream projections (full layer front end, used to build inputs of the small workloads)
# --------------------------------------------------------------------------------------

class Projections(NamedTuple):
    q_nope: np.ndarray      # (B, rows, H, d_h)
    q_rope_raw: np.ndarray  # (B, rows, H, d_r)  before rotation
    ckv_raw: np.ndarray     # (B, rows, r)       before RMSNorm
    krope_raw: np.ndarray   # (B, rows, d_r)     before rotation


def project_layer(x: np.ndarray, num_heads: int, head_dim: int, rope_dim: int,
                  w_dkv: np.ndarray, w_kr: np.ndarray, w_qr: np.ndarray,
                  w_q: Optional[np.ndarray] = None, w_dq: Optional[np.ndarray] = None,
                  w_uq: Optional[np.ndarray] = None, gamma_q: Optional[np.ndarray] = None,
                  eps: float = 1e-6) -> Projections:
    """Hidden states -> the four per-token inputs of the attention library.

    "MLA from scratch in PyTorch", The MLAAttention module: c_q = norm_q(W_DQ x),
    q = W_UQ c_q reshaped per head; c_kv = W_DKV x (normalised later, at append).
    "Multi-head latent attention", ``_project_mla``: the RoPE query and key are projected
    from x (``self.q_rope(x)``, ``self.k_rope(x)``); the key is one row shared by all heads.
    With no query rank (``w_q`` given) the query projection is full rank: q = W_Q x.
    Weights use the nn.Linear layout (out_features, in_features).
    """
    x = np.asarray(x, dtype=F64)
    B, n, _ = x.shape
    if w_q is not None:
        q = x @ w_q.T
    else:
        c_q = rms_norm(x @ w_dq.T, gamma_q, eps)
        q = c_q @ w_uq.T
    q_nope = q.reshape(B, n, num_heads, head_dim)
    q_rope_raw = (x @ w_qr.T).reshape(B, n, num_heads, rope_dim)
    ckv_raw = x @ w_dkv.T
    krope_raw = x @ w_kr.T
    return Projections(q_nope, q_rope_raw, ckv_raw, krope_raw)


# --------------------------------------------------------------------------------------
# Append: the cached row of one token
# --------------------------------------------------------------------------------------

def cache_rows(ckv_raw: np.ndarray, krope_raw: np.ndarray, gamma: np.ndarray, pos,
               eps: float, base: float, store_bf16: bool) -> np.ndarray:
    """[RMSNorm(c_kv) || RoPE(k_rope, pos)] per token, rounded to the cache's storage type.

    "Multi-head latent attention", Compress keys and values into one latent: the cache holds
    c_t and the rotated k_rope_t, r + d_r numbers per token per layer, concatenated in that
    order (``torch.cat((key, key_rope), -1)``). "MLA from scratch in PyTorch": c_kv is
    normalised by ``norm_kv`` before caching; the cache tensor is bfloat16.
    """
    c = rms_norm(np.asarray(ckv_raw, dtype=F64), np.asarray(gamma, dtype=F64), eps)
    k = rope_rotate(np.asarray(krope_raw, dtype=F64), pos, base)
    row = np.concatenate([c, k], axis=-1)
    return round_bf16(row) if store_bf16 else row


class Placement(NamedTuple):
    block: np.ndarray   # int64 per row
    slot: np.ndarray    # int64 per row
    valid: np.ndarray   # bool per row: block id in range and position inside the table


def paged_placement(seq_idx, pos, table: np.ndarray, block_size: int,
                    num_blocks: int) -> Placement:
    """Where each (sequence, position) lives in a paged pool: table[seq][pos // bs], pos % bs.

    "MLA from scratch in PyTorch", What's not in this implementation: a paged (vLLM-style)
    cache of fixed-size blocks. A row whose table column is past the table or whose block id
    is outside [0, num_blocks) is not placed.
    """
    seq_idx = np.asarray(seq_idx, dtype=np.int64)
    pos = np.asarray(pos, dtype=np.int64)
    col = pos // block_size
    slot = pos % block_size
    in_table = (pos >= 0) & (col < table.shape[1]) & (seq_idx >= 0) & (seq_idx < table.shape[0])
    block = np.full(pos.shape, -1, dtype=np.int64)
    block[in_table] = table[seq_idx[in_table], col[in_table]]
    valid = in_table & (block >= 0) & (block < num_blocks)
    return Placement(block, slot, valid)


def append_ref(pool: np.ndarray, ckv_raw, krope_raw, gamma, seq_idx, pos, table,
               block_size: int, eps: float, base: float, store_bf16: bool) -> Placement:
    """Write each token's cache row into ``pool`` (num_blocks, bs, r + d_r) in place."""
    rows = cache_rows(ckv_raw, krope_raw, gamma, pos, eps, base, store_bf16)
    pl = paged_placement(seq_idx, pos, table, block_size, pool.shape[0])
    pool[pl.block[pl.valid], pl.slot[pl.valid]] = rows[pl.valid]
    return pl


# --------------------------------------------------------------------------------------
# Attention: naive form (the authority) and absorbed form
# --------------------------------------------------------------------------------------

class DecodeOut(NamedTuple):
    o: np.ndarray       # (T, H, d_v)  per-head attention output (before W_O)
    o_lat: np.ndarray   # (T, H, r)    softmax-weighted sum of cached latents
    lse: np.ndarray     # (T, H)       natural-log log-sum-exp of the scaled scores


def _causal_lengths(total: int, T: int) -> np.ndarray:
    """Rows attended by query token t: 0 .. total - T + t (its own row included)."""
    return total - T + 1 + np.arange(T)


def naive_decode(c_kv: np.ndarray, k_rope: np.ndarray, q_nope: np.ndarray, q_rope: np.ndarray,
                 w_uk: np.ndarray, w_uv: np.ndarray, scale: float, dtype=F64) -> DecodeOut:
    """One sequence, the pages' expanded form: rebuild K and V per head from every cached latent.

    "MLA from scratch in PyTorch", The MLAAttention module: k = W_UK(c_kv_full),
    v = W_UV(c_kv_full) reshaped per head, attn = softmax(q k^T * scale) with the causal
    mask for several query tokens, out = attn v. "Multi-head latent attention",
    ``_project_mla``: the key is [k_content || k_rope] with the RoPE key broadcast to every
    head; the query is [q_nope || q_rope]. "Build a DeepSeek Model from Scratch" ch. 3, the
    cache-update figure: the whole updated latent cache is expanded into full per-head keys
    and values before the attention.

    c_kv (L, r) and k_rope (L, d_r) hold every row including the T new ones (already normed
    and rotated); q_nope (T, H, d_h), q_rope (T, H, d_r) rotated; w_uk (H, d_h, r) and
    w_uv (H, d_v, r) are the per-head blocks of the nn.Linear weights. ``dtype`` is the
    arithmetic type (float64 unless a test reproduces a float32 computation).
    """
    c_kv = np.asarray(c_kv, dtype=dtype)
    k_rope = np.asarray(k_rope, dtype=dtype)
    L = c_kv.shape[0]
    T, H, _ = q_nope.shape
    d_v, r = w_uv.shape[1], w_uv.shape[2]
    lengths = _causal_lengths(L, T)
    o = np.empty((T, H, d_v), dtype=dtype)
    o_lat = np.empty((T, H, r), dtype=dtype)
    lse = np.empty((T, H), dtype=dtype)
    keep = np.arange(L)[None, :] < lengths[:, None]                 # (T, L) causal mask
    for h in range(H):
        K = c_kv @ np.asarray(w_uk[h], dtype=dtype).T               # (L, d_h)
        V = c_kv @ np.asarray(w_uv[h], dtype=dtype).T               # (L, d_v)
        key = np.concatenate([K, k_rope], axis=1)                   # (L, d_h + d_r)
        qry = np.concatenate([np.asarray(q_nope[:, h], dtype=dtype),
                              np.asarray(q_rope[:, h], dtype=dtype)], axis=1)  # (T, d_h + d_r)
        s = (qry @ key.T) * dtype(scale)                            # (T, L)
        s = np.where(keep, s, -np.inf)
        p = softmax(s)
        o[:, h] = p @ V
        o_lat[:, h] = p @ c_kv
        lse[:, h] = logsumexp(s)
    return DecodeOut(o, o_lat, lse)


def expanded_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """Causal attention over per-head keys and values already expanded from the latent.

    "MLA from scratch in PyTorch", The MLAAttention module: attn = softmax(q k^T * scale) with
    the causal mask over the T new tokens, out = attn v. Q (T, H, D), K (L, H, D) and
    V (L, H, d_v) hold every head's query, key ([K_nope || k_rope]) and value; the T queries
    are the last T of the L rows. Returns o (T, H, d_v). Computed in float64 on the values
    given, so a caller that rounds Q, K or V first gets the attention of the rounded operands.
    """
    Q = np.asarray(Q, dtype=F64)
    K = np.asarray(K, dtype=F64)
    V = np.asarray(V, dtype=F64)
    T, L = Q.shape[0], K.shape[0]
    s = np.einsum("thd,lhd->htl", Q, K) * scale                     # (H, T, L)
    keep = np.arange(L)[None, :] < _causal_lengths(L, T)[:, None]     # (T, L)
    s = np.where(keep[None], s, -np.inf)
    p = softmax(s)
    return np.einsum("htl,lhd->thd", p, V)


def absorb_query(q_nope: np.ndarray, w_uk: np.ndarray, dtype=F64) -> np.ndarray:
    """q_lat[h] = W_UK[h]^T q_nope[h]: "DeepSeek MLA, Built From the Paper", 3 Matrix
    absorption -- q^T (W_UK c) = (W_UK^T q)^T c, so W_UK folds into the query once.
    q_nope (..., H, d_h), w_uk (H, d_h, r) -> (..., H, r)."""
    q = np.asarray(q_nope, dtype=dtype)
    return np.matmul(q[..., None, :], np.asarray(w_uk, dtype=dtype))[..., 0, :]


def absorbed_decode(c_kv: np.ndarray, k_rope: np.ndarray, q_nope: np.ndarray, q_rope: np.ndarray,
                    w_uk: np.ndarray, w_uv: np.ndarray, scale: float, dtype=F64) -> DecodeOut:
    """Same inputs and outputs as ``naive_decode``, computed in absorbed form.

    Scores are (W_UK^T q_nope) . c_kv + q_rope . k_rope ("Build a DeepSeek Model from
    Scratch" ch. 3: "the scores are the sum of the content-based scores and the
    position-based scores"); the weighted sum stays in latent space and W_UV is applied after
    it ("MLA from scratch in PyTorch", Absorbing projections: attend directly to latents).
    """
    c_kv = np.asarray(c_kv, dtype=dtype)
    k_rope = np.asarray(k_rope, dtype=dtype)
    L = c_kv.shape[0]
    T = q_nope.shape[0]
    q_lat = absorb_query(q_nope, w_uk, dtype)                       # (T, H, r)
    s = (q_lat @ c_kv.T + np.asarray(q_rope, dtype=dtype) @ k_rope.T) * dtype(scale)  # (T, H, L)
    keep = np.arange(L)[None, :] < _causal_lengths(L, T)[:, None]
    s = np.where(keep[:, None, :], s, -np.inf)
    p = softmax(s)
    o_lat = p @ c_kv                                                # (T, H, r)
    o = np.matmul(np.asarray(w_uv, dtype=dtype), o_lat[..., None])[..., 0]
    return DecodeOut(o, o_lat, logsumexp(s))


# --------------------------------------------------------------------------------------
# Stage references
# --------------------------------------------------------------------------------------

def absorb_ref(q_nope: np.ndarray, q_rope_raw: np.ndarray, pos, w_uk: np.ndarray,
               base: float) -> np.ndarray:
    """The packed absorbed query Q[n, h] = [W_UK[h]^T q_nope[n, h] || RoPE(q_rope[n, h], pos[n])].

    q_nope (N, H, d_h), q_rope_raw (N, H, d_r), pos (N,) -> (N, H, r + d_r) float64.
    """
    q_lat = absorb_query(q_nope, w_uk)
    pos = np.asarray(pos)
    q_rope = rope_rotate(np.asarray(q_rope_raw, dtype=F64), pos[:, None], base)
    return np.concatenate([q_lat, q_rope], axis=-1)


def latent_attention(Q: np.ndarray, rows: np.ndarray, kv_rank: int, scale: float,
                     T: int) -> DecodeOut:
    """Attention of packed absorbed queries over cached rows of one sequence.

    Q (T, H, r + d_r), rows (L, r + d_r): s = scale * Q . row, p = softmax (causal over the
    T new tokens), o_lat = p . row[:r], lse = logsumexp(s). Returns o = o_lat (no W_UV).
    """
    rows = np.asarray(rows, dtype=F64)
    L = rows.shape[0]
    s = (np.asarray(Q, dtype=F64) @ rows.T) * scale                   # (T, H, L)
    keep = np.arange(L)[None, :] < _causal_lengths(L, T)[:, None]
    s = np.where(keep[:, None, :], s, -np.inf)
    p = softmax(s)
    o_lat = p @ rows[:, :kv_rank]
    return DecodeOut(o_lat, o_lat, logsumexp(s))


def combine_ref(o_parts: Sequence[np.ndarray], lse_parts: Sequence[np.ndarray]):
    """Merge softmax-normalised partial results over disjoint key ranges.

    Each part i holds o_i = sum_j p_ij v_j / l_i and lse_i = log l_i (scores' log-sum-exp over
    its range). The full result is sum_i exp(lse_i - L) o_i with L = log sum_i exp(lse_i).
    """
    lse = np.stack([np.asarray(x, dtype=F64) for x in lse_parts])          # (n, ...)
    L = logsumexp(lse, axis=0)
    w = np.exp(lse - L)
    o = sum(w[i][..., None] * np.asarray(o_parts[i], dtype=F64) for i in range(len(o_parts)))
    return o, L


def output_ref(o_lat: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """o[n, h] = W_UV[h] o_lat[n, h]: the value up-projection applied after the weighted sum.

    "MLA from scratch in PyTorch", Absorbing projections; "Build a DeepSeek Model from
    Scratch" ch. 3, the figure on the output rearrangement (W_UV applied after the weighted
    sum).
    o_lat (N, H, r), w_uv (H, d_v, r) -> (N, H, d_v).
    """
    o_lat = np.asarray(o_lat, dtype=F64)
    return np.matmul(np.asarray(w_uv, dtype=F64), o_lat[..., None])[..., 0]


# --------------------------------------------------------------------------------------
# End-to-end helpers for one sequence from raw per-token inputs
# --------------------------------------------------------------------------------------

def decode_sequence_from_raw(ckv_raw, krope_raw, q_nope, q_rope_raw, w_uk, w_uv, gamma,
                             scale: float, eps: float, base: float, store_bf16: bool,
                             form: str = "naive") -> DecodeOut:
    """Build a sequence's cache rows 0..L-1 from raw inputs, rotate its T queries at positions
    L-T .. L-1, and run the chosen form ("naive" is the authority, "absorbed" the cross-form)."""
    L = np.asarray(ckv_raw).shape[0]
    T = np.asarray(q_nope).shape[0]
    r = np.asarray(ckv_raw).shape[1]
    rows = cache_rows(ckv_raw, krope_raw, gamma, np.arange(L), eps, base, store_bf16)
    qpos = np.arange(L - T, L)
    q_rope = rope_rotate(np.asarray(q_rope_raw, dtype=F64), qpos[:, None], base)
    fn = naive_decode if form == "naive" else absorbed_decode
    return fn(rows[:, :r], rows[:, r:], np.asarray(q_nope, dtype=F64), q_rope, w_uk, w_uv, scale)


def decode_sequence_bf16_query(ckv_raw, krope_raw, q_nope, q_rope_raw, w_uk, w_uv, gamma,
                               scale: float, eps: float, base: float) -> DecodeOut:
    """Absorbed form with the packed query [q_lat || q_rope] stored in bfloat16.

    On a bf16 model the absorbed query is a bfloat16 tensor like every other activation (the
    module of "MLA from scratch in PyTorch" computes in its parameters' dtype); rounding it
    once, to nearest even, separates that storage error -- which peaky attention amplifies --
    from the error of the attention arithmetic itself. Everything else is float64.
    """
    L = np.asarray(ckv_raw).shape[0]
    T = np.asarray(q_nope).shape[0]
    r = np.asarray(ckv_raw).shape[1]
    rows = cache_rows(ckv_raw, krope_raw, gamma, np.arange(L), eps, base, True)
    Q = round_bf16(absorb_ref(q_nope, q_rope_raw, np.arange(L - T, L), w_uk, base))
    lat = latent_attention(Q, rows, r, scale, T)
    return DecodeOut(output_ref(lat.o_lat, w_uv), lat.o_lat, lat.lse)
