"""Seeded synthetic inputs for MLA decode, shared by the tests, the CPU oracle and bench.py.

This module only draws random numbers and lays out integer bookkeeping (sequence lengths,
block tables). It contains none of the attention arithmetic: no normalisation, no rotary
embedding, no projection, no softmax. Both the CUDA path and the float64 oracle consume what
it returns, and neither imports the other.

Workload shapes follow the DeepSeek-V2 attention configuration restated in "MLA from scratch
in PyTorch" (section "Hyperparameters": d_model 5120, 128 heads, head dim 128, KV rank 512,
query rank 1536, RoPE dim 64) and its scaled-down variant (512 / 16 / 64 / 64 / 96 / 32).

Random streams: every tensor comes from ``numpy.random.default_rng([seed, stream_id])`` with a
fixed stream id, so any one sequence can be regenerated alone (the oracle recomputes sampled
sequences of the large configurations without drawing the whole batch).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

# Stream ids (fixed; changing one changes every derived fixture).
_S_WQ, _S_WDQ, _S_WUQ, _S_WQR, _S_WDKV, _S_WUK, _S_WUV, _S_WKR, _S_X, _S_GAMMA = range(1, 11)
_S_TABLE = 20
_S_LENS = 21
_S_NEEDLE = 22
_S_SEQ0 = 1000


@dataclasses.dataclass(frozen=True)
class Workload:
    """One MLA decode workload: model shape, batch shape and cache layout."""

    name: str
    d_model: int
    num_heads: int
    head_dim: int          # d_h (nope part of the query/key, and the value head dim)
    kv_rank: int           # r: width of the cached latent c_kv
    rope_dim: int          # d_r: width of the decoupled RoPE key
    q_rank: Optional[int]  # r_q: query latent width (None: full-rank query projection)
    batch: int
    cached: int            # S: rows already in the cache before this step
    new_tokens: int        # T: query tokens appended and attended this step
    dtype: str             # "f32" or "bf16": storage type of activations, weights and cache
    block_size: int        # tokens per cache block; 0 means contiguous (one block per sequence)
    permute_blocks: bool
    ragged_max: int = 0    # >0: S_b drawn uniformly from [1, ragged_max] per sequence
    rope_base: float = 10000.0
    rms_eps: float = 1e-6

    @property
    def head_dim_v(self) -> int:
        return self.head_dim

    @property
    def row_width(self) -> int:
        return self.kv_rank + self.rope_dim

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim + self.rope_dim)


WORKLOADS: Dict[str, Workload] = {
    # d_model=256, H=8, d_h=32, r=64, d_r=16, B=1, S=64, one new token, fp32.
    "tiny_fp32": Workload("tiny_fp32", 256, 8, 32, 64, 16, None, 1, 64, 1, "f32", 0, False),
    # Scaled-down DeepSeek-V2: d_model=512, H=16, d_h=64, r=64, r_q=96, d_r=32, B=8, S=1024.
    "small_fp32": Workload("small_fp32", 512, 16, 64, 64, 32, 96, 8, 1024, 1, "f32", 0, False),
    "small_bf16": Workload("small_bf16", 512, 16, 64, 64, 32, 96, 8, 1024, 1, "bf16", 0, False),
    # DeepSeek-V2 attention shape, B=64, S=8192, paged 64-token blocks, permuted table.
    "dsv2": Workload("dsv2", 5120, 128, 128, 512, 64, 1536, 64, 8192, 1, "bf16", 64, True),
    # Same shape, B=128, S_b ~ U[1, 32768].
    "ragged": Workload("ragged", 5120, 128, 128, 512, 64, 1536, 128, 0, 1, "bf16", 64, True,
                       ragged_max=32768),
    # Same shape, B=32, S=16384, 4 causal query tokens appended this step.
    "mtp": Workload("mtp", 5120, 128, 128, 512, 64, 1536, 32, 16384, 4, "bf16", 64, True),
}


def scaled(w: Workload, **changes) -> Workload:
    """A copy of ``w`` with some fields replaced (used for reduced test sizes)."""
    return dataclasses.replace(w, **changes)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, stream])


def _normal(seed: int, stream: int, shape, std: float = 1.0) -> np.ndarray:
    x = _rng(seed, stream).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def cached_lengths(w: Workload, seed: int = 0) -> np.ndarray:
    """S_b per sequence (rows already cached). Ragged workloads draw U[1, ragged_max]."""
    if w.ragged_max > 0:
        return _rng(seed, _S_LENS).integers(1, w.ragged_max + 1, size=w.batch).astype(np.int64)
    return np.full(w.batch, w.cached, dtype=np.int64)


def total_rows(w: Workload, seed: int = 0) -> np.ndarray:
    """Rows valid in each sequence after this step's append: S_b + T."""
    return cached_lengths(w, seed) + w.new_tokens


@dataclasses.dataclass
class CacheLayout:
    block_size: int
    num_blocks: int
    max_blocks: int
    table: np.ndarray      # (batch, max_blocks) int32; -1 in unused entries


def cache_layout(w: Workload, seed: int = 0, spare_blocks: int = 0) -> CacheLayout:
    """Block size, pool size and block table.

    Paged workloads give sequence b the next ceil(rows_b / bs) entries of a random
    permutation of all block ids; contiguous workloads use one block per sequence
    (block_size = max rows, table[b][0] = b). ``spare_blocks`` adds unused blocks to the
    pool (left at their sentinel value by the tests).
    """
    rows = total_rows(w, seed)
    if w.block_size == 0:
        bs = int(rows.max())
        nblk = np.ones(w.batch, dtype=np.int64)
    else:
        bs = w.block_size
        nblk = (rows + bs - 1) // bs
    total = int(nblk.sum())
    num_blocks = total + spare_blocks
    if w.permute_blocks:
        ids = _rng(seed, _S_TABLE).permutation(num_blocks)[:total]
    else:
        ids = np.arange(total)
    max_blocks = int(nblk.max())
    table = np.full((w.batch, max_blocks), -1, dtype=np.int32)
    off = 0
    for b in range(w.batch):
        table[b, : nblk[b]] = ids[off: off + nblk[b]]
        off += nblk[b]
    return CacheLayout(bs, num_blocks, max_blocks, table)


# ---------------------------------------------------------------------------------------
# Projection-level draws (library inputs drawn directly as N(0, 1)).
# ---------------------------------------------------------------------------------------

def up_projection_weights(w: Workload, seed: int = 0):
    """W_UK and W_UV as (H, d, r) float32, N(0, 1/r): nn.Linear(r, H*d) weights viewed per head."""
    std = 1.0 / math.sqrt(w.kv_rank)
    wuk = _normal(seed, _S_WUK, (w.num_heads, w.head_dim, w.kv_rank), std)
    wuv = _normal(seed, _S_WUV, (w.num_heads, w.head_dim_v, w.kv_rank), std)
    return wuk, wuv


def rms_gain(w: Workload, seed: int = 0, perturbed: bool = False) -> np.ndarray:
    """RMSNorm gain gamma: ones (the module default), or 1 + 0.1 N(0, 1) when ``perturbed``."""
    if not perturbed:
        return np.ones(w.kv_rank, dtype=np.float32)
    return (1.0 + 0.1 * _normal(seed, _S_GAMMA, (w.kv_rank,))).astype(np.float32)


@dataclasses.dataclass
class SequenceDraw:
    ckv_raw: np.ndarray     # (rows_b, r)   un-normalised latent rows (positions 0..rows_b-1)
    krope_raw: np.ndarray   # (rows_b, d_r) un-rotated RoPE key rows
    q_nope: np.ndarray      # (T, H, d_h)
    q_rope_raw: np.ndarray  # (T, H, d_r)  un-rotated


def sequence_draw(w: Workload, b: int, rows_b: int, seed: int = 0) -> SequenceDraw:
    """All per-sequence random inputs of sequence ``b`` (independent of the batch size)."""
    g = _rng(seed, _S_SEQ0 + b)
    f = np.float32
    ckv = g.standard_normal(size=(rows_b, w.kv_rank), dtype=f)
    kr = g.standard_normal(size=(rows_b, w.rope_dim), dtype=f)
    qn = g.standard_normal(size=(w.new_tokens, w.num_heads, w.head_dim), dtype=f)
    qr = g.standard_normal(size=(w.new_tokens, w.num_heads, w.rope_dim), dtype=f)
    return SequenceDraw(ckv, kr, qn, qr)


def plant_needle(w: Workload, draw: SequenceDraw, seed: int = 0, factor: float = 16.0) -> int:
    """Make attention peaky: scale one earlier RoPE-key row by ``factor``.

    Rotation preserves the row's norm, so for every head whose q_rope points the same way
    the score of that row becomes large and it dominates the softmax (about half the heads);
    for the others it is pushed far below the rest. Only a random index and a scaling of
    random data happen here. Returns the row index.
    """
    rows = draw.krope_raw.shape[0]
    j = int(_rng(seed, _S_NEEDLE).integers(0, max(1, rows - w.new_tokens)))
    draw.krope_raw[j] *= np.float32(factor)
    return j


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Input preparation: round float32 draws to bfloat16-representable float32 values.

    Uses torch's float32 -> bfloat16 conversion (round to nearest even), so that the device
    tensors and the oracle's float64 copies hold exactly the same numbers.
    """
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def storage_round(w: Workload, x: np.ndarray) -> np.ndarray:
    """The values the device stores for a workload input: bf16-rounded or plain float32."""
    x = np.asarray(x, dtype=np.float32)
    return round_to_bf16(x) if w.dtype == "bf16" else x


# ---------------------------------------------------------------------------------------
# Full-layer draws (hidden states and all eight projection weights), for the small configs.
# ---------------------------------------------------------------------------------------

@dataclasses.dataclass
class LayerDraw:
    x: np.ndarray                  # (B, S+T, d_model) hidden states, N(0, 1)
    w_q: Optional[np.ndarray]      # (H*d_h, d_model) full-rank query (q_rank None)
    w_dq: Optional[np.ndarray]     # (r_q, d_model)
    w_uq: Optional[np.ndarray]     # (H*d_h, r_q)
    w_qr: np.ndarray               # (H*d_r, d_model)
    w_dkv: np.ndarray              # (r, d_model)
    w_uk: np.ndarray               # (H*d_h, r)
    w_uv: np.ndarray               # (H*d_h, r)
    w_kr: np.ndarray               # (d_r, d_model)
    gamma_q: Optional[np.ndarray]  # (r_q,) ones
    gamma_kv: np.ndarray           # (r,)  ones


def layer_draw(w: Workload, seed: int = 0, x_rows: Optional[int] = None) -> LayerDraw:
    """Hidden states N(0, 1) and nn.Linear-shaped weights N(0, 1/fan_in), float64.

    x is (B, longest sequence, d_model), or (x_rows, d_model) when x_rows is given (the
    tokens of one step, for the front end alone).
    """
    H, dh, r, dr, dm = w.num_heads, w.head_dim, w.kv_rank, w.rope_dim, w.d_model
    x_shape = (w.batch, int(total_rows(w, seed).max()), dm) if x_rows is None else (x_rows, dm)

    def lin(stream, out_f, in_f):
        return _normal(seed, stream, (out_f, in_f), 1.0 / math.sqrt(in_f)).astype(np.float64)

    if w.q_rank is None:
        w_q, w_dq, w_uq, gq = lin(_S_WQ, H * dh, dm), None, None, None
    else:
        w_q = None
        w_dq = lin(_S_WDQ, w.q_rank, dm)
        w_uq = lin(_S_WUQ, H * dh, w.q_rank)
        gq = np.ones(w.q_rank)
    return LayerDraw(
        x=_normal(seed, _S_X, x_shape).astype(np.float64),
        w_q=w_q, w_dq=w_dq, w_uq=w_uq,
        w_qr=lin(_S_WQR, H * dr, dm),
        w_dkv=lin(_S_WDKV, r, dm),
        w_uk=lin(_S_WUK, H * dh, r),
        w_uv=lin(_S_WUV, H * dh, r),
        w_kr=lin(_S_WKR, dr, dm),
        gamma_q=gq,
        gamma_kv=np.ones(r),
    )


def positions_for_append(w: Workload, rows: np.ndarray, only_new: bool):
    """(seq_idx, pos) int32 pairs for the rows an append call writes.

    ``only_new``: the T rows of this step (positions S_b..S_b+T-1); otherwise every row
    0..rows_b-1 of every sequence (used to fill the cache before the step).
    """
    seq, pos = [], []
    for b, n in enumerate(rows):
        lo = n - w.new_tokens if only_new else 0
        seq.append(np.full(n - lo, b, dtype=np.int32))
        pos.append(np.arange(lo, n, dtype=np.int32))
    return np.concatenate(seq), np.concatenate(pos)


def sample_sequences(w: Workload, k: int, seed: int = 0) -> List[int]:
    """A fixed random subset of k sequence indices (for per-sequence oracle checks)."""
    k = min(k, w.batch)
    return sorted(_rng(seed, 30).choice(w.batch, size=k, replace=False).tolist())
