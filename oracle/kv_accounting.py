"""Cache-size and decode-cost arithmetic -- TEST INFRASTRUCTURE ONLY (part of the oracle).

Closed forms stated on the pages:

* "DeepSeek MLA, Built From the Paper", 1 The problem MLA solves: per token per layer the
  cache holds 2 * n_heads * d_head values for MHA, 2 * n_kv_heads * d_head for GQA and
  r_kv + d_rope for MLA (no head count in the last).
* "Multi-head latent attention", Compress keys and values into one latent: r numbers per
  token replace 2 * H * d_head; with the decoupled RoPE key the cache holds r + d_r.
* "MLA from scratch in PyTorch", Memory comparison and The up-projection cost at decode time:
  bf16 bytes for an (n_layers, B, max_seq, ...) cache, and the decode FLOPs of the naive form
  (two up-projections of every cached latent plus the attention itself).
"""
from __future__ import annotations


def cache_values_mha(n_heads: int, d_head: int) -> int:
    return 2 * n_heads * d_head


def cache_values_gqa(n_kv_heads: int, d_head: int) -> int:
    return 2 * n_kv_heads * d_head


def cache_values_mla(kv_rank: int, rope_dim: int) -> int:
    return kv_rank + rope_dim


def cache_bytes(values_per_token: int, n_layers: int, batch: int, seq: int,
                bytes_per_value: int = 2) -> int:
    """Bytes of a cache holding ``values_per_token`` per token per layer (bf16 by default)."""
    return values_per_token * n_layers * batch * seq * bytes_per_value


def reduction_fraction(mla_values: int, baseline_values: int) -> float:
    """1 - mla / baseline: the fraction of the baseline cache that MLA removes."""
    return 1.0 - mla_values / baseline_values


def gqa_crossover_rank(n_kv_heads: int, d_head: int, rope_dim: int) -> int:
    """Smallest latent rank r at which MLA's cache (r + d_r) is no longer below GQA's."""
    return cache_values_gqa(n_kv_heads, d_head) - rope_dim


def naive_decode_flops(seq_len: int, n_heads: int, d_head: int, kv_rank: int) -> int:
    """Decode FLOPs of the expanded form: rebuild K and V from every latent, then attend
    (the up-projection cost section of "MLA from scratch in PyTorch", restated)."""
    up_k = 2 * seq_len * kv_rank * n_heads * d_head
    up_v = 2 * seq_len * kv_rank * n_heads * d_head
    return up_k + up_v + 2 * n_heads * d_head * seq_len


def absorbed_decode_work(n_rows: int, n_heads: int, kv_rank: int, rope_dim: int,
                         bytes_per_value: int = 2):
    """Algorithmic work of absorbed decode over ``n_rows`` cached rows for one query token:
    every row is read once (r + d_r values), and each head does a (r + d_r)-wide dot product
    and an r-wide weighted accumulation. Returns (bytes, flops)."""
    width = kv_rank + rope_dim
    nbytes = n_rows * width * bytes_per_value
    flops = n_rows * n_heads * 2 * (width + kv_rank)
    return nbytes, flops
