"""Context-parallel decode: every sequence's cache rows split across the GPUs of a group.

A sequence whose cache outgrows one GPU ("MLA from scratch in PyTorch", Memory comparison:
the cache grows linearly with the context) is cut into contiguous, block-aligned slices of
rows, one per rank. Each rank runs mla_decode over its own slice with its own block table,
which gives every (sequence, query token) row group a softmax-normalised partial result and
its log-sum-exp; the ranks all-gather those (one collective) and merge them with
mla_combine_partials, the same log-sum-exp merge mla_decode applies to its own work ranges.

The split keeps the causal rule of several new query tokens local to one rank: query token t
of a sequence of S rows (T of them new) attends rows 0 .. S - T + t, so every row below
S - T + 1 is attended by every token. Ranks 0 .. world - 2 hold only such rows, whole cache
blocks of them, and decode each (sequence, token) pair as a sequence of its own over the whole
slice; the last rank holds the tail, the T new rows included, and decodes it with the causal
rule as mla_decode states it. Every slice must hold at least one row: sequences too short for
that are not split (a ValueError says so).

This module is host logic around the library calls: block-table slicing, the collective
(torch.distributed, NCCL between GPUs) and the order of the calls.
"""
from dataclasses import dataclass
from typing import Callable, List, Optional

import numpy as np
import torch

from . import Config, combine_partials, decode


def slice_cuts(seq_len: int, new_tokens: int, world: int, block_size: int) -> List[int]:
    """Row boundaries c_0 = 0 < c_1 < ... < c_world = seq_len of one sequence's slices.

    Rank k holds rows [c_k, c_k+1). The cuts are whole cache blocks, as even as the block count
    allows (c_k = block_size * floor(k * blocks / world)), and none lies above the last row
    that every query token attends (S - T), so the T new rows stay on the last rank.
    """
    if world < 1 or block_size < 1 or not (1 <= new_tokens <= seq_len):
        raise ValueError(f"cannot split {seq_len} rows with {new_tokens} new over {world} ranks")
    blocks = -(-seq_len // block_size)
    shared = (seq_len - new_tokens) // block_size  # whole blocks every token attends
    cuts = [block_size * min(k * blocks // world, shared) for k in range(world)] + [seq_len]
    if any(b <= a for a, b in zip(cuts[:-1], cuts[1:])):
        raise ValueError(f"a sequence of {seq_len} rows ({new_tokens} new) is too short to split "
                         f"over {world} ranks of {block_size}-row blocks")
    return cuts


@dataclass
class RankPlan:
    """One rank's mla_decode arguments for its slices (host arrays)."""
    table: np.ndarray     # (sequences, max_blocks) int32: the slice's block ids
    lens: np.ndarray      # (sequences,) int32: rows of each slice
    q_per_seq: int        # query tokens per decoded sequence
    row_groups: int       # batch * new_tokens, in the order b * new_tokens + t


def rank_plan(block_table: np.ndarray, seq_lens: np.ndarray, new_tokens: int, world: int,
              rank: int, block_size: int) -> RankPlan:
    """The decode arguments of `rank` for a batch whose block table and lengths are global.

    block_table (B, max_blocks) int32 maps a sequence's blocks to pool blocks; seq_lens (B,)
    counts the rows after this step's append. Ranks below world - 1 decode B * T sequences
    (sequence b repeated for each of its T query tokens, every one over the whole slice); the
    last rank decodes B sequences with T causal query tokens.
    """
    block_table = np.asarray(block_table)
    seq_lens = np.asarray(seq_lens)
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a group of {world}")
    B, T = len(seq_lens), int(new_tokens)
    bounds = [slice_cuts(int(s), T, world, block_size)[rank:rank + 2] for s in seq_lens]
    first = [lo // block_size for lo, _ in bounds]
    count = [-(-(hi - lo) // block_size) for lo, hi in bounds]
    width = max(count)
    table = np.zeros((B, width), dtype=np.int32)
    for b in range(B):
        table[b, :count[b]] = block_table[b, first[b]:first[b] + count[b]]
    lens = np.array([hi - lo for lo, hi in bounds], dtype=np.int32)
    if rank == world - 1 or T == 1:
        return RankPlan(table, lens, T, B * T)
    return RankPlan(np.repeat(table, T, axis=0), np.repeat(lens, T), 1, B * T)


def decode_slice(cfg: Config, plan: RankPlan, q, pool, workspace, out_latent, lse, dev_err,
                 stream=None, device=None):
    """mla_decode of this rank's slices: out_latent (B*T, H, r) and lse (B*T, H) receive the
    partial results in row-group order. `workspace` must hold
    mla_decode_workspace_size(cfg, len(plan.lens), plan.q_per_seq) bytes."""
    device = device if device is not None else q.device
    table = torch.from_numpy(plan.table).to(device)
    lens = torch.from_numpy(plan.lens).to(device)
    decode(cfg, q, pool, table, lens, plan.q_per_seq, workspace, out_latent, lse, dev_err, stream)


def gather_partials(out_latent: torch.Tensor, lse: torch.Tensor, group=None):
    """All ranks' partial results, part-major: (world, n, H, r) and (world, n, H)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    out = []
    for x in (out_latent.contiguous(), lse.contiguous()):
        # gathered as the concatenation along the first dimension (the form every backend
        # takes), which is the part-major layout
        parts = x.new_empty((world * x.shape[0],) + tuple(x.shape[1:]))
        dist.all_gather_into_tensor(parts, x, group=group)
        out.append(parts.view((world,) + tuple(x.shape)))
    return out[0], out[1]


def context_parallel_decode(cfg: Config, plan: RankPlan, q, pool, workspace, out_latent, lse,
                            dev_err, group=None, stream=None,
                            decode_slice_fn: Optional[Callable] = None,
                            combine_fn: Optional[Callable] = None):
    """This rank's slice decode, the all-gather of every rank's partials, and their merge into
    out_latent (B*T, H, r) and lse (B*T, H) (the same on every rank).

    decode_slice_fn(cfg, plan, q, pool, workspace, part_o, part_lse, dev_err, stream) and
    combine_fn(cfg, parts_o, parts_lse, out_latent, lse, stream) default to the library calls.
    """
    import contextlib

    decode_slice_fn = decode_slice_fn or decode_slice
    combine_fn = combine_fn or combine_partials
    # the collective is ordered after the work of torch's current stream: make `stream` current
    on_stream = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with on_stream:
        part_o = torch.empty_like(out_latent)
        part_l = torch.empty_like(lse)
        decode_slice_fn(cfg, plan, q, pool, workspace, part_o, part_l, dev_err, stream)
        parts_o, parts_l = gather_partials(part_o, part_l, group)
        combine_fn(cfg, parts_o, parts_l, out_latent, lse, stream)
