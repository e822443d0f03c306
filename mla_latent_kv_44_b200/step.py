"""Device state and one decode step of an MLA layer, driven through the C ABI.

A ``DecodeState`` owns the device buffers of one workload: W_UK and W_UV, the paged latent
cache (filled with rows 0 .. S_b-1 of every sequence through ``mla_append_latent``, as earlier
steps would have), the step's new-token inputs and the outputs. ``step()`` enqueues the four
calls of the hot path: absorb the query, append the new rows, decode, project with W_UV.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import numpy as np
import torch

import mla_inputs as mi

from . import (DECODE_AUTO, STAGES_ALL, Config, absorb_query, append_latent, decode,
               decode_step, decode_workspace_size, output)

POOL_SENTINEL = -1  # every bit set: NaN in both bf16 and fp32


def config_for(w: mi.Workload, block_size: int, decode_kernel: int = DECODE_AUTO) -> Config:
    return Config(num_heads=w.num_heads, head_dim=w.head_dim, kv_rank=w.kv_rank,
                  rope_dim=w.rope_dim, block_size=block_size, dtype=w.dtype,
                  head_dim_v=w.head_dim_v, rope_base=w.rope_base, rms_eps=w.rms_eps,
                  softmax_scale=w.softmax_scale, decode_kernel=decode_kernel)


class DecodeState:
    """Buffers for one decode step of workload ``w`` on ``device``.

    Inputs are either drawn here (``mla_inputs.sequence_draw``: projection outputs N(0, 1),
    W_UK/W_UV N(0, 1/r)) or passed in as arrays (``raw``), e.g. projections of hidden states.
    Values are rounded to the workload's storage type once, on the host.
    """

    def __init__(self, w: mi.Workload, seed: int = 0, device: str = "cuda",
                 decode_kernel: int = DECODE_AUTO, raw: Optional[dict] = None,
                 needle: float = 0.0, gamma_perturbed: bool = False, spare_blocks: int = 0,
                 sequences: Optional[Sequence[int]] = None):
        self.w = w
        self.device = torch.device(device)
        self.rows = mi.total_rows(w, seed)
        self.layout = mi.cache_layout(w, seed, spare_blocks)
        self.cfg = config_for(w, self.layout.block_size, decode_kernel)
        tdt = self.cfg.torch_dtype
        dev = self.device
        B, T, H = w.batch, w.new_tokens, w.num_heads
        D = w.row_width

        if raw is None:
            wuk, wuv = mi.up_projection_weights(w, seed)
            gamma = mi.rms_gain(w, seed, gamma_perturbed)
        else:
            wuk, wuv, gamma = raw["w_uk"], raw["w_uv"], raw["gamma"]
        self.w_uk_host = mi.storage_round(w, wuk)
        self.w_uv_host = mi.storage_round(w, wuv)
        self.gamma_host = np.asarray(gamma, dtype=np.float32)
        self.w_uk = torch.from_numpy(self.w_uk_host).to(dev, tdt)
        self.w_uv = torch.from_numpy(self.w_uv_host).to(dev, tdt)
        self.gamma = torch.from_numpy(self.gamma_host).to(dev)

        L = self.layout
        self.block_table = torch.from_numpy(L.table).to(dev)
        self.pool = torch.empty((L.num_blocks, L.block_size, D), dtype=tdt, device=dev)
        self.pool.view(torch.int16 if tdt == torch.bfloat16 else torch.int32).fill_(POOL_SENTINEL)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=dev)

        # new-token inputs of the step (rows S_b .. S_b+T-1), kept on the host for checks
        qn = np.empty((B * T, H, w.head_dim), np.float32)
        qr = np.empty((B * T, H, w.rope_dim), np.float32)
        ckv_new = np.empty((B * T, w.kv_rank), np.float32)
        kr_new = np.empty((B * T, w.rope_dim), np.float32)
        self.needle_rows = {}
        seqs = range(B) if sequences is None else sequences
        self.host_draws = {}
        for b in range(B):
            n = int(self.rows[b])
            if raw is None:
                d = mi.sequence_draw(w, b, n, seed)
                if needle:
                    self.needle_rows[b] = mi.plant_needle(w, d, seed, factor=needle)
                ckv, kr, q1, q2 = d.ckv_raw, d.krope_raw, d.q_nope, d.q_rope_raw
            else:
                ckv, kr = raw["ckv_raw"][b][:n], raw["krope_raw"][b][:n]
                q1, q2 = raw["q_nope"][b], raw["q_rope_raw"][b]
            ckv = mi.storage_round(w, ckv)
            kr = mi.storage_round(w, kr)
            q1 = mi.storage_round(w, q1)
            q2 = mi.storage_round(w, q2)
            if b in seqs:
                self.host_draws[b] = (ckv, kr, q1, q2)
            qn[b * T:(b + 1) * T] = q1
            qr[b * T:(b + 1) * T] = q2
            ckv_new[b * T:(b + 1) * T] = ckv[n - T:]
            kr_new[b * T:(b + 1) * T] = kr[n - T:]
            self._prefill(b, ckv[: n - T], kr[: n - T])
        torch.cuda.synchronize(dev)
        if int(self.dev_err.item()) != 0:
            raise RuntimeError(f"prefill append raised device error bits {int(self.dev_err.item())}")

        self.q_nope = torch.from_numpy(qn).to(dev, tdt)
        self.q_rope = torch.from_numpy(qr).to(dev, tdt)
        self.ckv_new = torch.from_numpy(ckv_new).to(dev, tdt)
        self.krope_new = torch.from_numpy(kr_new).to(dev, tdt)
        seq_new, pos_new = mi.positions_for_append(w, self.rows, only_new=True)
        self.seq_new = torch.from_numpy(seq_new).to(dev)
        self.pos_new = torch.from_numpy(pos_new).to(dev)
        self.seq_lens = torch.from_numpy(self.rows.astype(np.int32)).to(dev)

        self.q = torch.empty((B * T, H, D), dtype=tdt, device=dev)
        ws = decode_workspace_size(self.cfg, B, T)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.out_latent = torch.empty((B * T, H, w.kv_rank), dtype=torch.float32, device=dev)
        self.lse = torch.empty((B * T, H), dtype=torch.float32, device=dev)
        self.o = torch.empty((B * T, H, w.head_dim_v), dtype=tdt, device=dev)

    def _prefill(self, b: int, ckv: np.ndarray, kr: np.ndarray, chunk: int = 1 << 16):
        n = ckv.shape[0]
        tdt = self.cfg.torch_dtype
        for lo in range(0, n, chunk):
            hi = min(n, lo + chunk)
            c = torch.from_numpy(np.ascontiguousarray(ckv[lo:hi])).to(self.device, tdt)
            k = torch.from_numpy(np.ascontiguousarray(kr[lo:hi])).to(self.device, tdt)
            seq = torch.full((hi - lo,), b, dtype=torch.int32, device=self.device)
            pos = torch.arange(lo, hi, dtype=torch.int32, device=self.device)
            append_latent(self.cfg, c, k, self.gamma, seq, pos, self.block_table, self.pool,
                          self.dev_err)

    # ---- the hot path -------------------------------------------------------------------
    def absorb(self, stream=None):
        absorb_query(self.cfg, self.q_nope, self.q_rope, self.pos_new, self.w_uk, self.q, stream,
                     self.dev_err)

    def append(self, stream=None):
        append_latent(self.cfg, self.ckv_new, self.krope_new, self.gamma, self.seq_new,
                      self.pos_new, self.block_table, self.pool, self.dev_err, stream)

    def attend(self, stream=None, stages: int = STAGES_ALL):
        decode(self.cfg, self.q, self.pool, self.block_table, self.seq_lens, self.w.new_tokens,
               self.workspace, self.out_latent, self.lse, self.dev_err, stream, stages)

    def project(self, stream=None):
        output(self.cfg, self.out_latent, self.w_uv, self.o, stream, self.dev_err)

    def step(self, stream=None):
        """The four calls of the hot path, one after another."""
        self.absorb(stream)
        self.append(stream)
        self.attend(stream)
        self.project(stream)

    def fused_launches(self) -> int:
        """Kernel launches of step_fused: 4 where mla_decode_step fuses (bf16, the tensor-core
        attention shape, tensor-core projections), else the four calls' 6."""
        c = self.cfg
        fused = (c.dtype == "bf16" and c.decode_kernel != 1 and c.num_heads == 128 and
                 c.kv_rank == 512 and c.rope_dim == 64 and c.block_size == 64 and
                 c.head_dim % 64 == 0 and c.head_dim <= 256)
        return 4 if fused else 6

    def step_fused(self, stream=None):
        """The same step through mla_decode_step (one call; four launches where it can)."""
        decode_step(self.cfg, self.q_nope, self.q_rope, self.w_uk, self.ckv_new, self.krope_new,
                    self.gamma, self.seq_new, self.pos_new, self.block_table, self.pool,
                    self.seq_lens, self.w.new_tokens, self.q, self.workspace, self.out_latent,
                    self.lse, self.w_uv, self.o, self.dev_err, stream)

    # ---- helpers ------------------------------------------------------------------------
    def sequence_rows(self, b: int) -> np.ndarray:
        """Rows 0 .. rows_b-1 of sequence b read back from the pool (float32)."""
        n = int(self.rows[b])
        bs = self.layout.block_size
        ids = torch.from_numpy(self.layout.table[b, : (n + bs - 1) // bs].astype(np.int64))
        blocks = self.pool[ids.to(self.device)].float().reshape(-1, self.w.row_width)[:n]
        return blocks.cpu().numpy()

    def tokens_of(self, b: int) -> slice:
        T = self.w.new_tokens
        return slice(b * T, (b + 1) * T)


def chunked(seq: Sequence[int], n: int) -> List[List[int]]:
    return [list(seq[i:i + n]) for i in range(0, len(seq), n)]
