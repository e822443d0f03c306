"""Python binding of libmla (MLA absorbed decode for B200, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA kernels of
``libmla.so``. Tensors are passed as raw device pointers; PyTorch provides device memory and
streams. The library is loaded on the first call (so that the build step can import this
package before the library exists); that call fails loudly when the library has not been
built (``python -m mla_latent_kv_44_b200.build``). There is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla.so")
# The same library built with a test define that leaves out one K-slab load of the attention
# kernel's first work range (tests of the bounded-wait path load it instead of LIB_PATH).
TEST_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla_testhook.so")

MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_CUDA, MLA_ERR_WORKSPACE = range(5)
STATIC_WORKSPACE_BYTES = 40 << 20
MLA_F32, MLA_BF16 = 0, 1
DECODE_AUTO, DECODE_SIMT, DECODE_TENSOR = 0, 1, 2
DEV_OOB_BLOCK, DEV_OOB_POS, DEV_WAIT_TIMEOUT, DEV_BAD_LENGTH = 1, 2, 4, 8
STAGE_PLAN, STAGE_ATTEND, STAGE_COMBINE = 1, 2, 4
STAGES_ALL = STAGE_PLAN | STAGE_ATTEND | STAGE_COMBINE
MAX_COMBINE_PARTS = 256  # MLA_MAX_COMBINE_PARTS

_c_i32, _c_f32, _vp, _sz = ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class MlaConfig(ctypes.Structure):
    _fields_ = [("num_heads", _c_i32), ("head_dim", _c_i32), ("head_dim_v", _c_i32),
                ("kv_rank", _c_i32), ("rope_dim", _c_i32), ("block_size", _c_i32),
                ("rope_base", _c_f32), ("rms_eps", _c_f32), ("softmax_scale", _c_f32),
                ("dtype", _c_i32), ("decode_kernel", _c_i32)]


class MlaFrontConfig(ctypes.Structure):
    _fields_ = [("d_model", _c_i32), ("q_rank", _c_i32), ("q_rms_eps", _c_f32)]


class MlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m mla_latent_kv_44_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(MlaConfig)
    sig = {
        "mla_absorb_query": (_c_i32, [P, _vp, _vp, _vp, _vp, _vp, _c_i32, _vp, _vp]),
        "mla_append_latent": (_c_i32, [P, _vp, _vp, _vp, _vp, _vp, _vp, _c_i32, _c_i32, _vp,
                                       _c_i32, _c_i32, _vp, _vp]),
        "mla_decode_workspace_size": (_sz, [P, _c_i32, _c_i32]),
        "mla_decode": (_c_i32, [P, _vp, _vp, _vp, _c_i32, _c_i32, _vp, _c_i32, _c_i32, _vp, _sz,
                                _vp, _vp, _vp, _vp]),
        "mla_decode_stages": (_c_i32, [P, _c_i32, _vp, _vp, _vp, _c_i32, _c_i32, _vp, _c_i32,
                                       _c_i32, _vp, _sz, _vp, _vp, _vp, _vp]),
        "mla_output": (_c_i32, [P, _vp, _vp, _vp, _c_i32, _vp, _vp]),
        "mla_decode_static_workspace": (_c_i32, [P, _vp, _vp, _vp, _c_i32, _c_i32, _vp, _c_i32,
                                                 _c_i32, _vp, _vp, _vp, _vp]),
        "mla_decode_step": (_c_i32, [P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_i32, _vp,
                                     _c_i32, _vp, _c_i32, _c_i32, _vp, _vp, _sz, _vp, _vp, _vp,
                                     _vp, _vp, _vp]),
        "mla_combine_partials": (_c_i32, [P, _vp, _vp, _c_i32, _c_i32, _vp, _vp, _vp]),
        "mla_append_latent_fp8": (_c_i32, [P, _vp, _vp, _vp, _vp, _vp, _vp, _c_i32, _c_i32, _vp,
                                           _vp, _c_i32, _c_i32, _vp, _vp]),
        "mla_decode_fp8_workspace_size": (_sz, [P, _c_i32, _c_i32, _c_i32]),
        "mla_decode_fp8": (_c_i32, [P, _vp, _vp, _vp, _vp, _c_i32, _c_i32, _vp, _c_i32, _c_i32,
                                    _vp, _sz, _vp, _vp, _vp, _vp]),
        "mla_prefill_workspace_size": (_sz, [P, _c_i32]),
        "mla_prefill": (_c_i32, [P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_i32, _c_i32, _c_i32,
                                 _vp, _vp, _sz, _vp, _vp]),
        "mla_project_workspace_size": (_sz, [P, ctypes.POINTER(MlaFrontConfig), _c_i32]),
        "mla_project": (_c_i32, [P, ctypes.POINTER(MlaFrontConfig), _vp, _vp, _vp, _vp, _vp,
                                 _vp, _vp, _vp, _vp, _vp, _vp, _c_i32, _vp, _sz, _vp, _vp]),
        "mla_status_string": (ctypes.c_char_p, [_c_i32]),
        "mla_abi_version": (_c_i32, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


class _Lib:
    """libmla.so, loaded on first use."""

    _handle = None

    def __getattr__(self, name):
        if _Lib._handle is None:
            _Lib._handle = _load()
        return getattr(_Lib._handle, name)


lib = _Lib()


@dataclass
class Config:
    """Shape and numerics of one MLA layer's decode (mirrors ``mla_config``)."""

    num_heads: int
    head_dim: int
    kv_rank: int
    rope_dim: int
    block_size: int
    dtype: str = "bf16"            # "bf16" or "f32"
    head_dim_v: int = 0            # 0: same as head_dim
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    softmax_scale: float = 0.0     # 0: 1 / sqrt(head_dim + rope_dim)
    decode_kernel: int = DECODE_AUTO

    def c(self) -> MlaConfig:
        scale = self.softmax_scale or 1.0 / math.sqrt(self.head_dim + self.rope_dim)
        return MlaConfig(self.num_heads, self.head_dim, self.head_dim_v or self.head_dim,
                         self.kv_rank, self.rope_dim, self.block_size, self.rope_base,
                         self.rms_eps, scale, MLA_BF16 if self.dtype == "bf16" else MLA_F32,
                         self.decode_kernel)

    @property
    def row_width(self) -> int:
        return self.kv_rank + self.rope_dim

    @property
    def torch_dtype(self):
        import torch
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


def status_string(status: int) -> str:
    return lib.mla_status_string(status).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(st: int, where: str):
    if st != MLA_OK:
        raise MlaError(st, where)


def absorb_query(cfg: Config, q_nope, q_rope, pos, w_uk, q_out, stream=None, dev_err=None):
    """mla_absorb_query: q_out[n, h] = [W_UK[h]^T q_nope[n, h] || RoPE(q_rope[n, h], pos[n])]."""
    c = cfg.c()
    _check(lib.mla_absorb_query(ctypes.byref(c), _ptr(q_nope), _ptr(q_rope), _ptr(pos),
                                _ptr(w_uk), _ptr(q_out), int(q_nope.shape[0]), _ptr(dev_err),
                                _stream(stream)), "mla_absorb_query")


def append_latent(cfg: Config, ckv_raw, krope_raw, gamma, seq_idx, pos, block_table, pool,
                  dev_err, stream=None):
    """mla_append_latent: write [RMSNorm(c_kv) * gamma || RoPE(k_rope)] rows into the pool."""
    c = cfg.c()
    _check(lib.mla_append_latent(ctypes.byref(c), _ptr(ckv_raw), _ptr(krope_raw), _ptr(gamma),
                                 _ptr(seq_idx), _ptr(pos), _ptr(block_table),
                                 int(block_table.shape[0]), int(block_table.shape[1]), _ptr(pool),
                                 int(pool.shape[0]), int(ckv_raw.shape[0]), _ptr(dev_err),
                                 _stream(stream)), "mla_append_latent")


def decode_workspace_size(cfg: Config, batch: int, q_per_seq: int) -> int:
    c = cfg.c()
    return int(lib.mla_decode_workspace_size(ctypes.byref(c), batch, q_per_seq))


def decode(cfg: Config, q, pool, block_table, seq_lens, q_per_seq: int, workspace, out_latent,
           lse, dev_err, stream=None, stages: int = STAGES_ALL):
    """mla_decode (or a subset of its stages): split-KV absorbed attention over the pool."""
    c = cfg.c()
    _check(lib.mla_decode_stages(ctypes.byref(c), stages, _ptr(q), _ptr(pool), _ptr(block_table),
                                 int(block_table.shape[1]), int(pool.shape[0]), _ptr(seq_lens),
                                 int(seq_lens.shape[0]), q_per_seq, _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _ptr(out_latent),
                                 _ptr(lse), _ptr(dev_err), _stream(stream)), "mla_decode")


def decode_static_workspace(cfg: Config, q, pool, block_table, seq_lens, q_per_seq: int,
                            out_latent, lse, dev_err, stream=None):
    """mla_decode_static_workspace: mla_decode with the library's own fixed device workspace,
    for callers that cannot allocate device memory (see include/mla.h)."""
    c = cfg.c()
    _check(lib.mla_decode_static_workspace(ctypes.byref(c), _ptr(q), _ptr(pool),
                                           _ptr(block_table), int(block_table.shape[1]),
                                           int(pool.shape[0]), _ptr(seq_lens),
                                           int(seq_lens.shape[0]), q_per_seq, _ptr(out_latent),
                                           _ptr(lse), _ptr(dev_err), _stream(stream)),
           "mla_decode_static_workspace")


def decode_step(cfg: Config, q_nope, q_rope, w_uk, ckv_raw, krope_raw, gamma, seq_idx, pos,
                block_table, pool, seq_lens, q_per_seq: int, q_work, workspace, out_latent, lse,
                w_uv, o, dev_err, stream=None):
    """mla_decode_step: absorb, append, decode and output of one step in one call (see
    include/mla.h); batch = seq_lens.shape[0]."""
    c = cfg.c()
    _check(lib.mla_decode_step(ctypes.byref(c), _ptr(q_nope), _ptr(q_rope), _ptr(w_uk),
                               _ptr(ckv_raw), _ptr(krope_raw), _ptr(gamma), _ptr(seq_idx), _ptr(pos),
                               _ptr(block_table), int(block_table.shape[1]), _ptr(pool),
                               int(pool.shape[0]), _ptr(seq_lens), int(seq_lens.shape[0]),
                               q_per_seq, _ptr(q_work), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _ptr(out_latent),
                               _ptr(lse), _ptr(w_uv), _ptr(o), _ptr(dev_err), _stream(stream)),
           "mla_decode_step")


def output(cfg: Config, out_latent, w_uv, o, stream=None, dev_err=None):
    """mla_output: o[n, h] = W_UV[h] out_latent[n, h]."""
    c = cfg.c()
    _check(lib.mla_output(ctypes.byref(c), _ptr(out_latent), _ptr(w_uv), _ptr(o),
                          int(out_latent.shape[0]), _ptr(dev_err), _stream(stream)), "mla_output")


def combine_partials(cfg: Config, part_latent, part_lse, out_latent, lse=None, stream=None):
    """mla_combine_partials: merge part_latent (parts, n, H, r) / part_lse (parts, n, H), each
    part a decode over a disjoint set of the rows, into out_latent (n, H, r) and lse (n, H)."""
    c = cfg.c()
    _check(lib.mla_combine_partials(ctypes.byref(c), _ptr(part_latent), _ptr(part_lse),
                                    int(part_latent.shape[0]), int(part_latent.shape[1]),
                                    _ptr(out_latent), _ptr(lse), _stream(stream)),
           "mla_combine_partials")


def front_config(d_model: int, q_rank: int = 0, q_rms_eps: float = 1e-6) -> MlaFrontConfig:
    """mla_front_config: hidden size, query rank (0: full-rank query), RMSNorm eps of c_q."""
    return MlaFrontConfig(d_model, q_rank, q_rms_eps)


def project_workspace_size(cfg: Config, front: MlaFrontConfig, n_tokens: int) -> int:
    return int(lib.mla_project_workspace_size(ctypes.byref(cfg.c()), ctypes.byref(front),
                                              n_tokens))


def project(cfg: Config, front: MlaFrontConfig, x, w_dq, gamma_q, w_uq, w_qr, w_dkv, w_kr,
            q_nope, q_rope, ckv_raw, krope_raw, workspace, dev_err=None, stream=None):
    """mla_project: hidden states x (n, d_model) -> q_nope, q_rope, ckv_raw, krope_raw."""
    c = cfg.c()
    _check(lib.mla_project(ctypes.byref(c), ctypes.byref(front), _ptr(x), _ptr(w_dq),
                           _ptr(gamma_q), _ptr(w_uq), _ptr(w_qr), _ptr(w_dkv), _ptr(w_kr),
                           _ptr(q_nope), _ptr(q_rope), _ptr(ckv_raw), _ptr(krope_raw),
                           int(x.shape[0]), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _ptr(dev_err),
                           _stream(stream)), "mla_project")


def append_latent_fp8(cfg: Config, ckv_raw, krope_raw, gamma, seq_idx, pos, block_table, pool,
                      row_scale, dev_err, stream=None):
    """mla_append_latent_fp8: new rows as e4m3 codes (uint8 pool) with per-row scales."""
    c = cfg.c()
    _check(lib.mla_append_latent_fp8(ctypes.byref(c), _ptr(ckv_raw), _ptr(krope_raw), _ptr(gamma),
                                     _ptr(seq_idx), _ptr(pos), _ptr(block_table),
                                     int(block_table.shape[0]), int(block_table.shape[1]),
                                     _ptr(pool), _ptr(row_scale), int(pool.shape[0]),
                                     int(ckv_raw.shape[0]), _ptr(dev_err), _stream(stream)),
           "mla_append_latent_fp8")


def decode_fp8_workspace_size(cfg: Config, batch: int, q_per_seq: int, max_blocks: int) -> int:
    return int(lib.mla_decode_fp8_workspace_size(ctypes.byref(cfg.c()), batch, q_per_seq,
                                                 max_blocks))


def decode_fp8(cfg: Config, q, pool, row_scale, block_table, seq_lens, q_per_seq: int, workspace,
               out_latent, lse, dev_err, stream=None):
    """mla_decode_fp8: mla_decode over an fp8 pool (codes times the rows' scales)."""
    c = cfg.c()
    _check(lib.mla_decode_fp8(ctypes.byref(c), _ptr(q), _ptr(pool), _ptr(row_scale),
                              _ptr(block_table), int(block_table.shape[1]), int(pool.shape[0]),
                              _ptr(seq_lens), int(seq_lens.shape[0]), q_per_seq, _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _ptr(out_latent),
                              _ptr(lse), _ptr(dev_err), _stream(stream)), "mla_decode_fp8")


def prefill_workspace_size(cfg: Config, n_tokens: int) -> int:
    return int(lib.mla_prefill_workspace_size(ctypes.byref(cfg.c()), n_tokens))


def prefill(cfg: Config, q_nope, q_rope, pos, rows, w_uk, w_uv, cu_seqlens, max_seqlen: int, o,
            workspace, dev_err=None, stream=None):
    """mla_prefill: causal attention of packed prompts (cu_seqlens: batch + 1 offsets)."""
    c = cfg.c()
    _check(lib.mla_prefill(ctypes.byref(c), _ptr(q_nope), _ptr(q_rope), _ptr(pos), _ptr(rows),
                           _ptr(w_uk), _ptr(w_uv), _ptr(cu_seqlens), int(cu_seqlens.shape[0]) - 1,
                           int(max_seqlen), int(q_nope.shape[0]), _ptr(o), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _ptr(dev_err),
                           _stream(stream)), "mla_prefill")


def abi_version() -> int:
    return int(lib.mla_abi_version())
