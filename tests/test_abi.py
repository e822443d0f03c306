"""The C ABI library loads, exports every symbol the header declares, and validates arguments
synchronously (no GPU needed: every call here fails validation before any CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")


@pytest.fixture(scope="module")
def mla():
    from mla_latent_kv_44_b200 import build

    build.build()
    import mla_latent_kv_44_b200 as m

    return m


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("mla_absorb_query", "mla_append_latent", "mla_decode", "mla_output"):
        assert n in names


def test_every_declared_symbol_is_exported(mla):
    lib = ctypes.CDLL(mla.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_abi_version_and_status_strings(mla):
    assert mla.abi_version() == 8
    assert mla.status_string(0) == "MLA_OK"
    assert mla.status_string(4) == "MLA_ERR_WORKSPACE"
    assert mla.status_string(99) == "MLA_ERR_UNKNOWN"


def _cfg(mla, **kw):
    base = dict(num_heads=128, head_dim=128, kv_rank=512, rope_dim=64, block_size=64)
    base.update(kw)
    return mla.Config(**base).c()


def test_workspace_size_is_host_arithmetic(mla):
    c = _cfg(mla)
    n1 = mla.lib.mla_decode_workspace_size(ctypes.byref(c), 64, 1)
    n4 = mla.lib.mla_decode_workspace_size(ctypes.byref(c), 64, 4)
    assert n1 > 148 * 128 * 512 * 4           # partial outputs of 2 * 74 slots
    assert n4 > n1 and n1 % 256 == 0
    assert mla.lib.mla_decode_workspace_size(ctypes.byref(c), 0, 1) == 0
    assert mla.lib.mla_decode_workspace_size(None, 64, 1) == 0


@pytest.mark.parametrize("bad", [dict(kv_rank=48), dict(rope_dim=3), dict(num_heads=0),
                                 dict(block_size=0), dict(dtype="f16")])
def test_invalid_config_rejected(mla, bad):
    kw = dict(num_heads=128, head_dim=128, kv_rank=512, rope_dim=64, block_size=64)
    kw.update(bad)
    cfg = mla.Config(**kw)
    c = cfg.c()
    if bad.get("dtype") == "f16":
        c.dtype = 7
    st = mla.lib.mla_absorb_query(ctypes.byref(c), 1, 1, 1, 1, 1, 4, None, None)
    assert st == mla.MLA_ERR_INVALID_ARG


def test_null_pointers_rejected_without_launch(mla):
    c = _cfg(mla)
    assert mla.lib.mla_absorb_query(ctypes.byref(c), None, 1, 1, 1, 1, 4, None, None) == 1
    assert mla.lib.mla_output(ctypes.byref(c), None, 1, 1, 4, None, None) == 1
    assert mla.lib.mla_append_latent(ctypes.byref(c), 1, 1, 1, 1, 1, 1, 2, 2, 1, 4, 8, None,
                                     None) == 1
    ws = mla.lib.mla_decode_workspace_size(ctypes.byref(c), 2, 1)
    assert mla.lib.mla_decode(ctypes.byref(c), None, 256, 256, 2, 4, 256, 2, 1, 256, ws, 256,
                              None, 256, None) == 1


def test_workspace_too_small_or_misaligned(mla):
    c = _cfg(mla)
    ws = mla.lib.mla_decode_workspace_size(ctypes.byref(c), 2, 1)
    args = (256, 256, 256, 2, 4, 256, 2, 1)
    assert mla.lib.mla_decode(ctypes.byref(c), *args, 256, ws - 1, 256, None, 256, None) == 4
    assert mla.lib.mla_decode(ctypes.byref(c), *args, 257, ws, 256, None, 256, None) == 4


def test_empty_work_is_a_no_op(mla):
    c = _cfg(mla)
    assert mla.lib.mla_absorb_query(ctypes.byref(c), None, None, None, None, None, 0, None, None) == 0
    assert mla.lib.mla_output(ctypes.byref(c), None, None, None, 0, None, None) == 0
    assert mla.lib.mla_decode(ctypes.byref(c), None, None, None, 1, 1, None, 0, 1, None, 0, None,
                              None, None, None) == 0


def test_tensor_kernel_request_for_unsupported_shape(mla):
    c = _cfg(mla, num_heads=16, kv_rank=64, rope_dim=32)
    c.decode_kernel = mla.DECODE_TENSOR
    ws = mla.lib.mla_decode_workspace_size(ctypes.byref(c), 2, 1)
    st = mla.lib.mla_decode(ctypes.byref(c), 256, 256, 256, 2, 4, 256, 2, 1, 256, ws, 256, None,
                            256, None)
    assert st == mla.MLA_ERR_UNSUPPORTED


def test_product_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "mla_latent_kv_44_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in re.findall(r"^\s*(?:from|import)\s+(\w+)", text, re.M), f


def _decode_both(mla, c, batch, q_per_seq, **ptrs):
    """Status of mla_decode (with a large enough workspace) and of mla_decode_static_workspace
    for the same arguments; every case here fails or succeeds before any CUDA call."""
    p = dict(q=256, pool=256, table=256, lens=256, out=256, err=256)
    p.update(ptrs)
    ws = mla.lib.mla_decode_workspace_size(ctypes.byref(c), max(batch, 1), max(q_per_seq, 1))
    a = mla.lib.mla_decode(ctypes.byref(c), p["q"], p["pool"], p["table"], 4, 4, p["lens"], batch,
                           q_per_seq, 256, max(ws, 1), p["out"], None, p["err"], None)
    b = mla.lib.mla_decode_static_workspace(ctypes.byref(c), p["q"], p["pool"], p["table"], 4, 4,
                                            p["lens"], batch, q_per_seq, p["out"], None, p["err"],
                                            None)
    return a, b


def test_static_workspace_entry_point_returns_mla_decodes_statuses(mla):
    good = _cfg(mla)
    bad = _cfg(mla, kv_rank=48)
    # an invalid configuration is reported even when there is no work
    assert _decode_both(mla, bad, 0, 1) == (mla.MLA_ERR_INVALID_ARG, mla.MLA_ERR_INVALID_ARG)
    assert _decode_both(mla, good, 0, 1) == (mla.MLA_OK, mla.MLA_OK)
    assert _decode_both(mla, good, -1, 1) == (mla.MLA_ERR_INVALID_ARG, mla.MLA_ERR_INVALID_ARG)
    assert _decode_both(mla, good, 2, 0) == (mla.MLA_ERR_INVALID_ARG, mla.MLA_ERR_INVALID_ARG)
    assert _decode_both(mla, good, 2, 1, q=None) == (mla.MLA_ERR_INVALID_ARG,
                                                      mla.MLA_ERR_INVALID_ARG)
    # more (sequence, token) pairs than the schedule supports: unsupported, not invalid
    assert _decode_both(mla, good, 1 << 22, 8) == (mla.MLA_ERR_UNSUPPORTED, mla.MLA_ERR_UNSUPPORTED)
    # a workspace larger than the library's array is the static entry point's own error
    big = 100000
    assert mla.lib.mla_decode_workspace_size(ctypes.byref(good), big, 1) > mla.STATIC_WORKSPACE_BYTES
    st = mla.lib.mla_decode_static_workspace(ctypes.byref(good), 256, 256, 256, 4, 4, 256, big, 1,
                                             256, None, 256, None)
    assert st == mla.MLA_ERR_WORKSPACE


def test_combine_partials_validates_arguments(mla):
    c = _cfg(mla)
    f = mla.lib.mla_combine_partials
    assert f(ctypes.byref(c), 256, 256, 0, 4, 256, None, None) == mla.MLA_ERR_INVALID_ARG
    assert f(ctypes.byref(c), 256, 256, mla.MAX_COMBINE_PARTS + 1, 4, 256, None,
             None) == mla.MLA_ERR_INVALID_ARG
    assert f(ctypes.byref(c), None, 256, 2, 4, 256, None, None) == mla.MLA_ERR_INVALID_ARG
    assert f(ctypes.byref(c), 256, None, 2, 4, 256, None, None) == mla.MLA_ERR_INVALID_ARG
    assert f(ctypes.byref(c), 256, 256, 2, 4, None, None, None) == mla.MLA_ERR_INVALID_ARG
    assert f(ctypes.byref(c), 264, 256, 2, 4, 256, None, None) == mla.MLA_ERR_INVALID_ARG
    assert f(ctypes.byref(c), 256, 256, 2, 4, 260, None, None) == mla.MLA_ERR_INVALID_ARG
    assert f(ctypes.byref(c), 256, 256, 2, -1, 256, None, None) == mla.MLA_ERR_INVALID_ARG
    bad = _cfg(mla, kv_rank=48)
    assert f(ctypes.byref(bad), 256, 256, 2, 4, 256, None, None) == mla.MLA_ERR_INVALID_ARG
    # no row groups: nothing to do, whatever the pointers
    assert f(ctypes.byref(c), None, None, 2, 0, None, None, None) == mla.MLA_OK
