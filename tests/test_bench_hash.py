"""The bench keys its measured DRAM traffic to the attention kernel's code.

Edits to comments or layout keep the key (the kernel is the same); any change to the code
drops it, so the bench reports no traffic until the kernel is captured again.
"""
import os
import shutil

import bench


def _tree(tmp_path):
    dst = tmp_path / "mla_latent_kv_44_b200" / "csrc"
    dst.mkdir(parents=True)
    src = os.path.join(bench.ROOT, "mla_latent_kv_44_b200", "csrc")
    for f in bench.ATTEND_SOURCES:
        shutil.copy(os.path.join(src, f), dst / f)
    return dst


def _hash_at(root, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(root))
    return bench.attend_source_hash()


def test_comments_and_layout_do_not_change_the_key(tmp_path, monkeypatch):
    dst = _tree(tmp_path)
    before = _hash_at(tmp_path, monkeypatch)
    f = dst / "decode_tc.cu"
    text = f.read_text()
    f.write_text("// a new leading comment\n/* and a block\n   comment */\n" +
                 text.replace("\n\n", "\n\n\n", 3))
    assert _hash_at(tmp_path, monkeypatch) == before


def test_a_code_change_changes_the_key(tmp_path, monkeypatch):
    dst = _tree(tmp_path)
    before = _hash_at(tmp_path, monkeypatch)
    f = dst / "decode_tc.cu"
    text = f.read_text()
    assert "constexpr int kKStages = 4;" in text
    f.write_text(text.replace("constexpr int kKStages = 4;", "constexpr int kKStages = 3;"))
    assert _hash_at(tmp_path, monkeypatch) != before


def test_traffic_applies_to_its_workload_and_kernel_only():
    import argparse

    (workload, key), traffic = next(iter(bench.ATTEND_TRAFFIC.items()))
    assert isinstance(traffic, int) and traffic > 0
    here = bench.attend_source_hash()
    args = argparse.Namespace(decode_kernel="auto", workload=workload)
    assert bench.attend_traffic(args) == (traffic if key == here else None)
    other = [w for w in ("dsv2", "ragged", "mtp") if w != workload][0]
    assert bench.attend_traffic(argparse.Namespace(decode_kernel="auto", workload=other)) is None
    assert bench.attend_traffic(argparse.Namespace(decode_kernel="simt", workload=workload)) is None
