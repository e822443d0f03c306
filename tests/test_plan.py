"""The decode planner's integer output, bit for bit.

mla_decode's first stage cuts every (sequence, query token) row group into 64-row chunks, lays
all chunks end to end and cuts that list into R = min(74, chunks) equal work ranges (range q
starts at chunk floor(q * C / R)). A row group crossed by range starts becomes several
segments with consecutive partial-result slots. This test runs the planner stage alone,
reads the whole schedule back from the workspace and compares it with the same rule written
out here on the host, for batch shapes that exercise one-row groups, exactly one range per
group, hundreds of short groups, the ragged and multi-token DeepSeek-V2 workloads, and more
than 1024 row groups (the planner's multi-pass path).
"""
import numpy as np
import pytest
import torch

import mla_inputs as mi

RANGES = 74
CHUNK = 64


@pytest.fixture(scope="module")
def mla():
    import mla_latent_kv_44_b200 as m

    return m


def _align256(x):
    return (x + 255) // 256 * 256


def workspace_offsets(H, r, bt):
    """Byte offsets of the schedule's arrays in the decode workspace (each region 256-byte
    aligned, in this order: header, range starts, segments, per-row-group arrays; the partial
    results of split row groups, whose size depends on H and r, come after them)."""
    off, out = 0, {}
    for name, nbytes in (("header", 64 * 4), ("range_begin", (RANGES + 1) * 4),
                         ("segments", (RANGES + bt) * 16), ("bt_slot0", bt * 4),
                         ("bt_nseg", bt * 4), ("bt_len", bt * 4), ("bt_chunk0", bt * 4)):
        out[name] = off
        off = _align256(off + nbytes)
    return out


def expected_plan(seq_lens, T, cap):
    """The schedule the split rule defines, computed with plain integer arithmetic."""
    lens = []
    for sl in seq_lens:
        for t in range(T):
            lens.append(sl - T + 1 + t if T <= sl <= cap else 0)
    nch = [(L + CHUNK - 1) // CHUNK for L in lens]
    chunk0 = [0] * len(nch)
    for i in range(1, len(nch)):
        chunk0[i] = chunk0[i - 1] + nch[i - 1]
    C = sum(nch)
    R = min(RANGES, C)
    starts = [q * C // R for q in range(R)]
    start_of = {s: q for q, s in enumerate(starts)}
    segments, bt_slot0, bt_nseg = [], [], []
    range_begin = [None] * (R + 1)
    slot = 0
    for bt, n in enumerate(nch):
        if n == 0:
            bt_slot0.append(-1)
            bt_nseg.append(0)
            continue
        x, e = chunk0[bt], chunk0[bt] + n
        cuts = [x] + [s for s in starts if x < s < e] + [e]
        nseg = len(cuts) - 1
        for k in range(nseg):
            if cuts[k] in start_of:
                range_begin[start_of[cuts[k]]] = len(segments)
            segments.append((bt, cuts[k], cuts[k + 1], slot + k if nseg >= 2 else -1))
        bt_slot0.append(slot if nseg >= 2 else -1)
        bt_nseg.append(nseg)
        if nseg >= 2:
            slot += nseg
    range_begin[R] = len(segments)
    assert all(v is not None for v in range_begin)
    return dict(header=(len(segments), R, C), range_begin=range_begin, segments=segments,
                bt_slot0=bt_slot0, bt_nseg=bt_nseg, bt_len=lens, bt_chunk0=chunk0,
                slots=slot)


def run_plan(mla, seq_lens, T, cap=None, H=16, r=64, dr=32):
    """Run the planner alone (the schedule does not depend on the head count or widths)."""
    dev = "cuda"
    B = len(seq_lens)
    cap = max(seq_lens) if cap is None else cap
    max_blocks = max(1, (cap + CHUNK - 1) // CHUNK)
    cfg = mla.Config(num_heads=H, head_dim=128, kv_rank=r, rope_dim=dr, block_size=CHUNK,
                     dtype="bf16")
    ws = torch.zeros(mla.decode_workspace_size(cfg, B, T), dtype=torch.uint8, device=dev)
    ws.fill_(0xA5)  # the planner must write every field compared below
    q = torch.zeros((B * T, H, r + dr), dtype=torch.bfloat16, device=dev)
    pool = torch.zeros((1, CHUNK, r + dr), dtype=torch.bfloat16, device=dev)
    table = torch.zeros((B, max_blocks), dtype=torch.int32, device=dev)
    lens = torch.tensor(seq_lens, dtype=torch.int32, device=dev)
    out = torch.zeros((B * T, H, r), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    mla.decode(cfg, q, pool, table, lens, T, ws, out, None, err, stages=mla.STAGE_PLAN)
    torch.cuda.synchronize()
    return ws.cpu().numpy(), int(err.item()), max_blocks * CHUNK


def check(mla, seq_lens, T, cap=None):
    raw, err, cap = run_plan(mla, seq_lens, T, cap)
    exp = expected_plan(seq_lens, T, cap)
    bt = len(seq_lens) * T
    off = workspace_offsets(16, 64, bt)
    i32 = lambda name, n: raw[off[name]:off[name] + 4 * n].view(np.int32)  # noqa: E731
    nseg, R, C = exp["header"]
    assert tuple(i32("header", 3)) == exp["header"]
    assert list(i32("range_begin", R + 1)) == exp["range_begin"]
    segs = i32("segments", 4 * nseg).reshape(nseg, 4)
    assert [tuple(s) for s in segs] == exp["segments"]
    assert list(i32("bt_slot0", bt)) == exp["bt_slot0"]
    assert list(i32("bt_nseg", bt)) == exp["bt_nseg"]
    assert list(i32("bt_len", bt)) == exp["bt_len"]
    assert list(i32("bt_chunk0", bt)) == exp["bt_chunk0"]
    # coverage invariant: the segments tile every row group's chunks once, in order, and the
    # ranges cut the chunk list into pieces of equal size (floor(q * C / R))
    covered = [c for (_, lo, hi, _) in exp["segments"] for c in range(lo, hi)]
    assert covered == list(range(C))
    bad = any(not (T <= s <= cap) for s in seq_lens)
    assert err == (mla.DEV_BAD_LENGTH if bad else 0)
    return exp


@pytest.mark.gpu
def test_plan_one_long_sequence(mla):
    exp = check(mla, [8193], 1)
    assert exp["header"] == (74, 74, 129) and exp["slots"] == 74


@pytest.mark.gpu
def test_plan_74_sequences(mla):
    g = np.random.default_rng(11)
    check(mla, [int(x) for x in g.integers(1, 9000, 74)], 1)


@pytest.mark.gpu
def test_plan_300_short_sequences(mla):
    g = np.random.default_rng(12)
    check(mla, [int(x) for x in g.integers(1, 500, 300)], 1)


@pytest.mark.gpu
def test_plan_dsv2_workloads(mla):
    for name in ("dsv2", "ragged", "mtp"):
        w = mi.WORKLOADS[name]
        rows = [int(x) for x in mi.total_rows(w, 0)]
        check(mla, rows, w.new_tokens)


@pytest.mark.gpu
@pytest.mark.parametrize("B,T", [(1100, 1), (300, 4), (2500, 1)])
def test_plan_more_than_1024_row_groups(mla, B, T):
    g = np.random.default_rng(13 + B)
    check(mla, [int(x) for x in g.integers(T, 3000, B)], T)


@pytest.mark.gpu
def test_plan_with_invalid_lengths(mla):
    g = np.random.default_rng(14)
    lens = [int(x) for x in g.integers(1, 2000, 40)]
    lens[3] = 0        # shorter than the query tokens
    lens[17] = 5000    # beyond the 2048 rows the block table holds
    check(mla, lens, 1, cap=2048)
