"""Context-parallel decode: each sequence's cache rows split across ranks, merged by lse.

CPU: the split rule against brute force (every row on exactly one rank, whole blocks, the new
rows on the last rank, every slice non-empty), each rank's block table and lengths, and the
whole flow (slice decode, all-gather, merge) on 2 and 3 gloo ranks with the oracle standing in
for the device calls: the merged result must equal the oracle's decode over all rows.
GPU: the ranks emulated one after another on one GPU (each rank's mla_decode over its slices
into its part of the gathered buffer, then mla_combine_partials), checked against the oracle;
and the merge kernel's own edge cases.
"""
import os
import socket

import numpy as np
import pytest
import torch

import mla_inputs as mi
from oracle import mla_ref as ref


@pytest.fixture(scope="module")
def cp():
    from mla_latent_kv_44_b200 import build

    build.build()
    from mla_latent_kv_44_b200 import context_parallel

    return context_parallel


# ------------------------------------------------------------------------------- split rule
def test_slice_cuts_against_brute_force(cp):
    for bs in (4, 16):
        for T in (1, 2, 5):
            for world in (1, 2, 3, 4, 7):
                for S in range(T, 12 * bs):
                    try:
                        cuts = cp.slice_cuts(S, T, world, bs)
                    except ValueError:
                        # only short sequences: with at least `world` blocks, the largest
                        # even cut at most the blocks every token attends, all slices are
                        # non-empty
                        blocks = -(-S // bs)
                        shared = (S - T) // bs
                        assert not (blocks >= world and blocks - (-(-blocks // world)) <= shared)
                        continue
                    assert len(cuts) == world + 1 and cuts[0] == 0 and cuts[-1] == S
                    owner = np.full(S, -1)
                    for k in range(world):
                        assert cuts[k] < cuts[k + 1]                 # non-empty
                        assert cuts[k] % bs == 0                     # whole blocks
                        owner[cuts[k]:cuts[k + 1]] = k
                    assert np.all(owner >= 0)                        # every row, once
                    # rows of ranks below the last are attended by every query token
                    assert world == 1 or cuts[world - 1] <= S - T
                    assert np.all(owner[S - T:] == world - 1)        # new rows on the last rank


def test_rank_plan_tables_and_lengths(cp):
    g = np.random.default_rng([5, 1])
    bs, T, world = 8, 3, 3
    seq_lens = np.array([100, 37, 64, 250], dtype=np.int32)
    B, maxb = len(seq_lens), 40
    table = g.permutation(B * maxb).astype(np.int32).reshape(B, maxb)
    total = np.zeros(B, dtype=np.int64)
    for rank in range(world):
        plan = cp.rank_plan(table, seq_lens, T, world, rank, bs)
        assert plan.row_groups == B * T
        reps = 1 if rank == world - 1 else T
        assert plan.q_per_seq == (T if rank == world - 1 else 1)
        assert plan.table.shape[0] == B * reps and plan.lens.shape == (B * reps,)
        for b in range(B):
            cuts = cp.slice_cuts(int(seq_lens[b]), T, world, bs)
            lo, hi = cuts[rank], cuts[rank + 1]
            nb = -(-(hi - lo) // bs)
            for i in range(b * reps, (b + 1) * reps):
                assert plan.lens[i] == hi - lo
                assert np.array_equal(plan.table[i, :nb], table[b, lo // bs:lo // bs + nb])
            total[b] += hi - lo
    assert np.array_equal(total, seq_lens)


# -------------------------------------------------------------- the flow on gloo CPU ranks
def _oracle_slice_decode(pool_rows_of, r, scale):
    """mla_decode's contract, computed by the oracle: every local sequence i attends its
    plan.lens[i] rows (read through plan.table) with plan.q_per_seq causal tokens."""
    def run(cfg, plan, q, pool, workspace, part_o, part_l, dev_err, stream):
        qps = plan.q_per_seq
        for i in range(len(plan.lens)):
            rows = pool_rows_of(plan.table[i], int(plan.lens[i]))
            res = ref.latent_attention(q[i * qps:(i + 1) * qps].numpy(), rows, r, scale, qps)
            part_o[i * qps:(i + 1) * qps] = torch.from_numpy(res.o_lat)
            part_l[i * qps:(i + 1) * qps] = torch.from_numpy(res.lse)
    return run


def _oracle_combine(cfg, parts_o, parts_l, out, lse, stream):
    o, L = ref.combine_ref(list(parts_o.numpy()), list(parts_l.numpy()))
    out.copy_(torch.from_numpy(o))
    lse.copy_(torch.from_numpy(L))


def _flow_inputs(T):
    g = np.random.default_rng([7, T])
    bs, H, r, dr = 16, 4, 32, 16
    seq_lens = np.array([700, 300, 1000], dtype=np.int32)
    B, maxb = len(seq_lens), 64
    nblocks = B * maxb
    pool = g.standard_normal((nblocks, bs, r + dr))
    table = g.permutation(nblocks).astype(np.int32).reshape(B, maxb)
    q = g.standard_normal((B * T, H, r + dr))
    return bs, H, r, dr, seq_lens, pool, table, q


def _rank_main(rank, world, port, T, out):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from mla_latent_kv_44_b200 import context_parallel as cp

        bs, H, r, dr, seq_lens, pool, table, q = _flow_inputs(T)
        scale = 0.2

        def rows_of(blocks, n):
            return pool[np.asarray(blocks)].reshape(-1, r + dr)[:n]

        plan = cp.rank_plan(table, seq_lens, T, world, rank, bs)
        lat = torch.empty((len(seq_lens) * T, H, r), dtype=torch.float64)
        lse = torch.empty((len(seq_lens) * T, H), dtype=torch.float64)
        cp.context_parallel_decode(None, plan, torch.from_numpy(q), None, None, lat, lse, None,
                                   decode_slice_fn=_oracle_slice_decode(rows_of, r, scale),
                                   combine_fn=_oracle_combine)
        err = 0.0
        for b, S in enumerate(seq_lens):
            whole = ref.latent_attention(q[b * T:(b + 1) * T], rows_of(table[b], int(S)), r,
                                         scale, T)
            err = max(err, float(np.max(np.abs(lat[b * T:(b + 1) * T].numpy() - whole.o_lat))),
                      float(np.max(np.abs(lse[b * T:(b + 1) * T].numpy() - whole.lse))))
        out.put((rank, err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T", [(2, 1), (3, 1), (2, 4), (3, 3)])
def test_context_parallel_flow_on_gloo_ranks(cp, world, T):
    import torch.multiprocessing as mp

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(k, world, port, T, q)) for k in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(results) == list(range(world))
    assert max(results.values()) < 1e-10, results


# ------------------------------------------------------------------------------ GPU tests
@pytest.mark.gpu
@pytest.mark.parametrize("name,kw,world", [
    ("dsv2", dict(batch=4, cached=3000), 2),
    ("dsv2", dict(batch=4, cached=3000), 3),
    ("dsv2", dict(batch=2, cached=9000), 8),
    ("mtp", dict(batch=3, cached=1500), 2),
    ("mtp", dict(batch=3, cached=1500), 4),
])
def test_context_parallel_emulated_on_one_gpu(cp, name, kw, world):
    import mla_latent_kv_44_b200 as mla
    from mla_latent_kv_44_b200.step import DecodeState
    from tests.gpu_util import check_sequence, dev_err

    w = mi.scaled(mi.WORKLOADS[name], **kw)
    st = DecodeState(w)
    st.absorb()
    st.append()
    T, n = w.new_tokens, w.batch * w.new_tokens
    parts_o = torch.empty((world,) + tuple(st.out_latent.shape), device="cuda")
    parts_l = torch.empty((world,) + tuple(st.lse.shape), device="cuda")
    for rank in range(world):
        plan = cp.rank_plan(st.layout.table, st.rows, T, world, rank, st.layout.block_size)
        ws = torch.empty(mla.decode_workspace_size(st.cfg, len(plan.lens), plan.q_per_seq),
                         dtype=torch.uint8, device="cuda")
        cp.decode_slice(st.cfg, plan, st.q, st.pool, ws, parts_o[rank], parts_l[rank],
                        st.dev_err)
    mla.combine_partials(st.cfg, parts_o, parts_l, st.out_latent, st.lse)
    st.project()
    assert dev_err(st) == 0
    assert n == st.out_latent.shape[0]
    for b in range(w.batch):
        check_sequence(st, b, "absorbed")


@pytest.mark.gpu
def test_combine_partials_edge_cases():
    import mla_latent_kv_44_b200 as mla

    cfg = mla.Config(num_heads=6, head_dim=32, kv_rank=96, rope_dim=16, block_size=16)
    g = np.random.default_rng([9, 2])
    P, n, H, r = 5, 7, 6, 96
    o = g.standard_normal((P, n, H, r)).astype(np.float32)
    lse = (3.0 * g.standard_normal((P, n, H))).astype(np.float32)
    lse[1, 2] = -np.inf                      # part 1 has no rows for row group 2 ...
    o[1, 2] = np.nan                         # ... and its output is never read
    lse[:, 4, 3] = -np.inf                   # row group 4, head 3: no rows anywhere
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()  # noqa: E731
    out = torch.empty((n, H, r), device="cuda")
    L = torch.empty((n, H), device="cuda")
    mla.combine_partials(cfg, dev(o), dev(lse), out, L)
    # the oracle's merge of the same parts, the unread NaN block given as zeros (the oracle
    # multiplies it by its zero weight)
    clean = np.where(np.isnan(o), 0.0, o).astype(np.float64)
    with np.errstate(invalid="ignore"):
        exp_o, exp_L = ref.combine_ref(list(clean), list(lse.astype(np.float64)))
    got_o, got_L = out.cpu().numpy(), L.cpu().numpy()
    assert np.all(np.isfinite(got_o))
    assert np.all(got_o[4, 3] == 0) and got_L[4, 3] == -np.inf
    fin = np.isfinite(exp_L)
    assert np.count_nonzero(~fin) == 1
    assert np.max(np.abs(got_L[fin] - exp_L[fin])) < 1e-5
    assert np.max(np.abs(got_o[fin] - exp_o[fin])) < 1e-5 * np.max(np.abs(clean))
    # one part: the merge is the identity, bit for bit
    one = torch.empty((n, H, r), device="cuda")
    L1 = torch.empty((n, H), device="cuda")
    src = o[:1].copy()
    src[np.isnan(src)] = 0
    mla.combine_partials(cfg, dev(src), dev(lse[:1]), one, L1)
    keep = np.isfinite(lse[0])
    assert np.array_equal(one.cpu().numpy()[keep], src[0][keep])
    assert np.array_equal(L1.cpu().numpy()[keep], lse[0][keep])
    # an empty part appended last leaves every bit as it was
    two = torch.empty((n, H, r), device="cuda")
    L2 = torch.empty((n, H), device="cuda")
    o_e = np.concatenate([o, np.full((1, n, H, r), np.nan, np.float32)])
    l_e = np.concatenate([lse, np.full((1, n, H), -np.inf, np.float32)])
    mla.combine_partials(cfg, dev(o_e), dev(l_e), two, L2)
    assert np.array_equal(two.cpu().numpy(), got_o) and np.array_equal(L2.cpu().numpy(), got_L)
