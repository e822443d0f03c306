"""A model of the prefill attention kernel's barrier protocol, run under random interleavings.

prefill_tc_kernel (mla_latent_kv_44_b200/csrc/prefill_tc.cu) hands work between a TMA thread,
an MMA warp and two softmax groups of four warps through mbarriers: the two query tiles
(bar_q); key slabs through a ring of four slots (kfull/kfree, slab s of key tile j in slot
(3j + s) % 4, freed by the last score product that reads it); value tiles double-buffered
(vfull/vfree, freed by the last P . V that reads them); per query tile g the scores (s[g]),
the softmax's P (p[g], one arrival per warp) and the P . V completions (o[g]). This model
replays the same sequence of waits, arrivals, copies and commits as the kernel issues them,
with copies landing in any order and tensor-core commits completing in issue order, and checks
for every interleaving tried that:

* no role waits forever (the protocol cannot deadlock);
* every wait finds its barrier in the phase it waits for or one past it, never two past (a
  parity wait cannot be satisfied by an older or a later phase);
* no copy lands in a slot whose previous contents a product may still read;
* a tile's scores are never written over a P that its P . V has not consumed, and every
  product reads the key, value and P tile it means to.
"""
import random

import pytest

KSLOTS = 4


class _Bar:
    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.done += 1


def _run(nkt, seed):
    rnd = random.Random(seed)
    nk = max(nkt)
    q = _Bar("q")
    kfull = [_Bar(f"kfull{i}") for i in range(KSLOTS)]
    kfree = [_Bar(f"kfree{i}") for i in range(KSLOTS)]
    vfull = [_Bar(f"vfull{i}") for i in range(2)]
    vfree = [_Bar(f"vfree{i}") for i in range(2)]
    s_bar = [_Bar(f"s{g}") for g in range(2)]
    p_bar = [_Bar(f"p{g}", 4) for g in range(2)]
    o_bar = [_Bar(f"o{g}") for g in range(2)]
    kslot, vstage = [None] * KSLOTS, [None] * 2   # what each buffer holds
    scol = [None, None]                            # what query tile g's S columns hold
    pending = []                                   # copies and commits not yet landed

    def tma():  # the kernel's TMA thread
        pending.append(("copy", q, None))
        u = 0

        def load_k(j, sl):
            nonlocal u
            slot = u % KSLOTS
            if u >= KSLOTS:
                yield ("wait", kfree[slot], u // KSLOTS - 1)
            assert kslot[slot] is None, f"key slot {slot} refilled while in use"
            kslot[slot] = "loading"
            pending.append(("copy", kfull[slot], ("k", slot, (j, sl))))
            u += 1

        for j in range(nk):
            yield from load_k(j, 0)
            vs = j & 1
            if j >= 2:
                yield ("wait", vfree[vs], (j >> 1) - 1)
            assert vstage[vs] is None, f"value stage {vs} refilled while in use"
            vstage[vs] = "loading"
            pending.append(("copy", vfull[vs], ("v", vs, j)))
            yield from load_k(j, 1)
            yield from load_k(j, 2)

    def mma():  # the kernel's MMA warp
        def scores(g, j):
            last = g == 1 or nkt[1] <= j
            for sl in range(3):
                u = 3 * j + sl
                slot = u % KSLOTS
                yield ("wait", kfull[slot], u // KSLOTS)
                assert kslot[slot] == ("ready", (j, sl)), f"S_{g}({j}) read {kslot[slot]}"
                if last:
                    pending.append(("commit", kfree[slot], ("kfree", slot)))
            assert scol[g] in (None, "consumed"), f"S_{g}({j}) written over a live P"
            scol[g] = ("S", j)
            pending.append(("commit", s_bar[g], None))

        yield ("wait", q, 0)
        yield from scores(0, 0)
        if nkt[1] > 0:
            yield from scores(1, 0)
        for j in range(nk):
            vs = j & 1
            yield ("wait", vfull[vs], j >> 1)
            for g in range(2):
                if j >= nkt[g]:
                    continue
                yield ("wait", p_bar[g], j)
                assert vstage[vs] == ("ready", j), f"P.V_{g}({j}) read {vstage[vs]}"
                assert scol[g] == ("P", j), f"P.V_{g}({j}) read {scol[g]}"
                pending.append(("commit", o_bar[g], ("pv", g)))
                if g == 1 or nkt[1] <= j:
                    pending.append(("commit", vfree[vs], ("vfree", vs)))
                if j + 1 < nkt[g]:
                    yield ("wait", o_bar[g], j)
                    yield from scores(g, j + 1)

    def softmax(g, w):  # warp w of query tile g's softmax group
        for j in range(nkt[g]):
            yield ("wait", s_bar[g], j)
            if w == 0:
                assert scol[g] == ("S", j), f"softmax {g} tile {j} found {scol[g]}"
                scol[g] = ("P", j)
            p_bar[g].arrive()
            yield ("step", None, None)
        if nkt[g] > 0:
            yield ("wait", o_bar[g], nkt[g] - 1)

    actors = [tma(), mma()] + [softmax(g, w) for g in range(2) for w in range(4) if nkt[g] > 0]
    waiting = [None] * len(actors)
    alive = list(range(len(actors)))
    for _ in range(1_000_000):
        if not alive and not pending:
            return
        choices = [("actor", i) for i in alive] + ([("land", 0)] if pending else [])
        rnd.shuffle(choices)
        moved = False
        for kind, i in choices:
            if kind == "land":
                commits = [k for k, p in enumerate(pending) if p[0] == "commit"]
                k = rnd.randrange(len(pending))
                if pending[k][0] == "commit":
                    k = commits[0]  # tensor-core commits complete in issue order
                op, bar, info = pending.pop(k)
                if info is not None:
                    if info[0] == "k":
                        kslot[info[1]] = ("ready", info[2])
                    elif info[0] == "v":
                        vstage[info[1]] = ("ready", info[2])
                    elif info[0] == "kfree":
                        kslot[info[1]] = None
                    elif info[0] == "vfree":
                        vstage[info[1]] = None
                    elif info[0] == "pv":
                        scol[info[1]] = "consumed"
                bar.arrive()
                moved = True
                break
            if waiting[i] is not None:
                bar, n = waiting[i]
                assert bar.done in (n, n + 1), f"{bar.name}: phase {bar.done} for a wait on {n}"
                if bar.done == n:
                    continue
                waiting[i] = None
            try:
                op, bar, n = next(actors[i])
            except StopIteration:
                alive.remove(i)
                moved = True
                break
            if op == "wait":
                waiting[i] = (bar, n)
            moved = True
            break
        assert moved, "deadlock: " + ", ".join(
            f"{w[0].name} phase {w[0].done} for {w[1]}" for w in waiting if w)
    raise AssertionError("the model did not finish")


@pytest.mark.parametrize("nkt", [(1, 0), (1, 2), (2, 0), (3, 4), (7, 8), (16, 0), (31, 32)])
def test_prefill_barrier_protocol(nkt):
    # (key tiles of query tile A, of query tile B): a pair of 128-query tiles sees 2pr + 1
    # and 2pr + 2 key tiles, or A alone when B starts past the sequence end
    for seed in range(25):
        _run(nkt, seed)


def test_model_catches_a_missing_wait():
    """The model is not vacuous: without the wait for P . V before the next scores, some
    interleaving writes scores over a live P."""
    import inspect
    src = inspect.getsource(_run).replace(
        "                    yield (\"wait\", o_bar[g], j)\n", "")
    ns = {}
    exec(compile(src, "model", "exec"), {**globals()}, ns)
    with pytest.raises(AssertionError, match="written over a live P"):
        for seed in range(200):
            ns["_run"]((3, 4), seed)
