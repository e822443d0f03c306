"""A model of the prefill expansion kernel's barrier protocol, run under random interleavings.

expand_tc_kernel (mla_latent_kv_44_b200/csrc/prefill_tc.cu) is persistent: a CTA walks work
items (a 128-row weight tile, a chunk of token tiles). Its TMA thread refills the resident
weight tile slab by slab (wfull[s]/wfree[s]: slab s of an item is loaded once the previous
item's last products have read that slab) and streams the tokens' slabs through a ring of six
(xfull/xfree); its MMA warp accumulates each token tile into one of two TMEM accumulators
(afull, committed after the tile's last product; afree, one arrival per epilogue warp once
the four epilogue warps have read it). This model replays those waits, arrivals, copies and
commits with copies landing in any order and commits completing in issue order, and checks
that no interleaving deadlocks, that every wait finds its phase or one past it, that no buffer
is refilled while a product may still read it, and that every product and every epilogue
reads the data it means to.
"""
import random

import pytest

STAGES, SLABS = 6, 8


class _Bar:
    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.done += 1


def _run(items, seed):
    """items: token tiles of each work item this CTA takes, in order."""
    rnd = random.Random(seed)
    wfull = [_Bar(f"wfull{s}") for s in range(SLABS)]
    wfree = [_Bar(f"wfree{s}") for s in range(SLABS)]
    xfull = [_Bar(f"xfull{s}") for s in range(STAGES)]
    xfree = [_Bar(f"xfree{s}") for s in range(STAGES)]
    afull = [_Bar(f"afull{a}") for a in range(2)]
    afree = [_Bar(f"afree{a}", 4) for a in range(2)]
    wbuf, xbuf, acc = [None] * SLABS, [None] * STAGES, [None, None]
    pending = []

    def tma():
        kx = 0
        for li, nt in enumerate(items):
            for tt in range(nt):
                for s in range(SLABS):
                    if tt == 0:
                        if li > 0:
                            yield ("wait", wfree[s], li - 1)
                        assert wbuf[s] in (None, "free"), f"weight slab {s} refilled in use"
                        wbuf[s] = "loading"
                        pending.append(("copy", wfull[s], ("w", s, li)))
                    st = kx % STAGES
                    if kx >= STAGES:
                        yield ("wait", xfree[st], kx // STAGES - 1)
                    assert xbuf[st] in (None, "free"), f"token stage {st} refilled in use"
                    xbuf[st] = "loading"
                    pending.append(("copy", xfull[st], ("x", st, (li, tt, s))))
                    kx += 1

    def mma():
        kx = tcount = 0
        for li, nt in enumerate(items):
            for tt in range(nt):
                a = tcount & 1
                if tcount >= 2:
                    yield ("wait", afree[a], (tcount >> 1) - 1)
                assert acc[a] in (None, "read"), f"accumulator {a} overwritten before read"
                for s in range(SLABS):
                    st = kx % STAGES
                    if tt == 0:
                        yield ("wait", wfull[s], li)
                    yield ("wait", xfull[st], kx // STAGES)
                    assert wbuf[s] == ("ready", li), f"product read weight slab {wbuf[s]}"
                    assert xbuf[st] == ("ready", (li, tt, s)), f"product read {xbuf[st]}"
                    pending.append(("commit", xfree[st], ("xfree", st)))
                    if tt == nt - 1:
                        pending.append(("commit", wfree[s], ("wfree", s)))
                    kx += 1
                acc[a] = ("acc", li, tt)
                pending.append(("commit", afull[a], ("done", a, (li, tt))))
                tcount += 1

    def epilogue(w):
        tcount = 0
        for li, nt in enumerate(items):
            for tt in range(nt):
                a = tcount & 1
                yield ("wait", afull[a], tcount >> 1)
                assert acc[a] == ("done", li, tt), f"epilogue {w} read {acc[a]}"
                afree[a].arrive()
                if afree[a].pending == 0:
                    acc[a] = "read"
                yield ("step", None, None)
                tcount += 1

    actors = [tma(), mma()] + [epilogue(w) for w in range(4)]
    waiting = [None] * len(actors)
    alive = list(range(len(actors)))
    for _ in range(2_000_000):
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
                tag = info[0]
                if tag == "w":
                    wbuf[info[1]] = ("ready", info[2])
                elif tag == "x":
                    xbuf[info[1]] = ("ready", info[2])
                elif tag == "xfree":
                    xbuf[info[1]] = "free"
                elif tag == "wfree":
                    wbuf[info[1]] = "free"
                elif tag == "done":
                    acc[info[1]] = ("done",) + info[2]
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


@pytest.mark.parametrize("items", [[1], [1, 1, 1], [16, 16], [3, 1, 16], [2, 5]])
def test_expand_barrier_protocol(items):
    for seed in range(15):
        _run(items, seed)


def test_model_catches_a_missing_wait():
    """The model is not vacuous: without the epilogue's release of an accumulator, some
    interleaving overwrites it before it is read."""
    import inspect
    src = inspect.getsource(_run).replace(
        "                    yield (\"wait\", afree[a], (tcount >> 1) - 1)\n",
        "                    pass\n")
    ns = {}
    exec(compile(src, "model", "exec"), {**globals()}, ns)
    with pytest.raises(AssertionError, match="overwritten before read"):
        for seed in range(400):
            ns["_run"]([4, 4], seed)
