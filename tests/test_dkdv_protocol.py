"""A model of the dK/dV kernel's synchronisation (s2_bwd_dkdv_kernel in
csrc/s2_bwd.cu), run on the CPU like the forward's (test_fwd_protocol.py): the
producer (one K/V buffer per item, a ring of ST query stages), the two UMMA
issuers (A: S^T and dV; B: dP^T and dK; each in order, the tensor pipe running
the two streams in any interleaving), the elementwise warps with the item
epilogue, and the copies in flight landing in any order.  Items are kv tiles
of one rolled group, walked as the equal-work pairs of the schedule (tile t,
then tile T-1-t), each with rep x 2 (T - t) 64-row query sub-tiles; a launch
may take any contiguous range of the pairs (the split-dS backward's ranges).
Checks: no deadlock, no phase overrun, every UMMA reads the K/V, query stage
and score buffer it means, and nothing is overwritten while a reader still
needs it."""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.rem, self.done = count, count, 0

    def arrive(self, n=1):
        for _ in range(n):
            self.rem -= 1
            if self.rem == 0:
                self.done += 1
                self.rem = self.count


def items_for(T, rep, pairs):
    """Sub-tile counts of the items (kv tiles) a CTA walks over `pairs` of one group."""
    out = []
    for pj in pairs:
        out.append(rep * 2 * (T - pj))
        if T - 1 - pj != pj:
            out.append(rep * 2 * (T - (T - 1 - pj)))
    return out


def run(items, ST, seed):
    rnd = random.Random(seed)
    bars = {("kv",): Bar(1), ("kv_empty",): Bar(2), ("acc_full",): Bar(2), ("acc_free",): Bar(8)}
    for s in range(ST):
        bars[("full", s)], bars[("empty", s)] = Bar(1), Bar(2)
    for b in (0, 1):
        bars[("s", b)], bars[("dp", b)], bars[("pds", b)] = Bar(1), Bar(1), Bar(8)
    err = []
    # sub-tiles in walk order: (item, index inside the item)
    subs = [(n, it) for n, cnt in enumerate(items) for it in range(cnt)]
    kv = [None]       # the item whose K/V the buffer holds ("in flight" while loading)
    kv_reads = [0]    # S^T / dP^T UMMAs still to read it
    stage = [None] * ST
    stage_reads = [0] * ST  # S^T, dP^T, dV, dK UMMAs and the elementwise row statistics
    tbuf = {"S": [None, None], "dP": [None, None]}  # TMEM score buffers: ("raw"|"p", g)
    grads_done = set()
    acc_read = set()
    pipe = {0: [], 1: []}
    tma = []

    def producer():
        gi = 0
        for n, cnt in enumerate(items):
            if n >= 1:
                yield ("wait", ("kv_empty",), n - 1)
            if kv_reads[0]:
                err.append(f"K/V of item {n} loaded over {kv_reads[0]} pending reads")
            kv[0], kv_reads[0] = ("in flight",), 2 * cnt

            def land_kv(n=n):
                kv[0] = n
                bars[("kv",)].arrive()
            tma.append(land_kv)
            for it in range(cnt):
                s, f = gi % ST, gi // ST
                if f > 0:
                    yield ("wait", ("empty", s), f - 1)
                if stage_reads[s]:
                    err.append(f"stage {s} reloaded with {stage_reads[s]} reads pending")
                stage[s], stage_reads[s] = ("in flight",), 5

                def land_stage(s=s, g=gi):
                    stage[s] = g
                    bars[("full", s)].arrive()
                tma.append(land_stage)
                gi += 1

    def issuer(x):  # x = 0: A (S^T, dV), 1: B (dP^T, dK)
        buf = "S" if x == 0 else "dP"

        def wait_inputs(g):
            n, it = subs[g]
            if it == 0:
                yield ("wait", ("kv",), n)
            yield ("wait", ("full", g % ST), g // ST)

        def issue_sp(g):
            n, it = subs[g]
            pipe[x].append(("SP", x, g))
            pipe[x].append(("commit", (buf.lower() if x else "s", g & 1)))
            if it == items[n] - 1:
                pipe[x].append(("commit", ("kv_empty",)))

        if not subs:
            return
        yield from wait_inputs(0)
        issue_sp(0)
        for g in range(len(subs)):
            n, it = subs[g]
            nxt = g + 1 if g + 1 < len(subs) else None
            nxt_new = nxt is not None and subs[nxt][1] == 0
            if nxt is not None and not nxt_new:
                yield from wait_inputs(nxt)
                issue_sp(nxt)
            yield ("wait", ("pds", g & 1), g >> 1)
            if it == 0 and n > 0:
                yield ("wait", ("acc_free",), n - 1)
            pipe[x].append(("GRAD", x, g))
            pipe[x].append(("commit", ("empty", g % ST)))
            if it == items[n] - 1:
                pipe[x].append(("commit", ("acc_full",)))
            if nxt_new:
                yield from wait_inputs(nxt)
                issue_sp(nxt)

    def elementwise():
        for g, (n, it) in enumerate(subs):
            yield ("wait", ("full", g % ST), g // ST)
            yield ("wait", ("s", g & 1), g >> 1)
            yield ("wait", ("dp", g & 1), g >> 1)
            if stage[g % ST] != g:
                err.append(f"elementwise reads stage {g % ST} = {stage[g % ST]} for sub-tile {g}")
            stage_reads[g % ST] -= 1
            for b in ("S", "dP"):
                if tbuf[b][g & 1] != ("raw", g):
                    err.append(f"elementwise reads {b} buffer {g & 1} = {tbuf[b][g & 1]} for sub-tile {g}")
                tbuf[b][g & 1] = ("p", g)
            yield ("arrive", ("pds", g & 1), 8)
            if it == items[n] - 1:
                yield ("wait", ("acc_full",), n)
                if any((x, gg) not in grads_done for x in (0, 1) for gg, (nn, _) in enumerate(subs) if nn == n):
                    err.append(f"epilogue of item {n} before its gradient UMMAs")
                acc_read.add(n)
                yield ("arrive", ("acc_free",), 8)

    def execute(x):
        op = pipe[x].pop(0)
        if op[0] == "commit":
            bars[op[1]].arrive()
            return
        g = op[2]
        n, it = subs[g]
        s = g % ST
        if stage[s] != g:
            err.append(f"{op[0]}{x}({g}) reads stage {s} = {stage[s]}")
        stage_reads[s] -= 1
        b = "S" if x == 0 else "dP"
        if op[0] == "SP":
            if kv[0] != n:
                err.append(f"SP{x}({g}) reads the K/V of {kv[0]}, not item {n}")
            kv_reads[0] -= 1
            prev = tbuf[b][g & 1]
            if prev is not None and (prev[0] != "p" or (x, prev[1]) not in grads_done):
                err.append(f"SP{x}({g}) overwrites {b} buffer holding {prev}")
            tbuf[b][g & 1] = ("raw", g)
        else:
            if tbuf[b][g & 1] != ("p", g):
                err.append(f"GRAD{x}({g}) reads {b} buffer = {tbuf[b][g & 1]}")
            if it == 0 and n > 0 and (n - 1) not in acc_read:
                err.append(f"GRAD{x}({g}) restarts the accumulator before item {n - 1} was read out")
            grads_done.add((x, g))

    actors = {"producer": producer(), "issuer A": issuer(0), "issuer B": issuer(1), "elementwise": elementwise()}
    pending = {name: None for name in actors}
    finished = set()
    while not err:
        runnable = [a for a in actors if a not in finished and
                    (pending[a] is None or bars[pending[a][1]].done >= pending[a][2] + 1)]
        choices = runnable + [("pipe", x) for x in (0, 1) if pipe[x]] + (["tma"] if tma else [])
        if not choices:
            if len(finished) == len(actors):
                return []
            return ["deadlock: " + ", ".join(f"{a} waits {pending[a]}" for a in actors if a not in finished)]
        c = rnd.choice(choices)
        if isinstance(c, tuple):
            execute(c[1])
            continue
        if c == "tma":
            tma.pop(rnd.randrange(len(tma)))()
            continue
        while True:
            try:
                op = next(actors[c])
            except StopIteration:
                finished.add(c)
                pending[c] = None
                break
            if op[0] == "arrive":  # an arrival, then any other actor may run first
                bars[op[1]].arrive(op[2])
                pending[c] = None
                break
            done = bars[op[1]].done
            if done < op[2]:  # the barrier is a phase behind: a parity wait would pass at once
                return [f"{c}: parity wait ahead on {op[1]} (waits phase {op[2]}, {done} complete)"]
            if done >= op[2] + 2:
                return [f"{c}: phase overrun on {op[1]}"]
            if done >= op[2] + 1:
                continue
            pending[c] = op
            break
    return err[:3]


def cases():
    out = []
    for T in range(1, 9):
        npairs = (T + 1) // 2
        for rep in (1, 2, 3):
            out.append((items_for(T, rep, range(npairs)), 3))            # a CTA's pairs of one group
            out.append((items_for(T, rep, [0]) * 3, 3))                   # pair (0, T-1) of three groups
            out.append((items_for(T, rep, range(npairs))[1:], 2))         # a range starting inside a pair
            out.append((items_for(T, rep, [npairs - 1]) * 2, 4))          # the middle pair (one item when T is odd)
    return out


@pytest.mark.parametrize("idx", range(len(cases())))
def test_dkdv_protocol_runs_clean(idx):
    items, ST = cases()[idx]
    for seed in range(10):
        problems = run(list(items), ST, seed)
        assert not problems, (problems, items, ST)


PLANTED = {
    # the K/V buffer released after an item's first S^T / dP^T instead of its last
    "K/V released early": ("            if it == items[n] - 1:\n                pipe[x].append((\"commit\", (\"kv_empty\",)))",
                           "            if it == 0:\n                pipe[x].append((\"commit\", (\"kv_empty\",)))"),
    # a query stage reloaded without waiting for both issuers' gradient UMMAs
    "stage reused early": ("                if f > 0:\n                    yield (\"wait\", (\"empty\", s), f - 1)",
                           "                if f > 1:\n                    yield (\"wait\", (\"empty\", s), f - 2)"),
    # the elementwise warps not waiting for dP^T
    "dP not waited": ("            yield (\"wait\", (\"dp\", g & 1), g >> 1)\n", ""),
}


@pytest.mark.parametrize("name", sorted(PLANTED))
def test_model_catches_planted_mistakes(name):
    """Each planted protocol mistake makes the model report a problem on some
    interleaving: the checks are live."""
    import inspect
    import textwrap
    src = textwrap.dedent(inspect.getsource(run))
    old, new = PLANTED[name]
    assert old in src
    ns = dict(globals())
    exec(src.replace(old, new), ns)
    caught = 0
    for items, ST in cases()[:24]:
        caught += any(ns["run"](list(items), ST, seed) for seed in range(6))
    assert caught > 0
