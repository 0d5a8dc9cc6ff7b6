"""A model of the 128-query dK/dV kernel's synchronisation (s2_bwd_dkdv128_kernel
in csrc/s2_bwd_kv128.cu), run on the CPU like the other kernels' models: the
producer (one K/V buffer per item, a ring of ST stages of 128-row Q / dO
tiles with their row statistics), the two UMMA issuers (A: S^T and dV, B:
dP^T and dK; per query tile the scores, then the gradient UMMAs of each
64-query half once the elementwise warps have released it), the elementwise
warps (P^T and dS^T over the single S^T / dP^T buffers, half by half, and the
item's epilogue) and the copies in flight landing in any order; after every
wait and every arrival any other actor may go first.  Items are kv tiles of
one rolled group walked as the equal-work pairs of the schedule, item t
taking rep x (T - t) query tiles.  Checks: no deadlock, no parity wait
overrun or wait ahead of its barrier, every UMMA reads the K/V, stage and
score half it means, and nothing is overwritten while a reader still needs
it."""
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
    """Query-tile counts of the items (kv tiles) a CTA walks over `pairs` of one group."""
    out = []
    for pj in pairs:
        out.append(rep * (T - pj))
        if T - 1 - pj != pj:
            out.append(rep * (T - (T - 1 - pj)))
    return out


def run(items, ST, seed):
    rnd = random.Random(seed)
    bars = {("kv",): Bar(1), ("kv_empty",): Bar(2), ("s",): Bar(1), ("dp",): Bar(1), ("acc_full",): Bar(2),
            ("acc_free",): Bar(8)}
    for s in range(ST):
        bars[("full", s)], bars[("empty", s)] = Bar(1), Bar(2)
    for h in (0, 1):
        bars[("p", h)] = Bar(8)
    err = []
    subs = [(n, it) for n, cnt in enumerate(items) for it in range(cnt)]
    kv, kv_reads = [None], [0]
    stage, stage_reads = [None] * ST, [0] * ST
    tbuf = {0: [None, None], 1: [None, None]}  # per issuer's score buffer, per half: ("raw"|"p", g)
    grads_done, acc_read = set(), set()
    pipe = {0: [], 1: []}
    copies = []

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
            copies.append(land_kv)
            for it in range(cnt):
                s, f = gi % ST, gi // ST
                if f > 0:
                    yield ("wait", ("empty", s), f - 1)
                if stage_reads[s]:
                    err.append(f"stage {s} reloaded with {stage_reads[s]} reads pending")
                stage[s], stage_reads[s] = ("in flight",), 7  # two scores, four gradient halves, the row statistics

                def land(s=s, g=gi):
                    stage[s] = g
                    bars[("full", s)].arrive()
                copies.append(land)
                gi += 1

    def issuer(x):  # 0: A (S^T, dV), 1: B (dP^T, dK)
        for g, (n, it) in enumerate(subs):
            if it == 0:
                yield ("wait", ("kv",), n)
            yield ("wait", ("full", g % ST), g // ST)
            pipe[x].append(("SP", x, g))
            pipe[x].append(("commit", ("s",) if x == 0 else ("dp",)))
            if it == items[n] - 1:
                pipe[x].append(("commit", ("kv_empty",)))
            for h in (0, 1):
                yield ("wait", ("p", h), g)
                if h == 0 and it == 0 and n > 0:
                    yield ("wait", ("acc_free",), n - 1)
                pipe[x].append(("GRAD", x, g, h))
                if h == 1:
                    pipe[x].append(("commit", ("empty", g % ST)))
                    if it == items[n] - 1:
                        pipe[x].append(("commit", ("acc_full",)))

    def elementwise():
        for g, (n, it) in enumerate(subs):
            yield ("wait", ("full", g % ST), g // ST)
            yield ("wait", ("s",), g)
            yield ("wait", ("dp",), g)
            if stage[g % ST] != g:
                err.append(f"elementwise reads stage {g % ST} = {stage[g % ST]} for tile {g}")
            stage_reads[g % ST] -= 1
            for h in (0, 1):
                for x in (0, 1):
                    if tbuf[x][h] != ("raw", g):
                        err.append(f"elementwise reads half {h} of buffer {x} = {tbuf[x][h]} for tile {g}")
                    tbuf[x][h] = ("p", g)
                yield ("arrive", ("p", h), 8)
            if it == items[n] - 1:
                yield ("wait", ("acc_full",), n)
                if any((x, gg, h) not in grads_done for x in (0, 1) for h in (0, 1)
                       for gg, (nn, _) in enumerate(subs) if nn == n):
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
        if op[0] == "SP":
            if kv[0] != n:
                err.append(f"SP{x}({g}) reads the K/V of {kv[0]}, not item {n}")
            kv_reads[0] -= 1
            for h in (0, 1):
                prev = tbuf[x][h]
                if prev is not None and (prev[0] != "p" or (x, prev[1], h) not in grads_done):
                    err.append(f"SP{x}({g}) overwrites half {h} holding {prev}")
                tbuf[x][h] = ("raw", g)
        else:
            h = op[3]
            if tbuf[x][h] != ("p", g):
                err.append(f"GRAD{x}({g}, half {h}) reads {tbuf[x][h]}")
            if it == 0 and h == 0 and n > 0 and (n - 1) not in acc_read:
                err.append(f"GRAD{x}({g}) restarts the accumulator before item {n - 1} was read out")
            grads_done.add((x, g, h))

    actors = {"producer": producer(), "issuer A": issuer(0), "issuer B": issuer(1), "elementwise": elementwise()}
    pending = {name: None for name in actors}
    finished = set()
    while not err:
        runnable = [a for a in actors if a not in finished and
                    (pending[a] is None or bars[pending[a][1]].done >= pending[a][2] + 1)]
        choices = runnable + [("pipe", x) for x in (0, 1) if pipe[x]] + (["copy"] if copies else [])
        if not choices:
            if len(finished) == len(actors):
                return []
            return ["deadlock: " + ", ".join(f"{a} waits {pending[a]}" for a in actors if a not in finished)]
        c = rnd.choice(choices)
        if isinstance(c, tuple):
            execute(c[1])
            continue
        if c == "copy":
            copies.pop(rnd.randrange(len(copies)))()
            continue
        pending[c] = None
        while True:
            try:
                op = next(actors[c])
            except StopIteration:
                finished.add(c)
                break
            if op[0] == "arrive":  # then any other actor may run first
                bars[op[1]].arrive(op[2])
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
    for T in range(1, 8):
        npairs = (T + 1) // 2
        for rep in (1, 2):
            for ST in (2, 3):
                out.append((items_for(T, rep, range(npairs)), ST))     # a CTA's pairs of one group
                out.append((items_for(T, rep, range(npairs))[1:], ST))  # a range starting inside a pair
            out.append((items_for(T, rep, [0]) * 3, 2))                 # pair (0, T-1) of three groups
    return out


@pytest.mark.parametrize("idx", range(len(cases())))
def test_kv128_protocol_runs_clean(idx):
    items, ST = cases()[idx]
    for seed in range(10):
        problems = run(list(items), ST, seed)
        assert not problems, (problems, items, ST)


PLANTED = {
    # the K/V buffer released after an item's first scores instead of its last
    "K/V released early": ("            if it == items[n] - 1:\n                pipe[x].append((\"commit\", (\"kv_empty\",)))",
                           "            if it == 0:\n                pipe[x].append((\"commit\", (\"kv_empty\",)))"),
    # a stage released after the first half's gradient UMMAs instead of the second
    "stage released early": ("                if h == 1:\n                    pipe[x].append((\"commit\", (\"empty\", g % ST)))",
                             "                if h == 0:\n                    pipe[x].append((\"commit\", (\"empty\", g % ST)))"),
    # the elementwise warps not waiting for dP^T
    "dP not waited": ("            yield (\"wait\", (\"dp\",), g)\n", ""),
    # a half handed to the gradient UMMAs before P^T / dS^T are written into it
    "half handed over early": ("                    tbuf[x][h] = (\"p\", g)\n                yield (\"arrive\", (\"p\", h), 8)\n",
                               "                yield (\"arrive\", (\"p\", h), 8)\n                for x in (0, 1):\n"
                               "                    tbuf[x][h] = (\"p\", g)\n"),
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
    for items, ST in cases()[:30]:
        caught += any(ns["run"](list(items), ST, seed) for seed in range(6))
    assert caught > 0
