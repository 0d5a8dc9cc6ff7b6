"""A model of the dQ-from-dS kernel's synchronisation (s2_bwd_dq_ds_kernel in
csrc/s2_bwd_ds.cu), run on the CPU like the forward's and the dK/dV kernel's
(test_fwd_protocol.py, test_dkdv_protocol.py): the producer (a ring of ST
stages, each one stored dS block and the K tile it multiplies), the UMMA
issuer (dQ = dS.K into one of two TMEM accumulators, alternating per item, the
tensor pipe running its UMMAs and commits in order), the four epilogue warps
(each reads its 32 TMEM lanes of the accumulator, scales, converts and stages
its rows in shared memory, releases the accumulator and starts a bulk store
of its staged rows) and the copies in flight (loads landing and stores
reading their staged rows in any order).  Items are query tiles of one rolled
group, walked as the equal-work pairs of the schedule (tile t, then tile
T-1-t), item i taking i+1 dS blocks; a launch may take any contiguous range
of the pairs (the split-dS backward's ranges).  Checks: no deadlock, no
phase overrun, every UMMA reads the stage it means, no accumulator is
restarted before its last read-out, no epilogue reads an accumulator before
its UMMAs ran, and no staged row is overwritten while a store still reads it."""
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


def items_for(T, pairs):
    """dS block counts of the items (query tiles) a CTA walks over `pairs` of one group."""
    out = []
    for pj in pairs:
        out.append(pj + 1)
        if T - 1 - pj != pj:
            out.append(T - pj)
    return out


def run(items, ST, seed):
    rnd = random.Random(seed)
    bars = {("acc_full", a): Bar(1) for a in (0, 1)}
    bars.update({("acc_empty", a): Bar(4) for a in (0, 1)})
    for s in range(ST):
        bars[("full", s)], bars[("empty", s)] = Bar(1), Bar(1)
    err = []
    blocks = [(n, j) for n, cnt in enumerate(items) for j in range(cnt)]
    stage = [None] * ST           # the block a stage holds ("in flight" while loading)
    stage_reads = [0] * ST        # UMMAs still to read it
    acc = [None, None]            # per accumulator: (item, UMMAs accumulated)
    acc_read = set()              # (item, warp): read out of TMEM
    staged = [None] * 4           # per epilogue warp: the item whose rows its staging holds
    stores = [[] for _ in range(4)]  # per warp: items whose bulk store has not read its staging yet
    pipe = []
    copies = []

    def producer():
        for g, (n, j) in enumerate(blocks):
            s, f = g % ST, g // ST
            if f > 0:
                yield ("wait", ("empty", s), f - 1)
            if stage_reads[s]:
                err.append(f"stage {s} reloaded with {stage_reads[s]} reads pending")
            stage[s], stage_reads[s] = ("in flight",), 1

            def land(s=s, g=g):
                stage[s] = g
                bars[("full", s)].arrive()
            copies.append(land)

    def issuer():
        g = 0
        for n, cnt in enumerate(items):
            ab = n & 1
            if n >= 2:
                yield ("wait", ("acc_empty", ab), (n >> 1) - 1)
            for j in range(cnt):
                yield ("wait", ("full", g % ST), g // ST)
                pipe.append(("mma", g))
                pipe.append(("commit", ("empty", g % ST)))
                if j == cnt - 1:
                    pipe.append(("commit", ("acc_full", ab)))
                g += 1

    def read_out(w, n, cnt, ab):  # TMEM -> registers -> staging rows
        if acc[ab] != (n, cnt):
            err.append(f"warp {w} reads accumulator {ab} = {acc[ab]} for item {n} of {cnt} blocks")
        acc_read.add((n, w))
        if stores[w]:
            err.append(f"warp {w} stages item {n} while the store of {stores[w][0]} still reads it")
        staged[w] = n

    def epilogue(w):
        for n, cnt in enumerate(items):
            ab = n & 1
            yield ("wait", ("acc_full", ab), n >> 1)
            # the previous store has finished reading the staging rows
            yield ("until", lambda w=w: not stores[w])
            yield ("yield",)  # the TMEM loads in flight
            read_out(w, n, cnt, ab)
            yield ("arrive", ("acc_empty", ab), 1)
            stores[w].append(n)

            def store(w=w, n=n):
                if staged[w] != n:
                    err.append(f"store of item {n} (warp {w}) reads staging holding {staged[w]}")
                stores[w].remove(n)
            copies.append(store)

    def execute():
        op = pipe.pop(0)
        if op[0] == "commit":
            bars[op[1]].arrive()
            return
        g = op[1]
        n, j = blocks[g]
        s = g % ST
        if stage[s] != g:
            err.append(f"UMMA for block {g} reads stage {s} = {stage[s]}")
        stage_reads[s] -= 1
        ab = n & 1
        if j == 0:
            prev = acc[ab]
            if prev is not None and any((prev[0], w) not in acc_read for w in range(4)):
                err.append(f"item {n} restarts accumulator {ab} before item {prev[0]} was read out")
            acc[ab] = (n, 1)
        else:
            if acc[ab] != (n, j):
                err.append(f"UMMA {j} of item {n} accumulates onto {acc[ab]}")
            acc[ab] = (n, j + 1)

    actors = {"producer": producer(), "issuer": issuer()}
    actors.update({f"epilogue {w}": epilogue(w) for w in range(4)})
    pending = {name: None for name in actors}
    finished = set()

    def ready(a):
        op = pending[a]
        if op is None:
            return True
        if op[0] == "until":
            return op[1]()
        return bars[op[1]].done >= op[2] + 1

    while not err:
        runnable = [a for a in actors if a not in finished and ready(a)]
        choices = runnable + (["pipe"] if pipe else []) + (["copy"] if copies else [])
        if not choices:
            if len(finished) == len(actors):
                return []
            return ["deadlock: " + ", ".join(f"{a} waits {pending[a][:2]}" for a in actors if a not in finished)]
        c = rnd.choice(choices)
        if c == "pipe":
            execute()
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
            if op[0] == "arrive":  # an arrival, then any other actor may run first
                bars[op[1]].arrive(op[2])
                pending[c] = None
                break
            if op[0] == "yield":  # let the others run before this actor goes on
                break
            if op[0] == "until":
                if op[1]():
                    continue
                pending[c] = op
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
    for T in range(1, 11):
        npairs = (T + 1) // 2
        for ST in (2, 3, 4):  # 3 stages at head dim 128, 4 at 64
            out.append((items_for(T, range(npairs)), ST))              # a CTA's pairs of one group
            out.append((items_for(T, [0]) * 3, ST))                     # pair (0, T-1) of three groups
            out.append((items_for(T, range(npairs))[1:], ST))           # a range starting inside a pair
            out.append((items_for(T, [npairs - 1]) * 3, ST))            # the middle pair (one item when T is odd)
    return out


@pytest.mark.parametrize("idx", range(len(cases())))
def test_dq_ds_protocol_runs_clean(idx):
    items, ST = cases()[idx]
    for seed in range(10):
        problems = run(list(items), ST, seed)
        assert not problems, (problems, items, ST)


PLANTED = {
    # an accumulator released before the warp has read it out of TMEM
    "accumulator released early": (
        "            yield (\"yield\",)  # the TMEM loads in flight\n            read_out(w, n, cnt, ab)\n"
        "            yield (\"arrive\", (\"acc_empty\", ab), 1)\n",
        "            yield (\"arrive\", (\"acc_empty\", ab), 1)\n            yield (\"yield\",)\n"
        "            read_out(w, n, cnt, ab)\n"),
    # the issuer restarting an accumulator without waiting for its read-out
    "accumulator not waited": (
        "            if n >= 2:\n                yield (\"wait\", (\"acc_empty\", ab), (n >> 1) - 1)\n",
        ""),
    # a warp restaging rows without waiting for its previous store to read them
    "staging reused early": (
        "            yield (\"until\", lambda w=w: not stores[w])\n",
        ""),
    # a stage reloaded without waiting for the UMMA that reads it
    "stage reused early": (
        "            if f > 0:\n                yield (\"wait\", (\"empty\", s), f - 1)",
        "            if f > 1:\n                yield (\"wait\", (\"empty\", s), f - 2)"),
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
    for items, ST in cases()[:40]:
        caught += any(ns["run"](list(items), ST, seed) for seed in range(6))
    assert caught > 0
