"""A model of the split path's dQ kernel's synchronisation (s2_bwd_dq_kernel in
csrc/s2_bwd.cu: dQ with S and dP recomputed), run on the CPU like the other
kernels' models: the producer (one shared-memory Q/dO buffer per item, a ring
of ST K/V stages), three UMMA issuers (S = Q K^T and dP = dO V^T with Q / dO
read from TMEM, dQ += dS K), each in order and interleaved in any way by the
tensor pipe, the dS warps (they copy each item's Q / dO from shared memory
into TMEM, turn S and dP into dS over the dP buffer, and read dQ out of TMEM
at the end of the item) and the copies in flight landing in any order; after
every wait and every arrival any other actor may go first.  Items are query
tiles of one rolled group walked as the equal-work pairs of the schedule,
item t taking 2 (t + 1) 64-row kv sub-tiles (causal; a chunk over a whole
key segment takes the same count for every tile).  Checks: no deadlock, no
parity wait overrun, every UMMA reads the Q / dO, stage and buffer it means,
and nothing is overwritten while a reader still needs it."""
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


def items_for(T, pairs, causal=True, nkv=None):
    """Sub-tile counts of the items (query tiles) a CTA walks over `pairs` of one group."""
    def cnt(t):
        return 2 * (t + 1) if causal else 2 * nkv
    out = []
    for pj in pairs:
        out.append(cnt(pj))
        if T - 1 - pj != pj:
            out.append(cnt(T - 1 - pj))
    return out


def run(items, ST, seed):
    rnd = random.Random(seed)
    bars = {("q",): Bar(1), ("q_empty",): Bar(8), ("qt",): Bar(8), ("acc_full",): Bar(1), ("acc_free",): Bar(8)}
    for b in (0, 1):
        bars[("sdp", b)], bars[("ds", b)], bars[("dqd", b)] = Bar(2), Bar(8), Bar(1)
    for s in range(ST):
        bars[("kv", s)], bars[("empty", s)] = Bar(1), Bar(1)
    err = []
    subs = [(n, it) for n, cnt in enumerate(items) for it in range(cnt)]
    qsm = [None]                 # the item whose Q / dO the shared-memory buffer holds
    qt = [None]                  # the item whose Q / dO are in TMEM
    qt_pending = [0]             # S / dP UMMAs issued that still read them
    stage, stage_reads = [None] * ST, [0] * ST
    sbuf = [None, None]          # TMEM S buffers: ("S", g) or ("read", g)
    dpbuf = [None, None]         # TMEM dP buffers: ("dP", g), ("dS", g) or ("read", g)
    acc, acc_read = [None], set()
    pipes = {0: [], 1: [], 2: []}
    copies = []

    def producer():
        gi = 0
        for n, cnt in enumerate(items):
            if n >= 1:
                yield ("wait", ("q_empty",), n - 1)
            qsm[0] = ("in flight",)

            def land_q(n=n):
                qsm[0] = n
                bars[("q",)].arrive()
            copies.append(land_q)
            for it in range(cnt):
                s, f = gi % ST, gi // ST
                if f > 0:
                    yield ("wait", ("empty", s), f - 1)
                if stage_reads[s]:
                    err.append(f"stage {s} reloaded with {stage_reads[s]} reads pending")
                stage[s], stage_reads[s] = ("in flight",), 3

                def land(s=s, g=gi):
                    stage[s] = g
                    bars[("kv", s)].arrive()
                copies.append(land)
                gi += 1

    def issuer(role):  # 0: S, 1: dP, 2: dQ
        for g, (n, it) in enumerate(subs):
            b = g & 1
            if role < 2:
                if it == 0:
                    yield ("wait", ("qt",), n)
                yield ("wait", ("kv", g % ST), g // ST)
                if g >= 2:
                    yield ("wait", ("ds", b), (g - 2) >> 1)
                if role == 1 and g >= 2:
                    yield ("wait", ("dqd", b), (g - 2) >> 1)
                qt_pending[0] += 1
                pipes[role].append(("S" if role == 0 else "dP", g))
                pipes[role].append(("commit", ("sdp", b)))
            else:
                yield ("wait", ("ds", b), g >> 1)
                if it == 0 and n > 0:
                    yield ("wait", ("acc_free",), n - 1)
                pipes[2].append(("dQ", g))
                pipes[2].append(("commit", ("empty", g % ST)))
                pipes[2].append(("commit", ("dqd", b)))
                if it == items[n] - 1:
                    pipes[2].append(("commit", ("acc_full",)))

    def put_q(n):
        yield ("wait", ("q",), n)
        if qsm[0] != n:
            err.append(f"Q / dO of item {n} copied from a buffer holding {qsm[0]}")
        if qt_pending[0]:
            err.append(f"Q / dO of item {n} written to TMEM with {qt_pending[0]} S / dP reads pending")
        qt[0] = n
        yield ("arrive", ("qt",), 8)
        yield ("arrive", ("q_empty",), 8)

    def ds_warps():
        if not subs:
            return
        yield from put_q(0)
        for g, (n, it) in enumerate(subs):
            b = g & 1
            yield ("wait", ("sdp", b), g >> 1)
            if it == items[n] - 1 and n + 1 < len(items):
                yield from put_q(n + 1)
            if sbuf[b] != ("S", g) or dpbuf[b] != ("dP", g):
                err.append(f"dS warps read S {sbuf[b]} dP {dpbuf[b]} for sub-tile {g}")
            sbuf[b] = ("read", g)
            yield ("yield",)
            dpbuf[b] = ("dS", g)
            yield ("arrive", ("ds", b), 8)
            if it == items[n] - 1:
                yield ("wait", ("acc_full",), n)
                if acc[0] != (n, items[n]):
                    err.append(f"epilogue of item {n} reads the accumulator at {acc[0]}")
                acc_read.add(n)
                yield ("arrive", ("acc_free",), 8)

    def execute(role):
        op = pipes[role].pop(0)
        if op[0] == "commit":
            bars[op[1]].arrive()
            return
        g = op[1]
        n, it = subs[g]
        b, s = g & 1, g % ST
        if stage[s] != g:
            err.append(f"{op[0]}({g}) reads stage {s} = {stage[s]}")
        stage_reads[s] -= 1
        if op[0] in ("S", "dP"):
            if qt[0] != n:
                err.append(f"{op[0]}({g}) reads the Q / dO of item {qt[0]}, not {n}")
            qt_pending[0] -= 1
            buf = sbuf if op[0] == "S" else dpbuf
            if buf[b] is not None and buf[b] != ("read", g - 2):
                err.append(f"{op[0]}({g}) overwrites {buf[b]}")
            buf[b] = (op[0], g)
        else:
            if dpbuf[b] != ("dS", g):
                err.append(f"dQ({g}) reads {dpbuf[b]}")
            dpbuf[b] = ("read", g)
            if it == 0:
                if n > 0 and (n - 1) not in acc_read:
                    err.append(f"dQ of item {n} restarts the accumulator before item {n - 1} was read out")
                acc[0] = (n, 1)
            else:
                if acc[0] != (n, it):
                    err.append(f"dQ({g}) accumulates onto {acc[0]}")
                acc[0] = (n, it + 1)

    actors = {"producer": producer(), "issuer S": issuer(0), "issuer dP": issuer(1), "issuer dQ": issuer(2),
              "dS warps": ds_warps()}
    pending = {name: None for name in actors}
    finished = set()
    while not err:
        runnable = [a for a in actors if a not in finished and
                    (pending[a] is None or bars[pending[a][1]].done >= pending[a][2] + 1)]
        choices = runnable + [("pipe", r) for r in pipes if pipes[r]] + (["copy"] if copies else [])
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
            if op[0] in ("arrive", "yield"):  # then any other actor may run first
                if op[0] == "arrive":
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
    for T in range(1, 10):
        npairs = (T + 1) // 2
        for ST in (2, 3, 4):  # at most 3 at head dim 128, 3 or 4 at 64
            out.append((items_for(T, range(npairs)), ST))                      # a CTA's pairs of one group
            out.append((items_for(T, [0]) * 3, ST))                             # pair (0, T-1) of three groups
            out.append((items_for(T, range(npairs))[1:], ST))                   # a range starting inside a pair
        out.append((items_for(T, range(npairs), causal=False, nkv=3), 3))      # chunk over a 3-tile key segment
    return out


@pytest.mark.parametrize("idx", range(len(cases())))
def test_dq_protocol_runs_clean(idx):
    items, ST = cases()[idx]
    for seed in range(10):
        problems = run(list(items), ST, seed)
        assert not problems, (problems, items, ST)


PLANTED = {
    # dP overwriting its buffer without waiting for dQ(g-2), the last reader of the dS there
    "dS buffer reused early": (
        "                if role == 1 and g >= 2:\n                    yield (\"wait\", (\"dqd\", b), (g - 2) >> 1)\n",
        ""),
    # the next item's Q / dO written to TMEM before this item's last S / dP completed
    "Q / dO replaced early": (
        "            yield (\"wait\", (\"sdp\", b), g >> 1)\n            if it == items[n] - 1 and n + 1 < len(items):\n"
        "                yield from put_q(n + 1)\n",
        "            if it == items[n] - 1 and n + 1 < len(items):\n                yield from put_q(n + 1)\n"
        "            yield (\"wait\", (\"sdp\", b), g >> 1)\n"),
    # S overwriting its buffer without waiting for the dS warps to have read S(g-2)
    "S buffer reused early": (
        "                if g >= 2:\n                    yield (\"wait\", (\"ds\", b), (g - 2) >> 1)\n",
        "                if g >= 2 and role == 1:\n                    yield (\"wait\", (\"ds\", b), (g - 2) >> 1)\n"),
    # the Q / dO buffer reloaded before its copy into TMEM
    "Q buffer reused early": (
        "            if n >= 1:\n                yield (\"wait\", (\"q_empty\",), n - 1)\n",
        ""),
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
