"""A model of the 64-key forward kernel's synchronisation (s2_fwd64_kernel in
csrc/s2_fwd64.cu), run on the CPU like the 128-key forward's
(test_fwd_protocol.py): the TMA producer (Q ring of three 128-row tiles, K/V
ring of 64-row tiles), the UMMA issuer (per 64-key tile j: P V_A(j), S_A(j+2),
P V_B(j), S_B(j+2); the next item's first two scores of a warpgroup in the
places of S(n) and S(n+1)), the two softmax warpgroups with their two score
buffers each and their epilogues, the tensor pipe (in order) and the copies in
flight (landing in any order); after every wait and every arrival any other
actor may go first.  Checks: no deadlock, no parity wait overrun
(a barrier two phases ahead of the waiter, which a parity wait cannot tell
from the phase it wants), every UMMA reads the tile and buffer it means, and
nothing is overwritten while a reader still needs it.  The item sequences
are those of the 128-key model (test_fwd_protocol.items_for and friends)."""
import random

import pytest

from tests.test_fwd_protocol import items_for, pairs_order, sequences

NQ = 3


class Bar:
    def __init__(self, count):
        self.count, self.rem, self.done = count, count, 0

    def arrive(self, n=1):
        for _ in range(n):
            self.rem -= 1
            if self.rem == 0:
                self.done += 1
                self.rem = self.count


def n_tiles(it, w):
    """64-key tiles of warpgroup w in an item (two per 128-key tile up to its last)."""
    if w == 0:
        return 2 * (it["last_a"] + 1)
    return 2 * (it["last_b"] + 1) if it["has_b"] else 0


def run(items, seed, NS=8):
    rnd = random.Random(seed)
    bars = {}
    for s in range(NQ):
        bars[("qfull", s)], bars[("qempty", s)] = Bar(1), Bar(4)
    for s in range(NS):
        bars[("full", s)], bars[("empty", s)] = Bar(1), Bar(1)
    for w in (0, 1):
        for b in (0, 1):
            bars[("s", w, b)], bars[("p", w, b)] = Bar(1), Bar(4)
        bars[("o", w)], bars[("ofree", w)] = Bar(1), Bar(4)
    err = []
    qslot, qreads, ring, ringreads = [None] * NQ, [0] * NQ, [None] * NS, [0] * NS
    sbuf = [[None, None], [None, None]]  # per warpgroup and score buffer: ("S"|"P", item, tile)
    pv_done, o_read, pipe, tma = set(), set(), [], []

    def readers(k, j):
        return (j < n_tiles(items[k], 0)) + (j < n_tiles(items[k], 1))

    def producer():
        qu, L = 0, 0

        def load_q(k, w, present):
            nonlocal qu
            s, r = qu % NQ, qu // NQ
            if r > 0:
                yield ("wait", ("qempty", s), r - 1)
            if qreads[s]:
                err.append(f"Q slot {s} reloaded with S reads pending")
            qreads[s] = n_tiles(items[k], w) if present else 0
            qslot[s] = ("in flight",)

            def land(s=s, tile=((k, w) if present else None)):
                qslot[s] = tile
                bars[("qfull", s)].arrive()
            tma.append(land)
            qu += 1

        def load_kv(k, kind, j):
            nonlocal L
            s, r = L % NS, L // NS
            if r > 0:
                yield ("wait", ("empty", s), r - 1)
            if ringreads[s]:
                err.append(f"K/V slot {s} reloaded with {ringreads[s]} reads pending")
            ring[s], ringreads[s] = ("in flight",), readers(k, j)

            def land(s=s, tile=(k, kind, j)):
                ring[s] = tile
                bars[("full", s)].arrive()
            tma.append(land)
            L += 1

        yield from load_q(0, 0, True)
        yield from load_q(0, 1, items[0]["has_b"])
        qb_pending = False
        for k, it in enumerate(items):
            nx = k + 1 < len(items)
            n64 = n_tiles(it, 1 if it["has_b"] else 0)
            jq = min(5, n64 - 1)
            for j in range(n64):
                yield from load_kv(k, "K", j)
                yield from load_kv(k, "V", j)
                if j == 0 and qb_pending:
                    yield from load_q(k, 1, it["has_b"])
                if j == jq and nx:
                    yield from load_q(k + 1, 0, True)
            qb_pending = nx

    def issuer():
        n, L, pre = 0, 0, False
        npb = [[0, 0], [0, 0]]  # P tiles received per warpgroup and buffer

        def commit(name, times=1):
            pipe.extend([("commit", name)] * times)

        def full(Lx):
            return ("wait", ("full", Lx % NS), Lx // NS)

        def issue_s(w, k, j, qs, Lk, buf):
            yield full(Lk)
            pipe.append(("S", w, k, j, qs, Lk % NS, buf))
            commit(("s", w, buf))

        def pv(w, k, j, Lv):
            yield ("wait", ("p", w, j & 1), npb[w][j & 1])
            if j == 0 and n > 0:
                yield ("wait", ("ofree", w), n - 1)
            yield full(Lv)
            pipe.append(("PV", w, k, j, Lv % NS))
            commit(("o", w))
            npb[w][j & 1] += 1

        for k, it in enumerate(items):
            nx = items[k + 1] if k + 1 < len(items) else None
            ua, ub = 2 * n, 2 * n + 1
            sa, sb, san, sbn = ua % NQ, ub % NQ, (ua + 2) % NQ, (ub + 2) % NQ
            na, nb = n_tiles(it, 0), n_tiles(it, 1)
            n64 = max(na, nb)
            L0 = L
            L0n = L0 + 2 * n64
            if not pre:
                yield ("wait", ("qfull", sa), ua // NQ)
                yield ("wait", ("qfull", sb), ub // NQ)
                for e in (0, 1):
                    yield from issue_s(0, k, e, sa, L0 + 2 * e, e)
                    if it["has_b"]:
                        yield from issue_s(1, k, e, sb, L0 + 2 * e, e)
                    elif e == 0:
                        commit(("qempty", sb), 4)
                    commit(("empty", (L0 + 2 * e) % NS))
            elif not it["has_b"]:
                yield ("wait", ("qfull", sb), ub // NQ)
                commit(("qempty", sb), 4)

            def start_next_b():
                yield ("wait", ("qfull", sbn), (ub + 2) // NQ)
                for e in (0, 1):
                    yield from issue_s(1, k + 1, e, sbn, L0n + 2 * e, e)
                    commit(("empty", (L0n + 2 * e) % NS))

            for j in range(n64):
                Lv = L0 + 2 * j + 1
                if j < na:
                    yield from pv(0, k, j, Lv)
                    if j >= nb:
                        commit(("empty", Lv % NS))
                    t = j + 2
                    if t < na:
                        yield from issue_s(0, k, t, sa, L0 + 2 * t, t & 1)
                        if t >= nb:
                            commit(("empty", (L0 + 2 * t) % NS))
                    elif nx is not None:
                        e = t - na
                        yield ("wait", ("qfull", san), (ua + 2) // NQ)
                        yield from issue_s(0, k + 1, e, san, L0n + 2 * e, e)
                        if not nx["has_b"]:
                            commit(("empty", (L0n + 2 * e) % NS))
                        if e == 1 and nx["has_b"] and not it["has_b"]:
                            yield from start_next_b()
                if j < nb:
                    yield from pv(1, k, j, Lv)
                    commit(("empty", Lv % NS))
                    t = j + 2
                    if t < nb:
                        yield from issue_s(1, k, t, sb, L0 + 2 * t, t & 1)
                        commit(("empty", (L0 + 2 * t) % NS))
                    elif nx is not None and nx["has_b"] and t - nb == 1:
                        yield from start_next_b()
            L, n, pre = L0n, n + 1, nx is not None

    def softmax(w):
        nsb, no = [0, 0], 0
        for k, it in enumerate(items):
            nt = n_tiles(it, w)
            if nt == 0:
                yield ("arrive", ("ofree", w), 4)
                continue
            for j in range(nt):
                b = j & 1
                yield ("wait", ("s", w, b), nsb[b])
                nsb[b] += 1
                if sbuf[w][b] != ("S", k, j):
                    err.append(f"softmax {w} reads {sbuf[w][b]} for S({k},{j}) in buffer {b}")
                if j > 0 and rnd.random() < 0.2:  # lazy rescale of O after P V(j-1)
                    yield ("wait", ("o", w), no - 1)
                if j == nt - 1:
                    # the item's last P: P V(j-1) first, so that the epilogue's
                    # parity wait never has two P V phases outstanding
                    yield ("wait", ("o", w), no - 1)
                sbuf[w][b] = ("P", k, j)
                yield ("arrive", ("p", w, b), 4)
                no += 1
            yield ("wait", ("o", w), no - 1)
            if any(("PV", w, k, j) not in pv_done for j in range(nt)):
                err.append(f"epilogue {w} of item {k} before its P V")
            o_read.add((w, k))
            yield ("arrive", ("ofree", w), 4)
            slot = (2 * k + w) % NQ
            if qreads[slot]:
                err.append(f"epilogue {w} stages O over Q slot {slot} with S reads pending")
            yield ("arrive", ("qempty", slot), 4)

    def execute():
        op = pipe.pop(0)
        if op[0] == "commit":
            bars[op[1]].arrive()
            return
        kind, w, k, j = op[:4]
        if kind == "S":
            qs, ks, b = op[4], op[5], op[6]
            if qslot[qs] != (k, w) or ring[ks] != (k, "K", j):
                err.append(f"S{w}({k},{j}) reads Q {qslot[qs]} K {ring[ks]}")
            prev = sbuf[w][b]
            if prev is not None and (prev[0] != "P" or ("PV", w, prev[1], prev[2]) not in pv_done):
                err.append(f"S{w}({k},{j}) overwrites {prev} in buffer {b}")
            qreads[qs] -= 1
            ringreads[ks] -= 1
            sbuf[w][b] = ("S", k, j)
            return
        if ring[op[4]] != (k, "V", j):
            err.append(f"PV{w}({k},{j}) reads V {ring[op[4]]}")
        if sbuf[w][j & 1] != ("P", k, j):
            err.append(f"PV{w}({k},{j}) reads {sbuf[w][j & 1]}")
        prev = [kk for kk in range(k) if n_tiles(items[kk], w) > 0]
        if j == 0 and prev and (w, prev[-1]) not in o_read:
            err.append(f"PV{w}({k},0) overwrites O of item {prev[-1]} before it is read")
        ringreads[op[4]] -= 1
        pv_done.add(("PV", w, k, j))

    actors = {"producer": producer(), "issuer": issuer(), "softmax A": softmax(0), "softmax B": softmax(1)}
    pending = {name: None for name in actors}
    finished = set()
    while not err:
        runnable = [a for a in actors if a not in finished and
                    (pending[a] is None or bars[pending[a][1]].done >= pending[a][2] + 1)]
        choices = runnable + (["pipe"] if pipe else []) + (["tma"] if tma else [])
        if not choices:
            if len(finished) == len(actors):
                return []
            return ["deadlock: " + ", ".join(f"{a} waits {pending[a]}" for a in actors if a not in finished)]
        c = rnd.choice(choices)
        if c == "pipe":
            execute()
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
                return [f"{c}: phase overrun on {op[1]} (waits phase {op[2]}, {done} complete)"]
            if done >= op[2] + 1:
                continue
            pending[c] = op
            break
    return err[:3]


@pytest.mark.parametrize("idx", range(len(sequences())))
def test_fwd64_protocol_runs_clean(idx):
    items = [dict(x) for x in sequences()[idx]]
    for seed in range(12):
        problems = run([dict(x) for x in items], seed)
        assert not problems, (problems, [(x["last_a"], x["last_b"], x["has_b"]) for x in items])


def test_model_finds_the_epilogue_parity_race():
    """With the epilogue the kernel had (after the last P, a wait for P V(nt-2)
    and then for P V(nt-1)), both P V can complete before the first wait, and
    that parity wait then names a phase two behind the barrier: the model
    reports it.  The kernel now waits for P V(nt-2) before handing over its
    last P, and the epilogue waits for the last P V alone."""
    import inspect
    import textwrap
    src = textwrap.dedent(inspect.getsource(run))
    last = """                if j == nt - 1:
                    # the item's last P: P V(j-1) first, so that the epilogue's
                    # parity wait never has two P V phases outstanding
                    yield ("wait", ("o", w), no - 1)
"""
    epi = """            yield ("wait", ("o", w), no - 1)
            if any(("PV", w, k, j) not in pv_done"""
    assert last in src and epi in src
    src = src.replace(last, "").replace(epi, """            yield ("wait", ("o", w), no - 2)
            yield ("wait", ("o", w), no - 1)
            if any(("PV", w, k, j) not in pv_done""")
    ns = dict(globals())
    exec(src, ns)
    found = [p for items in sequences()[:12] for seed in range(8) for p in ns["run"]([dict(x) for x in items], seed)]
    assert any("phase overrun on ('o'" in p for p in found)


def test_fwd64_protocol_twelve_slots():
    """The 12-slot K/V ring head dim 64 can select."""
    for items in sequences()[::3]:
        for seed in range(4):
            problems = run([dict(x) for x in items], seed, NS=12)
            assert not problems, (problems, [(x["last_a"], x["last_b"], x["has_b"]) for x in items])
