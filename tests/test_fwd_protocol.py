"""A model of the forward kernel's synchronisation (csrc/s2_fwd.cu), run on the
CPU: the TMA producer, the UMMA issuer, the two softmax warpgroups with their
epilogues, the tensor pipe and the copies in flight (landing in any order), as
programs of mbarrier waits and arrivals with the kernel's arrival counts and
phases, interleaved at random (after every wait and every arrival any other
actor, the tensor pipe or a copy may go first).  It checks that
every program finishes (no deadlock), that no wait is overrun (a barrier two
phases ahead of the waiter, which a parity wait cannot tell apart), and that
every UMMA reads the tile it means and nothing is overwritten while a reader
still needs it.  The item sequences are what a CTA walks: equal-work pairs
(item i then item T/2-1-i of one group), longest first across groups, chunked
and HGA-offset diagonals, groups with an odd tile count (an item without a
second query tile).  The model follows the kernel's issuer step by step; it
found the deadlock the kernel had when an item without a second tile followed
one with it (fixed in the kernel: that tile's Q slot is released at the top of
its own item)."""
import random

import pytest

NQ = 3  # Q ring slots; the K/V ring has NS slots: 4 at head dim 128, 4, 6 or 8 at 64


class Bar:
    def __init__(self, count):
        self.count, self.rem, self.done = count, count, 0

    def arrive(self, n=1):
        for _ in range(n):
            self.rem -= 1
            if self.rem == 0:
                self.done += 1
                self.rem = self.count


def items_for(T, causal=True, nkt=None, nh=0):
    """The forward items of one group of T tiles: item i = query tiles 2i, 2i+1."""
    out = []
    for i in range((T + 1) // 2):
        ta = 2 * i
        has_b = ta + 1 < T
        if causal:
            last_a, last_b = ta + nh, (ta + 1 + nh if has_b else -1)
        else:
            last_a, last_b = nkt - 1, (nkt - 1 if has_b else -1)
        out.append(dict(has_b=has_b, last_a=last_a, last_b=last_b, nkv=(last_b if has_b else last_a) + 1))
    return out


def pairs_order(T, **kw):
    its = items_for(T, **kw)
    out = []
    for pj in range((len(its) + 1) // 2):
        out.append(its[pj])
        if len(its) - 1 - pj != pj:
            out.append(its[len(its) - 1 - pj])
    return out


def run(items, seed, NS=4):
    """Returns a list of problems (empty when the protocol ran clean)."""
    rnd = random.Random(seed)
    bars = {}
    for s in range(NQ):
        bars[("qfull", s)], bars[("qempty", s)] = Bar(1), Bar(4)
    for s in range(NS):
        bars[("full", s)], bars[("empty", s)] = Bar(1), Bar(1)
    for w in (0, 1):
        for name, cnt in (("s", 1), ("plo", 4), ("p", 4), ("o", 1), ("ofree", 4)):
            bars[(name, w)] = Bar(cnt)
    err = []
    qslot, qreads, ring, ringreads = [None] * NQ, [0] * NQ, [None] * NS, [0] * NS
    sbuf, pv_done, o_read, pipe = [None, None], set(), set(), []
    tma = []  # copies in flight: each lands (tile in its slot, barrier arrival) at a random later point

    def readers(k, j):
        it = items[k]
        return (j <= it["last_a"]) + (it["has_b"] and j <= it["last_b"])

    def producer():
        qu, L = 0, 0

        def load_q(k, w, present):
            nonlocal qu
            s, r = qu % NQ, qu // NQ
            if r > 0:
                yield ("wait", ("qempty", s), r - 1)
            if qreads[s]:
                err.append(f"Q slot {s} reloaded with S reads pending")
            # the S UMMAs that will read this tile: one per key tile of its warpgroup
            qreads[s] = (items[k]["last_a"] if w == 0 else items[k]["last_b"]) + 1 if present else 0
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
            jq = min(2, it["nkv"] - 1)
            for j in range(it["nkv"]):
                yield from load_kv(k, "K", j)
                yield from load_kv(k, "V", j)
                if j == 0 and qb_pending:
                    yield from load_q(k, 1, it["has_b"])
                if j == jq and nx:
                    yield from load_q(k + 1, 0, True)
            qb_pending = nx

    def issuer():
        n, L, pre, npw = 0, 0, False, [0, 0]

        def commit(name, times=1):
            pipe.extend([("commit", name)] * times)

        def full(Lx):
            return ("wait", ("full", Lx % NS), Lx // NS)

        def issue_s(w, k, j, qs, Lk):
            pipe.append(("S", w, k, j, qs, Lk % NS))
            commit(("s", w))

        def pv(w, k, j, Lv, need_v):
            yield ("wait", ("plo", w), npw[w])
            if j == 0 and n > 0:
                yield ("wait", ("ofree", w), n - 1)
            if need_v:
                yield full(Lv)
            pipe.append(("PVlo", w, k, j, Lv % NS))
            yield ("wait", ("p", w), npw[w])
            pipe.append(("PVhi", w, k, j, Lv % NS))
            commit(("o", w))
            npw[w] += 1

        for k, it in enumerate(items):
            nx = items[k + 1] if k + 1 < len(items) else None
            ua, ub = 2 * n, 2 * n + 1
            sa, sb, san, sbn = ua % NQ, ub % NQ, (ua + 2) % NQ, (ub + 2) % NQ
            la, lb = it["last_a"], (it["last_b"] if it["has_b"] else -1)
            L0 = L
            L0n = L0 + 2 * it["nkv"]
            if not pre:
                yield ("wait", ("qfull", sa), ua // NQ)
                yield full(L0)
                yield ("wait", ("qfull", sb), ub // NQ)
                issue_s(0, k, 0, sa, L0)
                if it["has_b"]:
                    issue_s(1, k, 0, sb, L0)
                else:
                    commit(("qempty", sb), 4)
                commit(("empty", L0 % NS))
            elif not it["has_b"]:
                yield ("wait", ("qfull", sb), ub // NQ)
                commit(("qempty", sb), 4)

            def start_next_a():
                if nx is None:
                    return
                yield ("wait", ("qfull", san), (ua + 2) // NQ)
                yield full(L0n)
                issue_s(0, k + 1, 0, san, L0n)
                if not nx["has_b"]:
                    commit(("empty", L0n % NS))

            def start_next_b():
                if nx is None or not nx["has_b"]:
                    return
                yield ("wait", ("qfull", sbn), (ub + 2) // NQ)
                issue_s(1, k + 1, 0, sbn, L0n)
                commit(("empty", L0n % NS))

            for j in range(it["nkv"]):
                Lv, Lk1 = L0 + 2 * j + 1, L0 + 2 * j + 2
                if j <= la:
                    yield from pv(0, k, j, Lv, True)
                    if j > lb:
                        commit(("empty", Lv % NS))
                    if j + 1 <= la:
                        yield full(Lk1)
                        issue_s(0, k, j + 1, sa, Lk1)
                        if j + 1 > lb:
                            commit(("empty", Lk1 % NS))
                    else:
                        yield from start_next_a()
                        if lb < 0:
                            yield from start_next_b()
                if j <= lb:
                    yield from pv(1, k, j, Lv, j > la)
                    commit(("empty", Lv % NS))
                    if j + 1 <= lb:
                        if j + 1 > la:
                            yield full(Lk1)
                        issue_s(1, k, j + 1, sb, Lk1)
                        commit(("empty", Lk1 % NS))
                    else:
                        yield from start_next_b()
            L, n, pre = L0n, n + 1, nx is not None

    def softmax(w):
        ns = no = 0
        for k, it in enumerate(items):
            if w == 1 and not it["has_b"]:
                yield ("arrive", ("ofree", w), 4)
                continue
            last = it["last_a"] if w == 0 else it["last_b"]
            for j in range(last + 1):
                yield ("wait", ("s", w), ns)
                ns += 1
                if sbuf[w] != ("S", k, j):
                    err.append(f"softmax {w} reads {sbuf[w]} for S({k},{j})")
                if j > 0 and rnd.random() < 0.2:  # lazy rescale of O after the previous P V
                    yield ("wait", ("o", w), no - 1)
                sbuf[w] = ("Plo", k, j)
                yield ("arrive", ("plo", w), 4)
                sbuf[w] = ("P", k, j)
                yield ("arrive", ("p", w), 4)
                no += 1
            yield ("wait", ("o", w), no - 1)
            if any(("PVhi", w, k, j) not in pv_done for j in range(last + 1)):
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
            qs, ks = op[4], op[5]
            if qslot[qs] != (k, w) or ring[ks] != (k, "K", j):
                err.append(f"S{w}({k},{j}) reads Q {qslot[qs]} K {ring[ks]}")
            prev = sbuf[w]
            if prev is not None and (prev[0] != "P" or ("PVhi", w, prev[1], prev[2]) not in pv_done):
                err.append(f"S{w}({k},{j}) overwrites {prev}")
            qreads[qs] -= 1
            ringreads[ks] -= 1
            sbuf[w] = ("S", k, j)
            return
        if ring[op[4]] != (k, "V", j):
            err.append(f"{kind}{w}({k},{j}) reads V {ring[op[4]]}")
        if kind == "PVlo":
            if sbuf[w] not in (("Plo", k, j), ("P", k, j)):
                err.append(f"PVlo{w}({k},{j}) reads {sbuf[w]}")
            prev = [kk for kk in range(k) if w == 0 or items[kk]["has_b"]]
            if j == 0 and prev and (w, prev[-1]) not in o_read:
                err.append(f"PV{w}({k},0) overwrites O of item {prev[-1]} before it is read")
        else:
            if sbuf[w] != ("P", k, j):
                err.append(f"PVhi{w}({k},{j}) reads {sbuf[w]}")
            ringreads[op[4]] -= 1
            pv_done.add(("PVhi", w, k, j))

    actors = {"producer": producer(), "issuer": issuer(), "softmax A": softmax(0), "softmax B": softmax(1)}
    pending = {name: None for name in actors}
    finished = set()
    while not err:
        runnable = [n for n in actors if n not in finished and
                    (pending[n] is None or bars[pending[n][1]].done >= pending[n][2] + 1)]
        choices = runnable + (["pipe"] if pipe else []) + (["tma"] if tma else [])
        if not choices:
            if len(finished) == len(actors):
                return []
            return ["deadlock: " + ", ".join(f"{n} waits {pending[n]}" for n in actors if n not in finished)]
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
                return [f"{c}: phase overrun on {op[1]}"]
            if done >= op[2] + 1:
                continue
            pending[c] = op
            break
    return err[:3]


def sequences():
    out = []
    for T in range(1, 12):
        out.append(pairs_order(T) * 2)                                  # equal-work pairs, two groups
        out.append(list(reversed(items_for(T))) + items_for(T))         # longest first, then the rest
        out.append(pairs_order(T, nh=2))                                 # HGA-offset diagonals
        out.append(pairs_order(T, causal=False, nkt=T + 1))              # chunk attending a whole key segment
    rnd = random.Random(3)
    for _ in range(40):                                                  # mixtures of groups of any length
        seq = []
        for _ in range(rnd.randint(2, 5)):
            its = items_for(rnd.randint(1, 11), nh=rnd.choice([0, 0, 2]))
            seq.append(its[rnd.randrange(len(its))])
        out.append(seq)
    return out


@pytest.mark.parametrize("idx", range(len(sequences())))
def test_forward_protocol_runs_clean(idx):
    items = [dict(x) for x in sequences()[idx]]
    for seed in range(12):
        problems = run([dict(x) for x in items], seed)
        assert not problems, (problems, [(x["last_a"], x["last_b"], x["has_b"]) for x in items])


@pytest.mark.parametrize("NS", [6, 8])
def test_forward_protocol_deeper_rings(NS):
    """The K/V ring depths head dim 64 can select."""
    for items in sequences()[::3]:
        for seed in range(4):
            problems = run([dict(x) for x in items], seed, NS)
            assert not problems, (problems, NS, [(x["last_a"], x["last_b"], x["has_b"]) for x in items])


def test_model_finds_the_fixed_deadlock():
    """The model with the issuer's old order (the absent second tile's Q slot
    released from the previous item's first-tile path) deadlocks on pair
    (0, last) of a 9-tile group: the check is not vacuous."""
    import inspect
    import textwrap
    src = textwrap.dedent(inspect.getsource(run))
    old = """            elif not it["has_b"]:
                yield ("wait", ("qfull", sb), ub // NQ)
                commit(("qempty", sb), 4)
"""
    assert old in src
    src = src.replace(old, "")
    src = src.replace("""                if not nx["has_b"]:
                    commit(("empty", L0n % NS))""", """                if not nx["has_b"]:
                    yield ("wait", ("qfull", sbn), (ub + 2) // NQ)
                    commit(("qempty", sbn), 4)
                    commit(("empty", L0n % NS))""")
    ns = dict(globals())
    exec(src, ns)
    its = items_for(9)
    assert any(p.startswith("deadlock") for seed in range(4) for p in ns["run"]([its[0], its[4]], seed))
    assert run([dict(its[0]), dict(its[4])], 0) == []
