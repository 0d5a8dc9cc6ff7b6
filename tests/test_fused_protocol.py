"""A model of the fused backward kernel's synchronisation (s2_bwd_fused_kernel in
csrc/s2_bwd_fused.cu), run on the CPU like the other kernels' models: the
producer (K and V single-buffered, each released by its item's last readers;
a ring of ST stages of Q / dO / row statistics), issuers A (S^T, dV) and B
(dP^T, dK), each issuing the next sub-tile's scores before this one's
gradients except at an item's end, issuer C (dQ^T into one of two TMEM
buffers, then the bulk reduction of the previous sub-tile's staged partial),
the elementwise warps (P^T / dS^T into a shared-memory pair per sub-tile
parity, the dQ^T partial of the previous sub-tile staged into its finished
pair, the item's epilogue) and the copies in flight (loads landing and the
bulk reductions reading their staged pair in any order); after every wait
and every arrival any other actor may go first.  Checks: no deadlock, no
parity wait overrun or wait ahead of its barrier, every UMMA and copy reads
the buffer contents it means, nothing is overwritten while a reader still
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
    bars = {("k",): Bar(1), ("v",): Bar(1), ("k_empty",): Bar(2), ("v_empty",): Bar(1), ("s",): Bar(1),
            ("dp",): Bar(1), ("sdp_free",): Bar(8), ("acc_full",): Bar(2), ("acc_free",): Bar(8)}
    for s in range(ST):
        bars[("full", s)], bars[("empty", s)] = Bar(1), Bar(2)
    for b in (0, 1):
        bars[("pds", b)], bars[("mma_done", b)], bars[("dq_free", b)] = Bar(8), Bar(3), Bar(8)
        bars[("stg_full", b)], bars[("buf_free", b)] = Bar(8), Bar(1)
    err = []
    subs = [(n, it) for n, cnt in enumerate(items) for it in range(cnt)]
    last_g = {n: max(g for g, (nn, _) in enumerate(subs) if nn == n) for n in range(len(items))}
    kbuf, vbuf, k_reads, v_reads = [None], [None], [0], [0]
    stage, stage_reads = [None] * ST, [0] * ST
    tS, tdP = [None], [None]             # TMEM scores: ("raw", g) or ("read", g)
    pair = [None, None]                  # shared-memory pair: ("ps", g) / ("stg", g) / ("free", g)
    pair_reads = [0, 0]                  # dV, dK, dQ^T still to read P^T / dS^T
    tdq = [None, None]                   # TMEM dQ^T buffers: ("dq", g) or ("read", g)
    acc, acc_read, grads = [None], set(), set()
    pipes = {0: [], 1: [], 2: []}
    copies = []
    reduce_pending = [[]]                # sub-tiles whose bulk reduction has not read its pair yet

    def producer():
        gi, nk, nv = 0, 0, 0

        def load_stage():
            nonlocal gi
            s, f = gi % ST, gi // ST
            if f > 0:
                yield ("wait", ("empty", s), f - 1)
            if stage_reads[s]:
                err.append(f"stage {s} reloaded with {stage_reads[s]} reads pending")
            stage[s], stage_reads[s] = ("in flight",), 5

            def land(s=s, g=gi):
                stage[s] = g
                bars[("full", s)].arrive()
            copies.append(land)
            gi += 1

        for n, cnt in enumerate(items):
            pre = min(cnt, ST)
            for _ in range(pre):
                yield from load_stage()
            for name, buf, reads, nn, per in (("v", vbuf, v_reads, nv, 1), ("k", kbuf, k_reads, nk, 2)):
                if nn > 0:
                    yield ("wait", (name + "_empty",), nn - 1)
                if reads[0]:
                    err.append(f"{name.upper()} of item {n} loaded over {reads[0]} pending reads")
                buf[0], reads[0] = ("in flight",), per * cnt

                def land(buf=buf, name=name, n=n):
                    buf[0] = n
                    bars[(name,)].arrive()
                copies.append(land)
            nv += 1
            nk += 1
            for _ in range(pre, cnt):
                yield from load_stage()

    def issuer_ab(x):  # 0: A (S^T, dV), 1: B (dP^T, dK)
        def issue_sp(g):
            n, it = subs[g]
            if it == 0:
                yield ("wait", ("k",) if x == 0 else ("v",), n)
            yield ("wait", ("full", g % ST), g // ST)
            if g > 0:
                yield ("wait", ("sdp_free",), g - 1)
            pipes[x].append(("SP", g))
            pipes[x].append(("commit", ("s",) if x == 0 else ("dp",)))
            if g == last_g[n]:
                pipes[x].append(("commit", ("k_empty",) if x == 0 else ("v_empty",)))

        def issue_grad(g):
            n, it = subs[g]
            yield ("wait", ("pds", g & 1), g >> 1)
            if it == 0 and n > 0:
                yield ("wait", ("acc_free",), n - 1)
            pipes[x].append(("GRAD", g))
            pipes[x].append(("commit", ("empty", g % ST)))
            pipes[x].append(("commit", ("mma_done", g & 1)))
            if g == last_g[n]:
                pipes[x].append(("commit", ("acc_full",)))

        if not subs:
            return
        yield from issue_sp(0)
        for g, (n, it) in enumerate(subs):
            nxt = g + 1 < len(subs)
            boundary = g == last_g[n]
            if not boundary and nxt:
                yield from issue_sp(g + 1)
            yield from issue_grad(g)
            if boundary and nxt:
                yield from issue_sp(g + 1)

    def issuer_c():
        def reduce(g):
            b = g & 1
            yield ("wait", ("stg_full", b), g >> 1)
            reduce_pending[0].append(g)

            def read(g=g, b=b):
                if pair[b] != ("stg", g):
                    err.append(f"bulk reduction of sub-tile {g} reads pair {b} = {pair[b]}")
                reduce_pending[0].remove(g)
            copies.append(read)
            yield ("until", lambda g=g: g not in reduce_pending[0])
            pair[b] = ("free", g)
            yield ("arrive", ("buf_free", b), 1)

        for g, (n, it) in enumerate(subs):
            b = g & 1
            yield ("wait", ("pds", b), g >> 1)
            if g >= 2:
                yield ("wait", ("dq_free", b), (g - 2) >> 1)
            pipes[2].append(("DQ", g))
            pipes[2].append(("commit", ("mma_done", b)))
            if g == last_g[n]:
                pipes[2].append(("commit", ("k_empty",)))
            if g >= 1:
                yield from reduce(g - 1)
        if subs:
            yield from reduce(len(subs) - 1)

    def stage_dq(gp):
        b = gp & 1
        yield ("wait", ("mma_done", b), gp >> 1)
        if tdq[b] != ("dq", gp):
            err.append(f"dQ^T staging of sub-tile {gp} reads TMEM buffer {b} = {tdq[b]}")
        tdq[b] = ("read", gp)
        yield ("arrive", ("dq_free", b), 8)
        if pair[b] != ("ps", gp) or pair_reads[b]:
            err.append(f"dQ^T of sub-tile {gp} staged over pair {b} = {pair[b]} with {pair_reads[b]} reads pending")
        pair[b] = ("stg", gp)
        yield ("arrive", ("stg_full", b), 8)

    def elementwise():
        for g, (n, it) in enumerate(subs):
            s, b = g % ST, g & 1
            yield ("wait", ("full", s), g // ST)
            yield ("wait", ("s",), g)
            yield ("wait", ("dp",), g)
            if stage[s] != g or tS[0] != ("raw", g) or tdP[0] != ("raw", g):
                err.append(f"elementwise reads stage {stage[s]}, S^T {tS[0]}, dP^T {tdP[0]} for sub-tile {g}")
            stage_reads[s] -= 1
            tS[0], tdP[0] = ("read", g), ("read", g)
            yield ("arrive", ("sdp_free",), 8)
            if g >= 2:
                yield ("wait", ("buf_free", b), (g - 2) >> 1)
            if pair[b] is not None and pair[b] != ("free", g - 2):
                err.append(f"P^T / dS^T of sub-tile {g} written over pair {b} = {pair[b]}")
            pair[b], pair_reads[b] = ("ps", g), 3
            yield ("arrive", ("pds", b), 8)
            if g >= 1:
                yield from stage_dq(g - 1)
            if g == last_g[n]:
                yield ("wait", ("acc_full",), n)
                if any((x, gg) not in grads for x in (0, 1) for gg, (nn, _) in enumerate(subs) if nn == n):
                    err.append(f"epilogue of item {n} before its gradient UMMAs")
                acc_read.add(n)
                yield ("arrive", ("acc_free",), 8)
        if subs:
            yield from stage_dq(len(subs) - 1)

    def execute(r):
        op = pipes[r].pop(0)
        if op[0] == "commit":
            bars[op[1]].arrive()
            return
        g = op[1]
        n, it = subs[g]
        s, b = g % ST, g & 1
        if op[0] == "SP":
            buf, kv, reads = (tS, kbuf, k_reads) if r == 0 else (tdP, vbuf, v_reads)
            if stage[s] != g or kv[0] != n:
                err.append(f"SP{r}({g}) reads stage {stage[s]}, K/V of {kv[0]}")
            if buf[0] is not None and buf[0] != ("read", g - 1):
                err.append(f"SP{r}({g}) overwrites {buf[0]}")
            stage_reads[s] -= 1
            reads[0] -= 1
            buf[0] = ("raw", g)
        elif op[0] == "GRAD":
            if stage[s] != g or pair[b] != ("ps", g):
                err.append(f"GRAD{r}({g}) reads stage {stage[s]}, pair {pair[b]}")
            stage_reads[s] -= 1
            pair_reads[b] -= 1
            if it == 0 and n > 0 and (n - 1) not in acc_read:
                err.append(f"GRAD{r}({g}) restarts the accumulator before item {n - 1} was read out")
            grads.add((r, g))
        else:
            if pair[b] != ("ps", g) or kbuf[0] != n:
                err.append(f"DQ({g}) reads pair {pair[b]}, K of {kbuf[0]}")
            if tdq[b] is not None and tdq[b] != ("read", g - 2):
                err.append(f"DQ({g}) overwrites TMEM buffer {b} = {tdq[b]}")
            pair_reads[b] -= 1
            k_reads[0] -= 1
            tdq[b] = ("dq", g)

    actors = {"producer": producer(), "issuer A": issuer_ab(0), "issuer B": issuer_ab(1), "issuer C": issuer_c(),
              "elementwise": elementwise()}
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
        choices = runnable + [("pipe", r) for r in pipes if pipes[r]] + (["copy"] if copies else [])
        if not choices:
            if len(finished) == len(actors):
                return []
            return ["deadlock: " + ", ".join(f"{a} waits {pending[a][:2]}" for a in actors if a not in finished)]
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
    for T in range(1, 7):
        npairs = (T + 1) // 2
        for rep in (1, 2):
            for ST in (2, 3):
                out.append((items_for(T, rep, range(npairs)), ST))     # a CTA's pairs of one group
            out.append((items_for(T, rep, range(npairs))[1:], 3))       # a range starting inside a pair
            out.append((items_for(T, rep, [0]) * 2, 2))                 # pair (0, T-1) of two groups
    return out


@pytest.mark.parametrize("idx", range(len(cases())))
def test_fused_protocol_runs_clean(idx):
    items, ST = cases()[idx]
    for seed in range(8):
        problems = run(list(items), ST, seed)
        assert not problems, (problems, items, ST)


PLANTED = {
    # the elementwise warps writing P^T / dS^T over a pair whose staged dQ^T is still being reduced
    "pair reused early": ("            if g >= 2:\n                yield (\"wait\", (\"buf_free\", b), (g - 2) >> 1)\n", ""),
    # the next scores written before the elementwise warps have read the current ones
    "scores overwritten early": ("            if g > 0:\n                yield (\"wait\", (\"sdp_free\",), g - 1)\n", ""),
    # the partial staged without waiting for the sub-tile's UMMAs
    "staged before the UMMAs": ("        yield (\"wait\", (\"mma_done\", b), gp >> 1)\n", ""),
    # the pair released before the bulk reduction has read it
    "pair released before the reduction read it": (
        "            yield (\"until\", lambda g=g: g not in reduce_pending[0])\n", ""),
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
