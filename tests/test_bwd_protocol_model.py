"""Event model of the tensor-core backward's barrier protocol, checked on the
CPU (the dq kernel; the dkdv kernel has the same structure).

The roles mirror the kernel:
- the loader issues the fixed Q/dO tiles and a 2-deep ring of K/V tiles;
- the MMA warp issues each block's S/dP as two 64-column halves, then after
  each half's P arrival that half's dQ product, and after the second half
  the ring-slot release;
- four element-wise warps turn each S/dP half into dS.

TMA copies complete after random delays and in any order; MMAs run in issue
order, and a commit arrives once every earlier op is done.  Checks: every
mbarrier wait lands on exactly its intended phase (no early pass, no phase
two ahead), no S/dP half, ring slot or dQ accumulator is read or overwritten
out of turn, and nothing deadlocks.  A planted missing wait must be caught.
"""
import pytest

import random


class Bar:
    def __init__(self, count):
        self.count, self.arr, self.tx, self.phase = count, 0, 0, 0

    def arrive(self):
        self.arr += 1
        self._c()

    def expect(self, b):
        self.tx += b
        self.arr += 1
        self._c()

    def done_tx(self, b):
        self.tx -= b
        self._c()

    def _c(self):
        if self.arr == self.count and self.tx == 0:
            self.arr = 0
            self.phase += 1


class V(Exception):
    pass


def run(n, seed, mutate=None):
    rng = random.Random(seed)
    B = {"fixed": Bar(1), ("ring", 0): Bar(1), ("ring", 1): Bar(1), ("free", 0): Bar(1),
         ("free", 1): Bar(1), ("S", 0): Bar(1), ("S", 1): Bar(1), ("P", 0): Bar(4), ("P", 1): Bar(4)}
    ring = [{"c": None, "w": False} for _ in range(2)]
    fixed = {"c": None}
    half = [{"c": None} for _ in range(2)]      # S/dP half h content: ('S', it) or ('dS', it, warps)
    dq = {"through": None}
    tma = []
    mma = []
    consumed = set()

    def W(bar, par, target, label):
        return ("wait", bar, par, target, label)

    def loader():
        if n == 0:
            return
        B["fixed"].expect(1)
        tma.append(("fixed", None, "fixed"))
        for it in range(n):
            s = it & 1
            yield W(("free", s), ((it >> 1) & 1) ^ 1, (it >> 1) - 1, f"slot {s} free for {it}")
            B[("ring", s)].expect(1)
            if ring[s]["w"]:
                raise V("ring written twice")
            ring[s]["w"] = True
            tma.append(("ring", s, it))
            yield ("step",)

    def mmaw():
        if n == 0:
            return
        yield W("fixed", 0, 0, "fixed")

        def issue_half(it, h):
            s = it & 1
            if h == 0:  # the second half reads the same ring slot
                yield W(("ring", s), (it >> 1) & 1, it >> 1, f"ring {it}")
            mma.append(("S", it, h))
            mma.append(("commit", ("S", h)))

        yield from issue_half(0, 0)
        yield from issue_half(0, 1)
        for it in range(n):
            for h in range(2):
                if mutate != "no_p_wait" or h == 0:
                    yield W(("P", h), it & 1, it, f"P {it} {h}")
                mma.append(("G", it, h))
                if h == 1:
                    mma.append(("commit", ("free", it & 1)))
                if it + 1 < n:
                    yield from issue_half(it + 1, h)

    def elem(w):
        for it in range(n):
            for h in range(2):
                yield W(("S", h), it & 1, it, f"S {it} {h} w{w}")
                c = half[h]["c"]
                if not (c and c[1] == it and c[0] in ("S", "dS")):
                    raise V(f"w{w} reads half {h} = {c} for block {it}")
                yield ("step",)
                c = half[h]["c"]  # another warp may have written its lanes meanwhile
                if c[0] == "S":
                    half[h]["c"] = ("dS", it, {w})
                else:
                    c[2].add(w)
                B[("P", h)].arrive()
        if n:
            gl = n - 1
            yield W(("free", gl & 1), (gl >> 1) & 1, gl >> 1, f"final w{w}")
            if dq["through"] != (n - 1, 1):
                raise V(f"final read of dQ through {dq['through']}")

    actors = {"loader": loader(), "mma": mmaw()}
    for w in range(4):
        actors[f"e{w}"] = elem(w)
    blocked, done = {}, set()

    def ok(req):
        _, bar, par, target, label = req
        b = B[bar]
        if (b.phase & 1) != par:
            if b.phase != target + 1 and not (target < 0 and b.phase == 0):
                raise V(f"'{label}' passed at phase {b.phase}, meant {target + 1}")
            return True
        if b.phase >= target + 2:
            raise V(f"'{label}' blocks forever at phase {b.phase}")
        return False

    def exe(op):
        if op[0] == "S":
            _, it, h = op
            s = it & 1
            if ring[s]["c"] != it or ring[s]["w"] or fixed["c"] is None:
                raise V(f"S({it},{h}) reads ring {ring[s]} fixed {fixed}")
            c = half[h]["c"]
            if c is not None and (c[0] != "dS" or (c[1], h) not in consumed):
                raise V(f"S({it},{h}) overwrites half {h} = {c}")
            half[h]["c"] = ("S", it)
        elif op[0] == "G":
            _, it, h = op
            s = it & 1
            c = half[h]["c"]
            if not (c and c[0] == "dS" and c[1] == it and len(c[2]) == 4):
                raise V(f"G({it},{h}) reads half {h} = {c}")
            if ring[s]["c"] != it or ring[s]["w"]:
                raise V(f"G({it},{h}) reads ring {ring[s]}")
            want = None if (it, h) == (0, 0) else ((it, 0) if h == 1 else (it - 1, 1))
            if dq["through"] != want:
                raise V(f"G({it},{h}) accumulates onto {dq['through']}")
            dq["through"] = (it, h)
            consumed.add((it, h))

    steps = 0
    while True:
        steps += 1
        if steps > 10 ** 6:
            raise V("no progress")
        run_ = [a for a in actors if a not in done and (a not in blocked or ok(blocked[a]))]
        ev = (["_tma"] if tma else []) + (["_mma"] if mma else [])
        if not run_ and not ev:
            if len(done) == len(actors):
                return
            raise V("deadlock: " + "; ".join(blocked[a][4] for a in blocked if a not in done))
        ch = rng.choice(run_ + ev * 2)
        if ch == "_tma":
            kind, s, it = tma.pop(rng.randrange(len(tma)))
            if kind == "fixed":
                fixed["c"] = 1
                B["fixed"].done_tx(1)
            else:
                ring[s]["c"], ring[s]["w"] = it, False
                B[("ring", s)].done_tx(1)
            continue
        if ch == "_mma":
            op = mma.pop(0)
            if op[0] == "commit":
                B[op[1]].arrive()
            else:
                exe(op)
            continue
        blocked.pop(ch, None)
        try:
            req = next(actors[ch])
        except StopIteration:
            done.add(ch)
            continue
        if req[0] == "wait" and not ok(req):
            blocked[ch] = req



@pytest.mark.parametrize("n", [0, 1, 2, 3, 4, 5, 8, 13])
def test_protocol_holds_under_random_timing(n):
    for seed in range(60):
        run(n, seed)


def test_model_catches_a_missing_wait():
    caught = 0
    for seed in range(30):
        try:
            run(6, seed, mutate="no_p_wait")
        except V:
            caught += 1
    assert caught >= 20, caught
