"""A discrete-event model of the persistent attention kernel's barrier
protocol (csrc/attn_sm100.cu), run on the CPU.

Each role of the kernel -- the row scheduler, the Q/K loader, the V loader
(which also stores O), the MMA issuer and the two softmax warp groups -- is a
Python generator that follows the kernel's loops and uses the same barrier
indices, arrival counts and phase formulas.  The tensor pipe executes MMAs in
issue order with random durations; TMA loads land in random order after
random delays.  The model checks that:

  * nothing deadlocks (every row finishes);
  * every wait on a barrier lands on the phase it means (an mbarrier wait by
    parity cannot tell a phase from the one two later, so a barrier that has
    run two phases ahead of a waiter is a protocol error);
  * no buffer is overwritten while it is still being read: an S buffer and
    its P, a K or V ring slot (also the O staging tile), the Q tile, O in
    tensor memory, the 1/l vector and a row descriptor.

It holds no arithmetic; the GPU parity tests check the numbers.
"""
import random

import pytest

STAGES = 3
ROW_SLOTS = 2
SOFTMAX_GROUPS = 2          # warps 0-3 and 4-7, 4 arrivals each
GROUP_WARPS = 4
EPILOGUE_WARPS = 4          # warps 8-11
ROW_USERS = 8 + 3           # softmax warps, MMA issuer, two loaders


class ProtocolError(AssertionError):
    pass


class Barrier:
    """An mbarrier: `count` arrivals complete a phase; `done` phases so far."""

    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self, n=1):
        self.pending += n
        if self.pending > self.count:
            raise ProtocolError(f"{self.name}: {self.pending} arrivals for {self.count}")
        if self.pending == self.count:
            self.pending = 0
            self.done += 1


class Sim:
    def __init__(self, rows, seed):
        self.rng = random.Random(seed)
        self.rows = rows            # list of block counts per CSR row
        self.bars = {}
        self.tickets = 0
        self.t = 0
        self.mma_queue = []         # in issue order: (kind, g, barrier)
        self.mma_busy_until = None
        self.tma = []               # (land_time, barrier, action)
        # resource state for the hazard checks
        self.s_state = {}           # S buffer -> g whose S/P it holds, and stage
        self.written_rows = set()
        self.o_row = None           # row whose PVs O holds
        self.o_reads = {}           # row -> number of epilogue warps that read O
        self.inv_l = {}             # parity slot -> (row, readers done)
        self.v_slot = {}            # slot -> ("V", g) or ("O", row)
        self.k_slot = {}
        self.q_row = None
        self.s_done = set()
        self.pv_done = set()
        self.desc = {}              # slot -> (k, readers)
        self.mutation = None        # a planted protocol mistake (tests of the model)
        self.early = 0              # rows whose first S products were issued early

    # 1/l and its LReady barrier alternate by row parity
    def lslot(self, orow):
        return 0 if self.mutation == "single_inv_l" else orow & 1

    def lphase(self, orow):
        return orow if self.mutation == "single_inv_l" else orow // 2

    def bar(self, name, count=1):
        if name not in self.bars:
            self.bars[name] = Barrier(name, count)
        return self.bars[name]

    # a wait that means phase `phase` (0-based) of barrier `b`
    def ready(self, b, phase):
        if b.done >= phase + 2:
            raise ProtocolError(f"{b.name}: waited for phase {phase} after {b.done} phases")
        return b.done >= phase + 1

    # ------------------------------------------------------------ the engine
    def run(self, roles, max_steps=2_000_000):
        state = [dict(gen=r, wait=None, done=False, name=n) for n, r in roles]
        for st in state:
            self._advance(st)
        for _ in range(max_steps):
            choices = [("role", st) for st in state if not st["done"] and st["wait"] is None]
            choices += [("role", st) for st in state if not st["done"] and st["wait"] is not None
                        and self.ready(*st["wait"])]
            if self.mma_queue:
                choices.append(("mma", None))
            choices += [("tma", i) for i in range(len(self.tma))]
            if not choices:
                if all(st["done"] for st in state):
                    return
                blocked = {st["name"]: (st["wait"][0].name, st["wait"][1]) for st in state if not st["done"]}
                raise ProtocolError(f"deadlock: {blocked}")
            kind, x = self.rng.choice(choices)
            if kind == "role":
                x["wait"] = None
                self._advance(x)
            elif kind == "mma":
                op = self.mma_queue.pop(0)
                op()
            else:
                land = self.tma.pop(x)
                land()
        raise ProtocolError("step limit")

    def _advance(self, st):
        while True:
            try:
                cmd = next(st["gen"])
            except StopIteration:
                st["done"] = True
                return
            if cmd[0] == "wait":
                b, phase = cmd[1], cmd[2]
                if phase < 0 or self.ready(b, phase):
                    continue
                st["wait"] = (b, phase)
                return
            if cmd[0] == "yield":
                return
            raise ProtocolError(f"unknown command {cmd}")

    # ----------------------------------------------- async work and hazards
    def W(self, name, phase):
        return ("wait", self.bar(name), phase)

    def arrive(self, name, n=1):
        self.bar(name).arrive(n)

    def mma_s(self, gs, row):
        """S(gs) = Q K^T into buffer gs % 3; commit SFull."""
        def op():
            b = gs % STAGES
            if self.q_row != row:
                raise ProtocolError(f"S({gs}) read Q of row {self.q_row}, not {row}")
            if self.k_slot.get(b) != gs:
                raise ProtocolError(f"S({gs}) read K slot {b} holding {self.k_slot.get(b)}")
            held = self.s_state.get(b)
            if held is not None and held[0] == "P" and held[1] not in self.pv_done:
                raise ProtocolError(f"S({gs}) overwrote P({held[1]}) before its PV")
            self.s_state[b] = ("S", gs)
            self.s_done.add(gs)
            self.arrive(f"SFull{b}")
        self.mma_queue.append(op)

    def mma_pv(self, gb, row, first):
        """O (+)= P(gb) V(gb); the row's first PV overwrites O; commit PVDone."""
        def op():
            b = gb % STAGES
            if self.s_state.get(b) != ("P", gb):
                raise ProtocolError(f"PV({gb}) read buffer {b} holding {self.s_state.get(b)}")
            if self.v_slot.get(b) != ("V", gb):
                raise ProtocolError(f"PV({gb}) read V slot {b} holding {self.v_slot.get(b)}")
            if first:
                if self.o_row is not None and self.o_reads.get(self.o_row, 0) != EPILOGUE_WARPS:
                    raise ProtocolError(f"PV({gb}) overwrote O of row {self.o_row} before it was read")
                self.o_row = row
            elif self.o_row != row:
                raise ProtocolError(f"PV({gb}) of row {row} accumulated onto row {self.o_row}")
            self.pv_done.add(gb)
            self.arrive(f"PVDone{b}")
        self.mma_queue.append(op)

    def tma_q(self, row, g_prev_last):
        if g_prev_last is not None and g_prev_last not in self.s_done:
            raise ProtocolError(f"Q of row {row} loaded before S({g_prev_last}) was done")
        def land():
            self.q_row = row
            self.arrive("Q")
        self.tma.append(land)

    def tma_k(self, g):
        b = g % STAGES
        if g >= STAGES and (g - STAGES) not in self.s_done:
            raise ProtocolError(f"K({g}) loaded before S({g - STAGES}) was done")
        def land():
            self.k_slot[b] = g
            self.arrive(f"KFull{b}")
        self.tma.append(land)

    def tma_v(self, g):
        b = g % STAGES
        held = self.v_slot.get(b)
        if held is not None and held[0] == "O":
            raise ProtocolError(f"V({g}) loaded over the unstored O of row {held[1]}")
        if g >= STAGES and (g - STAGES) not in self.pv_done:
            raise ProtocolError(f"V({g}) loaded before PV({g - STAGES}) was done")
        def land():
            self.v_slot[b] = ("V", g)
            self.arrive(f"VFull{b}")
        self.tma.append(land)

    def epilogue(self, orow, gl):
        """One of warps 8-11 writes out its quarter of row orow's O."""
        yield self.W(f"LReady{self.lslot(orow)}", self.lphase(orow))
        if self.inv_l.get(self.lslot(orow), (None,))[0] != orow:
            raise ProtocolError(f"1/l of row {orow} read as {self.inv_l.get(self.lslot(orow))}")
        yield self.W(f"PVDone{gl % STAGES}", gl // STAGES)
        if self.o_row != orow or gl not in self.pv_done:
            raise ProtocolError(f"O of row {orow} read while O holds row {self.o_row}")
        self.o_reads[orow] = self.o_reads.get(orow, 0) + 1
        row_, readers = self.inv_l[self.lslot(orow)]
        self.inv_l[self.lslot(orow)] = (row_, readers + 1)
        b = gl % STAGES
        held = self.v_slot.get(b)
        if held not in (("V", gl), ("O", orow)):
            raise ProtocolError(f"O of row {orow} staged over {held}")
        self.v_slot[b] = ("O", orow)
        self.arrive("OFree")
        self.arrive(f"OStaged{orow % STAGES}")
        yield ("yield",)

    # ------------------------------------------------------------ the roles
    def setup(self):
        for b in range(STAGES):
            self.bar(f"PFull{b}", 8)
            self.bar(f"OStaged{b}", EPILOGUE_WARPS)
            for name in ("KFull", "VFull", "SFull", "PVDone"):
                self.bar(f"{name}{b}", 1)
        for slot in range(ROW_SLOTS):
            self.bar(f"RowFull{slot}", 1)
            self.bar(f"RowFree{slot}", ROW_USERS)
            self.bar(f"LReady{slot}", 8)
        self.bar("OFree", EPILOGUE_WARPS)
        self.bar("Q", 1)

    def read_desc(self, k):
        d = self.desc[k & 1]
        if d["k"] != k:
            raise ProtocolError(f"descriptor {k} read as {d['k']}")
        return d

    def scheduler(self):
        g = orow = 0
        owe = [None, None]
        k = 0
        while True:
            slot = k & 1
            if k >= ROW_SLOTS:
                yield self.W(f"RowFree{slot}", (k - ROW_SLOTS) // 2)
            if owe[slot] is not None:
                yield from self.epilogue(*owe[slot])
                owe[slot] = None
            r = self.tickets
            self.tickets += 1
            if r >= len(self.rows):
                self.desc[slot] = dict(k=k, r=-1, n=0)
                self.arrive(f"RowFull{slot}")
                break
            n = self.rows[r]
            self.desc[slot] = dict(k=k, r=r, n=n)
            self.arrive(f"RowFull{slot}")
            if n > 0:
                owe[slot] = (orow, g + n - 1)
                orow += 1
                g += n
            k += 1
            yield ("yield",)
        if k >= 1 and owe[(k - 1) & 1] is not None:
            yield from self.epilogue(*owe[(k - 1) & 1])

    def qk_loader(self):
        g = orow = 0
        owe = None
        k = 0
        while True:
            yield self.W(f"RowFull{k & 1}", k // 2)
            d = self.read_desc(k)
            if d["r"] < 0:
                break
            self.arrive(f"RowFree{k & 1}")
            n = d["n"]
            if n == 0:
                k += 1
                continue
            if g > 0:
                yield self.W(f"SFull{(g - 1) % STAGES}", (g - 1) // STAGES)
            self.tma_q(orow, g - 1 if g > 0 else None)
            for it in range(n):
                yield self.W(f"SFull{g % STAGES}", g // STAGES - 1)
                self.tma_k(g)
                g += 1
                if owe is not None and (it == 2 or it == n - 1):
                    yield from self.epilogue(*owe)
                    owe = None
            owe = (orow, g - 1)
            orow += 1
            k += 1
        if owe is not None:
            yield from self.epilogue(*owe)

    def v_loader(self):
        g = orows = 0
        pending = []

        def share(p):
            if not p["shared"]:
                p["shared"] = True
                yield from self.epilogue(p["idx"], p["last"])

        def store_o():
            p = pending[0]
            yield from share(p)
            yield self.W(f"OStaged{p['idx'] % STAGES}", p["idx"] // STAGES)
            if self.v_slot.get(p["last"] % STAGES) != ("O", p["idx"]):
                raise ProtocolError(f"stored {self.v_slot.get(p['last'] % STAGES)} as O of row {p['idx']}")
            if self.o_reads.get(p["idx"]) != EPILOGUE_WARPS:
                raise ProtocolError(f"O of row {p['idx']} stored with {self.o_reads.get(p['idx'])} quarters")
            self.stored.append(p["idx"])
            self.v_slot[p["last"] % STAGES] = None  # the store has read the tile
            pending.pop(0)

        k = 0
        while True:
            for p in list(pending):
                if p["k"] <= k - 2 and self.mutation != "late_v_share":
                    yield from share(p)
            yield self.W(f"RowFull{k & 1}", k // 2)
            d = self.read_desc(k)
            if d["r"] < 0:
                break
            self.arrive(f"RowFree{k & 1}")
            n = d["n"]
            if n == 0:
                k += 1
                continue
            for it in range(n):
                if pending and pending[0]["last"] + STAGES == g:
                    yield from store_o()
                yield self.W(f"PVDone{g % STAGES}", g // STAGES - 1)
                self.tma_v(g)
                g += 1
            pending.append(dict(last=g - 1, idx=orows, k=k, shared=False))
            orows += 1
            k += 1
        while pending:
            yield from store_o()

    def mma_issuer(self):
        g = qrows = orow = 0
        owe = None
        ahead = 0
        k = 0
        while True:
            yield self.W(f"RowFull{k & 1}", k // 2)
            d = self.read_desc(k)
            if d["r"] < 0:
                break
            self.arrive(f"RowFree{k & 1}")
            n = d["n"]
            if n == 0:
                k += 1
                continue
            row = orow
            orow += 1
            if ahead == 0:
                yield self.W("Q", qrows)
                qrows += 1
            for it in range(ahead, min(STAGES, n)):
                yield self.W(f"KFull{(g + it) % STAGES}", (g + it) // STAGES)
                self.mma_s(g + it, row)
            ahead = 0
            if owe is not None:
                yield from self.epilogue(*owe)
                if self.mutation != "no_ofree_wait":
                    yield self.W("OFree", owe[0])
                owe = None
            for it in range(n):
                gb = g + it
                yield self.W(f"PFull{gb % STAGES}", gb // STAGES)
                yield self.W(f"VFull{gb % STAGES}", gb // STAGES)
                self.mma_pv(gb, row, it == 0)
                if it + STAGES < n:
                    gs = gb + STAGES
                    yield self.W(f"KFull{gs % STAGES}", gs // STAGES)
                    self.mma_s(gs, row)
                # before the last PV: the next row's first S products, if its
                # descriptor is out and its Q has landed (checks, no waits)
                if it == n - 2 and self.mutation != "no_early_s":
                    k1 = k + 1
                    if self.ready(self.bar(f"RowFull{k1 & 1}"), k1 // 2):
                        d1 = self.read_desc(k1)
                        if d1["r"] >= 0 and d1["n"] > 0 and self.ready(self.bar("Q"), qrows):
                            qrows += 1
                            self.early += 1
                            ahead = min(2, d1["n"])
                            for a in range(ahead):
                                gs = g + n + a
                                yield self.W(f"KFull{gs % STAGES}", gs // STAGES)
                                self.mma_s(gs, row + 1)
            owe = (row, g + n - 1)
            g += n
            k += 1
        if owe is not None:
            yield from self.epilogue(*owe)

    def softmax(self, group, reref):
        """Warps 0-3 (group 0) or 4-7 (group 1), arriving 4 at a time."""
        g = orows = 0
        k = 0
        while True:
            yield self.W(f"RowFull{k & 1}", k // 2)
            d = self.read_desc(k)
            if d["r"] < 0:
                break
            n = d["n"]
            if group == 1 and n > 1:
                yield self.W(f"SFull{(g + 1) % STAGES}", (g + 1) // STAGES)
            for it in range(n):
                gb = g + it
                b = gb % STAGES
                yield self.W(f"SFull{b}", gb // STAGES)
                held = self.s_state.get(b)
                if held not in (("S", gb), ("P", gb)):
                    raise ProtocolError(f"softmax read S({gb}) from buffer {b} holding {held}")
                if it > 0 and self.rng.random() < reref:
                    # a new reference: O is rescaled after PV(gb - 1)
                    yield self.W(f"PVDone{(gb - 1) % STAGES}", (gb - 1) // STAGES)
                    if self.o_row != orows:
                        raise ProtocolError(f"rescaled O of row {self.o_row} in row {orows}")
                self.s_state[b] = ("P", gb)
                self.arrive(f"PFull{b}", GROUP_WARPS)
                yield ("yield",)
            if n > 0:
                ls = self.lslot(orows)
                old = self.inv_l.get(ls)
                if old is not None and old[0] != orows and old[1] != EPILOGUE_WARPS:
                    raise ProtocolError(f"1/l of row {orows} overwrote row {old[0]} before it was read")
                if old is None or old[0] != orows:
                    self.inv_l[ls] = (orows, 0)
                self.arrive(f"LReady{ls}", GROUP_WARPS)
                orows += 1
            self.arrive(f"RowFree{k & 1}", GROUP_WARPS)
            g += n
            k += 1


def simulate(rows, seed, reref=0.05, mutation=None):
    sim = Sim(rows, seed)
    sim.mutation = mutation
    sim.stored = []
    sim.setup()
    roles = [("scheduler", sim.scheduler()), ("qk_loader", sim.qk_loader()),
             ("v_loader", sim.v_loader()), ("mma", sim.mma_issuer()),
             ("softmax0", sim.softmax(0, reref)), ("softmax1", sim.softmax(1, reref))]
    sim.run(roles)
    expected = list(range(sum(1 for n in rows if n > 0)))
    if sim.stored != expected:
        raise ProtocolError(f"stored rows {sim.stored}, expected {expected}")
    return sim


def _rows(rng, kinds):
    return [rng.choice(kinds) for _ in range(rng.randint(1, 14))]


@pytest.mark.parametrize("kinds", [
    (0, 1, 1, 2, 3, 4, 5, 8, 13),      # mixed lengths with empty rows
    (1,),                               # one-block rows: the tightest row hand-over
    (1, 2),                             # rows shorter than the rings
    (3, 4, 6, 20),                      # rows longer than the rings
])
def test_protocol_runs_clean(kinds):
    rng = random.Random(sum(kinds) * 131 + len(kinds))
    early = 0
    for seed in range(150):
        early += simulate(_rows(rng, kinds), seed).early
    # the early S issue before a row's last PV is exercised (rows of >= 2 blocks)
    assert early > 0 or max(kinds) < 2


@pytest.mark.parametrize("mutation,kinds", [
    ("single_inv_l", (1, 2, 3)),         # 1/l overwritten (LReady two phases ahead)
    ("late_v_share", (1,)),             # the V loader waits for a descriptor its share blocks
    ("no_ofree_wait", (1, 2, 5)),       # O overwritten before it is written out
])
def test_protocol_model_catches_planted_mistakes(mutation, kinds):
    rng = random.Random(7)
    caught = 0
    for seed in range(300):
        try:
            simulate(_rows(rng, kinds), seed, mutation=mutation)
        except ProtocolError:
            caught += 1
    assert caught > 0, mutation
