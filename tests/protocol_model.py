"""A model of the mbarrier protocol of the d = 128 backward main kernel
(io_aware_exact_30_b200/csrc/bwd128_sm100.cuh), for checking it on the CPU
under many random schedules.  Test infrastructure only.

Each role of the kernel is a generator that yields the same sequence of
barrier operations, with the same barriers, arrival counts and phase indices,
as the kernel's code; asynchronous work (TMA loads, MMAs and their commits,
the bulk stores) is queued and completed at random later points, in any order
the hardware allows (`AsyncWork`): a commit after everything its thread issued
before it, an MMA after the earlier MMAs of its thread on the same
accumulator, a copy at any time.  Buffers carry a version tag: every read
states the version it must see, every write sets one.  The work-item stream
(cluster launch control responses in two slots, a full and an empty barrier
each) is modelled for every role.  Each schedule gives every role a random
speed, so that some fall far behind the others.

Groups of threads that run the same code are modelled by a few agents each
(two per column half of the compute warps, two dQ warps), so the barriers'
arrival counts are the number of modelled agents, not of threads.

The checker reports:
  * a barrier test for phase k while the barrier is not in phase k or k + 1
    (the parity test would return a wrong answer: ahead, it succeeds on phase
    k - 2; two behind, it waits for a phase that needs the waiter itself),
  * an arrival that does not land in the phase it is meant for,
  * a read that sees another version than the one it needs,
  * a schedule in which nothing can move before every role has finished.

`Variant` switches reproduce protocol mistakes that were made while building
the kernel, so the tests can show that the checker catches each of them.
"""

import random
from dataclasses import dataclass, field


class ProtocolError(AssertionError):
    pass


@dataclass
class Variant:
    single_srd: bool = False      # one barrier (not one per S buffer) for the shared S^T read
    single_dsf: bool = False      # one barrier (not one per dS^T buffer) for dS^T ready
    epilogue_tile_wait: bool = False  # epilogue waits the last tile's staging-full barrier, not DQD
    no_dpe: bool = False          # dP^T(g) waits for dS^T(g-1) instead of the dP^T release
    # work items dealt in a fixed order (no mask) instead of taken through
    # cluster launch control responses (causal)
    static_items: bool = False
    clc_no_empty_wait: bool = False   # request into a slot without its consumers' release
    # an item without query tiles arrives DQD without waiting for the previous
    # item's epilogue (the mistake the checker found in the block-sparse walk)
    empty_item_no_epf_wait: bool = False
    # issuer B commits an empty item's FIN and KVE without waiting (the same)
    empty_item_no_b_wait: bool = False
    # a staging half is released without waiting for the previous tile's
    # reduction to have read it
    stg_half_no_read_wait: bool = False


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.completed = name, count, 0, 0

    def arrive(self, use):
        if self.completed != use:
            raise ProtocolError(f"{self.name}: arrival for phase {use} while in phase "
                                f"{self.completed}")
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.completed += 1

    def test(self, k):
        """The hardware's parity test for phase k, checked against its meaning."""
        if self.completed not in (k, k + 1):
            raise ProtocolError(f"{self.name}: test for phase {k} while in phase "
                                f"{self.completed}")
        return self.completed == k + 1


@dataclass
class World:
    bars: dict = field(default_factory=dict)
    buf: dict = field(default_factory=dict)

    def bar(self, name, count=1):
        if name not in self.bars:
            self.bars[name] = Barrier(name, count)
        return self.bars[name]

    def read(self, key, want):
        have = self.buf.get(key)
        if have != want:
            raise ProtocolError(f"read of {key}: wants {want}, holds {have}")

    def write(self, key, value):
        self.buf[key] = value


class AsyncWork:
    """Asynchronous operations in flight, per issuing unit (a TMA producer, an
    MMA-issuing thread, the bulk-store unit), completed in an order the
    hardware allows.  Each operation carries a tag:
      * "commit" (the default): a tcgen05.commit, or a bulk-group arrival.  It
        completes after every earlier operation of its unit.
      * "tma": a copy, which may complete at any time.
      * any other tag names the accumulator of a group of MMAs.  tcgen05.mma
        instructions of one thread are pipelined (kept in order) only when they
        share the accumulator and shape, so the group completes after the
        earlier groups of its unit on the same accumulator, in any order
        relative to the rest.
    With in_order=True every unit completes in issue order instead."""

    def __init__(self, in_order=False):
        self.units = {}
        self.in_order = in_order

    def push(self, unit, fn, tag="commit"):
        self.units.setdefault(unit, []).append((fn, tag))

    def pending(self):
        return any(self.units.values())

    def _eligible(self, ops, i):
        tag = ops[i][1]
        if self.in_order or tag == "commit":
            return i == 0
        if tag == "tma":
            return True
        return all(t != tag for _, t in ops[:i])

    def ready(self):
        return [(u, i) for u, ops in self.units.items() for i in range(len(ops))
                if self._eligible(ops, i)]

    def complete(self, unit, i):
        fn, _ = self.units[unit].pop(i)
        fn()


def item_request(world, t, dynamic, wait_empty=True):
    """The producer, once work item t's loads are issued, asks for the item
    after it (ItemStream::request): response k = t + 1 goes to slot k & 1,
    whose previous response every consumer must have read first."""
    if not dynamic:
        return
    k, slot, u = t + 1, (t + 1) & 1, t >> 1

    if u >= 1 and wait_empty:
        yield ("wait", [(f"CLCE{slot}", u - 1)])

    def land(k=k, slot=slot, u=u):
        world.write(("CLC", slot), k)
        world.bar(f"CLCF{slot}").arrive(u)
    yield ("async", "clc", land, "tma")


def item_advance(world, t, dynamic):
    """Every role (one agent of it) after work item t: waits for response
    t + 1, reads it and frees its slot (ItemStream::advance)."""
    if not dynamic:
        return
    k, slot, u = t + 1, (t + 1) & 1, t >> 1
    yield ("wait", [(f"CLCF{slot}", u)])
    yield ("read", ("CLC", slot), k)
    yield ("arrive", f"CLCE{slot}", u)


def run_roles(world, roles, seed, in_order=False, max_steps=200000):
    """Runs the roles (generators of operations) and their asynchronous work
    under one random schedule; raises ProtocolError on a violation or a
    deadlock.  Each schedule draws a speed for every role and for the
    asynchronous units, so that some roles lag far behind the others (a
    uniform choice at every step rarely lets one fall more than a few steps
    behind)."""
    rng = random.Random(seed)
    speed = {name: rng.choice((0.02, 0.2, 1.0, 1.0, 1.0, 4.0)) for name in roles}
    work_speed = rng.choice((0.1, 1.0, 1.0, 4.0))
    nxt = {name: None for name in roles}       # pending operation of each role
    work = AsyncWork(in_order)
    done = set()

    def advance(name):
        try:
            nxt[name] = next(roles[name])
        except StopIteration:
            nxt[name] = None
            done.add(name)

    def ready(op):
        # the kernel issues every test of a grouped wait before it looks at
        # any result, so every test is checked
        return all([world.bar(b).test(k) for b, k in op[1]])

    for name in roles:
        advance(name)
    for _ in range(max_steps):
        if len(done) == len(roles) and not work.pending():
            return
        choices = [("role", n) for n, op in nxt.items()
                   if op is not None and (op[0] != "wait" or ready(op))]
        choices += [("work", r) for r in work.ready()]
        if not choices:
            raise ProtocolError("deadlock: pending " + str(
                [(n, o[0], o[1] if o[0] == "wait" else "") for n, o in nxt.items() if o]))
        weights = [speed[c[1]] if c[0] == "role" else work_speed for c in choices]
        kind, name = rng.choices(choices, weights)[0]
        if kind == "work":
            work.complete(*name)
            continue
        op = nxt[name]
        if op[0] == "arrive":
            world.bar(op[1]).arrive(op[2])
        elif op[0] == "async":
            work.push(op[1], op[2], op[3] if len(op) > 3 else "commit")
        elif op[0] == "read":
            world.read(op[1], op[2])
        elif op[0] == "write":
            world.write(op[1], op[2])
        advance(name)
    raise ProtocolError("schedule did not finish")


ST = 3          # Q / dO / statistics stages
NCOMP = 4       # compute agents: (half, quarter) for half in 0,1 and quarter in 0,1
NDQ = 2         # dQ agents; agent 0 holds the reduction issuer


# ---------------------------------------------------------------------------
# Roles.  Operations yielded:
#   ("wait", [(bar, k), ...])          all tests must pass (tested together)
#   ("arrive", bar, use)
#   ("async", unit, fn[, tag])         fn() runs when the unit completes it
#                                      (completion order: AsyncWork)
#   ("read", key, version) / ("write", key, version)   a role's own access
# Every operation of a role is a step of its own, so any other step can fall
# between two of them; the effects of an MMA or a copy happen at once when it
# completes.  `plan` lists the number of 64-query tiles of each work item
# of one CTA, in the order the CTA takes them.
# ---------------------------------------------------------------------------

def producer(plan, v):
    g = 0
    for item, n_it in enumerate(plan):
        def load_tile(g):
            s, n = g % ST, g // ST
            yield ("wait", [(f"QE{s}", n - 1)])

            def land(g=g, s=s, n=n):
                W.write(("Q", s), g)
                W.write(("DO", s), g)
                W.write(("LD", s), g)
                W.bar(f"QF{s}").arrive(n)
            yield ("async", "tma", land, "tma")
        pre = min(ST, n_it)
        for _ in range(pre):
            yield from load_tile(g)
            g += 1
        if item > 0:
            yield ("wait", [("KVE", item - 1)])

        def land_kv(item=item):
            W.write("K", item)
            W.write("V", item)
            W.bar("KV").arrive(item)
        yield ("async", "tma", land_kv, "tma")
        for _ in range(pre, n_it):
            yield from load_tile(g)
            g += 1
        yield from item_request(W, item, not v.static_items, not v.clc_no_empty_wait)
        yield from item_advance(W, item, not v.static_items)


def issuer_a(plan, v):
    g = 0
    for item, n_it in enumerate(plan):
        # an item without query tiles (block-sparse: no query tile marked for
        # its key tile) only waits for its K and V to land
        waits = [("KV", item)]
        if n_it > 0:
            waits.append((f"QF{g % ST}", g // ST))
            if g >= 2:
                waits.append((f"DVD{g & 1}", (g - 2) >> 1))
        yield ("wait", waits)
        if n_it > 0:
            yield from mma_s(g, item)
        for it in range(n_it):
            s, g1, more = g % ST, g + 1, it + 1 < n_it
            waits = []
            if g >= 1:
                waits.append(("DSF0" if v.single_dsf else f"DSF{(g - 1) & 1}",
                              (g - 1) if v.single_dsf else (g - 1) >> 1) if v.no_dpe
                             else ("DPE", g - 1))
            if more:
                waits.append((f"QF{g1 % ST}", g1 // ST))
                if g1 >= 2:
                    waits.append((f"DVD{g1 & 1}", (g1 - 2) >> 1))
            yield ("wait", waits)

            def dp(g=g, s=s, item=item):
                W.read("V", item)
                W.read(("DO", s), g)
                W.write("DP", g)
            yield ("async", "A", dp, "DP")
            yield ("async", "A", lambda g=g: W.bar("DPF").arrive(g))
            yield ("async", "A", lambda s=s, g=g: W.bar(f"QE{s}", 2).arrive(g // ST))
            if more:
                yield from mma_s(g1, item)
            g += 1
        yield ("async", "A", lambda item=item: W.bar("KVE", 2).arrive(item))
        yield from item_advance(W, item, not v.static_items)


def mma_s(g, item):
    s = g % ST

    def run(g=g, s=s, item=item):
        W.read("K", item)
        W.read(("Q", s), g)
        for q in range(2):
            for r in ("R0", "R1", "R2", "R3"):   # S^T columns 0-15, 16-31, 32-47, 48-63
                W.write(("S", g & 1, q, r), ("S", g))
    yield ("async", "A", run, f"S{g & 1}")
    yield ("async", "A", lambda g=g: W.bar(f"SF{g & 1}").arrive(g >> 1))


def issuer_b(plan, v):
    g = 0
    for item, n_it in enumerate(plan):
        for it in range(n_it):
            s = g % ST
            waits = [(f"PTF{g & 1}", g >> 1), (f"QF{s}", g // ST)]
            if it == 0 and item > 0:
                waits.append(("ACCE", item - 1))
            yield ("wait", waits)

            def dv(g=g, s=s, item=item, it=it):
                for q in range(2):
                    W.read(("S", g & 1, q, "R0"), ("P", g))
                    W.read(("S", g & 1, q, "R1"), ("P", g))
                W.read(("DO", s), g)
                W.write("DVACC", (item, it + 1))
            yield ("async", "B", dv, "DV")
            yield ("async", "B", lambda g=g: W.bar(f"DVD{g & 1}").arrive(g >> 1))
            dsf = ("DSF0", g) if v.single_dsf else (f"DSF{g & 1}", g >> 1)
            waits = [dsf]
            if g >= 1:
                waits.append(("DQE", g - 1))
            if it == 0:
                waits.append(("KV", item))
            yield ("wait", waits)

            def dk(g=g, s=s, it=it, item=item):
                for h in range(2):
                    W.read(("DS", g & 1, h), g)
                W.read(("Q", s), g)
                W.write("DKACC", (item, it + 1))

            def dq(g=g, item=item):
                for h in range(2):
                    W.read(("DS", g & 1, h), g)
                W.read("K", item)
                W.write("DQ", g)
            yield ("async", "B", dk, "DK")
            yield ("async", "B", dq, "DQ")
            yield ("async", "B", lambda s=s, g=g: W.bar(f"QE{s}", 2).arrive(g // ST))
            yield ("async", "B", lambda g=g: W.bar("DQF").arrive(g))
            yield ("async", "B", lambda g=g: W.bar(f"DSTE{g & 1}").arrive(g >> 1))
            g += 1
        if n_it == 0 and not v.empty_item_no_b_wait:
            # An item without query tiles issues no MMA.  Its FIN and KVE commits
            # wait for the previous item's accumulator release (the compute
            # warps have passed the previous FIN) and for this item's K and V
            # (the producer has seen the previous KVE complete): otherwise
            # consecutive such items run both barriers two phases ahead.
            waits = [("KV", item)]
            if item > 0:
                waits.append(("ACCE", item - 1))
            yield ("wait", waits)
        yield ("async", "B", lambda item=item: W.bar("FIN").arrive(item))
        yield ("async", "B", lambda item=item: W.bar("KVE", 2).arrive(item))
        yield from item_advance(W, item, not v.static_items)


def compute(agent, plan, v):
    half, q = agent // 2, agent % 2
    g = 0
    for item, n_it in enumerate(plan):
        for it in range(n_it):
            s, b = g % ST, g & 1
            yield ("wait", [(f"QF{s}", g // ST)])
            yield ("wait", [(f"SF{b}", g >> 1)])
            yield ("read", ("LD", s), g)
            srd = ("SRD0", g) if v.single_srd else (f"SRD{b}", g >> 1)
            if half == 0:
                yield ("read", ("S", b, q, "R0"), ("S", g))
                yield ("read", ("S", b, q, "R1"), ("S", g))
                yield ("arrive", srd[0], srd[1])
                yield ("write", ("S", b, q, "R0"), ("P", g))
            else:
                yield ("read", ("S", b, q, "R2"), ("S", g))
                yield ("read", ("S", b, q, "R3"), ("S", g))
                yield ("wait", [srd])
                yield ("write", ("S", b, q, "R1"), ("P", g))
            yield ("arrive", f"PTF{b}", g >> 1)
            waits = [("DPF", g)]
            if g >= 2:
                waits.append((f"DSTE{b}", (g - 2) >> 1))
            yield ("wait", waits)
            yield ("read", "DP", g)
            yield ("read", ("LD", s), g)
            if not v.no_dpe:
                yield ("arrive", "DPE", g)
            yield ("write", ("DS", b, half), g)
            dsf = ("DSF0", g) if v.single_dsf else (f"DSF{b}", g >> 1)
            yield ("arrive", dsf[0], dsf[1])
            g += 1
        # epilogue
        yield ("wait", [("FIN", item)])
        if n_it > 0:
            yield ("read", "DVACC", (item, n_it))
            yield ("read", "DKACC", (item, n_it))
        # (an item without query tiles reads stale accumulators and writes zeros)
        yield ("arrive", "ACCE", item)
        if v.epilogue_tile_wait:
            yield ("wait", [("STGF1", g - 1)])
        else:
            yield ("wait", [("DQD", item)])
        # half h stages its 64 columns: dV into the staging tile's h-th 16 KB,
        # dK into dS^T buffer h (both column halves of the tile loop's layout)
        yield ("write", ("STG", half), ("dV", item))
        yield ("write", ("DS", half, 0), ("dK", item))
        yield ("write", ("DS", half, 1), ("dK", item))
        yield ("arrive", "EPS", item)
        if agent == 0:
            yield ("wait", [("EPS", item)])

            def store(item=item):
                for h in range(2):
                    W.read(("STG", h), ("dV", item))
                    W.read(("DS", h, 0), ("dK", item))
                    W.read(("DS", h, 1), ("dK", item))
                W.bar("EPF").arrive(item)
            yield ("async", "store", store)
        yield ("wait", [("EPF", item)])
        yield from item_advance(W, item, not v.static_items)


def dq_role(agent, plan, v):
    g = 0
    for item, n_it in enumerate(plan):
        for it in range(n_it):
            yield ("wait", [("DQF", g)])
            yield ("read", "DQ", g)
            yield ("arrive", "DQE", g)
            if SINGLE_STAGING:
                # the block-sparse instantiation: the whole 32 KB tile, one bulk
                # reduction, whose read the issuing lane waits for at once
                if g >= 1:
                    yield ("wait", [("STGE0", g - 1)])
                for h in range(2):
                    yield ("write", ("STG", h), ("dQ", g))
                yield ("arrive", "STGF0", g)
                if agent == 0:
                    yield ("wait", [("STGF0", g)])
                    for h in range(2):
                        yield ("read", ("STG", h), ("dQ", g))
                    yield ("arrive", "STGE0", g)
                    if it + 1 == n_it:
                        yield ("arrive", "DQD", item)
                g += 1
                continue
            # the staging tile in two 16 KB halves (32 queries each), each sent by
            # its own bulk reduction; agent 0 (the issuing lane) releases a half
            # once the previous tile's reduction of it has read it
            for h in range(2):
                if g >= 1:
                    if agent == 0:
                        if not v.stg_half_no_read_wait:
                            yield ("wait", [(f"RD{h}", g - 1)])
                        yield ("arrive", f"STGE{h}", g - 1)
                    yield ("wait", [(f"STGE{h}", g - 1)])
                # each dQ warp writes its feature column of the half
                yield ("write", ("STG", h), ("dQ", g))
                yield ("arrive", f"STGF{h}", g)
                if agent == 0:
                    yield ("wait", [(f"STGF{h}", g)])

                    def reduce(h=h, g=g):
                        W.read(("STG", h), ("dQ", g))
                        W.bar(f"RD{h}").arrive(g)
                    yield ("async", "bulk", reduce, "tma")
            if agent == 0 and it + 1 == n_it:
                # the epilogue reuses the staging tile once both reductions read it
                yield ("wait", [("RD0", g), ("RD1", g)])
                yield ("arrive", "DQD", item)
            g += 1
        if n_it == 0 and agent == 0:
            # An item without query tiles leaves the staging tile as it was.  Its
            # DQD arrival waits for the previous item's epilogue (EPF), which
            # follows the compute warps' wait for the previous DQD: otherwise
            # consecutive such items run DQD two phases ahead of that wait.
            if item > 0 and not v.empty_item_no_epf_wait:
                yield ("wait", [("EPF", item - 1)])
            yield ("arrive", "DQD", item)
        yield from item_advance(W, item, not v.static_items)


W = None  # the world of the schedule being run (the roles read it as a global)
SINGLE_STAGING = False  # dQ staging as one 32 KB tile (block-sparse) or two halves


def run_schedule(plan, seed, variant=None, max_steps=200000, in_order=False,
                 single_staging=False):
    """Runs one random schedule of one CTA working through `plan`; raises
    ProtocolError on a violation or a deadlock.  in_order: complete each
    unit's asynchronous work in issue order (a narrower set of schedules).
    single_staging: the block-sparse instantiation's dQ staging (one 32 KB
    tile per tile, one reduction) instead of the dense one's two halves."""
    global W, SINGLE_STAGING
    SINGLE_STAGING = single_staging
    v = variant or Variant()
    W = World()
    counts = {"KVE": 2, "ACCE": NCOMP, "PTF0": NCOMP, "PTF1": NCOMP, "DSF0": NCOMP,
              "DSF1": NCOMP, "DPE": NCOMP, "SRD0": NCOMP // 2, "SRD1": NCOMP // 2,
              "EPS": NCOMP, "DQE": NDQ, "STGF0": NDQ, "STGF1": NDQ}
    for s in range(ST):
        counts[f"QE{s}"] = 2
    if v.single_dsf:
        counts["DSF0"] = NCOMP
    # one arrival per modelled agent frees a response slot
    counts["CLCE0"] = counts["CLCE1"] = 3 + NCOMP + NDQ
    for name, c in counts.items():
        W.bar(name, c)
    roles = {"prod": producer(plan, v), "A": issuer_a(plan, v), "B": issuer_b(plan, v)}
    for a in range(NCOMP):
        roles[f"comp{a}"] = compute(a, plan, v)
    for a in range(NDQ):
        roles[f"dq{a}"] = dq_role(a, plan, v)
    run_roles(W, roles, seed, in_order, max_steps)
