"""A model of the mbarrier protocol of the d = 64 backward main kernel
(attn_bwd_main_kernel in io_aware_exact_30_b200/csrc/bwd_sm100.cuh), checked
on the CPU under random schedules with the rules of protocol_model.py.  Test
infrastructure only.

One CTA works on one 128-key tile (or, in the `persistent` design variant,
on a list of them, taking each K/V pair once the previous item's MMAs have
released the last: KVE, with the tile rings and barrier phases running on
across items and the accumulators reused after the epilogue read them: ACCE):
the producer loads K/V and streams
128-query tiles of Q (with the row statistics) and dO through two stages each;
one thread issues, per tile, S^T, dP^T, dV, then dK and dQ (in that order,
each group after its barriers); the compute warps (two column halves x row
quarters, modelled as four agents) write P^T over S^T (half 1 over columns half
0 reads, after the shared-read barrier), dS^T into shared memory, and drain dQ
into the accumulator.  After the epilogue, every agent arrives at ENDA; agent
0 counts the item on its head and publishes whether this CTA completed the
head, and all read that flag after ENDB (the counter itself and the dQ
conversion it gates are outside the model).  Asynchronous work completes in any order the hardware
allows (protocol_model.AsyncWork).
"""


from protocol_model import ProtocolError, World, item_advance, item_request, run_roles

QST = DOST = 2
NCOMP = 4    # (half, quarter) agents


class Variant:
    def __init__(self, no_srd=False, no_dsf_wait=False, no_acce=False, s_without_dvd_wait=False,
                 static_items=False, flag_without_endb=False):
        self.no_srd = no_srd              # mistake: half 1 writes P^T without the SRD wait
        self.no_dsf_wait = no_dsf_wait    # mistake: dK / dQ issued without waiting for dS^T
        # mistake: S^T(g+1) issued without waiting for dV(g), which reads P^T
        # from the same columns, trusting the issue order of one thread's MMAs
        self.s_without_dvd_wait = s_without_dvd_wait
        # persistent design: items dealt in a fixed order (no mask) instead of
        # taken through cluster launch control responses
        self.static_items = static_items
        # mistake: read the head-completion flag without waiting for ENDB
        self.flag_without_endb = flag_without_endb
        # persistent: the next item's first dV without the accumulator-release
        # wait.  Not a mistake: the compute warps read dV/dK in the epilogue
        # before they write the next item's P^T, which that dV waits for, so
        # the wait only guards the order.
        self.no_acce = no_acce


W = None
persistent = False  # the schedule runs a list of items (the persistent design)


def producer(plan, v):
    g = 0

    def load_tile(g):
        qs, qn, ds, dn = g % QST, g // QST, g % DOST, g // DOST
        yield ("wait", [(f"QE{qs}", qn - 1)])

        def land_q(g=g, qs=qs, qn=qn):
            W.write(("Q", qs), g)
            W.write(("LD", qs), g)
            W.bar(f"QF{qs}").arrive(qn)
        yield ("async", "tma", land_q, "tma")
        yield ("wait", [(f"DOE{ds}", dn - 1)])

        def land_do(g=g, ds=ds, dn=dn):
            W.write(("DO", ds), g)
            W.bar(f"DOF{ds}").arrive(dn)
        yield ("async", "tma", land_do, "tma")

    for item, n_it in enumerate(plan):
        # the persistent design loads an item's first query tiles ahead of its
        # K/V, which wait until the previous item's MMAs are done with K and V
        pre = min(QST, n_it) if persistent else 0
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
        if persistent:
            yield from item_request(W, item, not v.static_items)
            yield from item_advance(W, item, not v.static_items)


def issuer(plan, v):
    g = 0
    for item, n_it in enumerate(plan):
        yield ("wait", [("KV", item)])
        for it in range(n_it):
            qs, qn, ds, dn = g % QST, g // QST, g % DOST, g // DOST
            waits = [(f"QF{qs}", qn)]
            if g > 0 and not v.s_without_dvd_wait:
                waits.append(("DVD", g - 1))
            yield ("wait", waits)

            def s_mma(g=g, qs=qs, item=item):
                W.read("K", item)
                W.read(("Q", qs), g)
                for q in range(2):
                    for r in ("R0", "R1", "R2", "R3"):
                        W.write(("S", q, r), ("S", g))
            yield ("async", "mma", s_mma, "S")
            yield ("async", "mma", lambda g=g: W.bar("SF").arrive(g))
            yield ("wait", [(f"DOF{ds}", dn)])

            def dp_mma(g=g, ds=ds, item=item):
                W.read("V", item)
                W.read(("DO", ds), g)
                W.write("DP", g)
            yield ("async", "mma", dp_mma, "DP")
            yield ("async", "mma", lambda g=g: W.bar("DPF").arrive(g))
            waits = [("PTF", g)]
            if it == 0 and item > 0 and not v.no_acce:
                waits.append(("ACCE", item - 1))
            yield ("wait", waits)

            def dv_mma(g=g, ds=ds, item=item, it=it):
                for q in range(2):
                    W.read(("S", q, "R0"), ("P", g))
                    W.read(("S", q, "R1"), ("P", g))
                W.read(("DO", ds), g)
                W.write("DVACC", (item, it + 1))
            yield ("async", "mma", dv_mma, "DV")
            yield ("async", "mma", lambda g=g: W.bar("DVD").arrive(g))
            yield ("async", "mma", lambda ds=ds, dn=dn: W.bar(f"DOE{ds}").arrive(dn))
            waits = [] if v.no_dsf_wait else [("DSF", g)]
            if g > 0:
                waits.append(("DQE", g - 1))
            if waits:
                yield ("wait", waits)

            def dk_mma(g=g, qs=qs, item=item, it=it):
                for h in range(2):
                    W.read(("DS", h), g)
                W.read(("Q", qs), g)
                W.write("DKACC", (item, it + 1))

            def dq_mma(g=g, item=item):
                for h in range(2):
                    W.read(("DS", h), g)
                W.read("K", item)
                W.write("DQ", g)
            yield ("async", "mma", dk_mma, "DK")
            yield ("async", "mma", dq_mma, "DQ")
            yield ("async", "mma", lambda qs=qs, qn=qn: W.bar(f"QE{qs}").arrive(qn))
            yield ("async", "mma", lambda g=g: W.bar("DQF").arrive(g))
            g += 1
        yield ("async", "mma", lambda item=item: W.bar("FIN").arrive(item))
        yield ("async", "mma", lambda item=item: W.bar("KVE").arrive(item))
        if persistent:
            yield from item_advance(W, item, not v.static_items)


def compute(agent, plan, v):
    half, q = agent // 2, agent % 2
    g = 0
    for item, n_it in enumerate(plan):
        for it in range(n_it):
            qs, qn = g % QST, g // QST
            yield ("wait", [(f"QF{qs}", qn)])
            yield ("wait", [("SF", g)])
            for r in (("R0", "R1") if half == 0 else ("R2", "R3")):
                yield ("read", ("S", q, r), ("S", g))
            yield ("read", ("LD", qs), g)
            if half == 0:
                if not v.no_srd:
                    yield ("arrive", "SRD", g)
                yield ("write", ("S", q, "R0"), ("P", g))
            else:
                if not v.no_srd:
                    yield ("wait", [("SRD", g)])
                yield ("write", ("S", q, "R1"), ("P", g))
            yield ("arrive", "PTF", g)
            yield ("wait", [("DPF", g)])
            yield ("read", "DP", g)
            yield ("read", ("LD", qs), g)
            yield ("write", ("DS", half), g)
            yield ("arrive", "DSF", g)
            yield ("wait", [("DQF", g)])
            yield ("read", "DQ", g)
            yield ("arrive", "DQE", g)
            g += 1
        yield ("wait", [("FIN", item)])
        yield ("read", "DVACC", (item, n_it))
        yield ("read", "DKACC", (item, n_it))
        yield ("arrive", "ACCE", item)
        # the end-of-item handshake: every agent has written its dK/dV rows
        # (ENDA); agent 0 counts the item on its head and publishes whether the
        # CTA finished the head (the flag); all read the flag after ENDB
        yield ("arrive", "ENDA", item)
        if agent == 0:
            yield ("wait", [("ENDA", item)])
            yield ("write", "LASTFLAG", item)
            yield ("arrive", "ENDB", item)
        if not v.flag_without_endb:
            yield ("wait", [("ENDB", item)])
        yield ("read", "LASTFLAG", item)
        if persistent:
            yield from item_advance(W, item, not v.static_items)


def run_schedule(plan, seed, variant=None, max_steps=200000, in_order=False):
    """plan: the number of 128-query tiles of one work item (an int: the kernel
    as it is, one item per CTA), or of each item a persistent CTA takes.
    in_order: complete each unit's asynchronous work in issue order."""
    global W, persistent
    v = variant or Variant()
    persistent = not isinstance(plan, int)
    plan = [plan] if isinstance(plan, int) else list(plan)
    W = World()
    for name, c in {"PTF": NCOMP, "DSF": NCOMP, "DQE": NCOMP, "SRD": NCOMP // 2,
                    "ACCE": NCOMP, "ENDA": NCOMP}.items():
        W.bar(name, c)
    W.bar("CLCE0", 2 + NCOMP)
    W.bar("CLCE1", 2 + NCOMP)
    roles = {"prod": producer(plan, v), "mma": issuer(plan, v)}
    for a in range(NCOMP):
        roles[f"comp{a}"] = compute(a, plan, v)
    run_roles(W, roles, seed, in_order, max_steps)
