"""A model of the mbarrier protocol of the d = 64 backward main kernel
(attn_bwd_main_kernel in io_aware_exact_30_b200/csrc/bwd_sm100.cuh), checked
on the CPU under random schedules with the rules of protocol_model.py.  Test
infrastructure only.

One CTA works on one 128-key tile: the producer loads K/V and streams 128-query
tiles of Q (with the row statistics) and dO through two stages each; one thread
issues, per tile g, S^T, dP^T, dV, then dK and dQ (dQ into tensor-memory
buffer g mod 2), each group after its barriers; the compute warps (two column
halves x row quarters, modelled as four agents) write P^T over S^T (half 1
over columns half 0 reads, after the shared-read barrier), then, once dK and
dQ of tile g - 1 have read the dS^T buffer, write dS^T(g) into it, and only
then drain dQ of tile g - 1 into the accumulator (its product completed long
before); the last tile's dQ is drained after the loop.  After the epilogue,
every agent arrives at ENDA; agent 0 counts the item on its head and
publishes whether this CTA completed the head, and all read that flag after
ENDB (the counter itself and the dQ conversion it gates are outside the
model).  Asynchronous work completes in any order the hardware allows
(protocol_model.AsyncWork).
"""


from protocol_model import ProtocolError, World, run_roles  # noqa: F401

QST = DOST = 2
NCOMP = 4    # (half, quarter) agents


class Variant:
    def __init__(self, no_srd=False, no_dsf_wait=False, s_without_dvd_wait=False,
                 flag_without_endb=False, ds_without_dqf_wait=False, dq_without_dqe_wait=False):
        self.no_srd = no_srd              # mistake: half 1 writes P^T without the SRD wait
        self.no_dsf_wait = no_dsf_wait    # mistake: dK / dQ issued without waiting for dS^T
        # mistake: S^T(g+1) issued without waiting for dV(g), which reads P^T
        # from the same columns, trusting the issue order of one thread's MMAs
        self.s_without_dvd_wait = s_without_dvd_wait
        # mistake: read the head-completion flag without waiting for ENDB
        self.flag_without_endb = flag_without_endb
        # skip: dS^T(g) written without waiting for dK(g-1) and dQ(g-1) to
        # have read the buffer (implied: the dP^T(g) commit it waits on
        # follows them in issue order)
        self.ds_without_dqf_wait = ds_without_dqf_wait
        # skip: dQ(g) issued into its buffer without waiting for dQ(g-2) to be
        # drained (implied: the compute agents drain dQ(g-2) before they
        # publish dS^T(g), which dQ(g) waits for)
        self.dq_without_dqe_wait = dq_without_dqe_wait


W = None


def producer(n_it, v):
    yield ("async", "tma", land_kv, "tma")
    for g in range(n_it):
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


def land_kv():
    W.write("K", 0)
    W.write("V", 0)
    W.bar("KV").arrive(0)


def issuer(n_it, v):
    yield ("wait", [("KV", 0)])
    for g in range(n_it):
        qs, qn, ds, dn, b = g % QST, g // QST, g % DOST, g // DOST, g & 1
        waits = [(f"QF{qs}", qn)]
        if g > 0 and not v.s_without_dvd_wait:
            waits.append(("DVD", g - 1))
        yield ("wait", waits)

        def s_mma(g=g, qs=qs):
            W.read("K", 0)
            W.read(("Q", qs), g)
            for q in range(2):
                for r in ("R0", "R1", "R2", "R3"):
                    W.write(("S", q, r), ("S", g))
        yield ("async", "mma", s_mma, "S")
        yield ("async", "mma", lambda g=g: W.bar("SF").arrive(g))
        yield ("wait", [(f"DOF{ds}", dn)])

        def dp_mma(g=g, ds=ds):
            W.read("V", 0)
            W.read(("DO", ds), g)
            W.write("DP", g)
        yield ("async", "mma", dp_mma, "DP")
        yield ("async", "mma", lambda g=g: W.bar("DPF").arrive(g))
        yield ("wait", [("PTF", g)])

        def dv_mma(g=g, ds=ds):
            for q in range(2):
                W.read(("S", q, "R0"), ("P", g))
                W.read(("S", q, "R1"), ("P", g))
            W.read(("DO", ds), g)
            W.write("DVACC", g + 1)
        yield ("async", "mma", dv_mma, "DV")
        yield ("async", "mma", lambda g=g: W.bar("DVD").arrive(g))
        yield ("async", "mma", lambda ds=ds, dn=dn: W.bar(f"DOE{ds}").arrive(dn))
        waits = [] if v.no_dsf_wait else [("DSF", g)]
        if g >= 2 and not v.dq_without_dqe_wait:
            # dQ buffer b was last written by dQ(g - 2): drained
            waits.append((f"DQE{b}", (g >> 1) - 1))
        if waits:
            yield ("wait", waits)

        def dk_mma(g=g, qs=qs):
            for h in range(2):
                W.read(("DS", h), g)
            W.read(("Q", qs), g)
            W.write("DKACC", g + 1)

        def dq_mma(g=g, b=b):
            for h in range(2):
                W.read(("DS", h), g)
            W.read("K", 0)
            W.write(("DQ", b), g)
        yield ("async", "mma", dk_mma, "DK")
        yield ("async", "mma", dq_mma, f"DQ{b}")
        yield ("async", "mma", lambda qs=qs, qn=qn: W.bar(f"QE{qs}").arrive(qn))
        yield ("async", "mma", lambda g=g, b=b: W.bar(f"DQF{b}").arrive(g >> 1))
    yield ("async", "mma", lambda: W.bar("FIN").arrive(0))


def compute(agent, n_it, v):
    half, q = agent // 2, agent % 2

    def drain(t):
        b = t & 1
        yield ("read", ("DQ", b), t)
        yield ("arrive", f"DQE{b}", t >> 1)

    for g in range(n_it):
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
        waits = [("DPF", g)]
        if g >= 1 and not v.ds_without_dqf_wait:
            # dK(g - 1) and dQ(g - 1) have read the dS^T buffer
            waits.append((f"DQF{(g - 1) & 1}", (g - 1) >> 1))
        yield ("wait", waits)
        yield ("read", "DP", g)
        yield ("read", ("LD", qs), g)
        yield ("write", ("DS", half), g)
        yield ("arrive", "DSF", g)
        if g >= 1:
            if v.ds_without_dqf_wait:
                yield ("wait", [(f"DQF{(g - 1) & 1}", (g - 1) >> 1)])
            yield from drain(g - 1)
    if n_it > 0:
        t = n_it - 1
        yield ("wait", [(f"DQF{t & 1}", t >> 1)])
        yield from drain(t)
    yield ("wait", [("FIN", 0)])
    if n_it > 0:  # (no query tile: dK = dV = 0 are written without the accumulators)
        yield ("read", "DVACC", n_it)
        yield ("read", "DKACC", n_it)
    # the end-of-item handshake: every agent has written its dK/dV rows
    # (ENDA); agent 0 counts the item on its head and publishes whether the
    # CTA finished the head (the flag); all read the flag after ENDB
    yield ("arrive", "ENDA", 0)
    if agent == 0:
        yield ("wait", [("ENDA", 0)])
        yield ("write", "LASTFLAG", 0)
        yield ("arrive", "ENDB", 0)
    if not v.flag_without_endb:
        yield ("wait", [("ENDB", 0)])
    yield ("read", "LASTFLAG", 0)


def run_schedule(n_it, seed, variant=None, max_steps=200000, in_order=False):
    """n_it: the number of 128-query tiles of the CTA's key tile.  in_order:
    complete each unit's asynchronous work in issue order."""
    global W
    v = variant or Variant()
    W = World()
    for name, c in {"PTF": NCOMP, "DSF": NCOMP, "DQE0": NCOMP, "DQE1": NCOMP,
                    "SRD": NCOMP // 2, "ENDA": NCOMP}.items():
        W.bar(name, c)
    roles = {"prod": producer(n_it, v), "mma": issuer(n_it, v)}
    for a in range(NCOMP):
        roles[f"comp{a}"] = compute(a, n_it, v)
    run_roles(W, roles, seed, in_order, max_steps)
