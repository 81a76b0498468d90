"""A model of the mbarrier protocol of the d = 64 backward main kernel
(attn_bwd_main_kernel in io_aware_exact_30_b200/csrc/bwd_sm100.cuh), checked
on the CPU under random schedules with the rules of protocol_model.py.  Test
infrastructure only.

One CTA works on one 128-key tile: the producer loads K/V once and streams
128-query tiles of Q (with the row statistics) and dO through two stages each;
one thread issues, per tile, S^T, dP^T, dV, then dK and dQ (in that order,
each group after its barriers); the compute warps (two column halves x row
quarters, modelled as four agents) write P^T over S^T (half 1 over columns half
0 reads, after the shared-read barrier), dS^T into shared memory, and drain dQ
into the accumulator.  The per-head completion counters after the epilogue
are outside the model.
"""

import random

from protocol_model import ProtocolError, World

QST = DOST = 2
NCOMP = 4    # (half, quarter) agents


class Variant:
    def __init__(self, no_srd=False, no_dsf_wait=False):
        self.no_srd = no_srd              # mistake: half 1 writes P^T without the SRD wait
        self.no_dsf_wait = no_dsf_wait    # mistake: dK / dQ issued without waiting for dS^T


W = None


def producer(n_it, v):
    def land_kv():
        W.write("K", 0)
        W.write("V", 0)
        W.bar("KV").arrive(0)
    yield ("async", "tma", land_kv)
    for it in range(n_it):
        qs, qn, ds, dn = it % QST, it // QST, it % DOST, it // DOST
        yield ("wait", [(f"QE{qs}", qn - 1)])

        def land_q(it=it, qs=qs, qn=qn):
            W.write(("Q", qs), it)
            W.write(("LD", qs), it)
            W.bar(f"QF{qs}").arrive(qn)
        yield ("async", "tma", land_q)
        yield ("wait", [(f"DOE{ds}", dn - 1)])

        def land_do(it=it, ds=ds, dn=dn):
            W.write(("DO", ds), it)
            W.bar(f"DOF{ds}").arrive(dn)
        yield ("async", "tma", land_do)


def issuer(n_it, v):
    yield ("wait", [("KV", 0)])
    for it in range(n_it):
        qs, qn, ds, dn = it % QST, it // QST, it % DOST, it // DOST
        waits = [(f"QF{qs}", qn)]
        if it > 0:
            waits.append(("DVD", it - 1))
        yield ("wait", waits)

        def s_mma(it=it, qs=qs):
            W.read("K", 0)
            W.read(("Q", qs), it)
            for q in range(2):
                for r in ("R0", "R1", "R2", "R3"):
                    W.write(("S", q, r), ("S", it))
        yield ("async", "mma", s_mma)
        yield ("async", "mma", lambda it=it: W.bar("SF").arrive(it))
        yield ("wait", [(f"DOF{ds}", dn)])

        def dp_mma(it=it, ds=ds):
            W.read("V", 0)
            W.read(("DO", ds), it)
            W.write("DP", it)
        yield ("async", "mma", dp_mma)
        yield ("async", "mma", lambda it=it: W.bar("DPF").arrive(it))
        yield ("wait", [("PTF", it)])

        def dv_mma(it=it, ds=ds):
            for q in range(2):
                W.read(("S", q, "R0"), ("P", it))
                W.read(("S", q, "R1"), ("P", it))
            W.read(("DO", ds), it)
            W.write("DVACC", it + 1)
        yield ("async", "mma", dv_mma)
        yield ("async", "mma", lambda it=it: W.bar("DVD").arrive(it))
        yield ("async", "mma", lambda ds=ds, dn=dn: W.bar(f"DOE{ds}").arrive(dn))
        waits = [] if v.no_dsf_wait else [("DSF", it)]
        if it > 0:
            waits.append(("DQE", it - 1))
        if waits:
            yield ("wait", waits)

        def dkdq_mma(it=it, qs=qs):
            for h in range(2):
                W.read(("DS", h), it)
            W.read(("Q", qs), it)
            W.read("K", 0)
            W.write("DKACC", it + 1)
            W.write("DQ", it)
        yield ("async", "mma", dkdq_mma)
        yield ("async", "mma", lambda qs=qs, qn=qn: W.bar(f"QE{qs}").arrive(qn))
        yield ("async", "mma", lambda it=it: W.bar("DQF").arrive(it))
    yield ("async", "mma", lambda: W.bar("FIN").arrive(0))


def compute(agent, n_it, v):
    half, q = agent // 2, agent % 2
    for it in range(n_it):
        qs, qn = it % QST, it // QST
        yield ("wait", [(f"QF{qs}", qn)])
        yield ("wait", [("SF", it)])
        for r in (("R0", "R1") if half == 0 else ("R2", "R3")):
            yield ("read", ("S", q, r), ("S", it))
        yield ("read", ("LD", qs), it)
        if half == 0:
            if not v.no_srd:
                yield ("arrive", "SRD", it)
            yield ("write", ("S", q, "R0"), ("P", it))
        else:
            if not v.no_srd:
                yield ("wait", [("SRD", it)])
            yield ("write", ("S", q, "R1"), ("P", it))
        yield ("arrive", "PTF", it)
        yield ("wait", [("DPF", it)])
        yield ("read", "DP", it)
        yield ("read", ("LD", qs), it)
        yield ("write", ("DS", half), it)
        yield ("arrive", "DSF", it)
        yield ("wait", [("DQF", it)])
        yield ("read", "DQ", it)
        yield ("arrive", "DQE", it)
    yield ("wait", [("FIN", 0)])
    yield ("read", "DVACC", n_it)
    yield ("read", "DKACC", n_it)


def run_schedule(n_it, seed, variant=None, max_steps=200000):
    global W
    v = variant or Variant()
    W = World()
    for name, c in {"PTF": NCOMP, "DSF": NCOMP, "DQE": NCOMP, "SRD": NCOMP // 2}.items():
        W.bar(name, c)
    rng = random.Random(seed)
    roles = {"prod": producer(n_it, v), "mma": issuer(n_it, v)}
    for a in range(NCOMP):
        roles[f"comp{a}"] = compute(a, n_it, v)
    nxt = {n: None for n in roles}
    queues = {"tma": [], "mma": []}
    done = set()

    def advance(name):
        try:
            nxt[name] = next(roles[name])
        except StopIteration:
            nxt[name] = None
            done.add(name)

    for name in roles:
        advance(name)
    for _ in range(max_steps):
        if len(done) == len(roles) and not any(queues.values()):
            return
        choices = []
        for name, op in nxt.items():
            if op is None:
                continue
            if op[0] != "wait" or all(W.bar(b).test(k) for b, k in op[1]):
                choices.append(("role", name))
        choices += [("queue", qn) for qn, qu in queues.items() if qu]
        if not choices:
            raise ProtocolError("deadlock: " + str([(n, o) for n, o in nxt.items() if o]))
        kind, name = rng.choice(choices)
        if kind == "queue":
            queues[name].pop(0)()
            continue
        op = nxt[name]
        if op[0] == "arrive":
            W.bar(op[1]).arrive(op[2])
        elif op[0] == "async":
            queues[op[1]].append(op[2])
        elif op[0] == "read":
            W.read(op[1], op[2])
        elif op[0] == "write":
            W.write(op[1], op[2])
        advance(name)
    raise ProtocolError("schedule did not finish")
