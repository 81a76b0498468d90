"""A model of the mbarrier protocol of the fused causal linear-attention kernel
(linear_fused_kernel in io_aware_exact_30_b200/csrc/linear_sm100.cuh),
checked on the CPU under random schedules with the rules of protocol_model.py
(barrier tests in the phase they are for or the next, arrivals in their
phase, reads of the versions they need, no deadlock).  Test infrastructure
only.

Roles: the TMA producer, the MMA issuer, the row warps (P and the output,
two agents) and the state warps (two agents).  Per chunk c (stage c % 2 of
Q, K and half of V; buffers b = c % 2 of A/P and KV in tensor memory and of
the 16-bit state in shared memory) the issuer does A_c = Q_c K_c^T, KV_c =
K_c^T V_c, then O_c = Q_c S_{c-1} (once the output of chunk c - 1 is read and
S_{c-1} is stored), then, once P_c is written, O_c += P_c V_c.  The row warps
turn A_c into P_c and read O_c; the state warps add KV_c into their running
sum and store S_c for the next chunk.
"""

from protocol_model import AsyncWork, ProtocolError, World, run_roles  # noqa: F401

ST = 2      # Q/K/V stages
NA = 2      # agents per group of warps

W = None


class Variant:
    def __init__(self, no_se_wait=False, no_kve_wait=False, no_oe_wait=False,
                 no_pvd_wait=False, no_ssf_wait=False):
        # skip: the state warps overwrite a state buffer without waiting for
        # the Q S that read it (implied: the KV-full commit they waited on
        # follows that Q S)
        self.no_se_wait = no_se_wait
        # skip: KV of a chunk issued without waiting for the state warps to
        # have read the buffer (implied: the state stored after that read was
        # waited for one chunk earlier)
        self.no_kve_wait = no_kve_wait
        # mistake: Q S of the next chunk (which overwrites O) issued before the
        # row warps have read O
        self.no_oe_wait = no_oe_wait
        # skip: A of a chunk issued without waiting for the P V of two chunks
        # back, which read P from the same buffer (implied: the output read
        # after that P V was waited for one chunk earlier)
        self.no_pvd_wait = no_pvd_wait
        # mistake: Q S issued before the state warps stored the state it reads
        self.no_ssf_wait = no_ssf_wait


def producer(nc, v):
    for c in range(nc):
        s, n = c % ST, c // ST
        if n > 0:
            yield ("wait", [(f"KE{s}", n - 1)])

        def land(c=c, s=s, n=n):
            for x in ("Q", "K", "V"):
                W.write((x, s), c)
            W.bar(f"LD{s}").arrive(n)
        yield ("async", "tma", land, "tma")


def issuer(nc, v):
    for c in range(nc):
        s, n, b, u = c % ST, c // ST, c & 1, c >> 1
        waits = [(f"LD{s}", n)]
        if c >= 2:
            if not v.no_pvd_wait:
                waits.append((f"PVD{b}", u - 1))
            if not v.no_kve_wait:
                waits.append((f"KVE{b}", u - 1))
        yield ("wait", waits)

        def a_mma(c=c, s=s, b=b):
            W.read(("Q", s), c)
            W.read(("K", s), c)
            for a in range(NA):
                W.write(("A", b, a), ("A", c))
        yield ("async", "mma", a_mma, f"A{b}")
        yield ("async", "mma", lambda b=b, u=u: W.bar(f"AF{b}").arrive(u))

        def kv_mma(c=c, s=s, b=b):
            W.read(("K", s), c)
            W.read(("V", s), c)
            for a in range(NA):
                W.write(("KV", b, a), c)
        yield ("async", "mma", kv_mma, f"KV{b}")
        yield ("async", "mma", lambda b=b, u=u: W.bar(f"KVF{b}").arrive(u))
        if c >= 1:
            bp, up = (c - 1) & 1, (c - 1) >> 1
            waits = []
            if not v.no_oe_wait:
                waits.append(("OE", c - 1))
            if not v.no_ssf_wait:
                waits.append((f"SSF{bp}", up))
            if waits:
                yield ("wait", waits)

            def qs_mma(c=c, s=s, bp=bp):
                W.read(("Q", s), c)
                for a in range(NA):
                    W.read(("S", bp, a), c - 1)
                    W.write(("O", a), (c, "QS"))
            yield ("async", "mma", qs_mma, "O")
            yield ("async", "mma", lambda bp=bp, up=up: W.bar(f"SE{bp}").arrive(up))
        yield ("wait", [(f"PF{b}", u)])

        def pv_mma(c=c, s=s, b=b):
            W.read(("V", s), c)
            for a in range(NA):
                W.read(("A", b, a), ("P", c))
                if c >= 1:
                    W.read(("O", a), (c, "QS"))
                W.write(("O", a), (c, "PV"))
        yield ("async", "mma", pv_mma, "O")
        yield ("async", "mma", lambda c=c: W.bar("OD").arrive(c))
        yield ("async", "mma", lambda b=b, u=u: W.bar(f"PVD{b}").arrive(u))
        yield ("async", "mma", lambda s=s, n=n: W.bar(f"KE{s}").arrive(n))


def rows(agent, nc, v):
    for c in range(nc):
        b, u = c & 1, c >> 1
        yield ("wait", [(f"AF{b}", u)])
        yield ("read", ("A", b, agent), ("A", c))
        yield ("write", ("A", b, agent), ("P", c))
        yield ("arrive", f"PF{b}", u)
        yield ("wait", [("OD", c)])
        yield ("read", ("O", agent), (c, "PV"))
        yield ("arrive", "OE", c)


def state(agent, nc, v):
    for c in range(nc):
        b, u = c & 1, c >> 1
        yield ("wait", [(f"KVF{b}", u)])
        yield ("read", ("KV", b, agent), c)
        yield ("arrive", f"KVE{b}", u)
        if c == nc - 1:
            break
        if c >= 2 and not v.no_se_wait:
            yield ("wait", [(f"SE{b}", u - 1)])
        yield ("write", ("S", b, agent), c)
        yield ("arrive", f"SSF{b}", u)


def run_schedule(nc, seed, variant=None, in_order=False, max_steps=200000):
    """One random schedule of one CTA working through nc chunks; raises
    ProtocolError on a violation or a deadlock."""
    global W
    v = variant or Variant()
    W = World()
    for b in range(2):
        for name in ("PF", "KVE", "SSF"):
            W.bar(f"{name}{b}", NA)
    W.bar("OE", NA)
    roles = {"prod": producer(nc, v), "mma": issuer(nc, v)}
    for a in range(NA):
        roles[f"rows{a}"] = rows(a, nc, v)
        roles[f"state{a}"] = state(a, nc, v)
    run_roles(W, roles, seed, in_order, max_steps)
