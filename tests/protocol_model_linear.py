"""A model of the mbarrier protocol of the fused causal linear-attention kernel
(linear_fused_kernel in io_aware_exact_30_b200/csrc/linear_sm100.cuh),
checked on the CPU under random schedules with the rules of protocol_model.py
(barrier tests in the phase they are for or the next, arrivals in their
phase, reads of the versions they need, no deadlock).  Test infrastructure
only.

Roles: the TMA producer, the MMA issuer, the row warps (P and the output:
two key halves x two lane quarters, four agents) and the state warps (two
agents).  Per chunk c (stage c % 2 of Q, K and half of V; buffers b = c % 2
of A/P, O and KV in tensor memory and of the 16-bit state in shared memory)
the issuer does A_c = Q_c K_c^T, KV_c = K_c^T V_c, then O_c = Q_c S_{c-1}
(once the output of chunk c - 2 is read from O buffer b and S_{c-1} is
stored), then, once P_c is written, O_c += P_c V_c.
The row warps turn A_c into P_c (each key half over the first of its own two
32-column blocks: blocks 0 and 2), then read O_{c-1}; the state warps add
KV_c into their running sum and store S_c for the next chunk.
"""

from protocol_model import AsyncWork, ProtocolError, World, run_roles  # noqa: F401

ST = 2      # Q/K/V stages
NROW = 4    # row agents: (key half, lane quarter)
NSTATE = 2  # state agents

W = None


class Variant:
    def __init__(self, no_se_wait=False, no_kve_wait=False, no_oe_wait=False,
                 no_pvd_wait=False, no_ssf_wait=False, no_od_wait=False,
                 contiguous_p=False):
        # skip: the state warps overwrite a state buffer without waiting for
        # the Q S that read it (implied: the KV-full commit they waited on
        # follows that Q S)
        self.no_se_wait = no_se_wait
        # skip: KV of a chunk issued without waiting for the state warps to
        # have read its buffer (implied: the state stored after that read was
        # waited for one chunk earlier)
        self.no_kve_wait = no_kve_wait
        # mistake: Q S of a chunk (which overwrites its O buffer) issued before
        # the row warps have read the output of two chunks back from it
        self.no_oe_wait = no_oe_wait
        # skip: A of a chunk issued without waiting for the P V that read P from
        # the same buffer two chunks back (implied: the chunk's Q, K, V landed
        # in the stage that P V's commit released)
        self.no_pvd_wait = no_pvd_wait
        # mistake: Q S issued before the state warps stored the state it reads
        self.no_ssf_wait = no_ssf_wait
        # mistake: the row warps read O without waiting for its P V
        self.no_od_wait = no_od_wait
        # mistake: the upper key half packs its P next to the lower half's
        # (block 1), over columns the lower half may not have read yet
        self.contiguous_p = contiguous_p


def p_block(half, v):
    """The 32-column block of A buffer that a key half's P is packed into."""
    return 1 if (half == 1 and v.contiguous_p) else 2 * half


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
            for blk in range(4):
                for q in range(2):
                    W.write(("A", b, blk, q), ("A", c))
        yield ("async", "mma", a_mma, f"A{b}")
        yield ("async", "mma", lambda b=b, u=u: W.bar(f"AF{b}").arrive(u))

        def kv_mma(c=c, s=s, b=b):
            W.read(("K", s), c)
            W.read(("V", s), c)
            for a in range(NSTATE):
                W.write(("KV", b, a), c)
        yield ("async", "mma", kv_mma, f"KV{b}")
        yield ("async", "mma", lambda b=b, u=u: W.bar(f"KVF{b}").arrive(u))
        if c >= 1:
            bp, up = (c - 1) & 1, (c - 1) >> 1
            waits = []
            if c >= 2 and not v.no_oe_wait:
                waits.append((f"OE{b}", u - 1))
            if not v.no_ssf_wait:
                waits.append((f"SSF{bp}", up))
            if waits:
                yield ("wait", waits)

            def qs_mma(c=c, s=s, b=b, bp=bp):
                W.read(("Q", s), c)
                for a in range(NSTATE):
                    W.read(("S", bp, a), c - 1)
                for half in range(2):
                    for q in range(2):
                        W.write(("O", b, half, q), (c, "QS"))
            yield ("async", "mma", qs_mma, f"O{b}")
            yield ("async", "mma", lambda bp=bp, up=up: W.bar(f"SE{bp}").arrive(up))
        yield ("wait", [(f"PF{b}", u)])

        def pv_mma(c=c, s=s, b=b):
            W.read(("V", s), c)
            for half in range(2):
                for q in range(2):
                    W.read(("A", b, p_block(half, v), q), ("P", c, half))
                    if c >= 1:
                        W.read(("O", b, half, q), (c, "QS"))
                    W.write(("O", b, half, q), (c, "PV"))
        yield ("async", "mma", pv_mma, f"O{b}")
        yield ("async", "mma", lambda b=b, u=u: W.bar(f"OD{b}").arrive(u))
        yield ("async", "mma", lambda b=b, u=u: W.bar(f"PVD{b}").arrive(u))
        yield ("async", "mma", lambda s=s, n=n: W.bar(f"KE{s}").arrive(n))


def rows(agent, nc, v):
    half, q = agent // 2, agent % 2

    def store_o(c):
        b, u = c & 1, c >> 1
        if not v.no_od_wait:
            yield ("wait", [(f"OD{b}", u)])
        yield ("read", ("O", b, half, q), (c, "PV"))
        yield ("arrive", f"OE{b}", u)

    for c in range(nc):
        b, u = c & 1, c >> 1
        yield ("wait", [(f"AF{b}", u)])
        # the half's two 32-column blocks, read before P is packed over the first
        yield ("read", ("A", b, 2 * half, q), ("A", c))
        yield ("read", ("A", b, 2 * half + 1, q), ("A", c))
        yield ("write", ("A", b, p_block(half, v), q), ("P", c, half))
        yield ("arrive", f"PF{b}", u)
        if c >= 1:
            yield from store_o(c - 1)
    if nc > 0:
        yield from store_o(nc - 1)


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
        W.bar(f"PF{b}", NROW)
        W.bar(f"OE{b}", NROW)
        W.bar(f"KVE{b}", NSTATE)
        W.bar(f"SSF{b}", NSTATE)
    roles = {"prod": producer(nc, v), "mma": issuer(nc, v)}
    for a in range(NROW):
        roles[f"rows{a}"] = rows(a, nc, v)
    for a in range(NSTATE):
        roles[f"state{a}"] = state(a, nc, v)
    run_roles(W, roles, seed, in_order, max_steps)
