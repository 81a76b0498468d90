"""A model of the mbarrier protocol of the forward kernel
(io_aware_exact_30_b200/csrc/fwd_sm100.cuh), checked on the CPU under random
schedules with the same rules as protocol_model.py (the d = 128 backward).
Test infrastructure only.

Roles: the TMA producer, the single MMA issuer and, per query tile, the
softmax warps, modelled as two agents each.  Whether a softmax step moves the
kept max (and rescales O, which needs the previous P V complete) depends on
the data in the kernel; the model decides it at random.

A work item is a pair of query tiles.  Tile t attends to key tile j iff
act(t, j): j below its causal bound and, under a block mask, marked.  Every
role walks the union of the two tiles' key tiles in order (K and V are loaded
once per union tile); per union tile j the issuer does, for t = 0, 1: P_t V_j
if act(t, j), then S_t of the next union tile if tile t attends to it (after
the last P_t V, which read the same tensor-memory columns, has completed).
An item where neither tile attends to anything loads Q only; a tile with no
key tile writes zeros without touching tensor memory.

Every operation of a role (barrier tests and arrivals, its own reads and
writes) is a step of its own; the effects of an MMA or a copy happen at once
when it completes, in any order the hardware allows (protocol_model.AsyncWork:
MMA groups in issue order only per accumulator, a commit after all earlier
work of its thread, copies in any order).

Plan items: (n0, n1) for dense tiles (tile t attends to j < n_t), or
(n0, n1, mask0, mask1) with mask_t a sequence of 0/1 per key tile.

Two tensor-memory layouts: at d = 128 P_t is written over S_t (the next S_t
waits for the last P_t V); at d = 64 (p_own) P_t has columns of its own, so
the next S_t is issued as soon as P-ready shows the softmax is done with S_t,
ahead of the P_t V, and the softmax waits for that P_t V before it writes
P_t again.
"""

from protocol_model import ProtocolError, World, item_advance, item_request, run_roles  # noqa: F401

ST = 2      # K/V stages: 2 at d = 128, 3 for e4m3 scores at d = 128, 4 at d = 64
NSM = 2     # softmax agents per query tile


class Variant:
    def __init__(self, ke_before_pv=False, epilogue_no_od_wait=False, s_without_od_wait=False,
                 static_items=False, clc_no_empty_wait=False, s_wait_ignores_fresh_tile=False,
                 p_write_no_od_wait=False):
        # release the K/V stage before the tile-1 P V of the step is issued
        self.ke_before_pv = ke_before_pv
        # the epilogue reads O without waiting for the last P V
        self.epilogue_no_od_wait = epilogue_no_od_wait
        # mistake: the next S issued without waiting for the P V that reads
        # its columns, trusting the issue order (which the hardware keeps only
        # between MMAs on the same accumulator)
        self.s_without_od_wait = s_without_od_wait
        # work items dealt in a fixed order (no mask) instead of taken through
        # cluster launch control responses
        self.static_items = static_items
        # mistake: ask for the next item into a response slot before every
        # consumer has read the slot's previous response
        self.clc_no_empty_wait = clc_no_empty_wait
        # mistake (block-sparse walk): the wait for the last P_t V before the
        # next S_t is skipped when tile t issued no P V at this union tile (it
        # skipped a key tile the other tile attends to), as if the wait were
        # only needed right after issuing the P V.  With two K/V stages the
        # wait for the next K implies it (that stage was released by a commit
        # after the P V); with more stages it does not.  (A tile's first S of
        # an item needs no such wait either: the item's Q load follows the
        # previous item's last commit, which covers every earlier MMA.)
        self.s_wait_ignores_fresh_tile = s_wait_ignores_fresh_tile
        # mistake (P in columns of its own): the softmax writes P_t without
        # waiting for the last P_t V, which reads the same columns (the next
        # S_t goes out ahead of that P V, so S-full does not cover it)
        self.p_write_no_od_wait = p_write_no_od_wait


W = None
P_OWN = False  # d = 64: P_t in tensor-memory columns of its own


def p_cols(t, a):
    """Where agent a of tile t writes P_t (and P_t V reads it)."""
    return ("P", t, a) if P_OWN else ("S", t, a)


class Item:
    """Key tiles of one work item."""

    def __init__(self, spec):
        n0, n1 = spec[0], spec[1]
        masks = spec[2:] if len(spec) > 2 else None
        self.n = (n0, n1)
        self.nkv = max(n0, n1)
        self.act = [[j < self.n[t] and (masks is None or bool(masks[t][j]))
                     for j in range(self.nkv)] for t in range(2)]
        self.union = [j for j in range(self.nkv) if self.act[0][j] or self.act[1][j]]
        self.count = [sum(self.act[t]) for t in range(2)]


def producer(plan, v):
    kv = 0
    for item, spec in enumerate(plan):
        it = Item(spec)
        if item > 0:
            yield ("wait", [("QE", item - 1)])

        def land_q(item=item):
            W.write("Q", item)
            W.bar("Q").arrive(item)
        yield ("async", "tma", land_q, "tma")
        for u, _ in enumerate(it.union):
            kvj = kv + u
            s, n = kvj % ST, kvj // ST
            yield ("wait", [(f"KE{s}", n - 1)])

            def land_k(kvj=kvj, s=s, n=n):
                W.write(("K", s), kvj)
                W.bar(f"KF{s}").arrive(n)

            def land_v(kvj=kvj, s=s, n=n):
                W.write(("V", s), kvj)
                W.bar(f"VF{s}").arrive(n)
            yield ("async", "tma", land_k, "tma")
            yield ("async", "tma", land_v, "tma")
        kv += len(it.union)
        yield from item_request(W, item, not v.static_items, not v.clc_no_empty_wait)
        yield from item_advance(W, item, not v.static_items)


def issuer(plan, v):
    kv = 0
    n_pv, n_s, n_done = [0, 0], [0, 0], [0, 0]

    def issue_s(t, kvi, item):
        s = kvi % ST

        def run(t=t, kvi=kvi, s=s, item=item):
            W.read("Q", item)
            W.read(("K", s), kvi)
            for a in range(NSM):
                W.write(("S", t, a), ("S", kvi))
        yield ("async", "mma", run, f"S{t}")
        k = n_s[t]
        n_s[t] += 1
        yield ("async", "mma", lambda t=t, k=k: W.bar(f"SF{t}").arrive(k))

    for item, spec in enumerate(plan):
        it = Item(spec)
        U = it.union
        a0 = [bool(U) and it.act[t][U[0]] for t in range(2)]
        waits = [("Q", item)]
        if U:
            waits.append((f"KF{kv % ST}", kv // ST))
        if a0[0] and n_pv[0] > 0 and not P_OWN:
            waits.append(("OD0", n_pv[0] - 1))
        yield ("wait", waits)
        if a0[1] and n_pv[1] > 0 and not P_OWN:
            yield ("wait", [("OD1", n_pv[1] - 1)])
        for t in range(2):
            if a0[t]:
                yield from issue_s(t, kv, item)
        fresh = [True, True]  # no P_t V of this item issued yet
        for u, j in enumerate(U):
            kvj = kv + u
            s, n = kvj % ST, kvj // ST
            k1 = kvj + 1
            jn = U[u + 1] if u + 1 < len(U) else None
            k_next = False  # K of the next union tile has been waited for
            for t in range(2):
                act = it.act[t][j]
                waits = []
                if t == 0:
                    waits.append((f"VF{s}", n))
                if act:
                    waits.append((f"PF{t}", n_pv[t]))
                    if fresh[t] and n_done[t] > 0:
                        waits.append((f"OE{t}", n_done[t] - 1))
                if waits:
                    yield ("wait", waits)
                if t == 1 and v.ke_before_pv:
                    yield ("async", "mma", lambda s=s, n=n: W.bar(f"KE{s}").arrive(n))
                def do_pv(t=t, act=act, kvj=kvj, s=s, item=item, u=u):
                    if act:
                        def pv(t=t, kvj=kvj, s=s, item=item, u=u):
                            for a in range(NSM):
                                W.read(p_cols(t, a), ("P", kvj))
                            W.read(("V", s), kvj)
                            W.write(("O", t), (item, u))
                        yield ("async", "mma", pv, f"O{t}")
                        k = n_pv[t]
                        n_pv[t] += 1
                        fresh[t] = False
                        yield ("async", "mma", lambda t=t, k=k: W.bar(f"OD{t}").arrive(k))

                def do_next_s(t=t, act=act, k1=k1, item=item):
                    nonlocal k_next
                    if jn is not None and it.act[t][jn]:
                        # S_t of the next union tile takes the columns the last P_t V
                        # read: wait for that P V (of this item or an earlier one);
                        # with P in columns of its own, the softmax read S_t before
                        # the P-ready arrival the last P_t V waited for
                        waits = []
                        skip = (P_OWN or v.s_without_od_wait
                                or (v.s_wait_ignores_fresh_tile and not act))
                        if n_pv[t] > 0 and not skip:
                            waits.append((f"OD{t}", n_pv[t] - 1))
                        if not k_next:
                            waits.append((f"KF{k1 % ST}", k1 // ST))
                        if waits:
                            yield ("wait", waits)
                        k_next = True
                        yield from issue_s(t, k1, item)
                if P_OWN:
                    # the next S_t first: its columns were read before P-ready
                    yield from do_next_s()
                    yield from do_pv()
                else:
                    yield from do_pv()
                    yield from do_next_s()
            if not v.ke_before_pv:
                yield ("async", "mma", lambda s=s, n=n: W.bar(f"KE{s}").arrive(n))
        yield ("async", "mma", lambda item=item: W.bar("QE").arrive(item))
        kv += len(U)
        for t in range(2):
            if not fresh[t]:
                n_done[t] += 1
        yield from item_advance(W, item, not v.static_items)


def softmax(t, agent, plan, v, rng):
    kv = 0
    n_s = 0
    done = 0
    for item, spec in enumerate(plan):
        it = Item(spec)
        if it.n[t] == 0 or it.count[t] == 0:
            # no second tile, or a tile with no marked key tile: O = 0 and
            # LSE = -inf are written without touching tensor memory
            if it.n[t] > 0:
                yield ("write", ("OUT", t, agent), item)
            kv += len(it.union)
            yield from item_advance(W, item, not v.static_items)
            continue
        seen = 0
        for u, j in enumerate(it.union):
            if not it.act[t][j]:
                continue
            yield ("wait", [(f"SF{t}", n_s)])
            n_s += 1
            yield ("read", ("S", t, agent), ("S", kv + u))
            od_waited = False  # for the last P_t V
            if seen > 0 and rng.random() < 0.3:
                # the kept max moves: O is rescaled, which needs the last P V
                yield ("wait", [(f"OD{t}", n_s - 2)])
                od_waited = True
                yield ("read", ("O", t), (item, prev_u))
            if P_OWN and n_s >= 2 and not od_waited and not v.p_write_no_od_wait:
                # P_t's columns were last read by the previous P_t V
                yield ("wait", [(f"OD{t}", n_s - 2)])
            yield ("write", p_cols(t, agent), ("P", kv + u))
            yield ("arrive", f"PF{t}", n_s - 1)
            seen += 1
            prev_u = u
        if not v.epilogue_no_od_wait:
            yield ("wait", [(f"OD{t}", n_s - 1)])
        yield ("read", ("O", t), (item, prev_u))
        yield ("arrive", f"OE{t}", done)
        done += 1
        kv += len(it.union)
        yield from item_advance(W, item, not v.static_items)


def run_schedule(plan, seed, variant=None, max_steps=200000, in_order=False, stages=2,
                 p_own=False):
    """One random schedule of one CTA working through `plan`; raises
    ProtocolError on a violation or a deadlock.  in_order: complete each
    unit's asynchronous work in issue order.  stages: K/V pipeline depth.
    p_own: the d = 64 layout (P_t in columns of its own)."""
    import random
    global W, ST, P_OWN
    ST = stages
    P_OWN = p_own
    v = variant or Variant()
    W = World()
    for t in range(2):
        W.bar(f"PF{t}", NSM)
        W.bar(f"OE{t}", NSM)
    # one arrival per modelled agent frees a response slot
    n_consumers = 2 + 2 * NSM
    W.bar("CLCE0", n_consumers)
    W.bar("CLCE1", n_consumers)
    roles = {"prod": producer(plan, v), "mma": issuer(plan, v)}
    for t in range(2):
        for a in range(NSM):
            roles[f"sm{t}{a}"] = softmax(t, a, plan, v, random.Random(seed * 7 + 2 * t + a))
    run_roles(W, roles, seed, in_order, max_steps)
