"""A model of the mbarrier protocol of the forward kernel
(io_aware_exact_30_b200/csrc/fwd_sm100.cuh), checked on the CPU under random
schedules with the same rules as protocol_model.py (the d = 128 backward).
Test infrastructure only.

Roles: the TMA producer, the single MMA issuer (order per key tile j:
O_0 += P_0 V_j, S_0(j+1), O_1 += P_1 V_j, S_1(j+1)) and, per query tile, the
softmax warps, modelled as two agents each.  Whether a softmax step moves the
kept max (and rescales O, which needs the previous P V complete) depends on
the data in the kernel; the model decides it at random.

Every operation of a role (barrier tests and arrivals, its own reads and
writes) is a step of its own; the effects of an MMA or a copy happen at once
when it completes, in any order the hardware allows (protocol_model.AsyncWork:
MMA groups in issue order only per accumulator, a commit after all earlier
work of its thread, copies in any order).

A work item is given by (nkv_0, nkv_1), the key-tile steps of its two query
tiles: equal without the mask; under the causal mask tile 1 has one more, and
the last pair of an odd tile count has nkv_1 = 0.
"""

import random

from protocol_model import ProtocolError, World, item_advance, item_request, run_roles

ST = 2      # K/V stages (d = 128)
ST_DOUBLE = 4  # K/V stages of 64-key tiles (the s_double design)
NSM = 2     # softmax agents per query tile


class Variant:
    def __init__(self, ke_before_pv=False, epilogue_no_od_wait=False, split=False,
                 split_no_exchange_wait=False, order_c=False, s_without_od_wait=False,
                 static_items=False, clc_no_empty_wait=False, s_double=False,
                 s_double_no_od_wait=False):
        # release the K/V stage before the tile-1 P V of the step is issued
        self.ke_before_pv = ke_before_pv
        # the epilogue reads O without waiting for the last P V
        self.epilogue_no_od_wait = epilogue_no_od_wait
        # design variant: each tile's softmax split over two column halves (each
        # writing P over its own S columns), the row max exchanged through
        # shared memory per key tile (one barrier and one slot per step parity)
        # and the row sum per item
        self.split = split
        # mistake for the split design: read the other half's max without
        # waiting for the exchange barrier
        self.split_no_exchange_wait = split_no_exchange_wait
        # design variant: per key tile both tiles' P V first, then both next S
        # (each after its own P V has completed), so that each wait for a P V
        # is covered by MMAs already in the tensor pipe
        self.order_c = order_c
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
        # design variant: 64-key K/V tiles (4 stages) and two S buffers per
        # query tile, so S_t(j + 1) is computed while the softmax works on
        # S_t(j); per key tile both P V, then both S_t(j + 2) (each after the
        # P V that read its buffer)
        self.s_double = s_double
        # mistake for that design: S_t(j + 2) issued without waiting for
        # P_t(j) V, which reads the same buffer
        self.s_double_no_od_wait = s_double_no_od_wait


W = None


def stages(v):
    return ST_DOUBLE if v.s_double else ST


def producer(plan, v):
    ST = stages(v)
    kv = 0
    for item, (n0, n1) in enumerate(plan):
        nkv = max(n0, n1)
        if item > 0:
            yield ("wait", [("QE", item - 1)])

        def land_q(item=item):
            W.write("Q", item)
            W.bar("Q").arrive(item)
        yield ("async", "tma", land_q, "tma")
        for j in range(nkv):
            kvj = kv + j
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
        kv += nkv
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
            for a in range(nagents(v)):
                W.write(("S", t, a), ("S", kvi))
        yield ("async", "mma", run, f"S{t}")
        k = n_s[t]
        n_s[t] += 1
        yield ("async", "mma", lambda t=t, k=k: W.bar(f"SF{t}").arrive(k))

    for item, (n0, n1) in enumerate(plan):
        nkv_t = (n0, n1)
        nkv = max(n0, n1)
        waits = [("Q", item), (f"KF{kv % ST}", kv // ST)]
        if n0 > 0 and n_pv[0] > 0:
            waits.append(("OD0", n_pv[0] - 1))
        yield ("wait", waits)
        if n1 > 0 and n_pv[1] > 0:
            yield ("wait", [("OD1", n_pv[1] - 1)])
        for t in range(2):
            if nkv_t[t] > 0:
                yield from issue_s(t, kv, item)
        for j in range(nkv):
            kvj = kv + j
            s, n = kvj % ST, kvj // ST
            k1 = kvj + 1
            k_next = [False]  # K_{j+1} has been waited for

            def next_s(t, k1=k1, k_next=k_next, item=item):
                # S_t(j+1) takes the columns P_t(j) V read: wait for that P V
                waits = [] if v.s_without_od_wait else [(f"OD{t}", n_pv[t] - 1)]
                if not k_next[0]:
                    waits.append((f"KF{k1 % ST}", k1 // ST))
                if waits:
                    yield ("wait", waits)
                k_next[0] = True
                yield from issue_s(t, k1, item)

            for t in range(2):
                act = j < nkv_t[t]
                waits = []
                if t == 0:
                    waits.append((f"VF{s}", n))
                if act:
                    waits.append((f"PF{t}", n_pv[t]))
                    if j == 0 and n_done[t] > 0:
                        waits.append((f"OE{t}", n_done[t] - 1))
                if waits:
                    yield ("wait", waits)
                if t == 1 and v.ke_before_pv:
                    yield ("async", "mma", lambda s=s, n=n: W.bar(f"KE{s}").arrive(n))
                if not act:
                    continue

                def pv(t=t, kvj=kvj, s=s, item=item, j=j):
                    for a in range(nagents(v)):
                        W.read(("S", t, a), ("P", kvj))
                    W.read(("V", s), kvj)
                    for hh in range(2 if v.split else 1):
                        W.write(("O", t, hh), (item, j + 1))
                yield ("async", "mma", pv, f"O{t}")
                k = n_pv[t]
                n_pv[t] += 1
                yield ("async", "mma", lambda t=t, k=k: W.bar(f"OD{t}").arrive(k))
                if j + 1 < nkv_t[t] and not v.order_c:
                    yield from next_s(t)
            if v.order_c:
                if not v.ke_before_pv:
                    yield ("async", "mma", lambda s=s, n=n: W.bar(f"KE{s}").arrive(n))
                for t in range(2):
                    if j + 1 < nkv_t[t]:
                        yield from next_s(t)
            elif not v.ke_before_pv:
                yield ("async", "mma", lambda s=s, n=n: W.bar(f"KE{s}").arrive(n))
        yield ("async", "mma", lambda item=item: W.bar("QE").arrive(item))
        kv += nkv
        for t in range(2):
            if nkv_t[t] > 0:
                n_done[t] += 1
        yield from item_advance(W, item, not v.static_items)


def issuer_sdouble(plan, v):
    """The s_double design: S in two buffers per query tile."""
    stg = stages(v)
    kv = 0
    n_pv, n_s, n_done = [0, 0], [0, 0], [0, 0]

    def issue_s(t, kvi, item):
        s, b, use = kvi % stg, n_s[t] & 1, n_s[t] >> 1

        def run(t=t, kvi=kvi, s=s, b=b, item=item):
            W.read("Q", item)
            W.read(("K", s), kvi)
            for a in range(nagents(v)):
                W.write(("S", t, b, a), ("S", kvi))
        yield ("async", "mma", run, f"S{t}{b}")
        n_s[t] += 1
        yield ("async", "mma", lambda t=t, b=b, use=use: W.bar(f"SF{t}{b}").arrive(use))

    for item, (n0, n1) in enumerate(plan):
        nkv_t = (n0, n1)
        nkv = max(n0, n1)
        base = list(n_s)  # S count of each tile at the item's start
        # the previous item's last P V (committed after every earlier one)
        # read the buffers the first S take
        waits = [("Q", item), (f"KF{kv % stg}", kv // stg)]
        for t in range(2):
            if nkv_t[t] > 0 and n_pv[t] > 0:
                last = n_pv[t] - 1
                waits.append((f"OD{t}{last & 1}", last >> 1))
        yield ("wait", waits)
        for t in range(2):
            if nkv_t[t] > 0:
                yield from issue_s(t, kv, item)
        if nkv > 1:
            yield ("wait", [(f"KF{(kv + 1) % stg}", (kv + 1) // stg)])
            for t in range(2):
                if nkv_t[t] > 1:
                    yield from issue_s(t, kv + 1, item)
        for j in range(nkv):
            kvj = kv + j
            s, n = kvj % stg, kvj // stg
            for t in range(2):
                act = j < nkv_t[t]
                waits = []
                if t == 0:
                    waits.append((f"VF{s}", n))
                b = (base[t] + j) & 1
                if act:
                    # P ready, one barrier per S buffer: with S(j + 1) computed
                    # early, one agent can run a step ahead of another
                    waits.append((f"PF{t}{b}", n_pv[t] >> 1))
                    if j == 0 and n_done[t] > 0:
                        waits.append((f"OE{t}", n_done[t] - 1))
                if waits:
                    yield ("wait", waits)
                if not act:
                    continue

                def pv(t=t, kvj=kvj, s=s, b=b, item=item, j=j):
                    for a in range(nagents(v)):
                        W.read(("S", t, b, a), ("P", kvj))
                    W.read(("V", s), kvj)
                    W.write(("O", t, 0), (item, j + 1))
                yield ("async", "mma", pv, f"O{t}")
                k = n_pv[t]
                n_pv[t] += 1
                # P V done, one barrier per S buffer: two P V of a tile can be
                # in flight, and a parity test is only valid for the newest
                # phase or the one before
                yield ("async", "mma", lambda t=t, k=k: W.bar(f"OD{t}{k & 1}").arrive(k >> 1))
            yield ("async", "mma", lambda s=s, n=n: W.bar(f"KE{s}").arrive(n))
            k2, k_waited = kvj + 2, False
            for t in range(2):
                if j + 2 < nkv_t[t]:
                    k = n_pv[t] - 1
                    waits = [] if v.s_double_no_od_wait else [(f"OD{t}{k & 1}", k >> 1)]
                    if not k_waited:
                        waits.append((f"KF{k2 % stg}", k2 // stg))
                    k_waited = True
                    yield ("wait", waits)
                    yield from issue_s(t, k2, item)
        yield ("async", "mma", lambda item=item: W.bar("QE").arrive(item))
        kv += nkv
        for t in range(2):
            if nkv_t[t] > 0:
                n_done[t] += 1
        yield from item_advance(W, item, not v.static_items)


def softmax_sdouble(t, agent, plan, v, rng):
    kv = n_s = done = 0
    for item, nk in enumerate(plan):
        my, nkv = nk[t], max(nk)
        if my == 0:
            kv += nkv
            yield from item_advance(W, item, not v.static_items)
            continue
        for j in range(my):
            b, use = n_s & 1, n_s >> 1
            yield ("wait", [(f"SF{t}{b}", use)])
            n_s += 1
            yield ("read", ("S", t, b, agent), ("S", kv + j))
            if j > 0 and rng.random() < 0.3:
                # the kept max moves: O is rescaled, which needs P V(j-1)
                k = n_s - 2
                yield ("wait", [(f"OD{t}{k & 1}", k >> 1)])
                yield ("read", ("O", t, 0), (item, j))
            yield ("write", ("S", t, b, agent), ("P", kv + j))
            yield ("arrive", f"PF{t}{b}", use)
        k = n_s - 1
        yield ("wait", [(f"OD{t}{k & 1}", k >> 1)])
        yield ("read", ("O", t, 0), (item, my))
        yield ("arrive", f"OE{t}", done)
        done += 1
        kv += nkv
        yield from item_advance(W, item, not v.static_items)


def softmax(t, agent, plan, v, rng):
    kv = 0
    n_s = 0
    done = 0
    for item, nk in enumerate(plan):
        my = nk[t]
        nkv = max(nk)
        if my == 0:
            kv += nkv
            yield from item_advance(W, item, not v.static_items)
            continue
        for j in range(my):
            yield ("wait", [(f"SF{t}", n_s)])
            n_s += 1
            yield ("read", ("S", t, agent), ("S", kv + j))
            if j > 0 and rng.random() < 0.3:
                # the kept max moves: O is rescaled, which needs P V(j-1)
                yield ("wait", [(f"OD{t}", n_s - 2)])
                yield ("read", ("O", t, 0), (item, j))
            yield ("write", ("S", t, agent), ("P", kv + j))
            yield ("arrive", f"PF{t}", n_s - 1)
        if not v.epilogue_no_od_wait:
            yield ("wait", [(f"OD{t}", n_s - 1)])
        yield ("read", ("O", t, 0), (item, my))
        yield ("arrive", f"OE{t}", done)
        done += 1
        kv += nkv
        yield from item_advance(W, item, not v.static_items)


def nagents(v):
    return 2 * NSM if v.split else NSM


def softmax_split(t, h, qq, plan, v, seed):
    """Half h (key columns 64 h ..) of row quarter qq of tile t."""
    agent = h * NSM + qq
    kv = n_s = done = 0
    for item, nk in enumerate(plan):
        my, nkv = nk[t], max(nk)
        if my == 0:
            kv += nkv
            yield from item_advance(W, item, not v.static_items)
            continue
        for j in range(my):
            yield ("wait", [(f"SF{t}", n_s)])
            slot = n_s & 1
            n_s += 1
            yield ("read", ("S", t, agent), ("S", kv + j))
            yield ("write", ("PMAX", t, slot, h, qq), kv + j)
            mx = f"MX{t}{qq}{n_s - 1 & 1}"
            yield ("arrive", mx, (n_s - 1) >> 1)
            if not v.split_no_exchange_wait:
                yield ("wait", [(mx, (n_s - 1) >> 1)])
            yield ("read", ("PMAX", t, slot, 1 - h, qq), kv + j)
            # both halves see the same row max, so they take the same decision
            if j > 0 and random.Random(seed * 1009 + t * 97 + qq * 13 + n_s).random() < 0.3:
                yield ("wait", [(f"OD{t}", n_s - 2)])
                yield ("read", ("O", t, h), (item, j))
            yield ("write", ("S", t, agent), ("P", kv + j))
            yield ("arrive", f"PF{t}", n_s - 1)
        yield ("wait", [(f"OD{t}", n_s - 1)])
        yield ("write", ("PSUM", t, h, qq), item)
        yield ("arrive", f"LX{t}{qq}", done)
        yield ("wait", [(f"LX{t}{qq}", done)])
        yield ("read", ("PSUM", t, 1 - h, qq), item)
        yield ("read", ("O", t, h), (item, my))
        yield ("arrive", f"OE{t}", done)
        done += 1
        kv += nkv
        yield from item_advance(W, item, not v.static_items)


def run_schedule(plan, seed, variant=None, max_steps=200000, in_order=False):
    """One random schedule of one CTA working through `plan`; raises
    ProtocolError on a violation or a deadlock.  in_order: complete each
    unit's asynchronous work in issue order."""
    global W
    v = variant or Variant()
    W = World()
    for t in range(2):
        W.bar(f"PF{t}", nagents(v))
        for b in range(2):
            W.bar(f"PF{t}{b}", nagents(v))
        W.bar(f"OE{t}", nagents(v))
        for qq in range(NSM):
            W.bar(f"LX{t}{qq}", 2)
            for sl in range(2):
                W.bar(f"MX{t}{qq}{sl}", 2)
    # one arrival per modelled agent frees a response slot
    n_consumers = 2 + 2 * nagents(v)
    W.bar("CLCE0", n_consumers)
    W.bar("CLCE1", n_consumers)
    roles = {"prod": producer(plan, v),
             "mma": issuer_sdouble(plan, v) if v.s_double else issuer(plan, v)}
    for t in range(2):
        if v.s_double:
            for a in range(NSM):
                roles[f"sm{t}{a}"] = softmax_sdouble(t, a, plan, v,
                                                     random.Random(seed * 7 + 2 * t + a))
        elif v.split:
            for h in range(2):
                for qq in range(NSM):
                    roles[f"sm{t}{h}{qq}"] = softmax_split(t, h, qq, plan, v, seed)
        else:
            for a in range(NSM):
                roles[f"sm{t}{a}"] = softmax(t, a, plan, v, random.Random(seed * 7 + 2 * t + a))
    run_roles(W, roles, seed, in_order, max_steps)
