"""CPU model of attn_sdpa_host's stream and event protocol (csrc/attn.cu).

Streams are FIFOs of operations; cudaStreamWaitEvent refers to the most recent
cudaEventRecord of that event at the time of the wait call (none: no-op).  A
random scheduler runs any stream whose head is ready.  Buffers carry versions:
every read must see the version it needs, so a copy that overwrites a slot
still in use, or a kernel that reads a slot before its copy landed, fails.
Several calls run back to back on the same internal streams and events, and
the caller's stream consumes each call's host outputs after the call.
"""
import random

K_SLOTS = 3


class Sim:
    def __init__(self):
        self.streams = {n: [] for n in ("user", "in", "cmp", "out")}
        self.last_record = {}      # event -> record id (host order)
        self.done_records = set()  # record ids whose stream position was reached
        self.buf = {}
        self.rid = 0

    # host-side API, in host order
    def record(self, ev, stream):
        self.rid += 1
        rid = self.rid
        self.last_record[ev] = rid
        self.streams[stream].append(("record", rid))

    def wait(self, stream, ev):
        rid = self.last_record.get(ev)  # None: never recorded -> no-op
        self.streams[stream].append(("wait", rid))

    def op(self, stream, fn):
        self.streams[stream].append(("op", fn))

    # device side
    def ready(self, s):
        q = self.streams[s]
        if not q:
            return False
        kind, x = q[0]
        return kind != "wait" or x is None or x in self.done_records

    def step(self, rng):
        cand = [s for s in self.streams if self.ready(s)]
        if not cand:
            if any(self.streams.values()):
                raise AssertionError("deadlock")
            return False
        s = rng.choice(cand)
        kind, x = self.streams[s].pop(0)
        if kind == "record":
            self.done_records.add(x)
        elif kind == "op":
            x()
        return True

    def read(self, key, want):
        if self.buf.get(key) != want:
            raise AssertionError(f"read {key}: want {want}, have {self.buf.get(key)}")

    def write(self, key, val):
        self.buf[key] = val


def enqueue_call(sim, call, BH, hc, drop=()):
    """The enqueue sequence of attn_sdpa_host, in host order.  ``drop`` names
    waits to leave out (planted mistakes): start, drained, loaded, computed,
    done."""
    sim.record("start", "user")
    for s in ("in", "cmp", "out"):
        if "start" not in drop:
            sim.wait(s, "start")
    c, h0 = 0, 0
    while h0 < BH:
        n = min(hc, BH - h0)
        slot = c % K_SLOTS
        tag = (call, c)
        if "drained" not in drop:
            sim.wait("in", f"drained{slot}")

        def h2d(slot=slot, tag=tag, call=call, c=c):
            sim.read(("host_in", call), call)         # the caller's inputs of this call
            for t in ("q", "k", "v", "do"):
                sim.write((t, slot), tag)
        sim.op("in", h2d)
        sim.record(f"loaded{slot}", "in")
        if "loaded" not in drop:
            sim.wait("cmp", f"loaded{slot}")

        def kernels(slot=slot, tag=tag):
            for t in ("q", "k", "v", "do"):
                sim.read((t, slot), tag)
            sim.write(("ws",), tag)                  # the one backward workspace
            sim.write(("o", slot), tag)
            sim.read(("ws",), tag)
            for t in ("dq", "dk", "dv"):
                sim.write((t, slot), tag)
        sim.op("cmp", kernels)
        sim.record(f"computed{slot}", "cmp")
        if "computed" not in drop:
            sim.wait("out", f"computed{slot}")

        def d2h(slot=slot, tag=tag, call=call, c=c):
            for t in ("o", "dq", "dk", "dv"):
                sim.read((t, slot), tag)
                sim.write(("host_out", call, c, t), tag)
        sim.op("out", d2h)
        sim.record(f"drained{slot}", "out")
        c += 1
        h0 += hc
    sim.record("done", "out")
    if "done" not in drop:
        sim.wait("user", "done")
    return c


def run(seed, calls=3, BH=7, hc=2, drop=()):
    rng = random.Random(seed)
    sim = Sim()
    for call in range(calls):
        # the caller fills its host inputs for this call on its stream, calls,
        # then consumes the outputs after the call (stream order)
        sim.op("user", lambda call=call: sim.write(("host_in", call), call))
        nchunks = enqueue_call(sim, call, BH, hc, drop)

        def consume(call=call, nchunks=nchunks):
            for c in range(nchunks):
                for t in ("o", "dq", "dk", "dv"):
                    sim.read(("host_out", call, c, t), (call, c))
        sim.op("user", consume)
        # interleave some device progress with the host enqueueing
        for _ in range(rng.randrange(0, 40)):
            if not sim.step(rng):
                break
    while sim.step(rng):
        pass

