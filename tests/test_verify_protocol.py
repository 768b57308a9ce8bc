"""Random-schedule model of the tensor-memory verify kernel's cross-role protocol
(sparse_dense_kv_b200/csrc/verify_tc.cu), kept by hand in step with the kernel.

Roles: the K producer (claims chunk ids and publishes them, one ahead of its own progress,
through a ring of kRing slots with one barrier per slot, once the current chunk's first K
tile is issued; loads Q into one of two buffers one chunk ahead and the K tiles through its
2-stage ring), the V producer (reads the ids from the ring after its chunk's first V tile,
V tiles through its own 2-stage ring), the QK issuer (chunk after chunk: Q, a free S buffer,
each K tile) and the PV issuer (chunk after chunk: the whole P^T, a free O buffer, each V
tile), and 8 softmax warps in two warpgroups (S double buffer, per-tile P^T release by the
previous chunk's PV, O double buffer, warpgroup barriers). Each step of each role is an arrive or a wait on a phase-parity barrier, as in
the kernel; a scheduler picks a random role at every step.

Checked over many random schedules and chunk / tile counts: the roles never deadlock, and
no ring slot is overwritten before every read of its previous id (the V producer reads
each id once, the QK and the PV issuer once each, each softmax warp once). Over such schedules the smallest ring that never fails is 6 slots (5
fails now and then); the kernel has 16. A ring of 4 slots must fail the overwrite check
(negative control).
"""
import random

import pytest


class Bar:
    """An mbarrier: `count` arrivals complete a phase; a wait on parity p passes once the
    phase with that parity has completed."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.phases = 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier expects"
        if self.pending == 0:
            self.phases += 1
            self.pending = self.count

    def test(self, parity):
        return (self.phases & 1) != parity


def run(ntiles, ring, seed, kst=2, vst=2, KT=7, limit=20000):
    """One random schedule; returns None, "deadlock" or "overwrite"."""
    rnd = random.Random(seed)
    M = len(ntiles)
    bars = {}

    def bar(name, count=1):
        if name not in bars:
            bars[name] = Bar(count)
        return bars[name]

    for s in range(kst):
        bar(f"kfull{s}"), bar(f"kempty{s}")
    for s in range(vst):
        bar(f"vfull{s}"), bar(f"vempty{s}")
    for b in range(2):
        bar(f"qfull{b}"), bar(f"qempty{b}"), bar(f"sfull{b}"), bar(f"sempty{b}", 8)
        bar(f"ofull{b}"), bar(f"oempty{b}", 8)
    for t in range(8):
        bar(f"pfree{t}")
    for g in range(2):
        bar(f"wg{g}", 4)
    bar("pfull", 8)
    for s in range(ring):
        bar(f"item{s}")

    slot_item = {}                 # slot -> id published there last
    reads = {}                     # id -> reads done
    NEED = 1 + 2 + 8               # V producer, the QK and PV issuers, 8 softmax warps
    state = {"overwrite": False}

    def W(name, parity):
        return ("wait", name, parity)

    def A(name):
        return ("arrive", name)

    def publish(m):                # K producer: id m (M = no more work) into slot m % ring
        slot = m % ring
        prev = slot_item.get(slot)
        if prev is not None and reads.get(prev, 0) < NEED:
            state["overwrite"] = True
        slot_item[slot] = m
        reads[m] = 0
        return A(f"item{slot}")

    def read(m):                   # after the wait on the slot's barrier
        if slot_item.get(m % ring) != m:
            state["overwrite"] = True
        reads[m] = reads.get(m, 0) + 1
        return ("nop",)

    def W_item(m):
        return W(f"item{m % ring}", (m // ring) & 1)

    def kprod():
        # item m+1 is claimed and published, and its Q rows loaded, once item m's first K
        # tile is on its way
        g = 0
        yield publish(0)
        if M > 0:
            yield A("qfull0")
        for m in range(M):
            for t in range(ntiles[m]):
                s = g % kst
                if g >= kst:
                    yield W(f"kempty{s}", ((g // kst) - 1) & 1)
                yield A(f"kfull{s}")
                g += 1
                if t == 0:
                    yield publish(m + 1)
                    if m + 1 < M:
                        if m + 1 >= 2:
                            yield W(f"qempty{(m + 1) & 1}", ((m - 1) >> 1) & 1)
                        yield A(f"qfull{(m + 1) & 1}")

    def vprod():
        # the id of item m+1 is read from the ring once item m's first V tile is on its way
        g = 0
        yield W_item(0)
        yield read(0)
        for m in range(M):
            for t in range(ntiles[m]):
                s = g % vst
                if g >= vst:
                    yield W(f"vempty{s}", ((g // vst) - 1) & 1)
                yield A(f"vfull{s}")
                g += 1
                if t == 0:
                    yield W_item(m + 1)
                    yield read(m + 1)

    def qk():
        gk = 0
        for mk in range(M + 1):
            yield W_item(mk)
            yield read(mk)
            if mk == M:
                return
            yield W(f"qfull{mk & 1}", (mk >> 1) & 1)
            if mk >= 2:
                yield W(f"sempty{mk & 1}", ((mk - 2) >> 1) & 1)
            for _ in range(ntiles[mk]):
                s = gk % kst
                yield W(f"kfull{s}", (gk // kst) & 1)
                yield A(f"kempty{s}")
                gk += 1
            yield A(f"sfull{mk & 1}")
            yield A(f"qempty{mk & 1}")

    def pv():
        gv = 0
        for nv in range(M + 1):
            yield W_item(nv)
            yield read(nv)
            if nv == M:
                return
            yield W("pfull", nv & 1)
            if nv >= 2:
                yield W(f"oempty{nv & 1}", ((nv - 2) >> 1) & 1)
            for tv in range(ntiles[nv]):
                s = gv % vst
                yield W(f"vfull{s}", (gv // vst) & 1)
                yield A(f"vempty{s}")
                yield A(f"pfree{tv}")
                gv += 1
            for t in range(ntiles[nv], KT):
                yield A(f"pfree{t}")
            yield A(f"ofull{nv & 1}")

    def soft(w):
        sg = w // 4
        ph = 0
        n = 0
        while True:
            yield W_item(n)
            yield read(n)
            if n == M:
                break
            yield W(f"sfull{n & 1}", (n >> 1) & 1)
            yield A(f"wg{sg}")
            yield W(f"wg{sg}", ph)
            ph ^= 1
            yield A(f"wg{sg}")
            yield W(f"wg{sg}", ph)
            ph ^= 1
            for t in range(ntiles[n]):
                if n > 0:
                    yield W(f"pfree{t}", (n - 1) & 1)
            yield A(f"sempty{n & 1}")
            yield A("pfull")
            if n > 0:
                m = n - 1
                yield W(f"ofull{m & 1}", (m >> 1) & 1)
                yield A(f"oempty{m & 1}")
            yield A(f"wg{sg}")
            yield W(f"wg{sg}", ph)
            ph ^= 1
            n += 1
        if M > 0:
            yield A(f"wg{sg}")
            yield W(f"wg{sg}", ph)
            m = M - 1
            yield W(f"ofull{m & 1}", (m >> 1) & 1)
            yield A(f"oempty{m & 1}")

    roles = {"K": kprod(), "V": vprod(), "QK": qk(), "PV": pv()}
    for w in range(8):
        roles[f"S{w}"] = soft(w)
    cur = {r: next(g) for r, g in roles.items()}
    done = set()
    stall = 0
    while len(done) < len(roles):
        r = rnd.choice([x for x in roles if x not in done])
        op = cur[r]
        ok = True
        if op[0] == "wait":
            ok = bars[op[1]].test(op[2])
        elif op[0] == "arrive":
            bars[op[1]].arrive()
        elif op[0] == "idle":
            ok = False
        if ok or op[0] == "idle":
            try:
                cur[r] = next(roles[r])
            except StopIteration:
                done.add(r)
        if state["overwrite"]:
            return "overwrite"
        stall = 0 if ok else stall + 1
        if stall > limit:
            return "deadlock"
    return None


@pytest.mark.parametrize("block", range(4))
def test_protocol_has_no_deadlock_and_no_early_overwrite(block):
    for trial in range(block * 100, block * 100 + 100):
        rnd = random.Random(trial)
        M = rnd.randint(0, 40)
        ntiles = [rnd.randint(1, 7) for _ in range(M)]
        assert run(ntiles, ring=16, seed=trial) is None, (trial, ntiles)


def test_a_four_slot_ring_is_caught_overwriting():
    bad = 0
    for trial in range(200):
        rnd = random.Random(trial)
        ntiles = [rnd.randint(1, 7) for _ in range(rnd.randint(8, 30))]
        bad += run(ntiles, ring=4, seed=trial) == "overwrite"
    assert bad > 0
