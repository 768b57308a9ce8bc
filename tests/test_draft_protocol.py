"""CPU models of the persistent sparse draft kernel (sparse_dense_kv_b200/csrc/draft.cu),
kept by hand in step with it.

1. The work split: every CTA takes one share of the launch's (request, KV head) pairs laid
   end to end; the share is at least ceil(P / CTAs), a third of the longest pair and one
   64-position tile. Checked on random length mixes (including empty pairs, a single pair,
   far more CTAs than work): every position of every pair lands in exactly one segment,
   a pair has at most 4 segments (the records of the workspace), each segment's record
   index j is in [0, nseg), the tiles of a share are what the roles count, and the pair's
   segments agree on nseg.
2. The warp roles' barrier protocol under random schedules: the index warp (segment slots
   with their query rows, row-id slots kBatchTiles at a time), the gather warps (row ids ->
   K/V stage), the attention warps (stage -> compute, segment slots opened on a segment's
   first tile and released after its last). No schedule deadlocks, and no slot (segment,
   row ids, stage) is rewritten before every reader of its previous contents has read it.
   Smaller rings than the kernel's must still be safe; a model that drops the wait on a
   free row-id slot must be caught (negative control).
"""
import random

import numpy as np
import pytest

from tests.test_verify_protocol import Bar

TILE, SEGMAX = 64, 4


def split(A, nctas):
    """Segments per CTA as the kernel walks them: (pair, a0, a1, j, nseg)."""
    pref = np.concatenate([[0], np.cumsum(A)]).astype(np.int64)
    P, amax = int(pref[-1]), int(max(A) if len(A) else 0)
    share = max(-(-P // nctas), -(-amax // (SEGMAX - 1)), TILE)
    out = []
    for c in range(nctas):
        lo, hi = c * share, min(P, (c + 1) * share)
        segs = []
        if lo < hi:
            for p in range(len(A)):
                if pref[p + 1] <= lo or pref[p + 1] == pref[p]:
                    continue
                if pref[p] >= hi:
                    break
                a0, a1 = max(lo, pref[p]) - pref[p], min(hi, pref[p + 1]) - pref[p]
                cf, cl = pref[p] // share, (pref[p + 1] - 1) // share
                segs.append((p, int(a0), int(a1), int(c - cf), int(cl - cf + 1)))
        out.append(segs)
    return out, share


@pytest.mark.parametrize("seed", range(60))
def test_split_covers_every_position_once(seed):
    rng = np.random.default_rng(seed)
    npairs = int(rng.integers(1, 300))
    kind = seed % 4
    if kind == 0:
        A = rng.integers(1, 1300, npairs)
    elif kind == 1:
        A = rng.integers(0, 40, npairs)               # short pairs, some empty
    elif kind == 2:
        A = np.where(rng.random(npairs) < 0.1, rng.integers(3000, 5000, npairs), rng.integers(1, 100, npairs))
    else:
        A = np.full(npairs, int(rng.integers(1, 2000)))
    nctas = int(rng.choice([1, 3, 148, 1000]))
    segs, share = split(A, nctas)
    seen = [np.zeros(a, dtype=np.int64) for a in A]
    per_pair = {}
    for c, ss in enumerate(segs):
        for p, a0, a1, j, nseg in ss:
            assert 0 <= a0 < a1 <= A[p]
            seen[p][a0:a1] += 1
            assert 0 <= j < nseg <= SEGMAX
            per_pair.setdefault(p, set()).add((j, nseg))
    for p, a in enumerate(A):
        assert np.all(seen[p] == 1), p
        if a:
            js = per_pair[p]
            nseg = {n for _, n in js}
            assert len(nseg) == 1 and sorted(j for j, _ in js) == list(range(nseg.pop()))


def test_split_of_the_qwen3_8b_workload_is_balanced():
    rng = np.random.default_rng(2)
    L = rng.integers(8192, 24577, 32)
    n = np.maximum(-(-(L * 500) // 10000), 64)
    A = np.repeat(n, 8) + 4                         # draft step 3
    segs, share = split(A, 148)
    rows = [sum(a1 - a0 for _, a0, a1, _, _ in ss) for ss in segs]
    busy = [r for r in rows if r]
    assert max(busy) == share and len(busy) >= 147
    assert max(len(ss) for ss in segs) <= 5      # segments a share touches (8 segment slots)


# ------------------------------------------------------------------ protocol model ----
def run(seg_tiles, seed, nst=4, offr=16, segr=8, batch=4, drop_off_wait=False, limit=200000):
    """One random schedule of one CTA with the given tiles per segment. Returns None,
    "deadlock" or "overwrite"."""
    rnd = random.Random(seed)
    tiles = [(k, tl, n) for k, n in enumerate(seg_tiles) for tl in range(n)]
    T, S = len(tiles), len(seg_tiles)
    bars = {}

    def bar(name, count=1):
        if name not in bars:
            bars[name] = Bar(count)
        return bars[name]

    for s in range(nst):
        bar(f"full{s}", 2 * 32 + 1), bar(f"empty{s}", 4)
    for s in range(offr):
        bar(f"offfull{s}"), bar(f"offempty{s}", 2)
    for s in range(segr):
        bar(f"segfull{s}"), bar(f"segempty{s}")
    bar("grp", 4)
    slot = {"seg": {}, "off": {}, "stage": {}}
    reads = {}
    bad = {"overwrite": False}
    NEED = {"seg": 4 + 4, "off": 2, "stage": 4}    # readers of each slot's contents

    def write(kind, s, item):
        prev = slot[kind].get(s)
        if prev is not None and reads.get((kind, prev), 0) < NEED[kind]:
            bad["overwrite"] = True
        slot[kind][s] = item
        reads[(kind, item)] = 0
        return ("nop",)

    def read(kind, s, item):
        if slot[kind].get(s) != item:
            bad["overwrite"] = True
        reads[(kind, item)] = reads.get((kind, item), 0) + 1
        return ("nop",)

    W = lambda name, parity: ("wait", name, parity)   # noqa: E731
    A = lambda name: ("arrive", name)                 # noqa: E731

    def index():
        t = 0
        for k, n in enumerate(seg_tiles):
            ss = k % segr
            if k >= segr:
                yield W(f"segempty{ss}", ((k // segr) - 1) & 1)
            yield write("seg", ss, k)
            yield A(f"segfull{ss}")
            for tb in range(0, n, batch):
                nb = min(batch, n - tb)
                if not drop_off_wait:
                    for u in range(nb):
                        if t + u >= offr:
                            yield W(f"offempty{(t + u) % offr}", (((t + u) // offr) - 1) & 1)
                for u in range(nb):
                    yield write("off", (t + u) % offr, t + u)
                for u in range(nb):
                    yield A(f"offfull{(t + u) % offr}")
                t += nb

    def gather(g):
        for t in range(T):
            ts, s = t % offr, t % nst
            yield W(f"offfull{ts}", (t // offr) & 1)
            if t >= nst:
                yield W(f"empty{s}", ((t // nst) - 1) & 1)
            yield read("off", ts, t)
            if g == 0:
                yield write("stage", s, t)            # the tile's rows and its meta land here
            for _ in range(32):
                yield A(f"full{s}")                   # each lane's copies land
            if g == 0:
                yield A(f"full{s}")                   # the meta arrive
            yield A(f"offempty{ts}")

    def attn(w):
        segk, ph = 0, 0
        for t, (k, tl, n) in enumerate(tiles):
            s = t % nst
            yield W(f"full{s}", (t // nst) & 1)
            yield read("stage", s, t)
            if tl == 0:
                yield W(f"segfull{k % segr}", (segk // segr) & 1)
                yield read("seg", k % segr, k)        # each warp loads the query rows
            yield A(f"empty{s}")
            if tl == n - 1:
                yield read("seg", k % segr, k)        # each warp reads the description
                for _ in range(3):                    # group barriers of the segment's end
                    yield A("grp")
                    yield W("grp", ph)
                    ph ^= 1
                if w == 0:
                    yield A(f"segempty{k % segr}")
                segk += 1

    roles = [index(), gather(0), gather(1)] + [attn(w) for w in range(4)]
    pending = [None] * len(roles)
    done = [False] * len(roles)
    steps = 0
    while not all(done):
        steps += 1
        if steps > limit:
            return "deadlock"
        ready = []
        for i, g in enumerate(roles):
            if done[i]:
                continue
            op = pending[i]
            if op is not None and op[0] == "wait" and not bars[op[1]].test(op[2]):
                continue
            ready.append(i)
        if not ready:
            return "deadlock"
        i = rnd.choice(ready)
        op = pending[i]
        if op is not None and op[0] == "arrive":
            bars[op[1]].arrive()
        try:
            pending[i] = next(roles[i])
        except StopIteration:
            done[i] = True
        if bad["overwrite"]:
            return "overwrite"
    return None


@pytest.mark.parametrize("seed", range(40))
def test_roles_never_deadlock_or_overwrite(seed):
    rng = random.Random(seed)
    seg_tiles = [rng.choice([1, 1, 2, 3, 5, 9, 23]) for _ in range(rng.randint(1, 14))]
    assert run(seg_tiles, seed) is None
    # rings smaller than the kernel's are safe too (the protocol does not rely on depth)
    assert run(seg_tiles, seed + 1000, nst=2, offr=4, segr=2, batch=2) is None


def test_dropping_the_row_id_slot_wait_is_caught():
    fails = sum(run([9, 9, 9], s, offr=4, batch=4, drop_off_wait=True) == "overwrite" for s in range(30))
    assert fails > 0
