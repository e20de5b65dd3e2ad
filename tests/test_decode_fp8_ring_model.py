"""A model of the 8-bit decode kernel's load and hand-over protocol
(compressed_long_context_hca_b200/csrc/decode_fp8.cu) with the hardware's parity-wait
rule, checked over random schedules on the CPU.

mbarrier semantics modelled: a barrier counts completed phases; a phase completes when its
expected arrivals (and, for a TMA box, the box's bytes) have come in; a wait on parity P
returns as soon as the phase count's parity differs from P (so a wait on a phase two
ahead of the current one returns at once). A tcgen05.commit arrives once every MMA its
issuing thread issued before it has completed, so the commits of one thread arrive in
order; TMA landings complete in any order.

The roles, restated from the kernel:
- the K load warp streams the K boxes of the split's tiles, in tile order, into a K ring
  (4 boxes per e4m3 tile; the window tile's 8 after its bf16 query, which waits until the
  last e4m3 score MMA has completed), each slot reused once the score MMAs released it;
- the V load warp streams the e4m3 V boxes (ceil(n / 32) per e4m3 tile) into a V ring,
  each slot reused once both 16-key groups of its box were widened;
- the score warp issues S(c) once its K boxes landed and the softmax of tile c - 2 has
  released score buffer c & 1;
- the converter warps widen the V groups in order into a ring of f16 buffers (the window
  tile's groups arrive there by TMA instead);
- the P.V warp consumes the f16 groups after the softmax of their tile and releases the V
  ring slot of a box once it has both of its groups;
- the softmax of tile c waits for its scores and for the P buffer it writes: an e4m3
  tile's P alternates between two buffers (free once P.V(c - 2) is done), the window
  tile's two parts take both (free once P.V(c - 1) is done).

Checked, over many random schedules and tile lists (one compressed tile and the window,
several partial tiles, window only, no window): no role waits forever, every box or buffer
a consumer reads holds what it expects (landed and not replaced), no score buffer is
overwritten while the softmax reads it, and no P buffer is rewritten while a P.V product
that reads it is in flight. Two deliberately broken variants must fail those checks.
"""

import random
from collections import deque

KSTAGES = 3    # K ring slots of the kernel
V8STAGES = 3   # V ring slots
VSTAGES = 2    # f16 V buffers


class Bar:
    def __init__(self, count):
        self.count = count
        self.arrived = 0
        self.tx = 0
        self.phase = 0          # completed phases

    def arrive(self, tx=0):
        self.arrived += 1
        self.tx += tx
        self._check()

    def land(self, tx):
        self.tx -= tx
        self._check()

    def _check(self):
        if self.arrived == self.count and self.tx == 0:
            self.phase += 1
            self.arrived = 0

    def ready(self, parity):
        return (self.phase & 1) != parity


def run(tiles, rng, nbuf=2, v_release_early=False):
    """tiles: list of (kind, n) with kind 'c' (e4m3 tile of n keys) or 'r' (window tile).
    nbuf: P buffers an e4m3 tile's P alternates over (1 models writing a single buffer
    under the same waits). v_release_early: the P.V warp releases a V ring slot after the
    first group of its box instead of both. Returns None when every role finished with valid reads, else
    a failure string."""
    B = {}
    for s in range(KSTAGES):
        B[("k_full", s)] = Bar(1)
        B[("k_empty", s)] = Bar(1)
    for s in range(V8STAGES):
        B[("v8_full", s)] = Bar(1)
        B[("v8_empty", s)] = Bar(1)
    for s in range(VSTAGES):
        B[("v_full", s)] = Bar(1)
        B[("v_empty", s)] = Bar(1)
    for x in range(2):
        B[("s_full", x)] = Bar(1)
        B[("p_full", x)] = Bar(1)
        B[("o_done", x)] = Bar(1)
    for name in ("q8_free", "qb_full", "q_ready"):
        B[(name,)] = Bar(1)
    kslot = [None] * KSTAGES     # box id in each K ring slot (after it landed)
    vslot = [None] * V8STAGES
    vbuf = [None] * VSTAGES
    pbuf = [None, None]          # tile whose P each buffer holds
    p_reading = set()            # buffers read by P.V products not yet completed
    s_reading = [None, None]     # tile whose scores the softmax is reading, per buffer
    v_reading = set()            # V ring slots the converters are reading
    queues = {}
    nland = [0]
    fail = []
    ntiles = len(tiles)
    has_ring = ntiles > 0 and tiles[-1][0] == "r"
    nct = ntiles - (1 if has_ring else 0)

    def post(key, fn):
        queues.setdefault(key, deque()).append(fn)

    def land_later(fn):
        nland[0] += 1
        post(("tma", nland[0]), fn)

    def commit(name, who):
        post(who, lambda: B[name].arrive())

    def p_bufs(c):
        if tiles[c][0] == "r":
            return [0, 1]
        return [c % nbuf]

    def vboxes(t):
        return -(-t[1] // 32) if t[0] == "c" else 0

    # ------------------------------------------------------------ roles as generators
    def ring_load(full, empty, stages, slots, cnt, box_id):
        s = cnt % stages
        if cnt >= stages:
            yield ("wait", (empty, s), ((cnt // stages) - 1) & 1)
        if full == "v8_full" and s in v_reading:
            fail.append(f"V box {box_id} loaded over a slot the converters read")
        B[(full, s)].arrive(tx=1)

        def landing(s=s, box_id=box_id):
            slots[s] = box_id
            B[(full, s)].land(1)
        land_later(landing)

    def producer_k():
        cnt = 0
        for c in range(ntiles):
            t = tiles[c]
            if t[0] == "r":
                yield ("wait", ("q8_free",), 0)
                B[("qb_full",)].arrive(tx=1)
                land_later(lambda: B[("qb_full",)].land(1))
            for q in range(4 if t[0] == "c" else 8):
                yield from ring_load("k_full", "k_empty", KSTAGES, kslot, cnt, ("K", c, q))
                cnt += 1

    def producer_v():
        cnt = 0
        for c in range(ntiles):
            for q in range(vboxes(tiles[c])):
                yield from ring_load("v8_full", "v8_empty", V8STAGES, vslot, cnt, ("V", c, q))
                cnt += 1

    def umma_s():
        yield ("wait", ("q_ready",), 0)
        n = 0
        released = False
        for c in range(ntiles):
            if c >= 2:
                # score buffer c & 1 is free once the softmax of tile c - 2 is done
                yield ("wait", ("p_full", c & 1), ((c - 2) >> 1) & 1)
                if s_reading[c & 1] is not None:
                    fail.append(f"S({c}) overwrote the scores of tile {s_reading[c & 1]}")
            t = tiles[c]
            if t[0] == "r":
                if not released:
                    commit(("q8_free",), "s")
                    released = True
                yield ("wait", ("qb_full",), 0)
            for q in range(4 if t[0] == "c" else 8):
                s = n % KSTAGES
                yield ("wait", ("k_full", s), (n // KSTAGES) & 1)
                if kslot[s] != ("K", c, q):
                    fail.append(f"S read {kslot[s]} for K{(c, q)}")
                commit(("k_empty", s), "s")
                n += 1
            commit(("s_full", c & 1), "s")
            if has_ring and c + 1 == nct and not released:
                commit(("q8_free",), "s")
                released = True

    def umma_pv():
        nv = 0
        cv = 0
        for pc in range(ntiles):
            t = tiles[pc]
            vstart = nv
            nv += vboxes(t)
            yield ("wait", ("p_full", pc & 1), (pc >> 1) & 1)
            bufs = p_bufs(pc)
            for x in bufs:
                if pbuf[x] != pc:
                    fail.append(f"PV({pc}) read P buffer {x} holding {pbuf[x]}")
                p_reading.add(x)
            ng = t[1] // 16
            for g in range(ng):
                s = cv % VSTAGES
                yield ("wait", ("v_full", s), (cv // VSTAGES) & 1)
                if vbuf[s] != (pc, g):
                    fail.append(f"PV read {vbuf[s]} for group {(pc, g)}")
                # the converters have read the e4m3 box of this group: released once both
                # of its groups (or the tile's last) are in
                last = g == ng - 1 or (g % 2 == 0 if v_release_early else g % 2 == 1)
                if t[0] == "c" and last:
                    B[("v8_empty", (vstart + g // 2) % V8STAGES)].arrive()
                commit(("v_empty", s), "pv")
                cv += 1

            def pv_done(pc=pc, bufs=tuple(bufs)):
                for x in bufs:
                    p_reading.discard(x)
                B[("o_done", pc & 1)].arrive()
            post("pv", pv_done)

    def softmax():
        yield ("wait", ("q_ready",), 0)
        for c in range(ntiles):
            yield ("wait", ("s_full", c & 1), (c >> 1) & 1)
            s_reading[c & 1] = c
            pv = c - 1 if tiles[c][0] == "r" else c - 2
            if pv >= 0:
                yield ("wait", ("o_done", pv & 1), (pv >> 1) & 1)
            for x in p_bufs(c):
                if x in p_reading:
                    fail.append(f"softmax({c}) rewrote P buffer {x} under a P.V product")
                pbuf[x] = c
            s_reading[c & 1] = None
            B[("p_full", c & 1)].arrive()

    def converter():
        B[("q_ready",)].arrive()
        n = 0
        cv = 0
        for c in range(ntiles):
            t = tiles[c]
            ng = t[1] // 16
            for g in range(ng):
                vs = cv % VSTAGES
                if t[0] == "c" and g % 2 == 0:
                    sidx = n + g // 2
                    yield ("wait", ("v8_full", sidx % V8STAGES), (sidx // V8STAGES) & 1)
                if cv >= VSTAGES:
                    yield ("wait", ("v_empty", vs), ((cv // VSTAGES) - 1) & 1)
                if t[0] == "c":
                    rs = (n + g // 2) % V8STAGES
                    if vslot[rs] != ("V", c, g // 2):
                        fail.append(f"converter read {vslot[rs]} for V{(c, g // 2)}")
                    v_reading.add(rs)
                    vbuf[vs] = (c, g)
                    B[("v_full", vs)].arrive()
                    if g % 2 == 1 or g == ng - 1:
                        v_reading.discard(rs)
                else:
                    B[("v_full", vs)].arrive(tx=1)

                    def landing(vs=vs, key=(c, g)):
                        vbuf[vs] = key
                        B[("v_full", vs)].land(1)
                    land_later(landing)
                cv += 1
            n += vboxes(t)

    roles = {"producer_k": producer_k(), "producer_v": producer_v(), "umma_s": umma_s(),
             "umma_pv": umma_pv(), "softmax": softmax(), "converter": converter()}
    waiting = {name: None for name in roles}
    for _ in range(200000):
        runnable = [r for r in roles if waiting[r] is None or
                    B[waiting[r][0]].ready(waiting[r][1])]
        live = [k for k, q in queues.items() if q]
        if not runnable and not live:
            break
        if live and (not runnable or rng.random() < 0.3):
            queues[rng.choice(live)].popleft()()
            continue
        r = rng.choice(runnable)
        waiting[r] = None
        try:
            req = next(roles[r])
            waiting[r] = (req[1], req[2])
        except StopIteration:
            del roles[r]
            del waiting[r]
        if fail:
            return fail[0]
    if roles:
        return "deadlock: " + ", ".join(f"{r} waits {waiting[r]}" for r in roles)
    return None


def _tile_lists(rng):
    yield [("c", 80), ("r", 128)]           # one partial compressed tile + the window
    yield [("c", 128), ("r", 128)]
    yield [("c", 128)] * 3 + [("c", 48), ("r", 112)]
    yield [("r", 64)]                       # window only
    yield [("c", 128)] * 4                  # a split without the window
    yield [("c", 16)]
    for _ in range(20):
        n = rng.randint(1, 6)
        tl = [("c", 128)] * (n - 1) + [("c", 16 * rng.randint(1, 8))]
        if rng.random() < 0.6:
            tl.append(("r", 16 * rng.randint(1, 8)))
        yield tl


def test_protocol_never_misreads_or_deadlocks():
    rng = random.Random(7)
    for tiles in _tile_lists(random.Random(3)):
        for _ in range(30):
            res = run(tiles, rng)
            assert res is None, (tiles, res)


def test_one_p_buffer_with_the_same_waits_races():
    # writing every e4m3 tile's P to one buffer while waiting only for P.V(c - 2) rewrites
    # the buffer that P.V(c - 1) may still be reading
    rng = random.Random(5)
    failures = [run([("c", 128)] * 4 + [("r", 128)], rng, nbuf=1) for _ in range(200)]
    assert any(f is not None and "rewrote" in f for f in failures)


def test_v_box_released_after_one_group_is_caught():
    # releasing a V ring slot after the first of its two groups lets the V load warp
    # overwrite a box whose second group the converters still have to widen
    rng = random.Random(9)
    failures = [run([("c", 128)] * 3 + [("r", 128)], rng, v_release_early=True)
                for _ in range(200)]
    assert any(f is not None and ("converter read" in f or "loaded over" in f)
               for f in failures)
