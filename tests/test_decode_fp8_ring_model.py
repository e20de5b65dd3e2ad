"""A model of the 8-bit decode kernel's load ring (csrc/decode_fp8.cu) with the hardware's
parity-wait rule, checked over random schedules on the CPU.

mbarrier semantics modelled: a barrier counts completed phases; a phase completes when its
expected arrivals (and, for a TMA box, the box's bytes) have come in; a wait on parity P
returns as soon as the phase count's parity differs from P (so a wait on a phase two
ahead of the current one returns at once: the aliasing the kernel must avoid).

The roles, restated from the kernel: the load warp issues, in order, K(0), then per step
c >= 1: K(c), V(c - 1), into a ring of 5 slots (waiting for the slot's previous box to be
released); a compressed tile is 4 K boxes and ceil(n / 32) V boxes, the window tile 8 K
boxes (and its bf16 query, after the last e4m3 score MMA); one UMMA warp consumes the K
boxes in order for the score MMAs, S(c) once the softmax of tile c - 2 has released score
buffer c & 1, and a second UMMA warp consumes the V groups from a 3-slot buffer ring after
the softmax of each tile;
the converter warps consume the V boxes in order, two 16-key groups per box, into the
buffer ring, and the P.V warp releases a V box once it has both of its groups; the
softmax of tile c waits for its scores and for the P buffer it writes: an e4m3 tile's P
alternates between two buffers (free once P.V(c - 2) is done), the window tile's two
parts take both (free once P.V(c - 1) is done). Asynchronous completions (TMA landings,
MMA commits) happen at random later times.

Checked, over many random schedules and tile lists (one compressed tile and the window,
several partial tiles, window only, no window): no role waits forever, every box a
consumer reads is the box it expects (it has landed and has not been replaced), and no P
buffer is rewritten while a P.V product that reads it is in flight. The same
model with one shared full barrier per slot (the consumers waiting on parities of the
slot's position in the load order) must fail the second check for a split made of one
compressed tile and the window tile.
"""

import random

STAGES = 5    # load ring slots of the kernel
VSTAGES = 3   # V buffer slots


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


def run(tiles, typed, rng, nbuf=2):
    """tiles: list of (kind, n) with kind 'c' (e4m3 tile of n keys) or 'r' (window tile).
    nbuf: P buffers an e4m3 tile's P alternates over (1 models writing a single buffer
    under the same waits). Returns None when every role finished with valid reads, else a
    failure string."""

    def p_bufs(c):
        if tiles[c][0] == "r":
            return [0, 1]
        return [c % nbuf]
    B = {}
    for s in range(STAGES):
        B[("k_full", s)] = Bar(1)
        B[("v8_full", s)] = Bar(1)
        B[("ring_empty", s)] = Bar(1)
    for s in range(VSTAGES):
        B[("v_full", s)] = Bar(1)
        B[("v_empty", s)] = Bar(1)
    for x in range(2):
        B[("s_full", x)] = Bar(1)
        B[("p_full", x)] = Bar(1)
        B[("o_done", x)] = Bar(1)
    for name in ("q8_free", "qb_full", "q_ready"):
        B[(name,)] = Bar(1)
    slot_box = [None] * STAGES   # box id currently in the slot (after it landed)
    vbuf = [None] * VSTAGES
    pbuf = [None, None]          # tile whose P each buffer holds
    s_reading = [None, None]     # tile whose scores the softmax is reading, per buffer
    p_reading = set()            # buffers read by P.V products not yet completed
    pending = []                 # async events: (callable)
    fail = []
    ntiles = len(tiles)
    has_ring = ntiles > 0 and tiles[-1][0] == "r"
    nct = ntiles - (1 if has_ring else 0)

    def kboxes(t):
        return 4 if t[0] == "c" else 8

    def vboxes(t):
        return -(-t[1] // 32) if t[0] == "c" else 0

    def full_bar(kind, s):
        return B[(kind if typed else "k_full", s)]

    # ------------------------------------------------------------ roles as generators
    def producer():
        cnt = 0

        def load(kind, box_id):
            nonlocal cnt
            s = cnt % STAGES
            if cnt >= STAGES:
                yield ("wait", ("ring_empty", s), ((cnt // STAGES) - 1) & 1)
            bar = full_bar(kind, s)
            bar.arrive(tx=1)

            def landing(s=s, bar=bar, box_id=box_id):
                slot_box[s] = box_id
                bar.land(1)
            pending.append(landing)
            cnt += 1

        for c in range(ntiles + 1):
            if c < ntiles:
                t = tiles[c]
                if t[0] == "c":
                    for q in range(4):
                        yield from load("k_full", ("K", c, q))
                else:
                    yield ("wait", ("q8_free",), 0)
                    B[("qb_full",)].arrive(tx=1)
                    pending.append(lambda: B[("qb_full",)].land(1))
                    for q in range(8):
                        yield from load("k_full", ("K", c, q))
            if c >= 1:
                t = tiles[c - 1]
                for q in range(vboxes(t)):
                    yield from load("v8_full", ("V", c - 1, q))

    def commit(name):
        # a tcgen05.commit: arrives once the MMAs issued so far have completed
        pending.append(lambda: B[name].arrive())

    def umma_s():
        yield ("wait", ("q_ready",), 0)
        n = 0
        kph = [0] * STAGES
        released = False
        for c in range(ntiles):
            if c >= 2:
                n += vboxes(tiles[c - 2])
                # score buffer c & 1 is free once the softmax of tile c - 2 is done
                yield ("wait", ("p_full", c & 1), ((c - 2) >> 1) & 1)
                if s_reading[c & 1] is not None:
                    fail.append(f"S({c}) overwrote the scores of tile {s_reading[c & 1]}")
            t = tiles[c]
            if t[0] == "r":
                if not released:
                    commit(("q8_free",))
                    released = True
                yield ("wait", ("qb_full",), 0)
            for q in range(kboxes(t)):
                s = n % STAGES
                if typed:
                    yield ("wait", ("k_full", s), kph[s])
                    kph[s] ^= 1
                else:
                    yield ("wait", ("k_full", s), (n // STAGES) & 1)
                if slot_box[s] != ("K", c, q):
                    fail.append(f"UMMA read {slot_box[s]} for K{(c, q)}")
                commit(("ring_empty", s))
                n += 1
            commit(("s_full", c & 1))
            if has_ring and c + 1 == nct and not released:
                commit(("q8_free",))
                released = True

    def umma_pv():
        nk = kboxes(tiles[0]) if ntiles else 0
        nv = 0
        cv = 0
        for pc in range(ntiles):
            t = tiles[pc]
            if pc + 1 < ntiles:
                nk += kboxes(tiles[pc + 1])
            vstart = nk + nv
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
                if t[0] == "c" and (g % 2 == 1 or g == ng - 1):
                    B[("ring_empty", (vstart + g // 2) % STAGES)].arrive()
                commit(("v_empty", s))
                cv += 1

            def pv_done(pc=pc, bufs=tuple(bufs)):
                for x in bufs:
                    p_reading.discard(x)
                B[("o_done", pc & 1)].arrive()
            pending.append(pv_done)

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
        vph = [0] * STAGES
        cv = 0
        for c in range(ntiles + 1):
            if c < ntiles:
                n += kboxes(tiles[c])
            if c == 0:
                continue
            t = tiles[c - 1]
            ng = t[1] // 16
            if t[0] == "c":
                for g in range(ng):
                    sidx = n + (g >> 1)
                    rs = sidx % STAGES
                    if g % 2 == 0:
                        if typed:
                            yield ("wait", ("v8_full", rs), vph[rs])
                            vph[rs] ^= 1
                        else:
                            yield ("wait", ("k_full", rs), (sidx // STAGES) & 1)
                    vs = cv % VSTAGES
                    if cv >= VSTAGES:
                        yield ("wait", ("v_empty", vs), ((cv // VSTAGES) - 1) & 1)
                    if slot_box[rs] != ("V", c - 1, g >> 1):
                        fail.append(f"converter read {slot_box[rs]} for V{(c - 1, g >> 1)}")
                    vbuf[vs] = (c - 1, g)
                    B[("v_full", vs)].arrive()
                    cv += 1
                n += vboxes(t)
            else:
                for g in range(ng):
                    vs = cv % VSTAGES
                    if cv >= VSTAGES:
                        yield ("wait", ("v_empty", vs), ((cv // VSTAGES) - 1) & 1)
                    B[("v_full", vs)].arrive(tx=1)

                    def landing(vs=vs, key=(c - 1, g)):
                        vbuf[vs] = key
                        B[("v_full", vs)].land(1)
                    pending.append(landing)
                    cv += 1

    roles = {"producer": producer(), "umma_s": umma_s(), "umma_pv": umma_pv(),
             "softmax": softmax(), "converter": converter()}
    waiting = {name: None for name in roles}
    for _ in range(200000):
        runnable = [r for r in roles if waiting[r] is None or
                    B[waiting[r][0]].ready(waiting[r][1])]
        if not runnable and not pending:
            break
        if pending and (not runnable or rng.random() < 0.3):
            pending.pop(rng.randrange(len(pending)))()
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


def test_typed_ring_never_aliases_or_deadlocks():
    rng = random.Random(7)
    for tiles in _tile_lists(random.Random(3)):
        for _ in range(30):
            res = run(tiles, True, rng)
            assert res is None, (tiles, res)


def test_shared_parity_ring_aliases():
    # the same ring with one full barrier per slot: the converter's wait on a V box two
    # phases ahead returns at once and reads a slot that does not hold its box
    rng = random.Random(11)
    failures = [run([("c", 80), ("r", 128)], False, rng) for _ in range(200)]
    assert any(f is not None and "read" in f for f in failures)


def test_one_p_buffer_with_the_same_waits_races():
    # writing every e4m3 tile's P to one buffer while waiting only for P.V(c - 2) rewrites
    # the buffer that P.V(c - 1) may still be reading
    rng = random.Random(5)
    failures = [run([("c", 128)] * 4 + [("r", 128)], True, rng, nbuf=1) for _ in range(200)]
    assert any(f is not None and "rewrote" in f for f in failures)
