"""A model of the prefill pair kernel's K/V load streams and of the rule its abort path
(drain_loads in prefill_pair.cu) uses to find the loads still in flight.

Two CTAs (leader 0, peer 1) each run two producer streams over one sequence of loads
n = 0, 1, 2, ...: stream (cta, m) issues the n with n % 2 == m, in order, into ring slot
n % 3, and may issue n only once the slot's previous phase (load n - 3) has completed. The
leader's barrier phase of load n completes when the leader has armed it (the leader arms it
when it issues n) and both CTAs' halves have landed. Streams stop at random points (a
time-out), loads land at random times. The kernel's rule, restated here: per slot, the only
load that can still be in flight is n* = the largest n on the slot that any stream issued;
the leader completes the half the peer never issued, arms a load only the peer issued, and
waits on n*'s phase. The test checks, over many random runs, that after those actions every
issued load's phase is the one waited on or already complete -- nothing any CTA issued can
still be writing when the CTAs leave -- and that the parity wait is exact (the barrier is
at most one phase past n*).
"""

import random

STAGES = 3


def _run(rng, n_loads):
    issued = {0: set(), 1: set()}     # cta -> issued loads
    landed = {0: set(), 1: set()}
    next_n = {(c, m): m for c in (0, 1) for m in (0, 1)}
    stop = {}
    complete = set()

    def phase_done(n):
        return n in issued[0] and n in landed[0] and n in issued[1] and n in landed[1]

    while len(stop) < 4:
        ev = rng.random()
        live = [k for k in next_n if k not in stop]
        k = rng.choice(live)
        n = next_n[k]
        if ev < 0.04 or n >= n_loads:                      # this stream stops
            stop[k] = n
        elif ev < 0.6:                                     # try to issue its next load
            if n < STAGES or (n - STAGES) in complete:
                issued[k[0]].add(n)
                next_n[k] = n + 2
        else:                                              # some load in flight lands
            inflight = [(c, x) for c in (0, 1) for x in issued[c] if x not in landed[c]]
            if inflight:
                c, x = rng.choice(inflight)
                landed[c].add(x)
        complete |= {x for x in issued[0] | issued[1] if phase_done(x)}
    return issued, landed, stop, complete


def _drain_targets(stop):
    """The kernel's rule: per slot, n* and the leader / peer flags."""
    kv = [stop[(0, 0)], stop[(0, 1)], stop[(1, 0)], stop[(1, 1)]]
    out = {}
    for s in range(STAGES):
        nstar = -1
        for cm in range(4):
            for n in range(kv[cm] - 1, max(-1, kv[cm] - 7), -1):
                if n % 2 == cm % 2 and n % STAGES == s:
                    nstar = max(nstar, n)
                    break
        if nstar >= 0:
            out[s] = (nstar, nstar < kv[0 + nstar % 2], nstar < kv[2 + nstar % 2])
    return out


def test_drain_rule_covers_every_load_in_flight():
    rng = random.Random(1234)
    for trial in range(4000):
        issued, landed, stop, complete = _run(rng, rng.randint(1, 40))
        targets = _drain_targets(stop)
        for c in (0, 1):
            for n in issued[c]:
                # issued(cta, n) agrees with the published stops
                assert n < stop[(c, n % 2)]
                if n in complete:
                    continue
                # an issued load whose phase has not completed is the slot's n*
                s = n % STAGES
                assert s in targets and targets[s][0] == n, (trial, c, n, targets)
                nstar, L, P = targets[s]
                assert L == (n in issued[0]) and P == (n in issued[1])
        for s, (nstar, L, P) in targets.items():
            # nothing after n* on the slot was issued: its phase is pending or just done,
            # so the parity wait on it is exact
            assert all(x % STAGES != s or x <= nstar for x in issued[0] | issued[1])
            assert L or P
