"""A model of the GEMM kernels' TMA ring protocol, run under random
interleavings: two producer threads fill ring stages (each stage owned by the
producer with its parity), one consumer (the MMA issuer) drains them in order,
and every wait is an mbarrier parity wait (the phase of the given parity has
completed iff the barrier's current phase has the other parity).

Checks: a producer never refills a stage whose previous fill is unconsumed,
the consumer never reads an unfilled stage, nothing deadlocks, and each
producer's final drain (a wait on the full barrier of its last fill of every
stage it filled) refers to a completed phase.  The same model with the K
blocks dealt by iteration parity instead breaks the drain whenever the ring
depth is odd, which is why the kernels deal stages, not iterations."""
import random

import pytest


def _run(S, nkb, tiles, seed, owner):
    rnd = random.Random(seed)
    total = nkb * tiles
    consumed = [0] * S   # completed phases of empty[s]
    landed = [0] * S     # completed phases of full[s]
    filled = [0] * S
    prod = [dict(it=0, stage=0, phase=0, issued=0, last_par=0, done=False) for _ in range(2)]
    cons = dict(it=0, stage=0, phase=0)
    inflight = []

    def passes(count, parity):
        return (count & 1) != parity

    for _ in range(10 ** 6):
        acts = [("p", p) for p in range(2) if not prod[p]["done"]]
        if cons["it"] < total:
            acts.append(("c", 0))
        if inflight:
            acts.append(("land", 0))
        if not acts:
            break
        kind, p = rnd.choice(acts)
        if kind == "land":
            s, k = inflight.pop(rnd.randrange(len(inflight)))
            assert landed[s] == k
            landed[s] += 1
        elif kind == "p":
            P = prod[p]
            if P["it"] >= total:
                P["done"] = True
                continue
            st = P["stage"]
            if owner(st, P["it"]) == p:
                if not passes(consumed[st], P["phase"] ^ 1):
                    continue
                k = P["it"] // S
                assert filled[st] == k and consumed[st] == k, "refill of an unconsumed stage"
                filled[st] += 1
                inflight.append((st, k))
                P["issued"] |= 1 << st
                P["last_par"] = (P["last_par"] & ~(1 << st)) | (P["phase"] << st)
            P["it"] += 1
            P["stage"] += 1
            if P["stage"] == S:
                P["stage"], P["phase"] = 0, P["phase"] ^ 1
        else:
            st = cons["stage"]
            if not passes(landed[st], cons["phase"]):
                continue
            assert landed[st] == cons["it"] // S + 1, "consumed an unfilled stage"
            consumed[st] += 1
            cons["it"] += 1
            cons["stage"] += 1
            if cons["stage"] == S:
                cons["stage"], cons["phase"] = 0, cons["phase"] ^ 1
    else:
        raise AssertionError("deadlock")
    for P in prod:
        for s in range(S):
            if P["issued"] >> s & 1:
                assert passes(landed[s], P["last_par"] >> s & 1), "drain waits on a phase that never completes"


@pytest.mark.parametrize("S", range(3, 9))
def test_stage_owned_ring_is_safe(S):
    for nkb in (1, 2, 3, 5, 20):
        for seed in range(12):
            _run(S, nkb, 3, seed, lambda st, it: st & 1)


def test_iteration_dealt_ring_breaks_the_drain_for_odd_depth():
    with pytest.raises(AssertionError, match="drain"):
        for seed in range(50):
            _run(5, 20, 3, seed, lambda st, it: it & 1)
    for seed in range(12):   # even depth: each stage still has one owner
        _run(6, 20, 3, seed, lambda st, it: it & 1)
