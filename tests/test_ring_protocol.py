"""A model of the fused decode kernel's shared-memory slot ring, run over random interleavings.

The kernel streams each CTA's gate/up items and down pieces through R shared-memory slots: fill q
lands in slot q % R and completes one phase of that slot's mbarrier; a consumer of fill q waits
with the parity of phase q / R. A parity wait can only tell the current phase from the one before
it, so it is sound only if, at the wait, the slot has completed exactly q / R or q / R + 1 phases:
one fewer and the wait mistakes the older phase for its own; two more and it never returns.

The schedule modelled here is the kernel's: fills 0..R-1 are issued at the start, fill q + R
when fill q has been consumed; gate/up items alternate between two warp groups, each taking its
items in order, with an even R; after the CTA barrier that closes the gate/up phase the down
phase's warps take whole units (warp w: units w, w + 16, ...), a unit of piece d first waiting
until piece d - R is fully consumed. The test drives that schedule with fills landing and consumers advancing in random
order and checks the wait rule at every wait, and that the schedule never deadlocks. Variants
with the rules the kernel relies on removed (an odd R, no wait for the piece one ring behind,
items dealt to every warp) must break the rule, so the check is known to see the failure it
guards against.
"""
import random

import pytest

WARPS = 16


def simulate(n_mine, npieces, n_rb, dpu, nu_last, R, seed, even_ring=True, piece_wait=True, p2_owners=2):
    """Returns (violations, deadlocked). nu_last: units in the last piece (1..dpu). p2_owners:
    how many consumers the gate/up items are dealt to round-robin (the kernel: 2 warp groups)."""
    rng = random.Random(seed)
    if even_ring:
        assert R % 2 == 0
    n_total = n_mine + n_rb * npieces
    nu = (npieces - 1) * dpu + nu_last
    completed = [0] * R       # phases completed per slot
    in_flight = []            # fills issued, not yet landed
    violations = []

    def issue(q):
        if q < n_total:
            in_flight.append(q)

    for q in range(min(n_total, R)):
        issue(q)

    def wait_ok(q):
        """True if the parity wait for fill q returns now; records a violation if it returns wrongly."""
        s, p = q % R, q // R
        c = completed[s]
        returns = (c % 2) != (p % 2)
        if returns and c != p + 1:
            violations.append((q, c, p))
        return returns

    # P2: group g takes items g, g + 2, ... in order (the ring is even: a slot's items share a group)
    p2 = {g: [q for q in range(g, n_mine, p2_owners)] for g in range(p2_owners)}
    # P3 (after the barrier): per row block, warp w takes units w, w + 16, ...
    pcnt = {}
    p3 = None
    rb = 0
    steps = 0
    while True:
        steps += 1
        if steps > 100000:
            return violations, True
        actions = []
        if in_flight:
            actions.append("land")
        p2_left = any(p2[g] for g in p2)
        if p2_left:
            for g in p2:
                if p2[g] and wait_ok_peek(p2[g][0], completed, R):
                    actions.append(("p2", g))
        elif p3 is None:
            if rb == n_rb:
                break
            p3 = {w: list(range(w, nu, WARPS)) for w in range(WARPS)}
            pcnt = {d: 0 for d in range(npieces)}
            continue
        else:
            for w in range(WARPS):
                if not p3[w]:
                    continue
                u = p3[w][0]
                d = u // dpu
                if piece_wait and d >= R:
                    need = dpu if d - R < npieces - 1 else nu_last
                    if pcnt[d - R] < need:
                        continue
                qd = n_mine + rb * npieces + d
                if wait_ok_peek(qd, completed, R):
                    actions.append(("p3", w))
            if all(not v for v in p3.values()):
                p3 = None
                rb += 1
                continue
        if not actions:
            return violations, True
        a = rng.choice(actions)
        if a == "land":
            q = in_flight.pop(rng.randrange(len(in_flight)))
            completed[q % R] += 1
        elif a[0] == "p2":
            q = p2[a[1]].pop(0)
            wait_ok(q)
            issue(q + R)
        else:
            w = a[1]
            u = p3[w].pop(0)
            d = u // dpu
            qd = n_mine + rb * npieces + d
            wait_ok(qd)
            pcnt[d] += 1
            need = dpu if d < npieces - 1 else nu_last
            if pcnt[d] == need:
                issue(qd + R)
    return violations, False


def wait_ok_peek(q, completed, R):
    s, p = q % R, q // R
    return (completed[s] % 2) != (p % 2)


CONFIGS = [
    # (n_mine, npieces, n_rb, dpu, nu_last, R): shapes the kernel meets (T=1: 5 items, 3 pieces,
    # R=8; T=4: ~10 items, ~6 pieces, R=16; T=5 top-10: up to 23 items, 13 pieces, R=12) and
    # harder ones (more items and pieces than slots, two row blocks, small rings)
    (5, 3, 1, 4, 3, 8), (10, 6, 1, 4, 2, 16), (23, 13, 1, 4, 3, 12), (23, 13, 2, 4, 4, 12),
    (17, 9, 1, 2, 1, 4), (40, 30, 2, 1, 1, 6), (3, 5, 2, 4, 1, 2), (0, 7, 1, 3, 2, 4),
]


@pytest.mark.parametrize("cfg", CONFIGS)
def test_kernel_schedule_keeps_every_parity_wait_sound(cfg):
    for seed in range(60):
        violations, deadlocked = simulate(*cfg, seed=seed)
        assert not violations, (cfg, seed, violations[:3])
        assert not deadlocked, (cfg, seed)


def test_without_the_ordering_rules_a_wait_goes_wrong():
    # odd ring (a slot's items alternate between the two groups) and no wait for the piece one ring
    # behind: some interleaving lets a parity wait return on an older phase
    bad = 0
    for (n_mine, npieces, n_rb, dpu, nu_last) in [(23, 13, 1, 4, 3), (17, 9, 1, 2, 1), (40, 30, 2, 1, 1)]:
        for seed in range(60):
            violations, _ = simulate(n_mine, npieces, n_rb, dpu, nu_last, 7, seed=seed, even_ring=False,
                                     piece_wait=False)
            bad += bool(violations)
    assert bad > 0


def test_items_dealt_to_every_warp_break_the_rule():
    # gate/up items dealt round-robin to all 16 warps (a layout tried once) with a ring of 12 and
    # 23 items per CTA: a warp's second item can wait two phases ahead of its slot
    bad = sum(bool(simulate(23, 13, 1, 4, 3, 12, seed=seed, p2_owners=16)[0]) for seed in range(60))
    assert bad > 0


@pytest.mark.parametrize("even_ring,piece_wait", [(False, True), (True, False)])
def test_each_rule_is_needed(even_ring, piece_wait):
    # an odd ring alone breaks the gate/up waits; missing piece waits alone break the down waits
    cfgs = [(23, 13, 1, 4, 3), (17, 9, 1, 2, 1), (40, 30, 2, 1, 1)]
    R = 6 if even_ring else 7
    bad = sum(bool(simulate(*c, R, seed=seed, even_ring=even_ring, piece_wait=piece_wait)[0])
              for c in cfgs for seed in range(60))
    assert bad > 0
