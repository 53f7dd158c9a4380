"""The LLA-2D kernel's c^V ring protocol, simulated on the host.  No GPU.

The kernel keeps a tile's four c^V quarter slots on one barrier, vt_full[n % 4].  A slot is refilled
once the V GEMM of its previous tile m is complete, which is phase m / 2 of d_full[m % 2].  All waits
are parity waits on mbarriers.  A parity wait for phase k succeeds once the barrier's completed-phase
count c has odd distance to k.  It is only correct while c is k or k + 1, so here every wait checks
that invariant:
- at c = k - 1 it would pass a phase that has not happened;
- at c = k + 2 it would hang.

The producer also arrives on vt_full[n % 4] (expect_tx) before the tile's quarter waits, so the
barrier's previous phase (tile n - 4) must be complete by then.

The actors are the c^V producer, the copies in flight, the V-GEMM issuer and the compute warps
(P of tile n needs the V GEMM of tile n - 2 read back: the P buffers are double-buffered).  Every
enabled action is taken in a seeded random order, so many interleavings are tried.  The kernel
bounds the ring to NV <= 8 slots, and for those ring sizes no interleaving breaks an invariant.
A ring of 12 slots can run a producer wait a full d_full phase late: the check must catch that.

The per-head kernel's latent stage ring (ratio 21.3) is simulated the same way.  Its consumers
drift apart by up to three TMEM score buffers of eight stages, more than one ring round, so round
r of a slot lands on barrier set r % 4.  With one barrier per slot a consumer's wait can match a
fill two rounds back; with four sets, and 3 x 8 <= 4 x 10 as the kernel asserts, it cannot.
"""

import random

import pytest


class Barrier:
    def __init__(self):
        self.done = 0  # completed phases

    def wait_ok(self, k: int) -> bool:
        """A parity wait for phase k: checks the invariant, then returns whether it passes."""
        assert self.done in (k, k + 1), f"parity wait for phase {k} with {self.done} phases complete"
        return self.done == k + 1


def simulate(nv: int, tiles: int, seed: int) -> None:
    rng = random.Random(seed)
    vt_full = [Barrier() for _ in range(4)]
    vt_pending = [0] * 4      # quarter copies of the barrier's current phase still in flight
    vt_armed = [False] * 4    # expect_tx done for the current phase
    d_full = [Barrier() for _ in range(2)]
    v_issued = [False] * tiles
    v_done = [False] * tiles
    p_ready = [False] * tiles
    in_flight = []            # (tile) copies issued, not yet landed
    prod_tile, prod_q = 0, 0  # next quarter the producer fills
    mma_next = 0              # next V GEMM to issue
    comp_next = 0             # next tile whose P the compute warps write
    gemm_running = []         # V GEMMs issued, not complete

    def producer_step() -> bool:
        nonlocal prod_tile, prod_q
        if prod_tile >= tiles:
            return False
        n, q = prod_tile, prod_q
        b = n & 3
        if q == 0 and not vt_armed[b]:
            # arrive.expect_tx on vt_full[n % 4]: its previous phase (tile n - 4) must be complete
            assert vt_full[b].done == n // 4, f"tile {n}: barrier {b} still in phase of tile {n - 4}"
            vt_armed[b] = True
            vt_pending[b] = 4
        vk = 4 * n + q
        if vk >= nv:
            m = (vk - nv) // 4  # the slot's previous tile
            if not d_full[m & 1].wait_ok(m >> 1):
                return False
        in_flight.append(n)
        prod_q += 1
        if prod_q == 4:
            prod_tile, prod_q = prod_tile + 1, 0
        return True

    def land_step() -> bool:
        if not in_flight:
            return False
        n = in_flight.pop(rng.randrange(len(in_flight)))
        b = n & 3
        vt_pending[b] -= 1
        if vt_pending[b] == 0:
            vt_full[b].done += 1
            vt_armed[b] = False
        return True

    def mma_step() -> bool:
        nonlocal mma_next
        n = mma_next
        if n >= tiles or not p_ready[n]:
            return False
        if not vt_full[n & 3].wait_ok(n >> 2):
            return False
        v_issued[n] = True
        gemm_running.append(n)
        mma_next += 1
        return True

    def gemm_done_step() -> bool:
        if not gemm_running:
            return False
        n = gemm_running.pop(0)  # the tensor pipe completes in issue order
        v_done[n] = True
        d_full[n & 1].done += 1
        return True

    def compute_step() -> bool:
        nonlocal comp_next
        n = comp_next
        if n >= tiles:
            return False
        if n >= 2 and not v_done[n - 2]:  # P buffer n % 2 is free once tile n - 2's V GEMM is read
            return False
        p_ready[n] = True
        comp_next += 1
        return True

    actors = [producer_step, land_step, mma_step, gemm_done_step, compute_step]
    for _ in range(200 * tiles):
        order = actors[:]
        rng.shuffle(order)
        if not any(a() for a in order):
            break
    assert all(v_done), f"stalled: {sum(v_done)} of {tiles} V GEMMs done"


@pytest.mark.parametrize("nv", [4, 5, 6, 7, 8])
def test_cv_ring_waits_never_alias(nv):
    for seed in range(60):
        simulate(nv, tiles=40, seed=1000 * nv + seed)


def test_a_ring_deeper_than_two_tiles_can_alias():
    """The bound the kernel asserts is needed: with 12 slots some interleaving waits on d_full a
    full phase late (or arms vt_full early), and the invariants catch it."""
    caught = 0
    for seed in range(200):
        try:
            simulate(12, tiles=40, seed=seed)
        except AssertionError:
            caught += 1
    assert caught > 0


def simulate_stage_ring(nst: int, nbuf: int, tiles: int, seed: int, sets: int = 4) -> None:
    """The per-head kernel's stage ring at ratio 21.3: 16 heads per item in two TMEM groups of 8,
    one stage per (tile, head), two producers (even and odd heads), 16 compute warps (4 per lane
    quarter, warp f of a quarter taking heads f, f + 4, f + 8, f + 12).  Round r of slot s lands
    on barrier set r % sets (4 in the kernel), and a consumer waits for phase r / sets.  A warp starts head group
    gi only once the MMA has issued it, and the MMA issues group gi only once all 16 warps have
    released group gi - nbuf: so the warps drift apart by at most nbuf groups."""
    rng = random.Random(seed)
    H, HG, WPQ = 16, 8, 4
    groups = tiles * 2
    nstages = tiles * H
    full = [[Barrier() for _ in range(nst)] for _ in range(sets)]
    empty = [Barrier() for _ in range(nst)]
    empty_count = [0] * nst          # arrivals in the current phase of st_empty[slot] (4 per phase)
    tm_empty_count = [0] * groups    # warps done with group gi
    issued_groups = 0
    in_flight = []
    prod_next = [0, 1]               # next stage of each producer (even / odd heads)
    # warp (q, f): position in its sequence of (group, stage) steps
    seqs = {}
    for q in range(4):
        for f in range(WPQ):
            steps = []
            for t in range(tiles):
                for g in range(2):
                    heads = [hl for hl in (f, f + 4, f + 8, f + 12) if hl // HG == g]
                    steps.append(("group", t * 2 + g))
                    for hl in heads:
                        steps.append(("stage", t * H + hl))
                    steps.append(("release", t * 2 + g))
            seqs[(q, f)] = [steps, 0]

    def producer(i):
        k = prod_next[i]
        if k >= nstages:
            return False
        slot, rnd = k % nst, k // nst
        if rnd > 0 and not empty[slot].wait_ok(rnd - 1):
            return False
        in_flight.append(k)
        prod_next[i] += 2
        return True

    def land():
        if not in_flight:
            return False
        k = in_flight.pop(rng.randrange(len(in_flight)))
        slot, rnd = k % nst, k // nst
        full[rnd % sets][slot].done += 1
        return True

    def mma():
        nonlocal issued_groups
        gi = issued_groups
        if gi >= groups:
            return False
        if gi >= nbuf and tm_empty_count[gi - nbuf] < 16:
            return False
        issued_groups += 1
        return True

    def warp(key):
        steps, pos = seqs[key]
        if pos >= len(steps):
            return False
        kind, x = steps[pos]
        if kind == "group":
            if x >= issued_groups:
                return False
        elif kind == "stage":
            slot, rnd = x % nst, x // nst
            if not full[rnd % sets][slot].wait_ok(rnd // sets):
                return False
            empty_count[slot] += 1
            if empty_count[slot] == 4:  # the four quarter warps of the head released it
                empty_count[slot] = 0
                empty[slot].done += 1
        else:
            tm_empty_count[x] += 1
        seqs[key][1] = pos + 1
        return True

    actors = [lambda: producer(0), lambda: producer(1), land, mma] + [
        (lambda k=k: warp(k)) for k in seqs]
    for _ in range(400 * tiles * H):
        order = actors[:]
        rng.shuffle(order)
        if not any(a() for a in order):
            break
    assert all(p >= len(s) for s, p in seqs.values()), "stalled"


def test_stage_ring_barrier_sets_never_alias():
    """The kernel's configuration (10 slots, 3 score buffers: 3 x 8 <= 4 x 10 stages)."""
    for seed in range(20):
        simulate_stage_ring(nst=10, nbuf=3, tiles=6, seed=seed)


def test_stage_ring_needs_four_sets_for_the_drift():
    """With fewer slots than the drift allows (3 x 8 > 4 x 5) some interleaving waits on a
    barrier set at the wrong phase: the bound the kernel asserts is needed."""
    caught = 0
    for seed in range(40):
        try:
            simulate_stage_ring(nst=5, nbuf=3, tiles=6, seed=seed)
        except AssertionError:
            caught += 1
    assert caught > 0


def test_stage_ring_one_barrier_per_slot_aliases():
    """One barrier per slot, as before the barrier sets: the warps' drift (3 groups of 8 stages)
    exceeds a ring round (10), and a consumer's parity wait can match a fill two rounds back."""
    caught = 0
    for seed in range(40):
        try:
            simulate_stage_ring(nst=10, nbuf=3, tiles=6, seed=seed, sets=1)
        except AssertionError:
            caught += 1
    assert caught > 0
