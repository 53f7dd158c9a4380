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
