"""CPU model of the quantize+pack kernel's work split (csrc/quant_pack.cuh with
the plan of csrc/vq_api.cu), no GPU: for block sizes, bit widths, row widths
and unit counts of the workloads, every (unit, row, 16-byte vector) is read
exactly once in pass 1, every (unit, word row, vector) is encoded exactly once
in pass 2, and every (unit, vector) of scale/zero is written exactly once."""
import itertools

import pytest

WARPS, BATCH, TARGET_WARPS = 16, 16, 2048


def plan(units, W, n, V):
    P = 1
    while P < WARPS and units * P < TARGET_WARPS and 2 * P <= W:
        P *= 2
    rw = 1
    while rw * BATCH < n and rw * V < 32:
        rw *= 2
    TL = min(32, rw * V) if P == 1 else 32
    return P, -(-W // P), TL


def check(n, bits, V, units, grid):
    CPW = 32 // bits
    W = -(-n // CPW)
    P, WP, TL = plan(units, W, n, V)
    assert 32 % TL == 0 and TL % V == 0
    gpc, RW, upw = WARPS // P, TL // V, 32 // TL
    seen1, seen2, meta = set(), set(), set()
    for cta, warp in itertools.product(range(grid), range(WARPS)):
        grp, part = divmod(warp, P)
        u0 = (cta * gpc + grp) * upw
        while u0 < units:
            for lane in range(32):
                team, tl = divmod(lane, TL)
                j, rsub = tl % V, tl // V
                unit = u0 + team
                live = unit < units
                w0 = part * WP
                w1 = min(W, w0 + WP) if live else w0
                r0, r1 = w0 * CPW, min(n, w1 * CPW)
                r = r0 + rsub
                while r < r1:
                    for u in range(BATCH):
                        if r + u * RW < r1:  # the clamped repeats re-read row r1 - 1
                            k = (unit, r + u * RW, j)
                            assert k not in seen1
                            seen1.add(k)
                    r += BATCH * RW
                if live and part == 0 and rsub == 0:
                    assert (unit, j) not in meta
                    meta.add((unit, j))
                w = w0 + rsub
                while w < w1:
                    assert (unit, w, j) not in seen2
                    seen2.add((unit, w, j))
                    w += RW
            u0 += grid * gpc * upw
    assert len(seen1) == units * n * V
    assert len(seen2) == units * W * V
    assert len(meta) == units * V


@pytest.mark.parametrize("n", [1, 2, 4, 9, 16, 17, 25, 36, 64, 100, 256])
def test_quant_work_split_covers_every_vector_once(n):
    for bits, V, units, grid in itertools.product((2, 3, 4, 6, 8), (8, 16, 32), (3, 256, 1000), (1, 148)):
        if units * n <= 16000:
            check(n, bits, V, units, grid)


def test_quant_plan_small_blocks_share_warps():
    # VAR-d30 shapes (bf16, head_dim 64: 8 vectors per row; 7680 units): blocks of up to
    # 16 tokens take 4 units per warp, 25 tokens 2, larger blocks a whole warp
    tl = {n: plan(7680, -(-n // 10), n, 8)[2] for n in (1, 4, 9, 16, 25, 36, 64, 256)}
    assert tl == {1: 8, 4: 8, 9: 8, 16: 8, 25: 16, 36: 32, 64: 32, 256: 32}


# ------------------------------------------------------------------ ring kernel
RING_MAX_WARPS, RING_BUDGET = 12, 200 * 1024


def ring_plan(n, D, esize):
    slab = n * D * esize
    if not (8192 <= slab <= RING_BUDGET // 2):
        return None
    ns, rw = 2, RING_BUDGET // (2 * slab)
    if rw < RING_MAX_WARPS:
        ns, rw = 1, RING_BUDGET // slab
    rw = min(rw, RING_MAX_WARPS)
    return (rw, ns, slab, min(RING_MAX_WARPS // rw, 6)) if rw >= 2 else None


@pytest.mark.parametrize("D,esize", [(64, 2), (128, 2), (64, 4), (128, 4)])
def test_ring_quant_plan_and_protocol(D, esize):
    """Ring kernel: the slots fit the shared-memory budget (and the barrier
    arrays), every unit goes to exactly one team, and each slot is filled and
    drained in the same order (by the producer warp, or, for one-warp teams,
    by the team itself: its first NS units at once, then unit i + NS into the
    slot unit i leaves), so the parity of every full/empty wait is the use
    count of that slot."""
    ran = 0
    for n in (16, 36, 64, 100, 144, 169, 256, 300, 400, 576, 800):
        pl = ring_plan(n, D, esize)
        if pl is None:
            continue
        rw, ns, slab, rg = pl
        assert 2 <= rw <= RING_MAX_WARPS and ns in (1, 2) and slab % 16 == 0
        assert rw * ns * slab <= RING_BUDGET and rw * ns <= RING_MAX_WARPS * 4
        # teams: at most 12 consumer warps, named barriers 1 .. rw, and the
        # shared memory (barriers, slots, [rw][2][rg][2][D] partials) fits the opt-in
        assert 1 <= rg <= 6 and rw * rg <= RING_MAX_WARPS and rw + 1 <= 16
        assert 2 * RING_MAX_WARPS * 4 * 8 + rw * ns * slab + rw * 2 * rg * 2 * D * 4 <= 232448
        # the team's warps split rows (pass 1, 8 loads per lane per step) and
        # word rows (pass 2): every one is taken exactly once
        V = D * esize // 16
        RL = 32 // V
        for bits in (2, 3, 4, 6, 8):
            W = -(-n // (32 // bits))
            rows, wrows = [], []
            for gw in range(rg):
                for rsub in range(RL):
                    r = rsub + gw * RL
                    while r < n:
                        rows += [r + q * RL * rg for q in range(8) if r + q * RL * rg < n]
                        r += 8 * RL * rg
                    w = rsub + gw * RL
                    while w < W:
                        wrows.append(w)
                        w += RL * rg
            assert sorted(rows) == list(range(n)) and sorted(wrows) == list(range(W))
        for units, grid in ((7680, 148), (256, 148), (5, 3)):
            grid = min(grid, units)
            seen = {}
            for cta in range(grid):
                fills = []                     # producer order: (slot, use)
                k = 0
                while cta + k * grid < units:
                    w, s, use = k % rw, (k // rw) % ns, k // (rw * ns)
                    fills.append((w * ns + s, use, cta + k * grid))
                    k += 1
                for w in range(rw):          # consumer w: its own units in order
                    kk = w
                    drains = []
                    while cta + kk * grid < units:
                        u = cta + kk * grid
                        assert u not in seen
                        seen[u] = w
                        drains.append((w * ns + (kk // rw) % ns, kk // (rw * ns), u))
                        kk += rw
                    assert drains == [f for f in fills if f[0] // ns == w]
                    if rg == 1:
                        # self-copying team: units 0 .. ns-1 first, then unit i + ns
                        # into the slot unit i has just left
                        own = [d[:2] for d in drains[:ns]]
                        for i in range(len(drains) - ns):
                            assert drains[i + ns][:2] == (drains[i][0], drains[i][1] + 1)
                            own.append(drains[i + ns][:2])
                        assert own == [d[:2] for d in drains]
            assert len(seen) == units
            ran += 1
    assert ran > 0


def test_ring_plans_of_the_workload_slabs():
    """The ring plans the measurements chose, for the bf16 slabs of the VAR-d30
    (head_dim 64) and Infinity-2B (head_dim 128) blocks that take the ring:
    (teams, slots per team, slab bytes, warps per team). Two slots per team
    only for 8 KB slabs (twelve one-warp teams still fit); one slot and as
    many teams as the budget holds above that; the smallest slabs fall to the
    streaming kernel."""
    want = {
        (36, 64): None, (64, 64): (12, 2, 8192, 1), (100, 64): (12, 1, 12800, 1),
        (169, 64): (9, 1, 21632, 1), (256, 64): (6, 1, 32768, 2),
        (16, 128): None, (36, 128): (12, 1, 9216, 1), (64, 128): (12, 1, 16384, 1),
        (144, 128): (5, 1, 36864, 2), (256, 128): (3, 1, 65536, 4), (400, 128): (2, 1, 102400, 6),
        (576, 128): None,
    }
    for (n, D), plan in want.items():
        assert ring_plan(n, D, 2) == plan, (n, D)
