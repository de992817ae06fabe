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


# ------------------------------------------------------------------ register-resident kernel
REG_THREADS, REG_MAX_CLUSTER = 512, 16


def reg_tasks(bits):
    cpw = 32 // bits
    return 1 if cpw >= 16 else max(1, 10 // cpw)


def reg_plan(W, V, bits):
    """Mirror of plan_quant's register-resident branch: (TT, C) or None."""
    R = reg_tasks(bits)
    tasks, cap = W * V, REG_THREADS * R
    if tasks > cap * REG_MAX_CLUSTER:
        return None
    if tasks <= cap:
        TT = V
        while TT < 32 and TT < tasks:
            TT *= 2
        if TT >= 32:
            TT = 32
            while TT * R < tasks:
                TT *= 2
        return TT, 1
    C = 2
    while C * cap < tasks:
        C *= 2
    return REG_THREADS, C


def check_reg(n, bits, V, D, units, grid_ctas):
    """Every (unit, word row, vector) task is loaded and encoded by exactly one
    thread, the scale/zero vectors of a unit are written once, all threads of a
    CTA run the same rounds (barriers and shuffles line up), shuffle partners
    and named-barrier teams stay inside one unit, and the shared-memory
    partials stay inside their buffers."""
    CPW = 32 // bits
    W = -(-n // CPW)
    pl = reg_plan(W, V, bits)
    if pl is None:
        return False
    TT, C = pl
    R = reg_tasks(bits)
    tasks = W * V
    assert TT & (TT - 1) == 0 and TT % V == 0 and V <= TT <= REG_THREADS and R * TT * C >= tasks
    assert C in (1, 2, 4, 8, 16) and (C == 1 or TT == REG_THREADS)
    teams = REG_THREADS // TT
    assert TT <= 32 or teams <= 8      # named barrier ids 1..8 (sub-warp teams use none)
    grid = max(C, grid_ctas - grid_ctas % C)
    ncl = grid // C
    span = min(TT, 32)
    seen, meta = {}, set()
    rounds = None
    for cta in range(grid):
        cl, rank = divmod(cta, C)
        r0s = list(range(cl * teams, units, ncl * teams))
        if rounds is None:
            rounds = len(r0s)
        # every CTA of one cluster runs the same rounds (cluster barrier per round)
        if C > 1:
            assert len(r0s) == len(list(range((cta - rank) // C * teams, units, ncl * teams)))
        for r0 in r0s:
            for tid in range(REG_THREADS):
                team, i = divmod(tid, TT)
                j = i % V
                unit = r0 + team
                live = unit < units
                # shuffle partners (xor offsets V .. span/2) share the unit and the vector
                off = V
                while off < span:
                    partner = tid ^ off
                    assert partner // TT == team and (partner % TT) % V == j
                    off *= 2
                tfirst = rank * TT + i
                for k in range(R):
                    t = tfirst + k * TT * C
                    if live and t < tasks:
                        assert t % V == j
                        key = (unit, t // V, j)
                        assert key not in seen, key
                        seen[key] = cta
                if live and tfirst < V:
                    assert (unit, j) not in meta
                    meta.add((unit, j))
                if TT > 32:
                    wt = i >> 5
                    nw = TT // 32
                    # red[par][16][2][D]: this team's warps occupy slots team*nw .. +nw
                    assert 0 <= team * nw + wt < 16
    assert len(seen) == units * tasks
    assert len(meta) == units * V
    return True


@pytest.mark.parametrize("D,esize", [(64, 2), (128, 2), (64, 4), (128, 4)])
def test_reg_quant_covers_every_task_once(D, esize):
    V = D * esize // 16
    ran = 0
    for n in (1, 2, 3, 9, 16, 25, 36, 64, 100, 169, 256, 400, 1024, 1600, 4096, 4680):
        for bits in (2, 3, 4, 6, 8):
            units = 3 if n >= 1024 else 37
            ran += check_reg(n, bits, V, D, units, 12)
    assert ran > 40


def test_reg_quant_plans_of_the_workloads():
    # VAR-d30 INT3 (bf16, D 64): teams of 8 lanes up to 16 tokens, whole CTAs
    # never; the last block (26 word rows) takes a team of 8 warps
    assert reg_plan(-(-256 // 10), 8, 3) == (256, 1)
    assert reg_plan(-(-16 // 10), 8, 3) == (16, 1)
    assert reg_plan(1, 8, 3) == (8, 1)
    # Infinity-2B (D 128: 16 vectors per row), last block of 4096 tokens: a
    # cluster of 16 CTAs at INT3 and INT4; video chunks of 4680 tokens at INT6: 16
    assert reg_plan(-(-4096 // 10), 16, 3) == (512, 16)
    assert reg_plan(-(-4096 // 8), 16, 4) == (512, 16)
    assert reg_plan(-(-4680 // 5), 16, 6) == (512, 16)
