"""CPU models of the packed-KV attention kernel (csrc/attention_pipe.cuh), no GPU.

The kernel's constants and index arithmetic are restated here and checked
for every head_dim / bit width / query-tile mode it is launched with:

- the shared- and tensor-memory layout of PipeCfg fits one CTA and keeps the
  alignment the bulk copies and MMA descriptors need;
- the key-tile walker covers blocks 0..s exactly once, its staged word rows
  stay inside the stage buffers, and the unpack tasks write every
  (tensor, key, channel) of a tile exactly once with the right cached token;
- the mbarrier protocol between the producer, unpack, MMA and softmax roles
  (single K/V release and the split release of the two-slot ring) never
  deadlocks, never lets a parity wait see a barrier two phases ahead, and
  never overwrites a tile header before the softmax has read it. A planted
  hazard shows the simulation can fail.
"""
import itertools
import random

import pytest

SMEM_OPTIN = 232448  # bytes of dynamic shared memory one CTA may opt in to on sm_100a
MAX_TABLE = 4096     # kPipeMaxTable: tabled key counts per item


# ------------------------------------------------------------------ PipeCfg
def pipe_cfg(BITS, D, NQT):
    c = {}
    c["KT"] = KT = 64 if D == 64 else 48
    c["CPW"] = CPW = 32 // BITS
    c["MAXSEG"] = MAXSEG = 8 if D == 64 else 4
    c["MAXROWS"] = MAXROWS = -(-KT // CPW) + 2 * MAXSEG
    TM_QT = 512 // NQT
    c["Q_TMEM"] = Q_TMEM = D == 64
    c["NS"] = NS = 4 if NQT == 1 else 2
    c["NKV"] = NKV = 4 if D == 64 else (3 if NQT == 1 else 2)
    c["NSTG"] = NSTG = 3 if (D == 64 and BITS <= 4) else 2
    c["SPLIT"] = NKV <= 2
    STAGE_Q = D == 64
    QPF = 2 if (STAGE_Q and NQT == 1) else 1
    UW = 8 if NQT == 1 else 6
    Q_SZ = 0 if Q_TMEM else 128 * D * 2
    c["TILE_SZ"] = TILE_SZ = KT * D * 2
    KV0 = NQT * Q_SZ
    KV_SZ = 4 * TILE_SZ
    QST0 = KV0 + NKV * KV_SZ
    QST_SZ = 128 * D * 2 if STAGE_Q else 0
    STG0 = QST0 + NQT * QPF * QST_SZ
    STG_V = MAXROWS * D * 4
    STG_META = 2 * STG_V
    STG_SEG = STG_META + MAXSEG * 4 * D * 4
    STG_ROWS = STG_SEG + MAXSEG * 16
    STG_SZ = STG_ROWS + (2 * MAXSEG + 4) * 4
    HDR0 = STG0 + NSTG * STG_SZ
    NRED = 5
    RED0 = HDR0 + NKV * 16
    BARS = RED0 + NRED * UW * 4
    NBARS = 2 * NSTG + 4 * NKV + NRED + NQT * (1 + 3 * NS)
    TMEM_SLOT = BARS + NBARS * 8
    NKTAB = TMEM_SLOT + 16
    c["SMEM_ALLOC"] = NKTAB + MAX_TABLE + 1024
    c["checks"] = {
        "operand alignment": KV0 % 1024 == 0 and TILE_SZ % 1024 == 0 and Q_SZ % 1024 == 0,
        "stage alignment": STG0 % 16 == 0 and STG_SZ % 16 == 0 and STG_V % 16 == 0 and STG_META % 16 == 0,
        "header alignment": HDR0 % 16 == 0 and BARS % 8 == 0,
        "shared memory": c["SMEM_ALLOC"] <= SMEM_OPTIN,
        "exponent slots": NRED > NKV,
        "tensor memory": NS * KT + D + (D // 2 if Q_TMEM else 0) <= TM_QT,
        "threads": NQT * 128 + UW * 32 + 64 <= 512,
    }
    c["UW"] = UW
    return c


LAUNCHED = [(b, d, 2) for b in (2, 3, 4, 6, 8) for d in (64, 128)]  # every dispatched instantiation


@pytest.mark.parametrize("BITS,D,NQT", LAUNCHED)
def test_layout_fits_one_cta(BITS, D, NQT):
    c = pipe_cfg(BITS, D, NQT)
    bad = [k for k, ok in c["checks"].items() if not ok]
    assert not bad, (BITS, D, NQT, bad, c["SMEM_ALLOC"])


def warp_roles(NQT):
    """Role of each warp: softmax 0 .. 4 NQT - 1, then the unpack warps, the
    producer and the MMA warp."""
    UW = 8 if NQT == 1 else 6
    SOFT = 4 * NQT
    PROD, MMA = SOFT + UW, SOFT + UW + 1
    nwarps = MMA + 1
    roles = {}
    for w in range(nwarps):
        if w < SOFT:
            roles[w] = ("softmax", w // 4, w % 4)
        elif w in (MMA, PROD):
            roles[w] = ("mma",) if w == MMA else ("producer",)
        else:
            roles[w] = ("unpack", w - SOFT)
    return roles, nwarps, MMA, PROD, UW


@pytest.mark.parametrize("NQT", [1, 2])
def test_warp_roles(NQT):
    roles, nwarps, MMA, PROD, UW = warp_roles(NQT)
    assert nwarps * 32 <= 512 and MMA < nwarps and PROD < nwarps
    # every unpack index 0 .. UW-1 exactly once; softmax warps cover each
    # query tile's four tensor-memory lane quarters
    assert sorted(r[1] for r in roles.values() if r[0] == "unpack") == list(range(UW))
    assert sorted((r[1], r[2]) for r in roles.values() if r[0] == "softmax") == [
        (qt, q) for qt in range(NQT) for q in range(4)]


# ------------------------------------------------------------------ tiles and unpack
def sw128_offset(row, k, rows):
    slab, kin = k >> 6, k & 63
    return slab * rows * 128 + (row >> 3) * 1024 + (row & 7) * 128 + (((kin >> 3) ^ (row & 7)) << 4) + ((kin & 7) << 1)


def walk(blocks, s, KT, MAXSEG):
    """Tiles of the key walk over blocks 0..s: (keys, [(block, u0, take, key0)])."""
    kb, u, tiles = 0, 0, []
    while kb <= s:
        nk, segs, i = 0, [], 0
        while i < MAXSEG and nk < KT and kb <= s:
            take = min(KT - nk, blocks[kb] - u)
            segs.append((kb, u, take, nk))
            nk += take
            u += take
            if u >= blocks[kb]:
                kb, u = kb + 1, 0
            i += 1
        tiles.append((nk, segs))
    return tiles


def check_tiles(BITS, D, blocks):
    c = pipe_cfg(BITS, D, 2)
    KT, CPW, MAXSEG = c["KT"], c["CPW"], c["MAXSEG"]
    prefix = [0]
    for n in blocks:
        prefix.append(prefix[-1] + n)
    for s in range(len(blocks)):
        tiles = walk(blocks, s, KT, MAXSEG)
        covered = 0
        for nk, segs in tiles:
            assert 1 <= nk <= KT and 1 <= len(segs) <= MAXSEG
            rows, row0 = [], 0  # producer: staged word rows of each segment
            for kb, u0, take, key0 in segs:
                wa, wb = u0 // CPW, (u0 + take - 1) // CPW
                assert wb < -(-blocks[kb] // CPW)  # inside the block's packed rows
                rows.append((row0, wb - wa + 1))
                row0 += wb - wa + 1
            R = row0
            assert R <= c["MAXROWS"]
            OCT = D // 8
            written = {}
            for task in range(2 * R * OCT):  # unpack tasks (K tasks first, then V)
                tsel = 1 if task >= R * OCT else 0
                sr, jj = divmod(task - tsel * R * OCT, OCT)
                i = 0
                while i + 1 < len(segs) and rows[i + 1][0] <= sr:
                    i += 1
                kb, u0, take, key0 = segs[i]
                assert rows[i][0] <= sr < rows[i][0] + rows[i][1]
                ub = (u0 // CPW + (sr - rows[i][0])) * CPW
                kbase = key0 + ub - u0
                for sl in range(max(0, u0 - ub), min(CPW, u0 + take - ub)):
                    key = kbase + sl
                    assert 0 <= key < nk
                    off = sw128_offset(key, 8 * jj, KT)
                    assert off + 16 <= c["TILE_SZ"]
                    k = (tsel, key, jj)
                    assert k not in written
                    written[k] = (kb, ub + sl)
            for tsel, key, jj in itertools.product(range(2), range(nk), range(OCT)):
                gpos = covered + key
                kb = max(b for b in range(len(blocks)) if prefix[b] <= gpos)
                assert written[(tsel, key, jj)] == (kb, gpos - prefix[kb])
            covered += nk
        assert covered == prefix[s + 1]


VAR_BLOCKS = [1, 4, 9, 16, 25, 36, 64, 100, 169, 256]
INFINITY_BLOCKS = [1, 4, 16, 36, 64, 144, 256, 400, 576, 1024, 1600, 2304, 4096]


@pytest.mark.parametrize("BITS,D", [(b, d) for b in (2, 3, 4, 6, 8) for d in (64, 128)])
def test_tile_walk_and_unpack_cover_every_key_once(BITS, D):
    check_tiles(BITS, D, VAR_BLOCKS)
    check_tiles(BITS, D, [1, 2, 3, 4])
    rng = random.Random(BITS * 1000 + D)
    for _ in range(4):
        nb = rng.randint(1, 12)
        check_tiles(BITS, D, [rng.choice([1, 2, 3, 5, 7, 11, 16, 31, 64, 65, 127, 129, 300]) for _ in range(nb)])


def test_tile_walk_infinity_schedule():
    check_tiles(4, 128, INFINITY_BLOCKS[:10])


# ------------------------------------------------------------------ barrier protocol
class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, 0, 0

    def arrive(self, n=1):
        self.pending += n
        assert self.pending <= self.count, f"{self.name}: over-arrival"
        if self.pending == self.count:
            self.pending = 0
            self.phase += 1


def simulate(NQT, NS, NKV, T, n_items, grid, n_qt, cta, seed, ALT, SPLIT, hazard=False, NSTG=2, UW=4):
    """Cooperative run of every role of one CTA. Each role yields
    ('wait', barrier, use): wait for completion number `use` of that barrier.
    MMA commits and bulk copies complete after a random delay. Returns the
    list of protocol errors (empty when the run is clean)."""
    rng = random.Random(seed)
    n_groups = n_qt if ALT else -(-n_qt // NQT)
    items = list(range(cta, n_items, grid))

    def qts_of(k, item):
        return [k & 1] if ALT else list(range(min(NQT, n_qt - (item % n_groups) * NQT)))

    B = {}

    def bar(name, count):
        B[name] = Bar(name, count)

    for i in range(NSTG):
        bar(("stg_full", i), 1)
        bar(("stg_empty", i), 32 * UW)
    for i in range(NKV):
        bar(("k_full", i), 32 * UW)
        bar(("k_empty", i), 1)
        bar(("v_full", i), 32 * UW)
        bar(("v_empty", i), 1)
    for i in range(5):
        bar(("red", i), UW)
    for qt in range(NQT):
        bar(("q_full", qt), 4)
        for i in range(NS):
            bar(("s_full", qt, i), 1)
            bar(("p_full", qt, i), 4)
            bar(("pv_done", qt, i), 1)
    hdr = [None] * NKV
    asyncq, now, errors = [], [0], []

    def async_arrive(name):
        asyncq.append((now[0] + rng.randint(1, 30), name))

    def producer():
        for g in range(len(items) * T):
            st = g % NSTG
            if g >= NSTG:
                yield ("wait", ("stg_empty", st), g // NSTG - 1)
            async_arrive(("stg_full", st))

    def mma():
        nq, iq, prev, gt = [0] * NQT, [0] * NQT, None, 0
        for k_it, it in enumerate(items):
            qts = qts_of(k_it, it)
            for j in range(T):
                kvs = gt % NKV
                yield ("wait", ("k_full", kvs), gt // NKV)
                if j == 0:
                    for qt in qts:
                        yield ("wait", ("q_full", qt), iq[qt])
                        iq[qt] += 1
                for qt in qts:
                    n = nq[qt]
                    if n >= NS:
                        yield ("wait", ("pv_done", qt, n % NS), n // NS - 1)
                    async_arrive(("s_full", qt, n % NS))
                if SPLIT:
                    async_arrive(("k_empty", kvs))
                if prev:
                    yield from pv(prev)
                pn = [0] * NQT
                for qt in qts:
                    pn[qt] = nq[qt]
                    nq[qt] += 1
                prev = (qts, kvs, pn, gt)
                gt += 1
        if prev:
            yield from pv(prev)

    def pv(prev):
        pqts, pkvs, pn, pgt = prev
        if SPLIT:
            yield ("wait", ("v_full", pkvs), pgt // NKV)
        for qt in pqts:
            n = pn[qt]
            yield ("wait", ("p_full", qt, n % NS), n // NS)
            async_arrive(("pv_done", qt, n % NS))
        async_arrive(("v_empty", pkvs))

    def unpack(w):
        gt = 0
        if items:
            B[("red", 0)].arrive()
        for k, it in enumerate(items):
            yield ("wait", ("red", k % 5), k // 5)
            for j in range(T):
                st, kvs = gt % NSTG, gt % NKV
                yield ("wait", ("stg_full", st), gt // NSTG)
                if hazard and j == 0 and w == 0:
                    hdr[kvs] = gt  # planted: header written before the slot's V is free
                if SPLIT and gt >= NKV:
                    yield ("wait", ("k_empty", kvs), gt // NKV - 1)
                if SPLIT:
                    B[("k_full", kvs)].arrive(32)
                if gt >= NKV:
                    yield ("wait", ("v_empty", kvs), gt // NKV - 1)
                if j == 0 and w == 0 and not hazard:
                    hdr[kvs] = gt
                B[("stg_empty", st)].arrive(32)
                if not SPLIT:
                    B[("k_full", kvs)].arrive(32)
                B[("v_full", kvs)].arrive(32)
                if j == 0 and k + 1 < len(items):
                    B[("red", (k + 1) % 5)].arrive()
                gt += 1

    def softmax(qt, w):
        act = [it for k_it, it in enumerate(items) if qt in qts_of(k_it, it)]
        if act:
            B[("q_full", qt)].arrive()
        n, epi = 0, False
        for a, it in enumerate(act):
            gt0 = items.index(it) * T
            for j in range(T):
                yield ("wait", ("s_full", qt, n % NS), n // NS)
                if j == 0:
                    yield ("wait", ("v_full", gt0 % NKV), gt0 // NKV)
                    if hdr[gt0 % NKV] != gt0:
                        errors.append(f"soft{qt}.{w}: header of tile {gt0} overwritten")
                if j == T - 1 and a + 1 < len(act):
                    B[("q_full", qt)].arrive()
                if j >= 1 and rng.random() < 0.3:  # a rescale of O
                    yield ("wait", ("pv_done", qt, (n - 1) % NS), (n - 1) // NS)
                if j == 0 and epi:
                    epi = False
                    yield ("wait", ("pv_done", qt, (n - 1) % NS), (n - 1) // NS)
                B[("p_full", qt, n % NS)].arrive()
                n += 1
            epi = True
        if epi:
            yield ("wait", ("pv_done", qt, (n - 1) % NS), (n - 1) // NS)

    gens = {"mma": mma(), "prod": producer()}
    gens.update({f"unpack{w}": unpack(w) for w in range(UW)})
    gens.update({f"soft{qt}.{w}": softmax(qt, w) for qt in range(NQT) for w in range(4)})
    waiting = {name: None for name in gens}
    alive = set(gens)

    def step(name):
        try:
            waiting[name] = next(gens[name])
        except StopIteration:
            alive.discard(name)
            waiting[name] = None

    for name in list(alive):
        step(name)
    idle = 0
    while alive:
        now[0] += 1
        due = [x for x in asyncq if x[0] <= now[0]]
        rng.shuffle(due)
        for x in due:
            asyncq.remove(x)
            b = B[x[1]]
            b.arrive(b.count - b.pending if x[1][0] == "stg_full" else 1)
        progressed = bool(due)
        order = sorted(alive)
        rng.shuffle(order)
        for name in order:
            req = waiting[name]
            if req is None:
                continue
            b = B[req[1]]
            if b.phase > req[2] + 1:
                errors.append(f"{name}: {req[1]} two phases ahead of its parity wait")
                return errors
            if b.phase == req[2] + 1:
                step(name)
                progressed = True
        if not progressed and not asyncq:
            idle += 1
            if idle > 3:
                errors.append("deadlock: " + ", ".join(f"{n} waits {waiting[n]}" for n in sorted(alive) if waiting[n]))
                return errors
        else:
            idle = 0
        assert now[0] < 10 ** 6
    return errors


def protocol_cases(D, ALT, BITS=3):
    c = pipe_cfg(BITS, D, 2)
    for T in (1, 2, 3, 11):
        for n_qt in ((1, 2, 3) if ALT else (1, 2, 3, 5)):
            for grid, cta in ((1, 0), (3, 1), (7, 6)):
                n_groups = n_qt if ALT else -(-n_qt // 2)
                for bh in (1, 4, 9):
                    if cta < bh * n_groups:
                        yield dict(NQT=2, NS=c["NS"], NKV=c["NKV"], T=T, n_items=bh * n_groups, grid=grid,
                                   n_qt=n_qt, cta=cta, ALT=ALT, SPLIT=c["SPLIT"], NSTG=c["NSTG"], UW=c["UW"])


@pytest.mark.parametrize("D,ALT,BITS", [(64, True, 3), (64, False, 3), (128, True, 3), (128, False, 3),
                                         (64, True, 8), (64, False, 8)])
def test_barrier_protocol_is_clean(D, ALT, BITS):
    """Every ring configuration the kernel is built with: (3 K/V slots, 3 stages)
    and (3, 2) at head_dim 64 (8+ and fewer codes per word), (2, 2) at 128."""
    n = 0
    for case in protocol_cases(D, ALT, BITS):
        for seed in range(2):
            errs = simulate(seed=seed, **case)
            assert not errs, (case, seed, errs[:2])
            n += 1
    assert n > 50


def test_barrier_simulation_finds_a_planted_hazard():
    bad = 0
    for case in protocol_cases(128, True):
        if case["T"] == 1:
            bad += bool(simulate(seed=0, hazard=True, **case))
    assert bad > 0


# ------------------------------------------------------------------ CUDA-core kernel (attention.cuh)
CC_MAX_SMEM, CC_MAX_QUERIES, SMALL_MAX_QUERIES = 76 * 1024, 32, 4


def cc_layout(n_q, P, D):
    PP, NQP = (P + 31) & ~31, (n_q + 7) & ~7
    KS = PP + 1
    kt = 0
    vs = (kt + D * KS + 3) & ~3
    qs = vs + PP * D
    ps = qs + NQP * D
    linv = ps + NQP * PP
    return dict(PP=PP, NQP=NQP, KS=KS, kt=kt, vs=vs, qs=qs, ps=ps, linv=linv, floats=linv + NQP)


def dispatch(n_q, P, D):
    if n_q <= SMALL_MAX_QUERIES:
        return "small"
    if n_q <= CC_MAX_QUERIES and cc_layout(n_q, P, D)["floats"] * 4 <= CC_MAX_SMEM:
        return "cc"
    return "pipe"


def check_cc_block(sched, s, D, bits):
    CPW = 32 // bits
    n_q, P = sched[s], sum(sched[: s + 1])
    L = cc_layout(n_q, P, D)
    PP, NQP, KS = L["PP"], L["NQP"], L["KS"]
    assert L["vs"] % 4 == 0 and L["qs"] % 4 == 0 and L["ps"] % 4 == 0  # float4 rows stay 16-byte aligned
    kt_end, vs_end = L["kt"] + (D - 1) * KS + PP, L["vs"] + PP * D
    assert kt_end <= L["vs"] and vs_end <= L["qs"]
    assert L["qs"] + NQP * D <= L["ps"] and L["ps"] + NQP * PP <= L["linv"]
    # dequantize: every (block, word row, channel) item lands on keys < P, each key once
    keys, key = set(), 0
    for kb in range(s + 1):
        for w in range(-(-sched[kb] // CPW)):
            ns = min(CPW, sched[kb] - w * CPW)
            assert ns >= 1
            for i in range(ns):
                j = key + w * CPW + i
                assert j < P and j not in keys
                keys.add(j)
        key += sched[kb]
    assert keys == set(range(P))
    # bank pattern of the dequantize stores: a warp's 32 consecutive channels of one key
    assert len({(c * KS + 5) % 32 for c in range(32)}) == 32


@pytest.mark.parametrize("D", [64, 128])
def test_cc_kernel_layout_and_dispatch(D):
    rng = random.Random(D)
    scheds = [VAR_BLOCKS, INFINITY_BLOCKS, [1, 2, 7, 11, 81, 300, 1100, 4095], [300, 200, 5, 3]]
    scheds += [[rng.randint(1, 70) for _ in range(rng.randint(1, 10))] for _ in range(100)]
    for sched in scheds:
        for s in range(len(sched)):
            if dispatch(sched[s], sum(sched[: s + 1]), D) == "cc":
                for bits in (2, 3, 4, 6, 8):
                    check_cc_block(sched, s, D, bits)
    # the VAR schedule at head_dim 64: blocks 0-1 warp per query, 2-4 CUDA-core, 5-9 tensor cores
    if D == 64:
        got = [dispatch(n, sum(VAR_BLOCKS[: s + 1]), 64) for s, n in enumerate(VAR_BLOCKS)]
        assert got == ["small"] * 2 + ["cc"] * 3 + ["pipe"] * 5
    # few queries over many keys fall through to the tensor cores
    assert dispatch(5, 505, D) == "pipe"


# ------------------------------------------------------------------ work items -> query rows
def pipe_rows_written(n_q, BH, grid):
    """(bh, row) -> count of softmax threads that write it, for the launch mode
    the dispatch picks: two query tiles per item above 128 queries, otherwise
    one tile per item with the two warpgroups taking the CTA's items in turn."""
    ALT = n_q <= 128
    n_qt = -(-n_q // 128)
    n_groups = n_qt if ALT else -(-n_qt // 2)
    n_items = BH * n_groups

    def item_nqt(item):
        return 1 if ALT else min(2, n_qt - (item % n_groups) * 2)

    written = {}
    mma_tiles = {}
    for cta in range(min(grid, n_items)):
        # the MMA thread: k-th item of the CTA covers query tiles [qlo, qhi)
        for k, item in enumerate(range(cta, n_items, grid)):
            qlo, qhi = (k & 1, (k & 1) + 1) if ALT else (0, item_nqt(item))
            for qt in range(qlo, qhi):
                mma_tiles[(item, qt)] = mma_tiles.get((item, qt), 0) + 1
        for qt in range(2):
            roff = 128 - n_q if (ALT and qt == 1) else 0
            item = cta + (qt * grid if ALT else 0)
            if not ALT and item < n_items and item_nqt(item) <= qt:
                item += grid
                while item < n_items and item_nqt(item) <= qt:
                    item += grid
            while item < n_items:
                assert mma_tiles.get((item, qt)) == 1, (item, qt)  # the MMA thread serves this tile
                for row in range(128):
                    r = row - roff if ALT else (item % n_groups) * 256 + qt * 128 + row
                    if 0 <= r < n_q:
                        key = (item // n_groups, r)
                        written[key] = written.get(key, 0) + 1
                if ALT:
                    item += 2 * grid
                else:
                    item += grid
                    while item < n_items and item_nqt(item) <= qt:
                        item += grid
    return written


@pytest.mark.parametrize("n_q", [5, 16, 64, 100, 128, 129, 169, 256, 300, 576, 1024])
def test_every_query_row_is_written_once(n_q):
    for BH, grid in ((1, 1), (3, 2), (7, 148), (40, 148), (300, 148)):
        w = pipe_rows_written(n_q, BH, grid)
        assert set(w) == {(bh, r) for bh in range(BH) for r in range(n_q)}
        assert set(w.values()) == {1}
