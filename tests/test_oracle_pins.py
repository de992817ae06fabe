"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test checks the oracle against a fact the pages or the mathematics fix:
the KV-memory numbers printed in "VAR-Q results data (Tables 2-4)", the
nearest-grid-level property of asymmetric min/max quantization, exact special
cases, bit-level packing, exact rational arithmetic for the fused multiply-add,
and float64 brute force for the attention. `test_planted_mistakes_are_caught`
plants plausible mistakes in the oracle and checks that the pins fail.
"""
import math
import os
import shlex
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle.vq_oracle as vo
from workloads import WORKLOADS, make_kv, make_q

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "varq_kv_memory.txt")

# Model shapes behind the table rows: VAR-dN has N layers and hidden 64*N over the
# 10-scale 680-token schedule; Infinity-2B has 32 layers, hidden 2048, 13 scales,
# 10521 tokens. The KV figures count twice the stated batch (classifier-free
# guidance doubles the batch). Infinity-8B's shape is not known, so only its
# saving and the ratio to its own BF16 row are checked.
SHAPES = {"var20": (20, 1280, 680, 10), "var24": (24, 1536, 680, 10),
          "var30": (30, 1920, 680, 10), "infinity2": (32, 2048, 10521, 13),
          "infinity8": (None, None, 10521, 13)}


def _golden_rows():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        ds, table, setting, method, prec, kv, saving = shlex.split(line)
        batch = int(setting.split("batch")[-1])
        rows.append(dict(ds=ds, batch=batch, method=method,
                         bits=None if prec == "BF16" else int(prec[3:]),
                         kv=float(kv), saving=None if saving == "-" else float(saving)))
    return rows


def check_kv_memory(paper_kv_gib):
    rows = _golden_rows()
    assert len(rows) == 18
    bf16 = {r["ds"]: r["kv"] for r in rows if r["bits"] is None}
    for r in rows:
        L, hid, N, S = SHAPES[r["ds"]]
        if L is not None:
            gib, saving = paper_kv_gib(L, hid, N, S, 2 * r["batch"], r["bits"])
            assert round(gib, 2) == r["kv"], (r, gib)
        else:
            _, saving = paper_kv_gib(1, 1, N, S, 2 * r["batch"], r["bits"])
            if r["bits"] is not None:
                assert abs(bf16[r["ds"]] * (1 - saving / 100) - r["kv"]) <= 0.006, r
        if r["saving"] is not None:
            assert round(saving, 2) == r["saving"], (r, saving)


def test_kv_memory_matches_printed_tables():
    check_kv_memory(vo.paper_kv_gib)


# ------------------------------------------------------------------ quantizer
def _f32(v):
    return struct.unpack("f", struct.pack("f", v))[0]


def _rand_block(rng, B, H, n, D, kind="normal"):
    if kind == "normal":
        x = rng.standard_normal((B, H, n, D)).astype(np.float32)
        x[..., ::7] *= 30.0
        x += rng.uniform(-5, 5, size=(B, H, 1, 1)).astype(np.float32)
    elif kind == "bf16":
        t = torch.from_numpy(rng.standard_normal((B, H, n, D)).astype(np.float32) * 40).to(torch.bfloat16)
        x = t.float().numpy()
    return x


def check_grid_properties(quantize_pack_block, dequantize, rng):
    """Codes are in range, hit the extreme levels, and pick the nearest grid level."""
    for bits in (4, 3, 2, 6, 8):
        for n in (1, 2, 3, 5, 7, 10, 11, 16, 33):
            x = _rand_block(rng, 2, 2, n, 16)
            words, scale, zero = quantize_pack_block(x, bits)
            codes = vo.unpack(words, bits, n).astype(np.int64)
            assert codes.min() >= 0 and codes.max() <= (1 << bits) - 1
            mn = x.min(axis=2)
            mx = x.max(axis=2)
            # zero is the exact group min (x == min gets code 0); the max gets the top level
            np.testing.assert_array_equal(zero, mn + np.float32(0))
            for b in range(2):
                for h in range(2):
                    for c in range(16):
                        col = [float(v) for v in x[b, h, :, c]]
                        lo, hi = min(col), max(col)
                        s = float(scale[b, h, c])
                        if n == 1 or lo == hi:
                            assert s == 0.0 and all(codes[b, h, :, c] == 0)
                            continue
                        # grid step: the exact (max - min)/(2^b - 1) within one float32 rounding
                        exact = (Fraction(hi) - Fraction(lo)) / ((1 << bits) - 1)
                        assert abs(Fraction(s) - exact) <= exact * Fraction(1, 2**23)
                        tmin = col.index(lo)
                        tmax = col.index(hi)
                        assert codes[b, h, tmin, c] == 0
                        assert codes[b, h, tmax, c] == (1 << bits) - 1
                        for t in range(n):
                            k = int(codes[b, h, t, c])
                            dist = abs(col[t] - (lo + k * s))
                            # nearest level: no other level is closer by more than rounding slack
                            slack = 1e-5 * s + 4 * np.spacing(np.float32(abs(col[t]) + abs(lo)))
                            for k2 in (k - 1, k + 1):
                                if 0 <= k2 < (1 << bits):
                                    assert dist <= abs(col[t] - (lo + k2 * s)) + slack
            xh = dequantize(words, scale, zero, bits, n)
            err = np.abs(xh.astype(np.float64) - x.astype(np.float64))
            bound = scale[:, :, None, :].astype(np.float64) / 2 * (1 + 2.0 ** -16) + \
                np.spacing(np.abs(x) + np.abs(mn[:, :, None, :])).astype(np.float64)
            assert np.all(err <= bound)


def test_quantizer_grid_properties():
    check_grid_properties(vo.quantize_pack_block, vo.dequantize, np.random.default_rng(1))


def _tiny_range_blocks(rng):
    """Groups whose whole range is tiny: subnormal values (scale below 2^-128,
    where 1/scale overflows float32), normal values with a scale just under and
    over 2^-100, and the arithmetic progression 1e-40 * [0, 19]."""
    cols = [1e-40 * np.arange(20, dtype=np.float64),
            1e-40 * np.arange(20, dtype=np.float64)[::-1] - 3e-40,
            rng.uniform(-1, 1, 20) * 2.0 ** -135,
            rng.uniform(0, 1, 20) * 2.0 ** -146,
            2.0 ** -110 * (1 + rng.uniform(0, 2.0 ** -6, 20)),
            rng.uniform(-1, 1, 20) * 2.0 ** -96,
            rng.uniform(-1, 1, 20) * 2.0 ** -99,
            rng.standard_normal(20)]
    x = np.stack(cols, axis=-1).astype(np.float32)          # [20][8]
    return x.reshape(1, 1, 20, len(cols))


def check_tiny_range_groups(quantize_pack_block, dequantize, rng):
    """Exact-rational check of the nearest grid level on tiny-range groups.

    With t_exact = (x - min) / scale computed in exact rationals from the stored
    scale and clamped to [0, 2^b - 1], every code must be within 1/2 + 2^-16 of
    t_exact (the nearest level up to the float32 roundings of d and t), min -> 0,
    max -> 2^b - 1 where the scale is a normal float, and the dequantized value
    within scale/2 (1 + 2^-16) + one ulp of the input + (2^b - 1) 2^-150 (the
    rounding of a subnormal scale, accumulated over the levels).
    """
    for bits in (2, 3, 4, 6, 8):
        for n in (20, 11, 3):
            x = _tiny_range_blocks(rng)[:, :, :n]
            words, scale, zero = quantize_pack_block(x, bits)
            codes = vo.unpack(words, bits, n).astype(np.int64)
            for c in range(x.shape[-1]):
                col = [float(v) for v in x[0, 0, :, c]]
                lo, hi = min(col), max(col)
                s = float(scale[0, 0, c])
                if s == 0.0:
                    # flat group, or a range so small that (max - min)/(2^b - 1)
                    # rounds to zero (below half the smallest subnormal): codes 0
                    assert (Fraction(hi) - Fraction(lo)) / ((1 << bits) - 1) <= Fraction(1, 2**150)
                    assert all(codes[0, 0, :, c] == 0)
                    continue
                assert codes[0, 0, col.index(lo), c] == 0
                if s >= 2.0 ** -126:
                    # a normal scale is within 2^-24 of (max - min)/(2^b - 1), so the
                    # max is nearest the top level; a subnormal scale can be off by
                    # more than half a level over 2^b - 1 steps, and then the
                    # nearest-level check below is the property that holds
                    assert codes[0, 0, col.index(hi), c] == (1 << bits) - 1, (bits, n, c)
                for t in range(n):
                    # exact grid position, clamped to the 2^b levels (a subnormal
                    # scale can put the max past the top level)
                    t_exact = min(max((Fraction(col[t]) - Fraction(lo)) / Fraction(s), Fraction(0)),
                                  Fraction((1 << bits) - 1))
                    assert abs(codes[0, 0, t, c] - t_exact) <= Fraction(1, 2) + Fraction(1, 2**16), \
                        (bits, n, c, t, float(t_exact), codes[0, 0, t, c])
            xh = dequantize(words, scale, zero, bits, n)
            err = np.abs(xh.astype(np.float64) - x.astype(np.float64))
            mn = x.min(axis=2, keepdims=True)
            # plus (2^b - 1) * 2^-150: a subnormal scale is rounded to an absolute
            # 2^-150, so the top level can fall that far short of the max
            bound = scale[:, :, None, :].astype(np.float64) / 2 * (1 + 2.0 ** -16) + \
                np.spacing(np.abs(x) + np.abs(mn)).astype(np.float64) + ((1 << bits) - 1) * 2.0 ** -150
            flat = (scale == 0)[:, :, None, :]
            bound = np.where(flat, (x.max(axis=2, keepdims=True) - mn).astype(np.float64), bound)
            assert np.all(err <= bound), (bits, n, float(np.max(err / bound)))


def test_quantizer_tiny_range_groups():
    check_tiny_range_groups(vo.quantize_pack_block, vo.dequantize, np.random.default_rng(10))


def test_quantizer_bf16_inputs_and_min_max_exact():
    rng = np.random.default_rng(2)
    x = _rand_block(rng, 2, 3, 29, 64, kind="bf16")
    mn, mx = vo.group_min_max(x)
    for b in range(2):
        for h in range(3):
            for c in range(64):
                col = [float(v) for v in x[b, h, :, c]]
                assert mn[b, h, c] == min(col) and mx[b, h, c] == max(col)


def test_quantizer_matches_scalar_brute_force():
    """numpy float32 semantics vs scalar Python with float32 rounding after each op.

    +, -, *, / of float32 values done in float64 and rounded once to float32 give
    the correctly rounded float32 result (53 >= 2*24 + 2), so this scalar version
    is an independent check that the vectorised oracle really works in float32.
    """
    rng = np.random.default_rng(3)
    for bits in (4, 3, 6, 8):
        x = _rand_block(rng, 1, 2, 13, 8)
        words, scale, zero = vo.quantize_pack_block(x, bits)
        codes = vo.unpack(words, bits, 13)
        for h in range(2):
            for c in range(8):
                col = [float(v) for v in x[0, h, :, c]]
                lo, hi = min(col), max(col)
                s = _f32(_f32(hi - lo) / float((1 << bits) - 1))
                assert s == float(scale[0, h, c])
                inv = _f32(1.0 / s)
                for t in range(13):
                    tt = _f32(_f32(col[t] - lo) * inv)
                    k = min(max(int(round(tt)), 0), (1 << bits) - 1)  # Python round = half even
                    assert k == codes[0, h, t, c]


def test_special_cases_constant_equispaced_single_token():
    # constant group: scale 0, codes 0, exact reconstruction
    x = np.full((1, 1, 9, 4), 3.25, dtype=np.float32)
    w, s, z = vo.quantize_pack_block(x, 4)
    assert np.all(s == 0) and np.all(w == 0)
    np.testing.assert_array_equal(vo.dequantize(w, s, z, 4, 9), x)
    # exactly 2^b equispaced levels reconstruct exactly
    for bits in (2, 3, 4, 6):
        levels = (1 << bits)
        base = np.float32(-1.5)
        step = np.float32(0.25)
        vals = base + step * np.arange(levels, dtype=np.float32)
        x = np.tile(vals[::-1].reshape(1, 1, levels, 1), (1, 1, 1, 3)).astype(np.float32)
        w, s, z = vo.quantize_pack_block(x, bits)
        assert np.all(s == step) and np.all(z == base)
        np.testing.assert_array_equal(vo.dequantize(w, s, z, bits, levels), x)
        np.testing.assert_array_equal(vo.unpack(w, bits, levels)[0, 0, :, 0], np.arange(levels)[::-1])
    # one token: every group is flat
    x = np.random.default_rng(4).standard_normal((2, 2, 1, 8)).astype(np.float32)
    w, s, z = vo.quantize_pack_block(x, 3)
    assert np.all(s == 0) and np.all(w == 0)
    np.testing.assert_array_equal(vo.dequantize(w, s, z, 3, 1), x)
    # negative zero min is stored as +0
    x = np.array([-0.0, 1.0, 2.0], dtype=np.float32).reshape(1, 1, 3, 1)
    _, _, z = vo.quantize_pack_block(x, 4)
    assert np.signbit(z).sum() == 0


def test_pack_layout_bit_level_and_round_trip():
    rng = np.random.default_rng(5)
    for bits in (2, 3, 4, 6, 8):
        cpw = 32 // bits
        for n in (1, cpw - 1, cpw, cpw + 1, 3 * cpw + 2):
            codes = rng.integers(0, 1 << bits, size=(2, 1, n, 5)).astype(np.uint8)
            words = vo.pack(codes, bits)
            assert words.shape == (2, 1, (n + cpw - 1) // cpw, 5)
            np.testing.assert_array_equal(vo.unpack(words, bits, n), codes)
            for b in range(2):
                for c in range(5):
                    for w in range(words.shape[2]):
                        word = int(words[b, 0, w, c])
                        for pos in range(32):
                            bit = (word >> pos) & 1
                            slot, j = divmod(pos, bits)
                            t = w * cpw + slot
                            if slot >= cpw or t >= n:
                                assert bit == 0  # padding and unused high bits
                            else:
                                assert bit == (int(codes[b, 0, t, c]) >> j) & 1


def test_cache_layout_matches_enumeration():
    sched = (1, 4, 9, 16, 25)
    B, H, D = 2, 3, 8
    for bits in (4, 3):
        total, meta, offs = vo.cache_layout(sched, B, H, D, bits)
        idx = 0
        for s, n in enumerate(sched):
            assert offs[s] == idx
            for _b in range(B):
                for _h in range(H):
                    for _w in range(-(-n // (32 // bits))):
                        idx += D
        assert total == idx and meta == len(sched) * B * H * D
        x = np.random.default_rng(6).standard_normal((B, H, sum(sched), D)).astype(np.float32)
        packed, sc, z = vo.cache_append(x, sched, bits)
        t0 = 0
        for s, n in enumerate(sched):
            w, s1, z1 = vo.quantize_pack_block(x[:, :, t0:t0 + n], bits)
            np.testing.assert_array_equal(packed[offs[s]:offs[s + 1]], w.reshape(-1))
            np.testing.assert_array_equal(sc[s * B * H * D:(s + 1) * B * H * D], s1.reshape(-1))
            t0 += n


# ------------------------------------------------------------------ fma
def _round_f32_exact(fr: Fraction) -> np.float32:
    c = np.float32(float(fr))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    best = None
    for v in cands:
        d = abs(Fraction(float(v)) - fr)
        if best is None or d < best[0] or (d == best[0] and (np.float32(v).view(np.uint32) & 1) == 0):
            best = (d, v)
    return np.float32(best[1])


def check_fma(fma):
    rng = np.random.default_rng(7)
    a = rng.integers(0, 16, 400).astype(np.float32)
    b = (rng.standard_normal(400) * 10).astype(np.float32)
    c = (rng.standard_normal(400) * 100).astype(np.float32)
    # adversarial: a*b exactly on a float32 midpoint, c a tiny nudge either way
    a2 = np.array([1 + 2**-12] * 4 + [3.0] * 2, dtype=np.float32)
    b2 = np.array([1 + 2**-12] * 4 + [np.float32(1 + 2**-23)] * 2, dtype=np.float32)
    c2 = np.array([2**-60, -2**-60, 2**-30, 0.0, 2**-70, -2**-70], dtype=np.float32)
    a, b, c = np.concatenate([a, a2]), np.concatenate([b, b2]), np.concatenate([c, c2])
    got = fma(a, b, c)
    for i in range(len(a)):
        exact = Fraction(float(a[i])) * Fraction(float(b[i])) + Fraction(float(c[i]))
        assert got[i] == _round_f32_exact(exact), (i, a[i], b[i], c[i], got[i])


def test_fma_is_correctly_rounded():
    check_fma(vo.fma_f32)


# ------------------------------------------------------------------ attention
def _attn_brute(q, k, v, sigma):
    n, D = q.shape
    P = k.shape[0]
    out = np.zeros((n, D))
    for i in range(n):
        lg = [sigma * sum(float(q[i, c]) * float(k[t, c]) for c in range(D)) for t in range(P)]
        m = max(lg)
        e = [math.exp(l - m) for l in lg]
        z = sum(e)
        for c in range(D):
            out[i, c] = sum(e[t] * float(v[t, c]) for t in range(P)) / z
    return out


def check_attention(attention_f64):
    rng = np.random.default_rng(8)
    for n, P, D in ((1, 1, 4), (3, 5, 8), (4, 9, 6)):
        q = rng.standard_normal((1, 2, n, D)).astype(np.float32)
        k = (rng.standard_normal((1, 2, P, D)) * 3).astype(np.float32)
        v = rng.standard_normal((1, 2, P, D)).astype(np.float32)
        sigma = 0.37
        got = attention_f64(q, k, v, sigma)
        for h in range(2):
            ref = _attn_brute(q[0, h], k[0, h], v[0, h], float(np.float32(sigma)))
            np.testing.assert_allclose(got[0, h], ref, rtol=1e-12, atol=1e-12)
    # one key: the output is that key's value row
    q = rng.standard_normal((1, 1, 3, 4)).astype(np.float32)
    k = rng.standard_normal((1, 1, 1, 4)).astype(np.float32)
    v = rng.standard_normal((1, 1, 1, 4)).astype(np.float32)
    np.testing.assert_allclose(attention_f64(q, k, v, 0.5)[0, 0], np.repeat(v[0, 0], 3, 0), rtol=0, atol=0)
    # zero query: uniform weights, the mean of the values
    q = np.zeros((1, 1, 2, 4), dtype=np.float32)
    k = rng.standard_normal((1, 1, 6, 4)).astype(np.float32)
    v = rng.standard_normal((1, 1, 6, 4)).astype(np.float32)
    np.testing.assert_allclose(attention_f64(q, k, v, 0.5)[0, 0], np.repeat(v[0, 0].astype(np.float64).mean(0, keepdims=True), 2, 0), rtol=1e-14)
    # two keys: weight of key 0 is the logistic function of the logit difference
    q = rng.standard_normal((1, 1, 1, 4)).astype(np.float32)
    k = rng.standard_normal((1, 1, 2, 4)).astype(np.float32)
    v = np.eye(2, 4, dtype=np.float32).reshape(1, 1, 2, 4)
    d = 0.5 * float(np.dot(q[0, 0, 0].astype(np.float64), (k[0, 0, 1].astype(np.float64) - k[0, 0, 0].astype(np.float64))))
    w0 = 1.0 / (1.0 + math.exp(d))
    np.testing.assert_allclose(attention_f64(q, k, v, 0.5)[0, 0, 0, :2], [w0, 1 - w0], rtol=1e-13)


def test_attention_against_brute_force_and_closed_forms():
    check_attention(vo.attention_f64)


def test_tiny_workload_end_to_end_consistency():
    """Whole tiny decode: every block's cache region and attention via the oracle."""
    w = WORKLOADS["tiny"]
    k, v = make_kv(w, 0)
    q = make_q(w, 0)
    sched = w.block_tokens
    B, H, D = w.batch, w.heads, w.head_dim
    for bits in w.bits:
        pk, sk, zk = vo.cache_append(k.numpy(), sched, bits)
        pv, sv, zv = vo.cache_append(v.numpy(), sched, bits)
        for s in range(w.num_blocks):
            kh = vo.dequantize_cache(pk, sk, zk, sched, B, H, D, bits, s)
            vh = vo.dequantize_cache(pv, sv, zv, sched, B, H, D, bits, s)
            p0 = w.prefix(s)
            qs = q[:, :, p0:p0 + sched[s]].float().numpy()
            o = vo.attention_f64(qs, kh, vh, 0.125)
            assert o.shape == (B, H, sched[s], D) and np.all(np.isfinite(o))
            # the quantized cache stays within half a step of the input
            ks = k[:, :, :p0 + sched[s]].numpy()
            scales = np.concatenate([np.repeat(sk[j * D:(j + 1) * D].reshape(1, 1, 1, D), sched[j], 2) for j in range(s + 1)], 2)
            assert np.all(np.abs(kh - ks) <= scales / 2 * (1 + 2**-16) + np.spacing(np.abs(ks) + 60))


# ------------------------------------------------------------------ planted mistakes
def test_planted_mistakes_are_caught(monkeypatch):
    """Plausible oracle mistakes (wrong level count, floor instead of round, a
    saturated 1/scale without the power-of-two prescale, missing sigma,
    transposed value operand, double-rounded fma, payload 3 bits for INT3) each
    fail at least one pin above."""
    rng = np.random.default_rng(9)

    def wrong_levels(mn, mx, bits):
        levels = np.float32(1 << bits)
        return ((mx - mn) / levels).astype(np.float32), (mn + np.float32(0)).astype(np.float32)

    def qpb_with(scale_zero=None, rint=None, recip=None):
        def f(x, bits):
            x = np.asarray(x, dtype=np.float32)
            mn, mx = vo.group_min_max(x)
            sc, z = (scale_zero or vo.scale_zero)(mn, mx, bits)
            inv = (recip or vo.reciprocal)(sc)[:, :, None, :]
            pre = (vo.prescale(sc) if recip is None else np.ones_like(sc))[:, :, None, :]
            d = ((x - mn[:, :, None, :]).astype(np.float32) * pre).astype(np.float32)
            t = (d * inv).astype(np.float32)
            r = (rint or np.rint)(t)
            codes = np.where(sc[:, :, None, :] > 0, np.clip(r, 0, (1 << bits) - 1), 0).astype(np.uint8)
            return vo.pack(codes, bits), sc, z
        return f

    with pytest.raises(AssertionError):
        check_grid_properties(qpb_with(scale_zero=wrong_levels), vo.dequantize, rng)
    with pytest.raises(AssertionError):
        check_grid_properties(qpb_with(rint=np.floor), vo.dequantize, rng)

    def saturating_reciprocal(sc):
        # 1/scale capped at FLT_MAX, with no power-of-two prescale of d and scale
        with np.errstate(divide="ignore", over="ignore"):
            inv = (np.float32(1) / sc).astype(np.float32)
        return np.where(sc > 0, np.minimum(inv, np.finfo(np.float32).max), 0).astype(np.float32)

    with pytest.raises(AssertionError):
        check_tiny_range_groups(qpb_with(recip=saturating_reciprocal), vo.dequantize, rng)
    # the pins still pass through the same helper with the oracle's own steps
    check_tiny_range_groups(qpb_with(), vo.dequantize, rng)
    with pytest.raises(AssertionError):
        check_attention(lambda q, k, v, s: vo.attention_f64(q, k, v, 1.0))
    with pytest.raises(AssertionError):
        check_attention(lambda q, k, v, s: vo.attention_f64(q, k, v[..., ::-1, :], s))
    with pytest.raises(AssertionError):
        check_fma(lambda a, b, c: (a.astype(np.float64) * b + c).astype(np.float32))
    monkeypatch.setattr(vo, "payload_bits", lambda bits: float(bits))
    with pytest.raises(AssertionError):
        check_kv_memory(vo.paper_kv_gib)


# ------------------------------------------------------------------ paper-exact storage
VAR_SCHED = tuple(r * r for r in (1, 2, 3, 4, 5, 6, 8, 10, 13, 16))
INF_SCHED = tuple(r * r for r in (1, 2, 4, 6, 8, 12, 16, 20, 24, 32, 40, 48, 64))
# table shape -> (layers, heads, head_dim, schedule)
PAPER_SHAPES = {"var20": (20, 20, 64, VAR_SCHED), "var24": (24, 24, 64, VAR_SCHED),
                "var30": (30, 30, 64, VAR_SCHED), "infinity2": (32, 16, 128, INF_SCHED)}


def check_paper_layout(paper_layout):
    """Bytes of the paper storage format for every VAR-Q image row of Tables
    2a/2b whose model shape is known equal the printed KV GiB and saving."""
    n = 0
    for r in _golden_rows():
        if r["bits"] is None or r["ds"] not in PAPER_SHAPES:
            continue
        L, H, D, sched = PAPER_SHAPES[r["ds"]]
        words, meta, _ = paper_layout(sched, 2 * r["batch"], H, D, r["bits"])
        gib = L * 2 * (words + meta) * 4 / 2**30
        assert round(gib, 2) == r["kv"], (r, gib)
        bf16 = L * 2 * 2 * r["batch"] * H * D * sum(sched) * 2 / 2**30
        assert round(100 * (1 - gib / bf16), 2) == r["saving"], (r, gib)
        n += 1
    assert n == 9   # VAR-d20/d24/d30 INT4 and INT3, Infinity-2B INT8, INT4 and INT3


def test_paper_layout_reproduces_printed_kv_memory():
    check_paper_layout(vo.paper_layout)


def test_paper_stream_bit_layout_and_round_trip():
    rng = np.random.default_rng(11)
    for bits in (2, 3, 4, 6, 8):
        cpw = 32 // bits
        for B, H, n, D in ((1, 1, 1, 4), (2, 3, 5, 8), (1, 2, 7, 6)):
            codes = rng.integers(0, 1 << bits, size=(B, H, n, D)).astype(np.uint8)
            words = vo.paper_pack_block(codes, bits)
            assert words.shape == (-(-(B * H * n * D) // cpw),)
            np.testing.assert_array_equal(vo.paper_unpack_block(words, bits, B, H, n, D), codes)
            flat = codes.reshape(-1)
            for wi, word in enumerate(int(x) for x in words):
                for pos in range(32):
                    slot, j = divmod(pos, bits)
                    i = wi * cpw + slot
                    want = 0 if (slot >= cpw or i >= flat.size) else (int(flat[i]) >> j) & 1
                    assert (word >> pos) & 1 == want


def check_fp16_metadata_grid(quantize_pack_block, rng):
    """fp16 metadata: scale and zero are fp16 values (the pair packs into 32
    bits and unpacks exactly), zero is the min rounded to fp16, and every code
    is the nearest level of the stored grid, clamped to [0, 2^b - 1]."""
    for bits in (2, 3, 4, 6, 8):
        x = _rand_block(rng, 1, 2, 19, 8)
        words, scale, zero = quantize_pack_block(x, bits, meta_fp16=True)
        np.testing.assert_array_equal(scale, scale.astype(np.float16).astype(np.float32))
        np.testing.assert_array_equal(zero, zero.astype(np.float16).astype(np.float32))
        meta = vo.paper_meta(scale, zero)
        np.testing.assert_array_equal((meta & 0xffff).astype(np.uint16).view(np.float16).astype(np.float32), scale)
        np.testing.assert_array_equal((meta >> 16).astype(np.uint16).view(np.float16).astype(np.float32), zero)
        codes = vo.unpack(words, bits, 19).astype(np.int64)
        levels = (1 << bits) - 1
        for h in range(2):
            for c in range(8):
                col = [float(v) for v in x[0, h, :, c]]
                assert float(zero[0, h, c]) == float(np.float16(min(col)))
                s = Fraction(float(scale[0, h, c]))
                z = Fraction(float(zero[0, h, c]))
                for t in range(19):
                    if s == 0:
                        assert codes[0, h, t, c] == 0
                        continue
                    te = min(max((Fraction(col[t]) - z) / s, Fraction(0)), Fraction(levels))
                    assert abs(codes[0, h, t, c] - te) <= Fraction(1, 2) + Fraction(1, 2**16), (bits, h, c, t)


def test_fp16_metadata_grid():
    check_fp16_metadata_grid(vo.quantize_pack_block, np.random.default_rng(12))


def test_paper_from_cache_matches_per_block_streams():
    rng = np.random.default_rng(13)
    sched, B, H, D = (1, 4, 9, 16), 2, 3, 8
    x = rng.standard_normal((B, H, sum(sched), D)).astype(np.float32) * 5
    for bits in (3, 4):
        packed, sc, z = vo.cache_append(x, sched, bits, meta_fp16=True)
        stream, meta = vo.paper_from_cache(packed, sc, z, sched, B, H, D, bits)
        words, metaw, offs = vo.paper_layout(sched, B, H, D, bits)
        assert stream.size == words and meta.size == metaw
        t0 = 0
        for s, n in enumerate(sched):
            codes = vo.unpack(vo.quantize_pack_block(x[:, :, t0:t0 + n], bits, meta_fp16=True)[0], bits, n)
            np.testing.assert_array_equal(stream[offs[s]:offs[s + 1]], vo.paper_pack_block(codes, bits))
            t0 += n
