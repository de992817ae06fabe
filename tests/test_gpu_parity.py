"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Codes, packed words, scales and zeros must be bit-exact. Attention outputs must
be within max-abs 2e-3 x RMS(reference) of the float64 oracle run on the
oracle's own dequantized cache. Inputs come from the seeded workload generator
(drawn on the GPU, copied to the host for the oracle).
"""
import numpy as np
import pytest
import torch

import oracle.vq_oracle as vo
from workloads import WORKLOADS, Workload, default_softmax_scale, make_kv, make_q

pytestmark = pytest.mark.gpu

ATTN_TOL = 2e-3


@pytest.fixture(scope="module")
def vq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_kv_cache_25_b200 import vq as _vq
    return _vq


def _host(t):
    return t.float().cpu().numpy()


def _append_all(vq, w: Workload, bits, k, v):
    desc = vq.CacheDesc(w.batch, w.heads, w.head_dim, bits, w.block_tokens)
    cache = vq.LayerCache(desc)
    for s, n in enumerate(w.block_tokens):
        p0 = w.prefix(s)
        vq.vq_cache_append(desc, cache, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n])
    torch.cuda.synchronize()
    assert vq.vq_poll_device_error() == 0
    return desc, cache


def _check_cache_bit_exact(vq, w, bits, desc, cache, k, v, bsel):
    B, H, D = w.batch, w.heads, w.head_dim
    offs = cache.block_word_offset
    for name, x, packed, scale, zero in (("k", k, cache.packed_k, cache.scale_k, cache.zero_k),
                                         ("v", v, cache.packed_v, cache.scale_v, cache.zero_v)):
        xh = _host(x[bsel])
        pk = packed.cpu().numpy().view(np.uint32)
        sc = scale.cpu().numpy()
        zr = zero.cpu().numpy()
        for s, n in enumerate(w.block_tokens):
            p0 = w.prefix(s)
            W = desc.word_rows(s)
            words, s_ref, z_ref = vo.quantize_pack_block(xh[:, :, p0:p0 + n], bits)
            got_w = pk[offs[s]:offs[s + 1]].reshape(B, H, W, D)[bsel]
            got_s = sc[s * B * H * D:(s + 1) * B * H * D].reshape(B, H, D)[bsel]
            got_z = zr[s * B * H * D:(s + 1) * B * H * D].reshape(B, H, D)[bsel]
            np.testing.assert_array_equal(got_s.view(np.uint32), s_ref.view(np.uint32), err_msg=f"{name} scale s={s}")
            np.testing.assert_array_equal(got_z.view(np.uint32), z_ref.view(np.uint32), err_msg=f"{name} zero s={s}")
            if not np.array_equal(got_w, words):
                bad = np.argwhere(got_w != words)
                raise AssertionError(f"{name} packed words differ at block {s}: {len(bad)} words, first {bad[:3]}")


def _oracle_cache(w, bits, x_host):
    """Oracle's own cache of the selected batch rows: (packed, scale, zero)."""
    return vo.cache_append(x_host, w.block_tokens, bits)


def _check_attention(vq, w, bits, desc, cache, q, k, v, bsel, rows_for_block):
    sigma = default_softmax_scale(w)
    B, H, D = w.batch, w.heads, w.head_dim
    kh_host, vh_host = _host(k[bsel]), _host(v[bsel])
    ok_, sk, zk = _oracle_cache(w, bits, kh_host)
    ov_, sv, zv = _oracle_cache(w, bits, vh_host)
    nb = len(bsel)
    worst = 0.0
    for s, n in enumerate(w.block_tokens):
        rows = rows_for_block(s, n)
        if rows is None:
            continue
        p0 = w.prefix(s)
        out = torch.full((B, H, n, D), float("nan"), dtype=torch.float32, device="cuda")
        vq.vq_attention_block(desc, cache, s, q[:, :, p0:p0 + n], sigma, out)
        torch.cuda.synchronize()
        got = out[bsel].cpu().numpy()[:, :, rows]
        khat = vo.dequantize_cache(ok_, sk, zk, w.block_tokens, nb, H, D, bits, s)
        vhat = vo.dequantize_cache(ov_, sv, zv, w.block_tokens, nb, H, D, bits, s)
        qs = _host(q[bsel][:, :, p0:p0 + n])[:, :, rows]
        ref = vo.attention_f64(qs, khat, vhat, sigma)
        rms = float(np.sqrt(np.mean(ref ** 2)))
        err = float(np.max(np.abs(got - ref))) / rms
        worst = max(worst, err)
        assert np.all(np.isfinite(got)), f"block {s}: non-finite output"
        assert err <= ATTN_TOL, f"block {s}: max|err|/rms = {err:.3e}"
    assert vq.vq_poll_device_error() == 0
    return worst


def _all_rows(s, n):
    return slice(0, n)


def _sampled_rows(last_blocks):
    def f(s, n):
        if s >= last_blocks:
            return slice(0, n)
        return slice(0, min(n, 64))
    return f


# ---------------------------------------------------------------- small configs: everything
@pytest.mark.parametrize("name", ["tiny", "var_d16"])
def test_small_configs_full_parity(vq, name):
    w = WORKLOADS[name]
    k, v = make_kv(w, 0, device="cuda")
    q = make_q(w, 0, device="cuda")
    for bits in w.bits:
        desc, cache = _append_all(vq, w, bits, k, v)
        bsel = list(range(w.batch))
        _check_cache_bit_exact(vq, w, bits, desc, cache, k, v, bsel)
        _check_attention(vq, w, bits, desc, cache, q, k, v, bsel, _all_rows)


# ---------------------------------------------------------------- full-size configs, sampled
@pytest.mark.parametrize("name", ["var_d20", "var_d30", "infinity_2b"])
def test_full_size_configs_parity(vq, name):
    w = WORKLOADS[name]
    layer = 1
    k, v = make_kv(w, layer, device="cuda")
    q = make_q(w, layer, device="cuda")
    bsel = [0, w.batch - 1]
    for bits in w.bits:
        desc, cache = _append_all(vq, w, bits, k, v)
        _check_cache_bit_exact(vq, w, bits, desc, cache, k, v, bsel)
        last = w.num_blocks - 2
        _check_attention(vq, w, bits, desc, cache, q, k, v, bsel,
                         lambda s, n: (slice(0, n) if s >= last else (slice(0, min(n, 64)) if s % 3 == 0 else None)))
        del cache
        torch.cuda.empty_cache()


# ---------------------------------------------------------------- other bit widths, video shapes
@pytest.mark.parametrize("name", ["var_d16", "infinity_2b"])
def test_other_bit_widths_parity(vq, name):
    """INT2, INT6 and INT8 caches: bit-exact cache and attention parity on the
    VAR-d16 shape (every row of one layer) and the Infinity-2B shape (sampled)."""
    w = WORKLOADS[name]
    layer = 2
    k, v = make_kv(w, layer, device="cuda")
    q = make_q(w, layer, device="cuda")
    full = name == "var_d16"
    bsel = list(range(w.batch)) if full else [0, w.batch - 1]
    last = w.num_blocks - 2

    def rows(s, n):
        if full:
            return slice(0, n)
        if s >= last:
            return slice(0, min(n, 512))
        return slice(0, min(n, 64)) if s % 4 == 0 else None

    for bits in (2, 6, 8):
        desc, cache = _append_all(vq, w, bits, k, v)
        _check_cache_bit_exact(vq, w, bits, desc, cache, k, v, bsel)
        _check_attention(vq, w, bits, desc, cache, q, k, v, bsel, rows)
        del cache
        torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["video_self_forcing", "video_longlive"])
def test_video_chunk_parity(vq, name):
    """Next-frame video shapes (uniform 4680-token chunks, head_dim 128) at the
    video rows' INT6 and INT4: one layer, two batch entries, the first three
    chunks, 128 sampled query rows per chunk."""
    import dataclasses
    w0 = WORKLOADS[name]
    w = dataclasses.replace(w0, layers=1, batch=2, chunks=w0.chunks[:3])
    k, v = make_kv(w, 0, device="cuda")
    q = make_q(w, 0, device="cuda")
    for bits in w.bits:
        desc, cache = _append_all(vq, w, bits, k, v)
        _check_cache_bit_exact(vq, w, bits, desc, cache, k, v, [0, 1])
        _check_attention(vq, w, bits, desc, cache, q, k, v, [0, 1], lambda s, n: slice(n // 2, n // 2 + 128))


# ---------------------------------------------------------------- edge cases
def _ragged_kv(sched, D, H=3, B=1, dtype=torch.bfloat16, seed=5):
    g = torch.Generator(device="cuda").manual_seed(seed)
    N = sum(sched)
    k = torch.randn((B, H, N, D), generator=g, device="cuda") * 4
    k[..., 3] *= 40
    v = torch.randn((B, H, N, D), generator=g, device="cuda") + 2
    q = torch.randn((B, H, N, D), generator=g, device="cuda").to(torch.bfloat16)
    return k.to(dtype), v.to(dtype), q


@pytest.mark.parametrize("D", [64, 128])
def test_ragged_blocks_all_bit_widths(vq, D):
    """Odd block sizes (1, INT3 word-row tails, slabs split across warp groups) for bits 2/3/4/6/8;
    dequantize is bit-exact too, and attention is within the bar at every width."""
    sched = [1, 2, 7, 11, 81, 300, 1100, 4095]
    k, v, q = _ragged_kv(sched, D)
    B, H = 1, 3
    for bits in (2, 3, 4, 6, 8):
        desc = vq.CacheDesc(B, H, D, bits, sched)
        cache = vq.LayerCache(desc)
        p0 = 0
        kh = _host(k)
        vh = _host(v)
        for s, n in enumerate(sched):
            vq.vq_cache_append(desc, cache, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n])
            W = desc.word_rows(s)
            offs = cache.block_word_offset
            packed = cache.packed_k[offs[s]:offs[s + 1]]
            scale = cache.scale_k[s * B * H * D:(s + 1) * B * H * D]
            zero = cache.zero_k[s * B * H * D:(s + 1) * B * H * D]
            deq = torch.empty((B, H, n, D), dtype=torch.float32, device="cuda")
            vq.vq_dequantize(desc, s, packed, scale, zero, deq)
            torch.cuda.synchronize()
            words, s_ref, z_ref = vo.quantize_pack_block(kh[:, :, p0:p0 + n], bits)
            v_words, v_s, v_z = vo.quantize_pack_block(vh[:, :, p0:p0 + n], bits)
            np.testing.assert_array_equal(
                cache.packed_v[offs[s]:offs[s + 1]].cpu().numpy().view(np.uint32).reshape(B, H, W, D), v_words)
            np.testing.assert_array_equal(
                cache.scale_v[s * B * H * D:(s + 1) * B * H * D].cpu().numpy().view(np.uint32),
                v_s.reshape(-1).view(np.uint32))
            np.testing.assert_array_equal(packed.cpu().numpy().view(np.uint32).reshape(B, H, W, D), words)
            np.testing.assert_array_equal(scale.cpu().numpy().view(np.uint32), s_ref.reshape(-1).view(np.uint32))
            np.testing.assert_array_equal(zero.cpu().numpy().view(np.uint32), z_ref.reshape(-1).view(np.uint32))
            x_ref = vo.dequantize(words, s_ref, z_ref, bits, n)
            np.testing.assert_array_equal(deq.cpu().numpy().view(np.uint32), x_ref.view(np.uint32))
            p0 += n
        assert vq.vq_poll_device_error() == 0
        _check_ragged_attention(vq, desc, cache, sched, q, k, v, bits, D)


@pytest.mark.parametrize("D", [64, 128])
def test_ragged_blocks_fp32_inputs(vq, D):
    """fp32 K/V through both quantize kernels: slabs of 8-100 KB take the
    shared-memory ring (teams of 1 to 6 warps at these sizes), the rest the
    register-streaming kernel; codes, scales and zeros bit-exact, attention
    within the bar."""
    sched = [1, 33, 81, 300, 1100]
    k, v, q = _ragged_kv(sched, D, dtype=torch.float32, seed=9)
    B, H = 1, 3
    for bits in (3, 4):
        desc = vq.CacheDesc(B, H, D, bits, sched)
        cache = vq.LayerCache(desc)
        kh, vh = _host(k), _host(v)
        p0 = 0
        for s, n in enumerate(sched):
            vq.vq_cache_append(desc, cache, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n])
            torch.cuda.synchronize()
            W = desc.word_rows(s)
            offs = cache.block_word_offset
            for x, packed, scale, zero in ((kh, cache.packed_k, cache.scale_k, cache.zero_k),
                                           (vh, cache.packed_v, cache.scale_v, cache.zero_v)):
                words, s_ref, z_ref = vo.quantize_pack_block(x[:, :, p0:p0 + n], bits)
                np.testing.assert_array_equal(
                    packed[offs[s]:offs[s + 1]].cpu().numpy().view(np.uint32).reshape(B, H, W, D), words)
                np.testing.assert_array_equal(scale[s * B * H * D:(s + 1) * B * H * D].cpu().numpy().view(np.uint32),
                                              s_ref.reshape(-1).view(np.uint32))
                np.testing.assert_array_equal(zero[s * B * H * D:(s + 1) * B * H * D].cpu().numpy().view(np.uint32),
                                              z_ref.reshape(-1).view(np.uint32))
            p0 += n
        assert vq.vq_poll_device_error() == 0
        _check_ragged_attention(vq, desc, cache, sched, q, k, v, bits, D)


@pytest.mark.parametrize("D", [64, 128])
def test_few_queries_over_many_keys(vq, D):
    """Blocks of 5 and 3 queries after 500 cached tokens: too many keys for the
    CUDA-core kernel's shared memory, so they run on the tensor-core kernel
    with mostly empty query tiles."""
    sched = [300, 200, 5, 3]
    k, v, q = _ragged_kv(sched, D, H=2, B=2, seed=11)
    for bits in (3, 4):
        desc = vq.CacheDesc(2, 2, D, bits, sched)
        cache = vq.LayerCache(desc)
        p0 = 0
        for s, n in enumerate(sched):
            vq.vq_cache_append(desc, cache, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n])
            p0 += n
        _check_ragged_attention(vq, desc, cache, sched, q, k, v, bits, D, B=2, H=2)


@pytest.mark.parametrize("D", [64, 128])
def test_reference_moves_mid_item(vq, D):
    """Logits that jump far above an item's running reference maximum: keys
    aligned with every query, +50 nats in the middle of the second key tile,
    +110 nats in a later tile. The tensor-core kernel moves the reference
    inside a tile (rescaling the P chunks already written, O and the row
    sums) and still matches, for the paired query tiles (block 2, 200
    queries) and the alternating mode (block 1, 48 queries)."""
    sched = [64, 48, 200]
    B, H = 1, 2
    N = sum(sched)
    g = torch.Generator(device="cuda").manual_seed(17)
    u = torch.ones(D, device="cuda")
    q = (u + 0.5 * torch.randn((B, H, N, D), generator=g, device="cuda")).to(torch.bfloat16)
    k = torch.randn((B, H, N, D), generator=g, device="cuda")
    v = torch.randn((B, H, N, D), generator=g, device="cuda") + 1.0
    kt = 64 if D == 64 else 48
    first = [kt + 20 + i for i in range(6)]   # second key tile, a chunk after its first
    later = [kt * 4 + 3 + i for i in range(3)]  # a later tile's first chunk
    k[:, :, first, :] += (50.0 / D ** 0.5) * u
    k[:, :, later, :] += (110.0 / D ** 0.5) * u
    k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    for bits in (4, 8):
        desc = vq.CacheDesc(B, H, D, bits, sched)
        cache = vq.LayerCache(desc)
        p0 = 0
        for s, n in enumerate(sched):
            vq.vq_cache_append(desc, cache, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n])
            p0 += n
        _check_ragged_attention(vq, desc, cache, sched, q, k, v, bits, D, B=B, H=H)


def _check_ragged_attention(vq, desc, cache, sched, q, k, v, bits, D, B=1, H=3):
    sigma = 1.0 / np.sqrt(D)
    ok_, sk, zk = vo.cache_append(_host(k), sched, bits)
    ov_, sv, zv = vo.cache_append(_host(v), sched, bits)
    p0 = 0
    for s, n in enumerate(sched):
        out = torch.full((B, H, n, D), float("nan"), dtype=torch.float32, device="cuda")
        vq.vq_attention_block(desc, cache, s, q[:, :, p0:p0 + n], float(sigma), out)
        torch.cuda.synchronize()
        rows = slice(0, min(n, 300))
        khat = vo.dequantize_cache(ok_, sk, zk, sched, B, H, D, bits, s)
        vhat = vo.dequantize_cache(ov_, sv, zv, sched, B, H, D, bits, s)
        ref = vo.attention_f64(_host(q[:, :, p0:p0 + n])[:, :, rows], khat, vhat, sigma)
        got = out.cpu().numpy()[:, :, rows]
        err = np.max(np.abs(got - ref)) / np.sqrt(np.mean(ref ** 2))
        assert err <= ATTN_TOL, (bits, s, n, err)
        p0 += n
    assert vq.vq_poll_device_error() == 0


def test_strided_inputs_and_outputs(vq):
    """K/V/Q given as [B][N][H][D] tensors viewed as [B][H][N][D] (row stride H*D),
    output written into a [B][n][H][D] buffer; same bytes as contiguous inputs."""
    B, H, D, sched, bits = 2, 4, 64, [4, 16, 64, 256], 4
    N = sum(sched)
    g = torch.Generator(device="cuda").manual_seed(11)
    kt = (torch.randn((B, N, H, D), generator=g, device="cuda") * 3).to(torch.bfloat16)
    vt = torch.randn((B, N, H, D), generator=g, device="cuda").to(torch.bfloat16)
    qt = torch.randn((B, N, H, D), generator=g, device="cuda").to(torch.bfloat16)
    k, v, q = kt.permute(0, 2, 1, 3), vt.permute(0, 2, 1, 3), qt.permute(0, 2, 1, 3)
    desc = vq.CacheDesc(B, H, D, bits, sched)
    c1, c2 = vq.LayerCache(desc), vq.LayerCache(desc)
    p0 = 0
    for s, n in enumerate(sched):
        vq.vq_cache_append(desc, c1, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n])
        vq.vq_cache_append(desc, c2, s, k[:, :, p0:p0 + n].contiguous(), v[:, :, p0:p0 + n].contiguous())
        p0 += n
    torch.cuda.synchronize()
    assert torch.equal(c1.packed_k, c2.packed_k) and torch.equal(c1.packed_v, c2.packed_v)
    assert torch.equal(c1.scale_v, c2.scale_v) and torch.equal(c1.zero_k, c2.zero_k)
    s = len(sched) - 1
    n = sched[s]
    p0 = N - n
    o_strided = torch.empty((B, n, H, D), dtype=torch.float32, device="cuda")
    o_contig = torch.empty((B, H, n, D), dtype=torch.float32, device="cuda")
    vq.vq_attention_block(desc, c1, s, q[:, :, p0:p0 + n], 0.125, o_strided.permute(0, 2, 1, 3))
    vq.vq_attention_block(desc, c1, s, q[:, :, p0:p0 + n].contiguous(), 0.125, o_contig)
    torch.cuda.synchronize()
    assert torch.equal(o_strided.permute(0, 2, 1, 3), o_contig)


@pytest.mark.gpu
@pytest.mark.parametrize("n", [64, 169])
def test_ring_slot_refills_with_strided_rows(vq, n):
    """Slabs that take the shared-memory ring (8 KB with one-warp teams that copy
    their own units; 21.6 KB with three-warp teams served by the producer warp),
    with enough (batch, head) that every CTA refills its slots many times. Rows
    [B][N][H][D] viewed as [B][H][N][D] are copied row by row; the cache must
    hold the same bytes as from contiguous slabs, and those match the oracle
    on a sample of units."""
    B, H, D, bits = 128, 30, 64, 3
    sched = [n]
    g = torch.Generator(device="cuda").manual_seed(17 + n)
    kt = (torch.randn((B, n, H, D), generator=g, device="cuda") * 2).to(torch.bfloat16)
    vt = torch.randn((B, n, H, D), generator=g, device="cuda").to(torch.bfloat16)
    k, v = kt.permute(0, 2, 1, 3), vt.permute(0, 2, 1, 3)
    desc = vq.CacheDesc(B, H, D, bits, sched)
    c1, c2 = vq.LayerCache(desc), vq.LayerCache(desc)
    vq.vq_cache_append(desc, c1, 0, k, v)
    vq.vq_cache_append(desc, c2, 0, k.contiguous(), v.contiguous())
    torch.cuda.synchronize()
    assert vq.vq_poll_device_error() == 0
    for a, b in ((c1.packed_k, c2.packed_k), (c1.packed_v, c2.packed_v), (c1.scale_k, c2.scale_k),
                 (c1.zero_k, c2.zero_k), (c1.scale_v, c2.scale_v), (c1.zero_v, c2.zero_v)):
        assert torch.equal(a, b)
    # a sample of (b, h) units against the oracle: scale, zero and packed words of K and V
    W = -(-n // (32 // bits))
    pk = c2.packed_k.view(B, H, W, D).cpu().numpy().view(np.uint32)
    pv = c2.packed_v.view(B, H, W, D).cpu().numpy().view(np.uint32)
    sk, zk = c2.scale_k.view(B, H, D).cpu().numpy(), c2.zero_k.view(B, H, D).cpu().numpy()
    sv, zv = c2.scale_v.view(B, H, D).cpu().numpy(), c2.zero_v.view(B, H, D).cpu().numpy()
    rng = np.random.default_rng(n)
    for bb, hh in zip(rng.integers(0, B, 6), rng.integers(0, H, 6)):
        for x, pw, sc, ze in ((k, pk, sk, zk), (v, pv, sv, zv)):
            xs = _host(x[bb:bb + 1, hh:hh + 1])  # [1][1][n][D] float32
            words, s_o, z_o = vo.quantize_pack_block(xs, bits)
            np.testing.assert_array_equal(sc[bb, hh].view(np.uint32), s_o[0, 0].view(np.uint32))
            np.testing.assert_array_equal(ze[bb, hh].view(np.uint32), z_o[0, 0].view(np.uint32))
            np.testing.assert_array_equal(pw[bb, hh], words[0, 0])


def test_degenerate_groups(vq):
    """Constant channels (scale 0), a zero min stored as +0, a single-token block,
    and groups whose range is in the float32 subnormal range (scale below
    2^-128: the 2^64 prescale path), on both quantize kernels."""
    B, H, D = 1, 1, 64
    sched = [1, 20]
    x = torch.randn((B, H, 21, D), device="cuda", dtype=torch.float32)
    x[..., 5] = 3.0                          # constant channel
    x[..., 1:, 6] = x[..., 1:, 6].abs()      # channel with min exactly -0.0
    x[..., 1, 6] = -0.0
    x[..., 1:, 7] = 1e-40 * torch.arange(20, device="cuda", dtype=torch.float32)  # subnormal range
    for bits in (3, 4):
        desc = vq.CacheDesc(B, H, D, bits, sched)
        for s, (p0, n) in enumerate(((0, 1), (1, 20))):
            W = desc.word_rows(s)
            packed = torch.zeros(B * H * W * D, dtype=torch.int32, device="cuda")
            scale = torch.zeros(B * H * D, device="cuda")
            zero = torch.zeros(B * H * D, device="cuda")
            vq.vq_quantize_pack_block(desc, s, x[:, :, p0:p0 + n], packed, scale, zero)
            torch.cuda.synchronize()
            words, s_ref, z_ref = vo.quantize_pack_block(_host(x[:, :, p0:p0 + n]), bits)
            np.testing.assert_array_equal(packed.cpu().numpy().view(np.uint32).reshape(words.shape), words)
            np.testing.assert_array_equal(scale.cpu().numpy().view(np.uint32), s_ref.reshape(-1).view(np.uint32))
            np.testing.assert_array_equal(zero.cpu().numpy().view(np.uint32), z_ref.reshape(-1).view(np.uint32))
            if n == 1:
                assert torch.all(scale == 0) and torch.all(packed == 0)
    # a bf16 block large enough for the shared-memory ring kernel, with a
    # constant channel and channels whose range is subnormal (bf16 keeps the
    # float32 exponent range)
    n = 81
    xb = torch.randn((B, H, n, D), device="cuda", dtype=torch.float32) * 3
    xb[..., 5] = -2.0
    xb[..., 9] = 1e-39 * torch.arange(n, device="cuda", dtype=torch.float32)
    xb[..., 10] = 2.0 ** -128 * torch.randn(n, device="cuda")
    xb = xb.to(torch.bfloat16)
    for bits in (2, 3, 4, 6, 8):
        desc = vq.CacheDesc(B, H, D, bits, [n])
        W = desc.word_rows(0)
        packed = torch.zeros(B * H * W * D, dtype=torch.int32, device="cuda")
        scale = torch.zeros(B * H * D, device="cuda")
        zero = torch.zeros(B * H * D, device="cuda")
        vq.vq_quantize_pack_block(desc, 0, xb, packed, scale, zero)
        torch.cuda.synchronize()
        words, s_ref, z_ref = vo.quantize_pack_block(_host(xb), bits)
        np.testing.assert_array_equal(packed.cpu().numpy().view(np.uint32).reshape(words.shape), words)
        np.testing.assert_array_equal(scale.cpu().numpy().view(np.uint32), s_ref.reshape(-1).view(np.uint32))
        np.testing.assert_array_equal(zero.cpu().numpy().view(np.uint32), z_ref.reshape(-1).view(np.uint32))
    assert vq.vq_poll_device_error() == 0


def test_reappend_overwrites(vq):
    w = WORKLOADS["var_d16"]
    k, v = make_kv(w, 3, device="cuda")
    bits = 3
    desc, c1 = _append_all(vq, w, bits, k, v)
    snapshot = c1.packed_k.clone(), c1.scale_v.clone()
    s = 7
    p0, n = w.prefix(s), w.block_tokens[s]
    vq.vq_cache_append(desc, c1, s, v[:, :, p0:p0 + n], k[:, :, p0:p0 + n])   # different data
    vq.vq_cache_append(desc, c1, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n])   # original again
    torch.cuda.synchronize()
    assert torch.equal(c1.packed_k, snapshot[0]) and torch.equal(c1.scale_v, snapshot[1])


def test_bf16_output(vq):
    w = WORKLOADS["tiny"]
    k, v = make_kv(w, 0, device="cuda")
    q = make_q(w, 0, device="cuda")
    desc, cache = _append_all(vq, w, 4, k, v)
    s = w.num_blocks - 1
    p0, n = w.prefix(s), w.block_tokens[s]
    o32 = torch.empty((1, 1, n, 64), dtype=torch.float32, device="cuda")
    o16 = torch.empty((1, 1, n, 64), dtype=torch.bfloat16, device="cuda")
    vq.vq_attention_block(desc, cache, s, q[:, :, p0:p0 + n], 0.125, o32)
    vq.vq_attention_block(desc, cache, s, q[:, :, p0:p0 + n], 0.125, o16)
    torch.cuda.synchronize()
    assert torch.equal(o32.to(torch.bfloat16), o16)


@pytest.mark.parametrize("D", [64, 128])
def test_bf16_output_every_kernel(vq, D):
    """bf16 output = the float32 output rounded to nearest even, for every
    attention kernel's epilogue: a block of 3 queries (warp per query), 40
    (CUDA-core kernel), 100 (tensor cores, one query tile per item) and 200
    (tensor cores, two query tiles per item)."""
    sched = [3, 40, 100, 200]
    B, H = 1, 2
    k, v, q = _ragged_kv(sched, D, H=H, B=B, seed=13)
    for bits in (3, 4):
        desc = vq.CacheDesc(B, H, D, bits, sched)
        cache = vq.LayerCache(desc)
        p0 = 0
        for s, n in enumerate(sched):
            vq.vq_cache_append(desc, cache, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n])
            o32 = torch.empty((B, H, n, D), dtype=torch.float32, device="cuda")
            o16 = torch.empty((B, H, n, D), dtype=torch.bfloat16, device="cuda")
            vq.vq_attention_block(desc, cache, s, q[:, :, p0:p0 + n], 0.125, o32)
            vq.vq_attention_block(desc, cache, s, q[:, :, p0:p0 + n], 0.125, o16)
            torch.cuda.synchronize()
            assert torch.equal(o32.to(torch.bfloat16), o16), (bits, s, n)
            p0 += n
    assert vq.vq_poll_device_error() == 0


# ---------------------------------------------------------------- fused append + attention
def _fused_decode(vq, desc, cache, sched, k, v, q, sigma, B, H, D, out_dtype=torch.float32):
    outs = []
    p0 = 0
    for s, n in enumerate(sched):
        out = torch.full((B, H, n, D), float("nan"), dtype=out_dtype, device="cuda")
        vq.vq_append_attention_block(desc, cache, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n], q[:, :, p0:p0 + n],
                                     sigma, out)
        outs.append(out)
        p0 += n
    torch.cuda.synchronize()
    assert vq.vq_poll_device_error() == 0
    return outs


@pytest.mark.parametrize("D", [64, 128])
def test_fused_append_attention(vq, D):
    """vq_append_attention_block block by block: the cache is bit-exact with the
    oracle's append and every block's attention within the bar of the oracle's
    attention over it. Blocks of 3 and 20 queries run fused (warp per query and
    CUDA-core kernels, 4 (batch, head)); 100, 200 and 300 run append, then attend."""
    sched = [3, 20, 100, 200, 300]
    B, H = 2, 2
    k, v, q = _ragged_kv(sched, D, H=H, B=B, seed=17)
    sigma = float(1.0 / np.sqrt(D))
    for bits in (3, 4, 6):
        desc = vq.CacheDesc(B, H, D, bits, sched)
        cache = vq.LayerCache(desc)
        outs = _fused_decode(vq, desc, cache, sched, k, v, q, sigma, B, H, D)
        pk, sk, zk = vo.cache_append(_host(k), sched, bits)
        pv, sv, zv = vo.cache_append(_host(v), sched, bits)
        np.testing.assert_array_equal(cache.packed_k.cpu().numpy().view(np.uint32), pk)
        np.testing.assert_array_equal(cache.packed_v.cpu().numpy().view(np.uint32), pv)
        np.testing.assert_array_equal(cache.scale_k.cpu().numpy().view(np.uint32), sk.view(np.uint32))
        np.testing.assert_array_equal(cache.zero_v.cpu().numpy().view(np.uint32), zv.view(np.uint32))
        p0 = 0
        for s, n in enumerate(sched):
            khat = vo.dequantize_cache(pk, sk, zk, sched, B, H, D, bits, s)
            vhat = vo.dequantize_cache(pv, sv, zv, sched, B, H, D, bits, s)
            ref = vo.attention_f64(_host(q[:, :, p0:p0 + n]), khat, vhat, sigma)
            err = np.max(np.abs(outs[s].cpu().numpy() - ref)) / np.sqrt(np.mean(ref ** 2))
            assert err <= ATTN_TOL, (bits, s, n, err)
            p0 += n


def test_fused_matches_two_calls_strided(vq):
    """Permuted (strided) K/V/Q and output: the fused call leaves the same cache
    bytes and the same output as vq_cache_append followed by vq_attention_block."""
    B, H, D, sched, bits = 2, 4, 64, [4, 16, 64, 256], 3
    N = sum(sched)
    g = torch.Generator(device="cuda").manual_seed(23)
    kt = (torch.randn((B, N, H, D), generator=g, device="cuda") * 3).to(torch.bfloat16)
    vt = torch.randn((B, N, H, D), generator=g, device="cuda").to(torch.bfloat16)
    qt = torch.randn((B, N, H, D), generator=g, device="cuda").to(torch.bfloat16)
    k, v, q = kt.permute(0, 2, 1, 3), vt.permute(0, 2, 1, 3), qt.permute(0, 2, 1, 3)
    desc = vq.CacheDesc(B, H, D, bits, sched)
    c1, c2 = vq.LayerCache(desc), vq.LayerCache(desc)
    for c in (c1, c2):   # blocks not appended yet compare equal too
        for t in (c.packed_k, c.packed_v, c.scale_k, c.zero_k, c.scale_v, c.zero_v):
            t.zero_()
    p0 = 0
    for s, n in enumerate(sched):
        o1 = torch.empty((B, n, H, D), dtype=torch.float32, device="cuda").permute(0, 2, 1, 3)
        o2 = torch.empty((B, H, n, D), dtype=torch.float32, device="cuda")
        vq.vq_append_attention_block(desc, c1, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n], q[:, :, p0:p0 + n],
                                     0.125, o1)
        vq.vq_cache_append(desc, c2, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n])
        vq.vq_attention_block(desc, c2, s, q[:, :, p0:p0 + n], 0.125, o2)
        torch.cuda.synchronize()
        assert torch.equal(c1.packed_k, c2.packed_k) and torch.equal(c1.packed_v, c2.packed_v), s
        assert torch.equal(c1.scale_k, c2.scale_k) and torch.equal(c1.zero_v, c2.zero_v), s
        assert torch.equal(o1, o2), s
        p0 += n
    assert vq.vq_poll_device_error() == 0


# ---------------------------------------------------------------- fp16 metadata, storage format
@pytest.mark.parametrize("D", [64, 128])
def test_fp16_metadata_and_paper_format(vq, D):
    """Caches quantized with fp16 metadata: codes and the fp16-valued scale and
    zero bit-exact with the oracle (streaming, ring and fused quantize paths),
    attention within the bar over that cache, the storage format written by
    vq_paper_pack equal to the oracle's, and vq_paper_unpack restoring the
    word-row cache exactly."""
    sched = [1, 9, 81, 300]
    B, H = 2, 2
    k, v, q = _ragged_kv(sched, D, H=H, B=B, seed=29)
    sigma = float(1.0 / np.sqrt(D))
    for bits in (3, 4):
        desc = vq.CacheDesc(B, H, D, bits, sched, meta_fp16=True)
        cache = vq.LayerCache(desc)
        fused = vq.LayerCache(desc)
        p0 = 0
        for s, n in enumerate(sched):
            vq.vq_cache_append(desc, cache, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n])
            out = torch.empty((B, H, n, D), dtype=torch.float32, device="cuda")
            vq.vq_append_attention_block(desc, fused, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n],
                                         q[:, :, p0:p0 + n], sigma, out)
            p0 += n
        torch.cuda.synchronize()
        pk, sk, zk = vo.cache_append(_host(k), sched, bits, meta_fp16=True)
        pv, sv, zv = vo.cache_append(_host(v), sched, bits, meta_fp16=True)
        for c in (cache, fused):
            np.testing.assert_array_equal(c.packed_k.cpu().numpy().view(np.uint32), pk)
            np.testing.assert_array_equal(c.packed_v.cpu().numpy().view(np.uint32), pv)
            np.testing.assert_array_equal(c.scale_k.cpu().numpy().view(np.uint32), sk.view(np.uint32))
            np.testing.assert_array_equal(c.zero_v.cpu().numpy().view(np.uint32), zv.view(np.uint32))
        p0 = 0
        for s, n in enumerate(sched):
            out = torch.empty((B, H, n, D), dtype=torch.float32, device="cuda")
            vq.vq_attention_block(desc, cache, s, q[:, :, p0:p0 + n], sigma, out)
            torch.cuda.synchronize()
            khat = vo.dequantize_cache(pk, sk, zk, sched, B, H, D, bits, s)
            vhat = vo.dequantize_cache(pv, sv, zv, sched, B, H, D, bits, s)
            ref = vo.attention_f64(_host(q[:, :, p0:p0 + n]), khat, vhat, sigma)
            err = np.max(np.abs(out.cpu().numpy() - ref)) / np.sqrt(np.mean(ref ** 2))
            assert err <= ATTN_TOL, (bits, s, err)
            p0 += n
        words, meta, _ = vq.vq_paper_layout(desc)
        kw = torch.zeros(words, dtype=torch.int32, device="cuda")
        vw = torch.zeros(words, dtype=torch.int32, device="cuda")
        km = torch.zeros(meta, dtype=torch.int32, device="cuda")
        vm = torch.zeros(meta, dtype=torch.int32, device="cuda")
        vq.vq_paper_pack(desc, cache, kw, vw, km, vm)
        torch.cuda.synchronize()
        ref_kw, ref_km = vo.paper_from_cache(pk, sk, zk, sched, B, H, D, bits)
        ref_vw, ref_vm = vo.paper_from_cache(pv, sv, zv, sched, B, H, D, bits)
        np.testing.assert_array_equal(kw.cpu().numpy().view(np.uint32), ref_kw)
        np.testing.assert_array_equal(vw.cpu().numpy().view(np.uint32), ref_vw)
        np.testing.assert_array_equal(km.cpu().numpy().view(np.uint32), ref_km)
        np.testing.assert_array_equal(vm.cpu().numpy().view(np.uint32), ref_vm)
        back = vq.LayerCache(desc)
        vq.vq_paper_unpack(desc, kw, vw, km, vm, back)
        torch.cuda.synchronize()
        for a, b in ((back.packed_k, cache.packed_k), (back.packed_v, cache.packed_v), (back.scale_k, cache.scale_k),
                     (back.zero_k, cache.zero_k), (back.scale_v, cache.scale_v), (back.zero_v, cache.zero_v)):
            assert torch.equal(a, b)
    assert vq.vq_poll_device_error() == 0


# ---------------------------------------------------------------- failure path
def test_bounded_wait_timeout_sets_flag_and_context_survives(vq):
    """A wait that nothing completes gives up after its iteration limit: the
    kernel records flag 1 in the device error word and returns, the poll reads
    and clears it, and the context keeps working (a small append + attention
    afterwards is still bit-exact / within the bar)."""
    assert vq.vq_poll_device_error() == 0
    vq.vq_check_wait_timeout(2000)
    torch.cuda.synchronize()
    assert vq.vq_poll_device_error() == 1
    assert vq.vq_poll_device_error() == 0
    sched = [1, 9, 40]
    k, v, q = _ragged_kv(sched, 64, seed=3)
    desc = vq.CacheDesc(1, 3, 64, 4, sched)
    cache = vq.LayerCache(desc)
    p0 = 0
    for s, n in enumerate(sched):
        vq.vq_cache_append(desc, cache, s, k[:, :, p0:p0 + n], v[:, :, p0:p0 + n])
        p0 += n
    _check_ragged_attention(vq, desc, cache, sched, q, k, v, 4, 64)
