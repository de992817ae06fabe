"""CPU oracle for the VAR-Q-style packed low-bit KV cache.

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU
baseline leg may import this module. The library's product path never routes
through it and shares no code with it.

Source of the method: "VAR-Q: Tuning-Free KV Cache Quantization for Visual
Autoregressive Image and Video Generation", Abstract (paragraphs 1-3) and "Key
Contributions at a Glance". The abstract says visual AR models decode block by
block (paragraph 1) and that VAR-Q groups the KV cache "along the same two axes",
feature (channel) and block (paragraph 3). Block boundaries come from the
generation loop, with no calibration, and bit-packing kernels give the memory
reduction. Nothing else is specified there. The readings below (asymmetric
min/max, round-half-even, codes packed along tokens) are the plainest ones
consistent with "VAR-Q results data (Tables 2-4)". Its KV-memory column fits
exactly one 32-bit (scale, zero) pair per (block, channel) group and 10 INT3
codes per 32-bit word; `paper_kv_gib` checks that.

Every floating-point step is an IEEE binary32 operation done by numpy on float32
arrays, each as a separate statement, so no fused multiply-add can appear. The
exceptions are `dequantize`, which is defined as one fused multiply-add and
emulated exactly, and `attention_f64`, which is float64. Function by function:

  group_min_max     exact min/max over the block's tokens, per (b, h, channel)
  scale_zero        scale = (max - min) / (2^b - 1); zero = min (+0 for a zero min)
  encode            code = clamp(rint((x - min) * (1/scale)), 0, 2^b - 1); 0 if scale == 0;
                    float32 steps with an unbounded exponent (see `prescale`)
  pack / unpack     codes along tokens, floor(32/b) per 32-bit word, least significant first
  dequantize        x_hat = fma(code, scale, zero), one rounding
  attention_f64     softmax(sigma * q . k_hat) . v_hat over blocks 0..s, float64
  paper_kv_gib      KV-memory accounting of the results tables (closed form)
  scale_zero_fp16   scale and zero rounded to fp16: one 32-bit pair per group
  paper_*           the storage format those tables count: per block one
                    padding-free stream of codes over (b, h, token, channel),
                    floor(32/b) per word, and the 32-bit metadata pairs

Parity status: every function here is pinned by tests that do not re-type its
formula (brute force on tiny inputs, closed forms, special cases, the printed
numbers of the results tables). There is no "parity unpinned" function.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32
F64 = np.float64


# ---------------------------------------------------------------- layout
def codes_per_word(bits: int) -> int:
    """Codes held by one 32-bit word: 8 (INT4), 10 (INT3; bits 30-31 unused), 16 (INT2),
    5 (INT6; bits 30-31 unused), 4 (INT8)."""
    if bits not in (2, 3, 4, 6, 8):
        raise ValueError(f"unsupported bit width {bits}")
    return 32 // bits


def word_rows(n_tokens: int, bits: int) -> int:
    """Word-rows W_s = ceil(n_s / codes_per_word) of one block."""
    c = codes_per_word(bits)
    return (n_tokens + c - 1) // c


def cache_layout(block_tokens, batch: int, heads: int, head_dim: int, bits: int):
    """Offsets of the block-addressed cache of one layer and one tensor.

    Packed words of block s live at word offset B*H*D*sum_{k<s} W_k as
    [B][H][W_s][D]; scale and zero of block s live at s*B*H*D as [B][H][D].
    Returns (words_per_tensor, meta_per_tensor, block_word_offset[S+1]).
    """
    offs = [0]
    for n in block_tokens:
        offs.append(offs[-1] + batch * heads * head_dim * word_rows(n, bits))
    return offs[-1], len(block_tokens) * batch * heads * head_dim, offs


# ---------------------------------------------------------------- quantizer
def group_min_max(x: np.ndarray):
    """Min and max over the token axis of one block, per (b, h, channel).

    x: float32 [B][H][n_s][D] (bf16 inputs are widened exactly before this).
    The group is the (block, channel) cell of the abstract, paragraph 3.
    """
    x = np.asarray(x, dtype=F32)
    return x.min(axis=2), x.max(axis=2)


def scale_zero(mn: np.ndarray, mx: np.ndarray, bits: int):
    """Asymmetric uniform grid of 2^b levels spanning [min, max].

    scale = (max - min) / (2^b - 1) as one IEEE float32 subtraction and one
    IEEE float32 division; zero = min, with a zero min stored as +0.
    """
    levels = F32((1 << bits) - 1)
    diff = (mx.astype(F32) - mn.astype(F32)).astype(F32)
    scale = (diff / levels).astype(F32)
    zero = (mn.astype(F32) + F32(0.0)).astype(F32)
    return scale, zero


TINY_SCALE = F32(2.0 ** -100)
PRESCALE = F32(2.0 ** 64)


def prescale(scale: np.ndarray) -> np.ndarray:
    """Power of two applied to both d = x - min and scale before the reciprocal.

    2^64 where 0 < scale < 2^-100, else 1. Without it, 1/scale overflows float32
    for scales below 2^-128 (groups whose range lies in the subnormal range) and
    the codes stop being the nearest grid levels. Multiplying d and scale by the
    same power of two is exact here (the products stay normal and below 2^-28),
    so inv and t come out as float32 arithmetic with an unbounded exponent would
    give them: the asymmetric min/max grid of the abstract (paragraph 3) holds
    for every finite group, and every normal-range group is unaffected.
    """
    return np.where((scale > 0) & (scale < TINY_SCALE), PRESCALE, F32(1.0)).astype(F32)


def reciprocal(scale: np.ndarray) -> np.ndarray:
    """inv = 1/(scale * prescale(scale)), IEEE float32; 0 where scale == 0 (unused there).

    With |x| < 2^126 and at least 3 levels, scale < 2^126 and the scaled scale
    is at least 2^-85, so inv is a normal float32 that never overflows.
    """
    s2 = (scale * prescale(scale)).astype(F32)
    with np.errstate(divide="ignore", over="ignore"):
        inv = (F32(1.0) / s2).astype(F32)
    return np.where(scale > 0, inv, F32(0)).astype(F32)


def encode(x: np.ndarray, mn: np.ndarray, scale: np.ndarray, bits: int) -> np.ndarray:
    """Integer codes of one block: clamp(rint((x - min) * inv), 0, 2^b - 1).

    IEEE float32 steps, in this order: d = x - min, d = d * pre (pre =
    prescale(scale), exact), t = d * inv, then round half to even. A group
    whose scale is 0 (constant group, or a single token) encodes to 0
    everywhere.
    """
    x = np.asarray(x, dtype=F32)
    mn4 = mn[:, :, None, :]
    inv4 = reciprocal(scale)[:, :, None, :]
    pre4 = prescale(scale)[:, :, None, :]
    d = (x - mn4).astype(F32)
    d = (d * pre4).astype(F32)
    t = (d * inv4).astype(F32)
    r = np.rint(t)
    code = np.clip(r, 0, (1 << bits) - 1).astype(np.uint8)
    code = np.where(scale[:, :, None, :] > 0, code, np.uint8(0)).astype(np.uint8)
    return code


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack codes [B][H][n][D] into words [B][H][W][D] (uint32).

    Word (w, c) holds the codes of tokens w*cpw .. w*cpw+cpw-1 of channel c, token
    w*cpw+i in bits [b*i, b*i+b). Slots past the last token and bits past b*cpw
    are zero.
    """
    B, H, n, D = codes.shape
    cpw = codes_per_word(bits)
    W = word_rows(n, bits)
    words = np.zeros((B, H, W, D), dtype=np.uint32)
    for t in range(n):
        w, i = divmod(t, cpw)
        words[:, :, w, :] |= codes[:, :, t, :].astype(np.uint32) << np.uint32(bits * i)
    return words


def unpack(words: np.ndarray, bits: int, n_tokens: int) -> np.ndarray:
    """Inverse of `pack`: words [B][H][W][D] -> codes [B][H][n][D] (uint8)."""
    B, H, W, D = words.shape
    cpw = codes_per_word(bits)
    mask = np.uint32((1 << bits) - 1)
    codes = np.zeros((B, H, n_tokens, D), dtype=np.uint8)
    for t in range(n_tokens):
        w, i = divmod(t, cpw)
        codes[:, :, t, :] = ((words[:, :, w, :] >> np.uint32(bits * i)) & mask).astype(np.uint8)
    return codes


def to_fp16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest fp16 (ties to even), widened back exactly."""
    return np.asarray(x, dtype=F32).astype(np.float16).astype(F32)


def scale_zero_fp16(mn: np.ndarray, mx: np.ndarray, bits: int):
    """Metadata of one 32-bit (scale, zero) pair per group, the size the results
    tables count: the float32 scale and zero of `scale_zero`, each rounded to
    the nearest fp16. Codes are then taken against this stored grid (inputs
    must stay inside the fp16 range, |x| < 65504)."""
    scale, zero = scale_zero(mn, mx, bits)
    return to_fp16(scale), to_fp16(zero)


def quantize_pack_block(x: np.ndarray, bits: int, meta_fp16: bool = False):
    """One block of one tensor: float32 [B][H][n][D] -> (words, scale, zero).

    meta_fp16: scale and zero are the fp16-rounded pair and the codes the
    nearest levels of that grid, clamped to [0, 2^b - 1] (zero can sit above
    the min and zero + (2^b - 1) * scale below the max)."""
    x = np.asarray(x, dtype=F32)
    mn, mx = group_min_max(x)
    if meta_fp16:
        scale, zero = scale_zero_fp16(mn, mx, bits)
        codes = encode(x, zero, scale, bits)
    else:
        scale, zero = scale_zero(mn, mx, bits)
        codes = encode(x, mn, scale, bits)
    return pack(codes, bits), scale, zero


def cache_append(x_layer: np.ndarray, block_tokens, bits: int, meta_fp16: bool = False):
    """Quantize every block of one layer's tensor [B][H][N][D] into a full cache.

    Returns (packed words [words_per_tensor] uint32, scale [S*B*H*D], zero [S*B*H*D])
    in the block-addressed layout of `cache_layout`.
    """
    x_layer = np.asarray(x_layer, dtype=F32)
    B, H, N, D = x_layer.shape
    total, meta, offs = cache_layout(block_tokens, B, H, D, bits)
    packed = np.zeros(total, dtype=np.uint32)
    scale = np.zeros(meta, dtype=F32)
    zero = np.zeros(meta, dtype=F32)
    t0 = 0
    for s, n in enumerate(block_tokens):
        w, sc, z = quantize_pack_block(x_layer[:, :, t0:t0 + n, :], bits, meta_fp16)
        packed[offs[s]:offs[s + 1]] = w.reshape(-1)
        scale[s * B * H * D:(s + 1) * B * H * D] = sc.reshape(-1)
        zero[s * B * H * D:(s + 1) * B * H * D] = z.reshape(-1)
        t0 += n
    return packed, scale, zero


# ---------------------------------------------------------------- dequantize
def fma_f32(a: np.ndarray, b: np.ndarray, c: np.ndarray) -> np.ndarray:
    """Correctly rounded float32 a*b + c (one rounding), for float32 inputs.

    a*b is exact in float64 (24 + 24 significant bits). The float64 sum is then
    made round-to-odd: when the sum is inexact and its last bit is even, it is
    moved one ulp toward the exact value. Rounding a round-to-odd float64 value
    to float32 is then the correct single rounding, because 53 >= 2*24 + 2
    (Boldo and Melquiond, "Emulation of FMA and correctly rounded sums: proved
    algorithms using rounding to odd", IEEE Trans. Computers 57(4), 2008).
    """
    a64 = np.asarray(a, dtype=F32).astype(F64)
    b64 = np.asarray(b, dtype=F32).astype(F64)
    c64 = np.asarray(c, dtype=F32).astype(F64)
    p = a64 * b64
    s = p + c64
    # exact error of the addition (Knuth's TwoSum)
    bv = s - p
    av = s - bv
    err = (p - av) + (c64 - bv)
    bits = s.view(np.uint64)
    inexact_even = (err != 0) & ((bits & np.uint64(1)) == 0)
    toward = np.where(err > 0, np.inf, -np.inf)
    s = np.where(inexact_even, np.nextafter(s, toward), s)
    return s.astype(F32)


def dequantize(words: np.ndarray, scale: np.ndarray, zero: np.ndarray, bits: int, n_tokens: int) -> np.ndarray:
    """x_hat = fma(code, scale, zero) in float32 for one block -> [B][H][n][D]."""
    codes = unpack(words, bits, n_tokens).astype(F32)
    return fma_f32(codes, scale[:, :, None, :], zero[:, :, None, :])


def dequantize_cache(packed, scale, zero, block_tokens, B, H, D, bits, upto_block: int) -> np.ndarray:
    """Dequantized cache of blocks 0..upto_block of one tensor -> [B][H][P_s][D] float32."""
    _, _, offs = cache_layout(block_tokens, B, H, D, bits)
    parts = []
    for s in range(upto_block + 1):
        n = block_tokens[s]
        W = word_rows(n, bits)
        w = np.asarray(packed[offs[s]:offs[s + 1]]).reshape(B, H, W, D)
        sc = np.asarray(scale[s * B * H * D:(s + 1) * B * H * D], dtype=F32).reshape(B, H, D)
        z = np.asarray(zero[s * B * H * D:(s + 1) * B * H * D], dtype=F32).reshape(B, H, D)
        parts.append(dequantize(w, sc, z, bits, n))
    return np.concatenate(parts, axis=2)


# ---------------------------------------------------------------- attention
def attention_f64(q: np.ndarray, k_hat: np.ndarray, v_hat: np.ndarray, softmax_scale) -> np.ndarray:
    """Block-causal attention of one block's queries over the dequantized cache.

    q: [B][H][n_s][D] (bf16 values widened), k_hat, v_hat: [B][H][P_s][D] float32,
    the dequantized keys and values of blocks 0..s (the current block included in
    full). Returns float64 [B][H][n_s][D] = softmax(sigma * q k_hat^T) v_hat with
    exp in float64 and the row maximum subtracted first.
    """
    q64 = np.asarray(q, dtype=F32).astype(F64)
    k64 = np.asarray(k_hat, dtype=F32).astype(F64)
    v64 = np.asarray(v_hat, dtype=F32).astype(F64)
    sigma = F64(F32(softmax_scale))
    logits = sigma * np.matmul(q64, np.swapaxes(k64, -1, -2))      # [B][H][n_s][P_s]
    logits = logits - logits.max(axis=-1, keepdims=True)
    p = np.exp(logits)
    p = p / p.sum(axis=-1, keepdims=True)
    return np.matmul(p, v64)


# ---------------------------------------------------------------- accounting
def payload_bits(bits: int) -> float:
    """Stored bits per code in the results tables' accounting: b, except INT3 at
    10 codes per 32-bit word (3.2). (INT6 rows appear only for the video models
    of Table 4, whose token schedules the pages do not give, so no printed
    number fixes its accounting; 5 codes per word would be 6.4.)"""
    return 32.0 / codes_per_word(bits) if bits == 3 else float(bits)


def paper_kv_gib(layers: int, hidden: int, tokens: int, blocks: int, batch_eff: int, bits):
    """KV memory of the results tables (GiB) and the saving (%) versus BF16.

    BF16: layers * 2 (K, V) * tokens * hidden * 2 bytes * batch_eff. Quantized: the
    same element count at payload(b) + 32 * blocks / tokens bits per element,
    i.e. one 32-bit (scale, zero) pair per (block, channel) group. bits=None
    means BF16 (saving None).
    """
    elems = layers * 2 * tokens * hidden * batch_eff
    if bits is None:
        return elems * 2 / 2**30, None
    bpe = payload_bits(bits) + 32.0 * blocks / tokens
    return elems * bpe / 8 / 2**30, 100.0 * (1.0 - bpe / 16.0)


# ---------------------------------------------------------------- paper-exact storage
def paper_layout(block_tokens, batch: int, heads: int, head_dim: int, bits: int):
    """Storage the results tables count, for one layer and one tensor.

    Block s is one stream of its B*H*n_s*D codes in (b, h, token, channel)
    order, code i in word i // cpw at bits [b*(i % cpw), b*(i % cpw) + b): no
    per-(block, channel) padding, only the last word of the block may hold
    unused slots. Metadata: one 32-bit word per (block, b, h, channel), fp16
    scale in the low half, fp16 zero in the high half.
    Returns (words_per_tensor, meta_words_per_tensor, block_word_offset[S+1]).
    """
    cpw = codes_per_word(bits)
    offs = [0]
    for n in block_tokens:
        offs.append(offs[-1] + -(-(batch * heads * n * head_dim) // cpw))
    return offs[-1], len(block_tokens) * batch * heads * head_dim, offs


def paper_pack_block(codes: np.ndarray, bits: int) -> np.ndarray:
    """Codes [B][H][n][D] of one block -> its padding-free word stream (uint32)."""
    cpw = codes_per_word(bits)
    flat = np.asarray(codes, dtype=np.uint32).reshape(-1)
    nw = -(-flat.size // cpw)
    padded = np.zeros(nw * cpw, dtype=np.uint32)
    padded[:flat.size] = flat
    slots = padded.reshape(nw, cpw)
    words = np.zeros(nw, dtype=np.uint32)
    for i in range(cpw):
        words |= slots[:, i] << np.uint32(bits * i)
    return words


def paper_unpack_block(words: np.ndarray, bits: int, B: int, H: int, n: int, D: int) -> np.ndarray:
    """Inverse of `paper_pack_block`: the block's stream -> codes [B][H][n][D] (uint8)."""
    cpw = codes_per_word(bits)
    mask = np.uint32((1 << bits) - 1)
    w = np.asarray(words, dtype=np.uint32)
    slots = np.stack([(w >> np.uint32(bits * i)) & mask for i in range(cpw)], axis=1).reshape(-1)
    return slots[:B * H * n * D].reshape(B, H, n, D).astype(np.uint8)


def paper_meta(scale: np.ndarray, zero: np.ndarray) -> np.ndarray:
    """fp16 scale in the low 16 bits, fp16 zero in the high 16 bits, per group."""
    s16 = np.asarray(scale, dtype=F32).astype(np.float16).view(np.uint16).astype(np.uint32)
    z16 = np.asarray(zero, dtype=F32).astype(np.float16).view(np.uint16).astype(np.uint32)
    return s16 | (z16 << np.uint32(16))


def paper_from_cache(packed, scale, zero, block_tokens, B, H, D, bits):
    """A layer-tensor cache in the word-row layout -> (paper stream, metadata words)."""
    _, _, offs = cache_layout(block_tokens, B, H, D, bits)
    streams = []
    for s, n in enumerate(block_tokens):
        W = word_rows(n, bits)
        codes = unpack(np.asarray(packed[offs[s]:offs[s + 1]]).reshape(B, H, W, D), bits, n)
        streams.append(paper_pack_block(codes, bits))
    return np.concatenate(streams), paper_meta(scale, zero)
