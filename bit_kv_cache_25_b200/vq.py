"""Thin Python binding of libvq (ctypes): argument marshalling only.

Every computation runs in the CUDA kernels of libvq.so. This module turns torch
tensors into device pointers and strides, calls the C entry point of the same
name and raises VqError on a non-zero status. PyTorch is used only for device
memory and streams. If libvq.so is missing, importing this module raises: there
is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvq.so")

VQ_OK, VQ_ERR_INVALID_ARGUMENT, VQ_ERR_UNSUPPORTED, VQ_ERR_MISALIGNED, VQ_ERR_CUDA = range(5)
VQ_BF16, VQ_F32 = 0, 1


class VqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libvq status {status}: {message}")
        self.status = status


class vq_cache_desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("bits", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("block_tokens", ctypes.POINTER(ctypes.c_int32)), ("meta_fp16", ctypes.c_int32)]


class vq_layer_cache(ctypes.Structure):
    _fields_ = [("packed_k", ctypes.c_void_p), ("packed_v", ctypes.c_void_p),
                ("scale_k", ctypes.c_void_p), ("zero_k", ctypes.c_void_p),
                ("scale_v", ctypes.c_void_p), ("zero_v", ctypes.c_void_p)]


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is not built; run bit_kv_cache_25_b200.build.build() first")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I32, I64P, VP, F = ctypes.POINTER, ctypes.c_int32, ctypes.POINTER(ctypes.c_int64), ctypes.c_void_p, ctypes.c_float
    SZ = ctypes.c_size_t
    sig = {
        "vq_cache_layout": [P(vq_cache_desc), P(SZ), P(SZ), P(SZ)],
        "vq_quantize_pack_block": [P(vq_cache_desc), I32, VP, I32, I64P, VP, VP, VP, VP],
        "vq_cache_append": [P(vq_cache_desc), P(vq_layer_cache), I32, VP, VP, I32, I64P, I64P, VP],
        "vq_attention_block": [P(vq_cache_desc), P(vq_layer_cache), I32, VP, I64P, F, VP, I32, I64P, VP],
        "vq_append_attention_block": [P(vq_cache_desc), P(vq_layer_cache), I32, VP, VP, I32, I64P, I64P, VP, I64P, F,
                                      VP, I32, I64P, VP],
        "vq_dequantize": [P(vq_cache_desc), I32, VP, VP, VP, VP, VP],
        "vq_paper_layout": [P(vq_cache_desc), P(SZ), P(SZ), P(SZ)],
        "vq_paper_pack": [P(vq_cache_desc), P(vq_layer_cache), VP, VP, VP, VP, VP],
        "vq_paper_unpack": [P(vq_cache_desc), VP, VP, VP, VP, P(vq_layer_cache), VP],
        "vq_poll_device_error": [P(ctypes.c_uint32)],
        "vq_check_wait_timeout": [ctypes.c_uint32, VP],
        "vq_status_string": [I32],
        "vq_last_error": [],
        "vq_version": [],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name in ("vq_status_string", "vq_last_error") else ctypes.c_int32
    return lib


_lib = _load()

EXPORTED = ("vq_cache_layout", "vq_quantize_pack_block", "vq_cache_append", "vq_attention_block",
            "vq_append_attention_block", "vq_dequantize", "vq_paper_layout", "vq_paper_pack", "vq_paper_unpack",
            "vq_poll_device_error", "vq_check_wait_timeout", "vq_status_string", "vq_last_error", "vq_version")


def _check(status: int):
    if status != VQ_OK:
        raise VqError(status, _lib.vq_last_error().decode() or _lib.vq_status_string(status).decode())


class CacheDesc:
    """Host-side vq_cache_desc plus the int32 block schedule it points to."""

    def __init__(self, batch: int, heads: int, head_dim: int, bits: int, block_tokens: Sequence[int],
                 meta_fp16: bool = False):
        self.block_tokens = list(int(n) for n in block_tokens)
        self._arr = (ctypes.c_int32 * max(1, len(self.block_tokens)))(*self.block_tokens)
        self.c = vq_cache_desc(batch, heads, head_dim, bits, len(self.block_tokens), self._arr, int(bool(meta_fp16)))

    @property
    def batch(self): return self.c.batch

    @property
    def heads(self): return self.c.heads

    @property
    def head_dim(self): return self.c.head_dim

    @property
    def bits(self): return self.c.bits

    @property
    def num_blocks(self): return self.c.num_blocks

    @property
    def meta_fp16(self): return bool(self.c.meta_fp16)

    def word_rows(self, s: int) -> int:
        cpw = 32 // self.bits
        return (self.block_tokens[s] + cpw - 1) // cpw


def _strides(t: torch.Tensor, ndim_expected: int = 4):
    if t.dim() != ndim_expected:
        raise ValueError(f"expected a {ndim_expected}-d [B][H][T][D] tensor, got {tuple(t.shape)}")
    if t.stride(-1) != 1:
        raise ValueError("the channel dimension must be contiguous")
    return (ctypes.c_int64 * 3)(t.stride(0), t.stride(1), t.stride(2))


def _block_tokens(desc: "CacheDesc", block: int) -> int:
    if not 0 <= int(block) < desc.num_blocks:
        raise ValueError(f"block {block} out of range [0, {desc.num_blocks})")
    return desc.block_tokens[int(block)]


def _check_slab(name: str, t: torch.Tensor, desc: "CacheDesc", n: int):
    """t must be a [B][H][n][D] view of the block (any strides, channels contiguous)."""
    want = (desc.batch, desc.heads, n, desc.head_dim)
    if tuple(t.shape) != want:
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {want} ([B][H][n_s][D] of this block)")


def _check_flat(name: str, t: torch.Tensor, numel: int, dtypes):
    """t is written or read as a flat array of at least numel elements from data_ptr()."""
    if t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements, needs at least {numel}")


def _check_devices(*named):
    """Every tensor on the same CUDA device (a host pointer would become an
    out-of-bounds device access)."""
    dev = None
    for name, t in named:
        if not t.is_cuda:
            raise ValueError(f"{name} is on {t.device}, not a CUDA device")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other tensors on {dev}")


_WORDS = (torch.int32, torch.uint32) if hasattr(torch, "uint32") else (torch.int32,)
_F32 = (torch.float32,)


def _check_cache(desc: "CacheDesc", cache: "LayerCache"):
    words, meta, _ = vq_cache_layout(desc)
    for name in ("packed_k", "packed_v"):
        _check_flat(f"cache.{name}", getattr(cache, name), words, _WORDS)
    for name in ("scale_k", "zero_k", "scale_v", "zero_v"):
        _check_flat(f"cache.{name}", getattr(cache, name), meta, _F32)
    ptrs = (cache.packed_k.data_ptr(), cache.packed_v.data_ptr(), cache.scale_k.data_ptr(),
            cache.zero_k.data_ptr(), cache.scale_v.data_ptr(), cache.zero_v.data_ptr())
    if ptrs != (cache.c.packed_k, cache.c.packed_v, cache.c.scale_k, cache.c.zero_k, cache.c.scale_v, cache.c.zero_v):
        raise ValueError("cache tensors were replaced after the LayerCache was built")
    return [(f"cache.{n}", getattr(cache, n)) for n in
            ("packed_k", "packed_v", "scale_k", "zero_k", "scale_v", "zero_v")]


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return VQ_BF16
    if t.dtype == torch.float32:
        return VQ_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def vq_cache_layout(desc: CacheDesc):
    """-> (words_per_tensor, meta_per_tensor, block_word_offset list of S+1)."""
    w, m = ctypes.c_size_t(), ctypes.c_size_t()
    offs = (ctypes.c_size_t * (desc.num_blocks + 1))()
    _check(_lib.vq_cache_layout(ctypes.byref(desc.c), ctypes.byref(w), ctypes.byref(m), offs))
    return w.value, m.value, list(offs)


class LayerCache:
    """One layer's cache buffers, allocated by torch (the caller), in the layout
    vq_cache_layout describes."""

    def __init__(self, desc: CacheDesc, device="cuda"):
        words, meta, offs = vq_cache_layout(desc)
        self.desc = desc
        self.block_word_offset = offs
        self.packed_k = torch.empty(words, dtype=torch.int32, device=device)
        self.packed_v = torch.empty(words, dtype=torch.int32, device=device)
        self.scale_k = torch.empty(meta, dtype=torch.float32, device=device)
        self.zero_k = torch.empty(meta, dtype=torch.float32, device=device)
        self.scale_v = torch.empty(meta, dtype=torch.float32, device=device)
        self.zero_v = torch.empty(meta, dtype=torch.float32, device=device)
        self.c = vq_layer_cache(self.packed_k.data_ptr(), self.packed_v.data_ptr(), self.scale_k.data_ptr(),
                                self.zero_k.data_ptr(), self.scale_v.data_ptr(), self.zero_v.data_ptr())

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.packed_k, self.packed_v, self.scale_k, self.zero_k, self.scale_v, self.zero_v))


def vq_quantize_pack_block(desc: CacheDesc, block: int, x: torch.Tensor, packed: torch.Tensor,
                           scale: torch.Tensor, zero: torch.Tensor, stream=None):
    """Quantize + bit-pack one block of one tensor x [B][H][n_s][D] (bf16/fp32)."""
    n = _block_tokens(desc, block)
    _check_slab("x", x, desc, n)
    bhd = desc.batch * desc.heads * desc.head_dim
    _check_flat("packed", packed, bhd * desc.word_rows(block), _WORDS)
    _check_flat("scale", scale, bhd, _F32)
    _check_flat("zero", zero, bhd, _F32)
    _check_devices(("x", x), ("packed", packed), ("scale", scale), ("zero", zero))
    _check(_lib.vq_quantize_pack_block(ctypes.byref(desc.c), block, x.data_ptr(), _dtype(x), _strides(x),
                                       packed.data_ptr(), scale.data_ptr(), zero.data_ptr(), _stream(stream)))


def vq_cache_append(desc: CacheDesc, cache: LayerCache, block: int, k: torch.Tensor, v: torch.Tensor, stream=None):
    """Quantize block `block` of K and V ([B][H][n_s][D] views) into the layer cache."""
    if k.dtype != v.dtype:
        raise ValueError("k and v must have the same dtype")
    n = _block_tokens(desc, block)
    _check_slab("k", k, desc, n)
    _check_slab("v", v, desc, n)
    _check_devices(("k", k), ("v", v), *_check_cache(desc, cache))
    _check(_lib.vq_cache_append(ctypes.byref(desc.c), ctypes.byref(cache.c), block, k.data_ptr(), v.data_ptr(),
                                _dtype(k), _strides(k), _strides(v), _stream(stream)))


def vq_attention_block(desc: CacheDesc, cache: LayerCache, block: int, q: torch.Tensor, softmax_scale: float,
                       out: torch.Tensor, stream=None):
    """Attention of block `block`'s queries q [B][H][n_s][D] (bf16) over the packed
    cache of blocks 0..block; writes out [B][H][n_s][D] (fp32 or bf16)."""
    if q.dtype != torch.bfloat16:
        raise ValueError("q must be bfloat16")
    n = _block_tokens(desc, block)
    _check_slab("q", q, desc, n)
    _check_slab("out", out, desc, n)
    _check_devices(("q", q), ("out", out), *_check_cache(desc, cache))
    _check(_lib.vq_attention_block(ctypes.byref(desc.c), ctypes.byref(cache.c), block, q.data_ptr(), _strides(q),
                                   ctypes.c_float(softmax_scale), out.data_ptr(), _dtype(out), _strides(out),
                                   _stream(stream)))


def vq_append_attention_block(desc: CacheDesc, cache: LayerCache, block: int, k: torch.Tensor, v: torch.Tensor,
                              q: torch.Tensor, softmax_scale: float, out: torch.Tensor, stream=None):
    """Append block `block` of K and V ([B][H][n_s][D]) and attend its queries q
    over blocks 0..block in one call; the same cache and output as
    vq_cache_append followed by vq_attention_block."""
    if k.dtype != v.dtype:
        raise ValueError("k and v must have the same dtype")
    if q.dtype != torch.bfloat16:
        raise ValueError("q must be bfloat16")
    n = _block_tokens(desc, block)
    for name, t in (("k", k), ("v", v), ("q", q), ("out", out)):
        _check_slab(name, t, desc, n)
    _check_devices(("k", k), ("v", v), ("q", q), ("out", out), *_check_cache(desc, cache))
    _check(_lib.vq_append_attention_block(ctypes.byref(desc.c), ctypes.byref(cache.c), block, k.data_ptr(),
                                          v.data_ptr(), _dtype(k), _strides(k), _strides(v), q.data_ptr(),
                                          _strides(q), ctypes.c_float(softmax_scale), out.data_ptr(), _dtype(out),
                                          _strides(out), _stream(stream)))


def vq_paper_layout(desc: CacheDesc):
    """-> (words_per_tensor, meta_words_per_tensor, block_word_offset list of S+1) of the storage
    format the results tables count (one padding-free stream per block, 32-bit metadata pairs)."""
    w, m = ctypes.c_size_t(), ctypes.c_size_t()
    offs = (ctypes.c_size_t * (desc.num_blocks + 1))()
    _check(_lib.vq_paper_layout(ctypes.byref(desc.c), ctypes.byref(w), ctypes.byref(m), offs))
    return w.value, m.value, list(offs)


def vq_paper_pack(desc: CacheDesc, cache: LayerCache, k_words: torch.Tensor, v_words: torch.Tensor,
                  k_meta: torch.Tensor, v_meta: torch.Tensor, stream=None):
    """Write the layer cache in the storage format (lossless when desc.meta_fp16)."""
    words, meta, _ = vq_paper_layout(desc)
    for name, t, n in (("k_words", k_words, words), ("v_words", v_words, words), ("k_meta", k_meta, meta),
                       ("v_meta", v_meta, meta)):
        _check_flat(name, t, n, _WORDS)
    _check_devices(("k_words", k_words), ("v_words", v_words), ("k_meta", k_meta), ("v_meta", v_meta),
                   *_check_cache(desc, cache))
    _check(_lib.vq_paper_pack(ctypes.byref(desc.c), ctypes.byref(cache.c), k_words.data_ptr(), v_words.data_ptr(),
                              k_meta.data_ptr(), v_meta.data_ptr(), _stream(stream)))


def vq_paper_unpack(desc: CacheDesc, k_words: torch.Tensor, v_words: torch.Tensor, k_meta: torch.Tensor,
                    v_meta: torch.Tensor, cache: LayerCache, stream=None):
    """Fill the layer cache from the storage format."""
    words, meta, _ = vq_paper_layout(desc)
    for name, t, n in (("k_words", k_words, words), ("v_words", v_words, words), ("k_meta", k_meta, meta),
                       ("v_meta", v_meta, meta)):
        _check_flat(name, t, n, _WORDS)
    _check_devices(("k_words", k_words), ("v_words", v_words), ("k_meta", k_meta), ("v_meta", v_meta),
                   *_check_cache(desc, cache))
    _check(_lib.vq_paper_unpack(ctypes.byref(desc.c), k_words.data_ptr(), v_words.data_ptr(), k_meta.data_ptr(),
                                v_meta.data_ptr(), ctypes.byref(cache.c), _stream(stream)))


def vq_dequantize(desc: CacheDesc, block: int, packed: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor,
                  out: torch.Tensor, stream=None):
    """Check-only: dequantize one packed block into out [B][H][n_s][D] float32 (contiguous)."""
    if out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be contiguous float32")
    n = _block_tokens(desc, block)
    _check_slab("out", out, desc, n)
    bhd = desc.batch * desc.heads * desc.head_dim
    _check_flat("packed", packed, bhd * desc.word_rows(block), _WORDS)
    _check_flat("scale", scale, bhd, _F32)
    _check_flat("zero", zero, bhd, _F32)
    _check_devices(("packed", packed), ("scale", scale), ("zero", zero), ("out", out))
    _check(_lib.vq_dequantize(ctypes.byref(desc.c), block, packed.data_ptr(), scale.data_ptr(), zero.data_ptr(),
                              out.data_ptr(), _stream(stream)))


def vq_poll_device_error() -> int:
    code = ctypes.c_uint32()
    _check(_lib.vq_poll_device_error(ctypes.byref(code)))
    return code.value


def vq_check_wait_timeout(max_iters: int, stream=None):
    """Launch the self-test whose bounded wait times out (see vq.h); the device
    error word then holds flag 1 once the stream has run it."""
    _check(_lib.vq_check_wait_timeout(max_iters, _stream(stream)))


def vq_version() -> int:
    return _lib.vq_version()


def raw_lib():
    """The ctypes handle (for ABI tests)."""
    return _lib
