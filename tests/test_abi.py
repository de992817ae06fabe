"""The C-ABI library loads, exports every symbol include/vq.h declares, and
rejects bad arguments on the host before any CUDA call (no GPU needed)."""
import ctypes
import os
import re
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))  # the printed-table pins are shared

from bit_kv_cache_25_b200 import vq

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "vq.h")
BAD = 0x1000  # never dereferenced: validation fails first


def declared_symbols():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(vq_\w+)\s*\(", src, flags=re.M)))


def test_every_declared_symbol_is_exported():
    syms = declared_symbols()
    assert "vq_attention_block" in syms and "vq_cache_append" in syms and len(syms) >= 9
    lib = vq.raw_lib()
    for s in syms:
        assert hasattr(lib, s), s
    assert set(vq.EXPORTED) <= set(syms)


def test_status_strings_and_version():
    lib = vq.raw_lib()
    assert lib.vq_status_string(0) == b"ok"
    assert lib.vq_status_string(3) == b"misaligned"
    assert vq.vq_version() >= 100


def _desc(**kw):
    a = dict(batch=2, heads=3, head_dim=64, bits=3, block_tokens=[1, 4, 9, 16])
    a.update(kw)
    return vq.CacheDesc(**a)


@pytest.mark.parametrize("bits,cpw", [(2, 16), (3, 10), (4, 8), (6, 5), (8, 4)])
def test_layout_matches_definition(bits, cpw):
    d = _desc(bits=bits)
    words, meta, offs = vq.vq_cache_layout(d)
    W = [(n + cpw - 1) // cpw for n in d.block_tokens]
    assert offs == [2 * 3 * 64 * sum(W[:s]) for s in range(5)]
    assert words == offs[-1] and meta == 4 * 2 * 3 * 64


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=96), vq.VQ_ERR_UNSUPPORTED),
    (dict(bits=5), vq.VQ_ERR_UNSUPPORTED),
    (dict(bits=7), vq.VQ_ERR_UNSUPPORTED),
    (dict(batch=0), vq.VQ_ERR_INVALID_ARGUMENT),
    (dict(block_tokens=[3, 0]), vq.VQ_ERR_INVALID_ARGUMENT),
])
def test_bad_descriptor_rejected(kw, status):
    with pytest.raises(vq.VqError) as e:
        vq.vq_cache_layout(_desc(**kw))
    assert e.value.status == status


def _call_quant(d, block, x, strides, packed=BAD, scale=BAD, zero=BAD, dtype=vq.VQ_BF16):
    lib = vq.raw_lib()
    st = (ctypes.c_int64 * 3)(*strides)
    return lib.vq_quantize_pack_block(ctypes.byref(d.c), block, x, dtype, st, packed, scale, zero, None)


def test_host_validation_before_launch():
    lib = vq.raw_lib()
    d = _desc()
    assert _call_quant(d, 4, BAD, [3 * 30 * 64, 30 * 64, 64]) == vq.VQ_ERR_INVALID_ARGUMENT   # block out of range
    assert _call_quant(d, -1, BAD, [3 * 30 * 64, 30 * 64, 64]) == vq.VQ_ERR_INVALID_ARGUMENT
    assert _call_quant(d, 1, None, [3 * 30 * 64, 30 * 64, 64]) == vq.VQ_ERR_INVALID_ARGUMENT  # NULL x
    assert _call_quant(d, 1, BAD + 2, [3 * 30 * 64, 30 * 64, 64]) == vq.VQ_ERR_MISALIGNED     # misaligned x
    assert _call_quant(d, 1, BAD, [3 * 30 * 64, 30 * 64, 60]) == vq.VQ_ERR_MISALIGNED         # row stride
    assert _call_quant(d, 1, BAD, [3 * 30 * 64, 30 * 64, 64], dtype=7) == vq.VQ_ERR_UNSUPPORTED
    assert b"16 bytes" in lib.vq_last_error() or b"dtype" in lib.vq_last_error()
    # attention: at most 64 blocks; NULL cache (every case fails before a launch)
    d2 = _desc(bits=8, block_tokens=[1] * 70)
    st = (ctypes.c_int64 * 3)(3 * 30 * 64, 30 * 64, 64)
    cache = vq.vq_layer_cache(BAD, BAD, BAD, BAD, BAD, BAD)
    assert lib.vq_attention_block(ctypes.byref(d2.c), ctypes.byref(cache), 64, BAD, st, ctypes.c_float(0.125), BAD,
                                  vq.VQ_F32, st, None) == vq.VQ_ERR_UNSUPPORTED
    assert lib.vq_attention_block(ctypes.byref(d.c), None, 0, BAD, st, ctypes.c_float(0.125), BAD,
                                  vq.VQ_F32, st, None) == vq.VQ_ERR_INVALID_ARGUMENT
    assert lib.vq_attention_block(ctypes.byref(d.c), ctypes.byref(cache), 0, BAD, st, ctypes.c_float(-1.0), BAD,
                                  vq.VQ_F32, st, None) == vq.VQ_ERR_INVALID_ARGUMENT
    assert lib.vq_dequantize(ctypes.byref(d.c), 9, BAD, BAD, BAD, BAD, None) == vq.VQ_ERR_INVALID_ARGUMENT


def test_launch_without_gpu_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    d = _desc()
    assert _call_quant(d, 1, BAD, [3 * 30 * 64, 30 * 64, 64]) == vq.VQ_ERR_CUDA


def test_paper_layout_through_the_abi_reproduces_printed_kv_memory():
    """The C entry point's storage format sizes give the printed KV GiB of every
    VAR-Q image row of Tables 2a/2b (same check as the oracle's pin)."""
    import test_oracle_pins as pins

    def layout(sched, batch, heads, head_dim, bits):
        return vq.vq_paper_layout(vq.CacheDesc(batch, heads, head_dim, bits, sched))
    pins.check_paper_layout(layout)


def test_meta_fp16_flag_validated():
    d = _desc()
    d.c.meta_fp16 = 2
    with pytest.raises(vq.VqError):
        vq.vq_cache_layout(d)


def test_wait_timeout_selftest_validates_before_launch():
    """The error-path self-test rejects an iteration limit outside 1 .. 2^24
    before any CUDA call."""
    lib = vq.raw_lib()
    for bad in (0, (1 << 24) + 1):
        assert lib.vq_check_wait_timeout(bad, None) == vq.VQ_ERR_INVALID_ARGUMENT
