"""The Python binding rejects tensors that do not fit the call (wrong device,
shape, dtype or size) with ValueError before anything reaches the C ABI, so a
host tensor or a short slice can never become an out-of-bounds device access.
No GPU is needed: the checks run on CPU tensors."""
import pytest
import torch

from bit_kv_cache_25_b200 import vq

B, H, D, BITS = 2, 3, 64, 3
SCHED = [1, 4, 9, 16]


@pytest.fixture
def desc():
    return vq.CacheDesc(B, H, D, BITS, SCHED)


def _slab(n, dtype=torch.bfloat16):
    return torch.zeros((B, H, n, D), dtype=dtype)


def _meta():
    return torch.zeros(B * H * D, dtype=torch.float32)


def _words(desc, s):
    return torch.zeros(B * H * D * desc.word_rows(s), dtype=torch.int32)


def test_quantize_checks(desc):
    s = 3
    good = dict(x=_slab(16), packed=_words(desc, s), scale=_meta(), zero=_meta())
    cases = [
        (dict(x=_slab(9)), "shape"),                                   # wrong block length
        (dict(x=_slab(16).transpose(0, 1)), "shape"),                  # [H][B] order
        (dict(packed=_words(desc, s)[:-1]), "at least"),               # one word short
        (dict(scale=_meta()[:-4]), "at least"),
        (dict(zero=torch.zeros(B * H * D, dtype=torch.float64)), "dtype"),
        (dict(packed=torch.zeros(2 * B * H * D * desc.word_rows(s), dtype=torch.int32)[::2]), "contiguous"),
        ({}, "CUDA"),                                                  # host tensors
    ]
    for over, msg in cases:
        a = dict(good)
        a.update(over)
        with pytest.raises(ValueError, match=msg):
            vq.vq_quantize_pack_block(desc, s, a["x"], a["packed"], a["scale"], a["zero"])
    with pytest.raises(ValueError, match="out of range"):
        vq.vq_quantize_pack_block(desc, 4, good["x"], good["packed"], good["scale"], good["zero"])


def test_append_attention_dequantize_checks(desc):
    cache = vq.LayerCache(desc, device="cpu")
    s = 2
    k, v, q = _slab(9), _slab(9), _slab(9)
    out = _slab(9, torch.float32)
    with pytest.raises(ValueError, match="shape"):
        vq.vq_cache_append(desc, cache, s, k, _slab(4))
    with pytest.raises(ValueError, match="CUDA"):
        vq.vq_cache_append(desc, cache, s, k, v)
    with pytest.raises(ValueError, match="shape"):
        vq.vq_attention_block(desc, cache, s, q, 0.125, _slab(16, torch.float32))
    with pytest.raises(ValueError, match="CUDA"):
        vq.vq_attention_block(desc, cache, s, q, 0.125, out)
    short = vq.LayerCache(vq.CacheDesc(B, H, D, BITS, SCHED[:3]), device="cpu")
    with pytest.raises(ValueError, match="at least"):
        vq.vq_attention_block(desc, short, s, q, 0.125, out)       # cache sized for fewer blocks
    replaced = vq.LayerCache(desc, device="cpu")
    replaced.scale_v = torch.zeros_like(replaced.scale_v)          # not the buffer the C struct holds
    with pytest.raises(ValueError, match="replaced"):
        vq.vq_attention_block(desc, replaced, s, q, 0.125, out)
    with pytest.raises(ValueError, match="shape"):
        vq.vq_dequantize(desc, s, _words(desc, s), _meta(), _meta(), _slab(4, torch.float32))
    with pytest.raises(ValueError, match="at least"):
        vq.vq_dequantize(desc, s, _words(desc, 0)[:1], _meta(), _meta(), out)
    with pytest.raises(ValueError, match="CUDA"):
        vq.vq_dequantize(desc, s, _words(desc, s), _meta(), _meta(), out)
