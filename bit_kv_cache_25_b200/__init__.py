"""VAR-Q-style packed low-bit KV cache for block-by-block visual AR decoding on B200.

The compute lives in libvq.so (CUDA, sm_100a); `vq` is its ctypes binding.
"""
from . import vq  # noqa: F401
from .vq import (CacheDesc, LayerCache, VqError, vq_append_attention_block, vq_attention_block,  # noqa: F401
                 vq_cache_append,
                 vq_cache_layout, vq_dequantize, vq_poll_device_error, vq_quantize_pack_block, vq_version)
