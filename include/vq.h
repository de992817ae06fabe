/*
 * vq.h - C ABI of libvq, a packed low-bit KV cache for block-by-block visual
 * autoregressive decoding on NVIDIA B200 (sm_100a).
 *
 * Method: "VAR-Q: Tuning-Free KV Cache Quantization for Visual Autoregressive
 * Image and Video Generation", Abstract. Visual AR models decode block by block,
 * one scale of a next-scale model at a time (paragraph 1). VAR-Q groups the KV
 * cache along the feature (channel) and block axes, takes the block boundaries
 * from the generation loop with no calibration, and bit-packs the low-bit codes
 * (paragraph 3). "VAR-Q results data (Tables 2-4)", Tables 2a/2b, fixes the
 * storage: their KV-memory column fits one 32-bit metadata pair per
 * (block, channel) group and 10 INT3 codes per 32-bit word.
 *
 * What this library computes, per layer, per tensor (K or V) and per block s:
 *   group (b, h, s, c) = the n_s tokens of block s in channel c of head h of
 *   batch entry b;
 *   mn, mx  = exact min / max of the group (inputs widened exactly to float32);
 *   scale   = (mx - mn) / (2^bits - 1), one IEEE float32 division;
 *   zero    = mn (a zero min is stored as +0);
 *   inv     = min(1/scale, FLT_MAX) (IEEE float32), unused when scale == 0;
 *   code    = rint_half_even((x - mn) * inv), two separately rounded float32 ops;
 *             0 for every token when scale == 0;
 *   packing = codes along tokens: word (w, c) of block s holds tokens
 *             w*cpw .. w*cpw+cpw-1 of channel c, token w*cpw+i in bits
 *             [bits*i, bits*i+bits), cpw = floor(32/bits) (INT4: 8, INT3: 10,
 *             INT2: 16, INT6: 5, INT8: 4); unused slots and bits are 0.
 * Attention of block s (the page gives no attention kernel; this is the plainest
 * reading): every query of block s attends to every cached token of blocks
 * 0..s, its own block included. The cached K/V are the dequantized values
 * code*scale + zero. The result is softmax(softmax_scale * q . k^T) . v.
 *
 * Cache layout of one layer, one tensor (K and V have separate buffers):
 *   packed words: block s at word offset B*H*D*sum_{k<s} W_k, laid out
 *                 [B][H][W_s][D] (uint32), W_k = ceil(n_k / cpw);
 *   scale, zero:  block s at float offset s*B*H*D, laid out [B][H][D] (float32).
 * vq_cache_layout returns these sizes and offsets.
 *
 * Conventions that hold for every entry point:
 *   - Ownership: the caller allocates and owns every buffer. The library
 *     allocates no memory and holds no per-call state. The only global state
 *     is a thread-local text of the last error.
 *   - Host pointers: the descriptor and the stride arrays, read during the call
 *     only. Every other pointer is a device pointer.
 *   - Ordering: work is enqueued on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) and the call returns without waiting.
 *   - Errors: argument, alignment and capability errors return a status before
 *     anything is launched. A failed launch returns VQ_ERR_CUDA. Faults during
 *     execution surface at the caller's next synchronization.
 *     vq_last_error() gives a one-line reason for the last failure on this thread.
 *   - Alignment: every device pointer, and every stride times the element size,
 *     must be a multiple of 16 bytes. Channels are contiguous (stride 1).
 *   - Strides are in elements, ordered {batch, head, token}.
 *   - Inputs must be finite, with |x| < 2^126 so that max - min stays finite.
 *   - Supported: head_dim 64 or 128; bits 2, 3, 4, 6 or 8; K/V in bf16 or
 *     float32; queries in bf16; attention over at most 64 blocks.
 */
#ifndef VQ_H_
#define VQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VQ_OK = 0,
  VQ_ERR_INVALID_ARGUMENT = 1, /* null pointer, bad size, block index out of range */
  VQ_ERR_UNSUPPORTED = 2,      /* head_dim, bits, dtype or size this build does not handle */
  VQ_ERR_MISALIGNED = 3,       /* a pointer or stride breaks the 16-byte rule */
  VQ_ERR_CUDA = 4              /* a CUDA runtime call or launch failed */
} vq_status;

typedef enum { VQ_BF16 = 0, VQ_F32 = 1 } vq_dtype;

/* Static description of one model's cache; lives on the host. */
typedef struct {
  int32_t batch;               /* B >= 1 */
  int32_t heads;               /* H >= 1 */
  int32_t head_dim;            /* D: 64 or 128 */
  int32_t bits;                /* 2, 3, 4, 6 or 8 */
  int32_t num_blocks;          /* S >= 1: number of blocks (scales) in the schedule */
  const int32_t* block_tokens; /* host array [S]; n_s >= 1 tokens in block s */
  int32_t meta_fp16;           /* 0: float32 scale and zero; 1: both rounded to fp16 (one
                                  32-bit pair per group, the size "VAR-Q results data
                                  (Tables 2-4)", Tables 2a/2b, count) and the codes taken
                                  against that stored grid, clamped to [0, 2^bits - 1];
                                  inputs must then stay inside the fp16 range. The cache
                                  still stores them as float32 (exactly); vq_paper_pack
                                  writes the 32-bit pairs. */
} vq_cache_desc;

/* One layer's cache. All device pointers, owned by the caller, sized by
 * vq_cache_layout: packed_* hold words_per_tensor uint32 each, scale_* and
 * zero_* hold meta_per_tensor floats each. */
typedef struct {
  uint32_t* packed_k;
  uint32_t* packed_v;
  float* scale_k;
  float* zero_k;
  float* scale_v;
  float* zero_v;
} vq_layer_cache;

/* Sizes of one layer's cache for one tensor. `words_per_tensor` = uint32 words
 * of packed codes; `meta_per_tensor` = floats of scale (and as many of zero);
 * `block_word_offset` (may be NULL) receives S+1 word offsets, entry s being
 * where block s starts and entry S the total. Host only; no CUDA call. */
vq_status vq_cache_layout(const vq_cache_desc* desc, size_t* words_per_tensor,
                          size_t* meta_per_tensor, size_t* block_word_offset);

/* Quantize and bit-pack block `block` of ONE tensor.
 *   x:         device, block s's n_s tokens, element (b,h,t,c) at
 *              x[b*x_strides[0] + h*x_strides[1] + t*x_strides[2] + c]
 *              (t counted from the block's first token), dtype `x_dtype`;
 *   packed:    device, [B][H][W_s][D] uint32 (written in full, padding zero);
 *   scale, zero: device, [B][H][D] float32.
 * Groups are (b, h, c) over the block's n_s tokens ("VAR-Q ...", Abstract,
 * paragraph 3: grouping along the feature and block axes). */
vq_status vq_quantize_pack_block(const vq_cache_desc* desc, int32_t block,
                                 const void* x, vq_dtype x_dtype,
                                 const int64_t x_strides[3], uint32_t* packed,
                                 float* scale, float* zero, void* stream);

/* Quantize block `block` of K and V (one launch) and store it at block s's
 * place in `cache`. The generation loop supplies the block boundaries, so no
 * calibration is needed ("VAR-Q ...", Abstract, paragraph 3). Re-appending a
 * block overwrites it. k and v follow the x layout of vq_quantize_pack_block,
 * with their own strides. */
vq_status vq_cache_append(const vq_cache_desc* desc, const vq_layer_cache* cache,
                          int32_t block, const void* k, const void* v,
                          vq_dtype kv_dtype, const int64_t k_strides[3],
                          const int64_t v_strides[3], void* stream);

/* Block-causal attention of block s's queries over the packed cache of blocks
 * 0..s, read directly from the packed words with no dequantized copy. Blocks
 * 0..s must have been appended; this is not checked.
 *   q:   device bf16, element (b,h,t,c) at q[b*q_strides[0] + h*q_strides[1] + t*q_strides[2] + c],
 *        t in [0, n_s);
 *   out: device, same indexing with out_strides, dtype `out_dtype` (VQ_F32
 *        gives the accuracy the tests check; VQ_BF16 rounds the float32 result);
 *   softmax_scale: the logit multiplier, usually 1/sqrt(head_dim).
 * Arithmetic: float32 accumulation of logits, softmax and output over the
 * cache's dequantized values (on the tensor cores as hi/lo 16-bit operand
 * pairs: fp16 for K, bf16 for V and the probabilities); the result is within
 * 2e-3 x output RMS of float64 attention
 * over the same dequantized cache. See the kernel sources for the operand
 * precision of each kernel. */
vq_status vq_attention_block(const vq_cache_desc* desc, const vq_layer_cache* cache,
                             int32_t block, const void* q, const int64_t q_strides[3],
                             float softmax_scale, void* out, vq_dtype out_dtype,
                             const int64_t out_strides[3], void* stream);

/* Append and attend in one call: quantize block `block` of K and V into the
 * cache (as vq_cache_append) and run that block's attention (as
 * vq_attention_block). The cache bytes and the output are those of the two
 * calls in sequence. Block-by-block decoding appends each block just before
 * its queries attend ("VAR-Q ...", Abstract, paragraph 1; block boundaries
 * from the generation loop, paragraph 3), so both steps share one launch
 * where that is faster: blocks that run on the CUDA-core kernels (at most 32
 * queries) when batch * heads is at most four per SM; there each attention
 * CTA first quantizes the slabs of its own (batch, head), then attends, and
 * the fresh K/V is read from HBM once. Every other block runs the two
 * launches in order on `stream` (the quantize prologue serializes in front of
 * the attention and costs more than the extra launch). Arguments
 * are those of vq_cache_append and vq_attention_block, validated the same way
 * before anything is launched. */
vq_status vq_append_attention_block(const vq_cache_desc* desc, const vq_layer_cache* cache, int32_t block,
                                    const void* k, const void* v, vq_dtype kv_dtype,
                                    const int64_t k_strides[3], const int64_t v_strides[3], const void* q,
                                    const int64_t q_strides[3], float softmax_scale, void* out,
                                    vq_dtype out_dtype, const int64_t out_strides[3], void* stream);

/* Storage format counted by the KV-memory column of "VAR-Q results data
 * (Tables 2-4)", Tables 2a/2b, for one layer and one tensor: block s is one
 * padding-free stream of its B*H*n_s*D codes in (b, h, token, channel) order,
 * floor(32/bits) codes per 32-bit word (code i in word i / cpw, bits
 * [bits*(i % cpw), bits*(i % cpw) + bits)); the metadata is one 32-bit word per
 * (block, b, h, channel) group, fp16 scale in the low half and fp16 zero in the
 * high half. With the tables' shapes and effective batch its size reproduces
 * every printed VAR-Q image row to the digits shown. `words_per_tensor`: words
 * of all streams; `meta_words_per_tensor`: S*B*H*D; `block_word_offset` (may be
 * NULL) receives S+1 offsets. Host only; no CUDA call. */
vq_status vq_paper_layout(const vq_cache_desc* desc, size_t* words_per_tensor, size_t* meta_words_per_tensor,
                          size_t* block_word_offset);

/* Write a layer's cache (word-row layout) in the storage format above: k_words,
 * v_words hold words_per_tensor words each, k_meta, v_meta meta_words_per_tensor
 * words each (device, caller-owned). The metadata is rounded to fp16, so the
 * conversion is lossless for a cache quantized with desc->meta_fp16 = 1 (whose
 * scale and zero are fp16 values) and rounds the metadata otherwise. */
vq_status vq_paper_pack(const vq_cache_desc* desc, const vq_layer_cache* cache, uint32_t* k_words,
                        uint32_t* v_words, uint32_t* k_meta, uint32_t* v_meta, void* stream);

/* The inverse: fill a layer's cache (word-row layout, padding slots zero) from
 * the storage format. */
vq_status vq_paper_unpack(const vq_cache_desc* desc, const uint32_t* k_words, const uint32_t* v_words,
                          const uint32_t* k_meta, const uint32_t* v_meta, const vq_layer_cache* cache,
                          void* stream);

/* Check-only: dequantize one packed block, x_hat = fma(code, scale, zero) with
 * one float32 rounding, into out [B][H][n_s][D] (contiguous float32). packed,
 * scale and zero are in the layout written by vq_quantize_pack_block. */
vq_status vq_dequantize(const vq_cache_desc* desc, int32_t block, const uint32_t* packed,
                        const float* scale, const float* zero, float* out, void* stream);

/* Read and clear the device error word of the current device. Kernels OR a
 * flag into it instead of trapping: 1 = a bounded wait on a shared-memory
 * barrier gave up (the affected outputs are not written), 2 = a kernel saw
 * parameters its launcher should have rejected. Synchronizes with the device
 * (a blocking copy). */
vq_status vq_poll_device_error(uint32_t* code);

/* Self-test of the device error path (no counterpart on the pages; it checks
 * the library's own failure handling). Launches one thread on `stream` that
 * waits on a shared-memory barrier nothing arrives at, giving up after
 * max_iters polls (1 .. 2^24; each poll after the 64th sleeps ~100 ns), so
 * the wait times out: the kernel ORs flag 1 into the device error word and
 * returns normally, and the context stays usable. Read the flag with
 * vq_poll_device_error after the stream completes. Allocates nothing.
 * VQ_ERR_INVALID_ARGUMENT for max_iters outside the range. */
vq_status vq_check_wait_timeout(uint32_t max_iters, void* stream);

/* Static text for a status code. */
const char* vq_status_string(vq_status status);

/* One-line reason for the last failed call on the calling thread ("" if none). */
const char* vq_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int32_t vq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VQ_H_ */
