// libvq C ABI: argument validation, cache layout arithmetic and kernel launch.
// This file is the library's single translation unit; the kernels are
// included from their own headers. Every entry point validates all of its
// arguments on the host before it launches anything. See include/vq.h for the
// contract of each call.
#include "../../include/vq.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "vq_device.cuh"
#include "vq_internal.h"

#include "quant_pack.cuh"
#include "attention.cuh"
#include "dequant.cuh"
#include "paper.cuh"
#include "selftest.cuh"

namespace {

thread_local char g_last_error[256] = "";

vq_status fail(vq_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

vq_status ok() {
  g_last_error[0] = '\0';
  return VQ_OK;
}

vq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(VQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int codes_per_word(int bits) { return 32 / bits; }
int64_t word_rows(int64_t n, int bits) { return (n + codes_per_word(bits) - 1) / codes_per_word(bits); }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

vq_status check_desc(const vq_cache_desc* d) {
  if (!d) return fail(VQ_ERR_INVALID_ARGUMENT, "desc is NULL");
  if (d->batch < 1 || d->heads < 1) return fail(VQ_ERR_INVALID_ARGUMENT, "batch and heads must be >= 1");
  if (d->head_dim != 64 && d->head_dim != 128)
    return fail(VQ_ERR_UNSUPPORTED, "head_dim %d unsupported (64 or 128)", d->head_dim);
  if (d->bits != 2 && d->bits != 3 && d->bits != 4 && d->bits != 6 && d->bits != 8)
    return fail(VQ_ERR_UNSUPPORTED, "bits %d unsupported (2, 3, 4, 6 or 8)", d->bits);
  if (d->num_blocks < 1) return fail(VQ_ERR_INVALID_ARGUMENT, "num_blocks must be >= 1");
  if (d->meta_fp16 != 0 && d->meta_fp16 != 1) return fail(VQ_ERR_INVALID_ARGUMENT, "meta_fp16 must be 0 or 1");
  if (!d->block_tokens) return fail(VQ_ERR_INVALID_ARGUMENT, "block_tokens is NULL");
  int64_t total = 0;
  for (int s = 0; s < d->num_blocks; ++s) {
    if (d->block_tokens[s] < 1) return fail(VQ_ERR_INVALID_ARGUMENT, "block_tokens[%d] = %d < 1", s, d->block_tokens[s]);
    total += d->block_tokens[s];
  }
  if (total > (int64_t(1) << 30)) return fail(VQ_ERR_UNSUPPORTED, "sequence of %lld tokens too long", (long long)total);
  const int64_t bhd = int64_t(d->batch) * d->heads * d->head_dim;
  if (bhd * word_rows(total, d->bits) * 2 > (int64_t(1) << 40))
    return fail(VQ_ERR_UNSUPPORTED, "cache too large");
  return VQ_OK;
}

vq_status check_block(const vq_cache_desc* d, int32_t block) {
  if (block < 0 || block >= d->num_blocks)
    return fail(VQ_ERR_INVALID_ARGUMENT, "block %d out of range [0, %d)", block, d->num_blocks);
  return VQ_OK;
}

int64_t block_word_offset(const vq_cache_desc* d, int s) {
  int64_t off = 0;
  const int64_t bhd = int64_t(d->batch) * d->heads * d->head_dim;
  for (int k = 0; k < s; ++k) off += bhd * word_rows(d->block_tokens[k], d->bits);
  return off;
}

vq_status check_strides(const int64_t st[3], int esize, const char* name) {
  if (!st) return fail(VQ_ERR_INVALID_ARGUMENT, "%s strides are NULL", name);
  for (int i = 0; i < 3; ++i) {
    if (st[i] < 0) return fail(VQ_ERR_INVALID_ARGUMENT, "%s stride %d negative", name, i);
    if ((st[i] * esize) % 16 != 0)
      return fail(VQ_ERR_MISALIGNED, "%s stride %d (%lld elements) is not a multiple of 16 bytes", name, i,
                  (long long)st[i]);
  }
  return VQ_OK;
}

// Choose the warps per unit (P, enough units x warps to fill the GPU) and,
// with one warp per unit, the lanes per unit (TL): the fewest rows per team
// load that still cover the unit's rows in one batch of loads, so that small
// blocks put several units in flight per warp. Returns false if one slab is
// too large.
bool plan_quant(vq::QuantParams& p) {
  constexpr int64_t kTargetWarps = 2048;
  constexpr int kBatch = 16;  // loads in flight per lane in pass 1 (kQuantUnroll)
  int P = 1;
  while (P < vq::quant_warps() && int64_t(p.units) * P < kTargetWarps && 2 * P <= p.W) P *= 2;
  p.P = P;
  p.WP = (p.W + P - 1) / P;
  int rw = 1;
  while (rw * kBatch < p.n && rw * p.vecs_per_row < 32) rw *= 2;
  p.TL = (P == 1) ? rw * p.vecs_per_row : 32;
  if (p.TL > 32) p.TL = 32;
  // Ring kernel for slabs from 8 KB up to half the slot budget: every unit is
  // bulk-copied into a shared-memory slot and read from there twice. Two slots
  // per slot owner while that still leaves kRingMaxWarps owners, else one slot
  // each and as many owners as the budget holds (CUDA-graph A/B on VAR-d30:
  // 12.8 KB slabs 35.6 -> 33.5 us, 21.6 KB 57.8 -> 54.6 us per append against
  // two slots each; 8 KB slabs best with two); each owner is a team of warps
  // that shares its units' rows.
  p.ring = 0;
  const int64_t slab = int64_t(p.n) * p.D * p.esize;
  if (slab >= 8192 && slab <= vq::kRingSmemBudget / 2) {
    int ns = 2;
    int64_t rwarps = vq::kRingSmemBudget / (2 * slab);
    if (rwarps < vq::kRingMaxWarps) {
      ns = 1;
      rwarps = vq::kRingSmemBudget / slab;
    }
    if (rwarps > vq::kRingMaxWarps) rwarps = vq::kRingMaxWarps;
    if (rwarps >= 2) {
      p.ring = 1;
      p.RW = static_cast<int>(rwarps);
      p.NSLOT = ns;
      p.slot_bytes = static_cast<int>(slab);
      // the remaining consumer warps join the slot owners: teams of up to 6
      p.RG = std::min(vq::kRingMaxWarps / p.RW, 6);
    }
  }
  return true;
}

vq_status launch_quant(const vq_cache_desc* d, int32_t block, vq_dtype dt, int ntensors, const void* const x[2],
                       const int64_t* const strides[2], uint32_t* const packed[2], float* const scale[2],
                       float* const zero[2], void* stream) {
  if (dt != VQ_BF16 && dt != VQ_F32) return fail(VQ_ERR_UNSUPPORTED, "dtype %d unsupported", int(dt));
  const int esize = dt == VQ_BF16 ? 2 : 4;
  vq::QuantParams p{};
  p.B = d->batch;
  p.H = d->heads;
  p.D = d->head_dim;
  p.n = d->block_tokens[block];
  p.bits = d->bits;
  p.W = static_cast<int>(word_rows(p.n, p.bits));
  p.esize = esize;
  p.vecs_per_row = p.D * esize / 16;
  p.units = ntensors * p.B * p.H;
  p.meta16 = d->meta_fp16 ? 1 : 0;
  for (int i = 0; i < ntensors; ++i) {
    const char* nm = i == 0 ? "k/x" : "v";
    if (!x[i] || !packed[i] || !scale[i] || !zero[i]) return fail(VQ_ERR_INVALID_ARGUMENT, "%s: NULL pointer", nm);
    if (!aligned16(x[i]) || !aligned16(packed[i]) || !aligned16(scale[i]) || !aligned16(zero[i]))
      return fail(VQ_ERR_MISALIGNED, "%s: pointers must be 16-byte aligned", nm);
    vq_status st = check_strides(strides[i], esize, nm);
    if (st != VQ_OK) return st;
    p.t[i].x = x[i];
    p.t[i].sb = strides[i][0];
    p.t[i].sh = strides[i][1];
    p.t[i].st = strides[i][2];
    p.t[i].packed = packed[i];
    p.t[i].scale = scale[i];
    p.t[i].zero = zero[i];
  }
  plan_quant(p);
  cudaError_t e = vq::launch_quant_pack(p, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "quantize+pack launch");
  return ok();
}

// Validates the attention arguments and fills the kernel parameters.
vq_status build_attention(const vq_cache_desc* desc, const vq_layer_cache* cache, int32_t block, const void* q,
                          const int64_t q_strides[3], float softmax_scale, void* out, vq_dtype out_dtype,
                          const int64_t out_strides[3], vq::AttnParams& p) {
  vq_status st = check_desc(desc);
  if (st != VQ_OK) return st;
  if ((st = check_block(desc, block)) != VQ_OK) return st;
  if (block >= vq::kMaxBlocks) return fail(VQ_ERR_UNSUPPORTED, "attention supports at most %d blocks", vq::kMaxBlocks);
  if (!cache || !q || !out) return fail(VQ_ERR_INVALID_ARGUMENT, "NULL cache, q or out");
  if (!cache->packed_k || !cache->packed_v || !cache->scale_k || !cache->zero_k || !cache->scale_v || !cache->zero_v)
    return fail(VQ_ERR_INVALID_ARGUMENT, "cache has a NULL pointer");
  if (out_dtype != VQ_F32 && out_dtype != VQ_BF16) return fail(VQ_ERR_UNSUPPORTED, "out dtype unsupported");
  if (!(softmax_scale > 0.0f) || softmax_scale > 1e6f) return fail(VQ_ERR_INVALID_ARGUMENT, "softmax_scale must be in (0, 1e6]");
  if (!aligned16(q) || !aligned16(out) || !aligned16(cache->packed_k) || !aligned16(cache->packed_v) ||
      !aligned16(cache->scale_k) || !aligned16(cache->zero_k) || !aligned16(cache->scale_v) || !aligned16(cache->zero_v))
    return fail(VQ_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  if ((st = check_strides(q_strides, 2, "q")) != VQ_OK) return st;
  if ((st = check_strides(out_strides, out_dtype == VQ_F32 ? 4 : 2, "out")) != VQ_OK) return st;
  p = vq::AttnParams{};
  p.packed_k = cache->packed_k;
  p.packed_v = cache->packed_v;
  p.scale_k = cache->scale_k;
  p.zero_k = cache->zero_k;
  p.scale_v = cache->scale_v;
  p.zero_v = cache->zero_v;
  p.q = static_cast<const uint16_t*>(q);
  p.q_sb = q_strides[0];
  p.q_sh = q_strides[1];
  p.q_st = q_strides[2];
  p.out = out;
  p.o_sb = out_strides[0];
  p.o_sh = out_strides[1];
  p.o_st = out_strides[2];
  p.out_f32 = out_dtype == VQ_F32 ? 1 : 0;
  p.B = desc->batch;
  p.H = desc->heads;
  p.D = desc->head_dim;
  p.bits = desc->bits;
  p.s = block;
  p.n_q = desc->block_tokens[block];
  p.softmax_scale = softmax_scale;
  p.meta16 = desc->meta_fp16 ? 1 : 0;
  for (int k = 0; k <= block; ++k) {
    p.blk[k].word_off = block_word_offset(desc, k);
    p.blk[k].n = desc->block_tokens[k];
    p.blk[k].W = static_cast<int>(word_rows(desc->block_tokens[k], desc->bits));
  }
  return VQ_OK;
}

}  // namespace

extern "C" {

vq_status vq_cache_layout(const vq_cache_desc* desc, size_t* words_per_tensor, size_t* meta_per_tensor,
                          size_t* block_word_offset_out) {
  vq_status st = check_desc(desc);
  if (st != VQ_OK) return st;
  if (!words_per_tensor || !meta_per_tensor) return fail(VQ_ERR_INVALID_ARGUMENT, "output pointers are NULL");
  const int64_t total = block_word_offset(desc, desc->num_blocks);
  *words_per_tensor = static_cast<size_t>(total);
  *meta_per_tensor = static_cast<size_t>(int64_t(desc->num_blocks) * desc->batch * desc->heads * desc->head_dim);
  if (block_word_offset_out) {
    for (int s = 0; s <= desc->num_blocks; ++s) block_word_offset_out[s] = static_cast<size_t>(block_word_offset(desc, s));
  }
  return ok();
}

vq_status vq_quantize_pack_block(const vq_cache_desc* desc, int32_t block, const void* x, vq_dtype x_dtype,
                                 const int64_t x_strides[3], uint32_t* packed, float* scale, float* zero,
                                 void* stream) {
  vq_status st = check_desc(desc);
  if (st != VQ_OK) return st;
  if ((st = check_block(desc, block)) != VQ_OK) return st;
  const void* xs[2] = {x, nullptr};
  const int64_t* ss[2] = {x_strides, nullptr};
  uint32_t* ps[2] = {packed, nullptr};
  float* sc[2] = {scale, nullptr};
  float* zs[2] = {zero, nullptr};
  return launch_quant(desc, block, x_dtype, 1, xs, ss, ps, sc, zs, stream);
}

vq_status vq_cache_append(const vq_cache_desc* desc, const vq_layer_cache* cache, int32_t block, const void* k,
                          const void* v, vq_dtype kv_dtype, const int64_t k_strides[3], const int64_t v_strides[3],
                          void* stream) {
  vq_status st = check_desc(desc);
  if (st != VQ_OK) return st;
  if ((st = check_block(desc, block)) != VQ_OK) return st;
  if (!cache) return fail(VQ_ERR_INVALID_ARGUMENT, "cache is NULL");
  const int64_t woff = block_word_offset(desc, block);
  const int64_t moff = int64_t(block) * desc->batch * desc->heads * desc->head_dim;
  if (!cache->packed_k || !cache->packed_v || !cache->scale_k || !cache->zero_k || !cache->scale_v || !cache->zero_v)
    return fail(VQ_ERR_INVALID_ARGUMENT, "cache has a NULL pointer");
  const void* xs[2] = {k, v};
  const int64_t* ss[2] = {k_strides, v_strides};
  uint32_t* ps[2] = {cache->packed_k + woff, cache->packed_v + woff};
  float* sc[2] = {cache->scale_k + moff, cache->scale_v + moff};
  float* zs[2] = {cache->zero_k + moff, cache->zero_v + moff};
  return launch_quant(desc, block, kv_dtype, 2, xs, ss, ps, sc, zs, stream);
}

vq_status vq_attention_block(const vq_cache_desc* desc, const vq_layer_cache* cache, int32_t block, const void* q,
                             const int64_t q_strides[3], float softmax_scale, void* out, vq_dtype out_dtype,
                             const int64_t out_strides[3], void* stream) {
  vq::AttnParams p{};
  vq_status st = build_attention(desc, cache, block, q, q_strides, softmax_scale, out, out_dtype, out_strides, p);
  if (st != VQ_OK) return st;
  cudaError_t e = vq::launch_attention(p, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return ok();
}

vq_status vq_append_attention_block(const vq_cache_desc* desc, const vq_layer_cache* cache, int32_t block,
                                    const void* k, const void* v, vq_dtype kv_dtype, const int64_t k_strides[3],
                                    const int64_t v_strides[3], const void* q, const int64_t q_strides[3],
                                    float softmax_scale, void* out, vq_dtype out_dtype, const int64_t out_strides[3],
                                    void* stream) {
  vq::AttnParams p{};
  vq_status st = build_attention(desc, cache, block, q, q_strides, softmax_scale, out, out_dtype, out_strides, p);
  if (st != VQ_OK) return st;
  if (kv_dtype != VQ_BF16 && kv_dtype != VQ_F32) return fail(VQ_ERR_UNSUPPORTED, "dtype %d unsupported", int(kv_dtype));
  const int esize = kv_dtype == VQ_BF16 ? 2 : 4;
  if (!k || !v) return fail(VQ_ERR_INVALID_ARGUMENT, "k/v: NULL pointer");
  if (!aligned16(k) || !aligned16(v)) return fail(VQ_ERR_MISALIGNED, "k/v: pointers must be 16-byte aligned");
  if ((st = check_strides(k_strides, esize, "k")) != VQ_OK) return st;
  if ((st = check_strides(v_strides, esize, "v")) != VQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (vq::attention_fusable(p)) {
    // one launch: the attention CTAs quantize their own (batch, head) first
    p.fused = 1;
    p.x_esize = esize;
    p.xk = k;
    p.xv = v;
    p.xk_sb = k_strides[0];
    p.xk_sh = k_strides[1];
    p.xk_st = k_strides[2];
    p.xv_sb = v_strides[0];
    p.xv_sh = v_strides[1];
    p.xv_st = v_strides[2];
    cudaError_t e = vq::launch_attention(p, s);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "fused append+attention launch");
    return ok();
  }
  // several work items per (batch, head): the append, then the attention
  st = vq_cache_append(desc, cache, block, k, v, kv_dtype, k_strides, v_strides, stream);
  if (st != VQ_OK) return st;
  cudaError_t e = vq::launch_attention(p, s);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return ok();
}

vq_status vq_dequantize(const vq_cache_desc* desc, int32_t block, const uint32_t* packed, const float* scale,
                        const float* zero, float* out, void* stream) {
  vq_status st = check_desc(desc);
  if (st != VQ_OK) return st;
  if ((st = check_block(desc, block)) != VQ_OK) return st;
  if (!packed || !scale || !zero || !out) return fail(VQ_ERR_INVALID_ARGUMENT, "NULL pointer");
  if (!aligned16(packed) || !aligned16(scale) || !aligned16(zero) || !aligned16(out))
    return fail(VQ_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  vq::DequantParams p{};
  p.packed = packed;
  p.scale = scale;
  p.zero = zero;
  p.out = out;
  p.B = desc->batch;
  p.H = desc->heads;
  p.D = desc->head_dim;
  p.n = desc->block_tokens[block];
  p.bits = desc->bits;
  p.W = static_cast<int>(word_rows(p.n, p.bits));
  cudaError_t e = vq::launch_dequant(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
  return ok();
}

vq_status vq_paper_layout(const vq_cache_desc* desc, size_t* words_per_tensor, size_t* meta_words_per_tensor,
                          size_t* block_word_offset_out) {
  vq_status st = check_desc(desc);
  if (st != VQ_OK) return st;
  if (!words_per_tensor || !meta_words_per_tensor) return fail(VQ_ERR_INVALID_ARGUMENT, "output pointers are NULL");
  const int64_t bhd = int64_t(desc->batch) * desc->heads * desc->head_dim;
  const int cpw = codes_per_word(desc->bits);
  int64_t off = 0;
  for (int s = 0; s <= desc->num_blocks; ++s) {
    if (block_word_offset_out) block_word_offset_out[s] = static_cast<size_t>(off);
    if (s < desc->num_blocks) off += (bhd * desc->block_tokens[s] + cpw - 1) / cpw;
  }
  *words_per_tensor = static_cast<size_t>(off);
  *meta_words_per_tensor = static_cast<size_t>(int64_t(desc->num_blocks) * bhd);
  return ok();
}

namespace {

vq_status paper_convert(const vq_cache_desc* desc, const vq_layer_cache* cache, bool pack, uint32_t* const words[2],
                        uint32_t* const meta[2], void* stream) {
  vq_status st = check_desc(desc);
  if (st != VQ_OK) return st;
  if (!cache || !cache->packed_k || !cache->packed_v || !cache->scale_k || !cache->zero_k || !cache->scale_v ||
      !cache->zero_v)
    return fail(VQ_ERR_INVALID_ARGUMENT, "NULL cache or cache pointer");
  for (int t = 0; t < 2; ++t) {
    if (!words[t] || !meta[t]) return fail(VQ_ERR_INVALID_ARGUMENT, "NULL stream or metadata pointer");
    if (!aligned16(words[t]) || !aligned16(meta[t])) return fail(VQ_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  }
  if (!aligned16(cache->packed_k) || !aligned16(cache->packed_v) || !aligned16(cache->scale_k) ||
      !aligned16(cache->zero_k) || !aligned16(cache->scale_v) || !aligned16(cache->zero_v))
    return fail(VQ_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t BH = int64_t(desc->batch) * desc->heads;
  const int cpw = codes_per_word(desc->bits);
  uint32_t* const rows[2] = {cache->packed_k, cache->packed_v};
  float* const scale[2] = {cache->scale_k, cache->scale_v};
  float* const zero[2] = {cache->zero_k, cache->zero_v};
  for (int t = 0; t < 2; ++t) {
    int64_t soff = 0;
    for (int b = 0; b < desc->num_blocks; ++b) {
      const int n = desc->block_tokens[b];
      uint32_t* r = rows[t] + block_word_offset(desc, b);
      cudaError_t e = pack ? vq::launch_paper_block(desc->bits, true, r, words[t] + soff, BH, n, desc->head_dim, s)
                           : vq::launch_paper_block(desc->bits, false, words[t] + soff, r, BH, n, desc->head_dim, s);
      if (e != cudaSuccess) return cuda_fail(e, "paper format launch");
      soff += (BH * desc->head_dim * n + cpw - 1) / cpw;
    }
    const int64_t groups = int64_t(desc->num_blocks) * BH * desc->head_dim;
    cudaError_t e = vq::launch_paper_meta(pack, scale[t], zero[t], meta[t], scale[t], zero[t], groups, s);
    if (e != cudaSuccess) return cuda_fail(e, "paper metadata launch");
  }
  return ok();
}

}  // namespace

vq_status vq_paper_pack(const vq_cache_desc* desc, const vq_layer_cache* cache, uint32_t* k_words, uint32_t* v_words,
                        uint32_t* k_meta, uint32_t* v_meta, void* stream) {
  uint32_t* const w[2] = {k_words, v_words};
  uint32_t* const m[2] = {k_meta, v_meta};
  return paper_convert(desc, cache, true, w, m, stream);
}

vq_status vq_paper_unpack(const vq_cache_desc* desc, const uint32_t* k_words, const uint32_t* v_words,
                          const uint32_t* k_meta, const uint32_t* v_meta, const vq_layer_cache* cache, void* stream) {
  uint32_t* const w[2] = {const_cast<uint32_t*>(k_words), const_cast<uint32_t*>(v_words)};
  uint32_t* const m[2] = {const_cast<uint32_t*>(k_meta), const_cast<uint32_t*>(v_meta)};
  return paper_convert(desc, cache, false, w, m, stream);
}

vq_status vq_check_wait_timeout(uint32_t max_iters, void* stream) {
  if (max_iters < 1 || max_iters > (1u << 24))
    return fail(VQ_ERR_INVALID_ARGUMENT, "max_iters must be in [1, 2^24]");
  cudaError_t e = vq::launch_wait_timeout(max_iters, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "wait-timeout self-test launch");
  return ok();
}

vq_status vq_poll_device_error(uint32_t* code) {
  if (!code) return fail(VQ_ERR_INVALID_ARGUMENT, "code is NULL");
  uint32_t v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, vq::g_device_error, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(vq::g_device_error, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  *code = v;
  return ok();
}

const char* vq_status_string(vq_status status) {
  switch (status) {
    case VQ_OK: return "ok";
    case VQ_ERR_INVALID_ARGUMENT: return "invalid argument";
    case VQ_ERR_UNSUPPORTED: return "unsupported";
    case VQ_ERR_MISALIGNED: return "misaligned";
    case VQ_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* vq_last_error(void) { return g_last_error; }

int32_t vq_version(void) { return 100; }

}  // extern "C"
