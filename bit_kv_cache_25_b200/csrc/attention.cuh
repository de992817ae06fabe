// Packed-KV block attention: the queries of block s attend to every cached
// token of blocks 0..s, read straight from the bit-packed cache.
//
// The pages ("VAR-Q: Tuning-Free KV Cache Quantization ...", Abstract,
// paragraphs 1 and 3) give block-by-block decoding and a packed low-bit cache
// but no attention kernel. The plainest reading: block s is appended, then its
// queries attend to all of blocks 0..s (no mask within or across blocks).
//
// Scales are folded in. With k = code_k * sk + zk per (block, channel) and
// v = code_v * sv + zv:
//   logit(i, t) = sum_c (sigma q_ic sk_c) code_k(t, c) + sum_c sigma q_ic zk_c
//               = q'_i . code_k(t) + bias_i       (bias is per (query, block))
//   out_i = sum_blocks [ sv (.) (P code_v) + zv * rowsum(P) ] / l_i
// so the integer codes enter the products exactly and the per-block scales are
// applied once per (query, block, channel).
//
// This file holds the kernel for blocks with few queries (fewer than
// kTcMinQueries): one CTA per (b, h), one warp per query, lanes across
// channels. Each key's logit is a warp reduction over channels; the softmax is
// online in fp32 (one pass over the keys). The packed words of a word-row are
// read once per warp and serve its cpw keys from L1.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "vq_internal.h"

namespace vq {
namespace {

constexpr int kSmallWarps = 4;

__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;  // butterfly of commutative adds: identical on every lane
}

template <int BITS, int D>
__global__ void __launch_bounds__(kSmallWarps * 32) attention_small_kernel(const __grid_constant__ AttnParams p) {
  constexpr int CPW = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  constexpr int J = D / 32;  // channels per lane
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int bh = blockIdx.x;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int64_t BHD = static_cast<int64_t>(p.B) * p.H * D;

  for (int qi = warp; qi < p.n_q; qi += kSmallWarps) {
    const uint16_t* qrow = p.q + b * p.q_sb + h * p.q_sh + static_cast<int64_t>(qi) * p.q_st;
    float qs[J], o[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
      qs[j] = __fmul_rn(p.softmax_scale, bf16_to_f32(qrow[lane + 32 * j]));
      o[j] = 0.0f;
    }
    float m = -INFINITY, l = 0.0f;
    for (int kb = 0; kb <= p.s; ++kb) {
      const AttnBlockInfo bi = p.blk[kb];
      float qp[J], sv[J], zv[J], u[J];
      float bias = 0.0f;
#pragma unroll
      for (int j = 0; j < J; ++j) {
        const int64_t mo = kb * BHD + static_cast<int64_t>(bh) * D + lane + 32 * j;
        qp[j] = __fmul_rn(qs[j], p.scale_k[mo]);
        bias = fmaf(qs[j], p.zero_k[mo], bias);
        sv[j] = p.scale_v[mo];
        zv[j] = p.zero_v[mo];
        u[j] = 0.0f;
      }
      bias = warp_sum(bias);
      float rs = 0.0f;
      const uint32_t* pk = p.packed_k + bi.word_off + static_cast<int64_t>(bh) * bi.W * D;
      const uint32_t* pv = p.packed_v + bi.word_off + static_cast<int64_t>(bh) * bi.W * D;
      for (int w = 0; w < bi.W; ++w) {
        uint32_t wk[J], wv[J];
#pragma unroll
        for (int j = 0; j < J; ++j) {
          wk[j] = pk[static_cast<int64_t>(w) * D + lane + 32 * j];
          wv[j] = pv[static_cast<int64_t>(w) * D + lane + 32 * j];
        }
        const int nslot = min(CPW, bi.n - w * CPW);
#pragma unroll
        for (int i = 0; i < CPW; ++i) {
          if (i >= nslot) break;
          float dot = 0.0f;
#pragma unroll
          for (int j = 0; j < J; ++j) dot = fmaf(qp[j], static_cast<float>((wk[j] >> (BITS * i)) & MASK), dot);
          const float sc = warp_sum(dot) + bias;
          if (sc > m) {  // uniform across the warp
            const float alpha = expf(m - sc);
            m = sc;
            l *= alpha;
            rs *= alpha;
#pragma unroll
            for (int j = 0; j < J; ++j) {
              o[j] *= alpha;
              u[j] *= alpha;
            }
          }
          const float pr = expf(sc - m);
          l += pr;
          rs += pr;
#pragma unroll
          for (int j = 0; j < J; ++j) u[j] = fmaf(pr, static_cast<float>((wv[j] >> (BITS * i)) & MASK), u[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < J; ++j) o[j] = fmaf(u[j], sv[j], fmaf(rs, zv[j], o[j]));
    }
    const float inv = 1.0f / l;
    const int64_t obase = b * p.o_sb + h * p.o_sh + static_cast<int64_t>(qi) * p.o_st;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const float val = o[j] * inv;
      if (p.out_f32) {
        static_cast<float*>(p.out)[obase + lane + 32 * j] = val;
      } else {
        const uint32_t x = __float_as_uint(val);
        static_cast<uint16_t*>(p.out)[obase + lane + 32 * j] =
            static_cast<uint16_t>((x + 0x7fffu + ((x >> 16) & 1u)) >> 16);  // round to nearest even
      }
    }
  }
}

template <int BITS, int D>
cudaError_t launch_attention_small(const AttnParams& p, cudaStream_t stream) {
  attention_small_kernel<BITS, D><<<p.B * p.H, kSmallWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace
}  // namespace vq

#include "attention_pipe.cuh"

namespace vq {
namespace {

// Blocks with at least this many queries run on the tensor cores; smaller ones
// (mostly padding in a 128-row MMA tile) on the CUDA-core kernel.
constexpr int kTcMinQueries = 16;

}  // namespace

cudaError_t launch_attention(const AttnParams& p, cudaStream_t stream) {
  if (p.n_q >= kTcMinQueries) {
    // more than 128 queries: two query tiles per work item sharing every
    // dequantized K/V tile; otherwise one query tile per item, the two
    // softmax warpgroups taking the items in turn
    const bool pair = p.n_q > 128;
    if (p.bits == 4 && p.D == 64)
      return pair ? launch_attention_pipe<4, 64, 2, false>(p, stream) : launch_attention_pipe<4, 64, 2, true>(p, stream);
    if (p.bits == 4 && p.D == 128)
      return pair ? launch_attention_pipe<4, 128, 2, false>(p, stream) : launch_attention_pipe<4, 128, 2, true>(p, stream);
    if (p.bits == 3 && p.D == 64)
      return pair ? launch_attention_pipe<3, 64, 2, false>(p, stream) : launch_attention_pipe<3, 64, 2, true>(p, stream);
    if (p.bits == 3 && p.D == 128)
      return pair ? launch_attention_pipe<3, 128, 2, false>(p, stream) : launch_attention_pipe<3, 128, 2, true>(p, stream);
  }
  if (p.bits == 4 && p.D == 64) return launch_attention_small<4, 64>(p, stream);
  if (p.bits == 4 && p.D == 128) return launch_attention_small<4, 128>(p, stream);
  if (p.bits == 3 && p.D == 64) return launch_attention_small<3, 64>(p, stream);
  if (p.bits == 3 && p.D == 128) return launch_attention_small<3, 128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace vq
