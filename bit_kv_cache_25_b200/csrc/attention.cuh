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
// This is the general kernel: float32 CUDA-core arithmetic, one CTA per
// (b, h, 32 queries), 4 warps x 8 queries, 32 keys per step (one per lane),
// online softmax in float32.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "vq_internal.h"

namespace vq {
namespace {

constexpr int kAttnQ = 32;       // queries per CTA
constexpr int kAttnWarps = 4;    // 8 queries per warp
constexpr int kAttnQW = kAttnQ / kAttnWarps;
constexpr int kAttnKeys = 32;    // keys per step

__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

template <int D>
struct AttnF32Smem {
  float q[kAttnQ][D + 4];          // q' = sigma * q * sk for the current key block
  float qs[kAttnQ][D];             // sigma * q
  float bias[kAttnQ];              // sigma * q . zk
  float kt[D][kAttnKeys + 1];      // key codes, [channel][key]
  float v[kAttnKeys][D];           // value codes, [key][channel]
  float p[kAttnWarps][kAttnQW][kAttnKeys];
  float meta[4][D];                // sk, zk, sv, zv of the current block
};

template <int BITS, int D>
__global__ void __launch_bounds__(kAttnWarps * 32) attention_f32_kernel(const __grid_constant__ AttnParams p) {
  constexpr int CPW = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  constexpr int CPL = D / 32;  // output channels per lane
  extern __shared__ __align__(16) unsigned char attn_smem_raw[];
  AttnF32Smem<D>& S = *reinterpret_cast<AttnF32Smem<D>*>(attn_smem_raw);
  auto& sQ = S.q;
  auto& sQs = S.qs;
  auto& sBias = S.bias;
  auto& sKT = S.kt;
  auto& sV = S.v;
  auto& sP = S.p;
  auto& sMeta = S.meta;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int bh = blockIdx.y;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int q0 = blockIdx.x * kAttnQ;
  const int BHD = p.B * p.H * D;

  // sigma * q for this CTA's queries (rows past n_q are zero)
  for (int e = tid; e < kAttnQ * D; e += blockDim.x) {
    const int qi = e / D;
    const int c = e - qi * D;
    float v = 0.0f;
    if (q0 + qi < p.n_q) v = bf16_to_f32(p.q[b * p.q_sb + h * p.q_sh + int64_t(q0 + qi) * p.q_st + c]);
    sQs[qi][c] = __fmul_rn(p.softmax_scale, v);
  }

  float m[kAttnQW], l[kAttnQW], o[kAttnQW][CPL];
#pragma unroll
  for (int i = 0; i < kAttnQW; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < CPL; ++j) o[i][j] = 0.0f;
  }

  for (int kb = 0; kb <= p.s; ++kb) {
    const AttnBlockInfo bi = p.blk[kb];
    __syncthreads();
    for (int c = tid; c < D; c += blockDim.x) {
      const int64_t mo = int64_t(kb) * BHD + int64_t(bh) * D + c;
      sMeta[0][c] = p.scale_k[mo];
      sMeta[1][c] = p.zero_k[mo];
      sMeta[2][c] = p.scale_v[mo];
      sMeta[3][c] = p.zero_v[mo];
    }
    __syncthreads();
    for (int e = tid; e < kAttnQ * D; e += blockDim.x) {
      const int qi = e / D;
      const int c = e - qi * D;
      sQ[qi][c] = __fmul_rn(sQs[qi][c], sMeta[0][c]);
    }
    if (tid < kAttnQ) {
      float acc = 0.0f;
      for (int c = 0; c < D; ++c) acc = fmaf(sQs[tid][c], sMeta[1][c], acc);
      sBias[tid] = acc;
    }
    const uint32_t* pk = p.packed_k + bi.word_off + int64_t(bh) * bi.W * D;
    const uint32_t* pv = p.packed_v + bi.word_off + int64_t(bh) * bi.W * D;

    for (int t0 = 0; t0 < bi.n; t0 += kAttnKeys) {
      __syncthreads();
      for (int e = tid; e < kAttnKeys * D; e += blockDim.x) {
        const int kk = e / D;
        const int c = e - kk * D;
        const int t = t0 + kk;
        float ck = 0.0f, cv = 0.0f;
        if (t < bi.n) {
          const int w = t / CPW;
          const int sh = BITS * (t - w * CPW);
          ck = static_cast<float>((pk[int64_t(w) * D + c] >> sh) & MASK);
          cv = static_cast<float>((pv[int64_t(w) * D + c] >> sh) & MASK);
        }
        sKT[c][kk] = ck;
        sV[kk][c] = cv;
      }
      __syncthreads();
      const bool valid = (t0 + lane) < bi.n;
      const int nk = min(kAttnKeys, bi.n - t0);
#pragma unroll
      for (int i = 0; i < kAttnQW; ++i) {
        const int qi = warp * kAttnQW + i;
        float s = sBias[qi];
#pragma unroll 8
        for (int c = 0; c < D; ++c) s = fmaf(sQ[qi][c], sKT[c][lane], s);
        s = valid ? s : -INFINITY;
        float mx = s;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m[i], mx);
        const float alpha = expf(m[i] - m_new);  // exp(-inf) = 0 on the first step
        const float pr = valid ? expf(s - m_new) : 0.0f;
        float sum = pr;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        sP[warp][i][lane] = pr;
        __syncwarp();
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
          const int c = lane + 32 * j;
          float u = 0.0f;
          for (int t = 0; t < nk; ++t) u = fmaf(sP[warp][i][t], sV[t][c], u);
          o[i][j] = fmaf(o[i][j], alpha, fmaf(sMeta[2][c], u, sMeta[3][c] * sum));
        }
        l[i] = fmaf(l[i], alpha, sum);
        m[i] = m_new;
        __syncwarp();
      }
    }
  }

#pragma unroll
  for (int i = 0; i < kAttnQW; ++i) {
    const int qi = q0 + warp * kAttnQW + i;
    if (qi >= p.n_q) continue;
    const float inv = 1.0f / l[i];
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      const int c = lane + 32 * j;
      const float val = o[i][j] * inv;
      const int64_t off = b * p.o_sb + h * p.o_sh + int64_t(qi) * p.o_st + c;
      if (p.out_f32) {
        static_cast<float*>(p.out)[off] = val;
      } else {
        const uint32_t u = __float_as_uint(val);
        const uint32_t r = (u + 0x7fffu + ((u >> 16) & 1u)) >> 16;  // round to nearest even
        static_cast<uint16_t*>(p.out)[off] = static_cast<uint16_t>(r);
      }
    }
  }
}

template <int BITS, int D>
cudaError_t launch_attention_f32(const AttnParams& p, cudaStream_t stream) {
  dim3 grid((p.n_q + kAttnQ - 1) / kAttnQ, p.B * p.H);
  const int smem = static_cast<int>(sizeof(AttnF32Smem<D>));
  static bool configured[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(attention_f32_kernel<BITS, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  attention_f32_kernel<BITS, D><<<grid, kAttnWarps * 32, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace
}  // namespace vq

#include "attention_tc.cuh"

namespace vq {
namespace {

// Blocks with at least this many queries run on the tensor cores; smaller ones
// (mostly padding in a 128-row MMA tile) on the CUDA-core kernel.
constexpr int kTcMinQueries = 64;

}  // namespace

cudaError_t launch_attention(const AttnParams& p, cudaStream_t stream) {
  if (p.B * p.H > 65535) return cudaErrorInvalidConfiguration;
  if (p.n_q >= kTcMinQueries) {
    if (p.bits == 4 && p.D == 64) return launch_attention_tc<4, 64>(p, stream);
    if (p.bits == 4 && p.D == 128) return launch_attention_tc<4, 128>(p, stream);
    if (p.bits == 3 && p.D == 64) return launch_attention_tc<3, 64>(p, stream);
    if (p.bits == 3 && p.D == 128) return launch_attention_tc<3, 128>(p, stream);
  }
  if (p.bits == 4 && p.D == 64) return launch_attention_f32<4, 64>(p, stream);
  if (p.bits == 4 && p.D == 128) return launch_attention_f32<4, 128>(p, stream);
  if (p.bits == 3 && p.D == 64) return launch_attention_f32<3, 64>(p, stream);
  if (p.bits == 3 && p.D == 128) return launch_attention_f32<3, 128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace vq
