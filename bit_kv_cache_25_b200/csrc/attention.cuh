// Packed-KV block attention: the queries of block s attend to every cached
// token of blocks 0..s, read straight from the bit-packed cache.
//
// The pages ("VAR-Q: Tuning-Free KV Cache Quantization ...", Abstract,
// paragraphs 1 and 3) give block-by-block decoding and a packed low-bit cache
// but no attention kernel. The plainest reading: block s is appended, then its
// queries attend to all of blocks 0..s (no mask within or across blocks).
//
// Both kernels attend over the cache's own dequantized values
// x^ = fma(code, scale, zero) of each token's block (fp32), rebuilt on chip
// from the packed words tile by tile; no dequantized copy is kept in HBM.
//
// This file holds the two CUDA-core kernels and the dispatch between them and
// the tensor-core kernel (attention_pipe.cuh), by measured speed on the VAR
// and Infinity shapes: at most 4 queries -> attention_small_kernel; up to 32
// queries whose keys fit in shared memory -> attention_cc_kernel; the rest ->
// attention_pipe_kernel (a 128-row MMA tile is mostly padding below that).
//
// attention_cc_kernel: one CTA per (b, h). The cache's values of blocks 0..s
// are dequantized once into shared memory, x^ = fma(code, scale, zero) in
// fp32 (K^ transposed, [D][PP + 1]; V^ row-major), the queries are converted once
// (times sigma * log2 e), and the three steps run from shared memory in fp32:
//   S = q K^T        warp tasks of 8 rows x 32 keys (one key per lane)
//   P = 2^(S - max)  one warp per row, row sums kept for the output
//   O = P V^ / l     warp tasks of 8 rows x D channels (D / 32 per lane)
// Rows are padded to a multiple of 8 and keys to a multiple of 32 with zeros
// (padded keys are masked to p = 0), so no task needs a bounds check.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "tc_ptx.cuh"
#include "vq_internal.h"

namespace vq {
namespace {

// ---- blocks of at most kSmallMaxQueries queries: one CTA per (b, h), one warp
// per query, lanes across channels; each key's logit is a warp reduction over
// channels and the softmax is online in fp32 (one pass over the keys), with
// the integer codes in the products and the per-block scales applied once per
// (query, block, channel). No shared memory and no CTA barrier: the lowest
// latency for a handful of queries.
constexpr int kSmallMaxQueries = 4;
constexpr int kSmallWarps = 4;

__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;  // butterfly of commutative adds: identical on every lane
}

// Fused append: one warp quantizes tensor t (0 = K, 1 = V) of block s for
// (batch, head) bh into the cache, with the steps of the quantize kernel.
// (Not inlined: it runs once per CTA, and inlined its registers would crowd
// the attention loops.)
template <int BITS>
__device__ __noinline__ void fused_quantize_unit(const AttnParams& p, int bh, int t, int lane) {
  const int D = p.D;
  const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
  const AttnBlockInfo& bi = p.blk[p.s];
  const int64_t BHD = static_cast<int64_t>(p.B) * p.H * D;
  const unsigned char* x = static_cast<const unsigned char*>(t ? p.xv : p.xk);
  const int64_t sb = t ? p.xv_sb : p.xk_sb, sh = t ? p.xv_sh : p.xk_sh, st = t ? p.xv_st : p.xk_st;
  const unsigned char* slab = x + (b * sb + h * sh) * p.x_esize;
  uint32_t* packed = const_cast<uint32_t*>(t ? p.packed_v : p.packed_k) + bi.word_off + static_cast<int64_t>(bh) * bi.W * D;
  float* scale = const_cast<float*>(t ? p.scale_v : p.scale_k) + p.s * BHD + static_cast<int64_t>(bh) * D;
  float* zero = const_cast<float*>(t ? p.zero_v : p.zero_k) + p.s * BHD + static_cast<int64_t>(bh) * D;
  if (p.x_esize == 2)
    quantize_unit_warp<Bf16Vec, BITS>(slab, st * 2, bi.n, bi.W, D, packed, scale, zero, p.meta16 != 0, lane);
  else
    quantize_unit_warp<F32Vec, BITS>(slab, st * 4, bi.n, bi.W, D, packed, scale, zero, p.meta16 != 0, lane);
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
  if (p.fused) {  // this CTA's (b, h) of block s into the cache first (warps 0 and 1: K and V);
    // the cache is then read with plain loads, which see the CTA's own writes after the barrier
    if (warp < 2) fused_quantize_unit<BITS>(p, bh, warp, lane);
    __syncthreads();
  }

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


// ---- attention_cc_kernel
// Largest shared-memory plan; two CTAs per SM at this size (a third would need
// 3 x (76 + 1) KB, above the 228 KB of an SM), three at 74 KB or less.
constexpr int kCcMaxSmem = 76 * 1024;
constexpr int kCcMaxQueries = 32;  // from 36 queries on the tensor-core kernel is faster (VAR-d30 block 5)

// Shared-memory plan of one CTA (offsets in floats).
struct CcLayout {
  int PP, NQP;              // keys padded to 32, rows padded to 8
  int KS;                   // row stride of K^ (PP + 1: a warp's 32 channels of one key hit 32 banks)
  int kt, vs, qs, ps, linv; // K^ [D][KS], V^ [PP][D], q [NQP][D], S/P [NQP][PP], 1/l [NQP]
  int floats;
};

__host__ __device__ inline CcLayout cc_layout(int n_q, int P, int D) {
  CcLayout L;
  L.PP = (P + 31) & ~31;
  L.NQP = (n_q + 7) & ~7;
  L.KS = L.PP + 1;
  L.kt = 0;
  L.vs = (L.kt + D * L.KS + 3) & ~3;
  L.qs = L.vs + L.PP * D;
  L.ps = L.qs + L.NQP * D;
  L.linv = L.ps + L.NQP * L.PP;
  L.floats = L.linv + L.NQP;
  return L;
}

// THREADS: 128 for up to 16 queries, 256 above (more warps for the same
// shared memory once there are enough row and key tasks to share). The
// 128-thread form is held to 80 registers so that six CTAs fit an SM: its
// small blocks are latency-bound (VAR-d30 blocks 2-3 took 14 % less time
// than at three CTAs).
template <int BITS, int D, int THREADS>
__global__ void __launch_bounds__(THREADS, THREADS == 128 ? 6 : 3) attention_cc_kernel(const __grid_constant__ AttnParams p, int P) {
  constexpr int kCcThreads = THREADS;
  constexpr int kCcWarps = THREADS / 32;
  constexpr int kCcBatch = THREADS == 128 ? 4 : 2;  // dequantize items per thread with loads in flight together
  constexpr int CPW = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  constexpr int CH = D / 32;  // output channels per lane
  extern __shared__ __align__(16) float smc[];
  const int n_q = p.n_q;
  const CcLayout L = cc_layout(n_q, P, D);
  float* kt = smc + L.kt;
  float* vs = smc + L.vs;
  float* qs = smc + L.qs;
  float* ps = smc + L.ps;
  float* linv = smc + L.linv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x;
  const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
  const int64_t BHD = static_cast<int64_t>(p.B) * p.H * D;
  const int PP = L.PP, NQP = L.NQP, KS = L.KS;
  if (p.fused) {  // this CTA's (b, h) of block s into the cache first (warps 0 and 1: K and V)
    if (warp < 2) fused_quantize_unit<BITS>(p, bh, warp, lane);
    __syncthreads();
  }

  // ---- padding: keys [P, PP) of K^ and V^, rows [n_q, NQP) of q are zero
  for (int e = tid; e < D * (PP - P); e += kCcThreads) {
    const int c = e % D, j = P + e / D;
    kt[c * KS + j] = 0.0f;
    vs[j * D + c] = 0.0f;
  }
  for (int e = n_q * D + tid; e < NQP * D; e += kCcThreads) qs[e] = 0.0f;
  // ---- queries: bf16 -> fp32 times sigma * log2(e), 8 per 16-byte load
  const float qmul = p.softmax_scale * 1.4426950408889634f;
  for (int e = tid; e < n_q * (D / 8); e += kCcThreads) {
    const int i = e / (D / 8), c8 = e - i * (D / 8);
    const uint4 v = *reinterpret_cast<const uint4*>(p.q + b * p.q_sb + h * p.q_sh + static_cast<int64_t>(i) * p.q_st + 8 * c8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float* dst = qs + i * D + 8 * c8;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      dst[2 * k] = __uint_as_float(w[k] << 16) * qmul;
      dst[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u) * qmul;
    }
  }
  // ---- dequantize blocks 0..s: one (block, word row, channel) per item, kCcBatch items per thread in flight
  int E = 0;
  for (int kb = 0; kb <= p.s; ++kb) E += p.blk[kb].W * D;
  for (int e0 = tid; e0 < E; e0 += kCcBatch * kCcThreads) {
    uint32_t wk[kCcBatch], wv[kCcBatch];
    float sk[kCcBatch], zk[kCcBatch], sv[kCcBatch], zv[kCcBatch];
    int j0[kCcBatch], ns[kCcBatch], ch[kCcBatch];
#pragma unroll
    for (int u = 0; u < kCcBatch; ++u) {
      const int e = e0 + u * kCcThreads;
      ns[u] = 0;
      ch[u] = 0;
      j0[u] = 0;
      wk[u] = wv[u] = 0u;
      sk[u] = zk[u] = sv[u] = zv[u] = 0.0f;
      if (e < E) {
        int kb = 0, base = 0, key = 0;
        while (e >= base + p.blk[kb].W * D) {
          base += p.blk[kb].W * D;
          key += p.blk[kb].n;
          ++kb;
        }
        const int w = (e - base) / D, c = (e - base) - w * D;
        const AttnBlockInfo& bi = p.blk[kb];
        const int64_t off = bi.word_off + static_cast<int64_t>(bh) * bi.W * D + static_cast<int64_t>(w) * D + c;
        const int64_t mo = kb * BHD + static_cast<int64_t>(bh) * D + c;
        // plain loads (not the read-only path): with a fused append this CTA
        // wrote block s's words just before
        wk[u] = p.packed_k[off];
        wv[u] = p.packed_v[off];
        sk[u] = p.scale_k[mo];
        zk[u] = p.zero_k[mo];
        sv[u] = p.scale_v[mo];
        zv[u] = p.zero_v[mo];
        j0[u] = key + w * CPW;
        ns[u] = min(CPW, bi.n - w * CPW);
        ch[u] = c;
      }
    }
#pragma unroll
    for (int u = 0; u < kCcBatch; ++u) {
#pragma unroll
      for (int i = 0; i < CPW; ++i) {
        if (i < ns[u]) {
          const float ck = static_cast<float>((wk[u] >> (BITS * i)) & MASK);
          const float cv = static_cast<float>((wv[u] >> (BITS * i)) & MASK);
          kt[ch[u] * KS + j0[u] + i] = fmaf(ck, sk[u], zk[u]);
          vs[(j0[u] + i) * D + ch[u]] = fmaf(cv, sv[u], zv[u]);
        }
      }
    }
  }
  __syncthreads();

  // ---- S = q K^T: task (8 rows, 32 keys), key j = 32 kg + lane
  const int nkg = PP / 32;
  for (int t = warp; t < (NQP / 8) * nkg; t += kCcWarps) {
    const int i0 = (t / nkg) * 8, j = (t - (t / nkg) * nkg) * 32 + lane;
    float acc[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r] = 0.0f;
#pragma unroll 4
    for (int c = 0; c < D; c += 4) {
      const float k0 = kt[c * KS + j], k1 = kt[(c + 1) * KS + j], k2 = kt[(c + 2) * KS + j], k3 = kt[(c + 3) * KS + j];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float4 qv = *reinterpret_cast<const float4*>(qs + (i0 + r) * D + c);
        acc[r] = fmaf(qv.x, k0, fmaf(qv.y, k1, fmaf(qv.z, k2, fmaf(qv.w, k3, acc[r]))));
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) ps[(i0 + r) * PP + j] = acc[r];
  }
  __syncthreads();

  // ---- softmax: warp per row; keys past P get p = 0
  for (int i = warp; i < n_q; i += kCcWarps) {
    float m = -INFINITY;
    for (int j = lane; j < P; j += 32) m = fmaxf(m, ps[i * PP + j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.0f;
    for (int j = lane; j < PP; j += 32) {
      const float e = j < P ? tc::ex2(ps[i * PP + j] - m) : 0.0f;
      ps[i * PP + j] = e;
      l += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) linv[i] = 1.0f / l;
  }
  __syncthreads();

  // ---- O = P V^ / l: task of 8 rows, channels lane + 32 k
  for (int t = warp; t < NQP / 8; t += kCcWarps) {
    const int i0 = 8 * t;
    float acc[8][CH];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int k = 0; k < CH; ++k) acc[r][k] = 0.0f;
#pragma unroll 1
    for (int j = 0; j < PP; j += 4) {
      float vv[4][CH];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int k = 0; k < CH; ++k) vv[u][k] = vs[(j + u) * D + lane + 32 * k];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float4 pv = *reinterpret_cast<const float4*>(ps + (i0 + r) * PP + j);
#pragma unroll
        for (int k = 0; k < CH; ++k)
          acc[r][k] = fmaf(pv.x, vv[0][k], fmaf(pv.y, vv[1][k], fmaf(pv.z, vv[2][k], fmaf(pv.w, vv[3][k], acc[r][k]))));
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int i = i0 + r;
      if (i >= n_q) break;
      const float sc = linv[i];
      const int64_t obase = b * p.o_sb + h * p.o_sh + static_cast<int64_t>(i) * p.o_st;
#pragma unroll
      for (int k = 0; k < CH; ++k) {
        const float val = acc[r][k] * sc;
        if (p.out_f32) {
          static_cast<float*>(p.out)[obase + lane + 32 * k] = val;
        } else {
          const uint32_t x = __float_as_uint(val);
          static_cast<uint16_t*>(p.out)[obase + lane + 32 * k] =
              static_cast<uint16_t>((x + 0x7fffu + ((x >> 16) & 1u)) >> 16);  // round to nearest even
        }
      }
    }
  }
}

// Keys of blocks 0..s.
inline int attn_keys(const AttnParams& p) {
  int P = 0;
  for (int k = 0; k <= p.s; ++k) P += p.blk[k].n;
  return P;
}

inline bool cc_fits(const AttnParams& p) {
  const CcLayout L = cc_layout(p.n_q, attn_keys(p), p.D);
  return p.n_q <= kCcMaxQueries && static_cast<size_t>(L.floats) * 4 <= kCcMaxSmem;
}

template <int BITS, int D, int THREADS>
cudaError_t launch_attention_cc(const AttnParams& p, cudaStream_t stream) {
  static bool configured[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(attention_cc_kernel<BITS, D, THREADS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kCcMaxSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int P = attn_keys(p);
  const size_t smem = static_cast<size_t>(cc_layout(p.n_q, P, D).floats) * 4;
  attention_cc_kernel<BITS, D, THREADS><<<p.B * p.H, THREADS, smem, stream>>>(p, P);
  return cudaGetLastError();
}

}  // namespace
}  // namespace vq

#include "attention_pipe.cuh"

namespace vq {

namespace {

// Kernel choice per block, by measured speed on the VAR and Infinity shapes:
// few queries -> one warp per query; few queries over few keys -> the
// CUDA-core kernel (a 128-row MMA tile would be mostly padding); otherwise the
// tensor cores. More than 128 queries: two query tiles per work item sharing
// every dequantized K/V tile; otherwise one query tile per item, the two
// softmax warpgroups taking the items in turn.
}  // namespace

// Whether block s's append runs inside its attention launch: the CUDA-core
// kernels' CTAs (one per (batch, head)) then quantize their own (batch, head)
// slabs before attending. That saves a launch, but the CTA's quantize is a
// serial prologue, so it only pays while the grid is about one wave: measured
// with CUDA graphs, Infinity-2B blocks 0-2 (128 (batch, head)) took 6-12 us
// fused against 9-17 us as two launches, VAR-d30 blocks 0-4 (3840) 32-152
// against 16-128. On the tensor-core kernel the prologue never overlapped the
// attention (Infinity blocks 5-6 8-10 % slower, VAR-d30 blocks 5-9 4-15 %), so
// those blocks always run the two launches.
bool attention_fusable(const AttnParams& p) {
  if (!(p.n_q <= kSmallMaxQueries || cc_fits(p))) return false;
  static int sms[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (sms[dev] == 0 && cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    sms[dev] = 0;
    return false;
  }
  return static_cast<int64_t>(p.B) * p.H <= 4 * static_cast<int64_t>(sms[dev]);
}

namespace {

template <int BITS, int D>
cudaError_t launch_attention_typed(const AttnParams& p, cudaStream_t stream) {
  if (p.n_q <= kSmallMaxQueries) return launch_attention_small<BITS, D>(p, stream);
  if (cc_fits(p))
    return p.n_q > 16 ? launch_attention_cc<BITS, D, 256>(p, stream) : launch_attention_cc<BITS, D, 128>(p, stream);
  return p.n_q > 128 ? launch_attention_pipe<BITS, D, 2, false>(p, stream)
                     : launch_attention_pipe<BITS, D, 2, true>(p, stream);
}

template <int BITS>
cudaError_t launch_attention_bits(const AttnParams& p, cudaStream_t stream) {
  if (p.D == 64) return launch_attention_typed<BITS, 64>(p, stream);
  if (p.D == 128) return launch_attention_typed<BITS, 128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_attention(const AttnParams& p, cudaStream_t stream) {
  switch (p.bits) {
    case 2: return launch_attention_bits<2>(p, stream);
    case 3: return launch_attention_bits<3>(p, stream);
    case 4: return launch_attention_bits<4>(p, stream);
    case 6: return launch_attention_bits<6>(p, stream);
    case 8: return launch_attention_bits<8>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace vq
