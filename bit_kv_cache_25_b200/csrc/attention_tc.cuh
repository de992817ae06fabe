// Packed-KV block attention on the sm_100a tensor cores (tcgen05 + TMEM).
//
// Same computation as the CUDA-core kernel in attention.cuh: the queries of
// block s attend to every cached token of blocks 0..s. Scales are folded into
// the queries, so the MMAs multiply exact integer codes:
//   S = q'_scaled . code_k^T          q' = sigma * q (.) sk, one power-of-two
//                                     scale per (query, key block) so that
//                                     max |q'| sits in [2^10, 2^11)
//   logit = 2^e * S + sigma * q . zk
//   U    += P . code_v                (per key block, TMEM)
//   O    += U (.) sv + rowsum(P) * zv (folded once per key block, TMEM)
//
// Operand precision. One fp16 operand leaves the outputs of the pages'
// workloads outside a 2e-3 x RMS bound: fp16 probabilities alone give 2.5e-3 on
// the Infinity-2B-shaped INT4 cache. So every operand that is not an exact
// small integer is split into an fp16 hi part and an fp16 lo part
// (x = hi + lo + O(2^-22 x)): q' hi/lo times codes, then P hi/lo times codes,
// four MMAs per tile, all into fp32 accumulators. Codes 0..15 are exact in fp16.
//
// Tiles: 128 queries per CTA (M = 128, one TMEM lane per query row, one thread
// per row); key tiles of 8 packed word-rows (64 keys at INT4, 80 at INT3),
// never crossing a block boundary because the scales change per block. The
// unpacked operands are written to shared memory in the canonical K-major
// 128-byte-swizzle layout: K codes [keys][D], V codes [D][keys],
// P [128][keys], q' [128][D]. Online softmax in fp32 with a lazy reference
// maximum: rescaling happens only when a row maximum grows by more than
// kTau (p stays <= e^kTau, fine for fp16).
//
// This first tensor-core version runs its phases one after another inside a
// CTA (unpack -> QK MMA -> softmax -> PV MMA); overlap comes from co-resident
// CTAs.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tc_ptx.cuh"
#include "vq_device.cuh"
#include "vq_internal.h"

namespace vq {
namespace {

constexpr float kTau = 8.0f;          // lazy-rescale threshold (natural-log units)
constexpr int kTcThreads = 128;       // 4 warps = 128 TMEM lanes = 128 query rows

template <int BITS, int D>
struct TcCfg {
  static constexpr int CPW = 32 / BITS;
  static constexpr uint32_t MASK = (1u << BITS) - 1u;
  static constexpr int WT = 8;                  // word-rows per key tile
  static constexpr int KT = WT * CPW;           // keys per tile: 64 (INT4), 80 (INT3)
  static constexpr int KTP = ((KT + 63) / 64) * 64;  // key extent of V / P tiles, whole 64-key slabs
  static_assert(KT % 16 == 0 && KT <= 256, "key tile must be a multiple of 16, at most 256");
  // shared memory (byte offsets from a 1024-aligned base)
  static constexpr int Q_HI = 0;                       // [128][D] fp16
  static constexpr int Q_LO = Q_HI + 128 * D * 2;
  static constexpr int K_T = Q_LO + 128 * D * 2;       // [KT][D] fp16
  static constexpr int V_T = K_T + KT * D * 2;         // [D][KTP] fp16
  static constexpr int P_HI = V_T + D * KTP * 2;       // [128][KTP] fp16
  static constexpr int P_LO = P_HI + 128 * KTP * 2;
  static constexpr int META = P_LO + 128 * KTP * 2;    // sk, zk, sv, zv: [4][D] fp32
  static constexpr int BARS = META + 4 * D * 4;
  static constexpr int TMEM_SLOT = BARS + 16;
  static constexpr int SMEM = TMEM_SLOT + 16;
  static constexpr int SMEM_ALLOC = SMEM + 1024;       // room to align the base
  static_assert(K_T % 1024 == 0 && V_T % 1024 == 0 && P_HI % 1024 == 0 && P_LO % 1024 == 0, "tile alignment");
  // tensor memory columns
  static constexpr int COL_S = 0;                      // KT columns
  static constexpr int COL_U = 128;                    // D columns
  static constexpr int COL_O = 128 + D;                // D columns
  static constexpr int TMEM_COLS = (128 + 2 * D <= 256) ? 256 : 512;
};

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Two small non-negative integers (< 1024) as one fp16x2 word, exactly:
// 0x6400 is fp16 1024.0, so (0x6400 | c) is 1024 + c; subtracting 1024 leaves c.
__device__ __forceinline__ uint32_t codes_to_half2(uint32_t c0, uint32_t c1) {
  const uint32_t biased = (c0 | (c1 << 16)) | 0x64006400u;
  __half2 h = *reinterpret_cast<const __half2*>(&biased);
  const __half2 k = __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400));
  h = __hsub2(h, k);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int BITS, int D>
__global__ void __launch_bounds__(kTcThreads, 1) attention_tc_kernel(const __grid_constant__ AttnParams p) {
  using C = TcCfg<BITS, D>;
  constexpr int CPW = C::CPW;
  constexpr int KT = C::KT;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char* sm = smem_raw + (sbase - raw);
  float* meta = reinterpret_cast<float*>(sm + C::META);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::BARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::TMEM_SLOT);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int bh = blockIdx.y;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int q0 = blockIdx.x * 128;
  const int row = tid;
  const bool row_valid = (q0 + row) < p.n_q;
  const int64_t BHD = static_cast<int64_t>(p.B) * p.H * D;

  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    fence_barrier_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t idesc_qk = tc::idesc_f16_f32(128, KT);
  const uint32_t idesc_pv = tc::idesc_f16_f32(128, D);

  const uint16_t* qrow = p.q + b * p.q_sb + h * p.q_sh + static_cast<int64_t>(q0 + row) * p.q_st;
  uint32_t phase = 0;
  bool ok = true;
  float m_ref = -INFINITY;  // reference maximum of this row's logits
  float l_tot = 0.0f;       // sum of p over finished blocks (relative to m_ref)
  float rs = 0.0f;          // sum of p over the current block (relative to m_ref)
  bool have_o = false;      // O holds at least one folded block

  for (int kb = 0; kb <= p.s && ok; ++kb) {
    const AttnBlockInfo bi = p.blk[kb];
    __syncthreads();  // previous block's readers of meta are done
    for (int c = tid; c < D; c += kTcThreads) {
      const int64_t mo = kb * BHD + static_cast<int64_t>(bh) * D + c;
      meta[c] = p.scale_k[mo];
      meta[D + c] = p.zero_k[mo];
      meta[2 * D + c] = p.scale_v[mo];
      meta[3 * D + c] = p.zero_v[mo];
    }
    __syncthreads();

    // ---- q' = sigma * q * sk for this row, scaled by 2^-e, split into fp16 hi/lo
    float bias = 0.0f, amax = 0.0f;
    for (int c8 = 0; c8 < D; c8 += 8) {
      uint4 raw8 = make_uint4(0, 0, 0, 0);
      if (row_valid) raw8 = *reinterpret_cast<const uint4*>(qrow + c8);
      const uint32_t w4[4] = {raw8.x, raw8.y, raw8.z, raw8.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float qv = __uint_as_float((k & 1) ? (w4[k >> 1] & 0xffff0000u) : (w4[k >> 1] << 16));
        const float qs = __fmul_rn(p.softmax_scale, qv);
        const float qp = __fmul_rn(qs, meta[c8 + k]);
        amax = fmaxf(amax, fabsf(qp));
        bias = fmaf(qs, meta[D + c8 + k], bias);
      }
    }
    int e = 0;
    if (amax > 0.0f) {
      const int ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127;  // floor(log2) for normals
      e = max(-100, min(100, ex - 10));
    }
    const float down = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);   // 2^-e
    const float up = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);     // 2^e
    for (int c8 = 0; c8 < D; c8 += 8) {
      uint4 raw8 = make_uint4(0, 0, 0, 0);
      if (row_valid) raw8 = *reinterpret_cast<const uint4*>(qrow + c8);
      const uint32_t w4[4] = {raw8.x, raw8.y, raw8.z, raw8.w};
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int k2 = 0; k2 < 4; ++k2) {
        float x[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int k = 2 * k2 + u;
          const float qv = __uint_as_float(u ? (w4[k2] & 0xffff0000u) : (w4[k2] << 16));
          x[u] = __fmul_rn(__fmul_rn(__fmul_rn(p.softmax_scale, qv), meta[c8 + k]), down);
        }
        const __half2 hh = __floats2half2_rn(x[0], x[1]);
        const float2 hf = __half22float2(hh);
        hi[k2] = *reinterpret_cast<const uint32_t*>(&hh);
        lo[k2] = pack_half2(x[0] - hf.x, x[1] - hf.y);
      }
      const uint32_t off = tc::sw128_offset(row, c8, 128);
      tc::sts128(sbase + C::Q_HI + off, hi[0], hi[1], hi[2], hi[3]);
      tc::sts128(sbase + C::Q_LO + off, lo[0], lo[1], lo[2], lo[3]);
    }

    const uint32_t* pk = p.packed_k + bi.word_off + static_cast<int64_t>(bh) * bi.W * D;
    const uint32_t* pv = p.packed_v + bi.word_off + static_cast<int64_t>(bh) * bi.W * D;

    for (int w0 = 0; w0 < bi.W && ok; w0 += C::WT) {
      const int nkeys = min(KT, bi.n - w0 * CPW);
      const bool first_tile = (w0 == 0);

      // ---- unpack K codes: task = (word-row wl, channel octet j)
      for (int task = tid; task < C::WT * (D / 8); task += kTcThreads) {
        const int wl = task / (D / 8);
        const int j = task - wl * (D / 8);
        uint32_t wd[8];
        if (w0 + wl < bi.W) {
          const uint4* src = reinterpret_cast<const uint4*>(pk + static_cast<int64_t>(w0 + wl) * D + 8 * j);
          const uint4 a = src[0], bq = src[1];
          wd[0] = a.x; wd[1] = a.y; wd[2] = a.z; wd[3] = a.w;
          wd[4] = bq.x; wd[5] = bq.y; wd[6] = bq.z; wd[7] = bq.w;
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) wd[u] = 0u;
        }
#pragma unroll
        for (int i = 0; i < CPW; ++i) {
          uint32_t hv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            hv[u] = codes_to_half2((wd[2 * u] >> (BITS * i)) & C::MASK, (wd[2 * u + 1] >> (BITS * i)) & C::MASK);
          tc::sts128(sbase + C::K_T + tc::sw128_offset(wl * CPW + i, 8 * j, KT), hv[0], hv[1], hv[2], hv[3]);
        }
      }
      // ---- unpack V codes: task = (channel c, 8-key chunk kq); rows = channels
      for (int task = tid; task < D * (KT / 8); task += kTcThreads) {
        const int kq = task / D;
        const int c = task - kq * D;
        const int k0 = 8 * kq;
        const int wa = k0 / CPW;
        const int wb = (k0 + 7) / CPW;
        const uint32_t A = (w0 + wa < bi.W) ? pv[static_cast<int64_t>(w0 + wa) * D + c] : 0u;
        const uint32_t Bw = (wb == wa) ? A : ((w0 + wb < bi.W) ? pv[static_cast<int64_t>(w0 + wb) * D + c] : 0u);
        uint32_t cd[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int k = k0 + i;
          const int wr = k / CPW;
          const int slot = k - wr * CPW;
          cd[i] = (((wr == wa) ? A : Bw) >> (BITS * slot)) & C::MASK;
        }
        tc::sts128(sbase + C::V_T + tc::sw128_offset(c, k0, D), codes_to_half2(cd[0], cd[1]),
                   codes_to_half2(cd[2], cd[3]), codes_to_half2(cd[4], cd[5]), codes_to_half2(cd[6], cd[7]));
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();

      // ---- S = q'hi . K^T + q'lo . K^T
      if (tid == 0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          const uint64_t a = tc::sw128_desc(sbase + C::Q_HI + (kk >> 2) * 128 * 128 + koff);
          const uint64_t bd = tc::sw128_desc(sbase + C::K_T + (kk >> 2) * KT * 128 + koff);
          tc::mma_f16_ss(tmem + C::COL_S, a, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          const uint64_t a = tc::sw128_desc(sbase + C::Q_LO + (kk >> 2) * 128 * 128 + koff);
          const uint64_t bd = tc::sw128_desc(sbase + C::K_T + (kk >> 2) * KT * 128 + koff);
          tc::mma_f16_ss(tmem + C::COL_S, a, bd, idesc_qk, 1u);
        }
        tc::commit(&bar[0]);
      }
      ok = __syncthreads_and(mbar_wait_bounded(&bar[0], phase));
      phase ^= 1u;
      tc::fence_after_sync();
      if (!ok) break;

      // ---- softmax of this row's KT logits
      float s[KT];
#pragma unroll
      for (int c16 = 0; c16 < KT; c16 += 16) {
        uint32_t r[16];
        tc::tmem_ld16(tmem + lane_off + C::COL_S + c16, r);
        tc::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) s[c16 + u] = fmaf(__uint_as_float(r[u]), up, bias);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < KT; ++j) {
        if (j >= nkeys) s[j] = -INFINITY;
        mx = fmaxf(mx, s[j]);
      }
      float alpha = 1.0f;
      bool rescale = false;
      if (mx > m_ref + kTau) {
        if (m_ref != -INFINITY) {
          alpha = __expf(m_ref - mx);
          rescale = true;
        }
        m_ref = mx;
      }
      rs *= alpha;
      l_tot *= alpha;
      // rescale U (current block, only if it already holds tiles) and O in TMEM
      if (__any_sync(0xffffffffu, rescale)) {
        if (!first_tile) {
#pragma unroll 1
          for (int c16 = 0; c16 < D; c16 += 16) {
            uint32_t r[16];
            tc::tmem_ld16(tmem + lane_off + C::COL_U + c16, r);
            tc::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u) r[u] = __float_as_uint(__uint_as_float(r[u]) * alpha);
            tc::tmem_st16(tmem + lane_off + C::COL_U + c16, r);
          }
        }
        if (have_o) {
#pragma unroll 1
          for (int c16 = 0; c16 < D; c16 += 16) {
            uint32_t r[16];
            tc::tmem_ld16(tmem + lane_off + C::COL_O + c16, r);
            tc::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u) r[u] = __float_as_uint(__uint_as_float(r[u]) * alpha);
            tc::tmem_st16(tmem + lane_off + C::COL_O + c16, r);
          }
        }
        tc::tmem_wait_st();
      }
      // probabilities, split hi/lo, to shared memory; the row sum uses exactly hi + lo
#pragma unroll
      for (int c8 = 0; c8 < KT; c8 += 8) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float p0 = __expf(s[c8 + 2 * u] - m_ref);
          const float p1 = __expf(s[c8 + 2 * u + 1] - m_ref);
          const __half2 hh = __floats2half2_rn(p0, p1);
          const float2 hf = __half22float2(hh);
          const __half2 ll = __floats2half2_rn(p0 - hf.x, p1 - hf.y);
          const float2 lf = __half22float2(ll);
          rs += (hf.x + lf.x) + (hf.y + lf.y);
          hi[u] = *reinterpret_cast<const uint32_t*>(&hh);
          lo[u] = *reinterpret_cast<const uint32_t*>(&ll);
        }
        const uint32_t off = tc::sw128_offset(row, c8, 128);
        tc::sts128(sbase + C::P_HI + off, hi[0], hi[1], hi[2], hi[3]);
        tc::sts128(sbase + C::P_LO + off, lo[0], lo[1], lo[2], lo[3]);
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();

      // ---- U (+)= Phi . V + Plo . V
      if (tid == 0) {
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          const uint64_t a = tc::sw128_desc(sbase + C::P_HI + (kk >> 2) * 128 * 128 + koff);
          const uint64_t bd = tc::sw128_desc(sbase + C::V_T + (kk >> 2) * D * 128 + koff);
          tc::mma_f16_ss(tmem + C::COL_U, a, bd, idesc_pv, (first_tile && kk == 0) ? 0u : 1u);
        }
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          const uint64_t a = tc::sw128_desc(sbase + C::P_LO + (kk >> 2) * 128 * 128 + koff);
          const uint64_t bd = tc::sw128_desc(sbase + C::V_T + (kk >> 2) * D * 128 + koff);
          tc::mma_f16_ss(tmem + C::COL_U, a, bd, idesc_pv, 1u);
        }
        tc::commit(&bar[0]);
      }
      ok = __syncthreads_and(mbar_wait_bounded(&bar[0], phase));
      phase ^= 1u;
      tc::fence_after_sync();
    }
    if (!ok) break;

    // ---- fold this block: O = O + U (.) sv + rs * zv
#pragma unroll 1
    for (int c16 = 0; c16 < D; c16 += 16) {
      uint32_t u[16], o[16];
      tc::tmem_ld16(tmem + lane_off + C::COL_U + c16, u);
      if (have_o) tc::tmem_ld16(tmem + lane_off + C::COL_O + c16, o);
      tc::tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float base_o = have_o ? __uint_as_float(o[k]) : 0.0f;
        o[k] = __float_as_uint(fmaf(__uint_as_float(u[k]), meta[2 * D + c16 + k], fmaf(rs, meta[3 * D + c16 + k], base_o)));
      }
      tc::tmem_st16(tmem + lane_off + C::COL_O + c16, o);
    }
    tc::tmem_wait_st();
    l_tot += rs;
    rs = 0.0f;
    have_o = true;
  }

  // ---- epilogue: O / l to global memory. The TMEM loads are warp-collective,
  // so every lane takes them; rows past n_q only skip the stores.
  if (ok) {
    const float inv = 1.0f / l_tot;
    const int64_t obase = b * p.o_sb + h * p.o_sh + static_cast<int64_t>(q0 + row) * p.o_st;
#pragma unroll 1
    for (int c16 = 0; c16 < D; c16 += 16) {
      uint32_t o[16];
      tc::tmem_ld16(tmem + lane_off + C::COL_O + c16, o);
      tc::tmem_wait_ld();
      if (!row_valid) continue;
      if (p.out_f32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + obase + c16);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          dst[k] = make_float4(__uint_as_float(o[4 * k]) * inv, __uint_as_float(o[4 * k + 1]) * inv,
                               __uint_as_float(o[4 * k + 2]) * inv, __uint_as_float(o[4 * k + 3]) * inv);
      } else {
        uint32_t bf[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          uint32_t pair = 0;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const uint32_t x = __float_as_uint(__uint_as_float(o[2 * k + u]) * inv);
            const uint32_t r = (x + 0x7fffu + ((x >> 16) & 1u)) >> 16;
            pair |= r << (16 * u);
          }
          bf[k] = pair;
        }
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + obase + c16);
        dst[0] = make_uint4(bf[0], bf[1], bf[2], bf[3]);
        dst[1] = make_uint4(bf[4], bf[5], bf[6], bf[7]);
      }
    }
  }
  // (if a bounded wait gave up, the output stays unwritten and the error word is set)
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int BITS, int D>
cudaError_t launch_attention_tc(const AttnParams& p, cudaStream_t stream) {
  using C = TcCfg<BITS, D>;
  static bool configured[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(attention_tc_kernel<BITS, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  dim3 grid((p.n_q + 127) / 128, p.B * p.H);
  attention_tc_kernel<BITS, D><<<grid, kTcThreads, C::SMEM_ALLOC, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace
}  // namespace vq
