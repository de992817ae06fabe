// Quantize + bit-pack kernel: one decoding block of K and/or V into the
// block-addressed packed cache.
//
// Method ("VAR-Q: Tuning-Free KV Cache Quantization for Visual Autoregressive
// Image and Video Generation", Abstract, paragraph 3): groups along the feature
// (channel) and block axes. Group (b, h, s, c) = the n_s tokens of block s in
// channel c. Asymmetric min/max grid: scale = (max - min) / (2^bits - 1), zero =
// min; codes are bit-packed along tokens, floor(32/bits) per 32-bit word (10 per
// word for INT3, as the KV-memory column of "VAR-Q results data (Tables 2-4)"
// implies).
//
// Design (HBM-bound; ~2 B read + ~0.5 B written per bf16 element):
//   * work unit = (tensor, b, h): an n_s x D slab. A group of P warps (P = 1
//     when the block has thousands of units, up to 16 for a few large ones)
//     owns a unit at a time; groups walk the units with a grid-wide stride.
//     Nothing is staged and no CTA-wide barrier is taken: warp `part` of a
//     group streams its whole word-rows of the slab through registers with
//     16-byte loads (32/V rows per warp load, V = 16-byte vectors per row).
//   * pass 1: packed bf16x2 (or fp32) min/max per lane, kQuantUnroll loads in
//     flight (row indices past the part's end are clamped to its last row,
//     which min/max ignore), then shuffles across the lanes that share a
//     channel vector; with P > 1 the P partials meet in shared memory behind a
//     named barrier of the group. Min/max is exact, so the order of reduction
//     does not matter.
//   * scale/inv: one IEEE division and one IEEE reciprocal per group (every
//     lane computes its own channels' values); for a scale below 2^-100 both
//     d and scale are first multiplied by 2^64 (exact), so 1/scale never
//     overflows and the codes stay the nearest grid levels.
//   * pass 2: the warp re-reads its rows (now in L2), one word-row per lane and
//     vector, all cpw row loads issued first: d = x - min and t = d * inv, each
//     correctly rounded, t clamped to 2^bits - 1 (a subnormal scale can put
//     the max past the top level), then round half to even by adding 1.5*2^23.
//     The rounded value's low mantissa bits are the code. The codes are summed
//     into the word with shifts and a final constant correction, then stored
//     with 128-bit coalesced stores.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tc_ptx.cuh"
#include "vq_device.cuh"
#include "vq_internal.h"

namespace vq {

namespace {

constexpr int kQuantThreads = 512;  // 16 warps
constexpr int kQuantWarps = kQuantThreads / 32;
constexpr int kQuantUnroll = 16;  // pass-1 loads in flight per lane
constexpr uint32_t kRoundMagicBits = 0x4B400000u;  // bits of 1.5 * 2^23
constexpr float kRoundMagic = 12582912.0f;

// 8 bf16 channels of one 16-byte vector.
struct Bf16Vec {
  static constexpr int kCh = 8;
  static constexpr uint32_t kMnInit = 0x7F807F80u, kMxInit = 0xFF80FF80u;
  __device__ static void minmax_init(uint32_t (&mn)[4], uint32_t (&mx)[4], const uint4& v) {
    mn[0] = mx[0] = v.x;
    mn[1] = mx[1] = v.y;
    mn[2] = mx[2] = v.z;
    mn[3] = mx[3] = v.w;
  }
  __device__ static void minmax_acc(uint32_t (&mn)[4], uint32_t (&mx)[4], const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&w[k]);
      __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162*>(&mn[k]);
      __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162*>(&mx[k]);
      lo = __hmin2(lo, a);
      hi = __hmax2(hi, a);
      mn[k] = *reinterpret_cast<uint32_t*>(&lo);
      mx[k] = *reinterpret_cast<uint32_t*>(&hi);
    }
  }
  // channel c of the packed state as float (bf16 -> f32 is exact)
  __device__ static float ch(const uint32_t (&s)[4], int c) {
    const uint32_t w = s[c >> 1];
    return __uint_as_float((c & 1) ? (w & 0xffff0000u) : (w << 16));
  }
  __device__ static float elem(const uint4& v, int c) {
    const uint32_t w = (c >> 1) == 0 ? v.x : (c >> 1) == 1 ? v.y : (c >> 1) == 2 ? v.z : v.w;
    return __uint_as_float((c & 1) ? (w & 0xffff0000u) : (w << 16));
  }
};

// 4 fp32 channels of one 16-byte vector.
struct F32Vec {
  static constexpr int kCh = 4;
  static constexpr uint32_t kMnInit = 0x7F800000u, kMxInit = 0xFF800000u;
  __device__ static void minmax_init(uint32_t (&mn)[4], uint32_t (&mx)[4], const uint4& v) {
    mn[0] = mx[0] = v.x;
    mn[1] = mx[1] = v.y;
    mn[2] = mx[2] = v.z;
    mn[3] = mx[3] = v.w;
  }
  __device__ static void minmax_acc(uint32_t (&mn)[4], uint32_t (&mx)[4], const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = __uint_as_float(w[k]);
      mn[k] = __float_as_uint(fminf(__uint_as_float(mn[k]), a));
      mx[k] = __float_as_uint(fmaxf(__uint_as_float(mx[k]), a));
    }
  }
  __device__ static float ch(const uint32_t (&s)[4], int c) { return __uint_as_float(s[c]); }
  __device__ static float elem(const uint4& v, int c) {
    return __uint_as_float(c == 0 ? v.x : c == 1 ? v.y : c == 2 ? v.z : v.w);
  }
};

// Scale, zero and encode constants of one group from its exact min and max:
// scale = (max - min) / (2^bits - 1) and zero = min (+0 for a zero min), each
// rounded to fp16 when meta16 (one 32-bit metadata pair per group, the codes
// then taken against that stored grid); pre = 2^64 for a scale below 2^-100
// (1/scale would overflow from 2^-128 down: d and scale are both multiplied
// by it, exactly), inv = 1/(scale * pre), nmp = -zero * pre, so that
// d = fma(x, pre, nmp) = RN(x - zero) * pre.
__device__ __forceinline__ void group_params(float mn, float mx, float levels, bool meta16, float& scl, float& zer,
                                             float& inv, float& pre, float& nmp) {
  scl = __fdiv_rn(__fsub_rn(mx, mn), levels);
  zer = __fadd_rn(mn, 0.0f);
  if (meta16) {
    scl = __half2float(__float2half_rn(scl));
    zer = __half2float(__float2half_rn(zer));
  }
  pre = (scl > 0.0f && scl < 0x1p-100f) ? 0x1p64f : 1.0f;
  inv = (scl > 0.0f) ? __frcp_rn(__fmul_rn(scl, pre)) : 0.0f;
  nmp = __fmul_rn(-zer, pre);
}

// Channel pair (2k, 2k+1) of a 16-byte vector as two floats (exact widening).
template <class Vec>
__device__ __forceinline__ uint64_t vec_pair(const uint4& v, int k) {
  return tc::f2pack(Vec::elem(v, 2 * k), Vec::elem(v, 2 * k + 1));
}

// Encode rows 0 .. nvalid-1 of v (one 16-byte channel vector each) into the
// CH words of one word row, code of row i in bits [BITS*i, BITS*i + BITS).
// Every step is one IEEE float32 operation per channel: d = x - zero
// (fma(x, pre, -zero*pre) on the slow path), t = d * inv, on the slow path a
// clamp to [0, 2^BITS - 1], then round half to even by adding 1.5*2^23, whose
// low mantissa bits are the code. The clamp can act only for a subnormal scale
// (always behind a prescale) or fp16 metadata (zero rounded above the min);
// both take the slow path. Without a prescale the
// subtract and the multiply run on channel pairs as packed .rn operations
// (each lane rounded on its own, like the scalar operation); the rounding add
// is scalar.
template <class Vec, int BITS, int CPW>
__device__ __forceinline__ void encode_word_row(const uint4 (&v)[CPW], int nvalid, const float* nmp, const float* inv,
                                                const float* pre, bool tiny, uint32_t* words) {
  constexpr int CH = Vec::kCh;
  constexpr float kLevels = static_cast<float>((1 << BITS) - 1);
  uint32_t acc[CH];
#pragma unroll
  for (int c = 0; c < CH; ++c) acc[c] = 0u;
  uint32_t corr = 0u;
  if (!tiny) {
    uint64_t nm2[CH / 2], iv2[CH / 2];
#pragma unroll
    for (int k = 0; k < CH / 2; ++k) {
      nm2[k] = tc::f2pack(nmp[2 * k], nmp[2 * k + 1]);
      iv2[k] = tc::f2pack(inv[2 * k], inv[2 * k + 1]);
    }
#pragma unroll
    for (int i = 0; i < CPW; ++i) {
      if (i < nvalid) {
        corr += kRoundMagicBits << (BITS * i);
#pragma unroll
        for (int k = 0; k < CH / 2; ++k) {
          // packed d = x - min and t = d * inv; the rounding add stays scalar:
          // a packed multiply followed by a packed add was found contracted
          // into one rounding (codes differed from the oracle)
          const uint64_t t = tc::mul2(tc::add2(vec_pair<Vec>(v[i], k), nm2[k]), iv2[k]);
          acc[2 * k] += __float_as_uint(__fadd_rn(tc::f2lo(t), kRoundMagic)) << (BITS * i);
          acc[2 * k + 1] += __float_as_uint(__fadd_rn(tc::f2hi(t), kRoundMagic)) << (BITS * i);
        }
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < CPW; ++i) {
      if (i < nvalid) {
        corr += kRoundMagicBits << (BITS * i);
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const float d = __fmaf_rn(Vec::elem(v[i], c), pre[c], nmp[c]);
          const float tq = fminf(fmaxf(__fmul_rn(d, inv[c]), 0.0f), kLevels);
          acc[c] += __float_as_uint(__fadd_rn(tq, kRoundMagic)) << (BITS * i);
        }
      }
    }
  }
#pragma unroll
  for (int c = 0; c < CH; ++c) words[c] = acc[c] - corr;
}

__device__ __forceinline__ uint4 ldg128(const unsigned char* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

template <class Vec, int BITS>
__global__ void __launch_bounds__(kQuantThreads, 1) quant_pack_kernel(const __grid_constant__ QuantParams p) {
  constexpr int CPW = 32 / BITS;
  constexpr int CH = Vec::kCh;
  constexpr float kLevels = static_cast<float>((1 << BITS) - 1);
  extern __shared__ __align__(16) float qred[];  // [2][groups][P][2][D]
  const bool META16 = p.meta16 != 0;
  const int D = p.D;
  const int V = p.vecs_per_row;
  const int TL = p.TL;            // lanes per unit (team): a warp takes 32/TL units at once when P == 1
  const int RW = TL / V;          // rows per team load
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int P = p.P;
  const int gpc = kQuantWarps / P;
  const int grp = warp / P;
  const int part = warp - grp * P;
  const int team = lane / TL;
  const int tl = lane - team * TL;
  const int j = tl % V;
  const int rsub = tl / V;
  const int upw = 32 / TL;        // units per group step
  const int BH = p.B * p.H;
  int par = 0;
  // every lane of a warp runs the same rounds (shuffles below use the full
  // warp); a team whose unit is past the end only skips its loads and stores
  for (int u0 = (blockIdx.x * gpc + grp) * upw; u0 < p.units; u0 += gridDim.x * gpc * upw, par ^= 1) {
    const int unit = u0 + team;
    const bool live = unit < p.units;
    const QuantTensor& T = p.t[(live ? unit : u0) / BH];
    const int bh = (live ? unit : u0) % BH;
    const unsigned char* slab =
        static_cast<const unsigned char*>(T.x) + ((bh / p.H) * T.sb + (bh % p.H) * T.sh) * p.esize + j * 16;
    const int64_t rstride = T.st * p.esize;
    const int w0 = part * p.WP, w1 = live ? min(p.W, w0 + p.WP) : w0;
    const int r0 = w0 * CPW, r1 = min(p.n, w1 * CPW);
    uint32_t mn[4], mx[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      mn[k] = Vec::kMnInit;
      mx[k] = Vec::kMxInit;
    }
    // pass 1: rows past r1 re-read row r1-1 (min/max are idempotent), so
    // every load of a batch is issued before any is used
    for (int r = r0 + rsub; r < r1; r += kQuantUnroll * RW) {
      uint4 v[kQuantUnroll];
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u) v[u] = ldg128(slab + min(r + u * RW, r1 - 1) * rstride);
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u) Vec::minmax_acc(mn, mx, v[u]);
    }
    float fmn[CH], fmx[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      fmn[c] = Vec::ch(mn, c);
      fmx[c] = Vec::ch(mx, c);
    }
    for (int off = V; off < TL; off <<= 1) {
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        fmn[c] = fminf(fmn[c], __shfl_xor_sync(0xffffffffu, fmn[c], off));
        fmx[c] = fmaxf(fmx[c], __shfl_xor_sync(0xffffffffu, fmx[c], off));
      }
    }
    if (P > 1) {
      float* rb = qred + ((par * gpc + grp) * P) * 2 * D;
      if (rsub == 0) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          rb[part * 2 * D + CH * j + c] = fmn[c];
          rb[part * 2 * D + D + CH * j + c] = fmx[c];
        }
      }
      asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(32 * P) : "memory");
      for (int q = 0; q < P; ++q) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          fmn[c] = fminf(fmn[c], rb[q * 2 * D + CH * j + c]);
          fmx[c] = fmaxf(fmx[c], rb[q * 2 * D + D + CH * j + c]);
        }
      }
    }
    // pre = 2^64 for a scale below 2^-100 (1/scale would overflow from 2^-128
    // down): d and scale are both multiplied by it, exactly, so the encode
    // behaves as float32 with an unbounded exponent. d = fma(x, pre, -min*pre)
    // = RN(x - min) * pre bit for bit (one rounding of an exactly scaled
    // difference; a difference below 2^-126 is exact).
    float scl[CH], zer[CH], inv[CH], pre[CH], nmp[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      group_params(fmn[c], fmx[c], kLevels, META16, scl[c], zer[c], inv[c], pre[c], nmp[c]);
    }
    if (live && part == 0 && rsub == 0) {
      float* sd = T.scale + static_cast<size_t>(bh) * D + CH * j;
      float* zd = T.zero + static_cast<size_t>(bh) * D + CH * j;
#pragma unroll
      for (int q = 0; q < CH / 4; ++q) {
        reinterpret_cast<float4*>(sd)[q] = make_float4(scl[4 * q], scl[4 * q + 1], scl[4 * q + 2], scl[4 * q + 3]);
        reinterpret_cast<float4*>(zd)[q] = make_float4(zer[4 * q], zer[4 * q + 1], zer[4 * q + 2], zer[4 * q + 3]);
      }
    }
    bool tiny = false;
#pragma unroll
    for (int c = 0; c < CH; ++c) tiny |= (pre[c] != 1.0f);
    tiny = __any_sync(0xffffffffu, tiny) || META16;
    // pass 2: one word-row per lane and vector; every row load issued first
    for (int w = w0 + rsub; w < w1; w += RW) {
      const int tl0 = w * CPW;
      const int nvalid = min(CPW, p.n - tl0);
      uint4 v[CPW];
#pragma unroll
      for (int i = 0; i < CPW; ++i) v[i] = ldg128(slab + (tl0 + min(i, nvalid - 1)) * rstride);
      uint32_t wd[CH];
      encode_word_row<Vec, BITS, CPW>(v, nvalid, nmp, inv, pre, tiny, wd);
      uint32_t* dst = T.packed + (static_cast<size_t>(bh) * p.W + w) * D + CH * j;
#pragma unroll
      for (int q = 0; q < CH / 4; ++q)
        reinterpret_cast<uint4*>(dst)[q] = make_uint4(wd[4 * q], wd[4 * q + 1], wd[4 * q + 2], wd[4 * q + 3]);
    }
  }
}

// ---- ring variant: the slab of each unit is bulk-copied into a shared-memory
// slot, so min/max and the encode both read it from shared memory and HBM sees
// every input byte once. Consumer team t (RG warps) owns NSLOT slots and takes
// every RW-th unit of its CTA; a one-warp team copies its own units, larger
// teams are served by a producer warp (one lane). The team's
// warps split the unit's rows (pass 1) and word rows (pass 2) and merge their
// min/max partials in shared memory behind a named barrier of the team; no
// CTA-wide barrier: full/empty mbarriers per slot, waits bounded.
template <class Vec, int BITS>
__global__ void __launch_bounds__(32 * (1 + kRingMaxWarps), 1) quant_ring_kernel(const __grid_constant__ QuantParams p) {
  constexpr int CPW = 32 / BITS;
  constexpr int CH = Vec::kCh;
  constexpr float kLevels = static_cast<float>((1 << BITS) - 1);
  extern __shared__ __align__(128) unsigned char rsm[];
  const bool META16 = p.meta16 != 0;
  const int RW = p.RW, NS = p.NSLOT;
  uint64_t* full = reinterpret_cast<uint64_t*>(rsm);        // [RW][NS]
  uint64_t* empty = full + kRingMaxWarps * 4;               // [RW][NS]
  unsigned char* slots = rsm + 2 * kRingMaxWarps * 4 * 8;   // [RW][NS][slot_bytes]
  const int RG = p.RG;
  // [RW][2][RG][2][D] min/max partials of the team's warps (double-buffered),
  // then [RW][2] failed-wait marks (unit index + 1 of a wait that timed out)
  float* part = reinterpret_cast<float*>(slots + static_cast<size_t>(RW) * NS * p.slot_bytes);
  volatile int* tfail = reinterpret_cast<volatile int*>(part + static_cast<size_t>(RW) * 2 * RG * 2 * p.D);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = p.B * p.H;
  const int D = p.D, V = p.vecs_per_row;
  const int64_t rowb = static_cast<int64_t>(D) * p.esize;   // bytes of one token row
  if (threadIdx.x == 0) {
    for (int i = 0; i < RW * NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], RG);
    }
    for (int i = 0; i < 2 * RW; ++i) tfail[i] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // Copy of the CTA's k-th unit into slot (k % RW, (k / RW) % NS).
  auto issue = [&](int k) {
    const int u = blockIdx.x + k * gridDim.x;
    const int b = (k % RW) * NS + (k / RW) % NS;
    const QuantTensor& T = p.t[u / BH];
    const int bh = u % BH;
    const unsigned char* src =
        static_cast<const unsigned char*>(T.x) + ((bh / p.H) * T.sb + (bh % p.H) * T.sh) * p.esize;
    unsigned char* dst = slots + static_cast<size_t>(b) * p.slot_bytes;
    const uint32_t bytes = static_cast<uint32_t>(p.n * rowb);
    mbar_arrive_expect_tx(&full[b], bytes);
    if (T.st * p.esize == rowb) {
      bulk_copy_g2s(dst, src, bytes, &full[b]);  // contiguous rows: one copy
    } else {
      for (int r = 0; r < p.n; ++r)
        bulk_copy_g2s(dst + r * rowb, src + r * T.st * p.esize, static_cast<uint32_t>(rowb), &full[b]);
    }
  };
  // Teams of one warp copy their own units (each slot refilled as soon as its
  // warp has left it; measured faster on the 8 KB slabs of many one-warp
  // teams); larger teams are served by warp 0, which refills the slots in
  // unit order.
  const bool self_copy = (RG == 1);
  if (!self_copy && warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      for (int k = 0;; ++k) {
        const int u = blockIdx.x + k * gridDim.x;
        if (u >= p.units) break;
        const int b = (k % RW) * NS + (k / RW) % NS, use = k / (RW * NS);
        if (use > 0 && !mbar_wait_bounded(&empty[b], (use - 1) & 1)) break;
        issue(k);
      }
    }
    return;
  }
  // ------------------------------------------------------------------ consumers
  const int cw = self_copy ? warp : warp - 1;
  const int team = cw / RG, gw = cw - team * RG;
  if (team >= RW) return;
  if (self_copy && lane == 0) {
    for (int q = 0; q < NS; ++q)
      if (blockIdx.x + (team + q * RW) * gridDim.x < p.units) issue(team + q * RW);
  }
  const int j = lane % V;          // 16-byte channel vector of this lane
  const int rsub = lane / V;       // row (or word row) offset of this lane
  const int RL = 32 / V;           // rows (word rows) one warp step covers
  const int r0 = rsub + gw * RL;   // this warp's first row (word row); step RL * RG
  for (int k = team;; k += RW) {
    const int u = blockIdx.x + k * gridDim.x;
    if (u >= p.units) break;
    const int s = (k / RW) % NS, use = k / (RW * NS);
    const int b = team * NS + s;
    const int par = (k / RW) & 1;
    // a team leaves together: with more than one warp, a failed wait is
    // published and every warp of the team stops after the team's barrier
    const bool got = mbar_wait_bounded(&full[b], use & 1);
    if (RG == 1 && !got) break;
    const unsigned char* slab = slots + static_cast<size_t>(b) * p.slot_bytes + j * 16;
    const QuantTensor& T = p.t[u / BH];
    const int bh = u % BH;
    // pass 1: min/max of this lane's rows, 8 loads in flight
    uint32_t mn[4], mx[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      mn[q] = Vec::kMnInit;
      mx[q] = Vec::kMxInit;
    }
    for (int r = got ? r0 : p.n; r < p.n; r += 8 * RL * RG) {
      uint4 v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = lds128(slab + min(r + q * RL * RG, p.n - 1) * rowb);
#pragma unroll
      for (int q = 0; q < 8; ++q) Vec::minmax_acc(mn, mx, v[q]);  // repeats of row n-1 change nothing
    }
    float fmn[CH], fmx[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      fmn[c] = Vec::ch(mn, c);
      fmx[c] = Vec::ch(mx, c);
    }
    for (int off = V; off < 32; off <<= 1) {
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        fmn[c] = fminf(fmn[c], __shfl_xor_sync(0xffffffffu, fmn[c], off));
        fmx[c] = fmaxf(fmx[c], __shfl_xor_sync(0xffffffffu, fmx[c], off));
      }
    }
    if (RG > 1) {
      // the team's partials meet in shared memory (a buffer is written again
      // only after the team's next barrier, which every reader has passed)
      float* pb = part + static_cast<size_t>((team * 2 + par) * RG) * 2 * D;
      if (!got && lane == 0) tfail[team * 2 + par] = k + 1;
      if (rsub == 0) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          pb[gw * 2 * D + CH * j + c] = fmn[c];
          pb[gw * 2 * D + D + CH * j + c] = fmx[c];
        }
      }
      asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(32 * RG) : "memory");
      if (tfail[team * 2 + par] == k + 1) break;
      for (int q = 0; q < RG; ++q) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          fmn[c] = fminf(fmn[c], pb[q * 2 * D + CH * j + c]);
          fmx[c] = fmaxf(fmx[c], pb[q * 2 * D + D + CH * j + c]);
        }
      }
    }
    // scale, zero and encode constants (2^64 prescale of tiny scales, see the
    // streaming kernel)
    float inv[CH], pre[CH], nmp[CH];
    bool tiny = false;
    {
      float scl[CH], zer[CH];
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        group_params(fmn[c], fmx[c], kLevels, META16, scl[c], zer[c], inv[c], pre[c], nmp[c]);
        tiny |= (pre[c] != 1.0f);
      }
      if (rsub == 0 && gw == 0) {
        float* sd = T.scale + static_cast<size_t>(bh) * D + CH * j;
        float* zd = T.zero + static_cast<size_t>(bh) * D + CH * j;
#pragma unroll
        for (int q = 0; q < CH / 4; ++q) {
          reinterpret_cast<float4*>(sd)[q] = make_float4(scl[4 * q], scl[4 * q + 1], scl[4 * q + 2], scl[4 * q + 3]);
          reinterpret_cast<float4*>(zd)[q] = make_float4(zer[4 * q], zer[4 * q + 1], zer[4 * q + 2], zer[4 * q + 3]);
        }
      }
    }
    tiny = __any_sync(0xffffffffu, tiny) || META16;
    // pass 2: word rows of this lane's vector
    for (int w = r0; w < p.W; w += RL * RG) {
      const int t0 = w * CPW;
      const int nvalid = min(CPW, p.n - t0);
      uint4 v[CPW];
#pragma unroll
      for (int i = 0; i < CPW; ++i) v[i] = lds128(slab + (t0 + min(i, nvalid - 1)) * rowb);
      uint32_t wd[CH];
      encode_word_row<Vec, BITS, CPW>(v, nvalid, nmp, inv, pre, tiny, wd);
      uint32_t* dst = T.packed + (static_cast<size_t>(bh) * p.W + w) * D + CH * j;
#pragma unroll
      for (int q = 0; q < CH / 4; ++q)
        reinterpret_cast<uint4*>(dst)[q] = make_uint4(wd[4 * q], wd[4 * q + 1], wd[4 * q + 2], wd[4 * q + 3]);
    }
    __syncwarp();
    if (self_copy) {
      // this warp has left slot b: its unit NS ahead goes in
      if (lane == 0 && blockIdx.x + (k + NS * RW) * gridDim.x < p.units) {
        fence_proxy_async_smem();
        issue(k + NS * RW);
      }
    } else if (lane == 0) {
      mbar_arrive(&empty[b]);
    }
  }
}

size_t quant_ring_smem_bytes(const QuantParams& p) {
  return static_cast<size_t>(2 * kRingMaxWarps * 4 * 8) + static_cast<size_t>(p.RW) * p.NSLOT * p.slot_bytes +
         static_cast<size_t>(p.RW) * 2 * p.RG * 2 * p.D * sizeof(float) + static_cast<size_t>(p.RW) * 2 * sizeof(int);
}

template <class Vec, int BITS>
cudaError_t launch_ring(const QuantParams& p, cudaStream_t stream) {
  auto kern = quant_ring_kernel<Vec, BITS>;
  static int sm_count[kMaxDevices] = {};
  static bool configured[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             2 * kRingMaxWarps * 4 * 8 + kRingSmemBudget + kRingMaxWarps * 2 * 2 * 128 * 4 +
                                 kRingMaxWarps * 2 * 4);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int grid = p.units < sm_count[dev] ? p.units : sm_count[dev];
  // one warp per consumer, plus the producer warp for teams of several warps
  kern<<<grid, 32 * (p.RW * p.RG + (p.RG == 1 ? 0 : 1)), quant_ring_smem_bytes(p), stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

// One warp quantizes one unit (one tensor's n x D slab of one (batch, head)):
// the streaming kernel's steps with the whole warp on the unit, for the fused
// append+attention launches, whose CTAs quantize their own (batch, head) before
// attending. slab: the slab's first row; rstride: bytes between rows; packed:
// the unit's [W][D] words; scale, zero: its [D] vectors.
template <class Vec, int BITS>
__device__ void quantize_unit_warp(const unsigned char* slab, int64_t rstride, int n, int W, int D,
                                   uint32_t* packed, float* scale, float* zero, bool META16, int lane) {
  constexpr int CPW = 32 / BITS;
  constexpr int CH = Vec::kCh;
  constexpr float kLevels = static_cast<float>((1 << BITS) - 1);
  const int V = D / CH;        // 16-byte vectors per row
  const int RL = 32 / V;       // rows per warp load
  const int j = lane % V;
  const int rsub = lane / V;
  slab += j * 16;
  uint32_t mn[4], mx[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    mn[k] = Vec::kMnInit;
    mx[k] = Vec::kMxInit;
  }
  for (int r = rsub; r < n; r += kQuantUnroll * RL) {
    uint4 v[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) v[u] = ldg128(slab + min(r + u * RL, n - 1) * rstride);
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) Vec::minmax_acc(mn, mx, v[u]);  // repeats of row n-1 change nothing
  }
  float fmn[CH], fmx[CH];
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    fmn[c] = Vec::ch(mn, c);
    fmx[c] = Vec::ch(mx, c);
  }
  for (int off = V; off < 32; off <<= 1) {
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      fmn[c] = fminf(fmn[c], __shfl_xor_sync(0xffffffffu, fmn[c], off));
      fmx[c] = fmaxf(fmx[c], __shfl_xor_sync(0xffffffffu, fmx[c], off));
    }
  }
  float scl[CH], zer[CH], inv[CH], pre[CH], nmp[CH];
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    group_params(fmn[c], fmx[c], kLevels, META16, scl[c], zer[c], inv[c], pre[c], nmp[c]);
  }
  bool tiny = false;
#pragma unroll
  for (int c = 0; c < CH; ++c) tiny |= (pre[c] != 1.0f);
  tiny = __any_sync(0xffffffffu, tiny) || META16;
  if (rsub == 0) {
#pragma unroll
    for (int q = 0; q < CH / 4; ++q) {
      reinterpret_cast<float4*>(scale + CH * j)[q] = make_float4(scl[4 * q], scl[4 * q + 1], scl[4 * q + 2], scl[4 * q + 3]);
      reinterpret_cast<float4*>(zero + CH * j)[q] = make_float4(zer[4 * q], zer[4 * q + 1], zer[4 * q + 2], zer[4 * q + 3]);
    }
  }
  for (int w = rsub; w < W; w += RL) {
    const int t0 = w * CPW;
    const int nvalid = min(CPW, n - t0);
    uint4 v[CPW];
#pragma unroll
    for (int i = 0; i < CPW; ++i) v[i] = ldg128(slab + (t0 + min(i, nvalid - 1)) * rstride);
    uint32_t wd[CH];
    encode_word_row<Vec, BITS, CPW>(v, nvalid, nmp, inv, pre, tiny, wd);
    uint32_t* dst = packed + static_cast<size_t>(w) * D + CH * j;
#pragma unroll
    for (int q = 0; q < CH / 4; ++q)
      reinterpret_cast<uint4*>(dst)[q] = make_uint4(wd[4 * q], wd[4 * q + 1], wd[4 * q + 2], wd[4 * q + 3]);
  }
}

namespace {

template <class Vec, int BITS>
cudaError_t launch_typed(const QuantParams& p, cudaStream_t stream) {
  auto kern = quant_pack_kernel<Vec, BITS>;
  static int sm_count[kMaxDevices] = {};
  static bool configured[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(quant_smem_bytes(128)));
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int gpc = kQuantWarps / p.P;
  const int per_cta = gpc * (32 / p.TL);
  const int ctas = (p.units + per_cta - 1) / per_cta;
  const int grid = ctas < sm_count[dev] ? ctas : sm_count[dev];
  kern<<<grid, kQuantThreads, p.P > 1 ? quant_smem_bytes(p.D) : 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t quant_smem_bytes(int D) { return static_cast<size_t>(2) * kQuantWarps * 2 * D * sizeof(float); }

int quant_warps() { return kQuantWarps; }

cudaError_t launch_quant_pack(const QuantParams& p, cudaStream_t stream) {
  const bool bf16 = (p.esize == 2);
#define VQ_QP_CASE(B)                                                                         \
  case B:                                                                                     \
    if (p.ring) return bf16 ? launch_ring<Bf16Vec, B>(p, stream) : launch_ring<F32Vec, B>(p, stream); \
    return bf16 ? launch_typed<Bf16Vec, B>(p, stream) : launch_typed<F32Vec, B>(p, stream);
  switch (p.bits) {
    VQ_QP_CASE(2)
    VQ_QP_CASE(3)
    VQ_QP_CASE(4)
    VQ_QP_CASE(6)
    VQ_QP_CASE(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef VQ_QP_CASE
}

}  // namespace vq
