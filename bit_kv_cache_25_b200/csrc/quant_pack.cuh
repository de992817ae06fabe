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
#include <cuda_runtime.h>

#include <cstdint>

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

__device__ __forceinline__ uint4 ldg128(const unsigned char* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

template <class Vec, int BITS>
__global__ void __launch_bounds__(kQuantThreads, 1) quant_pack_kernel(const __grid_constant__ QuantParams p) {
  constexpr int CPW = 32 / BITS;
  constexpr int CH = Vec::kCh;
  constexpr float kLevels = static_cast<float>((1 << BITS) - 1);
  extern __shared__ __align__(16) float qred[];  // [2][groups][P][2][D]
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
      scl[c] = __fdiv_rn(__fsub_rn(fmx[c], fmn[c]), kLevels);
      zer[c] = __fadd_rn(fmn[c], 0.0f);
      pre[c] = (scl[c] > 0.0f && scl[c] < 0x1p-100f) ? 0x1p64f : 1.0f;
      inv[c] = (scl[c] > 0.0f) ? __frcp_rn(__fmul_rn(scl[c], pre[c])) : 0.0f;
      nmp[c] = __fmul_rn(-fmn[c], pre[c]);
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
    // pass 2: one word-row per lane and vector; every row load issued first
    for (int w = w0 + rsub; w < w1; w += RW) {
      const int tl0 = w * CPW;
      const int nvalid = min(CPW, p.n - tl0);
      uint4 v[CPW];
#pragma unroll
      for (int i = 0; i < CPW; ++i) v[i] = ldg128(slab + (tl0 + min(i, nvalid - 1)) * rstride);
      uint32_t acc[CH];
#pragma unroll
      for (int c = 0; c < CH; ++c) acc[c] = 0u;
      uint32_t corr = 0u;
#pragma unroll
      for (int i = 0; i < CPW; ++i) {
        if (i < nvalid) {
          corr += kRoundMagicBits << (BITS * i);
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            const float d = __fmaf_rn(Vec::elem(v[i], c), pre[c], nmp[c]);
            const float t = fminf(__fmul_rn(d, inv[c]), kLevels);
            const float rq = __fadd_rn(t, kRoundMagic);
            acc[c] += __float_as_uint(rq) << (BITS * i);
          }
        }
      }
      uint32_t* dst = T.packed + (static_cast<size_t>(bh) * p.W + w) * D + CH * j;
#pragma unroll
      for (int q = 0; q < CH / 4; ++q)
        reinterpret_cast<uint4*>(dst)[q] =
            make_uint4(acc[4 * q] - corr, acc[4 * q + 1] - corr, acc[4 * q + 2] - corr, acc[4 * q + 3] - corr);
    }
  }
}

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

// ---- register-resident variant: every input byte is loaded once.
// A task is one word row of one 16-byte channel vector (cpw rows x 16 bytes).
// A team of TT threads owns a unit; thread i holds tasks i, i + TT*C, ... (at
// most R) in registers, all loads issued before the first use. Teams of up to
// 32 threads live inside one warp (32 / TT units per warp); larger teams sync
// on a named barrier; a unit larger than one CTA is split over a cluster of C
// CTAs whose min/max meet in distributed shared memory. The group statistics
// then come from the registers, so the encode needs no second read.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float ld_dsmem_f32(const float* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

template <class Vec, int BITS>
struct QReg {
  static constexpr int CPW = 32 / BITS;
  static constexpr int CH = Vec::kCh;
  static constexpr int R = quant_reg_tasks(BITS);
  // the next unit's rows are loaded while this unit is encoded when two sets
  // of input registers fit (at most 40 registers each)
  static constexpr int PF = (R * CPW * 4 <= 40) ? 2 : 1;
  using Rows = uint4[R][CPW];
};

// Team-wide encode constants of one channel: inv = 1/(scale * pre),
// pre = 2^64 for a scale below 2^-100 (else 1), nmp = -min * pre.
__device__ __forceinline__ void qreg_params(float mn, float mx, float levels, float& scl, float& zer, float& inv,
                                            float& pre, float& nmp) {
  scl = __fdiv_rn(__fsub_rn(mx, mn), levels);
  zer = __fadd_rn(mn, 0.0f);
  pre = (scl > 0.0f && scl < 0x1p-100f) ? 0x1p64f : 1.0f;
  inv = (scl > 0.0f) ? __frcp_rn(__fmul_rn(scl, pre)) : 0.0f;
  nmp = __fmul_rn(-mn, pre);
}

template <class Vec, int BITS>
__global__ void __launch_bounds__(kQuantRegThreads, 1) quant_reg_kernel(const __grid_constant__ QuantParams p) {
  using Q = QReg<Vec, BITS>;
  constexpr int CPW = Q::CPW;
  constexpr int CH = Q::CH;
  constexpr int R = Q::R;
  constexpr float kLevels = static_cast<float>((1 << BITS) - 1);
  // shared memory: red [16 warps][2][D] partials, cred [2][2][D] per-CTA
  // partials read by the cluster, prm [8 teams][3][D] encode constants, and
  // per unit parity and team a "some group needs the prescale" flag
  extern __shared__ __align__(16) float qsm[];
  const int D = p.D;
  const int V = p.vecs_per_row;
  const int TT = p.TT;
  const int C = p.C;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int team = tid / TT;
  const int i = tid - team * TT;
  const int teams = kQuantRegThreads / TT;
  const int j = i % V;
  const int rank = (C > 1) ? static_cast<int>(cluster_rank()) : 0;
  const int cl = blockIdx.x / C, ncl = gridDim.x / C;
  const int tasks = p.W * V;
  const int tstride = TT * C;
  const int tfirst = rank * TT + i;
  const int BH = p.B * p.H;
  const int span = min(TT, 32);
  const int G = span / V;              // lanes of one team warp that share vector j
  const int kk = i / V;                // this lane's index among them (TT <= 32)
  float* red = qsm;                                  // [16][2][D]
  float* cred = red + 16 * 2 * D;                    // [2][2][D]
  float* prm = cred + 2 * 2 * D;                     // [8][3][D]
  int* tiny = reinterpret_cast<int*>(prm + 8 * 3 * D);  // [2][8]
  const int rstep = ncl * teams;

  auto unit_of = [&](int r0, int& bh, const QuantTensor*& T) -> bool {
    const int unit = r0 + team;
    const bool live = unit < p.units;
    T = &p.t[(live ? unit : r0) / BH];
    bh = (live ? unit : r0) % BH;
    return live;
  };
  // issue every load of this thread's tasks of round r0 (a thread without a
  // task reads row 0 of a valid slab for its first task and ignores it)
  auto load = [&](int r0, uint4 (&v)[R][CPW]) {
    int bh;
    const QuantTensor* T;
    const bool live = unit_of(r0, bh, T);
    const unsigned char* slab =
        static_cast<const unsigned char*>(T->x) + ((bh / p.H) * T->sb + (bh % p.H) * T->sh) * p.esize + j * 16;
    const int64_t rstride = T->st * p.esize;
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int t = tfirst + k * tstride;
      const bool has = live && t < tasks;
      const int w = has ? t / V : 0;
      if (k == 0 || has) {
#pragma unroll
        for (int c2 = 0; c2 < CPW; ++c2) v[k][c2] = ldg128(slab + min(w * CPW + c2, p.n - 1) * rstride);
      }
    }
  };
  auto process = [&](int r0, const uint4 (&v)[R][CPW], int par) {
    int bh;
    const QuantTensor* T;
    const bool live = unit_of(r0, bh, T);
    uint32_t mn[4], mx[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      mn[k] = Vec::kMnInit;
      mx[k] = Vec::kMxInit;
    }
#pragma unroll
    for (int k = 0; k < R; ++k) {
      if (live && tfirst + k * tstride < tasks) {
#pragma unroll
        for (int c2 = 0; c2 < CPW; ++c2) Vec::minmax_acc(mn, mx, v[k][c2]);  // rows past n repeat row n-1
      }
    }
    float fmn[CH], fmx[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      fmn[c] = Vec::ch(mn, c);
      fmx[c] = Vec::ch(mx, c);
    }
    for (int off = V; off < span; off <<= 1) {
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        fmn[c] = fminf(fmn[c], __shfl_xor_sync(0xffffffffu, fmn[c], off));
        fmx[c] = fmaxf(fmx[c], __shfl_xor_sync(0xffffffffu, fmx[c], off));
      }
    }
    // encode constants of this thread's CH channels
    float inv[CH], nmp[CH], pre[CH];
    bool any_tiny;
    if (TT <= 32) {
      // the G lanes of vector j split its channels: channel c is owned by lane
      // kk == c % G, which also writes its scale and zero
      bool t_own = false;
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        float scl, zer, iv, pr, nm;
        if (c % G == kk) {
          qreg_params(fmn[c], fmx[c], kLevels, scl, zer, iv, pr, nm);
          t_own |= (pr != 1.0f);
          if (live) {
            T->scale[static_cast<size_t>(bh) * D + CH * j + c] = scl;
            T->zero[static_cast<size_t>(bh) * D + CH * j + c] = zer;
          }
        } else {
          iv = pr = nm = 0.0f;
        }
        const int src = (lane - kk * V) + (c % G) * V;  // owner lane of channel c in this warp
        inv[c] = __shfl_sync(0xffffffffu, iv, src);
        pre[c] = __shfl_sync(0xffffffffu, pr, src);
        nmp[c] = __shfl_sync(0xffffffffu, nm, src);
      }
      any_tiny = __any_sync(0xffffffffu, t_own);
    } else {
      const int nw = TT / 32;
      const int wt = i >> 5;
      float* rb = red + (team * nw) * 2 * D;
      if (lane < V) {
#pragma unroll
        for (int q = 0; q < CH / 4; ++q) {
          reinterpret_cast<float4*>(rb + wt * 2 * D + CH * j)[q] =
              make_float4(fmn[4 * q], fmn[4 * q + 1], fmn[4 * q + 2], fmn[4 * q + 3]);
          reinterpret_cast<float4*>(rb + wt * 2 * D + D + CH * j)[q] =
              make_float4(fmx[4 * q], fmx[4 * q + 1], fmx[4 * q + 2], fmx[4 * q + 3]);
        }
      }
      float* pm = prm + team * 3 * D;
      if (C > 1) {
        __syncthreads();
        if (tid < D) {
          float a = INFINITY, b = -INFINITY;
          for (int q = 0; q < nw; ++q) {
            a = fminf(a, rb[q * 2 * D + tid]);
            b = fmaxf(b, rb[q * 2 * D + D + tid]);
          }
          cred[(par * 2) * D + tid] = a;
          cred[(par * 2 + 1) * D + tid] = b;
        }
        cluster_sync();
        // the flag of the other parity was last read before this unit's first
        // barrier and is next set after the next unit's: clear it here
        if (tid == 0) tiny[(par ^ 1) * 8] = 0;
        if (tid < D) {
          float a = INFINITY, b = -INFINITY;
          for (int q = 0; q < C; ++q) {
            a = fminf(a, ld_dsmem_f32(cred + (par * 2) * D + tid, q));
            b = fmaxf(b, ld_dsmem_f32(cred + (par * 2 + 1) * D + tid, q));
          }
          float scl, zer, iv, pr, nm;
          qreg_params(a, b, kLevels, scl, zer, iv, pr, nm);
          pm[tid] = iv;
          pm[D + tid] = pr;
          pm[2 * D + tid] = nm;
          if (pr != 1.0f) tiny[par * 8 + team] = 1;
          if (live && rank == 0) {
            T->scale[static_cast<size_t>(bh) * D + tid] = scl;
            T->zero[static_cast<size_t>(bh) * D + tid] = zer;
          }
        }
        __syncthreads();
      } else {
        asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(TT) : "memory");
        if (i == 0) tiny[(par ^ 1) * 8 + team] = 0;  // see the cluster branch
        for (int c = i; c < D; c += TT) {
          float a = INFINITY, b = -INFINITY;
          for (int q = 0; q < nw; ++q) {
            a = fminf(a, rb[q * 2 * D + c]);
            b = fmaxf(b, rb[q * 2 * D + D + c]);
          }
          float scl, zer, iv, pr, nm;
          qreg_params(a, b, kLevels, scl, zer, iv, pr, nm);
          pm[c] = iv;
          pm[D + c] = pr;
          pm[2 * D + c] = nm;
          if (pr != 1.0f) tiny[par * 8 + team] = 1;
          if (live) {
            T->scale[static_cast<size_t>(bh) * D + c] = scl;
            T->zero[static_cast<size_t>(bh) * D + c] = zer;
          }
        }
        asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(TT) : "memory");
      }
      any_tiny = tiny[par * 8 + team] != 0;
#pragma unroll
      for (int q = 0; q < CH / 4; ++q) {
        const float4 a = reinterpret_cast<const float4*>(pm + CH * j)[q];
        const float4 b = reinterpret_cast<const float4*>(pm + D + CH * j)[q];
        const float4 c4 = reinterpret_cast<const float4*>(pm + 2 * D + CH * j)[q];
        inv[4 * q] = a.x, inv[4 * q + 1] = a.y, inv[4 * q + 2] = a.z, inv[4 * q + 3] = a.w;
        pre[4 * q] = b.x, pre[4 * q + 1] = b.y, pre[4 * q + 2] = b.z, pre[4 * q + 3] = b.w;
        nmp[4 * q] = c4.x, nmp[4 * q + 1] = c4.y, nmp[4 * q + 2] = c4.z, nmp[4 * q + 3] = c4.w;
      }
    }
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int t = tfirst + k * tstride;
      if (live && t < tasks) {
        const int w = t / V;
        const int nvalid = min(CPW, p.n - w * CPW);
        uint32_t acc[CH];
#pragma unroll
        for (int c = 0; c < CH; ++c) acc[c] = 0u;
        uint32_t corr = 0u;
        if (!any_tiny) {
          // d = x - min: fma(x, 1, -min) is the same single rounding
#pragma unroll
          for (int c2 = 0; c2 < CPW; ++c2) {
            if (c2 < nvalid) {
              corr += kRoundMagicBits << (BITS * c2);
#pragma unroll
              for (int c = 0; c < CH; ++c) {
                const float d = __fadd_rn(Vec::elem(v[k][c2], c), nmp[c]);
                const float tq = fminf(__fmul_rn(d, inv[c]), kLevels);
                acc[c] += __float_as_uint(__fadd_rn(tq, kRoundMagic)) << (BITS * c2);
              }
            }
          }
        } else {
#pragma unroll
          for (int c2 = 0; c2 < CPW; ++c2) {
            if (c2 < nvalid) {
              corr += kRoundMagicBits << (BITS * c2);
#pragma unroll
              for (int c = 0; c < CH; ++c) {
                const float d = __fmaf_rn(Vec::elem(v[k][c2], c), pre[c], nmp[c]);
                const float tq = fminf(__fmul_rn(d, inv[c]), kLevels);
                acc[c] += __float_as_uint(__fadd_rn(tq, kRoundMagic)) << (BITS * c2);
              }
            }
          }
        }
        uint32_t* dst = T->packed + (static_cast<size_t>(bh) * p.W + w) * D + CH * j;
#pragma unroll
        for (int q = 0; q < CH / 4; ++q)
          reinterpret_cast<uint4*>(dst)[q] =
              make_uint4(acc[4 * q] - corr, acc[4 * q + 1] - corr, acc[4 * q + 2] - corr, acc[4 * q + 3] - corr);
      }
    }
  };

  if (tid < 16) tiny[tid] = 0;
  __syncthreads();
  // every thread of the CTA runs the same rounds (shuffles, barriers); the next
  // round's loads are issued before this round is processed
  int r0 = cl * teams;
  if (r0 < p.units) {
    if constexpr (Q::PF == 2) {
      uint4 va[R][CPW], vb[R][CPW];
      int par = 0;
      load(r0, va);
      while (true) {
        const int r1 = r0 + rstep;
        if (r1 < p.units) load(r1, vb);
        process(r0, va, par);
        par ^= 1;
        if (r1 >= p.units) break;
        const int r2 = r1 + rstep;
        if (r2 < p.units) load(r2, va);
        process(r1, vb, par);
        par ^= 1;
        if (r2 >= p.units) break;
        r0 = r2;
      }
    } else {
      uint4 va[R][CPW];
      int par = 0;
      for (; r0 < p.units; r0 += rstep, par ^= 1) {
        load(r0, va);
        process(r0, va, par);
      }
    }
  }
  // no CTA of a cluster may leave while another can still read its shared memory
  if (C > 1) cluster_sync();
}

size_t quant_reg_smem_bytes(int D) {
  return static_cast<size_t>(16 * 2 * D + 2 * 2 * D + 8 * 3 * D) * sizeof(float) + 16 * sizeof(int);
}

template <class Vec, int BITS>
cudaError_t launch_reg(const QuantParams& p, cudaStream_t stream) {
  auto kern = quant_reg_kernel<Vec, BITS>;
  static int sm_count[kMaxDevices] = {};
  static bool configured[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(quant_reg_smem_bytes(128)));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const size_t smem = quant_reg_smem_bytes(p.D);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(kQuantRegThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  if (p.C > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(p.C, 1, 1);
    int max_clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg);
    if (e != cudaSuccess || max_clusters < 1) {
      cudaGetLastError();  // clear a sticky-free query error; the streaming kernel takes the unit
      return launch_typed<Vec, BITS>(p, stream);
    }
    const int clusters = p.units < max_clusters ? p.units : max_clusters;
    cfg.gridDim = dim3(clusters * p.C, 1, 1);
  } else {
    const int teams = kQuantRegThreads / p.TT;
    const int ctas = (p.units + teams - 1) / teams;
    cfg.gridDim = dim3(ctas < sm_count[dev] ? ctas : sm_count[dev], 1, 1);
  }
  e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

size_t quant_smem_bytes(int D) { return static_cast<size_t>(2) * kQuantWarps * 2 * D * sizeof(float); }

int quant_warps() { return kQuantWarps; }

cudaError_t launch_quant_pack(const QuantParams& p, cudaStream_t stream) {
  const bool bf16 = (p.esize == 2);
#define VQ_QP_CASE(B)                                                                          \
  case B:                                                                                      \
    if (p.reg) return bf16 ? launch_reg<Bf16Vec, B>(p, stream) : launch_reg<F32Vec, B>(p, stream); \
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
