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
//   * work unit = (tensor, b, h): an n_s x D slab. A CTA stages whole slabs
//     (several small ones) or a chunk of word-rows of one large slab in shared
//     memory with 1-D bulk async copies (one per slab chunk when tokens are
//     contiguous). Large slabs are split over a thread-block cluster of up to
//     16 CTAs. The partial per-channel min/max are exchanged through
//     distributed shared memory, so HBM is read exactly once.
//   * task = (word-row w, 16-byte vector j of a row): a thread reads the cpw
//     rows of word-row w at vector j, i.e. 8 bf16 (or 4 fp32) channels.
//     Shared-memory reads are 128-bit, each quarter-warp on one contiguous
//     128-byte span, which is bank-conflict free.
//   * pass 1: per-task min/max (packed bf16x2 min/max for bf16), then integer
//     atomics on order-preserving keys into per-(unit, channel) shared slots.
//     Min/max is exact, so the order of reduction does not matter.
//   * scale/inv: one IEEE division and one IEEE reciprocal per group.
//   * pass 2: d = x - min and t = d * inv, each correctly rounded (no FMA
//     contraction), then round half to even by adding 1.5*2^23. The rounded
//     value's low mantissa bits are the code (t <= 2^bits - 1 + tiny, so no
//     clamp is needed). The codes are summed into the word with shifts and a
//     final constant correction, then stored with 128-bit coalesced stores.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "vq_device.cuh"
#include "vq_internal.h"

namespace vq {

namespace {

constexpr int kQuantThreads = 256;
constexpr uint32_t kRoundMagicBits = 0x4B400000u;  // bits of 1.5 * 2^23
constexpr float kRoundMagic = 12582912.0f;

struct QuantSmem {
  // layout inside dynamic shared memory (byte offsets)
  uint32_t bar, mnk, mxk, mn, inv, stage;
  uint32_t total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline QuantSmem quant_smem_layout(int G, int D, int rows_chunk, int rowbytes) {
  QuantSmem L;
  L.bar = 0;
  L.mnk = 16;
  L.mxk = L.mnk + 4u * G * D;
  L.mn = L.mxk + 4u * G * D;
  L.inv = L.mn + 4u * G * D;
  L.stage = align_up(L.inv + 4u * G * D, 128);
  L.total = L.stage + static_cast<uint32_t>(G) * rows_chunk * rowbytes;
  return L;
}

// 8 bf16 channels of one 16-byte vector.
struct Bf16Vec {
  static constexpr int kCh = 8;
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

template <class Vec, int BITS>
__global__ void __launch_bounds__(kQuantThreads) quant_pack_kernel(const __grid_constant__ QuantParams p) {
  constexpr int CPW = 32 / BITS;
  constexpr int CH = Vec::kCh;
  extern __shared__ __align__(128) unsigned char smem[];

  const int D = p.D;
  const int V = p.vecs_per_row;
  const int rowbytes = V * 16;
  const int rows_chunk = p.rows_chunk;
  const QuantSmem L = quant_smem_layout(p.G, D, rows_chunk, rowbytes);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L.bar);
  int32_t* mnk = reinterpret_cast<int32_t*>(smem + L.mnk);
  int32_t* mxk = reinterpret_cast<int32_t*>(smem + L.mxk);
  float* s_mn = reinterpret_cast<float*>(smem + L.mn);
  float* s_inv = reinterpret_cast<float*>(smem + L.inv);
  unsigned char* stage = smem + L.stage;

  const int C = p.C;
  const uint32_t rank = (C > 1) ? cluster_ctarank() : 0u;
  const int cta_unit0 = (C > 1) ? static_cast<int>(blockIdx.x) / C : static_cast<int>(blockIdx.x) * p.G;
  const int wr0 = static_cast<int>(rank) * p.wr_chunk;   // first word-row of this CTA's chunk
  const int row0 = wr0 * CPW;                            // first token of the chunk
  const int G = p.G;
  const int n = p.n;
  const int BH = p.B * p.H;
  const int tid = threadIdx.x;

  // number of this CTA's units that exist (the last CTA may be partial)
  const int units_here = min(G, p.units - cta_unit0);
  const int wr_here = max(0, min(p.wr_chunk, p.W - wr0));
  const int rows_here = max(0, min(rows_chunk, n - row0));

  // ---- stage the slab chunks in shared memory
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  for (int i = tid; i < G * D; i += blockDim.x) {
    mnk[i] = INT32_MAX;
    mxk[i] = INT32_MIN;
  }
  __syncthreads();

  if (tid < 32) {
    const uint32_t total = static_cast<uint32_t>(units_here) * rows_here * rowbytes;
    if (tid == 0) mbar_arrive_expect_tx(bar, total);
    __syncwarp();
    if (rows_here > 0) {
      for (int g = 0; g < units_here; ++g) {
        const int unit = cta_unit0 + g;
        const int tsel = unit / BH;
        const int bh = unit % BH;
        const QuantTensor& T = p.t[tsel];
        const int64_t base = (bh / p.H) * T.sb + (bh % p.H) * T.sh;
        const unsigned char* src = static_cast<const unsigned char*>(T.x) + (base + int64_t(row0) * T.st) * p.esize;
        unsigned char* dst = stage + static_cast<size_t>(g) * rows_chunk * rowbytes;
        if (T.st * p.esize == rowbytes) {
          if (tid == 0) bulk_copy_g2s(dst, src, static_cast<uint32_t>(rows_here) * rowbytes, bar);
        } else {
          for (int r = tid; r < rows_here; r += 32)
            bulk_copy_g2s(dst + r * rowbytes, src + int64_t(r) * T.st * p.esize, rowbytes, bar);
        }
      }
    }
  }
  const bool staged = mbar_wait_bounded(bar, 0);

  // ---- pass 1: per-channel min/max
  const int tasks_per_unit = wr_here * V;
  const int ntask = units_here * tasks_per_unit;
  if (staged) {
    for (int task = tid; task < ntask; task += blockDim.x) {
      const int g = task / tasks_per_unit;
      const int r = task - g * tasks_per_unit;
      const int wl = r / V;
      const int j = r - wl * V;
      const int tl0 = wl * CPW;
      const int nvalid = min(CPW, rows_here - tl0);
      const unsigned char* src = stage + (static_cast<size_t>(g) * rows_chunk + tl0) * rowbytes + j * 16;
      uint32_t mn[4], mx[4];
      Vec::minmax_init(mn, mx, lds128(src));
#pragma unroll
      for (int i = 1; i < CPW; ++i)
        if (i < nvalid) Vec::minmax_acc(mn, mx, lds128(src + i * rowbytes));
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        atomicMin(&mnk[g * D + j * CH + c], float_key(Vec::ch(mn, c)));
        atomicMax(&mxk[g * D + j * CH + c], float_key(Vec::ch(mx, c)));
      }
    }
  }
  __syncthreads();

  // ---- combine across the cluster (one unit per cluster)
  int32_t fmn = 0, fmx = 0;
  if (C > 1) {
    cluster_sync();  // every CTA's partials are complete and visible
    if (tid < D) {
      fmn = INT32_MAX;
      fmx = INT32_MIN;
      for (int r = 0; r < C; ++r) {
        fmn = min(fmn, dsmem_ld_s32(&mnk[tid], r));
        fmx = max(fmx, dsmem_ld_s32(&mxk[tid], r));
      }
    }
    cluster_arrive();  // done reading peers; the matching wait is at the end
  }

  // ---- per-group scale, zero, reciprocal
  for (int i = tid; i < units_here * D; i += blockDim.x) {
    const int32_t kmn = (C > 1) ? fmn : mnk[i];
    const int32_t kmx = (C > 1) ? fmx : mxk[i];
    const float mn = key_float(kmn);
    const float mx = key_float(kmx);
    const float diff = __fsub_rn(mx, mn);
    const float scale = __fdiv_rn(diff, static_cast<float>((1 << BITS) - 1));
    const float zero = __fadd_rn(mn, 0.0f);
    const float inv = (scale > 0.0f) ? fminf(__frcp_rn(scale), FLT_MAX) : 0.0f;
    s_mn[i] = mn;
    s_inv[i] = inv;
    if (rank == 0 && staged) {
      const int g = i / D;
      const int c = i - g * D;
      const int unit = cta_unit0 + g;
      const QuantTensor& T = p.t[unit / BH];
      const int bh = unit % BH;
      T.scale[static_cast<size_t>(bh) * D + c] = scale;
      T.zero[static_cast<size_t>(bh) * D + c] = zero;
    }
  }
  __syncthreads();

  // ---- pass 2: encode and pack
  if (staged) {
    for (int task = tid; task < ntask; task += blockDim.x) {
      const int g = task / tasks_per_unit;
      const int r = task - g * tasks_per_unit;
      const int wl = r / V;
      const int j = r - wl * V;
      const int tl0 = wl * CPW;
      const int nvalid = min(CPW, rows_here - tl0);
      const unsigned char* src = stage + (static_cast<size_t>(g) * rows_chunk + tl0) * rowbytes + j * 16;
      float mn[CH], inv[CH];
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        mn[c] = s_mn[g * D + j * CH + c];
        inv[c] = s_inv[g * D + j * CH + c];
      }
      uint32_t acc[CH];
#pragma unroll
      for (int c = 0; c < CH; ++c) acc[c] = 0u;
      uint32_t corr = 0u;
#pragma unroll
      for (int i = 0; i < CPW; ++i) {
        if (i < nvalid) {
          const uint4 v = lds128(src + i * rowbytes);
          corr += kRoundMagicBits << (BITS * i);
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            const float d = __fsub_rn(Vec::elem(v, c), mn[c]);
            const float t = __fmul_rn(d, inv[c]);
            const float rq = __fadd_rn(t, kRoundMagic);
            acc[c] += __float_as_uint(rq) << (BITS * i);
          }
        }
      }
      const int unit = cta_unit0 + g;
      const QuantTensor& T = p.t[unit / BH];
      const int bh = unit % BH;
      uint32_t* dst = T.packed + (static_cast<size_t>(bh) * p.W + wr0 + wl) * D + j * CH;
#pragma unroll
      for (int q = 0; q < CH / 4; ++q)
        reinterpret_cast<uint4*>(dst)[q] =
            make_uint4(acc[4 * q] - corr, acc[4 * q + 1] - corr, acc[4 * q + 2] - corr, acc[4 * q + 3] - corr);
    }
  }

  if (C > 1) cluster_wait();  // peers may still read this CTA's partials until here
}

template <class Vec, int BITS>
cudaError_t launch_typed(const QuantParams& p, cudaStream_t stream) {
  auto kern = quant_pack_kernel<Vec, BITS>;
  const int rowbytes = p.vecs_per_row * 16;
  const QuantSmem L = quant_smem_layout(p.G, p.D, p.rows_chunk, rowbytes);
  // Function attributes are set once per device and size, outside any stream
  // work, so launches can be captured into CUDA graphs.
  static int configured_smem[kMaxDevices] = {};
  static bool configured_cluster[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (static_cast<int>(L.total) > configured_smem[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(L.total));
    if (e != cudaSuccess) return e;
    configured_smem[dev] = static_cast<int>(L.total);
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(kQuantThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  if (p.C > 1) {
    if (p.C > 8 && !configured_cluster[dev]) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
      configured_cluster[dev] = true;
    }
    cfg.gridDim = dim3(p.units * p.C);
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  } else {
    cfg.gridDim = dim3((p.units + p.G - 1) / p.G);
  }
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

size_t quant_smem_bytes(int G, int D, int rows_chunk, int rowbytes) {
  return quant_smem_layout(G, D, rows_chunk, rowbytes).total;
}

int quant_threads() { return kQuantThreads; }

cudaError_t launch_quant_pack(const QuantParams& p, cudaStream_t stream) {
  const bool bf16 = (p.esize == 2);
#define VQ_QP_CASE(B)                                                                   \
  case B:                                                                               \
    return bf16 ? launch_typed<Bf16Vec, B>(p, stream) : launch_typed<F32Vec, B>(p, stream);
  switch (p.bits) {
    VQ_QP_CASE(2)
    VQ_QP_CASE(3)
    VQ_QP_CASE(4)
    VQ_QP_CASE(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef VQ_QP_CASE
}

}  // namespace vq
