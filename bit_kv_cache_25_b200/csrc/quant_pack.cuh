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
  uint32_t bar, mnk, mxk, mn, inv, stage, stage_bytes;
  uint32_t total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// `stages` staging buffers of G slabs of rows_chunk rows each.
__host__ __device__ inline QuantSmem quant_smem_layout(int G, int D, int rows_chunk, int rowbytes, int stages) {
  QuantSmem L;
  L.bar = 0;    // up to 4 mbarriers
  L.mnk = 32;
  L.mxk = L.mnk + 4u * G * D;
  L.mn = L.mxk + 4u * G * D;
  L.inv = L.mn + 4u * G * D;
  L.stage = align_up(L.inv + 4u * G * D, 128);
  L.stage_bytes = align_up(static_cast<uint32_t>(G) * rows_chunk * rowbytes, 128);
  L.total = L.stage + stages * L.stage_bytes;
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

// Work of one CTA-step: `units` consecutive units starting at `unit0`, each
// restricted to the token rows [row0, row0 + rows) / word-rows [wr0, wr0 + wrs).
struct QuantStep {
  int unit0, units, row0, rows, wr0, wrs;
};

// Warp 0: stage the slabs of one step into `stage` (completion on `bar`).
__device__ __forceinline__ void quant_issue_copies(const QuantParams& p, const QuantStep& st, unsigned char* stage,
                                                   uint64_t* bar, int rowbytes) {
  const int tid = threadIdx.x;
  if (tid >= 32) return;
  const uint32_t total = static_cast<uint32_t>(st.units) * st.rows * rowbytes;
  if (tid == 0) mbar_arrive_expect_tx(bar, total);
  __syncwarp();
  const int BH = p.B * p.H;
  for (int g = 0; g < st.units; ++g) {
    const int unit = st.unit0 + g;
    const QuantTensor& T = p.t[unit / BH];
    const int bh = unit % BH;
    const int64_t base = (bh / p.H) * T.sb + (bh % p.H) * T.sh;
    const unsigned char* src = static_cast<const unsigned char*>(T.x) + (base + int64_t(st.row0) * T.st) * p.esize;
    unsigned char* dst = stage + static_cast<size_t>(g) * p.rows_chunk * rowbytes;
    if (T.st * p.esize == rowbytes) {
      if (tid == 0) bulk_copy_g2s(dst, src, static_cast<uint32_t>(st.rows) * rowbytes, bar);
    } else {
      for (int r = tid; r < st.rows; r += 32)
        bulk_copy_g2s(dst + r * rowbytes, src + int64_t(r) * T.st * p.esize, rowbytes, bar);
    }
  }
}

// Pass 1: per-task min/max over the task's cpw rows, merged into the
// per-(unit, channel) key slots. When a whole warp works on one unit, the
// lanes that share a channel vector (lane % V) first combine their keys with
// shuffles and only V lanes issue shared-memory atomics; otherwise every lane
// issues its own. Min and max are idempotent, so any merge order is exact.
template <class Vec, int BITS>
__device__ __forceinline__ void quant_pass1(const QuantParams& p, const QuantStep& st, const unsigned char* stage,
                                            int32_t* mnk, int32_t* mxk) {
  constexpr int CPW = 32 / BITS;
  constexpr int CH = Vec::kCh;
  const int V = p.vecs_per_row;
  const int rowbytes = V * 16;
  const int D = p.D;
  const int tpu = st.wrs * V;
  const int ntask = st.units * tpu;
  const int lane = threadIdx.x & 31;
  const int wbase = threadIdx.x & ~31;
  for (int base = 0; base < ntask; base += blockDim.x) {
    const int task = base + threadIdx.x;
    const bool valid = task < ntask;
    const int g = valid ? task / tpu : 0;
    const int r = task - g * tpu;
    const int wl = r / V;
    const int j = r - wl * V;
    int32_t kmn[CH], kmx[CH];
    if (valid) {
      const int tl0 = wl * CPW;
      const int nvalid = min(CPW, st.rows - tl0);
      const unsigned char* src = stage + (static_cast<size_t>(g) * p.rows_chunk + tl0) * rowbytes + j * 16;
      uint32_t mn[4], mx[4];
      Vec::minmax_init(mn, mx, lds128(src));
#pragma unroll
      for (int i = 1; i < CPW; ++i)
        if (i < nvalid) Vec::minmax_acc(mn, mx, lds128(src + i * rowbytes));
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        kmn[c] = float_key(Vec::ch(mn, c));
        kmx[c] = float_key(Vec::ch(mx, c));
      }
    } else {
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        kmn[c] = INT32_MAX;
        kmx[c] = INT32_MIN;
      }
    }
    const int t_first = base + wbase;
    const bool uniform = (t_first + 31 < ntask) && (t_first / tpu == (t_first + 31) / tpu);
    if (uniform) {  // warp-uniform branch
      for (int off = V; off < 32; off <<= 1) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          kmn[c] = min(kmn[c], __shfl_xor_sync(0xffffffffu, kmn[c], off));
          kmx[c] = max(kmx[c], __shfl_xor_sync(0xffffffffu, kmx[c], off));
        }
      }
      if (lane < V) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          atomicMin(&mnk[g * D + j * CH + c], kmn[c]);
          atomicMax(&mxk[g * D + j * CH + c], kmx[c]);
        }
      }
    } else if (valid) {
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        atomicMin(&mnk[g * D + j * CH + c], kmn[c]);
        atomicMax(&mxk[g * D + j * CH + c], kmx[c]);
      }
    }
  }
}

// Per group: scale = (max - min) / (2^b - 1) (IEEE division), zero = min + 0,
// inv = min(1/scale, FLT_MAX) (IEEE reciprocal), written to shared memory for
// pass 2 and (when `write`) to the output arrays.
template <int BITS>
__device__ __forceinline__ void quant_finalize(const QuantParams& p, const QuantStep& st, int32_t kmn, int32_t kmx,
                                               int i, float* s_mn, float* s_inv, bool write) {
  const int D = p.D;
  const float mn = key_float(kmn);
  const float mx = key_float(kmx);
  const float diff = __fsub_rn(mx, mn);
  const float scale = __fdiv_rn(diff, static_cast<float>((1 << BITS) - 1));
  const float zero = __fadd_rn(mn, 0.0f);
  const float inv = (scale > 0.0f) ? fminf(__frcp_rn(scale), FLT_MAX) : 0.0f;
  s_mn[i] = mn;
  s_inv[i] = inv;
  if (write) {
    const int BH = p.B * p.H;
    const int g = i / D;
    const int c = i - g * D;
    const int unit = st.unit0 + g;
    const QuantTensor& T = p.t[unit / BH];
    const int bh = unit % BH;
    T.scale[static_cast<size_t>(bh) * D + c] = scale;
    T.zero[static_cast<size_t>(bh) * D + c] = zero;
  }
}

// Pass 2: encode and pack. d = x - min and t = d * inv, each correctly rounded
// (__fsub_rn / __fmul_rn are never contracted into an FMA), then round half to
// even by adding 1.5 * 2^23: the rounded value's low mantissa bits are the code
// (t <= 2^b - 1 + tiny, so no clamp is needed). Codes are summed into the word
// with shifts; the magic bits are removed once. (Packed f32x2 arithmetic is
// not used here: ptxas may fuse a packed multiply and add into one rounding.)
template <class Vec, int BITS>
__device__ __forceinline__ void quant_pass2(const QuantParams& p, const QuantStep& st, const unsigned char* stage,
                                            const float* s_mn, const float* s_inv) {
  constexpr int CPW = 32 / BITS;
  constexpr int CH = Vec::kCh;
  const int V = p.vecs_per_row;
  const int rowbytes = V * 16;
  const int D = p.D;
  const int BH = p.B * p.H;
  const int tpu = st.wrs * V;
  for (int task = threadIdx.x; task < st.units * tpu; task += blockDim.x) {
    const int g = task / tpu;
    const int r = task - g * tpu;
    const int wl = r / V;
    const int j = r - wl * V;
    const int tl0 = wl * CPW;
    const int nvalid = min(CPW, st.rows - tl0);
    const unsigned char* src = stage + (static_cast<size_t>(g) * p.rows_chunk + tl0) * rowbytes + j * 16;
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
    const int unit = st.unit0 + g;
    const QuantTensor& T = p.t[unit / BH];
    const int bh = unit % BH;
    uint32_t* dst = T.packed + (static_cast<size_t>(bh) * p.W + st.wr0 + wl) * D + j * CH;
#pragma unroll
    for (int q = 0; q < CH / 4; ++q)
      reinterpret_cast<uint4*>(dst)[q] =
          make_uint4(acc[4 * q] - corr, acc[4 * q + 1] - corr, acc[4 * q + 2] - corr, acc[4 * q + 3] - corr);
  }
}

// Blocks whose (tensor, b, h) slab fits one CTA: a persistent loop over groups
// of G units with a p.stages-deep bulk-copy pipeline, so the next groups'
// slabs are in flight while this group is reduced, encoded and stored.
template <class Vec, int BITS>
__global__ void __launch_bounds__(kQuantThreads) quant_pack_stream_kernel(const __grid_constant__ QuantParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int D = p.D;
  const int rowbytes = p.vecs_per_row * 16;
  const int NST = p.stages;
  const QuantSmem L = quant_smem_layout(p.G, D, p.rows_chunk, rowbytes, NST);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L.bar);
  int32_t* mnk = reinterpret_cast<int32_t*>(smem + L.mnk);
  int32_t* mxk = reinterpret_cast<int32_t*>(smem + L.mxk);
  float* s_mn = reinterpret_cast<float*>(smem + L.mn);
  float* s_inv = reinterpret_cast<float*>(smem + L.inv);
  const int tid = threadIdx.x;
  const int groups = (p.units + p.G - 1) / p.G;

  auto step_of = [&](int grp) {
    QuantStep st;
    st.unit0 = grp * p.G;
    st.units = min(p.G, p.units - st.unit0);
    st.row0 = 0;
    st.rows = p.n;
    st.wr0 = 0;
    st.wrs = p.W;
    return st;
  };

  if (tid == 0) {
    for (int i = 0; i < NST; ++i) mbar_init(&bar[i], 1);
    fence_barrier_init();
  }
  __syncthreads();
  // prologue: the first NST-1 groups of this CTA
  for (int k = 0; k < NST - 1; ++k) {
    const int grp = blockIdx.x + k * gridDim.x;
    if (grp < groups) quant_issue_copies(p, step_of(grp), smem + L.stage + k * L.stage_bytes, &bar[k], rowbytes);
  }
  bool ok = true;
  int it = 0;
  for (int grp = blockIdx.x; grp < groups; ++it, grp += gridDim.x) {
    const QuantStep st = step_of(grp);
    const int stg = it % NST;
    // keep NST-1 groups in flight: the stage refilled here was last read by
    // the previous iteration, which ended with a barrier
    const int ahead = grp + (NST - 1) * gridDim.x;
    if (ahead < groups) {
      const int s2 = (it + NST - 1) % NST;
      quant_issue_copies(p, step_of(ahead), smem + L.stage + s2 * L.stage_bytes, &bar[s2], rowbytes);
    }
    for (int i = tid; i < st.units * D; i += blockDim.x) {
      mnk[i] = INT32_MAX;
      mxk[i] = INT32_MIN;
    }
    ok = __syncthreads_and(mbar_wait_bounded(&bar[stg], (it / NST) & 1));
    if (!ok) break;
    const unsigned char* stage = smem + L.stage + stg * L.stage_bytes;
    quant_pass1<Vec, BITS>(p, st, stage, mnk, mxk);
    __syncthreads();
    for (int i = tid; i < st.units * D; i += blockDim.x) quant_finalize<BITS>(p, st, mnk[i], mxk[i], i, s_mn, s_inv, true);
    __syncthreads();
    quant_pass2<Vec, BITS>(p, st, stage, s_mn, s_inv);
    fence_proxy_async_smem();  // generic reads of this stage before a later bulk copy overwrites it
    __syncthreads();
  }
}

// Blocks whose slab is split over a cluster of C CTAs: each CTA stages its
// chunk of word-rows; the per-channel partial min/max are combined through
// distributed shared memory, so HBM is read exactly once.
template <class Vec, int BITS>
__global__ void __launch_bounds__(kQuantThreads) quant_pack_cluster_kernel(const __grid_constant__ QuantParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int D = p.D;
  const int rowbytes = p.vecs_per_row * 16;
  const QuantSmem L = quant_smem_layout(1, D, p.rows_chunk, rowbytes, 1);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L.bar);
  int32_t* mnk = reinterpret_cast<int32_t*>(smem + L.mnk);
  int32_t* mxk = reinterpret_cast<int32_t*>(smem + L.mxk);
  float* s_mn = reinterpret_cast<float*>(smem + L.mn);
  float* s_inv = reinterpret_cast<float*>(smem + L.inv);
  constexpr int CPW = 32 / BITS;
  const int C = p.C;
  const uint32_t rank = cluster_ctarank();
  const int tid = threadIdx.x;

  QuantStep st;
  st.unit0 = static_cast<int>(blockIdx.x) / C;
  st.units = 1;
  st.wr0 = static_cast<int>(rank) * p.wr_chunk;
  st.wrs = max(0, min(p.wr_chunk, p.W - st.wr0));
  st.row0 = st.wr0 * CPW;
  st.rows = max(0, min(p.rows_chunk, p.n - st.row0));

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  for (int i = tid; i < D; i += blockDim.x) {
    mnk[i] = INT32_MAX;
    mxk[i] = INT32_MIN;
  }
  __syncthreads();
  quant_issue_copies(p, st, smem + L.stage, bar, rowbytes);
  const bool staged = __syncthreads_and(mbar_wait_bounded(bar, 0));
  if (staged) quant_pass1<Vec, BITS>(p, st, smem + L.stage, mnk, mxk);
  __syncthreads();

  cluster_sync();  // every CTA's partials are complete and visible
  int32_t fmn = INT32_MAX, fmx = INT32_MIN;
  if (tid < D) {
    for (int r = 0; r < C; ++r) {
      fmn = min(fmn, dsmem_ld_s32(&mnk[tid], r));
      fmx = max(fmx, dsmem_ld_s32(&mxk[tid], r));
    }
  }
  cluster_arrive();  // done reading peers; the matching wait is at the end
  if (tid < D) quant_finalize<BITS>(p, st, fmn, fmx, tid, s_mn, s_inv, rank == 0 && staged);
  __syncthreads();
  if (staged) quant_pass2<Vec, BITS>(p, st, smem + L.stage, s_mn, s_inv);
  cluster_wait();  // peers may still read this CTA's partials until here
}

template <class Vec, int BITS>
cudaError_t launch_typed(const QuantParams& p, cudaStream_t stream) {
  const bool cluster = p.C > 1;
  auto kern = cluster ? quant_pack_cluster_kernel<Vec, BITS> : quant_pack_stream_kernel<Vec, BITS>;
  const int rowbytes = p.vecs_per_row * 16;
  const QuantSmem L = quant_smem_layout(cluster ? 1 : p.G, p.D, p.rows_chunk, rowbytes, cluster ? 1 : p.stages);
  // Function attributes are set once per device and size, outside any stream
  // work, so launches can be captured into CUDA graphs.
  static int configured_smem[2][kMaxDevices] = {};
  static bool configured_cluster[kMaxDevices] = {};
  static int sm_count[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (static_cast<int>(L.total) > configured_smem[cluster][dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(L.total));
    if (e != cudaSuccess) return e;
    configured_smem[cluster][dev] = static_cast<int>(L.total);
  }
  if (sm_count[dev] == 0) {
    e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(kQuantThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  if (cluster) {
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
    // persistent: enough CTAs to fill every SM at the residency shared memory allows
    const int groups = (p.units + p.G - 1) / p.G;
    const int per_sm = max(1, min(8, static_cast<int>((227u * 1024u) / (L.total + 1024u))));
    cfg.gridDim = dim3(min(groups, sm_count[dev] * per_sm));
  }
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

size_t quant_smem_bytes(int G, int D, int rows_chunk, int rowbytes, int stages) {
  return quant_smem_layout(G, D, rows_chunk, rowbytes, stages).total;
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
