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
// Tiles. A CTA owns 128 queries (M = 128: one thread and one TMEM lane per
// query row). Keys are walked in tiles of 64 keys that never cross a block
// boundary (the scales change per block); a tile's MMAs and softmax only cover
// its valid keys rounded up to 16. Operands live in shared memory in the
// canonical 128-byte-swizzle layout: K codes [64][D] and V codes [64][D] (the
// same layout and unpacking; V is read as an MN-major operand), P [128][64] and
// q' [128][D] (K-major).
//
// Pipeline (one warpgroup; thread 0 also issues the MMAs and bulk copies):
//   bulk copy of tile g+2's packed words  |  unpack tile g+1 into the other
//   operand buffer  |  QK^T of tile g+1 (tensor core)  while  softmax of tile g
//   (CUDA cores)  ->  PV of tile g (tensor core)  while  unpack of tile g+2.
// S is double-buffered in TMEM. Online softmax in fp32 with a lazy reference
// maximum: U and O are rescaled only when a row maximum grows by more than
// kTau (p stays <= e^kTau, fine for fp16).
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
constexpr int kKT = 64;               // keys per tile

template <int BITS, int D>
struct TcCfg {
  static constexpr int CPW = 32 / BITS;
  static constexpr uint32_t MASK = (1u << BITS) - 1u;
  static constexpr int MAXW = (kKT + CPW - 1) / CPW + 1;  // packed word-rows one tile can touch
  static constexpr int STAGE_WORDS = MAXW * D;            // per tensor
  // shared memory (byte offsets from a 1024-aligned base)
  static constexpr int Q_HI = 0;                          // [128][D] fp16
  static constexpr int Q_LO = Q_HI + 128 * D * 2;
  static constexpr int KB0 = Q_LO + 128 * D * 2;          // 2 x [64][D] fp16
  static constexpr int KB_SZ = kKT * D * 2;
  static constexpr int VB0 = KB0 + 2 * KB_SZ;             // 2 x [64][D] fp16 (read MN-major)
  static constexpr int VB_SZ = kKT * D * 2;
  static constexpr int STG0 = VB0 + 2 * VB_SZ;           // 2 x {K words, V words}
  static constexpr int STG_SZ = 2 * STAGE_WORDS * 4;
  static constexpr int META = STG0 + 2 * STG_SZ;          // 2 x [4][D] fp32: sk, zk, sv, zv
  static constexpr int BARS = META + 2 * 4 * D * 4;       // s[2], pv[2], stage[2]
  static constexpr int TMEM_SLOT = BARS + 6 * 8;
  static constexpr int SMEM = TMEM_SLOT + 16;
  static constexpr int SMEM_ALLOC = SMEM + 1024;          // room to align the base
  static_assert(KB0 % 1024 == 0 && VB0 % 1024 == 0, "tile alignment");
  static_assert(STG0 % 128 == 0 && STG_SZ % 128 == 0, "stage alignment");
  // tensor memory columns
  static constexpr int COL_S = 0;                         // 2 x 64 columns
  static constexpr int COL_U = 128;                       // D columns
  static constexpr int COL_O = 128 + D;                   // D columns
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

// Walks the key tiles of blocks 0..s in order: (block kb, first key t0).
struct TileIter {
  int kb, t0;
  __device__ __forceinline__ void next(const AttnParams& p) {
    if (kb > p.s) return;
    t0 += kKT;
    if (t0 >= p.blk[kb].n) {
      ++kb;
      t0 = 0;
    }
  }
  __device__ __forceinline__ bool valid(const AttnParams& p) const { return kb <= p.s; }
};

template <int BITS, int D>
__global__ void __launch_bounds__(kTcThreads, (D == 64) ? 2 : 1) attention_tc_kernel(const __grid_constant__ AttnParams p) {
  using C = TcCfg<BITS, D>;
  constexpr int CPW = C::CPW;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char* sm = smem_raw + (sbase - raw);
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(sm + C::BARS);
  uint64_t* bar_pv = bar_s + 2;
  uint64_t* bar_stg = bar_s + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::TMEM_SLOT);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int bh = blockIdx.y;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int q0 = blockIdx.x * 128;
  const int row = tid;
  const bool row_valid = (q0 + row) < p.n_q;
  // warps whose 32 rows are all past n_q skip the per-row work (q', softmax,
  // fold, epilogue); their P and U rows are never read back
  const bool warp_active = __any_sync(0xffffffffu, row_valid);
  const int64_t BHD = static_cast<int64_t>(p.B) * p.H * D;

  // zero the K/V operand buffers once: rows past a tile's valid keys are read by
  // the MMAs (multiplied by zero probabilities) and must hold finite values
  for (int i = C::KB0 + tid * 16; i < C::STG0; i += kTcThreads * 16) tc::sts128(sbase + i, 0u, 0u, 0u, 0u);
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 6; ++i) mbar_init(&bar_s[i], 1);
    fence_barrier_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t idesc_pv = tc::idesc_f16_f32(128, D, /*b_mn_major=*/true);
  // this row's query (bf16 pairs): kept in registers at D = 64, re-read from
  // global memory (L1/L2 hits) once per key block at D = 128
  constexpr bool kQRegs = (D == 64);
  const uint16_t* qrow = p.q + b * p.q_sb + h * p.q_sh + static_cast<int64_t>(q0 + row) * p.q_st;
  uint32_t qreg[kQRegs ? D / 2 : 1];
  if constexpr (kQRegs) {
#pragma unroll
    for (int c8 = 0; c8 < D; c8 += 8) {
      uint4 raw8 = make_uint4(0, 0, 0, 0);
      if (row_valid) raw8 = *reinterpret_cast<const uint4*>(qrow + c8);
      qreg[c8 / 2] = raw8.x;
      qreg[c8 / 2 + 1] = raw8.y;
      qreg[c8 / 2 + 2] = raw8.z;
      qreg[c8 / 2 + 3] = raw8.w;
    }
  }
  auto qword = [&](int k2) -> uint32_t {  // bf16 pair (2*k2, 2*k2+1)
    if constexpr (kQRegs) {
      return qreg[k2];
    } else {
      return row_valid ? reinterpret_cast<const uint32_t*>(qrow)[k2] : 0u;
    }
  };

  // ---- thread 0: bulk copy of one tile's packed K and V words into a stage
  auto issue_copy = [&](const TileIter& t, int stage) {
    const AttnBlockInfo& bi = p.blk[t.kb];
    const int wa = t.t0 / CPW;
    const int wb = min(bi.W - 1, (t.t0 + kKT - 1) / CPW);
    const uint32_t bytes = static_cast<uint32_t>(wb - wa + 1) * D * 4;
    const int64_t off = bi.word_off + static_cast<int64_t>(bh) * bi.W * D + static_cast<int64_t>(wa) * D;
    unsigned char* dst = sm + C::STG0 + stage * C::STG_SZ;
    mbar_arrive_expect_tx(&bar_stg[stage], 2 * bytes);
    bulk_copy_g2s(dst, p.packed_k + off, bytes, &bar_stg[stage]);
    bulk_copy_g2s(dst + C::STAGE_WORDS * 4, p.packed_v + off, bytes, &bar_stg[stage]);
  };

  // ---- all threads: meta of block kb into meta buffer kb % 2
  auto load_meta = [&](int kb) {
    float* meta = reinterpret_cast<float*>(sm + C::META) + (kb & 1) * 4 * D;
    for (int c = tid; c < D; c += kTcThreads) {
      const int64_t mo = kb * BHD + static_cast<int64_t>(bh) * D + c;
      meta[c] = p.scale_k[mo];
      meta[D + c] = p.zero_k[mo];
      meta[2 * D + c] = p.scale_v[mo];
      meta[3 * D + c] = p.zero_v[mo];
    }
  };

  // ---- this row's q' for block kb, split into fp16 hi/lo; returns bias, 2^e
  auto build_q = [&](int kb, float& bias_out, float& up_out) {
    const float* meta = reinterpret_cast<const float*>(sm + C::META) + (kb & 1) * 4 * D;
    float bias = 0.0f, amax = 0.0f;
#pragma unroll
    for (int c = 0; c < D; ++c) {
      const uint32_t w = qword(c >> 1);
      const float qv = __uint_as_float((c & 1) ? (w & 0xffff0000u) : (w << 16));
      const float qs = __fmul_rn(p.softmax_scale, qv);
      amax = fmaxf(amax, fabsf(__fmul_rn(qs, meta[c])));
      bias = fmaf(qs, meta[D + c], bias);
    }
    int e = 0;
    if (amax > 0.0f) {
      const int ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127;
      e = max(-100, min(100, ex - 10));
    }
    const float down = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
#pragma unroll
    for (int c8 = 0; c8 < D; c8 += 8) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int k2 = 0; k2 < 4; ++k2) {
        const uint32_t w = qword(c8 / 2 + k2);
        float x[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float qv = __uint_as_float(u ? (w & 0xffff0000u) : (w << 16));
          x[u] = __fmul_rn(__fmul_rn(__fmul_rn(p.softmax_scale, qv), meta[c8 + 2 * k2 + u]), down);
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
    bias_out = bias;
    up_out = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
  };

  // ---- all threads: unpack a staged tile into operand buffer `buf`. K and V
  // codes land in the same [64 keys][D] layout; task = (tensor, staged
  // word-row, channel octet) -> up to CPW keys, one 16-byte store per key.
  auto unpack = [&](const TileIter& ti, int stage, int buf) {
    const AttnBlockInfo& bi = p.blk[ti.kb];
    const int wa = ti.t0 / CPW;
    const int wb = min(bi.W - 1, (ti.t0 + kKT - 1) / CPW);
    const int nw = wb - wa + 1;
    const uint32_t* words = reinterpret_cast<const uint32_t*>(sm + C::STG0 + stage * C::STG_SZ);
    const int per = nw * (D / 8);
    for (int task = tid; task < 2 * per; task += kTcThreads) {
      const int tsel = task >= per ? 1 : 0;
      const int r = task - tsel * per;
      const int wl = r / (D / 8);
      const int j = r - wl * (D / 8);
      const uint32_t* src = words + tsel * C::STAGE_WORDS + wl * D + 8 * j;
      const uint4 a = *reinterpret_cast<const uint4*>(src);
      const uint4 bq = *reinterpret_cast<const uint4*>(src + 4);
      const uint32_t wd[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
      const uint32_t dst = sbase + (tsel ? (C::VB0 + buf * C::VB_SZ) : (C::KB0 + buf * C::KB_SZ));
      const int kbase = (wa + wl) * CPW - ti.t0;  // tile-local key of slot 0
#pragma unroll
      for (int i = 0; i < CPW; ++i) {
        const int key = kbase + i;
        if (key < 0 || key >= kKT) continue;
        uint32_t hv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          hv[u] = codes_to_half2((wd[2 * u] >> (BITS * i)) & C::MASK, (wd[2 * u + 1] >> (BITS * i)) & C::MASK);
        tc::sts128(dst + tc::sw128_offset(key, 8 * j, kKT), hv[0], hv[1], hv[2], hv[3]);
      }
    }
  };

  auto issue_qk = [&](const TileIter& t, int buf) {
    const int nk = min(kKT, p.blk[t.kb].n - t.t0);
    const int nk16 = (nk + 15) & ~15;
    const uint32_t idesc = tc::idesc_f16_f32(128, nk16);
    const uint32_t kbuf = sbase + C::KB0 + buf * C::KB_SZ;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t koff = (kk & 3) * 32;
      tc::mma_f16_ss(tmem + C::COL_S + buf * 64, tc::sw128_desc(sbase + C::Q_HI + (kk >> 2) * 128 * 128 + koff),
                     tc::sw128_desc(kbuf + (kk >> 2) * kKT * 128 + koff), idesc, kk > 0 ? 1u : 0u);
    }
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t koff = (kk & 3) * 32;
      tc::mma_f16_ss(tmem + C::COL_S + buf * 64, tc::sw128_desc(sbase + C::Q_LO + (kk >> 2) * 128 * 128 + koff),
                     tc::sw128_desc(kbuf + (kk >> 2) * kKT * 128 + koff), idesc, 1u);
    }
    tc::commit(&bar_s[buf]);
  };

  // PV of tile `buf`: A = P from TMEM, written in place over S[buf] (per 16-key
  // chunk kk: 8 columns of P hi, then 8 columns of P lo), B = V codes (MN-major).
  auto issue_pv = [&](int nk16, int buf, bool first_of_block) {
    const uint32_t vbuf = sbase + C::VB0 + buf * C::VB_SZ;
    constexpr uint32_t kLbo = kKT * 128;  // 64-channel groups of the [64][D] V tile
    const uint32_t pa = tmem + C::COL_S + buf * 64;
    for (int kk = 0; kk < nk16 / 16; ++kk) {
      tc::mma_f16_ts(tmem + C::COL_U, pa + 16 * kk, tc::sw128_desc_mn(vbuf + kk * 2048, kLbo), idesc_pv,
                     (first_of_block && kk == 0) ? 0u : 1u);
    }
    for (int kk = 0; kk < nk16 / 16; ++kk) {
      tc::mma_f16_ts(tmem + C::COL_U, pa + 16 * kk + 8, tc::sw128_desc_mn(vbuf + kk * 2048, kLbo), idesc_pv, 1u);
    }
    tc::commit(&bar_pv[buf]);
  };

  // ---------------------------------------------------------------- prologue
  TileIter cur{0, 0};
  TileIter cp = cur;  // next tile to copy (thread 0's view; every thread keeps it identical)
  if (tid == 0) {
    issue_copy(cp, 0);
  }
  cp.next(p);
  if (tid == 0 && cp.valid(p)) issue_copy(cp, 1);
  cp.next(p);

  load_meta(0);
  __syncthreads();
  float bias_q[2] = {0.0f, 0.0f}, up_q[2] = {1.0f, 1.0f};
  if (warp_active) build_q(0, bias_q[0], up_q[0]);
  bool ok = __syncthreads_and(mbar_wait_bounded(&bar_stg[0], 0));
  if (ok) unpack(cur, 0, 0);
  fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (tid == 0 && ok) issue_qk(cur, 0);

  float m_ref = -INFINITY;  // reference maximum of this row's logits
  float l_tot = 0.0f;       // sum of p over folded blocks (relative to m_ref)
  float rs = 0.0f;          // sum of p over the current block (relative to m_ref)
  bool have_o = false;      // O holds at least one folded block
  int prev_kb = -1;

  // ---------------------------------------------------------------- main loop over tiles
  int g = 0;
  for (; ok && cur.valid(p); ++g) {
    TileIter nxt = cur;
    nxt.next(p);
    const bool has_next = nxt.valid(p);
    const int nk = min(kKT, p.blk[cur.kb].n - cur.t0);
    const int nk16 = (nk + 15) & ~15;
    const bool first_of_block = (cur.t0 == 0);

    // (1) PV(g-1) done: its V buffer, the P buffer and U are free
    if (g >= 1) ok = __syncthreads_and(mbar_wait_bounded(&bar_pv[(g - 1) & 1], ((g - 1) >> 1) & 1));
    if (!ok) break;
    // (2) unpack tile g+1 into the other operand buffer
    if (has_next) {
      ok = __syncthreads_and(mbar_wait_bounded(&bar_stg[(g + 1) & 1], ((g + 1) >> 1) & 1));
      if (!ok) break;
      unpack(nxt, (g + 1) & 1, (g + 1) & 1);
    }
    // (3) S(g) ready
    ok = __syncthreads_and(mbar_wait_bounded(&bar_s[g & 1], (g >> 1) & 1));
    if (!ok) break;
    tc::fence_after_sync();
    // (4) fold the previous block into O when tile g starts a new block (PV(g-1),
    // the last PV of that block, is complete); this must precede (5), which may
    // reuse the previous block's meta buffer
    if (first_of_block && prev_kb >= 0 && warp_active) {
      const float* meta = reinterpret_cast<const float*>(sm + C::META) + (prev_kb & 1) * 4 * D;
#pragma unroll 1
      for (int c16 = 0; c16 < D; c16 += 16) {
        uint32_t u[16], o[16];
        tc::tmem_ld16(tmem + lane_off + C::COL_U + c16, u);
        if (have_o) tc::tmem_ld16(tmem + lane_off + C::COL_O + c16, o);
        tc::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float base_o = have_o ? __uint_as_float(o[k]) : 0.0f;
          o[k] = __float_as_uint(
              fmaf(__uint_as_float(u[k]), meta[2 * D + c16 + k], fmaf(rs, meta[3 * D + c16 + k], base_o)));
        }
        tc::tmem_st16(tmem + lane_off + C::COL_O + c16, o);
      }
      tc::tmem_wait_st();
      l_tot += rs;
      rs = 0.0f;
      have_o = true;
    }
    prev_kb = cur.kb;

    // (5) q' for tile g+1's block, if it starts a new one (QK(g) no longer reads q')
    if (has_next && nxt.kb != cur.kb) {
      __syncthreads();  // every thread's fold has finished reading the meta buffer reused here
      load_meta(nxt.kb);
      __syncthreads();
      if (warp_active) build_q(nxt.kb, bias_q[nxt.kb & 1], up_q[nxt.kb & 1]);
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // (6) QK(g+1) and the bulk copy of tile g+2 (into the stage tile g came through)
    if (tid == 0) {
      if (has_next) issue_qk(nxt, (g + 1) & 1);
      if (cp.valid(p)) issue_copy(cp, g & 1);
    }
    if (cp.valid(p)) cp.next(p);

    // (7) softmax of tile g. Pass 1: row maximum of the raw S (up > 0 is a power
    // of two, so max(S * up + bias) = max(S) * up + bias). Pass 2 re-reads S from
    // TMEM: p = 2^(S * up * log2 e + (bias - m) * log2 e), one FFMA and one EX2;
    // hi = p with its low 13 mantissa bits cleared (exact in fp16 for
    // p >= 2^-14), lo = p - hi (exact); both rounded to fp16.
    if (warp_active) {
    const float bias = bias_q[cur.kb & 1];
    const float up = up_q[cur.kb & 1];
    const uint32_t t_s = tmem + lane_off + C::COL_S + (g & 1) * 64;
    const bool partial = nk < nk16;  // columns [nk, nk16) are padding
    // all of this row's S in one TMEM round trip (up to 64 columns)
    uint32_t sr[kKT];
#pragma unroll
    for (int c16 = 0; c16 < kKT; c16 += 16)
      if (c16 < nk16) tc::tmem_ld16(t_s + c16, *reinterpret_cast<uint32_t(*)[16]>(&sr[c16]));
    tc::tmem_wait_ld();
    float smax = -INFINITY;
#pragma unroll
    for (int j = 0; j < kKT; ++j)
      if (j < nk) smax = fmaxf(smax, __uint_as_float(sr[j]));
    const float mx = fmaf(smax, up, bias);
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
    if (__any_sync(0xffffffffu, rescale)) {
      if (!first_of_block) {
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
    constexpr float kLog2e = 1.4426950408889634f;
    const float up2 = up * kLog2e;
    const float c2 = (bias - m_ref) * kLog2e;
    const uint64_t up2x2 = tc::f2pack(up2, up2);
    const uint64_t c2x2 = tc::f2pack(c2, c2);
    const uint64_t neg1x2 = tc::f2pack(-1.0f, -1.0f);
    uint64_t rs2 = tc::f2pack(0.0f, 0.0f);
#pragma unroll
    for (int c16 = 0; c16 < kKT; c16 += 16) {
      if (c16 < nk16) {
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j0 = c16 + 2 * u;
          const uint64_t arg =
              tc::fma2(tc::f2pack(__uint_as_float(sr[j0]), __uint_as_float(sr[j0 + 1])), up2x2, c2x2);
          float p0 = tc::ex2(tc::f2lo(arg));
          float p1 = tc::ex2(tc::f2hi(arg));
          if (partial) {
            p0 = (j0 < nk) ? p0 : 0.0f;
            p1 = (j0 + 1 < nk) ? p1 : 0.0f;
          }
          const uint64_t pp = tc::f2pack(p0, p1);
          const float h0 = __uint_as_float(__float_as_uint(p0) & 0xffffe000u);
          const float h1 = __uint_as_float(__float_as_uint(p1) & 0xffffe000u);
          const uint64_t lo2 = tc::fma2(tc::f2pack(h0, h1), neg1x2, pp);
          rs2 = tc::add2(rs2, pp);
          hi[u] = tc::cvt_half2(h0, h1);
          lo[u] = tc::cvt_half2(tc::f2lo(lo2), tc::f2hi(lo2));
        }
        // S of this row is in registers: P hi and lo replace it in place
        tc::tmem_st8(t_s + c16, hi);
        tc::tmem_st8(t_s + c16 + 8, lo);
      }
    }
    tc::tmem_wait_st();
    rs += tc::f2lo(rs2) + tc::f2hi(rs2);
    }  // warp_active
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // (8) PV(g)
    if (tid == 0) issue_pv(nk16, g & 1, first_of_block);
    cur = nxt;
  }

  // ---------------------------------------------------------------- last fold + epilogue
  if (ok && g >= 1) {
    // g tiles were walked; the PV of the last one is the pending commit
    ok = __syncthreads_and(mbar_wait_bounded(&bar_pv[(g - 1) & 1], ((g - 1) >> 1) & 1));
    tc::fence_after_sync();
  }
  if (ok && warp_active) {
    const float* meta = reinterpret_cast<const float*>(sm + C::META) + (prev_kb & 1) * 4 * D;
    const float inv = 1.0f / (l_tot + rs);
    const int64_t obase = b * p.o_sb + h * p.o_sh + static_cast<int64_t>(q0 + row) * p.o_st;
#pragma unroll 1
    for (int c16 = 0; c16 < D; c16 += 16) {
      uint32_t u[16], o[16];
      tc::tmem_ld16(tmem + lane_off + C::COL_U + c16, u);
      if (have_o) tc::tmem_ld16(tmem + lane_off + C::COL_O + c16, o);
      tc::tmem_wait_ld();
      float v[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float base_o = have_o ? __uint_as_float(o[k]) : 0.0f;
        v[k] = fmaf(__uint_as_float(u[k]), meta[2 * D + c16 + k], fmaf(rs, meta[3 * D + c16 + k], base_o)) * inv;
      }
      if (!row_valid) continue;
      if (p.out_f32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + obase + c16);
#pragma unroll
        for (int k = 0; k < 4; ++k) dst[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
      } else {
        uint32_t bf[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          uint32_t pair = 0;
#pragma unroll
          for (int uu = 0; uu < 2; ++uu) {
            const uint32_t x = __float_as_uint(v[2 * k + uu]);
            pair |= ((x + 0x7fffu + ((x >> 16) & 1u)) >> 16) << (16 * uu);
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
