// Packed-KV block attention on the sm_100a tensor cores, warp-specialized.
//
// Same arithmetic as attention_tc.cuh (scales folded into the queries, exact
// integer codes as MMA operands, q' and P split into fp16 hi/lo, fp32
// accumulators in TMEM; see that file for the reasoning). What changes is the
// schedule. Three roles run concurrently in one CTA and hand work to each other
// through mbarrier rings, so the tensor cores, the unpacking and the softmax
// overlap:
//   control warp (1 thread): bulk copies of packed words (3-stage ring) and
//     every tcgen05.mma: QK^T of tile g into S[g % 2], then PV of tile g-1;
//   unpack warpgroup (128 threads): packed words -> fp16 K and V code tiles
//     (2-buffer ring), the same [64 keys][D] 128B-swizzled layout for both;
//   softmax warpgroups (NQT of them, 128 threads each, one query row per
//     thread): read S from TMEM, write P hi/lo, rebuild q' once per key block,
//     fold each finished block's U into O and write the output.
// With NQT = 2 (head_dim 64) a CTA owns 256 queries: both query tiles share
// every unpacked K/V tile, and the two softmax warpgroups take turns on the
// tensor cores (one computes while the other's MMAs run).
// Barriers (count): stg_full (tx bytes), stg_empty (128), kv_full (128),
// kv_empty (MMA commit), and per query tile: q_full (128), s_full (commit),
// s_empty (128), p_full (128), p_empty (commit; also "PV of that tile is done").
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tc_ptx.cuh"
#include "vq_device.cuh"
#include "vq_internal.h"

namespace vq {
namespace {

template <int BITS, int D, int NQT>
struct WsCfg {
  static constexpr int THREADS = NQT * 128 + 128 + 32;    // softmax WGs, unpack WG, control warp
  static constexpr int UNPACK_T0 = NQT * 128;             // first unpack thread
  static constexpr int CTRL_WARP = NQT * 4 + 4;
  static constexpr int CPW = 32 / BITS;
  static constexpr uint32_t MASK = (1u << BITS) - 1u;
  static constexpr int KT = 64;                           // keys per tile
  static constexpr int MAXW = (KT + CPW - 1) / CPW + 1;   // packed word-rows one tile can touch
  static constexpr int STAGE_WORDS = MAXW * D;            // per tensor
  static constexpr int NSTG = (D == 64) ? 3 : 2;          // packed-word stages
  static constexpr int NKV = 2;                           // fp16 K/V tile buffers
  static constexpr int NPB = (NQT == 1) ? 2 : 1;          // P buffers per query tile
  // shared memory (byte offsets from a 1024-aligned base)
  static constexpr int Q_SZ = 128 * D * 2;                // one of hi / lo
  static constexpr int Q0 = 0;                            // NQT x {q' hi [128][D], q' lo [128][D]}
  static constexpr int KV0 = Q0 + NQT * 2 * Q_SZ;         // NKV x {K [64][D], V [64][D]}
  static constexpr int TILE_SZ = KT * D * 2;
  static constexpr int KV_SZ = 2 * TILE_SZ;
  static constexpr int P0 = KV0 + NKV * KV_SZ;            // NQT x NPB x {P hi [128][64], P lo [128][64]}
  static constexpr int PT_SZ = 128 * KT * 2;
  static constexpr int P_SZ = 2 * PT_SZ;
  static constexpr int STG0 = P0 + NQT * NPB * P_SZ;
  static constexpr int STG_SZ = 2 * STAGE_WORDS * 4;
  static constexpr int META = STG0 + NSTG * STG_SZ;       // NQT x 3 x [4][D] fp32: sk, zk, sv, zv
  static constexpr int BARS = META + NQT * 3 * 4 * D * 4;
  static constexpr int NBARS = 2 * NSTG + 2 * NKV + NQT * (1 + 2 + 2 + 2 * NPB);
  static constexpr int TMEM_SLOT = BARS + NBARS * 8;
  static constexpr int SMEM = TMEM_SLOT + 16;
  static constexpr int SMEM_ALLOC = SMEM + 1024;
  static_assert(KV0 % 1024 == 0 && TILE_SZ % 1024 == 0 && P0 % 1024 == 0 && PT_SZ % 1024 == 0, "tile alignment");
  static_assert(STG0 % 128 == 0 && STG_SZ % 128 == 0, "stage alignment");
  static_assert(SMEM_ALLOC <= 232448, "shared memory");
  // tensor memory columns: per query tile qt, S[2] at qt*128, U and O after all S
  static constexpr int COL_S = 0;
  static constexpr int COL_U = NQT * 128;                 // + qt * D
  static constexpr int COL_O = NQT * 128 + NQT * D;       // + qt * D
  static constexpr int TMEM_USED = NQT * (128 + 2 * D);
  static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "tensor memory");
};

// Bounded wait that works for every role: on timeout the device error word is
// set and the caller stops its loop.
__device__ __forceinline__ bool ws_wait(uint64_t* bar, uint32_t parity) { return mbar_wait_bounded(bar, parity); }

// Tile sequence helpers (every role walks the same sequence).
struct WsTile {
  int kb, t0;
};
__device__ __forceinline__ void ws_next(const AttnParams& p, WsTile& t) {
  if (t.kb > p.s) return;
  t.t0 += 64;
  if (t.t0 >= p.blk[t.kb].n) {
    ++t.kb;
    t.t0 = 0;
  }
}

template <int BITS, int D, int NQT>
__global__ void __launch_bounds__(WsCfg<BITS, D, NQT>::THREADS, 1)
    attention_ws_kernel(const __grid_constant__ AttnParams p) {
  using C = WsCfg<BITS, D, NQT>;
  constexpr int CPW = C::CPW;
  constexpr int KT = C::KT;
  constexpr int NPB = C::NPB;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char* sm = smem_raw + (sbase - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::BARS);
  uint64_t* stg_full = bars;
  uint64_t* stg_empty = stg_full + C::NSTG;
  uint64_t* kv_full = stg_empty + C::NSTG;
  uint64_t* kv_empty = kv_full + C::NKV;
  uint64_t* qbars = kv_empty + C::NKV;  // per query tile: q_full, s_full[2], s_empty[2], p_full[NPB], p_empty[NPB]
  constexpr int QB = 1 + 2 + 2 + 2 * NPB;
  auto q_full = [&](int qt) { return qbars + qt * QB; };
  auto s_full = [&](int qt, int i) { return qbars + qt * QB + 1 + i; };
  auto s_empty = [&](int qt, int i) { return qbars + qt * QB + 3 + i; };
  auto p_full = [&](int qt, int i) { return qbars + qt * QB + 5 + i; };
  auto p_empty = [&](int qt, int i) { return qbars + qt * QB + 5 + NPB + i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::TMEM_SLOT);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int bh = blockIdx.y;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int cta_q0 = blockIdx.x * 128 * NQT;
  // query tiles of this CTA that hold at least one query
  const int nqt = min(NQT, (p.n_q - cta_q0 + 127) / 128);
  const int64_t BHD = static_cast<int64_t>(p.B) * p.H * D;

  // ---- set-up: TMEM (warp 0), barriers (thread 0), zeroed K/V tiles (unpack WG)
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < C::NSTG; ++i) {
      mbar_init(&stg_full[i], 1);
      mbar_init(&stg_empty[i], 128);
    }
    for (int i = 0; i < C::NKV; ++i) {
      mbar_init(&kv_full[i], 128);
      mbar_init(&kv_empty[i], 1);
    }
    for (int qt = 0; qt < NQT; ++qt) {
      mbar_init(q_full(qt), 128);
      for (int i = 0; i < 2; ++i) {
        mbar_init(s_full(qt, i), 1);
        mbar_init(s_empty(qt, i), 128);
      }
      for (int i = 0; i < NPB; ++i) {
        mbar_init(p_full(qt, i), 128);
        mbar_init(p_empty(qt, i), 1);
      }
    }
    fence_barrier_init();
  }
  if (tid >= C::UNPACK_T0 && tid < C::UNPACK_T0 + 128) {
    // rows past a tile's valid keys are read by the MMAs (times zero
    // probabilities) and must hold finite values
    for (int i = C::KV0 + (tid - C::UNPACK_T0) * 16; i < C::P0; i += 128 * 16) tc::sts128(sbase + i, 0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::CTRL_WARP) {
    // =========================================================== control warp
    if ((tid & 31) == 0) {
      auto issue_copy = [&](const WsTile& t, int stage) {
        const AttnBlockInfo& bi = p.blk[t.kb];
        const int wa = t.t0 / CPW;
        const int wb = min(bi.W - 1, (t.t0 + KT - 1) / CPW);
        const uint32_t bytes = static_cast<uint32_t>(wb - wa + 1) * D * 4;
        const int64_t off = bi.word_off + static_cast<int64_t>(bh) * bi.W * D + static_cast<int64_t>(wa) * D;
        unsigned char* dst = sm + C::STG0 + stage * C::STG_SZ;
        mbar_arrive_expect_tx(&stg_full[stage], 2 * bytes);
        bulk_copy_g2s(dst, p.packed_k + off, bytes, &stg_full[stage]);
        bulk_copy_g2s(dst + C::STAGE_WORDS * 4, p.packed_v + off, bytes, &stg_full[stage]);
      };
      const uint32_t idesc_pv = tc::idesc_f16_f32(128, D, /*b_mn_major=*/true);
      constexpr uint32_t kLbo = KT * 128;
      auto issue_pv = [&](int qt, int gp, int nk16, bool first) {
        const uint32_t vbuf = sbase + C::KV0 + (gp % C::NKV) * C::KV_SZ + C::TILE_SZ;
        const uint32_t pb = sbase + C::P0 + (qt * NPB + gp % NPB) * C::P_SZ;
        const uint32_t tu = tmem + C::COL_U + qt * D;
        for (int kk = 0; kk < nk16 / 16; ++kk)
          tc::mma_f16_ss(tu, tc::sw128_desc(pb + kk * 32), tc::sw128_desc_mn(vbuf + kk * 2048, kLbo), idesc_pv,
                         (first && kk == 0) ? 0u : 1u);
        for (int kk = 0; kk < nk16 / 16; ++kk)
          tc::mma_f16_ss(tu, tc::sw128_desc(pb + C::PT_SZ + kk * 32), tc::sw128_desc_mn(vbuf + kk * 2048, kLbo),
                         idesc_pv, 1u);
        tc::commit(p_empty(qt, gp % NPB));
      };
      // prefetch the first NSTG tiles
      WsTile cp{0, 0};
      for (int k = 0; k < C::NSTG && cp.kb <= p.s; ++k, ws_next(p, cp)) issue_copy(cp, k);

      bool ok = true;
      WsTile t{0, 0};
      int prev_nk16 = 0;
      bool prev_first = true;
      int g = 0;
      for (; t.kb <= p.s; ++g) {
        const int nk = min(KT, p.blk[t.kb].n - t.t0);
        const int nk16 = (nk + 15) & ~15;
        const bool first = (t.t0 == 0);
        // refill the stage tile g-1 came through
        if (g >= 1 && cp.kb <= p.s) {
          const int st = (g - 1) % C::NSTG;
          if (!(ok = ws_wait(&stg_empty[st], ((g - 1) / C::NSTG) & 1))) break;
          issue_copy(cp, st);
          ws_next(p, cp);
        }
        // ---- QK(g) of every query tile -> S[qt][g % 2]
        if (!(ok = ws_wait(&kv_full[g % C::NKV], (g / C::NKV) & 1))) break;
        const uint32_t idesc = tc::idesc_f16_f32(128, nk16);
        const uint32_t kbuf = sbase + C::KV0 + (g % C::NKV) * C::KV_SZ;
        for (int qt = 0; qt < nqt && ok; ++qt) {
          if (first && !(ok = ws_wait(q_full(qt), t.kb & 1))) break;
          if (!(ok = ws_wait(s_empty(qt, g & 1), ((g >> 1) & 1) ^ 1))) break;
          tc::fence_after_sync();
          const uint32_t qb = sbase + C::Q0 + qt * 2 * C::Q_SZ;
          const uint32_t ts = tmem + C::COL_S + qt * 128 + (g & 1) * 64;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk & 3) * 32;
            tc::mma_f16_ss(ts, tc::sw128_desc(qb + (kk >> 2) * 128 * 128 + koff),
                           tc::sw128_desc(kbuf + (kk >> 2) * KT * 128 + koff), idesc, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk & 3) * 32;
            tc::mma_f16_ss(ts, tc::sw128_desc(qb + C::Q_SZ + (kk >> 2) * 128 * 128 + koff),
                           tc::sw128_desc(kbuf + (kk >> 2) * KT * 128 + koff), idesc, 1u);
          }
          tc::commit(s_full(qt, g & 1));
        }
        if (!ok) break;
        // ---- PV(g-1) of every query tile -> U[qt]
        if (g >= 1) {
          const int gp = g - 1;
          for (int qt = 0; qt < nqt && ok; ++qt) {
            if (!(ok = ws_wait(p_full(qt, gp % NPB), (gp / NPB) & 1))) break;
            tc::fence_after_sync();
            issue_pv(qt, gp, prev_nk16, prev_first);
          }
          if (!ok) break;
          tc::commit(&kv_empty[gp % C::NKV]);
        }
        prev_nk16 = nk16;
        prev_first = first;
        ws_next(p, t);
      }
      // ---- PV of the last tile
      if (ok && g >= 1) {
        const int gp = g - 1;
        for (int qt = 0; qt < nqt && ok; ++qt) {
          if (!(ok = ws_wait(p_full(qt, gp % NPB), (gp / NPB) & 1))) break;
          tc::fence_after_sync();
          issue_pv(qt, gp, prev_nk16, prev_first);
        }
        if (ok) tc::commit(&kv_empty[gp % C::NKV]);
      }
    }
  } else if (tid >= C::UNPACK_T0) {
    // =========================================================== unpack warpgroup
    const int ut = tid - C::UNPACK_T0;
    WsTile t{0, 0};
    for (int g = 0; t.kb <= p.s; ++g, ws_next(p, t)) {
      const int st = g % C::NSTG;
      const int kvb = g % C::NKV;
      if (!ws_wait(&stg_full[st], (g / C::NSTG) & 1)) break;
      if (!ws_wait(&kv_empty[kvb], ((g / C::NKV) & 1) ^ 1)) break;
      const AttnBlockInfo& bi = p.blk[t.kb];
      const int wa = t.t0 / CPW;
      const int wb = min(bi.W - 1, (t.t0 + KT - 1) / CPW);
      const int nw = wb - wa + 1;
      const uint32_t* words = reinterpret_cast<const uint32_t*>(sm + C::STG0 + st * C::STG_SZ);
      const uint32_t kvbase = sbase + C::KV0 + kvb * C::KV_SZ;
      const int per = nw * (D / 8);
      for (int task = ut; task < 2 * per; task += 128) {
        const int tsel = task >= per ? 1 : 0;
        const int r = task - tsel * per;
        const int wl = r / (D / 8);
        const int j = r - wl * (D / 8);
        const uint32_t* src = words + tsel * C::STAGE_WORDS + wl * D + 8 * j;
        // lanes j and j+4 of a quarter-warp would hit the same banks with
        // 32-byte strided 16-byte loads; odd quads read their halves swapped
        const int sw = (j >> 2) & 1;
        const uint4 a0 = *reinterpret_cast<const uint4*>(src + 4 * sw);
        const uint4 a1 = *reinterpret_cast<const uint4*>(src + 4 * (sw ^ 1));
        const uint4 a = sw ? a1 : a0;
        const uint4 bq = sw ? a0 : a1;
        const uint32_t wd[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
        const uint32_t dst = kvbase + tsel * C::TILE_SZ;
        const int kbase = (wa + wl) * CPW - t.t0;
#pragma unroll
        for (int i = 0; i < CPW; ++i) {
          const int key = kbase + i;
          if (key < 0 || key >= KT) continue;
          uint32_t hv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            hv[u] = codes_to_half2((wd[2 * u] >> (BITS * i)) & C::MASK, (wd[2 * u + 1] >> (BITS * i)) & C::MASK);
          tc::sts128(dst + tc::sw128_offset(key, 8 * j, KT), hv[0], hv[1], hv[2], hv[3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&stg_empty[st]);
      mbar_arrive(&kv_full[kvb]);
    }
  } else if ((tid >> 7) < nqt) {
    // =========================================================== softmax warpgroup qt
    const int qt = tid >> 7;
    const int row = tid & 127;
    const int q0 = cta_q0 + qt * 128;
    const bool row_valid = (q0 + row) < p.n_q;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t col_u = C::COL_U + qt * D;
    const uint32_t col_o = C::COL_O + qt * D;
    const uint32_t qb = sbase + C::Q0 + qt * 2 * C::Q_SZ;
    const uint16_t* qrow = p.q + b * p.q_sb + h * p.q_sh + static_cast<int64_t>(q0 + row) * p.q_st;
    // each query tile keeps its own three meta buffers (blocks kb % 3): the
    // tiles of a CTA may be up to two key tiles apart
    auto meta_of = [&](int kb) { return reinterpret_cast<float*>(sm + C::META) + (qt * 3 + kb % 3) * 4 * D; };
    // named barrier among this warpgroup's 128 threads only
    auto wg_sync = [&]() { asm volatile("bar.sync %0, 128;" ::"r"(1 + qt) : "memory"); };
    auto load_meta = [&](int kb) {
      float* meta = meta_of(kb);
      for (int c = row; c < D; c += 128) {
        const int64_t mo = kb * BHD + static_cast<int64_t>(bh) * D + c;
        meta[c] = p.scale_k[mo];
        meta[D + c] = p.zero_k[mo];
        meta[2 * D + c] = p.scale_v[mo];
        meta[3 * D + c] = p.zero_v[mo];
      }
    };
    // q' = sigma * q * sk of block kb, scaled by 2^-e, split into fp16 hi/lo
    auto build_q = [&](int kb, float& bias_out, float& up_out) {
      const float* meta = meta_of(kb);
      float bias = 0.0f, amax = 0.0f;
      for (int c2 = 0; c2 < D / 2; ++c2) {
        const uint32_t w = row_valid ? reinterpret_cast<const uint32_t*>(qrow)[c2] : 0u;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float qv = __uint_as_float(u ? (w & 0xffff0000u) : (w << 16));
          const float qs = __fmul_rn(p.softmax_scale, qv);
          amax = fmaxf(amax, fabsf(__fmul_rn(qs, meta[2 * c2 + u])));
          bias = fmaf(qs, meta[D + 2 * c2 + u], bias);
        }
      }
      int e = 0;
      if (amax > 0.0f) {
        const int ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127;
        e = max(-100, min(100, ex - 10));
      }
      const float down = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
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
            const float qv = __uint_as_float(u ? (w4[k2] & 0xffff0000u) : (w4[k2] << 16));
            x[u] = __fmul_rn(__fmul_rn(__fmul_rn(p.softmax_scale, qv), meta[c8 + 2 * k2 + u]), down);
          }
          const __half2 hh = __floats2half2_rn(x[0], x[1]);
          const float2 hf = __half22float2(hh);
          hi[k2] = *reinterpret_cast<const uint32_t*>(&hh);
          lo[k2] = pack_half2(x[0] - hf.x, x[1] - hf.y);
        }
        const uint32_t off = tc::sw128_offset(row, c8, 128);
        tc::sts128(qb + off, hi[0], hi[1], hi[2], hi[3]);
        tc::sts128(qb + C::Q_SZ + off, lo[0], lo[1], lo[2], lo[3]);
      }
      bias_out = bias;
      up_out = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
    };
    auto fold = [&](int kb, float rsum, bool have_o) {  // O = O + U (.) sv + rsum * zv
      const float* meta = meta_of(kb);
#pragma unroll 1
      for (int c16 = 0; c16 < D; c16 += 16) {
        uint32_t u[16], o[16];
        tc::tmem_ld16(tmem + lane_off + col_u + c16, u);
        if (have_o) tc::tmem_ld16(tmem + lane_off + col_o + c16, o);
        tc::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float base_o = have_o ? __uint_as_float(o[k]) : 0.0f;
          o[k] = __float_as_uint(
              fmaf(__uint_as_float(u[k]), meta[2 * D + c16 + k], fmaf(rsum, meta[3 * D + c16 + k], base_o)));
        }
        tc::tmem_st16(tmem + lane_off + col_o + c16, o);
      }
      tc::tmem_wait_st();
    };
    auto scale_tmem = [&](uint32_t col, float alpha) {
#pragma unroll 1
      for (int c16 = 0; c16 < D; c16 += 16) {
        uint32_t r[16];
        tc::tmem_ld16(tmem + lane_off + col + c16, r);
        tc::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) r[u] = __float_as_uint(__uint_as_float(r[u]) * alpha);
        tc::tmem_st16(tmem + lane_off + col + c16, r);
      }
      tc::tmem_wait_st();
    };

    float bias_q[3], up_q[3];
    load_meta(0);
    wg_sync();
    build_q(0, bias_q[0], up_q[0]);
    fence_proxy_async_smem();
    mbar_arrive(q_full(qt));

    bool ok = true;
    float m_ref = -INFINITY, l_tot = 0.0f, rs = 0.0f;
    bool have_o = false;
    int last_kb = 0;
    WsTile t{0, 0};
    int g = 0;
    for (; t.kb <= p.s; ++g) {
      WsTile nx = t;
      ws_next(p, nx);
      const int nk = min(64, p.blk[t.kb].n - t.t0);
      const int nk16 = (nk + 15) & ~15;
      const bool first = (t.t0 == 0);
      const bool last_of_block = (nx.kb != t.kb);
      if (!(ok = ws_wait(s_full(qt, g & 1), (g >> 1) & 1))) break;
      tc::fence_after_sync();
      // q' for the next block: QK(g) (the last one reading q') has completed
      if (last_of_block && nx.kb <= p.s) {
        load_meta(nx.kb);
        wg_sync();
        build_q(nx.kb, bias_q[nx.kb % 3], up_q[nx.kb % 3]);
        fence_proxy_async_smem();
        mbar_arrive(q_full(qt));
      }
      // fold the previous block once its last PV (tile g-1) is done
      if (first && g >= 1) {
        if (!(ok = ws_wait(p_empty(qt, (g - 1) % NPB), ((g - 1) / NPB) & 1))) break;
        tc::fence_after_sync();
        fold(last_kb, rs, have_o);
        l_tot += rs;
        rs = 0.0f;
        have_o = true;
      }
      last_kb = t.kb;
      // softmax of S[qt][g % 2]
      const float bias = bias_q[t.kb % 3];
      const float up = up_q[t.kb % 3];
      const uint32_t t_s = tmem + lane_off + C::COL_S + qt * 128 + (g & 1) * 64;
      const bool partial = nk < nk16;
      float smax = -INFINITY;
#pragma unroll
      for (int c16 = 0; c16 < 64; c16 += 16) {
        if (c16 < nk16) {
          uint32_t r[16];
          tc::tmem_ld16(t_s + c16, r);
          tc::tmem_wait_ld();
          if (partial) {
#pragma unroll
            for (int u = 0; u < 16; ++u)
              if (c16 + u < nk) smax = fmaxf(smax, __uint_as_float(r[u]));
          } else {
#pragma unroll
            for (int u = 0; u < 16; ++u) smax = fmaxf(smax, __uint_as_float(r[u]));
          }
        }
      }
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
      // PV(g - NPB) has finished reading the P buffer written below; with
      // NPB == 1 that is PV(g-1), which also makes U safe to rescale
      const bool any_rescale = __any_sync(0xffffffffu, rescale);
      if ((NPB == 1 || (any_rescale && !first)) && g >= 1) {
        if (!(ok = ws_wait(p_empty(qt, (g - 1) % NPB), ((g - 1) / NPB) & 1))) break;
        tc::fence_after_sync();
      }
      if (NPB == 2 && g >= 2) {
        if (!(ok = ws_wait(p_empty(qt, g % NPB), ((g - 2) / NPB) & 1))) break;
      }
      if (any_rescale && !first) scale_tmem(col_u, alpha);
      if (any_rescale && have_o) scale_tmem(col_o, alpha);
      constexpr float kLog2e = 1.4426950408889634f;
      const uint64_t up2x2 = tc::f2pack(up * kLog2e, up * kLog2e);
      const float c2 = (bias - m_ref) * kLog2e;
      const uint64_t c2x2 = tc::f2pack(c2, c2);
      const uint64_t neg1x2 = tc::f2pack(-1.0f, -1.0f);
      uint64_t rs2 = tc::f2pack(0.0f, 0.0f);
      const uint32_t pb = sbase + C::P0 + (qt * NPB + g % NPB) * C::P_SZ;
#pragma unroll
      for (int c16 = 0; c16 < 64; c16 += 16) {
        if (c16 < nk16) {
          uint32_t r[16];
          tc::tmem_ld16(t_s + c16, r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c8 = 0; c8 < 16; c8 += 8) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int j0 = c16 + c8 + 2 * u;
              const uint64_t arg =
                  tc::fma2(tc::f2pack(__uint_as_float(r[c8 + 2 * u]), __uint_as_float(r[c8 + 2 * u + 1])), up2x2, c2x2);
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
            const uint32_t off = tc::sw128_offset(row, c16 + c8, 128);
            tc::sts128(pb + off, hi[0], hi[1], hi[2], hi[3]);
            tc::sts128(pb + C::PT_SZ + off, lo[0], lo[1], lo[2], lo[3]);
          }
        }
      }
      rs += tc::f2lo(rs2) + tc::f2hi(rs2);
      // S[qt][g % 2] fully read, P written, U/O rescales complete
      fence_proxy_async_smem();
      tc::fence_before_sync();
      mbar_arrive(s_empty(qt, g & 1));
      mbar_arrive(p_full(qt, g % NPB));
      t = nx;
    }
    // ---- last block: wait for its final PV, fold and write the output
    if (ok && g >= 1) ok = ws_wait(p_empty(qt, (g - 1) % NPB), ((g - 1) / NPB) & 1);
    if (ok && g >= 1) {
      tc::fence_after_sync();
      const float* meta = meta_of(last_kb);
      const float inv = 1.0f / (l_tot + rs);
      const int64_t obase = b * p.o_sb + h * p.o_sh + static_cast<int64_t>(q0 + row) * p.o_st;
#pragma unroll 1
      for (int c16 = 0; c16 < D; c16 += 16) {
        uint32_t u[16], o[16];
        tc::tmem_ld16(tmem + lane_off + col_u + c16, u);
        if (have_o) tc::tmem_ld16(tmem + lane_off + col_o + c16, o);
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
  }

  // ---- teardown: every role has left its loop
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int BITS, int D, int NQT>
cudaError_t launch_attention_ws(const AttnParams& p, cudaStream_t stream) {
  using C = WsCfg<BITS, D, NQT>;
  static bool configured[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(attention_ws_kernel<BITS, D, NQT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  dim3 grid((p.n_q + 128 * NQT - 1) / (128 * NQT), p.B * p.H);
  attention_ws_kernel<BITS, D, NQT><<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace
}  // namespace vq
