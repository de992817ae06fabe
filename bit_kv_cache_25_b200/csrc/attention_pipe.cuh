// Packed-KV block attention: persistent, warp-specialized, on the sm_100a
// tensor cores (tcgen05.mma, fp32 accumulators in tensor memory, bulk copies).
//
// The queries of block s attend to every cached token of blocks 0..s.
//
// Operands. The cached tokens of blocks 0..s are walked as one sequence, in
// key tiles of KT tokens (64 at head_dim 64, 48 at 128) that may
// span several blocks (at most MAXSEG block segments per tile). Each tile is
// dequantized in shared memory to the cache's own fp32 values
// x^ = fma(code, scale, zero) of each token's block and split into two 16-bit
// parts. K, whose rounding moves every logit, takes fp16, after a power of two
// 2^-e chosen per (batch, head) so that the largest |K^| over blocks 0..s lies
// in [2^14, 2^15): hi = x^ with its mantissa cut to 10 bits (exact in fp16),
// lo = x^ - hi rounded to fp16, so hi + lo = x^ (1 + O(2^-21)). V takes bf16,
// as P does, with no scaling (bf16 has the range of fp32): hi = x^ rounded to
// bf16, lo = x^ - hi rounded to bf16, so hi + lo = x^ (1 + O(2^-16)). (With
// fp16 hi/lo for P alone, or for V alone, or bf16 hi/lo for K, the worst
// output error on the VAR-d30 and Infinity-2B shapes rose to 1e-3 .. 7e-3 of
// the output RMS in a float64 emulation, against 1e-4 here.) The bf16 queries are exact in fp16 after a
// power-of-two scale per row. Per tile, for the 128 query rows of a work item,
// all accumulation in fp32:
//   S  = q . (K^hi + K^lo)^T                      2 fp16 MMAs per 16-wide k-step
//   O += Phi . V^hi + Plo . V^hi + Phi . V^lo     3 bf16 MMAs per 16-key step
// with P = exp(logit - m) split into bf16 hi/lo and written to tensor memory
// over S. The dropped Plo . V^lo term is below 2^-16 of each product. bf16
// has the range of fp32, so P may sit far above its reference maximum without
// overflowing: O is rescaled only when a row maximum grows by more than
// kPipeTau = 40 (natural-log units), which the data essentially never does.
// The scales live in the operands, so O collects every block directly.
//
// Roles of one CTA (one CTA per SM, 512 threads, NQT = 1 or 2 query tiles of
// 128 rows of one (batch, head) per work item):
//   one softmax warpgroup per query tile (one query row per thread,
//     tensor-memory lanes 0-127 of that tile's columns): query load and
//     conversion, online softmax with a lazy reference maximum (O is rescaled
//     in tensor memory only when a row maximum grows by more than kPipeTau),
//     normalisation and output. With two query tiles the two warpgroups take
//     turns on the tensor cores and hide each other's tensor-memory latency;
//   unpack warps (8 with one query tile, 6 with two): staged packed words ->
//     dequantized hi/lo K (fp16) and V (bf16) tiles (ring of NKV slots) shared by the
//     item's query tiles, and the per-(batch, head) powers of two. With a
//     two-slot ring (head_dim 128) K and V of a slot are released and refilled
//     separately: the next K overlaps the PV that still reads this slot's V;
//   producer warp, one thread: bulk copies of each tile's packed K/V word
//     rows and of its blocks' scale/zero vectors into a stage ring;
//   MMA warp: every tcgen05.mma and commit, issued by one elected lane while
//     the whole warp runs the (warp-uniform) loop, with shared-memory
//     descriptors built once and advanced by constant offsets: QK^T of tile g
//     for each query tile, then PV of tile g-1 for each (the hi/lo parts of one
//     k-step back to back). At head_dim 64 the QK^T MMAs read q from tensor
//     memory (written there by the softmax warpgroup), K from shared memory.
// The CTA is persistent: it walks work items (batch*head, group of NQT query
// tiles) with a stride of gridDim.x. Every ring runs on across items, so the
// next item's copies, unpacking and first QK^T overlap this item's last tiles,
// and an item's output is written while the next item's first softmax is done.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tc_ptx.cuh"
#include "vq_device.cuh"
#include "vq_internal.h"

namespace vq {
namespace {

// lazy-rescale threshold (natural-log units): p <= e^40 < 2^58 as bf16, and
// O <= 2^15 * e^40 * (2^15 keys) stays far below the fp32 maximum
constexpr float kPipeTau = 40.0f;
constexpr float kPipeHead = 2.5f;  // an item's first reference maximum sits this far above its first tile's
constexpr int kPipeMaxTable = 4096;  // tiles per item whose key counts are tabled in shared memory

template <int BITS, int D, int NQT>
struct PipeCfg {
  static constexpr int KT = (D == 64) ? 64 : 48;           // keys per tile: S of a row fits in registers
  static constexpr int CPW = 32 / BITS;
  static constexpr uint32_t MASK = (1u << BITS) - 1u;
  static constexpr int MAXSEG = (D == 64) ? 8 : 4;         // block segments per tile
  static constexpr int MAXROWS = (KT + CPW - 1) / CPW + 2 * MAXSEG;  // staged word rows per tensor
  static constexpr int TM_QT = 512 / NQT;                  // tensor-memory columns per query tile
  // head_dim 64: the queries live in tensor memory (the QK^T MMAs then read
  // only K from shared memory); at 128 their D/2 columns do not fit
  static constexpr bool Q_TMEM = (D == 64);
  static constexpr int NS = (NQT == 1) ? 4 : 2;            // S slots per query tile
  static constexpr int NKV = (D == 64) ? 4 : (NQT == 1 ? 3 : 2);  // K/V tile slots
  // packed-word stages: a third fits only at head_dim 64 with at least 8 codes per word
  static constexpr int NSTG = (D == 64 && BITS <= 4) ? 3 : 2;
  // K and V of a tile are unpacked as two phases, each announced on its own,
  // when the K/V ring is short (K of a later tile then overlaps the PV that
  // still holds the slot's V); otherwise as one
  static constexpr bool SPLIT_KV = (NKV <= 2);
  static constexpr bool STAGE_Q = (D == 64);               // queries of later items prefetched by cp.async
  static constexpr int QPF = (STAGE_Q && NQT == 1) ? 2 : 1;  // items ahead the query staging runs
  static constexpr int UNPACK_WARPS = (NQT == 1) ? 8 : 6;
  static constexpr int UNPACK_THREADS = UNPACK_WARPS * 32;
  // Warp roles: softmax warps 0 .. 4 NQT - 1 (warp w reads tensor-memory lanes
  // 32 (w % 4) ..), then the unpack warps, the producer and the MMA warp. (With
  // the MMA warp and the producer moved next to the softmax warps only, the
  // MMA issue was no faster: the tensor pipe itself takes 68-93 cycles per
  // M=128, K=16 MMA of N <= 128, and the unpack warps lost a sub-partition.)
  static constexpr int SOFTMAX_WARPS = 4 * NQT;
  static constexpr int UNPACK_T0 = SOFTMAX_WARPS * 32;
  static constexpr int PROD_WARP = SOFTMAX_WARPS + UNPACK_WARPS;
  static constexpr int MMA_WARP = PROD_WARP + 1;
  static constexpr int THREADS = (MMA_WARP + 1) * 32;
  // index of warp w among the unpack warps, -1 for the other roles
  static __host__ __device__ constexpr int unpack_index(int w) {
    return (w < SOFTMAX_WARPS || w >= PROD_WARP) ? -1 : w - SOFTMAX_WARPS;
  }
  // ---- shared memory (byte offsets from a 1024-aligned base)
  static constexpr int Q_SZ = Q_TMEM ? 0 : 128 * D * 2;    // fp16 q [128][D] per query tile, K-major SW128
  static constexpr int Q0 = 0;
  static constexpr int TILE_SZ = KT * D * 2;               // 16-bit [KT][D], K-major SW128
  static constexpr int KV0 = Q0 + NQT * Q_SZ;              // NKV x {K hi, K lo, V hi, V lo}
  static constexpr int KV_SZ = 4 * TILE_SZ;
  static constexpr int QST0 = KV0 + NKV * KV_SZ;           // QPF x bf16 [128][D] query staging per query tile
  static constexpr int QST_SZ = STAGE_Q ? 128 * D * 2 : 0;
  static constexpr int STG0 = QST0 + NQT * QPF * QST_SZ;         // NSTG x {K rows, V rows, meta, segment table}
  static constexpr int STG_V = MAXROWS * D * 4;
  static constexpr int STG_META = 2 * STG_V;               // MAXSEG x [4][D] fp32: sk, zk, sv, zv
  static constexpr int STG_SEG = STG_META + MAXSEG * 4 * D * 4;  // MAXSEG x int4 {block, u0, take, key0}
  static constexpr int STG_ROWS = STG_SEG + MAXSEG * 16;   // MAXSEG x {first staged row, rows}, segment count
  static constexpr int STG_SZ = STG_ROWS + (2 * MAXSEG + 4) * 4;
  static constexpr int HDR0 = STG0 + NSTG * STG_SZ;        // NKV x {2^eK, 2^eV, -, -}
  static constexpr int NRED = 5;                           // exponent reduction slots (> NKV)
  static constexpr int RED0 = HDR0 + NKV * 16;             // NRED x UNPACK_WARPS floats (K maxima)
  static constexpr int BARS = RED0 + NRED * UNPACK_WARPS * 4;
  static constexpr int QBARS = 1 + 3 * NS;                 // per query tile: q_full, s_full, p_full, pv_done
  static constexpr int NBARS = 2 * NSTG + 4 * NKV + NRED + NQT * QBARS;
  static constexpr int TMEM_SLOT = BARS + NBARS * 8;
  static constexpr int NKTAB = TMEM_SLOT + 16;             // kPipeMaxTable x uint8: keys of each tile of an item
  static constexpr int SMEM = NKTAB + kPipeMaxTable;
  static constexpr int SMEM_ALLOC = SMEM + 1024;           // room to align the base
  static_assert(THREADS <= 512, "one CTA per SM at 128 registers per thread");
  static_assert(KV0 % 1024 == 0 && TILE_SZ % 1024 == 0 && Q_SZ % 1024 == 0, "operand alignment");
  static_assert(STG0 % 16 == 0 && STG_SZ % 16 == 0 && STG_V % 16 == 0 && STG_META % 16 == 0, "stage alignment");
  static_assert(HDR0 % 16 == 0 && BARS % 8 == 0, "header alignment");
  static_assert(SMEM_ALLOC <= 232448, "shared memory per CTA");
  static_assert(NRED > NKV, "exponent slots");
  // ---- tensor memory: query tile qt owns columns [qt * TM_QT, +TM_QT): NS S
  // slots of KT columns, then O (D columns), then (Q_TMEM) q as fp16 pairs:
  // column COL_Q + c/2 holds channels c, c+1 of the lane's query row
  static constexpr int COL_O = NS * KT;
  static constexpr int COL_Q = COL_O + D;
  static constexpr int TMEM_COLS = 512;
  static_assert(NS * KT + D + (Q_TMEM ? D / 2 : 0) <= TM_QT, "tensor memory");
};

// 16-byte asynchronous copy global -> shared (L2 only); src_bytes = 0 fills zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// 2^e and 2^-e with amax * 2^-e in [2^14, 2^15) (e = 0 for amax == 0; e clamped to [-100, 100]).
__device__ __forceinline__ void pipe_pow2(float amax, float& mul, float& inv) {
  int e = 0;
  if (amax > 0.0f) {
    e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127 - 14;
    e = max(-100, min(100, e));
  }
  mul = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
  inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
}

// Key-tile walker over the tokens of blocks 0..s: a tile takes up to KT tokens
// and at most MAXSEG block segments. (kb, u): the block and the block-relative
// token where the next tile starts.
template <int KT, int MAXSEG>
struct PipeWalk {
  int kb, u;
  __device__ __forceinline__ void reset() { kb = 0, u = 0; }
  // Advances over one tile and returns its key count; seg(i, kb, u0, take,
  // key0) is called for each of its block segments.
  template <typename F>
  __device__ __forceinline__ int next(const AttnParams& p, F&& seg) {
    int nk = 0;
    for (int i = 0; i < MAXSEG && nk < KT && kb <= p.s; ++i) {
      const int take = min(KT - nk, p.blk[kb].n - u);
      seg(i, kb, u, take, nk);
      nk += take;
      u += take;
      if (u >= p.blk[kb].n) {
        ++kb;
        u = 0;
      }
    }
    return nk;
  }
  __device__ __forceinline__ int next(const AttnParams& p) {
    return next(p, [](int, int, int, int, int) {});
  }
};

// ALT (with NQT == 2): every work item is one query tile and the two softmax
// warpgroups take the CTA's items in turn (even, odd), so one item's softmax
// overlaps the other's query conversion, epilogue and tensor-core round trips.
template <int BITS, int D, int NQT, bool ALT>
__global__ void __launch_bounds__(PipeCfg<BITS, D, NQT>::THREADS, 1)
    attention_pipe_kernel(const __grid_constant__ AttnParams p) {
  static_assert(!ALT || NQT == 2, "alternating items need two softmax warpgroups");
  using C = PipeCfg<BITS, D, NQT>;
  constexpr int CPW = C::CPW;
  constexpr int KT = C::KT;
  constexpr int NS = C::NS;
  constexpr int NKV = C::NKV;
  constexpr int NSTG = C::NSTG;
  using Walk = PipeWalk<KT, C::MAXSEG>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char* sm = smem_raw + (sbase - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::BARS);
  uint64_t* stg_full = bars;
  uint64_t* stg_empty = stg_full + NSTG;
  uint64_t* k_full = stg_empty + NSTG;  // K (and, unsplit, V) of a slot unpacked
  uint64_t* v_full = k_full + NKV;      // V of a slot unpacked; the slot's header written
  uint64_t* k_empty = v_full + NKV;     // QK^T of the slot's tile complete
  uint64_t* v_empty = k_empty + NKV;    // PV of the slot's tile complete
  uint64_t* red_bar = v_empty + NKV;
  uint64_t* qbars = red_bar + C::NRED;
  auto q_full = [&](int qt) { return qbars + qt * C::QBARS; };
  auto s_full = [&](int qt, int i) { return qbars + qt * C::QBARS + 1 + i; };
  auto p_full = [&](int qt, int i) { return qbars + qt * C::QBARS + 1 + NS + i; };
  auto pv_done = [&](int qt, int i) { return qbars + qt * C::QBARS + 1 + 2 * NS + i; };
  float* hdr = reinterpret_cast<float*>(sm + C::HDR0);
  float* red = reinterpret_cast<float*>(sm + C::RED0);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::TMEM_SLOT);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int64_t BHD = static_cast<int64_t>(p.B) * p.H * D;
  const int n_qt = (p.n_q + 127) / 128;
  const int n_groups = ALT ? n_qt : (n_qt + NQT - 1) / NQT;
  const int n_items = p.B * p.H * n_groups;
  auto item_nqt = [&](int item) { return ALT ? 1 : min(NQT, n_qt - (item % n_groups) * NQT); };
  // query tiles [qlo, qhi) of the k-th item of this CTA
  auto item_qlo = [&](int k) { return ALT ? (k & 1) : 0; };
  auto item_qhi = [&](int k, int item) { return ALT ? (k & 1) + 1 : item_nqt(item); };
  // key tiles per item (the same for every item), and the key count of each
  // of the first kPipeMaxTable tiles in shared memory (thread 0 writes it; the
  // set-up barrier below publishes it)
  uint8_t* nktab = sm + C::NKTAB;
  int T = 0;
  {
    Walk w;
    w.reset();
    while (w.kb <= p.s) {
      const int nk = w.next(p);
      if (tid == 0 && T < kPipeMaxTable) nktab[T] = static_cast<uint8_t>(nk);
      ++T;
    }
  }
  const bool tabled = T <= kPipeMaxTable;

  // ---- set-up: TMEM (warp 0), barriers (thread 0), zeroed K/V slots (unpack warps)
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < NSTG; ++i) {
      mbar_init(&stg_full[i], 1);
      mbar_init(&stg_empty[i], C::UNPACK_THREADS);
    }
    for (int i = 0; i < NKV; ++i) {
      mbar_init(&k_full[i], C::UNPACK_THREADS);
      mbar_init(&v_full[i], C::UNPACK_THREADS);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < C::NRED; ++i) mbar_init(&red_bar[i], C::UNPACK_WARPS);
    for (int qt = 0; qt < NQT; ++qt) {
      mbar_init(q_full(qt), 4);
      for (int i = 0; i < NS; ++i) {
        mbar_init(s_full(qt, i), 1);
        mbar_init(p_full(qt, i), 4);
        mbar_init(pv_done(qt, i), 1);
      }
    }
    fence_barrier_init();
  }
  if (C::unpack_index(warp) >= 0) {
    // key rows past a tile's valid keys are read by the MMAs (times zero
    // probabilities) and must hold finite values
    for (int i = C::KV0 + (C::unpack_index(warp) * 32 + lane) * 16; i < C::KV0 + NKV * C::KV_SZ;
         i += C::UNPACK_THREADS * 16)
      tc::sts128(sbase + i, 0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // The CTA holds all 512 columns (one CTA per SM), so its allocation starts
  // at lane 0, column 0: the MMA warp then uses constant tensor-memory
  // addresses. Anything else is recorded and every role skips its work.
  const bool tmem_at_zero = (tmem == 0u);
  if (!tmem_at_zero && tid == 0) atomicOr(&g_device_error, kDevErrBadShape);
  if (!tmem_at_zero) {
    // (recorded above: straight to the teardown)
  } else if (warp == C::PROD_WARP) {
    // =========================================================== producer thread
    if (lane == 0) {
      bool ok = true;
      int g = 0;
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
        const int bh = item / n_groups;
        Walk w;
        w.reset();
        for (int j = 0; j < T; ++j, ++g) {
          const int st = g % NSTG;
          if (g >= NSTG && !(ok = mbar_wait_bounded(&stg_empty[st], ((g / NSTG) - 1) & 1))) break;
          unsigned char* stage = sm + C::STG0 + st * C::STG_SZ;
          int4* segt = reinterpret_cast<int4*>(stage + C::STG_SEG);
          int* rows = reinterpret_cast<int*>(stage + C::STG_ROWS);
          // segment table (generic stores, published by the arrive below) and byte count
          int nseg = 0, row0 = 0;
          w.next(p, [&](int i, int kb, int u0, int take, int key0) {
            const int wa = u0 / CPW, wb = (u0 + take - 1) / CPW;
            segt[i] = make_int4(kb, u0, take, key0);
            rows[2 * i] = row0;
            rows[2 * i + 1] = wb - wa + 1;
            row0 += wb - wa + 1;
            nseg = i + 1;
          });
          rows[2 * C::MAXSEG] = nseg;
          constexpr uint32_t kMetaBytes = D * 4;
          mbar_arrive_expect_tx(&stg_full[st],
                                static_cast<uint32_t>(row0) * D * 4 * 2 + static_cast<uint32_t>(nseg) * 4 * kMetaBytes);
          for (int i = 0; i < nseg; ++i) {
            const int4 sg = segt[i];
            const AttnBlockInfo& bi = p.blk[sg.x];
            const int wa = sg.y / CPW;
            const uint32_t bytes = static_cast<uint32_t>(rows[2 * i + 1]) * D * 4;
            const int64_t off = bi.word_off + static_cast<int64_t>(bh) * bi.W * D + static_cast<int64_t>(wa) * D;
            const int64_t mo = sg.x * BHD + static_cast<int64_t>(bh) * D;
            unsigned char* dst = stage + rows[2 * i] * D * 4;
            bulk_copy_g2s(dst, p.packed_k + off, bytes, &stg_full[st]);
            bulk_copy_g2s(dst + C::STG_V, p.packed_v + off, bytes, &stg_full[st]);
            unsigned char* md = stage + C::STG_META + i * 4 * kMetaBytes;
            bulk_copy_g2s(md, p.scale_k + mo, kMetaBytes, &stg_full[st]);
            bulk_copy_g2s(md + kMetaBytes, p.zero_k + mo, kMetaBytes, &stg_full[st]);
            bulk_copy_g2s(md + 2 * kMetaBytes, p.scale_v + mo, kMetaBytes, &stg_full[st]);
            bulk_copy_g2s(md + 3 * kMetaBytes, p.zero_v + mo, kMetaBytes, &stg_full[st]);
          }
        }
      }
    }
  } else if (warp == C::MMA_WARP) {
    // =========================================================== MMA warp
    // The whole warp runs this loop (warp-uniform waits and descriptors); one
    // elected lane issues each tcgen05 instruction. With a single thread
    // running it, consecutive MMAs issued 85-110 cycles apart in the kernel.
    {
      constexpr uint32_t tm = 0u;  // tensor-memory base (checked at set-up)
      constexpr uint32_t kLbo = KT * 128;  // 64-channel groups of a [KT][D] V tile read MN-major
      const uint32_t idesc_pv = tc::idesc_f16_f32(128, D, /*b_mn_major=*/true, /*bf16=*/true);
      const uint64_t qdesc = tc::sw128_desc(sbase + C::Q0);
      const uint64_t kdesc0 = tc::sw128_desc(sbase + C::KV0);
      const uint64_t vdesc0 = tc::sw128_desc_mn(sbase + C::KV0 + 2 * C::TILE_SZ, kLbo);
      // The issue loops stay rolled, to keep this warp's code small (unrolled,
      // the single-thread version issued 100-190 cycles apart: instruction-cache
      // misses on code that no other warp shares).
      auto issue_qk = [&](int qt, int slot, int kvs, int nk16) {
        const uint32_t idesc = tc::idesc_f16_f32(128, nk16);
        const uint64_t kd = kdesc0 + static_cast<uint64_t>((kvs * C::KV_SZ) >> 4);
        const uint32_t d = tm + qt * C::TM_QT + slot * KT;
        constexpr int kSlabA = 128 * 128, kSlabB = KT * 128;
        if constexpr (C::Q_TMEM) {
          // A = q from tensor memory: 8 columns (16 fp16 channels) per k-step
          const uint32_t qa = tm + qt * C::TM_QT + C::COL_Q;
#pragma unroll 1
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t b = kd + static_cast<uint64_t>(((kk >> 2) * kSlabB + (kk & 3) * 32) >> 4);
            tc::mma_f16_ts_warp(d, qa + 8 * kk, b, idesc, kk > 0 ? 1u : 0u);                         // q . K^hi
            tc::mma_f16_ts_warp(d, qa + 8 * kk, b + static_cast<uint64_t>(C::TILE_SZ >> 4), idesc, 1u);  // q . K^lo
          }
        } else {
          const uint64_t qd = qdesc + static_cast<uint64_t>((qt * C::Q_SZ) >> 4);
#pragma unroll 1
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = qd + static_cast<uint64_t>(((kk >> 2) * kSlabA + (kk & 3) * 32) >> 4);
            const uint64_t b = kd + static_cast<uint64_t>(((kk >> 2) * kSlabB + (kk & 3) * 32) >> 4);
            tc::mma_f16_ss_warp(d, a, b, idesc, kk > 0 ? 1u : 0u);                         // q . K^hi
            tc::mma_f16_ss_warp(d, a, b + static_cast<uint64_t>(C::TILE_SZ >> 4), idesc, 1u);  // q . K^lo
          }
        }
        tc::commit_warp(s_full(qt, slot));
      };
      auto issue_pv = [&](int qt, int slot, int kvs, int nk16, bool first) {
        const uint64_t vd = vdesc0 + static_cast<uint64_t>((kvs * C::KV_SZ) >> 4);
        const uint32_t pa = tm + qt * C::TM_QT + slot * KT;
        const uint32_t o = tm + qt * C::TM_QT + C::COL_O;
        const int nkk = nk16 / 16;
        // per 16-key step: (P hi, V hi), (P lo, V hi), (P hi, V lo); P lo sits 8 columns after P hi
#pragma unroll 1
        for (int kk = 0; kk < nkk; ++kk) {
          const uint64_t v = vd + static_cast<uint64_t>((kk * 2048) >> 4);
          const uint32_t a = pa + 16 * kk;
          tc::mma_f16_ts_warp(o, a, v, idesc_pv, (first && kk == 0) ? 0u : 1u);
          tc::mma_f16_ts_warp(o, a + 8, v, idesc_pv, 1u);
          tc::mma_f16_ts_warp(o, a, v + static_cast<uint64_t>(C::TILE_SZ >> 4), idesc_pv, 1u);
        }
        tc::commit_warp(pv_done(qt, slot));
      };

      bool ok = true;
      bool prev = false, prev_first = false;
      int prev_nk16 = 0, prev_qlo = 0, prev_qhi = 0, prev_kvs = 0, prev_g = 0;
      int nq[NQT], iq[NQT], prev_n[NQT];  // per query tile: tiles so far, items so far, last tile
#pragma unroll
      for (int qt = 0; qt < NQT; ++qt) nq[qt] = iq[qt] = prev_n[qt] = 0;
      int g = 0;
      for (int item = blockIdx.x, k = 0; ok && item < n_items; item += gridDim.x, ++k) {
        const int qlo = item_qlo(k), qhi = item_qhi(k, item);
        Walk w;
        w.reset();
        for (int j = 0; j < T; ++j, ++g) {
          const int nk = tabled ? nktab[j] : w.next(p);
          const int nk16 = (nk + 15) & ~15;
          const int kvs = g % NKV;
          if (!(ok = mbar_wait_warp(&k_full[kvs], (g / NKV) & 1))) break;
          if (j == 0) {
#pragma unroll
            for (int qt = 0; qt < NQT; ++qt)
              if (qt >= qlo && qt < qhi && ok) ok = mbar_wait_warp(q_full(qt), iq[qt]++ & 1);
            if (!ok) break;
          }
#pragma unroll
          for (int qt = 0; qt < NQT; ++qt) {
            if (qt >= qlo && qt < qhi && ok) {
              const int n = nq[qt];
              const int slot = n % NS;
              if (n >= NS) ok = mbar_wait_warp(pv_done(qt, slot), ((n / NS) - 1) & 1);
              if (ok) {
                tc::fence_after_sync();
                issue_qk(qt, slot, kvs, nk16);
              }
            }
          }
          if (!ok) break;
          if constexpr (C::SPLIT_KV) tc::commit_warp(&k_empty[kvs]);
          if (prev) {
            if (C::SPLIT_KV && !(ok = mbar_wait_warp(&v_full[prev_kvs], (prev_g / NKV) & 1))) break;
#pragma unroll
            for (int qt = 0; qt < NQT; ++qt) {
              if (qt >= prev_qlo && qt < prev_qhi && ok) {
                const int n = prev_n[qt];
                ok = mbar_wait_warp(p_full(qt, n % NS), (n / NS) & 1);
                if (ok) {
                  tc::fence_after_sync();
                  issue_pv(qt, n % NS, prev_kvs, prev_nk16, prev_first);
                }
              }
            }
            if (!ok) break;
            tc::commit_warp(&v_empty[prev_kvs]);
          }
          prev = true;
          prev_first = (j == 0);
          prev_nk16 = nk16;
          prev_qlo = qlo;
          prev_qhi = qhi;
          prev_kvs = kvs;
          prev_g = g;
#pragma unroll
          for (int qt = 0; qt < NQT; ++qt)
            if (qt >= qlo && qt < qhi) prev_n[qt] = nq[qt]++;
        }
      }
      if (C::SPLIT_KV && ok && prev) ok = mbar_wait_warp(&v_full[prev_kvs], (prev_g / NKV) & 1);
      if (ok && prev) {
#pragma unroll
        for (int qt = 0; qt < NQT; ++qt) {
          if (qt >= prev_qlo && qt < prev_qhi && ok) {
            const int n = prev_n[qt];
            ok = mbar_wait_warp(p_full(qt, n % NS), (n / NS) & 1);
            if (ok) {
              tc::fence_after_sync();
              issue_pv(qt, n % NS, prev_kvs, prev_nk16, prev_first);
            }
          }
        }
        if (ok) tc::commit_warp(&v_empty[prev_kvs]);
      }
    }
  } else if (warp >= C::SOFTMAX_WARPS) {
    // =========================================================== unpack warps
    const int ut = C::unpack_index(warp) * 32 + lane;
    const float cmax = static_cast<float>(C::MASK);
    // Power of two of the k-th item's keys: max |K^| over blocks 0..s.
    // Each warp reduces its share of the scale/zero vectors and posts its
    // maxima in slot k % NRED; the item's first tile reads them all. A warp
    // runs at most NKV - 1 tiles ahead of another, so NRED > NKV slots never
    // alias a slot that is still to be read.
    auto pow2_post = [&](int item, int k) {
      const int bh = item / n_groups;
      float ak = 0.0f;
      // up to kPow2Batch (block, channel) pairs per thread in flight at once
      constexpr int kPow2Batch = 8;
      for (int base = 0; base < (p.s + 1) * D; base += kPow2Batch * C::UNPACK_THREADS) {
        float sk[kPow2Batch], zk[kPow2Batch];
#pragma unroll
        for (int u = 0; u < kPow2Batch; ++u) {
          const int idx = base + u * C::UNPACK_THREADS + ut;
          sk[u] = zk[u] = 0.0f;
          if (idx < (p.s + 1) * D) {
            const int kb = idx / D;
            const int64_t mo = kb * BHD + static_cast<int64_t>(bh) * D + (idx - kb * D);
            sk[u] = __ldcg(p.scale_k + mo);
            zk[u] = __ldcg(p.zero_k + mo);
          }
        }
#pragma unroll
        for (int u = 0; u < kPow2Batch; ++u) ak = fmaxf(ak, fmaxf(fabsf(zk[u]), fabsf(fmaf(cmax, sk[u], zk[u]))));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ak = fmaxf(ak, __shfl_xor_sync(0xffffffffu, ak, o));
      const int slot = k % C::NRED;
      if (lane == 0) {
        red[slot * C::UNPACK_WARPS + (ut >> 5)] = ak;
        mbar_arrive(&red_bar[slot]);
      }
      __syncwarp();
    };
    auto pow2_take = [&](int k, float& kmul, float& kinv) -> bool {
      const int slot = k % C::NRED;
      if (!mbar_wait_bounded(&red_bar[slot], (k / C::NRED) & 1)) return false;
      const float* r = red + slot * C::UNPACK_WARPS;
      float ak = 0.0f;
#pragma unroll
      for (int w = 0; w < C::UNPACK_WARPS; ++w) ak = fmaxf(ak, r[w]);
      pipe_pow2(ak, kmul, kinv);
      return true;
    };

    // V needs no power of two: bf16 hi/lo keeps the cache's values at any magnitude
    constexpr float vmul = 1.0f, vinv = 1.0f;
    float kmul = 1.0f, kinv = 1.0f;
    if (static_cast<int>(blockIdx.x) < n_items) pow2_post(blockIdx.x, 0);
    int g = 0;
    bool ok = true;
    for (int item = blockIdx.x, k = 0; ok && item < n_items; item += gridDim.x, ++k) {
      if (!(ok = pow2_take(k, kmul, kinv))) break;
      for (int j = 0; j < T; ++j, ++g) {
        const int st = g % NSTG;
        const int kvs = g % NKV;
        if (!(ok = mbar_wait_bounded(&stg_full[st], (g / NSTG) & 1))) break;
        // (unsplit, the slot's V release below also covers its K)
        if (C::SPLIT_KV && !(ok = mbar_wait_bounded(&k_empty[kvs], ((g / NKV) & 1) ^ 1))) break;
        const unsigned char* stage = sm + C::STG0 + st * C::STG_SZ;
        const int4* segt = reinterpret_cast<const int4*>(stage + C::STG_SEG);
        const int* rows = reinterpret_cast<const int*>(stage + C::STG_ROWS);
        const int nseg = rows[2 * C::MAXSEG];
        const int R = rows[2 * (nseg - 1)] + rows[2 * (nseg - 1) + 1];  // staged word rows
        const uint32_t kvbase = sbase + C::KV0 + kvs * C::KV_SZ;
        constexpr int OCT = D / 8;
        // task t < R * OCT: K, word row t / OCT, channels 8 (t % OCT) ..; then V likewise
        auto unpack_tasks = [&](int t0, int t1) {
          for (int task = t0 + ut; task < t1; task += C::UNPACK_THREADS) {
            const int tsel = task >= R * OCT ? 1 : 0;
            const int r = task - tsel * R * OCT;
            const int sr = r / OCT;
            const int jj = r - sr * OCT;
            // the segment of staged row sr
            int i = 0;
            while (i + 1 < nseg && rows[2 * (i + 1)] <= sr) ++i;
            const int4 sg = segt[i];  // {block, u0, take, key0}
            const uint32_t* src = reinterpret_cast<const uint32_t*>(stage + tsel * C::STG_V) + sr * D + 8 * jj;
            // lanes jj and jj+4 of a quarter-warp would hit the same banks with
            // 32-byte strided 16-byte loads; odd quads read their halves swapped
            const int sw = (jj >> 2) & 1;
            const uint4 a0 = *reinterpret_cast<const uint4*>(src + 4 * sw);
            const uint4 a1 = *reinterpret_cast<const uint4*>(src + 4 * (sw ^ 1));
            const uint4 a = sw ? a1 : a0;
            const uint4 bq = sw ? a0 : a1;
            const uint32_t wd[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
            const float* meta =
                reinterpret_cast<const float*>(stage + C::STG_META) + (i * 4 + 2 * tsel) * D + 8 * jj;
            const float mul = tsel ? vinv : kinv;
            uint64_t sc2[4], ze2[4];  // scale and zero of the 8 channels, times 2^-e (exact), in pairs
            const uint64_t kMagic2 = tc::f2pack(8388608.0f, 8388608.0f);
            {
              const uint4 s0 = *reinterpret_cast<const uint4*>(meta + 4 * sw);
              const uint4 s1 = *reinterpret_cast<const uint4*>(meta + 4 * (sw ^ 1));
              const uint4 z0 = *reinterpret_cast<const uint4*>(meta + D + 4 * sw);
              const uint4 z1 = *reinterpret_cast<const uint4*>(meta + D + 4 * (sw ^ 1));
              const uint4 sa = sw ? s1 : s0, sb = sw ? s0 : s1;
              const uint4 za = sw ? z1 : z0, zb = sw ? z0 : z1;
              const uint32_t sv8[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
              const uint32_t zv8[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                sc2[u] = tc::f2pack(__uint_as_float(sv8[2 * u]) * mul, __uint_as_float(sv8[2 * u + 1]) * mul);
                ze2[u] = tc::f2pack(__uint_as_float(zv8[2 * u]) * mul, __uint_as_float(zv8[2 * u + 1]) * mul);
              }
            }
            // block token of slot 0 of this word row, and its tile key
            const int ub = (sg.y / CPW + (sr - rows[2 * i])) * CPW;
            const int kbase = sg.w + ub - sg.y;
            const int s_lo = max(0, sg.y - ub), s_hi = min(CPW, sg.y + sg.z - ub);  // valid slots
            // key row r of the [KT][D] tile: byte r * 128 + ((octet ^ (r & 7)) << 4) in its 64-channel slab
            const uint32_t dst = kvbase + tsel * 2 * C::TILE_SZ + (jj >> 3) * KT * 128;
            const uint32_t oct = jj & 7;
#pragma unroll 1
            for (int s = s_lo; s < s_hi; ++s) {
              const int sh = BITS * s;
              const uint32_t row = static_cast<uint32_t>(kbase + s);
              uint32_t hi[4], lo[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                // codes c as the floats 2^23 + c, minus 2^23 (exact), then
                // fma(c, scale, zero) * 2^-e, two channels per packed op
                const uint64_t cb = tc::f2pack(__uint_as_float(((wd[2 * u] >> sh) & C::MASK) | 0x4B000000u),
                                               __uint_as_float(((wd[2 * u + 1] >> sh) & C::MASK) | 0x4B000000u));
                const uint64_t x = tc::fma2(tc::sub2(cb, kMagic2), sc2[u], ze2[u]);
                if (tsel) {
                  // V: bf16 hi rounded to nearest, lo = x - hi (exact in fp32) rounded
                  const uint32_t hb = tc::cvt_bf162(tc::f2lo(x), tc::f2hi(x));
                  const uint64_t l = tc::sub2(x, tc::bf162_to_f2(hb));
                  hi[u] = hb;
                  lo[u] = tc::cvt_bf162(tc::f2lo(l), tc::f2hi(l));
                } else {
                  // K: fp16 hi = x cut to 10 mantissa bits, lo = x - hi rounded
                  const float h0 = __uint_as_float(__float_as_uint(tc::f2lo(x)) & 0xffffe000u);
                  const float h1 = __uint_as_float(__float_as_uint(tc::f2hi(x)) & 0xffffe000u);
                  const uint64_t l = tc::sub2(x, tc::f2pack(h0, h1));
                  hi[u] = tc::cvt_half2(h0, h1);
                  lo[u] = tc::cvt_half2(tc::f2lo(l), tc::f2hi(l));
                }
              }
              const uint32_t off = row * 128 + ((oct ^ (row & 7)) << 4);
              tc::sts128(dst + off, hi[0], hi[1], hi[2], hi[3]);
              tc::sts128(dst + C::TILE_SZ + off, lo[0], lo[1], lo[2], lo[3]);
            }
          }
        };
        if constexpr (C::SPLIT_KV) {
          unpack_tasks(0, R * OCT);
          fence_proxy_async_smem();
          mbar_arrive(&k_full[kvs]);
        }
        // V of this slot's previous tile is free once its PV has completed
        if (!(ok = mbar_wait_bounded(&v_empty[kvs], ((g / NKV) & 1) ^ 1))) break;
        if (j == 0 && ut == 0) {
          hdr[kvs * 4 + 0] = kmul;
          hdr[kvs * 4 + 1] = vmul;
        }
        unpack_tasks(C::SPLIT_KV ? R * OCT : 0, 2 * R * OCT);
        fence_proxy_async_smem();
        mbar_arrive(&stg_empty[st]);
        if constexpr (!C::SPLIT_KV) mbar_arrive(&k_full[kvs]);
        mbar_arrive(&v_full[kvs]);
        // the next item's maxima, while this item's tiles run
        if (j == 0 && item + static_cast<int>(gridDim.x) < n_items) pow2_post(item + gridDim.x, k + 1);
      }
    }
  } else {
    // =========================================================== softmax warpgroup qt
    const int qt = tid >> 7;
    const int row = tid & 127;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tq = tmem + lane_off + qt * C::TM_QT;
    const uint32_t qs = sbase + C::Q0 + qt * C::Q_SZ;
    const uint32_t qst = sbase + C::QST0 + qt * C::QPF * C::QST_SZ;
    // query row held by this thread's tensor-memory lane. With alternating
    // items (one tile of n_q <= 128 queries) the second warpgroup puts its
    // rows at the top of the tile, so the two groups' busy warps sit on
    // different SM sub-partitions when n_q is small.
    const int roff = (ALT && qt == 1) ? 128 - p.n_q : 0;
    auto row_of = [&](int item) {
      return ALT ? row - roff : (item % n_groups) * NQT * 128 + qt * 128 + row;
    };
    auto row_ok = [&](int item) {
      const int r = row_of(item);
      return r >= 0 && r < p.n_q;
    };
    // next item of this CTA in which query tile qt holds queries
    auto next_item = [&](int item) {
      if constexpr (ALT) {
        return item + 2 * static_cast<int>(gridDim.x);
      } else {
        for (item += gridDim.x; item < n_items && item_nqt(item) <= qt; item += gridDim.x) {
        }
        return item;
      }
    };
    auto q_ptr = [&](int item) -> const uint16_t* {
      const int bh = item / n_groups;
      const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
      return p.q + b * p.q_sb + h * p.q_sh + static_cast<int64_t>(row_of(item)) * p.q_st;
    };
    // a later item's query row -> staging buffer `buf` (chunk c of the row at
    // c ^ (row & 7)); one commit group per call, empty when there is no item
    auto stage_q = [&](int item, int buf) {
      if (item < n_items) {
        const bool valid = row_ok(item);
        const uint16_t* src = valid ? q_ptr(item) : p.q;
#pragma unroll
        for (int c = 0; c < D / 8; ++c)
          cp_async16(qst + buf * C::QST_SZ + (row * (D / 8) + (c ^ (row & 7))) * 16, src + 8 * c, valid ? 16u : 0u);
      }
      cp_async_commit();
    };
    // query row of `item` -> fp16 q * 2^-eq in the K-major SW128 A tile; returns 2^eq.
    // Two passes over the row (maximum, then conversion), 8 values at a time.
    auto q_chunk = [&](int item, int buf, int c) -> uint4 {
      if constexpr (C::STAGE_Q) {
        return lds128(sm + C::QST0 + (qt * C::QPF + buf) * C::QST_SZ + (row * (D / 8) + (c ^ (row & 7))) * 16);
      } else {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (row_ok(item)) v = *reinterpret_cast<const uint4*>(q_ptr(item) + 8 * c);
        return v;
      }
    };
    auto convert_q = [&](int item, int buf) -> float {
      // the staging group of `item` is complete once at most QPF - 1 newer ones are pending
      if constexpr (C::STAGE_Q) {
        if constexpr (C::QPF == 2) {
          asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
          cp_async_wait_all();
        }
      }
      // two passes over the row (8 values per 16-byte chunk): the maximum |q|
      // on the magnitudes as packed 16-bit integers (same order as the values)
      // in four independent accumulators, then the conversion
      uint32_t am[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        const uint4 v = q_chunk(item, buf, c);
        am[0] = __vmaxu2(am[0], v.x & 0x7fff7fffu);
        am[1] = __vmaxu2(am[1], v.y & 0x7fff7fffu);
        am[2] = __vmaxu2(am[2], v.z & 0x7fff7fffu);
        am[3] = __vmaxu2(am[3], v.w & 0x7fff7fffu);
      }
      const uint32_t a2 = __vmaxu2(__vmaxu2(am[0], am[1]), __vmaxu2(am[2], am[3]));
      float mul, inv;
      pipe_pow2(__uint_as_float(max(a2 & 0xffffu, a2 >> 16) << 16), mul, inv);
      if constexpr (C::Q_TMEM) {
        // fp16 pairs of the row into this lane's D/2 tensor-memory columns
#pragma unroll 1
        for (int c8 = 0; c8 < D / 16; ++c8) {
          uint32_t h[8];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const uint4 v = q_chunk(item, buf, 2 * c8 + cc);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k)
              h[4 * cc + k] =
                  tc::cvt_half2(__uint_as_float(w[k] << 16) * inv, __uint_as_float(w[k] & 0xffff0000u) * inv);
          }
          tc::tmem_st8(tq + C::COL_Q + 8 * c8, h);
        }
        tc::tmem_wait_st();
        tc::fence_before_sync();
      } else {
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
          const uint4 v = q_chunk(item, buf, c);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          uint32_t h[4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            h[k] = tc::cvt_half2(__uint_as_float(w[k] << 16) * inv, __uint_as_float(w[k] & 0xffff0000u) * inv);
          tc::sts128(qs + tc::sw128_offset(row, 8 * c, 128), h[0], h[1], h[2], h[3]);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full(qt));
      return mul;
    };
    auto epilogue = [&](int item, float l, float vmul) {
      const int r = row_of(item);
      const bool valid = row_ok(item);
      const int bh = item / n_groups;
      const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
      const int64_t obase = b * p.o_sb + h * p.o_sh + static_cast<int64_t>(r) * p.o_st;
      const float scl = vmul / l;
      // 32 columns per round: two loads in flight, one wait
#pragma unroll 1
      for (int c32 = 0; c32 < D; c32 += 32) {
        uint32_t o[32];
#pragma unroll
        for (int k = 0; k < 2; ++k)
          tc::tmem_ld16(tq + C::COL_O + c32 + 16 * k, *reinterpret_cast<uint32_t(*)[16]>(&o[16 * k]));
        tc::tmem_wait_ld();
        if (!valid) continue;
        if (p.out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + obase + c32);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_float4(__uint_as_float(o[4 * k]) * scl, __uint_as_float(o[4 * k + 1]) * scl,
                                 __uint_as_float(o[4 * k + 2]) * scl, __uint_as_float(o[4 * k + 3]) * scl);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + obase + c32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t bf[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              uint32_t pair = 0;
#pragma unroll
              for (int uu = 0; uu < 2; ++uu) {
                const uint32_t x = __float_as_uint(__uint_as_float(o[8 * q + 2 * k + uu]) * scl);
                pair |= ((x + 0x7fffu + ((x >> 16) & 1u)) >> 16) << (16 * uu);
              }
              bf[k] = pair;
            }
            dst[q] = make_uint4(bf[0], bf[1], bf[2], bf[3]);
          }
        }
      }
    };
    // (rare: runs while the tile's S is held in registers, so 16 columns at a time)
    auto scale_o = [&](float alpha) {
#pragma unroll 1
      for (int c16 = 0; c16 < D; c16 += 16) {
        uint32_t r[16];
        tc::tmem_ld16(tq + C::COL_O + c16, r);
        tc::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) r[u] = __float_as_uint(__uint_as_float(r[u]) * alpha);
        tc::tmem_st16(tq + C::COL_O + c16, r);
      }
      tc::tmem_wait_st();
    };
    // S columns [c0, c0 + 64) of slot t_s into sr: 16-column chunks below nk16
    // are loaded, columns from nk on read as -inf
    auto load_s64 = [&](uint32_t t_s, int c0, int nk16, uint32_t (&sr)[64], int nk) {
#pragma unroll
      for (int c16 = 0; c16 < 64; c16 += 16)
        if (c0 + c16 < nk16) tc::tmem_ld16(t_s + c0 + c16, *reinterpret_cast<uint32_t(*)[16]>(&sr[c16]));
      tc::tmem_wait_ld();
      if (c0 + 64 > nk) {
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if (c0 + k >= nk) sr[k] = 0xff800000u;
      }
    };

    bool ok = true;
    int item = blockIdx.x + (ALT ? qt * static_cast<int>(gridDim.x) : 0);
    if (!ALT && item < n_items && item_nqt(item) <= qt) item = next_item(item);
    float qmul = 1.0f;  // 2^eq of the current item's row
    int kq = 0;         // items of this query tile so far (staging buffer of item k: k % QPF)
    if (item < n_items) {
      if constexpr (C::STAGE_Q) {
        stage_q(item, 0);
        if constexpr (C::QPF == 2) stage_q(next_item(item), 1);
      }
      qmul = convert_q(item, 0);
    }
    int g = 0;  // tiles of this query tile so far (S/P slot counter)
    bool epi = false;
    int epi_item = 0;
    float epi_l = 1.0f, epi_vmul = 1.0f;
    bool epi_active = false;
    constexpr float kLog2e = 1.4426950408889634f;
    while (ok && item < n_items) {
      const int nxt = next_item(item);
      // this item's first tile in the CTA-wide tile sequence (K/V slot and header)
      const int gt0 = ((item - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x)) * T;
      const bool warp_active = __any_sync(0xffffffffu, row_ok(item));
      // queries of the item QPF ahead, into the buffer item kq just freed
      if constexpr (C::STAGE_Q) stage_q(C::QPF == 2 ? (nxt < n_items ? next_item(nxt) : n_items) : nxt, kq % C::QPF);
      float up = 0.0f, vmul = 1.0f, m_ref = -INFINITY, l = 0.0f, qmul_next = qmul;
      Walk w;
      w.reset();
      for (int j = 0; j < T; ++j, ++g) {
        const int nk = tabled ? nktab[j] : w.next(p);
        const int nk16 = (nk + 15) & ~15;
        const int slot = g % NS;
        if (!(ok = mbar_wait_bounded(s_full(qt, slot), (g / NS) & 1))) break;
        tc::fence_after_sync();
        if (j == 0) {
          // the unpack warps' powers of two for this item (header of its first tile)
          if (!(ok = mbar_wait_bounded(&v_full[gt0 % NKV], (gt0 / NKV) & 1))) break;
          up = p.softmax_scale * qmul * hdr[(gt0 % NKV) * 4 + 0];
          vmul = hdr[(gt0 % NKV) * 4 + 1];
        }
        // last QK^T of this item has completed: q of the next item can replace it
        if (j == T - 1 && nxt < n_items) qmul_next = convert_q(nxt, (kq + 1) % C::QPF);
        if (warp_active) {
          const uint32_t t_s = tq + slot * KT;
          uint32_t sr[64];
          // pass 1: the tile's row maximum. Columns past nk (within the last
          // 16-column chunk) are set to -inf, which the maximum ignores and
          // pass 2 turns into p = 0.
          float smax = -INFINITY;
#pragma unroll 1
          for (int c0 = 0; c0 < KT; c0 += 64) {
            if (c0 < nk16) {
              load_s64(t_s, c0, nk16, sr, nk);
#pragma unroll
              for (int k = 0; k < 64; k += 4)
                smax = tc::max3(smax, tc::max3(__uint_as_float(sr[k]), __uint_as_float(sr[k + 1]),
                                               __uint_as_float(sr[k + 2])),
                                __uint_as_float(sr[k + 3]));
            }
          }
          const float mx = smax * up;
          float alpha = 1.0f;
          bool rescale = false;
          if (m_ref == -INFINITY) {
            // first tile of the item: start the reference above its maximum so
            // that later tiles rarely need a rescale (p >= e^-kPipeHead here)
            m_ref = mx + kPipeHead;
          } else if (mx > m_ref + kPipeTau) {
            alpha = __expf(m_ref - mx);
            rescale = true;
            m_ref = mx;
          }
          l *= alpha;
          if (__any_sync(0xffffffffu, rescale)) {
            // O holds PV up to tile g-1 once that PV completes
            if (!(ok = mbar_wait_bounded(pv_done(qt, (g - 1) % NS), ((g - 1) / NS) & 1))) break;
            tc::fence_after_sync();
            scale_o(alpha);
          }
          const float up2 = up * kLog2e;
          const float c2 = -m_ref * kLog2e;
          const uint64_t up2v = tc::f2pack(up2, up2), c2v = tc::f2pack(c2, c2);
          uint64_t rs2 = tc::f2pack(0.0f, 0.0f);
          // pass 2: p = 2^(S up log2e - m log2e); hi = p rounded to bf16,
          // lo = p - hi rounded to bf16; both as bf16 pairs in place over S
#pragma unroll 1
          for (int c0 = 0; c0 < KT; c0 += 64) {
            if (c0 < nk16) {
              if (KT > 64) load_s64(t_s, c0, nk16, sr, nk);  // (KT == 64: still in sr from pass 1)
#pragma unroll
              for (int c16 = 0; c16 < 64; c16 += 16) {
                if (c0 + c16 < nk16) {
                  uint32_t hi[8], lo[8];
#pragma unroll
                  for (int u = 0; u < 8; ++u) {
                    // two keys per packed op: t = S up log2e - m log2e, p = 2^t,
                    // hi = bf16(p), lo = bf16(p - hi)
                    const uint64_t t = tc::fma2(tc::f2pack(__uint_as_float(sr[c16 + 2 * u]),
                                                           __uint_as_float(sr[c16 + 2 * u + 1])), up2v, c2v);
                    const float p0 = tc::ex2(tc::f2lo(t)), p1 = tc::ex2(tc::f2hi(t));
                    const uint64_t pp = tc::f2pack(p0, p1);
                    const uint32_t hb = tc::cvt_bf162(p0, p1);
                    const uint64_t l = tc::sub2(pp, tc::bf162_to_f2(hb));
                    rs2 = tc::add2(rs2, pp);
                    hi[u] = hb;
                    lo[u] = tc::cvt_bf162(tc::f2lo(l), tc::f2hi(l));
                  }
                  // keys c0+c16 .. +15: P hi at the 8 columns from c0+c16, lo at the 8 after
                  tc::tmem_st8(t_s + c0 + c16, hi);
                  tc::tmem_st8(t_s + c0 + c16 + 8, lo);
                }
              }
            }
          }
          tc::tmem_wait_st();
          l += tc::f2lo(rs2) + tc::f2hi(rs2);
        }
        // the previous item's output, once its last PV is done (before this
        // item's first PV overwrites O)
        if (j == 0 && epi) {
          epi = false;
          if (epi_active) {
            if (!(ok = mbar_wait_bounded(pv_done(qt, (g - 1) % NS), ((g - 1) / NS) & 1))) break;
            tc::fence_after_sync();
            epilogue(epi_item, epi_l, epi_vmul);
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(qt, slot));
      }
      if (!ok) break;
      epi = true;
      epi_item = item;
      epi_l = l;
      epi_vmul = vmul;
      epi_active = warp_active;
      qmul = qmul_next;
      item = nxt;
      ++kq;
    }
    if (ok && epi && epi_active) {
      if (mbar_wait_bounded(pv_done(qt, (g - 1) % NS), ((g - 1) / NS) & 1)) {
        tc::fence_after_sync();
        epilogue(epi_item, epi_l, epi_vmul);
      }
    }
  }

  // ---- teardown: every role has left its loop
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int BITS, int D, int NQT, bool ALT>
cudaError_t launch_attention_pipe(const AttnParams& p, cudaStream_t stream) {
  using C = PipeCfg<BITS, D, NQT>;
  static bool configured[kMaxDevices] = {};
  static int sms[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(attention_pipe_kernel<BITS, D, NQT, ALT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attention_pipe_kernel<BITS, D, NQT, ALT>, C::THREADS,
                                                      C::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    configured[dev] = true;
  }
  const int n_qt = (p.n_q + 127) / 128;
  const int64_t n_items = static_cast<int64_t>(p.B) * p.H * (ALT ? n_qt : (n_qt + NQT - 1) / NQT);
  if (n_items > (int64_t(1) << 30)) return cudaErrorInvalidConfiguration;
  // one CTA per SM: all 512 tensor-memory columns are this CTA's
  const int grid = static_cast<int>(n_items < sms[dev] ? n_items : sms[dev]);
  attention_pipe_kernel<BITS, D, NQT, ALT><<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace
}  // namespace vq
