// Internal (C++) interface between the C-ABI entry points and the kernels.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace vq {

// One tensor of a quantize+pack launch: the block's input slab and where the
// packed words and per-group scale/zero of that block go.
struct QuantTensor {
  const void* x;        // element (b,h,t,c) at x[b*sb + h*sh + t*st + c]
  int64_t sb, sh, st;   // strides in elements
  uint32_t* packed;     // [B][H][W][D]
  float* scale;         // [B][H][D]
  float* zero;          // [B][H][D]
};

struct QuantParams {
  QuantTensor t[2];     // K then V (or a single tensor)
  int B, H, D;
  int n;                // tokens in the block
  int W;                // word-rows of the block
  int bits;
  int esize;            // 2 (bf16) or 4 (fp32)
  int vecs_per_row;     // D * esize / 16
  int units;            // tensors * B * H
  int P;                // warps per unit (1, 2, 4, 8 or 16)
  int WP;               // word-rows per warp of a unit (ceil(W / P))
  int TL;               // lanes per unit when P == 1 (vecs_per_row * rows per load; 32 / TL units per warp)
  int meta16;           // scale and zero rounded to fp16, codes against that grid
  // ring kernel (ring == 1): each unit's slab is bulk-copied into a shared-memory
  // slot of slot_bytes; RW consumer teams of RG warps, NSLOT slots per team
  int ring;
  int RW;
  int RG;
  int NSLOT;
  int slot_bytes;
};

constexpr int kRingMaxWarps = 12;            // consumer warps per CTA (teams x warps per team)
constexpr int kRingSmemBudget = 200 * 1024;  // bytes of slots per CTA


size_t quant_smem_bytes(int D);
int quant_warps();
cudaError_t launch_quant_pack(const QuantParams& p, cudaStream_t stream);

struct DequantParams {
  const uint32_t* packed;  // [B][H][W][D]
  const float* scale;      // [B][H][D]
  const float* zero;
  float* out;              // [B][H][n][D]
  int B, H, D, n, W, bits;
};
cudaError_t launch_dequant(const DequantParams& p, cudaStream_t stream);

// Conversions between the word-row cache and the storage format the results
// tables count (paper.cuh).
cudaError_t launch_paper_block(int bits, bool pack, const uint32_t* src, uint32_t* dst, int64_t BH, int n, int D,
                               cudaStream_t stream);
cudaError_t launch_paper_meta(bool pack, const float* scale, const float* zero, uint32_t* meta, float* scale_out,
                              float* zero_out, int64_t n, cudaStream_t stream);

// Attention of one block's queries over the packed cache of blocks 0..s.
struct AttnBlockInfo {
  int64_t word_off;  // word offset of block k's packed region (per tensor)
  int n;             // tokens of block k
  int W;             // word-rows of block k
};

constexpr int kMaxBlocks = 64;
constexpr int kMaxDevices = 64;  // per-process device ordinals with cached function attributes

struct AttnParams {
  const uint32_t* packed_k;
  const uint32_t* packed_v;
  const float* scale_k;
  const float* zero_k;
  const float* scale_v;
  const float* zero_v;
  const uint16_t* q;           // bf16
  int64_t q_sb, q_sh, q_st;
  void* out;
  int64_t o_sb, o_sh, o_st;
  int out_f32;                 // 1: float32 output, 0: bf16
  int B, H, D, bits;
  int s;                       // current block
  int n_q;                     // queries (tokens of block s)
  float softmax_scale;
  // fused append (fused != 0): block s's fresh K and V, which the attention
  // CTAs quantize into the cache for their own (batch, head) before attending
  int fused;
  int meta16;                  // the cache's metadata is fp16-valued (quantize against it)
  int x_esize;                 // 2 (bf16) or 4 (float32)
  const void* xk;
  const void* xv;
  int64_t xk_sb, xk_sh, xk_st, xv_sb, xv_sh, xv_st;
  AttnBlockInfo blk[kMaxBlocks];
};
cudaError_t launch_attention(const AttnParams& p, cudaStream_t stream);
bool attention_fusable(const AttnParams& p);

}  // namespace vq
