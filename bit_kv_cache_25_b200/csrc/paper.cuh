// The storage format "VAR-Q results data (Tables 2-4)" counts in its KV-memory
// column (Tables 2a/2b): per block one padding-free stream of the block's
// B*H*n*D codes in (b, h, token, channel) order, floor(32/bits) per 32-bit word
// (code i in word i / cpw at bits bits*(i % cpw)), and one 32-bit metadata pair
// per (block, b, h, channel): fp16 scale in the low half, fp16 zero in the high
// half. Its byte count reproduces the printed GiB of every VAR-Q image row.
//
// These kernels convert one layer-tensor cache between the word-row layout the
// attention reads ([B][H][W_s][D] per block, words along tokens) and this
// format, for storage. One thread per output word; the word-row layout is read
// through L1/L2 (each of its words feeds several stream words).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "vq_internal.h"

namespace vq {
namespace {

// Word-row layout of block s (region of B*H*W*D words) -> its stream.
template <int BITS>
__global__ void paper_pack_kernel(const uint32_t* __restrict__ rows, uint32_t* __restrict__ stream, int64_t n_words,
                                  int64_t n_codes, int n, int D, int W) {
  constexpr int CPW = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  const int64_t nd = static_cast<int64_t>(n) * D;
  for (int64_t wi = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; wi < n_words;
       wi += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    uint32_t out = 0u;
#pragma unroll
    for (int i = 0; i < CPW; ++i) {
      const int64_t idx = wi * CPW + i;
      if (idx < n_codes) {
        const int64_t bh = idx / nd;
        const int64_t r = idx - bh * nd;
        const int t = static_cast<int>(r / D);
        const int c = static_cast<int>(r - static_cast<int64_t>(t) * D);
        const uint32_t word = rows[(bh * W + t / CPW) * D + c];
        out |= ((word >> (BITS * (t % CPW))) & MASK) << (BITS * i);
      }
    }
    stream[wi] = out;
  }
}

// Stream of block s -> its word-row layout (padding slots zero).
template <int BITS>
__global__ void paper_unpack_kernel(const uint32_t* __restrict__ stream, uint32_t* __restrict__ rows,
                                    int64_t n_rows_words, int n, int D, int W) {
  constexpr int CPW = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < n_rows_words;
       k += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(k % D);
    const int64_t r = k / D;
    const int w = static_cast<int>(r % W);
    const int64_t bh = r / W;
    uint32_t out = 0u;
#pragma unroll
    for (int i = 0; i < CPW; ++i) {
      const int t = w * CPW + i;
      if (t < n) {
        const int64_t idx = (bh * n + t) * D + c;
        const uint32_t word = stream[idx / CPW];
        out |= ((word >> (BITS * static_cast<int>(idx % CPW))) & MASK) << (BITS * i);
      }
    }
    rows[k] = out;
  }
}

// float32 scale/zero -> 32-bit (fp16 scale | fp16 zero << 16) pairs, and back.
__global__ void paper_meta_pack_kernel(const float* __restrict__ scale, const float* __restrict__ zero,
                                       uint32_t* __restrict__ meta, int64_t n) {
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < n;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t s16 = __half_as_ushort(__float2half_rn(scale[g]));
    const uint32_t z16 = __half_as_ushort(__float2half_rn(zero[g]));
    meta[g] = s16 | (z16 << 16);
  }
}

__global__ void paper_meta_unpack_kernel(const uint32_t* __restrict__ meta, float* __restrict__ scale,
                                         float* __restrict__ zero, int64_t n) {
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < n;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t m = meta[g];
    scale[g] = __half2float(__ushort_as_half(static_cast<unsigned short>(m & 0xffffu)));
    zero[g] = __half2float(__ushort_as_half(static_cast<unsigned short>(m >> 16)));
  }
}

inline int paper_grid(int64_t work) {
  const int64_t g = (work + 255) / 256;
  return static_cast<int>(g < 1 ? 1 : (g > 148 * 8 ? 148 * 8 : g));
}

template <int BITS>
cudaError_t launch_paper_block(bool pack, const uint32_t* src, uint32_t* dst, int64_t BH, int n, int D,
                               cudaStream_t stream) {
  constexpr int CPW = 32 / BITS;
  const int W = (n + CPW - 1) / CPW;
  if (pack) {
    const int64_t codes = BH * n * D;
    const int64_t words = (codes + CPW - 1) / CPW;
    paper_pack_kernel<BITS><<<paper_grid(words), 256, 0, stream>>>(src, dst, words, codes, n, D, W);
  } else {
    const int64_t rows = BH * W * D;
    paper_unpack_kernel<BITS><<<paper_grid(rows), 256, 0, stream>>>(src, dst, rows, n, D, W);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_paper_block(int bits, bool pack, const uint32_t* src, uint32_t* dst, int64_t BH, int n, int D,
                               cudaStream_t stream) {
  switch (bits) {
    case 2: return launch_paper_block<2>(pack, src, dst, BH, n, D, stream);
    case 3: return launch_paper_block<3>(pack, src, dst, BH, n, D, stream);
    case 4: return launch_paper_block<4>(pack, src, dst, BH, n, D, stream);
    case 6: return launch_paper_block<6>(pack, src, dst, BH, n, D, stream);
    case 8: return launch_paper_block<8>(pack, src, dst, BH, n, D, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_paper_meta(bool pack, const float* scale, const float* zero, uint32_t* meta, float* scale_out,
                              float* zero_out, int64_t n, cudaStream_t stream) {
  if (pack)
    paper_meta_pack_kernel<<<paper_grid(n), 256, 0, stream>>>(scale, zero, meta, n);
  else
    paper_meta_unpack_kernel<<<paper_grid(n), 256, 0, stream>>>(meta, scale_out, zero_out, n);
  return cudaGetLastError();
}

}  // namespace vq
