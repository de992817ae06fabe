// Check-only dequantization of one packed block: x_hat = fma(code, scale, zero)
// (one float32 rounding), the inverse map of the asymmetric min/max grid of
// "VAR-Q: Tuning-Free KV Cache Quantization ...", Abstract, paragraph 3.
// One thread per packed word; a warp covers 32 consecutive channels, so each
// token row it writes is a coalesced 128-byte store.
#include <cuda_runtime.h>

#include <cstdint>

#include "vq_internal.h"

namespace vq {
namespace {

template <int BITS>
__global__ void dequant_kernel(const __grid_constant__ DequantParams p) {
  constexpr int CPW = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  const int64_t total = static_cast<int64_t>(p.B) * p.H * p.W * p.D;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % p.D);
    const int64_t r = idx / p.D;
    const int w = static_cast<int>(r % p.W);
    const int64_t bh = r / p.W;
    const uint32_t word = p.packed[idx];
    const float s = p.scale[bh * p.D + c];
    const float z = p.zero[bh * p.D + c];
    float* out = p.out + (bh * p.n + static_cast<int64_t>(w) * CPW) * p.D + c;
#pragma unroll
    for (int i = 0; i < CPW; ++i) {
      if (w * CPW + i < p.n) {
        const float code = static_cast<float>((word >> (BITS * i)) & MASK);
        out[static_cast<int64_t>(i) * p.D] = __fmaf_rn(code, s, z);
      }
    }
  }
}

}  // namespace

cudaError_t launch_dequant(const DequantParams& p, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(p.B) * p.H * p.W * p.D;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int grid = static_cast<int>(want < 148 * 16 ? (want < 1 ? 1 : want) : 148 * 16);
  switch (p.bits) {
    case 2: dequant_kernel<2><<<grid, threads, 0, stream>>>(p); break;
    case 3: dequant_kernel<3><<<grid, threads, 0, stream>>>(p); break;
    case 4: dequant_kernel<4><<<grid, threads, 0, stream>>>(p); break;
    case 6: dequant_kernel<6><<<grid, threads, 0, stream>>>(p); break;
    case 8: dequant_kernel<8><<<grid, threads, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace vq
