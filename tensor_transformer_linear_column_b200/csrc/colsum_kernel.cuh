// colsum_kernel.cuh -- column sums of a bf16 [rows, cols] matrix (the bias
// gradients of the backward pass: db = sum over tokens of the output
// gradient), fp32 accumulation in a fixed order, one bf16 rounding.
#pragma once

#include "ptx.cuh"

namespace tpb {

constexpr int kColsumWarps = 8;

// Block b owns columns [64 b, 64 b + 64); lane l of warp w reads the bf16 pair
// at columns 64 b + 2 l, +1 of rows w, w + 8, w + 16, ... (a warp reads one
// 128-byte row segment per step), then the eight warps' partial sums are added
// in warp order.  The result does not depend on timing.
__global__ void __launch_bounds__(kColsumWarps * 32)
    colsum_kernel(const uint16_t* __restrict__ in, int rows, int cols, uint16_t* __restrict__ out) {
  __shared__ float part[kColsumWarps][64];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x * 64 + 2 * lane;
  float s0 = 0.0f, s1 = 0.0f;
  if (c < cols) {
    const uint32_t* base = reinterpret_cast<const uint32_t*>(in + c);
    const size_t stride = static_cast<size_t>(cols) / 2;  // in 32-bit words
    for (int r = warp; r < rows; r += kColsumWarps) {
      const uint32_t v = __ldg(base + static_cast<size_t>(r) * stride);
      s0 += __uint_as_float(v << 16);
      s1 += __uint_as_float(v & 0xFFFF0000u);
    }
  }
  part[warp][2 * lane] = s0;
  part[warp][2 * lane + 1] = s1;
  __syncthreads();
  if (threadIdx.x < 64) {
    const int col = blockIdx.x * 64 + threadIdx.x;
    float acc = part[0][threadIdx.x];
#pragma unroll
    for (int w = 1; w < kColsumWarps; ++w) acc += part[w][threadIdx.x];
    if (col < cols) {
      const __nv_bfloat16 h = __float2bfloat16_rn(acc);
      out[col] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
}

}  // namespace tpb
