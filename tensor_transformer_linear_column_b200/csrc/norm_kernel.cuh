// norm_kernel.cuh -- the sequence-parallel region between two sublayers:
// residual add and RMSNorm, token shard by token shard.
//
// Sequence parallelism splits the parts of a layer that tensor parallelism
// leaves whole (normalisation, dropout) along the sequence inside the
// tensor-parallel group (drpranayjha.com "AI Infrastructure series, Part 5",
// section "What about MoE models and very long prompts?"): after the
// row-parallel linear, shard s keeps only the summed rows of its tokens
// [s T/t, (s+1) T/t) (a reduce-scatter instead of the all-reduce), adds the
// residual stream and normalises those rows; an all-gather hands every token to
// the next column-parallel linear.  On one GPU the row-parallel kernel has
// already summed every row; this kernel is the per-token-shard region, one CTA
// per token row:
//   r = residual + y              (fp32, stored once as bf16)
//   n = r / sqrt(mean_j r_j^2 + eps) * gamma    (from the fp32 r, one bf16 rounding)
// HBM-bound: y and the residual read once, r and n written once.
#pragma once

#include "ptx.cuh"

namespace tpb {

constexpr int kNormThreads = 256;
constexpr int kNormVecPerThread = 8;  // 16-byte pieces a thread keeps: rows up to 16384 wide

// One CTA per token row.  Rows of up to kNormThreads * kNormVecPerThread * 8
// elements are read once: each thread keeps its pieces of r = residual + y in
// fp32 registers between the sum of squares and the normalisation.  Wider
// rows take a second pass that re-reads y and the residual (from L2).
template <bool kInRegisters>
__global__ void __launch_bounds__(kNormThreads)
    add_rmsnorm_kernel(const uint16_t* __restrict__ y, const uint16_t* __restrict__ res,
                       const uint16_t* __restrict__ gamma, int H, float eps,
                       uint16_t* __restrict__ r_out, uint16_t* __restrict__ n_out) {
  __shared__ float warp_sums[kNormThreads / 32];
  grid_dependency_wait();  // y comes from the preceding kernel
  const size_t row = blockIdx.x;
  const uint4* y4 = reinterpret_cast<const uint4*>(y + row * H);
  const uint4* r4 = reinterpret_cast<const uint4*>(res + row * H);
  uint4* ro4 = reinterpret_cast<uint4*>(r_out + row * H);
  const int nvec = H / 8;  // 16-byte pieces of the row
  float keep[kInRegisters ? kNormVecPerThread * 8 : 1];
  // pass 1: r = residual + y, stored; this thread's sum of r^2 in fixed order
  float ss = 0.0f;
#pragma unroll
  for (int k = 0; k < (kInRegisters ? kNormVecPerThread : 1); ++k) {
    for (int v = threadIdx.x + k * kNormThreads; v < nvec;
         v += kInRegisters ? nvec : kNormThreads) {
      const uint4 a = __ldg(y4 + v), b = __ldg(r4 + v);
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
      uint32_t packed[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float r0 = __uint_as_float(bw[q] << 16) + __uint_as_float(aw[q] << 16);
        const float r1 = __uint_as_float(bw[q] & 0xFFFF0000u) + __uint_as_float(aw[q] & 0xFFFF0000u);
        ss = fmaf(r0, r0, ss);
        ss = fmaf(r1, r1, ss);
        packed[q] = pack_bf16x2(r0, r1);
        if constexpr (kInRegisters) {
          keep[k * 8 + 2 * q] = r0;
          keep[k * 8 + 2 * q + 1] = r1;
        }
      }
      ro4[v] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
  }
  // the row's sum: warp butterfly, then the eight warps in order
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = ss;
  __syncthreads();
  float total = warp_sums[0];
#pragma unroll
  for (int w = 1; w < kNormThreads / 32; ++w) total += warp_sums[w];
  const float inv = rsqrtf(total / static_cast<float>(H) + eps);
  // pass 2: n = r * inv * gamma from the fp32 r
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
  uint4* n4 = reinterpret_cast<uint4*>(n_out + row * H);
#pragma unroll
  for (int k = 0; k < (kInRegisters ? kNormVecPerThread : 1); ++k) {
    for (int v = threadIdx.x + k * kNormThreads; v < nvec;
         v += kInRegisters ? nvec : kNormThreads) {
      const uint4 g = __ldg(g4 + v);
      const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
      float rr[8];
      if constexpr (kInRegisters) {
#pragma unroll
        for (int e = 0; e < 8; ++e) rr[e] = keep[k * 8 + e];
      } else {
        const uint4 a = __ldg(y4 + v), b = __ldg(r4 + v);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          rr[2 * q] = __uint_as_float(bw[q] << 16) + __uint_as_float(aw[q] << 16);
          rr[2 * q + 1] = __uint_as_float(bw[q] & 0xFFFF0000u) + __uint_as_float(aw[q] & 0xFFFF0000u);
        }
      }
      uint32_t packed[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        packed[q] = pack_bf16x2(rr[2 * q] * inv * __uint_as_float(gw[q] << 16),
                                rr[2 * q + 1] * inv * __uint_as_float(gw[q] & 0xFFFF0000u));
      n4[v] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
  }
  grid_launch_dependents();
}

}  // namespace tpb
