// tiled_kernel.cuh -- persistent tensor-core GEMM for many tokens (prefill).
//
// out[M, N] = epilogue(A[M, K] @ B[N, K]^T) with bf16 operands, fp32
// accumulation in tensor memory (TMEM) and 128 x 256 output tiles.
//
// Roles (320 threads): warp 0 issues TMA loads of A / B k-blocks into a
// 4-stage shared-memory ring; one thread of warp 1 issues tcgen05.mma into one
// of two TMEM accumulators (2 x 256 columns); warps 2..9 drain accumulators
// through registers and store bf16.  The grid is at most one CTA per SM and
// walks the tiles in a grouped order so CTAs running together share operand
// k-blocks in L2.  The accumulator double buffer lets the epilogue of one tile
// overlap the main loop of the next.
//
// Column-parallel mode (one accumulation segment per tile): the epilogue adds
// the bias, applies the activation and rounds once to bf16.  Which shard owns
// a column changes nothing numerically, so the t shards are simply the
// column ranges of the tiles (iloveeagents.com "How do tensor parallelism (TP)
// and pipeline parallelism (PP) split large model weights", section "Example").
//
// Row-parallel mode (t segments per tile): segment s accumulates shard s's
// partial P_s = A[:, K_s] @ B[:, K_s]^T from zero in TMEM; the epilogue warps
// fold P_0, P_1, ... into an fp32 running sum held in registers in ascending
// s, then add the bias once and round once.  That is the all-reduce of the
// row-parallel layer (xingyuzhitong.com "Tensor vs Pipeline Parallelism",
// section "Tensor parallelism: split inside each layer"), done in the GEMM
// epilogue with no partial ever written to global memory.
#pragma once

#include "ptx.cuh"

namespace tpb {

constexpr int kTiledBM = 128;
constexpr int kTiledBN = 256;
constexpr int kTiledBK = 64;
constexpr int kTiledStages = 4;
constexpr int kTiledThreads = 320;
constexpr int kTiledABytes = kTiledBM * kTiledBK * 2;             // 16 KB
constexpr int kTiledBBytes = kTiledBN * kTiledBK * 2;             // 32 KB
constexpr int kTiledStageBytes = kTiledABytes + kTiledBBytes;     // 48 KB
constexpr int kTiledTmemCols = 2 * kTiledBN;                      // 512
constexpr int kTiledEpiWarps = 8;
constexpr int kTiledSmemBytes =
    1024 + kTiledStages * kTiledStageBytes + (2 * kTiledStages + 4 + 1) * 8 + 16;

struct TiledParams {
  int M, N, K;
  int kb_total;   // K / 64
  int segs;       // accumulation segments per tile: 1, or t in row-parallel mode
  int m_tiles, n_tiles, tiles;
  int group_m;    // tiles are walked in groups of group_m row-tiles
  int act;
  int prefetch_w;  // issue the first stages' weight (B) loads before waiting for the previous grid
  const uint16_t* bias;  // [N] or nullptr
  uint16_t* out;         // [M, N]
  // activation-gradient epilogue of the CTA-pair kernel only:
  const uint16_t* aux;   // [M, N] pre-activation z the gradient flows through
  uint16_t* out2;        // [M, N] act(z), written beside the gradient
};

__device__ __forceinline__ void tiled_coords(int tile, const TiledParams& p, int& m, int& n) {
  const int group = p.group_m * p.n_tiles;
  const int g = tile / group;
  const int first_m = g * p.group_m;
  const int rem = p.m_tiles - first_m;
  const int gm = rem < p.group_m ? rem : p.group_m;
  const int r = tile - g * group;
  m = first_m + r % gm;
  n = r / gm;
}

// 32 fp32 values -> bias, activation -> 32 bf16 stored at dst (16-byte aligned).
__device__ __forceinline__ void store_row_chunk32(uint16_t* dst, const float (&v)[32],
                                                  const uint16_t* bias_chunk, int act) {
  float b[32];
  if (bias_chunk != nullptr) {
    const uint4* bp = reinterpret_cast<const uint4*>(bias_chunk);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 u = __ldg(bp + q);
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        b[q * 8 + h * 2 + 0] = __uint_as_float(w4[h] << 16);
        b[q * 8 + h * 2 + 1] = __uint_as_float(w4[h] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) b[j] = 0.0f;
  }
  uint32_t packed[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float a0 = v[2 * j] + b[2 * j];
    float a1 = v[2 * j + 1] + b[2 * j + 1];
    if (act == 1) {
      a0 = gelu_tanh_f32(a0);
      a1 = gelu_tanh_f32(a1);
    }
    packed[j] = pack_bf16x2(a0, a1);
  }
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d4[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
}

template <bool kRowpar>
__global__ void __launch_bounds__(kTiledThreads, 1)
    tiled_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                      const __grid_constant__ CUtensorMap tmap_b, const TiledParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTiledStages * kTiledStageBytes);
  uint64_t* full_bar = bars;                         // [stages]
  uint64_t* empty_bar = bars + kTiledStages;         // [stages]
  uint64_t* tfull_bar = bars + 2 * kTiledStages;     // [2]
  uint64_t* tempty_bar = bars + 2 * kTiledStages + 2;  // [2]
  uint64_t* final_bar = bars + 2 * kTiledStages + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTiledStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull_bar[b]), 1);
      mbar_init(smem_u32(&tempty_bar[b]), kTiledEpiWarps);
    }
    mbar_init(smem_u32(final_bar), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTiledTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the next kernel in the stream may start its own set-up now
  grid_launch_dependents();

  const int kb_seg = p.kb_total / p.segs;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      prefetch_tmap(&tmap_a);
      prefetch_tmap(&tmap_b);
      int last_phase[kTiledStages];
#pragma unroll
      for (int s = 0; s < kTiledStages; ++s) last_phase[s] = -1;
      int it = 0;
      bool ok = true;
      // weights (B) are read-only model parameters: with prefetch_w the first
      // stages' weight tiles are requested before the previous grid finishes
      int pre = 0;
      if (p.prefetch_w && blockIdx.x < p.tiles) {
        int m0, n0;
        tiled_coords(blockIdx.x, p, m0, n0);
        pre = p.kb_total < kTiledStages ? p.kb_total : kTiledStages;
        for (int kb = 0; kb < pre; ++kb) {
          const uint32_t sa = smem_u32(smem + kb * kTiledStageBytes);
          mbar_arrive_expect_tx(smem_u32(&full_bar[kb]), kTiledStageBytes);
          tma_load_2d(sa + kTiledABytes, &tmap_b, smem_u32(&full_bar[kb]), kb * kTiledBK,
                      n0 * kTiledBN);
          last_phase[kb] = 0;
        }
      }
      grid_dependency_wait();  // activations may come from the previous grid
      for (int tile = blockIdx.x; ok && tile < p.tiles; tile += gridDim.x) {
        int m, n;
        tiled_coords(tile, p, m, n);
        for (int kb = 0; kb < p.kb_total; ++kb, ++it) {
          const int s = it % kTiledStages;
          const uint32_t ph = static_cast<uint32_t>(it / kTiledStages) & 1u;
          const uint32_t sa = smem_u32(smem + s * kTiledStageBytes);
          const uint32_t fb = smem_u32(&full_bar[s]);
          if (it < pre) {  // weight half already requested
            tma_load_2d(sa, &tmap_a, fb, kb * kTiledBK, m * kTiledBM);
            continue;
          }
          if (!wait_parity(smem_u32(&empty_bar[s]), ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(fb, kTiledStageBytes);
          tma_load_2d(sa, &tmap_a, fb, kb * kTiledBK, m * kTiledBM);
          tma_load_2d(sa + kTiledABytes, &tmap_b, fb, kb * kTiledBK, n * kTiledBN);
          last_phase[s] = static_cast<int>(ph);
        }
      }
      if (!ok) {
        for (int s = 0; s < kTiledStages; ++s)
          if (last_phase[s] >= 0)
            drain_wait(smem_u32(&full_bar[s]), static_cast<uint32_t>(last_phase[s]),
                       50ull * 1000ull * 1000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(kTiledBM, kTiledBN);
      int it = 0, acc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.tiles; tile += gridDim.x) {
        for (int seg = 0; ok && seg < p.segs; ++seg, ++acc) {
          const int buf = acc & 1;
          const uint32_t aph = static_cast<uint32_t>(acc >> 1) & 1u;
          if (!wait_parity(smem_u32(&tempty_bar[buf]), aph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + static_cast<uint32_t>(buf * kTiledBN);
          for (int kb = 0; kb < kb_seg; ++kb, ++it) {
            const int s = it % kTiledStages;
            const uint32_t ph = static_cast<uint32_t>(it / kTiledStages) & 1u;
            if (!wait_parity(smem_u32(&full_bar[s]), ph, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + s * kTiledStageBytes);
#pragma unroll
            for (int kk = 0; kk < kTiledBK / 16; ++kk) {
              umma_bf16(d, desc_kmajor_sw128(sa + kk * 32),
                        desc_kmajor_sw128(sa + kTiledABytes + kk * 32), idesc,
                        (kb > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(smem_u32(&empty_bar[s]));
          }
          if (ok) umma_commit(smem_u32(&tfull_bar[buf]));
        }
      }
      // every MMA issued by this thread is complete once final_bar flips
      umma_commit(smem_u32(final_bar));
      drain_wait(smem_u32(final_bar), 0, 50ull * 1000ull * 1000ull);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue warps 2..9
    grid_dependency_wait();  // outputs may still be read by the previous grid
    const int q = warp & 3;                   // TMEM lane quarter this warp may access
    const int ch = (warp - 2) >> 2;           // which 128-column half of the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int acc = 0;
    float run[kRowpar ? 128 : 1];
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x) {
      int m, n;
      tiled_coords(tile, p, m, n);
      const int row = m * kTiledBM + q * 32 + lane;
      const int col0 = n * kTiledBN + ch * 128;
      bool ok = true;
      for (int seg = 0; seg < p.segs; ++seg, ++acc) {
        const int buf = acc & 1;
        const uint32_t aph = static_cast<uint32_t>(acc >> 1) & 1u;
        const bool got = wait_parity(smem_u32(&tfull_bar[buf]), aph, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tbase = tmem_base + lane_base + static_cast<uint32_t>(buf * kTiledBN + ch * 128);
        if constexpr (!kRowpar) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tbase + c * 32, r);
            tmem_wait_ld();
            if (c == 3) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(smem_u32(&tempty_bar[buf]));
            }
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
            const int col = col0 + c * 32;
            if (row < p.M && col < p.N)
              store_row_chunk32(p.out + static_cast<size_t>(row) * p.N + col, v,
                                p.bias != nullptr ? p.bias + col : nullptr, p.act);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tbase + c * 32, r);
            tmem_wait_ld();
            if (seg == 0) {
#pragma unroll
              for (int j = 0; j < 32; ++j) run[c * 32 + j] = __uint_as_float(r[j]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) run[c * 32 + j] += __uint_as_float(r[j]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&tempty_bar[buf]));
        }
      }
      if (!ok) break;
      if constexpr (kRowpar) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = run[c * 32 + j];
          const int col = col0 + c * 32;
          if (row < p.M && col < p.N)
            store_row_chunk32(p.out + static_cast<size_t>(row) * p.N + col, v,
                              p.bias != nullptr ? p.bias + col : nullptr, 0);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTiledTmemCols);
  }
}

}  // namespace tpb
