// pair_kernel.cuh -- persistent tensor-core GEMM on CTA pairs (prefill).
//
// Same arithmetic and epilogues as tiled_kernel.cuh, on 256 x 256 output tiles
// computed by a pair of CTAs on two SMs with one M = 256 tcgen05.mma
// (cta_group::2).  Each CTA of the pair stages only its own 128 rows of A and
// its own half (128 rows) of B per k-block, so per SM the operand traffic from
// L2 is 32 KB per 128 x 256 x 64 step instead of 48 KB, and six stages fit in
// shared memory.
//
// Pair protocol (cluster of 2, rank 0 = leader):
//   * both CTAs' TMA loads complete on the leader's full barrier; only the
//     leader posts the pair's expected byte count;
//   * the leader's single MMA thread waits on that barrier, issues the MMAs and
//     commits to both CTAs' empty / accumulator-full barriers at once;
//   * each CTA's epilogue warps drain their own TMEM rows and release the
//     accumulator by arriving on the leader's accumulator-empty barrier.
// No load uses cluster multicast.
//
// Column-parallel and row-parallel modes are as in tiled_kernel.cuh: the
// row-parallel mode accumulates each of the t shards from zero in its own
// TMEM accumulation segment and the epilogue folds them in ascending order
// (xingyuzhitong.com "Tensor vs Pipeline Parallelism", section "Tensor
// parallelism: split inside each layer": the partial results of the
// row-split layer are summed).
//
// Operand layouts (template flags kAmn, kBmn): an operand is K-major (the
// forward pass: activations [rows, K] and weights [out, in]) or MN-major, read
// straight from a row-major [K][MN] matrix with no transpose in memory (the
// backward pass: dy W2 reads W2 [H, F] with F as N; dz^T x reads dz [T, F] and
// x [T, H] with the tokens as K).  An MN-major 128-row operand half arrives as
// two TMA boxes of 64 MN x 64 K.  The backward pass's third epilogue
// (kEpiDact) multiplies the product by act'(z) for a stored pre-activation z
// and also writes act(z).
#pragma once

#include "ptx.cuh"
#include "tiled_kernel.cuh"

namespace tpb {

constexpr int kPairBM = 256;                              // rows per pair tile
constexpr int kPairBN = 256;
constexpr int kPairBK = 64;
constexpr int kPairStages = 6;
constexpr int kPairThreads = 320;
constexpr int kPairHalfBytes = 128 * kPairBK * 2;         // 16 KB: 128 rows x 64 columns
constexpr int kPairStageBytes = 2 * kPairHalfBytes;       // own A rows + own B half
constexpr int kPairTmemCols = 2 * kPairBN;                // two 256-column accumulators
constexpr int kPairSmemBytes = 1024 + kPairStages * kPairStageBytes + (2 * kPairStages + 5) * 8 + 16;

// epilogues: bias + activation (one segment per tile), the row-parallel shard
// sum (t segments per tile), and the activation gradient (one segment)
constexpr int kEpiAct = 0;
constexpr int kEpiRowpar = 1;
constexpr int kEpiDact = 2;

// 32 fp32 products g at columns [col, col + 32) of one row, and the stored
// pre-activations z at the same places: dst = g * act'(z), dst2 = act(z)
// (act = none: dst = g, dst2 = z), each rounded once to bf16.
__device__ __forceinline__ void store_row_chunk32_dact(uint16_t* dst, uint16_t* dst2,
                                                       const uint16_t* z_chunk,
                                                       const float (&g)[32], int act) {
  const uint4* zp = reinterpret_cast<const uint4*>(z_chunk);
  uint32_t pd[16], ph[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = __ldg(zp + q);
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int j = q * 8 + h * 2;
      const float z0 = __uint_as_float(w4[h] << 16);
      const float z1 = __uint_as_float(w4[h] & 0xFFFF0000u);
      float a0 = z0, a1 = z1, d0 = 1.0f, d1 = 1.0f;
      if (act == 1) {
        gelu_tanh_and_grad_f32(z0, a0, d0);
        gelu_tanh_and_grad_f32(z1, a1, d1);
      }
      pd[q * 4 + h] = pack_bf16x2(g[j] * d0, g[j + 1] * d1);
      ph[q * 4 + h] = pack_bf16x2(a0, a1);
    }
  }
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  uint4* h4 = reinterpret_cast<uint4*>(dst2);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    d4[q] = make_uint4(pd[4 * q], pd[4 * q + 1], pd[4 * q + 2], pd[4 * q + 3]);
    h4[q] = make_uint4(ph[4 * q], ph[4 * q + 1], ph[4 * q + 2], ph[4 * q + 3]);
  }
}

// Load this CTA's 128 rows of one operand for k-block kb into `dst` (16 KB):
// K-major, one box {64 K, 128 rows} at (kb * 64, row0); MN-major, two boxes
// {64 MN, 64 K} at (row0, kb * 64) and (row0 + 64, kb * 64), 8 KB apart.
template <bool kMn>
__device__ __forceinline__ void pair_load_half(uint32_t dst, const CUtensorMap* map,
                                               uint32_t bar_cluster, int kb, int row0) {
  if constexpr (kMn) {
    tma_load_2d_pair(dst, map, bar_cluster, row0, kb * kPairBK);
    tma_load_2d_pair(dst + kPairHalfBytes / 2, map, bar_cluster, row0 + 64, kb * kPairBK);
  } else {
    tma_load_2d_pair(dst, map, bar_cluster, kb * kPairBK, row0);
  }
}

// Descriptor of MMA step kk (K = 16) of a 128-row operand half at `base`.
template <bool kMn>
__device__ __forceinline__ uint64_t pair_desc(uint32_t base, int kk) {
  if constexpr (kMn)
    return desc_mnmajor_sw128(base + static_cast<uint32_t>(kk) * 2048u, kPairHalfBytes / 2);
  else
    return desc_kmajor_sw128(base + static_cast<uint32_t>(kk) * 32u);
}

// 320 threads: registers are granted per group of four warps, so the ten warps
// count as twelve and 168 registers per thread is the ceiling.
template <int kEpi, bool kAmn, bool kBmn>
__global__ void __launch_bounds__(kPairThreads, 1)
    pair_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b, const TiledParams p) {
  constexpr bool kRowpar = kEpi == kEpiRowpar;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPairStages * kPairStageBytes);
  uint64_t* full_bar = bars;                            // [stages] (used in the leader)
  uint64_t* empty_bar = bars + kPairStages;             // [stages]
  uint64_t* tfull_bar = bars + 2 * kPairStages;         // [2]
  uint64_t* tempty_bar = bars + 2 * kPairStages + 2;    // [2] (used in the leader)
  uint64_t* final_bar = bars + 2 * kPairStages + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull_bar[b]), 1);
      mbar_init(smem_u32(&tempty_bar[b]), 2 * kTiledEpiWarps);
    }
    mbar_init(smem_u32(final_bar), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kPairTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // both CTAs' barriers and TMEM exist before any cross-CTA arrival or load
  cluster_sync_all();
  grid_launch_dependents();

  const uint32_t leader_full0 = dsmem_map(smem_u32(&full_bar[0]), 0);
  const uint32_t leader_tempty0 = dsmem_map(smem_u32(&tempty_bar[0]), 0);
  const int kb_seg = p.kb_total / p.segs;
  const int half_row = static_cast<int>(rank) * 128;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs): own A rows and own B half
      prefetch_tmap(&tmap_a);
      prefetch_tmap(&tmap_b);
      uint32_t issued = 0u, phases = 0u;
      int it = 0;
      bool ok = true;
      // weights (B) are read-only model parameters: with prefetch_w the first
      // stages' weight halves are requested before the preceding grid finishes
      int pre = 0;
      if (p.prefetch_w && pair < p.tiles) {
        int m0, n0;
        tiled_coords(pair, p, m0, n0);
        pre = p.kb_total < kPairStages ? p.kb_total : kPairStages;
        for (int kb = 0; kb < pre; ++kb) {
          const uint32_t sa = smem_u32(smem + kb * kPairStageBytes);
          if (leader) mbar_arrive_expect_tx(smem_u32(&full_bar[kb]), 2 * kPairStageBytes);
          pair_load_half<kBmn>(sa + kPairHalfBytes, &tmap_b, leader_full0 + kb * 8, kb,
                               n0 * kPairBN + half_row);
          issued |= 1u << kb;
        }
      }
      grid_dependency_wait();  // activations may come from the preceding grid
      for (int tile = pair; ok && tile < p.tiles; tile += npairs) {
        int m, n;
        tiled_coords(tile, p, m, n);
        for (int kb = 0; kb < p.kb_total; ++kb, ++it) {
          const int s = it % kPairStages;
          const uint32_t ph = static_cast<uint32_t>(it / kPairStages) & 1u;
          const uint32_t sa = smem_u32(smem + s * kPairStageBytes);
          if (it < pre) {  // weight half already requested
            pair_load_half<kAmn>(sa, &tmap_a, leader_full0 + s * 8, kb, m * kPairBM + half_row);
            continue;
          }
          if (!wait_parity(smem_u32(&empty_bar[s]), ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(smem_u32(&full_bar[s]), 2 * kPairStageBytes);
          pair_load_half<kAmn>(sa, &tmap_a, leader_full0 + s * 8, kb, m * kPairBM + half_row);
          pair_load_half<kBmn>(sa + kPairHalfBytes, &tmap_b, leader_full0 + s * 8, kb,
                               n * kPairBN + half_row);
          issued |= 1u << s;
          phases = (phases & ~(1u << s)) | (ph << s);
        }
      }
      if (!ok) {
        // loads already issued must land before shared memory is released
        if (leader) {
          for (int s = 0; s < kPairStages; ++s)
            if (issued & (1u << s))
              drain_wait(smem_u32(&full_bar[s]), (phases >> s) & 1u, 50ull * 1000ull * 1000ull);
        } else {
          // their completion is counted in the leader: allow them ample time
          const unsigned long long t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 2000000ull) {
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer for the pair (leader only)
      const uint32_t idesc = idesc_bf16_f32(kPairBM, kPairBN, kAmn, kBmn);
      int it = 0, acc = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < p.tiles; tile += npairs) {
        for (int seg = 0; ok && seg < p.segs; ++seg, ++acc) {
          const int buf = acc & 1;
          const uint32_t aph = static_cast<uint32_t>(acc >> 1) & 1u;
          if (!wait_parity_cluster(smem_u32(&tempty_bar[buf]), aph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + static_cast<uint32_t>(buf * kPairBN);
          for (int kb = 0; kb < kb_seg; ++kb, ++it) {
            const int s = it % kPairStages;
            const uint32_t ph = static_cast<uint32_t>(it / kPairStages) & 1u;
            if (!wait_parity(smem_u32(&full_bar[s]), ph, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + s * kPairStageBytes);
#pragma unroll
            for (int kk = 0; kk < kPairBK / 16; ++kk) {
              umma_bf16_pair(d, pair_desc<kAmn>(sa, kk), pair_desc<kBmn>(sa + kPairHalfBytes, kk),
                             idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit_pair(smem_u32(&empty_bar[s]), 0x3);
          }
          if (ok) umma_commit_pair(smem_u32(&tfull_bar[buf]), 0x3);
        }
      }
      // every MMA of the pair is complete once final_bar flips
      umma_commit_pair(smem_u32(final_bar), 0x1);
      drain_wait(smem_u32(final_bar), 0, 50ull * 1000ull * 1000ull);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue warps 2..9 (both CTAs): own 128 rows of the tile
    grid_dependency_wait();  // outputs may still be read by the preceding grid
    const int q = warp & 3;
    const int ch = (warp - 2) >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int acc = 0;
    float run[kRowpar ? 128 : 1];
    for (int tile = pair; tile < p.tiles; tile += npairs) {
      int m, n;
      tiled_coords(tile, p, m, n);
      const int row = m * kPairBM + half_row + q * 32 + lane;
      const int col0 = n * kPairBN + ch * 128;
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
        const uint32_t tbase = tmem_base + lane_base + static_cast<uint32_t>(buf * kPairBN + ch * 128);
        if constexpr (!kRowpar) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tbase + c * 32, r);
            tmem_wait_ld();
            if (c == 3) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) {
                if (leader)
                  mbar_arrive(smem_u32(&tempty_bar[buf]));
                else
                  mbar_arrive_remote(leader_tempty0 + buf * 8);
              }
            }
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
            const int col = col0 + c * 32;
            if (row < p.M && col < p.N) {
              const size_t off = static_cast<size_t>(row) * p.N + col;
              if constexpr (kEpi == kEpiDact)
                store_row_chunk32_dact(p.out + off, p.out2 + off, p.aux + off, v, p.act);
              else
                store_row_chunk32(p.out + off, v, p.bias != nullptr ? p.bias + col : nullptr,
                                  p.act);
            }
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
          if (lane == 0) {
            if (leader)
              mbar_arrive(smem_u32(&tempty_bar[buf]));
            else
              mbar_arrive_remote(leader_tempty0 + buf * 8);
          }
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

  // teardown: the pair's MMAs are done (leader drained them) and neither CTA
  // touches the other's shared memory or TMEM after this barrier
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kPairTmemCols);
  }
}

}  // namespace tpb
