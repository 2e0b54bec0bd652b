// stream_kernel.cuh -- weight-streaming kernel for few tokens (decode).
//
// With T <= 256 tokens the layer is bound by reading the weight once from HBM
// (drpranayjha.com "AI Infrastructure series, Part 5", section "Reason 2": in
// decode every token needs a read of every weight).  The kernel streams each
// weight byte exactly once with TMA and does the arithmetic on the tensor
// cores with the operands swapped: a 128-row slice of the weight is the MMA's
// M = 128 operand and the (zero-padded) tokens are its N operand, so
//   D[feature, token] = sum_k W[feature, k] * x[token, k]
// accumulates in TMEM.
//
// Work split: CTA (nt, c) of the grid owns output features [128 nt, 128 nt +
// 128) and a contiguous range of the reduction dimension; the `csize` CTAs
// that share an n-tile form one thread-block cluster.
//
// Row-parallel mode (the all-reduce of the row-parallel layer, done on chip):
// the reduction dimension is cut into t shards.  Either a shard is split over
// `jsplit` consecutive CTAs (csize = t * jsplit), or a CTA owns `spc`
// consecutive whole shards (t = csize * spc).  In the second case each shard
// is accumulated from zero in its own TMEM region (two regions, so the MMA
// runs on while the previous shard is drained) and the four epilogue warps fold
// the shard partials, in ascending shard order, into an fp32 running sum held
// in registers.  Column-parallel mode is the same kernel with one shard.
//
// Each CTA writes its fp32 partial [t_pad][128] to its own shared memory.
// After a cluster barrier, CTA r sums rows [r R, (r+1) R) (R = 128 / csize)
// across the cluster in a fixed order through distributed shared memory
// (16-byte loads), adds the bias, applies the activation and stores bf16.
// Nothing intermediate goes to global memory and there are no atomics, so the
// result is bit-identical from run to run for a given shape and t.
//
// Threads: warps 0-3 drain TMEM (warp w may access TMEM lanes 32w..32w+31)
// and do the reduction; warp 4 issues TMA; one thread of warp 5 issues MMAs.
#pragma once

#include "ptx.cuh"

namespace tpb {

struct StreamParams {
  int T;          // tokens (rows of x / out)
  int K;          // reduction dimension
  int N;          // output features
  int kb_total;   // K / 64
  int csize;      // CTAs per cluster along K (1, 2, 4 or 8)
  int jsplit;     // CTAs per reduction group (>= 1); csize / jsplit groups are summed in order
  int spc;        // shards per CTA: accumulation segments, each from zero (>= 1)
  int shards;     // shards of the reduction dimension (1 for column-parallel)
  int t_pad;      // MMA N: tokens rounded up to 16
  int tmem_cols;  // columns of one TMEM region (power of two >= max(32, t_pad))
  int stages;     // smem pipeline depth (<= 8)
  int stage_bytes;
  int act;        // tp_act
  int prefetch_w; // issue the first stages' weight loads before waiting for the previous grid
  const uint16_t* bias;  // [N] or nullptr
  uint16_t* out;         // [T, N]
};

constexpr int kStreamThreads = 192;
constexpr int kStreamProducerWarp = 4;
constexpr int kStreamMmaWarp = 5;
constexpr int kStreamTileM = 128;
constexpr int kStreamTileK = 64;
constexpr int kStreamWBytes = kStreamTileM * kStreamTileK * 2;  // 16 KB
constexpr int kStreamMaxStages = 8;
constexpr int kStreamRunCols = 64;  // register running sum: t_pad <= 64 when spc > 1

// Shared memory layout (dynamic, base rounded up to 1024 B):
//   [0, stages * stage_bytes)   pipeline: per stage W tile (16 KB) then x tile (t_pad * 128 B);
//                               reused after the main loop for the fp32 partial [t_pad][128]
//   then barriers: full[stages], empty[stages], seg_full[2], seg_empty[2], final, tmem slot,
//   abort flag
__host__ __device__ inline int stream_partial_bytes(int t_pad) { return t_pad * kStreamTileM * 4; }

__host__ __device__ inline int stream_data_bytes(int stages, int stage_bytes, int t_pad) {
  int a = stages * stage_bytes;
  int b = stream_partial_bytes(t_pad);
  return a > b ? a : b;
}

__host__ inline int stream_smem_bytes(int stages, int stage_bytes, int t_pad) {
  return 1024 /*alignment slack*/ + stream_data_bytes(stages, stage_bytes, t_pad) +
         (2 * stages + 5) * 8 + 16;
}

// k-block range [lo, hi) of cluster rank `crank`; never straddles a shard.
__host__ __device__ inline void stream_cta_range(const StreamParams& p, int crank, int& lo,
                                                 int& hi) {
  const int kbs = p.kb_total / p.shards;  // k-blocks per shard
  if (p.spc > 1) {
    lo = crank * p.spc * kbs;
    hi = lo + p.spc * kbs;
  } else {
    const int groups = p.csize / p.jsplit;       // == shards covered by the cluster
    const int per_group = p.kb_total / groups;   // k-blocks of one group's range
    const int g = crank / p.jsplit;
    const int sub = crank % p.jsplit;
    lo = g * per_group + (sub * per_group) / p.jsplit;
    hi = g * per_group + ((sub + 1) * per_group) / p.jsplit;
  }
}

__global__ void __launch_bounds__(kStreamThreads, 1)
    stream_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_x, const StreamParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int data_bytes = stream_data_bytes(p.stages, p.stage_bytes, p.t_pad);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + data_bytes);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + p.stages;
  uint64_t* seg_full = bars + 2 * p.stages;       // [2]
  uint64_t* seg_empty = bars + 2 * p.stages + 2;  // [2]
  uint64_t* final_bar = bars + 2 * p.stages + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x;
  const int crank = static_cast<int>(cluster_ctarank());  // == blockIdx.y

  int kb_lo, kb_hi;
  stream_cta_range(p, crank, kb_lo, kb_hi);
  const int nkb = kb_hi - kb_lo;
  const int kb_seg = nkb / p.spc;  // k-blocks per accumulation segment
  const uint32_t tcols_alloc = static_cast<uint32_t>(p.spc > 1 ? 2 * p.tmem_cols : p.tmem_cols);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&seg_full[b]), 1);
      mbar_init(smem_u32(&seg_empty[b]), 4);
    }
    mbar_init(smem_u32(final_bar), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kStreamMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), tcols_alloc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  // the next kernel in the stream may start its own set-up now
  grid_launch_dependents();

  const uint32_t x_bytes = static_cast<uint32_t>(p.t_pad) * kStreamTileK * 2;
  const uint32_t tx_bytes = kStreamWBytes + x_bytes;

  if (warp == kStreamProducerWarp) {
    if (lane == 0) {
      // ---------------- TMA producer
      prefetch_tmap(&tmap_w);
      prefetch_tmap(&tmap_x);
      const uint64_t pol_w = policy_evict_first();
      uint32_t issued = 0u, phases = 0u;  // per stage: a load was issued / its phase bit
      // weights are read-only model parameters: with prefetch_w the first
      // stages' weight tiles are requested before the previous grid finishes
      const int pre = p.prefetch_w ? (nkb < p.stages ? nkb : p.stages) : 0;
      for (int i = 0; i < pre; ++i) {
        const uint32_t st = smem_u32(smem + i * p.stage_bytes);
        mbar_arrive_expect_tx(smem_u32(&full_bar[i]), tx_bytes);
        tma_load_2d_hint(st, &tmap_w, smem_u32(&full_bar[i]), (kb_lo + i) * kStreamTileK,
                         n_tile * kStreamTileM, pol_w);
        issued |= 1u << i;
      }
      grid_dependency_wait();  // activations may come from the previous grid
      for (int i = 0; i < pre; ++i) {
        const uint32_t st = smem_u32(smem + i * p.stage_bytes);
        tma_load_2d(st + kStreamWBytes, &tmap_x, smem_u32(&full_bar[i]),
                    (kb_lo + i) * kStreamTileK, 0);
      }
      for (int i = pre; i < nkb; ++i) {
        const int s = i % p.stages;
        const uint32_t ph = static_cast<uint32_t>(i / p.stages) & 1u;
        if (!wait_parity(smem_u32(&empty_bar[s]), ph ^ 1u, abort_flag)) break;
        const uint32_t st = smem_u32(smem + s * p.stage_bytes);
        mbar_arrive_expect_tx(smem_u32(&full_bar[s]), tx_bytes);
        const int kc = (kb_lo + i) * kStreamTileK;
        tma_load_2d_hint(st, &tmap_w, smem_u32(&full_bar[s]), kc, n_tile * kStreamTileM, pol_w);
        tma_load_2d(st + kStreamWBytes, &tmap_x, smem_u32(&full_bar[s]), kc, 0);
        issued |= 1u << s;
        phases = (phases & ~(1u << s)) | (ph << s);
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA can exit
        for (int s = 0; s < p.stages; ++s)
          if (issued & (1u << s))
            drain_wait(smem_u32(&full_bar[s]), (phases >> s) & 1u, 50ull * 1000ull * 1000ull);
      }
    }
    __syncwarp();
  } else if (warp == kStreamMmaWarp) {
    if (lane == 0) {
      // ---------------- MMA issuer: spc segments, segment g into TMEM region g % 2
      const uint32_t idesc = idesc_bf16_f32(kStreamTileM, p.t_pad);
      bool ok = true;
      int i = 0;
      for (int g = 0; ok && g < p.spc; ++g) {
        const int region = g & 1;
        if (g >= 2) {
          if (!wait_parity(smem_u32(&seg_empty[region]), static_cast<uint32_t>((g >> 1) - 1) & 1u,
                           abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const uint32_t d = tmem_d + static_cast<uint32_t>(region * p.tmem_cols);
        for (int kb = 0; kb < kb_seg; ++kb, ++i) {
          const int s = i % p.stages;
          const uint32_t ph = static_cast<uint32_t>(i / p.stages) & 1u;
          if (!wait_parity(smem_u32(&full_bar[s]), ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * p.stage_bytes);
#pragma unroll
          for (int kk = 0; kk < kStreamTileK / 16; ++kk) {
            umma_bf16(d, desc_kmajor_sw128(st + kk * 32),
                      desc_kmajor_sw128(st + kStreamWBytes + kk * 32), idesc,
                      (kb > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(smem_u32(&empty_bar[s]));
        }
        if (ok) umma_commit(smem_u32(&seg_full[region]));
      }
      if (!ok) {
        // every MMA issued so far must finish before TMEM / smem are released
        umma_commit(smem_u32(final_bar));
        drain_wait(smem_u32(final_bar), 0, 50ull * 1000ull * 1000ull);
      }
    }
    __syncwarp();
  } else {
    // ---------------- warps 0-3: drain TMEM, fold shards in order
    grid_dependency_wait();
    float* part = reinterpret_cast<float*>(smem);
    const int row = warp * 32 + lane;  // TMEM lane == weight row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    if (p.spc == 1) {
      const bool ok = __all_sync(0xffffffffu, wait_parity(smem_u32(&seg_full[0]), 0, abort_flag));
      tc_fence_after();
      // once seg_full completed every MMA is done, so the pipeline buffers are dead
      for (int c0 = 0; c0 < p.t_pad && c0 < p.T; c0 += 16) {
        uint32_t r[16];
        if (ok && nkb > 0) {
          tmem_ld16(tmem_d + lane_addr + static_cast<uint32_t>(c0), r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) r[j] = 0u;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) part[(c0 + j) * kStreamTileM + row] = __uint_as_float(r[j]);
      }
    } else {
      float run[kStreamRunCols];
#pragma unroll
      for (int j = 0; j < kStreamRunCols; ++j) run[j] = 0.0f;
      bool ok = true;
      for (int g = 0; g < p.spc; ++g) {
        const int region = g & 1;
        ok = __all_sync(0xffffffffu,
                        wait_parity(smem_u32(&seg_full[region]), static_cast<uint32_t>(g >> 1) & 1u,
                                    abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint32_t base = tmem_d + lane_addr + static_cast<uint32_t>(region * p.tmem_cols);
#pragma unroll
        for (int c = 0; c < kStreamRunCols / 16; ++c) {
          if (c * 16 < p.t_pad) {
            uint32_t r[16];
            tmem_ld16(base + static_cast<uint32_t>(c * 16), r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float v = __uint_as_float(r[j]);
              run[c * 16 + j] = (g == 0) ? v : run[c * 16 + j] + v;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&seg_empty[region]));
      }
#pragma unroll
      for (int c = 0; c < kStreamRunCols / 16; ++c) {
        if (c * 16 < p.t_pad) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            part[(c * 16 + j) * kStreamTileM + row] = ok ? run[c * 16 + j] : 0.0f;
        }
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == kStreamMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_d, tcols_alloc);
  }

  // ---------------- cluster reduction of the partials, fixed order
  cluster_sync_all();
  if (warp < 4) {
    const int R = kStreamTileM / p.csize;  // rows this CTA finalises (multiple of 16)
    const int row0 = crank * R;
    const int groups4 = R / 4;
    const int total = groups4 * p.T;
    const uint32_t part_base = smem_u32(smem);
    for (int e = threadIdx.x; e < total; e += 128) {
      const int tok = e / groups4;
      const int rr = row0 + (e % groups4) * 4;
      const uint32_t off = part_base + static_cast<uint32_t>((tok * kStreamTileM + rr) * 4);
      float4 v[8];
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (c < p.csize) v[c] = dsmem_ld_f32x4(dsmem_map(off, static_cast<uint32_t>(c)));
      float4 y = make_float4(0.f, 0.f, 0.f, 0.f), ps = y;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (c < p.csize) {
          const int jj = c % p.jsplit;
          if (jj == 0) {
            ps = v[c];
          } else {
            ps.x += v[c].x; ps.y += v[c].y; ps.z += v[c].z; ps.w += v[c].w;
          }
          if (jj == p.jsplit - 1) {
            if (c == p.jsplit - 1) {
              y = ps;
            } else {
              y.x += ps.x; y.y += ps.y; y.z += ps.z; y.w += ps.w;
            }
          }
        }
      }
      const int n = n_tile * kStreamTileM + rr;
      if (n < p.N) {
        float o[4] = {y.x, y.y, y.z, y.w};
        if (p.bias != nullptr) {
          const uint2 bb = *reinterpret_cast<const uint2*>(p.bias + n);
          o[0] += __uint_as_float(bb.x << 16);
          o[1] += __uint_as_float(bb.x & 0xFFFF0000u);
          o[2] += __uint_as_float(bb.y << 16);
          o[3] += __uint_as_float(bb.y & 0xFFFF0000u);
        }
        if (p.act == 1) {
#pragma unroll
          for (int q = 0; q < 4; ++q) o[q] = gelu_tanh_f32(o[q]);
        }
        uint2 packed = make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
        *reinterpret_cast<uint2*>(p.out + static_cast<size_t>(tok) * p.N + n) = packed;
      }
    }
  }
  // peers may still be reading this CTA's partial
  cluster_sync_all();
}

}  // namespace tpb
