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
// 128) and the c-th slice of the reduction dimension.  The `csize` CTAs that
// share an n-tile form one thread-block cluster.  Each writes its fp32
// partial to its own shared memory; after a cluster barrier, CTA r sums the
// partials of rows [r R, (r+1) R) (R = 128 / csize) across the cluster in a
// fixed order through distributed shared memory, adds the bias, applies the
// activation and stores bf16.  Nothing intermediate goes to global memory and
// there are no atomics, so the result is bit-identical from run to run.
//
// Row-parallel mode: the cluster covers the t shards of the reduction
// dimension, `jsplit` CTAs per shard (csize = t * jsplit).  Shard s's partial
// P_s is the in-order sum of its CTAs' partials, each started from zero, and
// the output is ((P_0 + P_1) + ...) + b: the all-reduce of the row-parallel
// layer done on chip.
#pragma once

#include "ptx.cuh"

namespace tpb {

struct StreamParams {
  int T;          // tokens (rows of x / out)
  int K;          // reduction dimension
  int N;          // output features
  int kb_total;   // K / 64
  int csize;      // CTAs per cluster along K
  int shards;     // number of reduction shards the cluster's sum is grouped by (1 for column-parallel)
  int jsplit;     // CTAs per shard (csize / shards)
  int t_pad;      // MMA N: tokens rounded up to 16
  int tmem_cols;  // power of two >= max(32, t_pad)
  int stages;     // smem pipeline depth
  int stage_bytes;
  int act;        // tp_act
  const uint16_t* bias;  // [N] or nullptr
  uint16_t* out;         // [T, N]
};

constexpr int kStreamThreads = 128;
constexpr int kStreamTileM = 128;
constexpr int kStreamTileK = 64;
constexpr int kStreamWBytes = kStreamTileM * kStreamTileK * 2;  // 16 KB

// Shared memory layout (dynamic, base rounded up to 1024 B):
//   [0, stages * stage_bytes)        pipeline: per stage W tile (16 KB) then x tile (t_pad * 128 B)
//                                    (reused after the main loop for the fp32 partial [t_pad][128])
//   then barriers: full[stages], empty[stages], acc_full, tmem slot, abort flag
__host__ __device__ inline int stream_partial_bytes(int t_pad) { return t_pad * kStreamTileM * 4; }

__host__ __device__ inline int stream_data_bytes(int stages, int stage_bytes, int t_pad) {
  int a = stages * stage_bytes;
  int b = stream_partial_bytes(t_pad);
  return a > b ? a : b;
}

__host__ inline int stream_smem_bytes(int stages, int stage_bytes, int t_pad) {
  return 1024 /*alignment slack*/ + stream_data_bytes(stages, stage_bytes, t_pad) +
         (2 * stages + 1) * 8 + 16;
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
  uint64_t* acc_bar = bars + 2 * p.stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * p.stages + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x;
  const int crank = static_cast<int>(cluster_ctarank());  // == blockIdx.y

  // this CTA's k-block range, never straddling a shard boundary
  const int kb_per_shard = p.kb_total / p.shards;
  const int shard = crank / p.jsplit;
  const int sub = crank % p.jsplit;
  const int kb_lo = shard * kb_per_shard + (sub * kb_per_shard) / p.jsplit;
  const int kb_hi = shard * kb_per_shard + ((sub + 1) * kb_per_shard) / p.jsplit;
  const int nkb = kb_hi - kb_lo;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(acc_bar), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), static_cast<uint32_t>(p.tmem_cols));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  // inputs may be produced by the preceding kernel in the stream
  grid_dependency_wait();

  const uint32_t x_bytes = static_cast<uint32_t>(p.t_pad) * kStreamTileK * 2;
  const uint32_t tx_bytes = kStreamWBytes + x_bytes;
  int last_phase[8];  // phase of the latest load issued into each stage (-1 = none)
#pragma unroll
  for (int s = 0; s < 8; ++s) last_phase[s] = -1;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_x);
    const uint64_t pol_w = policy_evict_first();
    for (int i = 0; i < nkb; ++i) {
      const int s = i % p.stages;
      const uint32_t ph = static_cast<uint32_t>(i / p.stages) & 1u;
      if (!wait_parity(smem_u32(&empty_bar[s]), ph ^ 1u, abort_flag)) break;
      const uint32_t st = smem_u32(smem + s * p.stage_bytes);
      mbar_arrive_expect_tx(smem_u32(&full_bar[s]), tx_bytes);
      const int kc = (kb_lo + i) * kStreamTileK;
      tma_load_2d_hint(st, &tmap_w, smem_u32(&full_bar[s]), kc, n_tile * kStreamTileM, pol_w);
      tma_load_2d(st + kStreamWBytes, &tmap_x, smem_u32(&full_bar[s]), kc, 0);
      if (s < 8) last_phase[s] = static_cast<int>(ph);
    }
    if (*abort_flag) {
      // let copies already in flight land before the CTA can exit
      for (int s = 0; s < p.stages && s < 8; ++s)
        if (last_phase[s] >= 0)
          drain_wait(smem_u32(&full_bar[s]), static_cast<uint32_t>(last_phase[s]),
                     50ull * 1000ull * 1000ull);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer (single thread)
    const uint32_t idesc = idesc_bf16_f32(kStreamTileM, p.t_pad);
    bool ok = true;
    for (int i = 0; i < nkb; ++i) {
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
        const uint64_t da = desc_kmajor_sw128(st + kk * 32);
        const uint64_t db = desc_kmajor_sw128(st + kStreamWBytes + kk * 32);
        umma_bf16(tmem_d, da, db, idesc, (i > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(smem_u32(&empty_bar[s]));
    }
    // signals the epilogue (and, on the error path, that issued MMAs are done)
    umma_commit(smem_u32(acc_bar));
    if (!ok) drain_wait(smem_u32(acc_bar), 0, 50ull * 1000ull * 1000ull);
  }
  __syncwarp();

  // ---------------- partial: TMEM -> registers -> own shared memory [t_pad][128] fp32
  float* part = reinterpret_cast<float*>(smem);
  // block-uniform (the TMEM loads below are warp-collective); the barrier also
  // orders the producer's and issuer's error-path drains before the pipeline
  // buffers are reused: they are dead once acc_bar completed (all MMAs done)
  const bool have_acc = __syncthreads_and(wait_parity(smem_u32(acc_bar), 0, abort_flag) ? 1 : 0) != 0;
  tc_fence_after();
  const int row = warp * 32 + lane;  // TMEM lane == weight row within the tile
  for (int c0 = 0; c0 < p.t_pad; c0 += 16) {
    if (c0 >= p.T) break;
    uint32_t r[16];
    if (have_acc && nkb > 0) {
      tmem_ld16(tmem_d + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c0), r);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) r[j] = 0u;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) part[(c0 + j) * kStreamTileM + row] = __uint_as_float(r[j]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem_d, static_cast<uint32_t>(p.tmem_cols));

  // ---------------- cluster reduction of the partials, fixed order
  cluster_sync_all();
  {
    const int R = kStreamTileM / p.csize;  // rows this CTA finalises
    const int row0 = crank * R;
    const int total = R * p.T;
    const uint32_t part_base = smem_u32(part);
    for (int e = threadIdx.x; e < total; e += kStreamThreads) {
      const int tok = e / R;
      const int rr = row0 + (e % R);
      const int n = n_tile * kStreamTileM + rr;
      const uint32_t off = part_base + static_cast<uint32_t>((tok * kStreamTileM + rr) * 4);
      float y = 0.0f;
      for (int s = 0; s < p.shards; ++s) {
        float ps = dsmem_ld_f32(dsmem_map(off, static_cast<uint32_t>(s * p.jsplit)));
        for (int j = 1; j < p.jsplit; ++j)
          ps += dsmem_ld_f32(dsmem_map(off, static_cast<uint32_t>(s * p.jsplit + j)));
        y = (s == 0) ? ps : y + ps;
      }
      if (n < p.N) {
        if (p.bias != nullptr) y += bf16_to_f32(p.bias[n]);
        if (p.act == 1) y = gelu_tanh_f32(y);
        __nv_bfloat16 o = __float2bfloat16_rn(y);
        p.out[static_cast<size_t>(tok) * p.N + n] = *reinterpret_cast<uint16_t*>(&o);
      }
    }
  }
  // peers may still be reading this CTA's partial
  cluster_sync_all();
  grid_launch_dependents();
}

}  // namespace tpb
