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
// runs on while the previous shard is drained) and the four epilogue warps
// fold the shard partials, in ascending shard order, into an fp32 running sum
// held in registers.  Column-parallel mode is the same kernel with one shard.
//
// Cross-CTA sum: CTA r of the cluster owns rows [r R, (r+1) R) of the tile
// (R = 128 / csize).  Every CTA stages its fp32 partial per owner in its idle
// pipeline buffers and sends each owner its rows with one bulk shared-memory
// copy (cp.async.bulk, cluster scope) whose bytes complete on an mbarrier in
// the owner; each owner waits for exactly those bytes, sums the csize partials
// of its rows in a fixed order from its own shared memory, adds the bias,
// applies the activation and stores bf16.  Nothing intermediate goes to global memory and there are no
// atomics, so the result is bit-identical from run to run for a given shape
// and t.
//
// Weight traffic: a ring of 3-8 stages, deeper for CTAs that stream longer;
// with static weights the first stages are requested before the kernel waits
// for the preceding grid, overlapping that grid's tail.
//
// Threads: warps 0-3 drain TMEM (warp w may access TMEM lanes 32w..32w+31),
// push and reduce; warp 4 issues TMA; one thread of warp 5 issues MMAs.
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
  int prefetch_w; // weights may be read before the preceding grid completes
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
//   [0, stages * stage_bytes)   pipeline: per stage W tile (16 KB) then x tile (t_pad * 128 B)
//   [.., + recv_bytes)          receive buffer [csize][T][R] fp32 (<= 128 * t_pad * 4 bytes)
//   After the main loop the pipeline buffers hold the staging [owner][T][R] fp32 of this CTA's
//   partial (so stages * stage_bytes >= 128 * T * 4 is required: T <= 128).
//   then barriers: full[stages], empty[stages], seg_full[2], seg_empty[2], final, recv,
//   tmem slot, abort flag
// (no receive buffer when the cluster is a single CTA: it stores directly)
__host__ __device__ inline int stream_recv_bytes(int t_pad, int csize) {
  return csize > 1 ? t_pad * kStreamTileM * 4 : 0;
}

__host__ __device__ inline int stream_data_bytes(int stages, int stage_bytes, int t_pad, int csize) {
  return stages * stage_bytes + stream_recv_bytes(t_pad, csize);
}

__host__ inline int stream_smem_bytes(int stages, int stage_bytes, int t_pad, int csize) {
  return 1024 /*alignment slack*/ + stream_data_bytes(stages, stage_bytes, t_pad, csize) +
         (2 * stages + 6) * 8 + 16;
}

// Epilogue of one value: bias, activation, round to bf16, store.
__device__ __forceinline__ void stream_store(const StreamParams& p, int tok, int n, float v,
                                             float bias) {
  v += bias;
  if (p.act == 1) v = gelu_tanh_f32(v);
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  p.out[static_cast<size_t>(tok) * p.N + n] = *reinterpret_cast<uint16_t*>(&h);
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

// kShards = false: one accumulation segment per CTA (spc == 1); registers are
// bounded so three CTAs fit on an SM (six warps are granted registers as
// eight), which lets the next call's CTAs start and prefetch weights while
// this call drains.  kShards = true: several shards per CTA (spc >= 1).
template <bool kShards>
__global__ void __launch_bounds__(kStreamThreads, kShards ? 1 : 3)
    stream_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_x, const StreamParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* recv = reinterpret_cast<float*>(smem + p.stages * p.stage_bytes);
  const int data_bytes = stream_data_bytes(p.stages, p.stage_bytes, p.t_pad, p.csize);
  const bool multi = p.csize > 1;  // partials are summed across a cluster
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + data_bytes);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + p.stages;
  uint64_t* seg_full = bars + 2 * p.stages;       // [2]
  uint64_t* seg_empty = bars + 2 * p.stages + 2;  // [2]
  uint64_t* final_bar = bars + 2 * p.stages + 4;
  uint64_t* recv_bar = bars + 2 * p.stages + 5;  // bytes of the peers' partials for my rows
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(recv_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x;
  const int crank = static_cast<int>(cluster_ctarank());  // == blockIdx.y
  const int R = kStreamTileM / p.csize;                   // rows each CTA finalises

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
    mbar_init(smem_u32(recv_bar), 1);
    // expect csize partials of T x R fp32 before any peer can send (phase 1)
    mbar_arrive_expect_tx(smem_u32(recv_bar), static_cast<uint32_t>(p.csize * p.T * R * 4));
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
  // cluster phase 1: "this CTA has started" (waited on before any remote copy)
  if (multi) cluster_arrive_relaxed();
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
      const int w_row = n_tile * kStreamTileM;
      uint32_t issued = 0u, phases = 0u;  // per stage: a load was issued / its phase bit
      // weights are read-only model parameters: with prefetch_w the first
      // stages' weight tiles are requested before the preceding grid finishes
      const int pre = p.prefetch_w ? (nkb < p.stages ? nkb : p.stages) : 0;
      for (int i = 0; i < pre; ++i) {
        const uint32_t st = smem_u32(smem + i * p.stage_bytes);
        mbar_arrive_expect_tx(smem_u32(&full_bar[i]), tx_bytes);
        tma_load_2d_hint(st, &tmap_w, smem_u32(&full_bar[i]), (kb_lo + i) * kStreamTileK, w_row,
                         pol_w);
        issued |= 1u << i;
      }
      grid_dependency_wait();  // activations may come from the preceding grid
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
        tma_load_2d_hint(st, &tmap_w, smem_u32(&full_bar[s]), kc, w_row, pol_w);
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
    if (multi) cluster_wait_acquire();  // phase 1 (this warp copies nothing)
  } else {
    // ---------------- warps 0-3: drain TMEM, fold shards in order, stage rows per owner
    grid_dependency_wait();
    const int row = warp * 32 + lane;  // TMEM lane == weight row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    // staging (the idle pipeline buffers): [owner][tok][row % R] fp32
    float* stage_row = reinterpret_cast<float*>(smem) + (row / R) * p.T * R + (row % R);
    // single-CTA cluster: this thread's row is final, store it directly
    const int n_row = n_tile * kStreamTileM + row;
    const float bias_row = (!multi && p.bias != nullptr && n_row < p.N) ? bf16_to_f32(p.bias[n_row]) : 0.0f;
    if (!kShards || p.spc == 1) {
      const bool ok = __all_sync(0xffffffffu, wait_parity(smem_u32(&seg_full[0]), 0, abort_flag));
      tc_fence_after();
      // once seg_full completed every MMA is done, so the pipeline buffers are free
      for (int c0 = 0; c0 < p.T; c0 += 16) {
        uint32_t r[16];
        if (ok && nkb > 0) {
          tmem_ld16(tmem_d + lane_addr + static_cast<uint32_t>(c0), r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) r[j] = 0u;
        }
        if (multi) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < p.T) stage_row[(c0 + j) * R] = __uint_as_float(r[j]);
        } else if (n_row < p.N) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < p.T) stream_store(p, c0 + j, n_row, __uint_as_float(r[j]), bias_row);
        }
      }
    } else if constexpr (kShards) {
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
      if (multi) {
#pragma unroll
        for (int c = 0; c < kStreamRunCols; ++c)
          if (c < p.T) stage_row[c * R] = ok ? run[c] : 0.0f;
      } else if (n_row < p.N) {
#pragma unroll
        for (int c = 0; c < kStreamRunCols; ++c)
          if (c < p.T) stream_store(p, c, n_row, run[c], bias_row);
      }
    }
    tc_fence_before();
    if (multi) {
      fence_proxy_async_smem();  // staging is read by the bulk-copy engine
      cluster_wait_acquire();    // phase 1: every CTA of the cluster has started
      named_barrier(1, 128);     // all four warps have staged their rows
    }
    if (multi && threadIdx.x < p.csize) {
      // one bulk copy per owner, issued by lane o: my rows of owner o's range ->
      // its receive slot [crank] (each completes on the owner's byte count)
      const uint32_t bytes = static_cast<uint32_t>(p.T * R * 4);
      const int o = threadIdx.x;
      const uint32_t src = smem_u32(smem) + static_cast<uint32_t>(o) * bytes;
      const uint32_t dst = dsmem_map(smem_u32(recv) + static_cast<uint32_t>(crank) * bytes,
                                     static_cast<uint32_t>(o));
      bulk_copy_to_peer(dst, src, bytes, dsmem_map(smem_u32(recv_bar), static_cast<uint32_t>(o)));
    }
  }
  if (multi && warp == kStreamProducerWarp) cluster_wait_acquire();  // phase 1 (copies nothing)

  __syncthreads();
  if (warp == kStreamMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_d, tcols_alloc);
  }
  if (!multi) return;
  if (warp >= 4) cluster_arrive_release();  // phase 2 for the warps that receive nothing

  // ---------------- owner: fixed-order sum of the csize partials of its rows
  if (warp < 4) {
    // every peer always issues its copy, so this completes within microseconds
    if (!drain_wait(smem_u32(recv_bar), 0, 50ull * 1000ull * 1000ull))
      atomicOr(&g_tp_device_error, kErrTimeout);
    // phase 2: my incoming copies have landed (so the peers' sources were read)
    cluster_arrive_release();
    const int groups4 = R / 4;
    const int total = groups4 * p.T;
    for (int e = threadIdx.x; e < total; e += 128) {
      const int tok = e / groups4;
      const int q4 = (e % groups4) * 4;
      float4 v[8];
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (c < p.csize)
          v[c] = *reinterpret_cast<const float4*>(recv + (c * p.T + tok) * R + q4);
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
      const int n = n_tile * kStreamTileM + crank * R + q4;
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
  // phase 2: every CTA's incoming copies have landed, so this CTA's staging
  // (the source of its outgoing copies) is no longer read and it may exit
  cluster_wait_acquire();
}

}  // namespace tpb
