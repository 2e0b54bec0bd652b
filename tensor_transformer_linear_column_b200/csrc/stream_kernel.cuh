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
// Issue rate: one thread issues a tcgen05.mma (any N up to 256) about every
// 140 cycles, so with a handful of tokens the tensor pipe is bound by MMA
// issue, not arithmetic: 4 KB of weight per instruction.  Two warps therefore
// issue MMAs, one for the even and one for the odd pipeline stages, into two
// accumulators that the epilogue adds in a fixed order.
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
// (R = 128 / csize).  Every CTA sends each owner its fp32 partial of the
// owner's rows straight from registers with asynchronous remote stores
// (st.async, cluster scope) whose bytes complete on an mbarrier in the owner;
// each owner waits for exactly those bytes, sums the csize partials of its rows
// in a fixed order from its own shared memory, adds the bias, applies the
// activation and stores bf16.  A split cluster barrier closes the exchange:
// every thread arrives once it has issued its last remote store, and a CTA
// waits for that phase before it exits (the owner warps after their sum), so
// no CTA leaves while a peer may still write into its shared memory, also
// when a bounded wait has run out somewhere in the cluster (every wait before a
// send is bounded, so the phase always completes).  Nothing intermediate goes
// to global memory and there are no atomics, so the result is bit-identical
// from run to run for a given shape and t.
//
// Weight traffic: a ring of 2-8 stages of one or two k-blocks each (3-D TMA
// boxes), deeper for CTAs that stream longer.  With static weights the first
// ring's worth is requested before the kernel waits for the preceding grid,
// and CTAs with short streams send the next two boxes to L2, overlapping that
// grid's tail.
//
// 8-bit weights (kW8): the weight is FP8 E4M3 with one fp32 scale per row
// (drpranayjha.com "AI Infrastructure series, Part 5", section "Reason 2":
// decode reads 8-bit weights).  TMA brings each k-block's 8 KB of E4M3 codes
// into the stage (64-byte swizzle, so a thread reading its own row's 64 codes
// hits every bank once per eight lanes; two k-blocks per box, 16 KB requests,
// where four such stages fit the ring); the four epilogue warps, idle while
// the weights stream, convert them (exact: every E4M3 value is a bf16 value)
// and store the bf16 tile straight into tensor memory, one row per thread, as
// the MMA's A operand.  So per k-block shared memory carries only the codes
// (written by TMA, read once) and x, not a bf16 tile written and read again.
// TMEM A slots decouple conversion from the MMAs: four of 32 columns (one
// k-block each), or two of 64 with two k-blocks per box.  The row scale
// multiplies the fp32 sum before bias and activation; HBM traffic is halved.
//
// Threads: warps 0-3 drain TMEM (warp w may access TMEM lanes 32w..32w+31),
// push and reduce, and with 8-bit weights first convert the weight tiles;
// warp 4 issues TMA; one thread each of warps 5 and 6 issues MMAs.
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
  int kpb;        // k-blocks per TMA box and pipeline stage (1 or 2)
  int l2_ahead;   // boxes after the ring's first fill prefetched into L2 before the grid wait
  int stages;     // smem pipeline depth (<= 8)
  int stage_bytes;
  int act;        // tp_act
  int prefetch_w; // weights may be read before the preceding grid completes
  const uint16_t* bias;  // [N] or nullptr
  const float* w_scale;  // [N] row scales of an 8-bit weight (kW8), else unused
  uint16_t* out;         // [T, N]
};

constexpr int kStreamThreads = 224;
constexpr int kStreamProducerWarp = 4;
constexpr int kStreamMmaWarp = 5;   // MMA issuers: warps 5 and 6
constexpr int kStreamMmaWarps = 2;
constexpr int kStreamTileM = 128;
constexpr int kStreamTileK = 64;
constexpr int kStreamW8Bytes = kStreamTileM * kStreamTileK;  // one k-block of 8-bit W: 8 KB
constexpr int kStreamMaxStages = 8;
constexpr int kStreamMaxStagesW8 = 12;  // 8 KB code stages: a deeper ring in the same memory
constexpr int kStreamReleaseBack = 2;  // boxes still to issue when the next grid is released
constexpr int kStreamRunCols = 64;  // register running sum: t_pad <= 64 when spc > 1
constexpr int kStreamW8Slots = 4;   // 8-bit weights: bf16 k-blocks in TMEM (A operand slots)

// TMEM columns a CTA allocates: two accumulator regions of tmem_cols each,
// and with 8-bit weights 128 columns of A slots (four of 32, or two of 64).
__host__ __device__ inline int stream_tmem_alloc_cols(int tmem_cols, bool w8) {
  const int need = 2 * tmem_cols + (w8 ? kStreamW8Slots * 32 : 0);
  int c = 32;
  while (c < need) c <<= 1;
  return c;
}

// Shared memory layout (dynamic, base rounded up to 1024 B):
//   [0, stages * stage_bytes)   pipeline: per stage kpb W tiles (16 KB each) then kpb x
//                               tiles (t_pad * 128 B each); with 8-bit weights (kpb = 1)
//                               the W tile is the 8 KB E4M3 tile [128][64] bytes
//                               (64-byte swizzle), converted into TMEM
//   [.., + recv_bytes)          receive buffer [csize][R][RS] fp32: sender, row, token
//   then barriers: full[stages], empty[stages], seg_full[2], seg_empty[2], final[2], recv,
//   a_full[4], a_empty[4] (8-bit weights: TMEM A slots; two used with two
//   k-blocks per box), tmem slot, abort flag
// (no receive buffer when the cluster is a single CTA: it stores directly)
//
// Row stride RS of the receive buffer: T rounded up to 4 floats (one 16-byte
// store carries four tokens of a row), plus 4 when that is a multiple of 32
// floats, so eight consecutive rows read as float4 fall in distinct banks.
__host__ __device__ inline int stream_recv_stride(int T) {
  const int rs = (T + 3) / 4 * 4;
  return rs % 32 == 0 ? rs + 4 : rs;
}

__host__ __device__ inline int stream_recv_bytes(int T, int csize) {
  return csize > 1 ? kStreamTileM * stream_recv_stride(T) * 4 : 0;
}

__host__ __device__ inline int stream_data_bytes(int stages, int stage_bytes, int T, int csize) {
  return stages * stage_bytes + stream_recv_bytes(T, csize);
}

// Barriers after the data: full[stages], empty[stages], seg_full[2],
// seg_empty[2], final[2], recv, then `stream_extra_bars` more: a_full[4] and
// a_empty[4] with 8-bit weights, an unused [stages] otherwise.
__host__ __device__ inline int stream_extra_bars(int stages, bool w8) {
  return w8 ? 2 * kStreamW8Slots : stages;
}

__host__ inline int stream_smem_bytes(int stages, int stage_bytes, int T, int csize, bool w8) {
  return 1024 /*alignment slack*/ + stream_data_bytes(stages, stage_bytes, T, csize) +
         (2 * stages + 7 + stream_extra_bars(stages, w8)) * 8 + 16;
}

// Epilogue of one value: bias, activation, round to bf16, store.
__device__ __forceinline__ void stream_store(const StreamParams& p, int tok, int n, float v,
                                             float bias) {
  v += bias;
  if (p.act == 1) v = gelu_tanh_f32(v);
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  p.out[static_cast<size_t>(tok) * p.N + n] = *reinterpret_cast<uint16_t*>(&h);
}

// Send tokens [c0, c0 + 16) of this thread's row, values v, to the owner's
// receive row at cluster address `dst_row`: four tokens per 16-byte store, one
// at a time past the last full group.  Exactly T values per row are sent, the
// byte count each owner waits for.
__device__ __forceinline__ void stream_send16(uint32_t dst_row, uint32_t peer_bar, int c0, int T,
                                              const float* v) {
#pragma unroll
  for (int j = 0; j < 16; j += 4) {
    const int tok = c0 + j;
    const uint32_t dst = dst_row + static_cast<uint32_t>(tok * 4);
    if (tok + 4 <= T) {
      st_async_f32x4(dst, v[j], v[j + 1], v[j + 2], v[j + 3], peer_bar);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (tok + q < T) st_async_f32(dst + static_cast<uint32_t>(q * 4), v[j + q], peer_bar);
    }
  }
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

// Registers are granted to a CTA per group of four warps, so the seven-warp
// CTA is charged as eight; the bounds below are stated for 256 threads to make
// the compiler budget for that.  kShards = false: one accumulation segment per CTA
// (spc == 1), at most 85 registers so three CTAs fit on an SM, which lets the
// next call's CTAs start and prefetch weights while this call drains.
// kShards = true: several shards per CTA (spc > 1) folded in a register
// running sum, at most 128 registers (two CTAs per SM).
constexpr int kStreamRegThreads = 256;
template <bool kShards, bool kW8>
__global__ void __launch_bounds__(kStreamRegThreads, kShards ? 2 : 3)
    stream_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_x, const StreamParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* recv = reinterpret_cast<float*>(smem + p.stages * p.stage_bytes);
  const int data_bytes = stream_data_bytes(p.stages, p.stage_bytes, p.T, p.csize);
  const bool multi = p.csize > 1;  // partials are summed across a cluster
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + data_bytes);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + p.stages;
  uint64_t* seg_full = bars + 2 * p.stages;       // [2]
  uint64_t* seg_empty = bars + 2 * p.stages + 2;  // [2]
  uint64_t* final_bar = bars + 2 * p.stages + 4;  // [2], one per MMA issuer
  uint64_t* recv_bar = bars + 2 * p.stages + 6;   // bytes of the peers' partials for my rows
  uint64_t* a_full = bars + 2 * p.stages + 7;     // [4]: 8-bit weights, A slot converted (4 warps)
  uint64_t* a_empty = a_full + kStreamW8Slots;    // [4]: A slot read by the MMAs (commit)
  uint32_t* tmem_slot =
      reinterpret_cast<uint32_t*>(bars + 2 * p.stages + 7 + stream_extra_bars(p.stages, kW8));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x;
  float bias_own = 0.0f;   // bias of the row this thread finalises as owner
  float scale_own = 1.0f;  // and its 8-bit weight scale
  const int crank = static_cast<int>(cluster_ctarank());  // == blockIdx.y
  const int R = kStreamTileM / p.csize;                   // rows each CTA finalises

  int kb_lo, kb_hi;
  stream_cta_range(p, crank, kb_lo, kb_hi);
  const int nkb = kb_hi - kb_lo;
  const int kpb = p.kpb;            // k-blocks per box (divides every CTA's range)
  const int nbox = nkb / kpb;       // boxes (pipeline stages' worth) of this CTA
  const int box_seg = nbox / p.spc;  // boxes per accumulation segment
  // two TMEM regions: the two issuers' accumulators (one segment), or
  // alternate shards (several segments)
  // (8-bit weights: then the A slots, 128 columns: four of one bf16 k-block
  // each, or two of two k-blocks)
  const uint32_t a_col0 = static_cast<uint32_t>(2 * p.tmem_cols);
  const uint32_t tcols_alloc = static_cast<uint32_t>(stream_tmem_alloc_cols(p.tmem_cols, kW8));

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    if constexpr (kW8) {
      for (int a = 0; a < kStreamW8Slots; ++a) {
        mbar_init(smem_u32(&a_full[a]), 4);  // one arrive per converting warp
        mbar_init(smem_u32(&a_empty[a]), 1);
      }
    }
    for (int b = 0; b < 2; ++b) {
      // one segment: both issuers commit to seg_full[0]
      mbar_init(smem_u32(&seg_full[b]), kShards ? 1 : kStreamMmaWarps);
      mbar_init(smem_u32(&seg_empty[b]), 4);
      mbar_init(smem_u32(&final_bar[b]), 1);
    }
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

  const uint32_t x_bytes = static_cast<uint32_t>(p.t_pad) * kStreamTileK * 2;
  // one k-block of W: 16 KB of bf16, or 8 KB of E4M3 codes (kpb == 1)
  const uint32_t w_bytes = kW8 ? kStreamW8Bytes : kStreamTileM * kStreamTileK * 2;
  const uint32_t xoff = static_cast<uint32_t>(kpb) * w_bytes;  // x tiles follow the W tiles
  const uint32_t wdst = 0u;
  const uint32_t tx_bytes = static_cast<uint32_t>(kpb) * (w_bytes + x_bytes);

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
      // box i holds k-blocks kb_lo + i kpb .. + kpb - 1 (3-D maps: column in
      // the block, row, k-block)
      const int pre = p.prefetch_w ? (nbox < p.stages ? nbox : p.stages) : 0;
      for (int i = 0; i < pre; ++i) {
        const uint32_t st = smem_u32(smem + i * p.stage_bytes);
        mbar_arrive_expect_tx(smem_u32(&full_bar[i]), tx_bytes);
        tma_load_3d_hint(st + wdst, &tmap_w, smem_u32(&full_bar[i]), 0, w_row, kb_lo + i * kpb,
                         pol_w);
        issued |= 1u << i;
      }
      // the next l2_ahead boxes go to L2 only: a short look-ahead keeps HBM
      // busy while the preceding grid drains; a longer one delays this grid's
      // own first loads
      if (p.prefetch_w) {
        const int l2_end = nbox < pre + p.l2_ahead ? nbox : pre + p.l2_ahead;
        for (int i = pre; i < l2_end; ++i) tma_prefetch_l2_3d(&tmap_w, 0, w_row, kb_lo + i * kpb);
      }
      // the next kernel in the stream is released once this CTA has issued
      // all but its last kStreamReleaseBack weight boxes: earlier, its weight
      // requests slow this grid's last round trips; later, its own weight
      // prefetch starts too late to cover this grid's tail
      const int release_at = nbox - 1 - kStreamReleaseBack;
      bool released = release_at < pre;
      if (released) grid_launch_dependents();
      grid_dependency_wait();  // activations may come from the preceding grid
      for (int i = 0; i < pre; ++i) {
        const uint32_t st = smem_u32(smem + i * p.stage_bytes);
        tma_load_3d(st + xoff, &tmap_x, smem_u32(&full_bar[i]), 0, 0, kb_lo + i * kpb);
      }
      // stage s and pass parity ph of box i, advanced without divisions
      int s = pre == p.stages ? 0 : pre;
      uint32_t ph = pre == p.stages ? 1u : 0u;
      for (int i = pre; i < nbox; ++i) {
        if (!wait_parity(smem_u32(&empty_bar[s]), ph ^ 1u, abort_flag)) break;
        const uint32_t st = smem_u32(smem + s * p.stage_bytes);
        mbar_arrive_expect_tx(smem_u32(&full_bar[s]), tx_bytes);
        const int kb = kb_lo + i * kpb;
        tma_load_3d_hint(st + wdst, &tmap_w, smem_u32(&full_bar[s]), 0, w_row, kb, pol_w);
        tma_load_3d(st + xoff, &tmap_x, smem_u32(&full_bar[s]), 0, 0, kb);
        issued |= 1u << s;
        phases = (phases & ~(1u << s)) | (ph << s);
        if (++s == p.stages) {
          s = 0;
          ph ^= 1u;
        }
        if (i == release_at) {
          grid_launch_dependents();
          released = true;
        }
      }
      if (!released) grid_launch_dependents();  // the loop stopped early
      if (*abort_flag) {
        // let copies already in flight land before the CTA can exit
        for (int s = 0; s < p.stages; ++s)
          if (issued & (1u << s))
            drain_wait(smem_u32(&full_bar[s]), (phases >> s) & 1u, 50ull * 1000ull * 1000ull);
      }
    }
    __syncwarp();
  } else if (warp >= kStreamMmaWarp) {
    const int me = warp - kStreamMmaWarp;  // issuer 0 or 1
    if (lane == 0 && (!kShards || me == 0)) {
      // ---------------- MMA issuers.  One segment: issuer j takes the boxes in
      // the odd (j = 1) or even (j = 0) pipeline stages, into TMEM region j;
      // each stage has a single consumer, so its fills are taken in order.
      // Several segments (one issuer): segment g into region g % 2.
      const uint32_t idesc = idesc_bf16_f32(kStreamTileM, p.t_pad);
      // descriptors of stage 0; a byte offset b within the ring adds b >> 4
      const uint64_t desc0 = desc_kmajor_sw128(smem_u32(smem));
      // every stage needs activations from the preceding grid: park in the
      // hardware wait instead of polling the first stage while it drains
      grid_dependency_wait();
      bool ok = true;
      int i = 0;        // box index
      int s = 0;        // its stage
      uint32_t ph = 0u;  // its pass parity
      // 8-bit weights: box i's A slot and its pass parity, below
      for (int g = 0; ok && g < p.spc; ++g) {
        const int region = kShards ? (g & 1) : me;
        if (kShards && g >= 2) {
          if (!wait_parity(smem_u32(&seg_empty[region]), static_cast<uint32_t>((g >> 1) - 1) & 1u,
                           abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const uint32_t d = tmem_d + static_cast<uint32_t>(region * p.tmem_cols);
        const int end = (g + 1) * box_seg;
        bool first = true;
        for (; i < end; ++i) {
          // 8-bit weights with two k-blocks per box: two A slots of 64 columns,
          // box i in slot i % 2 and to issuer i % 2, so each slot has one
          // consumer; one k-block per box: four slots of 32, issuers by stage
          if (kShards || ((kW8 && kpb == 2) ? (i & 1) : (s & 1)) == me) {
            const int a = kpb == 2 ? (i & 1) : (i & (kStreamW8Slots - 1));
            const uint32_t aph = static_cast<uint32_t>(kpb == 2 ? (i >> 1) : (i >> 2)) & 1u;
            if (!wait_parity(smem_u32(kW8 ? &a_full[a] : &full_bar[s]), kW8 ? aph : ph,
                             abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t st = static_cast<uint32_t>(s * p.stage_bytes);
            for (int c = 0; c < kpb; ++c) {
              const uint64_t db = desc0 + ((st + xoff + static_cast<uint32_t>(c) * x_bytes) >> 4);
              if constexpr (kW8) {
                // A: the converted bf16 k-block c of slot a, 8 columns per K = 16
                const uint32_t ta = tmem_d + a_col0 + static_cast<uint32_t>((a * kpb + c) * 32);
#pragma unroll
                for (int kk = 0; kk < kStreamTileK / 16; ++kk) {
                  umma_bf16_ta(d, ta + static_cast<uint32_t>(kk * 8), db + static_cast<uint64_t>(kk * 2),
                               idesc, first ? 0u : 1u);
                  first = false;
                }
              } else {
                const uint64_t da = desc0 + ((st + static_cast<uint32_t>(c) * w_bytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < kStreamTileK / 16; ++kk) {
                  umma_bf16(d, da + static_cast<uint64_t>(kk * 2), db + static_cast<uint64_t>(kk * 2),
                            idesc, first ? 0u : 1u);
                  first = false;
                }
              }
            }
            umma_commit(smem_u32(&empty_bar[s]));
            if constexpr (kW8) umma_commit(smem_u32(&a_empty[a]));
          }
          if (++s == p.stages) {
            s = 0;
            ph ^= 1u;
          }
        }
        // an issuer without boxes commits at once; its region is not read
        if (ok) umma_commit(smem_u32(&seg_full[kShards ? region : 0]));
      }
      if (!ok) {
        // every MMA issued so far must finish before TMEM / smem are released
        umma_commit(smem_u32(&final_bar[me]));
        drain_wait(smem_u32(&final_bar[me]), 0, 50ull * 1000ull * 1000ull);
      }
    }
    __syncwarp();
    if (multi) cluster_wait_acquire();  // phase 1 (these warps send nothing)
  } else {
    if constexpr (kW8) {
      // ---------------- warps 0-3, first: E4M3 -> bf16 into TMEM.  Thread t
      // owns TMEM lane t = weight row t of the tile: for each k-block c of the
      // box it reads its row's 64 codes (four 16-byte chunks; chunk q sits at
      // chunk q ^ ((t / 2) % 4) of the row under the 64-byte swizzle),
      // converts them and stores the 64 bf16 values as 32 columns of box i's
      // A slot, at column offset 32 c.  Every converter thread takes every box
      // in order, whatever its waits returned, so the warps' arrivals stay
      // matched.
      const int t = static_cast<int>(threadIdx.x);
      const uint32_t lane_addr_c = static_cast<uint32_t>(warp * 32) << 16;
      const int sw = (t >> 1) & 3;
      int s = 0;
      uint32_t ph = 0u;
      bool ok = true;
      for (int i = 0; i < nbox; ++i) {
        const int a = kpb == 2 ? (i & 1) : (i & (kStreamW8Slots - 1));
        const uint32_t aph = static_cast<uint32_t>(kpb == 2 ? (i >> 1) : (i >> 2)) & 1u;
        ok = ok && wait_parity(smem_u32(&full_bar[s]), ph, abort_flag);
        ok = ok && wait_parity(smem_u32(&a_empty[a]), aph ^ 1u, abort_flag);
        // the warp stores only when all its lanes' waits succeeded (the store
        // is warp-wide); every warp arrives for every box whatever happened
        if (__all_sync(0xffffffffu, ok)) {
          for (int c = 0; c < kpb; ++c) {
            const uint8_t* row = smem + s * p.stage_bytes + c * kStreamW8Bytes + t * kStreamTileK;
            uint32_t w[32];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 v = *reinterpret_cast<const uint4*>(row + ((q ^ sw) << 4));
              const uint4 lo = e4m3x8_to_bf16x8(make_uint2(v.x, v.y));
              const uint4 hi = e4m3x8_to_bf16x8(make_uint2(v.z, v.w));
              w[8 * q + 0] = lo.x; w[8 * q + 1] = lo.y; w[8 * q + 2] = lo.z; w[8 * q + 3] = lo.w;
              w[8 * q + 4] = hi.x; w[8 * q + 5] = hi.y; w[8 * q + 6] = hi.z; w[8 * q + 7] = hi.w;
            }
            tmem_st32(tmem_d + lane_addr_c + a_col0 + static_cast<uint32_t>((a * kpb + c) * 32), w);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&a_full[a]));
        if (++s == p.stages) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    // ---------------- warps 0-3: drain TMEM, fold shards in order, send rows to their owners
    grid_dependency_wait();
    const int row = warp * 32 + lane;  // TMEM lane == weight row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    // single-CTA cluster: this thread's row is final, store it directly
    const int n_row = n_tile * kStreamTileM + row;
    const float bias_row = (!multi && p.bias != nullptr && n_row < p.N) ? bf16_to_f32(p.bias[n_row]) : 0.0f;
    const float scale_row = (kW8 && !multi && n_row < p.N) ? p.w_scale[n_row] : 1.0f;
    // owner rows: item e of the final sum is row e % R, and R divides 128, so
    // each thread finalises one row and can fetch its bias now, off the tail
    const int n_own = n_tile * kStreamTileM + crank * R + static_cast<int>(threadIdx.x) % R;
    bias_own = (multi && p.bias != nullptr && n_own < p.N) ? bf16_to_f32(p.bias[n_own]) : 0.0f;
    scale_own = (kW8 && multi && n_own < p.N) ? p.w_scale[n_own] : 1.0f;
    uint32_t dst_row = 0u, peer_bar = 0u;
    if (multi) {
      // phase 1: every CTA of the cluster has started, so its receive barrier is armed
      cluster_wait_acquire();
      const uint32_t owner = static_cast<uint32_t>(row / R);
      const int RS = stream_recv_stride(p.T);
      dst_row = dsmem_map(smem_u32(recv) + static_cast<uint32_t>(((crank * R + row % R) * RS) * 4),
                          owner);
      peer_bar = dsmem_map(smem_u32(recv_bar), owner);
    }
    if constexpr (!kShards) {
      const bool ok = __all_sync(0xffffffffu, wait_parity(smem_u32(&seg_full[0]), 0, abort_flag));
      tc_fence_after();
      // the issuers' accumulators that received a box, added in issuer order
      const int na = ok ? (nbox < kStreamMmaWarps ? nbox : kStreamMmaWarps) : 0;
      // 32 tokens per round: two TMEM loads in flight, one wait
      for (int c0 = 0; c0 < p.T; c0 += 32) {
        const bool two = c0 + 16 < p.T;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.0f;
        for (int a = 0; a < na; ++a) {
          uint32_t r0[16], r1[16];
          const uint32_t col = tmem_d + lane_addr + static_cast<uint32_t>(a * p.tmem_cols + c0);
          tmem_ld16(col, r0);
          if (two) {
            tmem_ld16(col + 16u, r1);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) r1[j] = 0u;
          }
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            v[j] = a == 0 ? __uint_as_float(r0[j]) : v[j] + __uint_as_float(r0[j]);
            v[16 + j] = a == 0 ? __uint_as_float(r1[j]) : v[16 + j] + __uint_as_float(r1[j]);
          }
        }
        if (multi) {
          stream_send16(dst_row, peer_bar, c0, p.T, v);
          if (two) stream_send16(dst_row, peer_bar, c0 + 16, p.T, v + 16);
        } else if (n_row < p.N) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0 + j < p.T) stream_store(p, c0 + j, n_row, kW8 ? v[j] * scale_row : v[j], bias_row);
        }
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
      if (!ok) {
#pragma unroll
        for (int j = 0; j < kStreamRunCols; ++j) run[j] = 0.0f;
      }
      if (multi) {
#pragma unroll
        for (int c = 0; c < kStreamRunCols; c += 16)
          if (c < p.T) stream_send16(dst_row, peer_bar, c, p.T, run + c);
      } else if (n_row < p.N) {
#pragma unroll
        for (int c = 0; c < kStreamRunCols; ++c)
          if (c < p.T) stream_store(p, c, n_row, kW8 ? run[c] * scale_row : run[c], bias_row);
      }
    }
    tc_fence_before();
  }
  if (multi && warp == kStreamProducerWarp) cluster_wait_acquire();  // phase 1 (sends nothing)
  // cluster phase 2: "this thread has issued its last remote store".  Warps 0-3
  // arrive after their sends; the others have none.
  if (multi) cluster_arrive_release();

  __syncthreads();
  if (warp == kStreamMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_d, tcols_alloc);
  }
  if (!multi) return;
  if (warp >= 4) {
    // no CTA of the cluster exits before every peer has issued all of its
    // remote stores (the owner warps take the same wait after their sum)
    cluster_wait_acquire();
    return;
  }

  // ---------------- owner: fixed-order sum of the csize partials of its rows.
  // Every peer always sends its T values per row, so this completes within
  // microseconds; if it ever ran out, the sum would read a partial buffer
  // (the error word says so) and the closing barrier below still keeps this
  // CTA alive until every late store has been issued.
  if (!drain_wait(smem_u32(recv_bar), 0, 50ull * 1000ull * 1000ull))
    atomicOr(&g_tp_device_error, kErrTimeout);
  const int RS = stream_recv_stride(p.T);
  const int groups = (p.T + 3) / 4;  // four tokens of one row per item
  const int n0 = n_tile * kStreamTileM + crank * R;
  // csize, R = 128 / csize and jsplit = csize / shards are powers of two
  const int r_shift = __ffs(R) - 1;
  const uint32_t recv_s = smem_u32(recv);
  const int j_mask = p.jsplit - 1;
  for (int e = threadIdx.x; e < R * groups; e += 128) {
    const int lr = e & (R - 1);
    const int tok0 = (e >> r_shift) * 4;
    float4 v[8];
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (c < p.csize) v[c] = ld_shared_f32x4(recv_s + static_cast<uint32_t>(((c * R + lr) * RS + tok0) * 4));
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f), ps = y;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c < p.csize) {
        const int jj = c & j_mask;
        if (jj == 0) {
          ps = v[c];
        } else {
          ps.x += v[c].x; ps.y += v[c].y; ps.z += v[c].z; ps.w += v[c].w;
        }
        if (jj == j_mask) {
          if (c == j_mask) {
            y = ps;
          } else {
            y.x += ps.x; y.y += ps.y; y.z += ps.z; y.w += ps.w;
          }
        }
      }
    }
    const int n = n0 + lr;
    if (n < p.N) {
      const float o[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (tok0 + q < p.T) stream_store(p, tok0 + q, n, kW8 ? o[q] * scale_own : o[q], bias_own);
    }
  }
  cluster_wait_acquire();  // phase 2, see above
}

}  // namespace tpb
