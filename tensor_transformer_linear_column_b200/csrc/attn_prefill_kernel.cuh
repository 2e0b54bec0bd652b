// attn_prefill_kernel.cuh -- the attention core when many tokens arrive at
// once (a prompt, or a long chunk of one appended to a cache): every query row
// of a head attends over the keys it may see, 128 query rows per CTA.
//
// Same operation as attn_decode_kernel (grouped-query causal attention, scores
// q.k / sqrt(d), query head h reads key-value head h / G, new token i at
// position past + i sees keys 0 .. past + i), with the heads split across the
// tensor-parallel shards and no exchange (xingyuzhitong.com "Tensor vs
// Pipeline Parallelism", section "Tensor parallelism: split inside each
// layer").  The decode kernel puts keys on the MMA's M side because a decode
// step has few query rows; here the queries fill M = 128 and each softmax
// thread owns one query row, so the row maximum and sum need no shuffles.
//
// Kernels:
//   kv_append_kernel      copies the new tokens' K and V (columns of qkv) into
//                         rows [past, past + T) of the caches;
//   attn_prefill_kernel   CTA (query head h, tile of 128 new tokens); key
//                         blocks of 128 from 0 up to the tile's last visible
//                         key, each block:
//     S = Q K_b^T            tcgen05.mma into TMEM columns [0, 128), fp32
//     softmax (warps 0-3)    thread r = query row r: masks keys past its
//                            position (the diagonal blocks only), takes the
//                            block maximum, p = 2^(s log2(e)/sqrt(d) - m)
//                            rounded to bf16 and written back into the same
//                            TMEM columns (two per 32-bit column), adds p to
//                            the row sum l
//     O += P V_b             tcgen05.mma with A = P read from TMEM, B = V
//                            read MN-major from its [key][d] tile, into TMEM
//                            columns [128, 256)
//   The running maximum m is raised only when a block's maximum exceeds it by
//   more than 8 (in log2 units): p then stays below 2^8, and O and l, which
//   are always relative to the same m, are rescaled by 2^(m_old - m_new) far
//   less often than once per block.  The result is the same softmax; only
//   the rounding differs.
//   Two CTAs share an SM (256 TMEM columns and ~100 KB of shared memory each),
//   so one CTA's softmax overlaps the other's MMAs.  Used for an odd number
//   of query heads per key-value head;
//   attn_prefill2_kernel  an even number: two heads of one key-value group
//                         per work item, sharing every K and V block, on a
//                         persistent grid; P goes through shared memory so
//                         the next scores need not wait for P V (below).
#pragma once

#include "attn_kernel.cuh"

namespace tpb {

constexpr int kPrefillRows = 128;        // query rows (tokens of one head) per CTA
constexpr int kPrefillThreads = 192;     // warps 0-3 softmax (thread 0 issues the MMAs), warp 4 TMA, warp 5 TMEM
constexpr int kPrefillTmemCols = 256;    // S / P [0, 128), O [128, 256)
constexpr float kPrefillRescaleLog2 = 8.0f;

// 2^x from the hardware approximation (PTX ex2.approx.ftz.f32, relative error
// near 2^-22, far below a bf16 rounding that follows); 2^-inf = +0.
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct PrefillParams {
  int T;        // new tokens
  int past;     // cached tokens before them
  int L;        // past + T
  int nq, G;    // query heads, query heads per key-value head
  int ntiles;   // ceil(T / 128)
  float scale_log2;  // log2(e) / sqrt(d)
  uint16_t* ctx;     // [T, nq * d]
};

// Shared memory (dynamic, base rounded up to 1024 B): Q [2 d halves][128][64],
// one K and one V stage of the same shape, barriers, the TMEM address and the
// abort flag.
__host__ __device__ constexpr int prefill_smem_bytes() {
  return 1024 + 3 * kAttnBlockBytes + 10 * 8 + 16;
}

// One thread per 16-byte piece: piece fastest, then the K heads and V heads in
// qkv's column order, then tokens, so reads of a token row are contiguous.
__global__ void kv_append_kernel(const uint16_t* __restrict__ qkv, int T, int past, int nq,
                                 int nkv, int max_len, uint16_t* __restrict__ k_cache,
                                 uint16_t* __restrict__ v_cache) {
  grid_dependency_wait();  // qkv comes from the preceding kernel
  constexpr int kVec = kAttnHeadDim / 8;
  const size_t per_tok = static_cast<size_t>(2) * nkv * kVec;
  const size_t n = static_cast<size_t>(T) * per_tok;
  const size_t ld = static_cast<size_t>(nq + 2 * nkv) * kAttnHeadDim;
  for (size_t e = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t tok = e / per_tok;
    const int rest = static_cast<int>(e - tok * per_tok);
    const int piece = rest % kVec;
    const int hh = (rest / kVec) % nkv;
    const int which = rest / (kVec * nkv);  // 0 = K, 1 = V
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(
        qkv + tok * ld + static_cast<size_t>(nq) * kAttnHeadDim) + rest);
    uint16_t* cache = which ? v_cache : k_cache;
    reinterpret_cast<uint4*>(cache + (static_cast<size_t>(hh) * max_len + past + tok) *
                                         kAttnHeadDim)[piece] = v;
  }
  grid_launch_dependents();
}

__global__ void __launch_bounds__(kPrefillThreads, 2)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,
                        const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* qs = smem;
  uint8_t* ks = smem + kAttnBlockBytes;
  uint8_t* vs = smem + 2 * kAttnBlockBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 3 * kAttnBlockBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 2;   // S of the stage's block done
  uint64_t* v_full = bars + 3;
  uint64_t* v_empty = bars + 4;   // P V of the stage's block done
  uint64_t* s_full = bars + 5;    // scores of a block in TMEM
  uint64_t* o_done = bars + 7;    // the block's P V product done
  uint64_t* final_bar = bars + 8; // every MMA of the issuer done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x;                     // heads fastest: a key-value group's
  const int tile = p.ntiles - 1 - blockIdx.y;   // heads run together; longest tiles first
  const int q0 = tile * kPrefillRows;
  const int g = h / p.G;
  const int kend = p.past + q0 + kPrefillRows < p.L ? p.past + q0 + kPrefillRows : p.L;
  const int nblk = (kend + kAttnBlockKeys - 1) / kAttnBlockKeys;  // >= 1

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    mbar_init(smem_u32(k_full), 1);
    mbar_init(smem_u32(k_empty), 1);
    mbar_init(smem_u32(v_full), 1);
    mbar_init(smem_u32(v_empty), 1);
    mbar_init(smem_u32(s_full), 1);
    mbar_init(smem_u32(o_done), 1);
    mbar_init(smem_u32(final_bar), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), static_cast<uint32_t>(kPrefillTmemCols));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t kOCol = 128;

  if (warp == 4) {
    if (lane == 0) {
      // ---------------- TMA producer: Q once, then K_b and V_b per block, one
      // stage each; a stage is refilled once the MMA that reads it is done
      grid_dependency_wait();  // qkv and the appended cache rows come from preceding kernels
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
      const uint32_t qb = smem_u32(q_full);
      mbar_arrive_expect_tx(qb, kAttnBlockBytes);
      tma_load_2d(smem_u32(qs), &tmap_q, qb, h * kAttnHeadDim, q0);
      tma_load_2d(smem_u32(qs) + kAttnHalfBytes, &tmap_q, qb, h * kAttnHeadDim + 64, q0);
      int kissued = 0, vissued = 0;
      for (int b = 0; b < nblk; ++b) {
        const int key = b * kAttnBlockKeys;
        if (!wait_parity(smem_u32(k_empty), (b & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(smem_u32(k_full), kAttnBlockBytes);
        tma_load_3d(smem_u32(ks), &tmap_k, smem_u32(k_full), 0, key, g);
        tma_load_3d(smem_u32(ks) + kAttnHalfBytes, &tmap_k, smem_u32(k_full), 64, key, g);
        ++kissued;
        if (!wait_parity(smem_u32(v_empty), (b & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(smem_u32(v_full), kAttnBlockBytes);
        tma_load_3d(smem_u32(vs), &tmap_v, smem_u32(v_full), 0, key, g);
        tma_load_3d(smem_u32(vs) + kAttnHalfBytes, &tmap_v, smem_u32(v_full), 64, key, g);
        ++vissued;
      }
      if (*abort_flag) {
        // a stage is refilled only after its previous fill was consumed, so
        // the last fill of each is the only one that can still be in flight
        drain_wait(qb, 0, 50ull * 1000ull * 1000ull);
        if (kissued > 0)
          drain_wait(smem_u32(k_full), (kissued - 1) & 1, 50ull * 1000ull * 1000ull);
        if (vissued > 0)
          drain_wait(smem_u32(v_full), (vissued - 1) & 1, 50ull * 1000ull * 1000ull);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    __syncwarp();  // allocates and frees the TMEM; the MMAs come from softmax thread 0
  } else {
    // ---------------- warps 0-3: thread r owns query row r (TMEM lane r).
    // Every thread takes the same arrivals whatever its waits returned.
    grid_dependency_wait();  // ctx may still be read by a preceding kernel
    const int r = threadIdx.x;
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const int pos = p.past + q0 + r;  // rows at or past T are padding, never stored
    const float c = p.scale_log2;
    float m_used = neg_inf();
    float l = 0.0f;
    bool ok = true;
    // Thread 0 issues the MMAs: S_b = Q K_b^T into TMEM columns [0, 128), and
    // after the four warps have written P_b (a named barrier, not a round
    // trip through another warp), O += P_b V_b.  S_{b+1} overwrites P_b, so
    // it waits until P_b V_b is done.
    const uint32_t idesc_s = idesc_bf16_f32(128, kAttnBlockKeys);              // Q, K K-major
    const uint32_t idesc_o = idesc_bf16_f32(128, kAttnHeadDim, false, true);   // V MN-major
    bool issuer_ok = true;
    auto issue_s = [&](int b) {
      if (!issuer_ok || !wait_parity(smem_u32(k_full), b & 1, abort_flag)) {
        issuer_ok = false;
        return;
      }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kAttnHeadDim / 16; ++kk) {
        const uint32_t off = static_cast<uint32_t>(kk >> 2) * kAttnHalfBytes +
                             static_cast<uint32_t>(kk & 3) * 32u;
        umma_bf16(tmem, desc_kmajor_sw128(smem_u32(qs) + off), desc_kmajor_sw128(smem_u32(ks) + off),
                  idesc_s, kk > 0 ? 1u : 0u);
      }
      umma_commit(smem_u32(k_empty));
      umma_commit(smem_u32(s_full));
    };
    if (r == 0) {
      issuer_ok = wait_parity(smem_u32(q_full), 0, abort_flag);
      issue_s(0);
    }
    for (int b = 0; b < nblk; ++b) {
      ok = __all_sync(0xffffffffu, ok && wait_parity(smem_u32(s_full), b & 1, abort_flag));
      tc_fence_after();
      uint32_t s[kAttnBlockKeys];
      if (ok) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tmem_ld32(tmem + lane_addr + static_cast<uint32_t>(32 * q),
                    *reinterpret_cast<uint32_t(*)[32]>(s + 32 * q));
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int k = 0; k < kAttnBlockKeys; ++k) s[k] = 0u;
      }
      const int key0 = b * kAttnBlockKeys;
      if (key0 + kAttnBlockKeys - 1 > p.past + q0) {  // a block on the diagonal
#pragma unroll
        for (int k = 0; k < kAttnBlockKeys; ++k)
          if (key0 + k > pos) s[k] = __float_as_uint(neg_inf());
      }
      float mx4[4] = {neg_inf(), neg_inf(), neg_inf(), neg_inf()};  // four independent chains
#pragma unroll
      for (int k = 0; k < kAttnBlockKeys; ++k) mx4[k & 3] = fmaxf(mx4[k & 3], __uint_as_float(s[k]));
      const float mb = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * c;  // c > 0, so the maximum commutes with the scaling
      const bool raise = mb > m_used + kPrefillRescaleLog2;  // also the first visible key
      float alpha = 1.0f;
      if (raise) {
        alpha = m_used == neg_inf() ? 0.0f : exp2_approx(m_used - mb);
        m_used = mb;
      }
      l *= alpha;
      // P in 16-column pieces, so each piece's scores die as it is stored
      const float neg_m = -m_used;
      float sum0 = 0.0f, sum1 = 0.0f;
#pragma unroll
      for (int q = 0; q < kAttnBlockKeys / 32; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float p0 = exp2_approx(fmaf(__uint_as_float(s[32 * q + 2 * k]), c, neg_m));
          const float p1 = exp2_approx(fmaf(__uint_as_float(s[32 * q + 2 * k + 1]), c, neg_m));
          sum0 += p0;
          sum1 += p1;
          pk[k] = pack_bf16x2(p0, p1);
        }
        if (ok) tmem_st16(tmem + lane_addr + static_cast<uint32_t>(16 * q), pk);
      }
      l += sum0 + sum1;
      if (b > 0 && ok && __any_sync(0xffffffffu, raise)) {
        // O holds the products of blocks 0 .. b - 1 (all done: S_b was issued
        // after P_{b-1} V_{b-1} completed); lanes that keep m use alpha = 1
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t o[32];
          const uint32_t a = tmem + lane_addr + kOCol + static_cast<uint32_t>(32 * q);
          tmem_ld32(a, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(a, o);
        }
      }
      if (ok) tmem_wait_st();
      tc_fence_before();
      named_barrier_sync(1, kPrefillRows);  // P_b and O's rescale are in TMEM
      if (r == 0) {
        tc_fence_after();
        if (issuer_ok && wait_parity(smem_u32(v_full), b & 1, abort_flag)) {
          // K = keys in steps of 16: P columns 8 kk .. 8 kk + 7 (two keys per
          // column); V rows 16 kk .. 16 kk + 15 = two 1024-byte core groups
#pragma unroll
          for (int kk = 0; kk < kAttnBlockKeys / 16; ++kk)
            umma_bf16_ta(tmem + kOCol, tmem + static_cast<uint32_t>(kk * 8),
                         desc_mnmajor_sw128(smem_u32(vs) + static_cast<uint32_t>(kk) * 2048u,
                                            kAttnHalfBytes),
                         idesc_o, (b > 0 || kk > 0) ? 1u : 0u);
          umma_commit(smem_u32(v_empty));
          umma_commit(smem_u32(o_done));
        } else {
          issuer_ok = false;
        }
        if (b + 1 < nblk) {
          if (issuer_ok && !wait_parity(smem_u32(o_done), b & 1, abort_flag)) issuer_ok = false;
          issue_s(b + 1);
        }
      }
    }
    if (r == 0) {
      // every MMA issued must finish before the TMEM is freed
      umma_commit(smem_u32(final_bar));
      drain_wait(smem_u32(final_bar), 0, 50ull * 1000ull * 1000ull);
    }
    ok = __all_sync(0xffffffffu, ok && wait_parity(smem_u32(o_done), (nblk - 1) & 1, abort_flag));
    tc_fence_after();
    if (ok) {
      const float inv = 1.0f / l;
      const bool valid = q0 + r < p.T;
      uint4* dst = reinterpret_cast<uint4*>(p.ctx + static_cast<size_t>(q0 + r) * p.nq * kAttnHeadDim +
                                            static_cast<size_t>(h) * kAttnHeadDim);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_addr + kOCol + static_cast<uint32_t>(32 * q), o);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int w = 0; w < 4; ++w)
            dst[4 * q + w] = make_uint4(
                pack_bf16x2(__uint_as_float(o[8 * w]) * inv, __uint_as_float(o[8 * w + 1]) * inv),
                pack_bf16x2(__uint_as_float(o[8 * w + 2]) * inv, __uint_as_float(o[8 * w + 3]) * inv),
                pack_bf16x2(__uint_as_float(o[8 * w + 4]) * inv, __uint_as_float(o[8 * w + 5]) * inv),
                pack_bf16x2(__uint_as_float(o[8 * w + 6]) * inv, __uint_as_float(o[8 * w + 7]) * inv));
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  grid_launch_dependents();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(kPrefillTmemCols));
  }
}

// ---------------------------------------------------------------------------
// attn_prefill2_kernel: the same operation for an even number G of query heads
// per key-value head.  A work item is two query tiles (heads h0 and h0 + 1 of
// one key-value group, the same 128 tokens), which share every K and V block.
// The grid is persistent, one CTA per SM: CTA c takes the items of its
// column of a boustrophedon order over the list sorted longest first (c,
// 2 C - 1 - c, 2 C + c, ...), so the CTAs' total key blocks agree to a few
// per cent, and the next item's Q, K and scores are loaded while the current
// one drains.  P goes to shared memory (a K-major A operand of the P V MMA)
// instead of back into the score columns, so a tile's softmax gives its
// score slot back as soon as it has loaded the scores: the MMA warp then
// computes the next block's scores while the softmax runs.
//   TMEM (512 columns): tile t's S at 256 t, its O at 256 t + 128.
//   Shared memory: Q_0, Q_1, a ring of three 32 KB stages, P_0, P_1 (32 KB
//   each: [2 halves of 64][128 rows][64] bf16, 128-byte swizzle).  The ring
//   carries, per item, K_0, K_1, V_0, K_2, V_1, K_3, V_2, ... in the order
//   the MMA warp reads them, so K_{b+1} is loaded once P_{b-2} V_{b-2} is
//   done and V_b once S_b is done: both well before they are needed.
//   Barrier phases run on across items: the ring by its item count, the
//   per-tile score / P / product barriers by a running block count, the Q
//   and O-release barriers by the item count.
//   Warps: 0-3 softmax of tile 0, 4-7 of tile 1 (thread r of a tile owns
//   query row r), 8 TMA, 9 MMA and TMEM allocation.
constexpr int kPrefill2Threads = 320;
constexpr int kPrefill2Stages = 3;

__host__ __device__ constexpr int prefill2_smem_bytes() {
  return 1024 + (2 + kPrefill2Stages + 2) * kAttnBlockBytes + 24 * 8 + 16;
}

// Ring item i (of 2 nblk) of a work item: K_0, then K_{b+1} and V_b for
// b = 0 .. nblk - 2, then V_{nblk-1}.
__device__ __forceinline__ bool ring_is_k(int i, int nblk) {
  return i == 0 || (i < 2 * nblk - 1 && ((i - 1) & 1) == 0);
}
__device__ __forceinline__ int ring_block(int i, int nblk) {
  if (i == 0) return 0;
  if (i == 2 * nblk - 1) return nblk - 1;
  return ((i - 1) >> 1) + (((i - 1) & 1) == 0 ? 1 : 0);
}

// The r-th work item of CTA c among C (index into the longest-first list of
// nwork items), or -1 past the end; increasing in r.
__device__ __forceinline__ int prefill2_item(int r, int c, int C, int nwork) {
  const int j = r * C + ((r & 1) ? (C - 1 - c) : c);
  return j < nwork ? j : -1;
}

// Work item j: head pair j mod npairs (heads fastest, so a key-value group's
// heads run together), tile ntiles - 1 - j / npairs (longest first).
struct Prefill2Item {
  int h0, q0, g, nblk;
};
__device__ __forceinline__ Prefill2Item prefill2_decode(int j, const PrefillParams& p) {
  const int npairs = p.nq / 2;
  Prefill2Item it;
  it.h0 = (j % npairs) * 2;
  it.q0 = (p.ntiles - 1 - j / npairs) * kPrefillRows;
  it.g = it.h0 / p.G;  // G even: h0 and h0 + 1 share it
  const int kend = p.past + it.q0 + kPrefillRows < p.L ? p.past + it.q0 + kPrefillRows : p.L;
  it.nblk = (kend + kAttnBlockKeys - 1) / kAttnBlockKeys;  // >= 1
  return it;
}

__global__ void __launch_bounds__(kPrefill2Threads, 1)
    attn_prefill2_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* qs = smem;                                     // [2 tiles][32 KB]
  uint8_t* ring = qs + 2 * kAttnBlockBytes;               // [kPrefill2Stages][32 KB]
  uint8_t* ps = ring + kPrefill2Stages * kAttnBlockBytes;  // [2 tiles][32 KB]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ps + 2 * kAttnBlockBytes);
  uint64_t* q_full = bars;        // an item's two Q tiles landed
  uint64_t* q_empty = bars + 1;   // the item's last S MMAs done: Q may be replaced
  uint64_t* full = bars + 2;      // [3] per ring stage
  uint64_t* empty = bars + 5;     // [3] both tiles' MMAs that read the stage done
  uint64_t* s_full = bars + 8;    // [2] per tile: S of a block in TMEM
  uint64_t* s_free = bars + 10;   // [2] per tile: the softmax has read S (128 arrivals)
  uint64_t* p_full = bars + 12;   // [2] per tile: P in shared memory, O rescaled (128)
  uint64_t* o_done = bars + 14;   // [2] per tile: the block's P V product done
  uint64_t* o_free = bars + 16;   // [2] per tile: the item's O read out (128)
  uint64_t* final_bar = bars + 18;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nwork = (p.nq / 2) * p.ntiles;
  const int c = blockIdx.x, C = gridDim.x;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    mbar_init(smem_u32(q_empty), 1);
    for (int i = 0; i < kPrefill2Stages; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), kPrefillRows);
      mbar_init(smem_u32(&p_full[i]), kPrefillRows);
      mbar_init(smem_u32(&o_done[i]), 1);
      mbar_init(smem_u32(&o_free[i]), kPrefillRows);
    }
    mbar_init(smem_u32(final_bar), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512u);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    if (lane == 0) {
      // ---------------- TMA producer: per item, both Q tiles (once the last
      // item's last S is done), then its ring items
      grid_dependency_wait();  // qkv and the appended cache rows come from preceding kernels
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
      int ri = 0;  // ring items issued
      int nq_loads = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int j = prefill2_item(r, c, C, nwork);
        if (j < 0) break;
        const Prefill2Item it = prefill2_decode(j, p);
        if (r > 0 && !wait_parity(smem_u32(q_empty), (r - 1) & 1, abort_flag)) break;
        const uint32_t qb = smem_u32(q_full);
        mbar_arrive_expect_tx(qb, 2 * kAttnBlockBytes);
        for (int t = 0; t < 2; ++t) {
          const uint32_t dst = smem_u32(qs + t * kAttnBlockBytes);
          tma_load_2d(dst, &tmap_q, qb, (it.h0 + t) * kAttnHeadDim, it.q0);
          tma_load_2d(dst + kAttnHalfBytes, &tmap_q, qb, (it.h0 + t) * kAttnHeadDim + 64, it.q0);
        }
        ++nq_loads;
        for (int i = 0; i < 2 * it.nblk; ++i, ++ri) {
          const int st = ri % kPrefill2Stages;
          if (!wait_parity(smem_u32(&empty[st]), ((ri / kPrefill2Stages) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          const int key = ring_block(i, it.nblk) * kAttnBlockKeys;
          const uint32_t fb = smem_u32(&full[st]);
          const uint32_t dst = smem_u32(ring + st * kAttnBlockBytes);
          mbar_arrive_expect_tx(fb, kAttnBlockBytes);
          if (ring_is_k(i, it.nblk)) {
            tma_load_3d(dst, &tmap_k, fb, 0, key, it.g);
            tma_load_3d(dst + kAttnHalfBytes, &tmap_k, fb, 64, key, it.g);
          } else {
            tma_load_3d(dst, &tmap_v, fb, 0, key, it.g);
            tma_load_3d(dst + kAttnHalfBytes, &tmap_v, fb, 64, key, it.g);
          }
        }
      }
      if (*abort_flag) {
        // a buffer is refilled only after its previous fill was consumed, so
        // the last fill of each is the only one that can be in flight
        if (nq_loads > 0)
          drain_wait(smem_u32(q_full), (nq_loads - 1) & 1, 50ull * 1000ull * 1000ull);
        for (int i = ri - kPrefill2Stages < 0 ? 0 : ri - kPrefill2Stages; i < ri; ++i)
          drain_wait(smem_u32(&full[i % kPrefill2Stages]), (i / kPrefill2Stages) & 1,
                     50ull * 1000ull * 1000ull);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    if (lane == 0) {
      // ---------------- MMA issuer.  Per block b: both tiles' S_{b+1} as soon
      // as each tile's softmax has read S_b out of TMEM, then both tiles'
      // O += P_b V_b as soon as each P_b is in shared memory.
      const uint32_t idesc_s = idesc_bf16_f32(128, kAttnBlockKeys);              // Q, K K-major
      const uint32_t idesc_o = idesc_bf16_f32(128, kAttnHeadDim, false, true);   // P K-major, V MN-major
      int ci = 0;  // ring items consumed
      int gb0 = 0;  // running index of the item's block 0
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int j = prefill2_item(r, c, C, nwork);
        if (j < 0) break;
        const int nblk = prefill2_decode(j, p).nblk;
        if (!wait_parity(smem_u32(q_full), r & 1, abort_flag)) {
          ok = false;
          break;
        }
        for (int i = 0; i < 2 * nblk && ok; ++i, ++ci) {
          const int st = ci % kPrefill2Stages;
          if (!wait_parity(smem_u32(&full[st]), (ci / kPrefill2Stages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t base = smem_u32(ring + st * kAttnBlockBytes);
          const int blk = ring_block(i, nblk);
          const int gblk = gb0 + blk;
          if (ring_is_k(i, nblk)) {
            for (int t = 0; t < 2 && ok; ++t) {  // S_blk = Q K_blk^T
              if (gblk > 0 && !wait_parity(smem_u32(&s_free[t]), (gblk - 1) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t qbase = smem_u32(qs + t * kAttnBlockBytes);
#pragma unroll
              for (int kk = 0; kk < kAttnHeadDim / 16; ++kk) {
                const uint32_t off = static_cast<uint32_t>(kk >> 2) * kAttnHalfBytes +
                                     static_cast<uint32_t>(kk & 3) * 32u;
                umma_bf16(tmem + static_cast<uint32_t>(t * 256), desc_kmajor_sw128(qbase + off),
                          desc_kmajor_sw128(base + off), idesc_s, kk > 0 ? 1u : 0u);
              }
              umma_commit(smem_u32(&s_full[t]));
            }
            if (ok && blk == nblk - 1) umma_commit(smem_u32(q_empty));  // Q read for the last time
          } else {
            for (int t = 0; t < 2 && ok; ++t) {  // O += P_blk V_blk
              if (!wait_parity(smem_u32(&p_full[t]), gblk & 1, abort_flag)) {
                ok = false;
                break;
              }
              // the first product of an item overwrites O: the last item's
              // O must have been read out
              if (blk == 0 && r > 0 && !wait_parity(smem_u32(&o_free[t]), (r - 1) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t pbase = smem_u32(ps + t * kAttnBlockBytes);
              // K = keys in steps of 16: P in the layout of Q (K-major, 128-byte
              // swizzle); V rows 16 kk .. 16 kk + 15 = two 1024-byte core groups
#pragma unroll
              for (int kk = 0; kk < kAttnBlockKeys / 16; ++kk) {
                const uint32_t off = static_cast<uint32_t>(kk >> 2) * kAttnHalfBytes +
                                     static_cast<uint32_t>(kk & 3) * 32u;
                umma_bf16(tmem + static_cast<uint32_t>(t * 256 + 128), desc_kmajor_sw128(pbase + off),
                          desc_mnmajor_sw128(base + static_cast<uint32_t>(kk) * 2048u, kAttnHalfBytes),
                          idesc_o, (blk > 0 || kk > 0) ? 1u : 0u);
              }
              umma_commit(smem_u32(&o_done[t]));
            }
          }
          if (ok) umma_commit(smem_u32(&empty[st]));
        }
        gb0 += nblk;
      }
      // every MMA issued must finish before the TMEM is freed
      umma_commit(smem_u32(final_bar));
      drain_wait(smem_u32(final_bar), 0, 50ull * 1000ull * 1000ull);
    }
    __syncwarp();
  } else {
    // ---------------- warps 0-7: tile t = warp / 4; thread r of the tile owns
    // query row r (TMEM lane r).  Every thread takes the same arrivals
    // whatever its waits returned.
    grid_dependency_wait();  // ctx may still be read by a preceding kernel
    const int t = warp >> 2;
    const int r = threadIdx.x & (kPrefillRows - 1);
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_tm = tmem + lane_addr + static_cast<uint32_t>(t * 256);
    const uint32_t o_tm = s_tm + 128u;
    // row r of P: 16-byte piece j (keys 8 j .. 8 j + 7) of d-half j / 8 sits at
    // piece (j mod 8) xor (r mod 8) of the row's 128 bytes
    const uint32_t p_row = smem_u32(ps + t * kAttnBlockBytes) + static_cast<uint32_t>(r) * 128u;
    const uint32_t sw = static_cast<uint32_t>(r & 7);
    const float c2 = p.scale_log2;
    bool ok = true;
    int gb0 = 0;  // running index of the item's block 0
    for (int wi = 0;; ++wi) {
      const int j = prefill2_item(wi, c, C, nwork);
      if (j < 0) break;
      const Prefill2Item it = prefill2_decode(j, p);
      const int pos = p.past + it.q0 + r;  // rows at or past T are padding, never stored
      float m_used = neg_inf();
      float l = 0.0f;
      for (int b = 0; b < it.nblk; ++b) {
        const int gb = gb0 + b;
        ok = __all_sync(0xffffffffu, ok && wait_parity(smem_u32(&s_full[t]), gb & 1, abort_flag));
        tc_fence_after();
        uint32_t s[kAttnBlockKeys];
        if (ok) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            tmem_ld32(s_tm + static_cast<uint32_t>(32 * q), *reinterpret_cast<uint32_t(*)[32]>(s + 32 * q));
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < kAttnBlockKeys; ++k) s[k] = 0u;
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&s_free[t]));  // the next S may overwrite the columns
        const int key0 = b * kAttnBlockKeys;
        if (key0 + kAttnBlockKeys - 1 > p.past + it.q0) {  // a block on the diagonal
#pragma unroll
          for (int k = 0; k < kAttnBlockKeys; ++k)
            if (key0 + k > pos) s[k] = __float_as_uint(neg_inf());
        }
        float mx4[4] = {neg_inf(), neg_inf(), neg_inf(), neg_inf()};  // four independent chains
#pragma unroll
        for (int k = 0; k < kAttnBlockKeys; ++k) mx4[k & 3] = fmaxf(mx4[k & 3], __uint_as_float(s[k]));
        const float mb = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * c2;  // c2 > 0, so the maximum commutes with the scaling
        const bool raise = mb > m_used + kPrefillRescaleLog2;  // also the first visible key
        float alpha = 1.0f;
        if (raise) {
          alpha = m_used == neg_inf() ? 0.0f : exp2_approx(m_used - mb);
          m_used = mb;
        }
        const float neg_m = -m_used;
        float sum0 = 0.0f, sum1 = 0.0f;
        uint32_t pk[kAttnBlockKeys / 2];
#pragma unroll
        for (int k = 0; k < kAttnBlockKeys / 2; ++k) {
          const float p0 = exp2_approx(fmaf(__uint_as_float(s[2 * k]), c2, neg_m));
          const float p1 = exp2_approx(fmaf(__uint_as_float(s[2 * k + 1]), c2, neg_m));
          sum0 += p0;
          sum1 += p1;
          pk[k] = pack_bf16x2(p0, p1);
        }
        l = l * alpha + (sum0 + sum1);
        // P replaces the previous block's P (also the last item's) and O is
        // rescaled: both wait for the previous P V product
        if (gb > 0)
          ok = __all_sync(0xffffffffu, ok && wait_parity(smem_u32(&o_done[t]), (gb - 1) & 1, abort_flag));
        tc_fence_after();
#pragma unroll
        for (int jj = 0; jj < kAttnBlockKeys / 8; ++jj) {
          const uint32_t a = p_row + static_cast<uint32_t>(jj >> 3) * kAttnHalfBytes +
                             ((static_cast<uint32_t>(jj & 7) ^ sw) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * jj]),
                       "r"(pk[4 * jj + 1]), "r"(pk[4 * jj + 2]), "r"(pk[4 * jj + 3])
                       : "memory");
        }
        if (b > 0 && ok && __any_sync(0xffffffffu, raise)) {
          // lanes that keep m use alpha = 1
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t o[32];
            const uint32_t a = o_tm + static_cast<uint32_t>(32 * q);
            tmem_ld32(a, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(a, o);
          }
          tmem_wait_st();
        }
        fence_proxy_async_smem();  // P is read by the MMA (async proxy)
        tc_fence_before();
        mbar_arrive(smem_u32(&p_full[t]));
      }
      gb0 += it.nblk;
      ok = __all_sync(0xffffffffu, ok && wait_parity(smem_u32(&o_done[t]), (gb0 - 1) & 1, abort_flag));
      tc_fence_after();
      if (ok) {
        const float inv = 1.0f / l;
        const bool valid = it.q0 + r < p.T;
        uint4* dst = reinterpret_cast<uint4*>(p.ctx + static_cast<size_t>(it.q0 + r) * p.nq * kAttnHeadDim +
                                              static_cast<size_t>(it.h0 + t) * kAttnHeadDim);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t o[32];
          tmem_ld32(o_tm + static_cast<uint32_t>(32 * q), o);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int w = 0; w < 4; ++w)
              dst[4 * q + w] = make_uint4(
                  pack_bf16x2(__uint_as_float(o[8 * w]) * inv, __uint_as_float(o[8 * w + 1]) * inv),
                  pack_bf16x2(__uint_as_float(o[8 * w + 2]) * inv, __uint_as_float(o[8 * w + 3]) * inv),
                  pack_bf16x2(__uint_as_float(o[8 * w + 4]) * inv, __uint_as_float(o[8 * w + 5]) * inv),
                  pack_bf16x2(__uint_as_float(o[8 * w + 6]) * inv, __uint_as_float(o[8 * w + 7]) * inv));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&o_free[t]));  // the next item's first product may overwrite O
    }
  }
  __syncthreads();
  grid_launch_dependents();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512u);
  }
}

}  // namespace tpb
