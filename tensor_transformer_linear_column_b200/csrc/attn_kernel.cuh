// attn_kernel.cuh -- the attention core between the QKV projection and the
// output projection, for decode: the T new tokens of one sequence attend over
// its key-value cache, head by head.
//
// Tensor parallelism gives each shard whole attention heads and the KV cache
// of its key-value heads, so the core needs no exchange (xingyuzhitong.com
// "Tensor vs Pipeline Parallelism", section "Tensor parallelism: split inside
// each layer"; drpranayjha.com "AI Infrastructure series, Part 5", section
// "How does tensor parallelism split a layer?").  On one GPU the t shards are
// the groups of key-value heads the grid walks; nothing is summed across them.
//
// What is computed (grouped-query causal attention, scores q.k / sqrt(d)):
// query head h reads key-value head g = h / G (G = nq / nkv); new token i sits
// at position past + i and sees cached keys 0 .. past + i.  The kernels:
//   attn_decode_kernel    CTA (chunk c, key-value head g, token group z):
//                         keys [c C, (c + 1) C) of head g against the queries
//                         of its G heads x Tq tokens; writes an unnormalised
//                         partial (running max m, sum l, sum of p v).  The
//                         CTAs whose chunk holds rows [past, past + T) first
//                         copy the new tokens' K and V from qkv into them;
//   attn_combine_kernel   per (token, query head): the partials of all chunks
//                         merged in a fixed order, divided by the total sum.
//
// attn_decode_kernel, per CTA (blocks of 128 keys; a 32 KB ring stage holds
// one block of K or of V, loaded by TMA in the order K_0, K_1, V_0, K_2, V_1, ...):
//   S_b^T[key, n] = K_b Q^T    tcgen05.mma, keys as M, the N = G Tq query rows
//                              (token-major, head-minor) as N, d = 128 as K, into
//                              one of two TMEM score slots
//   softmax of block b         the four epilogue warps (one key per thread):
//                              mask, the block maximum per query row, the
//                              running maximum m of accumulator b % 2,
//                              p = 2^(s - m) rounded to bf16 into one of two
//                              shared-memory P slots (the next MMA's K-major B
//                              operand), the running sum l rescaled by
//                              alpha = 2^(m_old - m), and that accumulator
//                              rescaled by alpha in TMEM
//   O_{b%2}^T[d, n] += V_b^T P_b^T   tcgen05.mma, d as M: V is read MN-major
//                              straight from its [key][d] tile, keys as K
// Even and odd blocks accumulate into separate O's with their own running
// maxima and sums, merged at the end: block b's softmax then waits only for
// block b - 2's P V product (long done), never for block b - 1's, so the
// MMA of one block overlaps the softmax of the next.  The scores of block
// b + 1 are also computed while block b's softmax runs.  HBM traffic is
// the cache read once per token group (K and V, 512 bytes per key at d = 128)
// plus partials of (d + 2) * 4 bytes per query row per chunk.
#pragma once

#include "ptx.cuh"

namespace tpb {

constexpr int kAttnHeadDim = 128;
constexpr int kAttnBlockKeys = 128;
constexpr int kAttnMaxStages = 2;  // the two MMA issuers rely on exactly two (see below)
// warp 0 TMA; warp 1 issues the score MMAs, warp 6 the P V MMAs; warps 2-5
// softmax / epilogue
constexpr int kAttnThreads = 224;
constexpr int kAttnBlockBytes = kAttnBlockKeys * kAttnHeadDim * 2;  // 32 KB
constexpr int kAttnHalfBytes = kAttnBlockBytes / 2;                // one 64-wide d half
__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

struct AttnParams {
  int T;          // new tokens
  int past;       // cached tokens before them
  int L;          // past + T: keys visible to the last token
  int nq, nkv, G; // query heads, key-value heads, G = nq / nkv
  int Tq;         // tokens per token group (grid z)
  int n_pad;      // query rows per CTA: G * Tq, 16 or 32
  int nblk;       // key blocks of 128 in [0, L)
  int nb;         // key blocks per chunk (the last chunk may have fewer)
  int chunks;     // chunks per key-value head
  int stages;     // ring depth
  int tmem_cols;  // TMEM columns allocated (power of two)
  float scale_log2;  // log2(e) / sqrt(d)
  float* part_o;  // [groups][nkv][chunks][n_pad][d] unnormalised sums of p v
  float* part_ml; // [groups][nkv][chunks][n_pad][2]  (max m, sum l) in base-2 units
  // the new tokens' keys and values, copied into the caches by the CTAs whose
  // chunk holds rows [past, past + T)
  const uint16_t* qkv;  // [T, (nq + 2 nkv) d]
  uint16_t* k_cache;    // [nkv, max_len, d]
  uint16_t* v_cache;
  int max_len;
};

// Order this thread's generic-proxy global writes before later async-proxy
// (TMA) reads of them.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Shared memory (dynamic, base rounded up to 1024 B): ring [stages][32 KB],
// Q [2 d halves][n_pad][64] bf16, P [2 slots][2 key halves][n_pad][64] bf16,
// reduction scratch [2][4][32] floats, m / l [2 accumulators][32] and alpha
// [32] floats, barriers.
__host__ __device__ inline int attn_q_bytes(int n_pad) { return n_pad * kAttnHeadDim * 2; }
__host__ __device__ inline int attn_smem_bytes(int stages, int n_pad) {
  return 1024 + stages * kAttnBlockBytes + 3 * attn_q_bytes(n_pad) + 2 * 4 * 32 * 4 + 5 * 32 * 4 +
         (2 * kAttnMaxStages + 11) * 8 + 16;
}

// Reduce kRows per-lane values (one per query row) over the 32 lanes of a warp
// with a transposing butterfly: at offset o a lane keeps the half of its rows
// selected by bit o of its lane index and trades the other half with lane
// ^ o, so kRows - 1 shuffles in total instead of 5 kRows.  On return v[0] holds
// the warp's reduction of row ((lane >> 1) & 15) for kRows = 16 (lanes 2c and
// 2c + 1 both hold row c), or of row `lane` for kRows = 32.
template <int kRows, bool kMax>
__device__ __forceinline__ float warp_rows_reduce(float (&v)[kRows], int lane) {
  int n = kRows;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (n > 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < kRows / 2; ++i) {
        if (i < n / 2) {
          const float send = upper ? v[i] : v[i + n / 2];
          const float keep = upper ? v[i + n / 2] : v[i];
          const float recv = __shfl_xor_sync(0xffffffffu, send, o);
          v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
        }
      }
      n >>= 1;
    } else {
      const float recv = __shfl_xor_sync(0xffffffffu, v[0], o);
      v[0] = kMax ? fmaxf(v[0], recv) : v[0] + recv;
    }
  }
  return v[0];
}

// Two CTAs per SM (the ring of one overlaps the softmax of the other): at most
// 170 registers per thread.  kRows = n_pad (16 or 32).
template <int kRows>
__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tmap_q,
                       const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr uint32_t kQHalf = kRows * 128u;  // bytes of one 64-wide half of a [kRows][128] tile
  uint8_t* ring = smem;
  uint8_t* qs = ring + p.stages * kAttnBlockBytes;
  uint8_t* ps = qs + 2 * kQHalf;                          // [2 slots][2 halves][kRows][128 B]
  float* red_m = reinterpret_cast<float*>(ps + 4 * kQHalf);  // [4][32]
  float* red_s = red_m + 4 * 32;                             // [4][32]
  float* m_s = red_s + 4 * 32;                               // [2][32] running maxima
  float* l_s = m_s + 2 * 32;                                 // [2][32] running sums
  float* a_s = l_s + 2 * 32;                                 // [32] this block's alpha
  uint64_t* bars = reinterpret_cast<uint64_t*>(a_s + 32);
  uint64_t* full_bar = bars;                         // [kAttnMaxStages]
  uint64_t* empty_bar = bars + kAttnMaxStages;       // [kAttnMaxStages]
  uint64_t* q_bar = bars + 2 * kAttnMaxStages;
  uint64_t* s_full = q_bar + 1;                      // [2] scores of a block in TMEM slot
  uint64_t* s_free = q_bar + 3;                      // [2] slot read by the softmax (128)
  uint64_t* p_full = q_bar + 5;                      // [2] P slot written, O rescaled (128)
  uint64_t* o_done = q_bar + 7;                      // [2] the P V product into O_slot done
  uint64_t* final_bar = q_bar + 9;                   // [2] one per MMA issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  const int g = blockIdx.y;
  const int grp = blockIdx.z;
  const int blk0 = chunk * p.nb;
  const int nbc = p.nblk - blk0 < p.nb ? p.nblk - blk0 : p.nb;  // blocks of this chunk
  const int key0 = blk0 * kAttnBlockKeys;
  const int tok0 = grp * p.Tq;
  const int nload = 2 * nbc;
  const int stages = p.stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(q_bar), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), 128);
      mbar_init(smem_u32(&p_full[i]), 128);
      mbar_init(smem_u32(&o_done[i]), 1);
    }
    mbar_init(smem_u32(&final_bar[0]), 1);
    mbar_init(smem_u32(&final_bar[1]), 1);
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
  // S slots at columns 0 and kRows, O_0 at 2 kRows, O_1 at 3 kRows
  const uint32_t tmem = *tmem_slot;
  const uint32_t o_col = 2u * kRows;

  // load / MMA item i: K_0, then K_b, V_{b-1} for b = 1 .. nbc-1, then V_{nbc-1}
  auto item = [nload](int i, bool& is_v) -> int {
    if (i == 0) { is_v = false; return 0; }
    if (i == nload - 1) { is_v = true; return (nload >> 1) - 1; }
    is_v = (i & 1) == 0;
    return is_v ? (i >> 1) - 1 : (i + 1) >> 1;
  };

  if (warp == 0) {
    // ---------------- the new tokens' K and V rows of head g that fall in this
    // chunk go into the caches first (the whole warp, 16 bytes per lane per
    // step), then the warp's writes are ordered before the TMA loads of them
    grid_dependency_wait();  // qkv comes from the preceding kernel
    {
      const int r0 = key0 > p.past ? key0 : p.past;
      const int kend = key0 + nbc * kAttnBlockKeys;
      const int r1 = kend < p.L ? kend : p.L;
      constexpr int kVec = kAttnHeadDim / 8;  // 16-byte pieces of a head row
      const size_t ld = static_cast<size_t>(p.nq + 2 * p.nkv) * kAttnHeadDim;
      for (int e = lane; e < (r1 - r0) * kVec * 2; e += 32) {
        const int piece = e % kVec;
        const int which = (e / kVec) & 1;  // 0 = K, 1 = V
        const int row = r0 + e / (2 * kVec);
        const int tok = row - p.past;
        const uint4* src = reinterpret_cast<const uint4*>(
            p.qkv + static_cast<size_t>(tok) * ld +
            static_cast<size_t>(p.nq + which * p.nkv + g) * kAttnHeadDim) + piece;
        uint16_t* cache = which ? p.v_cache : p.k_cache;
        uint4* dst = reinterpret_cast<uint4*>(
            cache + (static_cast<size_t>(g) * p.max_len + row) * kAttnHeadDim) + piece;
        *dst = __ldg(src);
      }
      fence_proxy_async_global();
      __syncwarp();
    }
    if (lane == 0) {
      // ---------------- TMA producer
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
      const uint32_t qb = smem_u32(q_bar);
      mbar_arrive_expect_tx(qb, 2u * kQHalf);
      tma_load_3d(smem_u32(qs), &tmap_q, qb, 0, g * p.G, tok0);
      tma_load_3d(smem_u32(qs) + kQHalf, &tmap_q, qb, 64, g * p.G, tok0);
      uint32_t issued = 0u, phases = 0u;
      int s = 0;
      uint32_t ph = 0u;
      for (int i = 0; i < nload; ++i) {
        if (!wait_parity(smem_u32(&empty_bar[s]), ph ^ 1u, abort_flag)) break;
        bool is_v;
        const int b = item(i, is_v);
        const uint32_t fb = smem_u32(&full_bar[s]);
        const uint32_t dst = smem_u32(ring + s * kAttnBlockBytes);
        const CUtensorMap* map = is_v ? &tmap_v : &tmap_k;
        const int kb = key0 + b * kAttnBlockKeys;
        mbar_arrive_expect_tx(fb, kAttnBlockBytes);
        tma_load_3d(dst, map, fb, 0, kb, g);
        tma_load_3d(dst + kAttnHalfBytes, map, fb, 64, kb, g);
        issued |= 1u << s;
        phases = (phases & ~(1u << s)) | (ph << s);
        if (++s == stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (*abort_flag) {
        drain_wait(qb, 0, 50ull * 1000ull * 1000ull);
        for (int st = 0; st < stages; ++st)
          if (issued & (1u << st))
            drain_wait(smem_u32(&full_bar[st]), (phases >> st) & 1u, 50ull * 1000ull * 1000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 6) {
    if (lane == 0) {
      // ---------------- MMA issuers: warp 1 takes the K items (scores), warp 6
      // the V items (P V); both walk the load order to track ring stages.
      // With two stages, stage 0 holds K_0 and then only V blocks, and stage 1
      // only K blocks except the last item, V_{nbc-1}.  Where a stage changes
      // hands (K_0 -> V_0, K_{nbc-1} -> V_{nbc-1}), the P V issuer waits for
      // that block's P first, which needs the block's scores, so the previous
      // fill has landed: a parity wait never matches an older phase.  The
      // score MMAs so never queue behind a P V product that waits for its
      // softmax.
      const bool pv_role = warp == 6;
      const uint32_t idesc_s = idesc_bf16_f32(128, kRows);               // K, Q both K-major
      const uint32_t idesc_o = idesc_bf16_f32(128, kRows, true, false);  // V^T MN-major, P K-major
      bool ok = pv_role || wait_parity(smem_u32(q_bar), 0, abort_flag);
      tc_fence_after();
      int s = 0;
      uint32_t ph = 0u;
      for (int i = 0; ok && i < nload; ++i) {
        bool is_v;
        const int b = item(i, is_v);
        const int slot = b & 1;
        if (is_v != pv_role) {  // the other issuer's item
          if (++s == stages) {
            s = 0;
            ph ^= 1u;
          }
          continue;
        }
        if (!is_v) {
          // the score slot must have been read by the softmax of block b - 2
          if (b >= 2 && !wait_parity(smem_u32(&s_free[slot]), ((b - 2) >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
        } else {
          // P_b written and O rescaled for block b
          if (!wait_parity(smem_u32(&p_full[slot]), (b >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
        }
        if (!wait_parity(smem_u32(&full_bar[s]), ph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(ring + s * kAttnBlockBytes);
        if (!is_v) {
          // S_b^T = K_b Q^T, K = d in steps of 16: steps 0-3 in d half 0, 4-7 in half 1
          const uint32_t d = tmem + static_cast<uint32_t>(slot * kRows);
#pragma unroll
          for (int kk = 0; kk < kAttnHeadDim / 16; ++kk) {
            const uint32_t hk = static_cast<uint32_t>(kk >> 2), ck = static_cast<uint32_t>(kk & 3);
            umma_bf16(d, desc_kmajor_sw128(st + hk * kAttnHalfBytes + ck * 32u),
                      desc_kmajor_sw128(smem_u32(qs) + hk * kQHalf + ck * 32u), idesc_s,
                      kk > 0 ? 1u : 0u);
          }
          umma_commit(smem_u32(&empty_bar[s]));
          umma_commit(smem_u32(&s_full[slot]));
        } else {
          // O^T += V_b^T P_b^T, K = keys in steps of 16: V MN-major (d halves
          // 16 KB apart, 8-key groups 1024 B apart); P slot's two 64-key halves
          const uint32_t pb = smem_u32(ps) + static_cast<uint32_t>(slot) * 2u * kQHalf;
#pragma unroll
          for (int kk = 0; kk < kAttnBlockKeys / 16; ++kk) {
            const uint32_t hk = static_cast<uint32_t>(kk >> 2), ck = static_cast<uint32_t>(kk & 3);
            umma_bf16(tmem + o_col + static_cast<uint32_t>(slot * kRows),
                      desc_mnmajor_sw128(st + static_cast<uint32_t>(kk) * 2048u, kAttnHalfBytes),
                      desc_kmajor_sw128(pb + hk * kQHalf + ck * 32u), idesc_o,
                      (b >= 2 || kk > 0) ? 1u : 0u);
          }
          umma_commit(smem_u32(&empty_bar[s]));
          umma_commit(smem_u32(&o_done[slot]));
        }
        if (++s == stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      // every MMA issued by this thread is complete once its final barrier flips
      umma_commit(smem_u32(&final_bar[pv_role ? 1 : 0]));
      drain_wait(smem_u32(&final_bar[pv_role ? 1 : 0]), 0, 50ull * 1000ull * 1000ull);
    }
    __syncwarp();
  } else {
    // ---------------- warps 2-5: softmax per block, O rescale, the partial.
    // Thread r of the 128 owns TMEM lane r: key r of each block, and d = r of O.
    // Every thread takes the same named barriers and arrivals whatever its
    // waits returned, so a timed-out wait cannot leave a barrier short.
    grid_dependency_wait();  // the partial buffers may still be read by a preceding kernel
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int et = threadIdx.x - 64;  // 0..127
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    const int g_shift = __ffs(p.G) - 1;  // G is a power of two
    int lim[kRows];                      // last key each query row may see (-1: padding)
#pragma unroll
    for (int j = 0; j < kRows; ++j) {
      const int tok = tok0 + (j >> g_shift);
      lim[j] = tok < p.T ? p.past + tok : -1;
    }
    if (et < kRows) {
      m_s[et] = m_s[32 + et] = neg_inf();
      l_s[et] = l_s[32 + et] = 0.0f;
    }
    // P half (key / 64) of row n: 128-byte rows, 16-byte chunk (key % 64) / 8
    // stored at chunk ^ (n % 8)
    const int kc = (r & 63) >> 3, kw = (r & 7) * 2;
    bool ok = true;
    for (int b = 0; b < nbc; ++b) {
      const int slot = b & 1;
      ok = __all_sync(0xffffffffu, ok && wait_parity(smem_u32(&s_full[slot]), (b >> 1) & 1,
                                                     abort_flag));
      tc_fence_after();
      uint32_t v[kRows];
      if (ok) {
#pragma unroll
        for (int c = 0; c < kRows; c += 16)
          tmem_ld16(tmem + lane_addr + static_cast<uint32_t>(slot * kRows + c),
                    *reinterpret_cast<uint32_t(*)[16]>(v + c));
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < kRows; ++j) v[j] = 0u;
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&s_free[slot]));
      const int key = key0 + b * kAttnBlockKeys + r;
      float sc[kRows];
#pragma unroll
      for (int j = 0; j < kRows; ++j)
        sc[j] = key <= lim[j] ? __uint_as_float(v[j]) * p.scale_log2 : neg_inf();
      // the block maximum per row: a transposing warp butterfly, then the four
      // warps in order
      const int my_row = kRows == 32 ? lane : (lane >> 1) & 15;
      {
        float mx[kRows];
#pragma unroll
        for (int j = 0; j < kRows; ++j) mx[j] = sc[j];
        const float m = warp_rows_reduce<kRows, true>(mx, lane);
        if (kRows == 32 || (lane & 1) == 0) red_m[q4 * 32 + my_row] = m;
      }
      named_barrier_sync(1, 128);
      float* ms = m_s + slot * 32;  // accumulator b % 2's running state
      float* ls = l_s + slot * 32;
      if (et < kRows) {
        const float mb = fmaxf(fmaxf(red_m[et], red_m[32 + et]), fmaxf(red_m[64 + et], red_m[96 + et]));
        const float mo = ms[et];
        const float mn = fmaxf(mo, mb);
        a_s[et] = mo == neg_inf() ? 0.0f : exp2f(mo - mn);
        ms[et] = mn;
      }
      named_barrier_sync(1, 128);
      // the P slot and accumulator b % 2 are free once block b - 2's P V
      // product is done
      if (b >= 2)
        ok = __all_sync(0xffffffffu, ok && wait_parity(smem_u32(&o_done[slot]),
                                                       ((b - 2) >> 1) & 1, abort_flag));
      uint8_t* pslot = ps + static_cast<size_t>(slot) * 2u * kQHalf + static_cast<size_t>(r >> 6) * kQHalf;
      {
        // p of rows j (this lane's key) as bf16; lanes 2m and 2m + 1 (keys
        // 2m, 2m + 1) then trade one value per row pair so that each writes one
        // 4-byte word: the even lane row j, the odd lane row j + 1
        float pr[kRows];
        uint16_t pb16[kRows];
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
          const float m = ms[j];
          const float e = sc[j] == neg_inf() ? 0.0f : exp2f(sc[j] - m);
          const __nv_bfloat16 hb = __float2bfloat16_rn(e);
          pb16[j] = *reinterpret_cast<const uint16_t*>(&hb);
          pr[j] = __bfloat162float(hb);
        }
        const bool odd = (lane & 1) != 0;
        const int kw4 = kw & ~3;  // the word of keys 2m, 2m + 1
#pragma unroll
        for (int j = 0; j < kRows; j += 2) {
          // even lane sends its row j + 1 value, odd lane its row j value
          const uint32_t give = odd ? pb16[j] : pb16[j + 1];
          const uint32_t got = __shfl_xor_sync(0xffffffffu, give, 1);
          const int row = odd ? j + 1 : j;
          const uint32_t word = odd ? (got | (static_cast<uint32_t>(pb16[j + 1]) << 16))
                                    : (static_cast<uint32_t>(pb16[j]) | (got << 16));
          *reinterpret_cast<uint32_t*>(pslot + row * 128 + ((kc ^ (row & 7)) << 4) + kw4) = word;
        }
        const float sm = warp_rows_reduce<kRows, false>(pr, lane);
        if (kRows == 32 || (lane & 1) == 0) red_s[q4 * 32 + my_row] = sm;
      }
      named_barrier_sync(1, 128);
      if (et < kRows)
        ls[et] = fmaf(ls[et], a_s[et],
                      ((red_s[et] + red_s[32 + et]) + red_s[64 + et]) + red_s[96 + et]);
      // O_{b%2} (the P V products of blocks b - 2, b - 4, ...) times alpha;
      // block b - 2's product was waited for above
      if (b >= 2 && ok) {
        tc_fence_after();
        const uint32_t oc = o_col + static_cast<uint32_t>(slot * kRows);
        uint32_t o[kRows];
#pragma unroll
        for (int c = 0; c < kRows; c += 16)
          tmem_ld16(tmem + lane_addr + oc + static_cast<uint32_t>(c),
                    *reinterpret_cast<uint32_t(*)[16]>(o + c));
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < kRows; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * a_s[j]);
#pragma unroll
        for (int c = 0; c < kRows; c += 16)
          tmem_st16(tmem + lane_addr + oc + static_cast<uint32_t>(c),
                    *reinterpret_cast<uint32_t(*)[16]>(o + c));
        tmem_wait_st();
      }
      fence_proxy_async_smem();  // P is read by the MMA through the async proxy
      tc_fence_before();
      mbar_arrive(smem_u32(&p_full[slot]));
    }
    // the last P V products of both accumulators, then the partial: the two
    // merged with weights 2^(m_x - M), M = max(m_0, m_1); O^T has lane = d,
    // column = query row
    if (nbc > 0)
      ok = __all_sync(0xffffffffu, ok && wait_parity(smem_u32(&o_done[(nbc - 1) & 1]),
                                                     ((nbc - 1) >> 1) & 1, abort_flag));
    if (nbc > 1)
      ok = __all_sync(0xffffffffu, ok && wait_parity(smem_u32(&o_done[nbc & 1]),
                                                     ((nbc - 2) >> 1) & 1, abort_flag));
    named_barrier_sync(1, 128);  // every thread's m / l updates are visible
    float* w0s = red_m;          // [32] weight of O_0, [32 + n] weight of O_1
    if (et < kRows) {
      const float m0 = m_s[et], m1 = nbc > 1 ? m_s[32 + et] : neg_inf();
      const float M = fmaxf(m0, m1);
      const float w0 = m0 == neg_inf() ? 0.0f : exp2f(m0 - M);
      const float w1 = m1 == neg_inf() ? 0.0f : exp2f(m1 - M);
      w0s[et] = w0;
      w0s[32 + et] = w1;
      const float L = w0 * l_s[et] + (nbc > 1 ? w1 * l_s[32 + et] : 0.0f);
      const size_t slot = (static_cast<size_t>(grp) * p.nkv + g) * p.chunks + chunk;
      float* pml = p.part_ml + slot * static_cast<size_t>(kRows) * 2;
      pml[2 * et] = ok ? M : neg_inf();
      pml[2 * et + 1] = ok ? L : 0.0f;
    }
    named_barrier_sync(1, 128);
    tc_fence_after();
    const size_t slot = (static_cast<size_t>(grp) * p.nkv + g) * p.chunks + chunk;
    float* po = p.part_o + slot * static_cast<size_t>(kRows) * kAttnHeadDim;
#pragma unroll
    for (int c = 0; c < kRows; c += 16) {
      uint32_t v0[16], v1[16];
      if (ok) {
        tmem_ld16(tmem + lane_addr + o_col + static_cast<uint32_t>(c), v0);
        if (nbc > 1) tmem_ld16(tmem + lane_addr + o_col + kRows + static_cast<uint32_t>(c), v1);
        tmem_wait_ld();
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        // O_1 is read only when it was written (nbc > 1): unwritten TMEM may
        // hold any bit pattern, and 0 * NaN is NaN
        float o = ok ? w0s[c + j] * __uint_as_float(v0[j]) : 0.0f;
        if (ok && nbc > 1) o = fmaf(w0s[32 + c + j], __uint_as_float(v1[j]), o);
        po[static_cast<size_t>(c + j) * kAttnHeadDim + r] = o;
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  grid_launch_dependents();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
  }
}

// One CTA of kCombineWarps warps per (token i, query head h): merge the chunk
// partials of head h.  M = max_c m_c; ctx = sum_c 2^(m_c - M) o_c /
// sum_c 2^(m_c - M) l_c, one bf16 rounding.  Warp w takes chunks w,
// w + kCombineWarps, ... in order with a running maximum M_w (its sums are
// rescaled by 2^(M_w,old - M_w,new) when a chunk raises it), lane l owning
// d = 4 l .. 4 l + 3, all of its chunks' loads issued before the first use;
// warp 0 then takes M = max_w M_w and adds the warps' sums scaled by
// 2^(M_w - M) in warp order.  Every order is fixed, so the result is
// bit-identical from run to run, and a merge costs one memory round trip.
constexpr int kCombineWarps = 8;
constexpr int kCombineMaxPerWarp = 8;  // chunks per warp held in registers at once
__global__ void __launch_bounds__(kCombineWarps * 32)
    attn_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                        int T, int nq, int nkv, int G, int Tq, int n_pad, int chunks,
                        uint16_t* __restrict__ ctx) {
  __shared__ float4 red_o[kCombineWarps][32];
  __shared__ float red_l[kCombineWarps];
  __shared__ float red_m[kCombineWarps];
  grid_dependency_wait();
  const int wid = blockIdx.x;  // (token, query head)
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int i = wid / nq;
  const int h = wid % nq;
  const int g = h / G;
  const int grp = i / Tq;
  const int n = (i - grp * Tq) * G + (h - g * G);
  const size_t base = (static_cast<size_t>(grp) * nkv + g) * chunks;
  const float* ml = part_ml + (base * n_pad + n) * 2;  // chunk c at ml[c * n_pad * 2]
  const size_t ml_stride = static_cast<size_t>(n_pad) * 2;
  const float* po = part_o + (base * n_pad + n) * kAttnHeadDim + 4 * lane;
  const size_t o_stride = static_cast<size_t>(n_pad) * kAttnHeadDim;
  float Mw = neg_inf();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = 0.0f;
  for (int c0 = warp; c0 < chunks; c0 += kCombineWarps * kCombineMaxPerWarp) {
    float2 mlv[kCombineMaxPerWarp];
    float4 ov[kCombineMaxPerWarp];
#pragma unroll
    for (int k = 0; k < kCombineMaxPerWarp; ++k) {
      const int c = c0 + k * kCombineWarps;
      if (c < chunks) {
        mlv[k] = __ldg(reinterpret_cast<const float2*>(ml + c * ml_stride));
        ov[k] = __ldg(reinterpret_cast<const float4*>(po + c * o_stride));
      }
    }
#pragma unroll
    for (int k = 0; k < kCombineMaxPerWarp; ++k) {
      const int c = c0 + k * kCombineWarps;
      if (c < chunks && mlv[k].x != neg_inf()) {
        if (mlv[k].x > Mw) {
          const float s = Mw == neg_inf() ? 0.0f : exp2f(Mw - mlv[k].x);
          acc.x *= s;
          acc.y *= s;
          acc.z *= s;
          acc.w *= s;
          L *= s;
          Mw = mlv[k].x;
        }
        const float w = exp2f(mlv[k].x - Mw);
        acc.x = fmaf(w, ov[k].x, acc.x);
        acc.y = fmaf(w, ov[k].y, acc.y);
        acc.z = fmaf(w, ov[k].z, acc.z);
        acc.w = fmaf(w, ov[k].w, acc.w);
        L = fmaf(w, mlv[k].y, L);
      }
    }
  }
  red_o[warp][lane] = acc;
  if (lane == 0) {
    red_l[warp] = L;
    red_m[warp] = Mw;
  }
  __syncthreads();
  if (warp != 0) return;
  float M = red_m[0];
#pragma unroll
  for (int w = 1; w < kCombineWarps; ++w) M = fmaxf(M, red_m[w]);
  float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.0f;
#pragma unroll
  for (int w = 0; w < kCombineWarps; ++w) {
    const float mw = red_m[w];
    const float s = mw == neg_inf() ? 0.0f : exp2f(mw - M);
    const float4 v = red_o[w][lane];
    sum.x = fmaf(s, v.x, sum.x);
    sum.y = fmaf(s, v.y, sum.y);
    sum.z = fmaf(s, v.z, sum.z);
    sum.w = fmaf(s, v.w, sum.w);
    lsum = fmaf(s, red_l[w], lsum);
  }
  const float inv = 1.0f / lsum;
  uint2 packed;
  packed.x = pack_bf16x2(sum.x * inv, sum.y * inv);
  packed.y = pack_bf16x2(sum.z * inv, sum.w * inv);
  *reinterpret_cast<uint2*>(ctx + static_cast<size_t>(i) * nq * kAttnHeadDim +
                            static_cast<size_t>(h) * kAttnHeadDim + 4 * lane) = packed;
}

}  // namespace tpb
