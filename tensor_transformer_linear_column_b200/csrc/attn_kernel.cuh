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
//   kv_append_kernel      copies the new tokens' K and V from qkv into the
//                         cache rows [past, past + T);
//   attn_decode_kernel    CTA (chunk c, key-value head g, token group z):
//                         keys [c C, (c + 1) C) of head g against the queries
//                         of its G heads x Tq tokens; writes an unnormalised
//                         partial (running max m, sum l, sum of p v);
//   attn_combine_kernel   per (token, query head): the partials of all chunks
//                         merged in chunk order, divided by the total sum.
//
// attn_decode_kernel, per CTA (one M = 128 key block = 32 KB of K or V per
// ring stage, loaded by TMA):
//   S^T[key, n] = K_blk Q^T    tcgen05.mma, keys as M, the N = G Tq query rows
//                              (token-major, head-minor) as N, d = 128 as K;
//                              every block of the chunk into its own TMEM slice
//   softmax                    the four epilogue warps (one key per thread)
//                              mask, take the chunk maximum per query row,
//                              p = 2^(s - m) rounded to bf16 into shared memory
//                              as the next MMA's K-major B operand, sum l
//   O^T[d, n] += V_blk^T P^T   tcgen05.mma, d as M: V is read MN-major straight
//                              from its [key][d] tile, keys as K
// Because the maximum over the whole chunk is known before any P V product,
// no accumulator is ever rescaled.  HBM traffic is the cache read once per
// token group (K and V, 512 bytes per key at d = 128) plus partials of
// (d + 2) * 4 bytes per query row per chunk.
#pragma once

#include "ptx.cuh"

namespace tpb {

constexpr int kAttnHeadDim = 128;
constexpr int kAttnBlockKeys = 128;
constexpr int kAttnStages = 2;
constexpr int kAttnThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2-5 softmax / epilogue
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
  int nb;         // key blocks per chunk
  int chunks;     // chunks per key-value head
  int tmem_cols;  // TMEM columns allocated (power of two)
  float scale_log2;  // log2(e) / sqrt(d)
  float* part_o;  // [groups][nkv][chunks][n_pad][d] unnormalised sums of p v
  float* part_ml; // [groups][nkv][chunks][n_pad][2]  (max m, sum l) in base-2 units
};

// Shared memory (dynamic, base rounded up to 1024 B): ring [kAttnStages][32 KB],
// Q [2 halves][n_pad][64] bf16, P [nb][2 halves][n_pad][64] bf16, reduction
// scratch [4][16] floats, m / l [n_pad] floats, barriers.
__host__ __device__ inline int attn_q_bytes(int n_pad) { return n_pad * kAttnHeadDim * 2; }
__host__ __device__ inline int attn_p_bytes(int nb, int n_pad) {
  return nb * n_pad * kAttnBlockKeys * 2;
}
__host__ __device__ inline int attn_smem_bytes(int nb, int n_pad) {
  return 1024 + kAttnStages * kAttnBlockBytes + attn_q_bytes(n_pad) + attn_p_bytes(nb, n_pad) +
         4 * 16 * 4 + 2 * n_pad * 4 + (2 * kAttnStages + 5) * 8 + 16;
}

// Copy the new tokens' keys and values into the cache: for token i and
// key-value head g, qkv[i, (nq + g) d ..] -> k_cache[g, past + i, :] and
// qkv[i, (nq + nkv + g) d ..] -> v_cache[g, past + i, :], 16 bytes per thread.
__global__ void kv_append_kernel(const uint16_t* __restrict__ qkv, uint16_t* __restrict__ kc,
                                 uint16_t* __restrict__ vc, int T, int past, int max_len, int nq,
                                 int nkv) {
  grid_dependency_wait();  // qkv comes from the preceding kernel
  constexpr int kVec = kAttnHeadDim / 8;  // 16-byte pieces per head row
  const int total = T * nkv * kVec * 2;
  const size_t ld = static_cast<size_t>(nq + 2 * nkv) * kAttnHeadDim;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x) {
    const int piece = e % kVec;
    const int rest = e / kVec;
    const int g = rest % nkv;
    const int which = (rest / nkv) & 1;  // 0 = K, 1 = V
    const int i = rest / (2 * nkv);
    const uint4* src = reinterpret_cast<const uint4*>(
        qkv + static_cast<size_t>(i) * ld + static_cast<size_t>(nq + which * nkv + g) * kAttnHeadDim) + piece;
    uint16_t* cache = which ? vc : kc;
    uint4* dst = reinterpret_cast<uint4*>(
        cache + (static_cast<size_t>(g) * max_len + past + i) * kAttnHeadDim) + piece;
    *dst = *src;
  }
  grid_launch_dependents();
}

// Two CTAs per SM (the ring of one overlaps the softmax of the other): at most
// 170 registers per thread.
__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tmap_q,
                       const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint8_t* qs = ring + kAttnStages * kAttnBlockBytes;
  uint8_t* ps = qs + attn_q_bytes(p.n_pad);
  float* red = reinterpret_cast<float*>(ps + attn_p_bytes(p.nb, p.n_pad));  // [4][16]
  float* m_s = red + 4 * 16;                                                 // [n_pad]
  float* l_s = m_s + p.n_pad;                                                // [n_pad]
  uint64_t* bars = reinterpret_cast<uint64_t*>(l_s + p.n_pad);
  uint64_t* full_bar = bars;                       // [stages]
  uint64_t* empty_bar = bars + kAttnStages;        // [stages]
  uint64_t* q_bar = bars + 2 * kAttnStages;
  uint64_t* s_bar = q_bar + 1;                     // every S block is in TMEM
  uint64_t* p_bar = q_bar + 2;                     // P is in shared memory (128 arrivals)
  uint64_t* o_bar = q_bar + 3;                     // O is in TMEM
  uint64_t* final_bar = q_bar + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  const int g = blockIdx.y;
  const int grp = blockIdx.z;
  const int key0 = chunk * p.nb * kAttnBlockKeys;
  const int tok0 = grp * p.Tq;
  const int n_pad = p.n_pad;
  const uint32_t q_half = static_cast<uint32_t>(n_pad) * 128u;  // bytes of one d half of Q

  if (threadIdx.x == 0) {
    for (int s = 0; s < kAttnStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(q_bar), 1);
    mbar_init(smem_u32(s_bar), 1);
    mbar_init(smem_u32(p_bar), 128);
    mbar_init(smem_u32(o_bar), 1);
    mbar_init(smem_u32(final_bar), 1);
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
  const uint32_t tmem = *tmem_slot;
  const int nload = 2 * p.nb;  // K blocks, then V blocks

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer: Q once, then K_0 .. K_nb-1, V_0 .. V_nb-1
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
      grid_dependency_wait();  // qkv and the appended cache rows come from preceding kernels
      const uint32_t qb = smem_u32(q_bar);
      mbar_arrive_expect_tx(qb, 2u * q_half);
      tma_load_3d(smem_u32(qs), &tmap_q, qb, 0, g * p.G, tok0);
      tma_load_3d(smem_u32(qs) + q_half, &tmap_q, qb, 64, g * p.G, tok0);
      uint32_t issued = 0u, phases = 0u;
      int s = 0;
      uint32_t ph = 0u;
      for (int i = 0; i < nload; ++i) {
        if (!wait_parity(smem_u32(&empty_bar[s]), ph ^ 1u, abort_flag)) break;
        const uint32_t fb = smem_u32(&full_bar[s]);
        const uint32_t dst = smem_u32(ring + s * kAttnBlockBytes);
        const CUtensorMap* map = i < p.nb ? &tmap_k : &tmap_v;
        const int kb = key0 + (i < p.nb ? i : i - p.nb) * kAttnBlockKeys;
        mbar_arrive_expect_tx(fb, kAttnBlockBytes);
        tma_load_3d(dst, map, fb, 0, kb, g);
        tma_load_3d(dst + kAttnHalfBytes, map, fb, 64, kb, g);
        issued |= 1u << s;
        phases = (phases & ~(1u << s)) | (ph << s);
        if (++s == kAttnStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (*abort_flag) {
        drain_wait(qb, 0, 50ull * 1000ull * 1000ull);
        for (int st = 0; st < kAttnStages; ++st)
          if (issued & (1u << st))
            drain_wait(smem_u32(&full_bar[st]), (phases >> st) & 1u, 50ull * 1000ull * 1000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t idesc_s = idesc_bf16_f32(128, n_pad);               // K, Q both K-major
      const uint32_t idesc_o = idesc_bf16_f32(128, n_pad, true, false);  // V^T MN-major, P K-major
      const uint32_t o_col = static_cast<uint32_t>(p.nb * n_pad);
      bool ok = wait_parity(smem_u32(q_bar), 0, abort_flag);
      tc_fence_after();
      int s = 0;
      uint32_t ph = 0u;
      for (int i = 0; ok && i < nload; ++i) {
        if (i == p.nb) {
          // all S blocks issued: tell the softmax warps, then wait for P
          umma_commit(smem_u32(s_bar));
          if (!wait_parity(smem_u32(p_bar), 0, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        if (!wait_parity(smem_u32(&full_bar[s]), ph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(ring + s * kAttnBlockBytes);
        if (i < p.nb) {
          // S_b^T = K_b Q^T, K = d in steps of 16: steps 0-3 in d half 0, 4-7 in half 1
          const uint32_t d = tmem + static_cast<uint32_t>(i * n_pad);
#pragma unroll
          for (int kk = 0; kk < kAttnHeadDim / 16; ++kk) {
            const uint32_t hk = static_cast<uint32_t>(kk >> 2), ck = static_cast<uint32_t>(kk & 3);
            umma_bf16(d, desc_kmajor_sw128(st + hk * kAttnHalfBytes + ck * 32u),
                      desc_kmajor_sw128(smem_u32(qs) + hk * q_half + ck * 32u), idesc_s,
                      kk > 0 ? 1u : 0u);
          }
        } else {
          // O^T += V_b^T P_b^T, K = keys in steps of 16: V MN-major (d halves
          // 16 KB apart, 8-key groups 1024 B apart); P_b's two 64-key halves
          const int b = i - p.nb;
          const uint32_t pb = smem_u32(ps) + static_cast<uint32_t>(b) * 2u * q_half;
#pragma unroll
          for (int kk = 0; kk < kAttnBlockKeys / 16; ++kk) {
            const uint32_t hk = static_cast<uint32_t>(kk >> 2), ck = static_cast<uint32_t>(kk & 3);
            umma_bf16(tmem + o_col,
                      desc_mnmajor_sw128(st + static_cast<uint32_t>(kk) * 2048u, kAttnHalfBytes),
                      desc_kmajor_sw128(pb + hk * q_half + ck * 32u), idesc_o,
                      (b > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(smem_u32(&empty_bar[s]));
        if (++s == kAttnStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (ok) umma_commit(smem_u32(o_bar));
      // every MMA issued by this thread is complete once final_bar flips
      umma_commit(smem_u32(final_bar));
      drain_wait(smem_u32(final_bar), 0, 50ull * 1000ull * 1000ull);
    }
    __syncwarp();
  } else {
    // ---------------- warps 2-5: softmax and the partial's write-out.
    // Thread r of the 128 owns TMEM lane r: key r of each block, then d = r.
    grid_dependency_wait();  // the partial buffers may still be read by a preceding kernel
    const int q4 = warp & 3;                 // TMEM lane quarter of this warp
    const int r = q4 * 32 + lane;
    const int et = threadIdx.x - 64;         // 0..127, for shared-memory roles
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    bool ok = __all_sync(0xffffffffu, wait_parity(smem_u32(s_bar), 0, abort_flag));
    tc_fence_after();
    const int g_shift = __ffs(p.G) - 1;  // G is a power of two
    for (int c0 = 0; c0 < n_pad; c0 += 16) {
      // the last key each of these 16 query rows may see (-1: a padding row)
      int lim[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int tok = tok0 + ((c0 + j) >> g_shift);
        lim[j] = tok < p.T ? p.past + tok : -1;
      }
      // pass 1: the chunk maximum of columns c0 .. c0 + 15 (masked scores
      // -inf); two blocks' scores per TMEM round trip
      float mx[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) mx[j] = neg_inf();
      for (int b = 0; ok && b < p.nb; b += 2) {
        const bool two = b + 1 < p.nb;
        uint32_t v0[16], v1[16];
        tmem_ld16(tmem + lane_addr + static_cast<uint32_t>(b * n_pad + c0), v0);
        if (two) tmem_ld16(tmem + lane_addr + static_cast<uint32_t>((b + 1) * n_pad + c0), v1);
        tmem_wait_ld();
        const int key = key0 + b * kAttnBlockKeys + r;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (key <= lim[j]) mx[j] = fmaxf(mx[j], __uint_as_float(v0[j]) * p.scale_log2);
          if (two && key + kAttnBlockKeys <= lim[j])
            mx[j] = fmaxf(mx[j], __uint_as_float(v1[j]) * p.scale_log2);
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], o));
      }
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) red[q4 * 16 + j] = mx[j];
      }
      named_barrier_sync(1, 128);
      if (et < 16) {
        const float m = fmaxf(fmaxf(red[et], red[16 + et]), fmaxf(red[32 + et], red[48 + et]));
        m_s[c0 + et] = m;
      }
      named_barrier_sync(1, 128);
      float msafe[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float m = m_s[c0 + j];
        msafe[j] = m == neg_inf() ? 0.0f : m;  // a row with nothing visible: p = 0
      }
      // pass 2: p = 2^(s - m) as bf16 into P (row n = column of S, key r of the
      // block), and the sum of the rounded p of each row
      float sum[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) sum[j] = 0.0f;
      // P_b half (key / 64), row n: 128-byte rows, 16-byte chunk (key % 64) / 8
      // stored at chunk ^ (n % 8)
      const int kc = (r & 63) >> 3, kw = (r & 7) * 2;
      for (int b = 0; ok && b < p.nb; b += 2) {
        const bool two = b + 1 < p.nb;
        uint32_t v0[16], v1[16];
        tmem_ld16(tmem + lane_addr + static_cast<uint32_t>(b * n_pad + c0), v0);
        if (two) tmem_ld16(tmem + lane_addr + static_cast<uint32_t>((b + 1) * n_pad + c0), v1);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h == 1 && !two) break;
          const int bb = b + h;
          const int key = key0 + bb * kAttnBlockKeys + r;
          uint8_t* pb = ps + static_cast<size_t>(bb) * 2u * q_half + static_cast<size_t>(r >> 6) * q_half;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = c0 + j;
            const float sv = __uint_as_float(h == 0 ? v0[j] : v1[j]);
            const float e = key <= lim[j] ? exp2f(sv * p.scale_log2 - msafe[j]) : 0.0f;
            const __nv_bfloat16 hb = __float2bfloat16_rn(e);
            sum[j] += __bfloat162float(hb);
            *reinterpret_cast<__nv_bfloat16*>(pb + n * 128 + ((kc ^ (n & 7)) << 4) + kw) = hb;
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum[j] += __shfl_xor_sync(0xffffffffu, sum[j], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) red[q4 * 16 + j] = sum[j];
      }
      named_barrier_sync(1, 128);
      if (et < 16) l_s[c0 + et] = ((red[et] + red[16 + et]) + red[32 + et]) + red[48 + et];
      named_barrier_sync(1, 128);
    }
    // P is complete: make the generic-proxy writes visible to the MMA
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(smem_u32(p_bar));
    ok = __all_sync(0xffffffffu, ok && wait_parity(smem_u32(o_bar), 0, abort_flag));
    tc_fence_after();
    // O^T in TMEM: lane = d, column = query row n.  Partial of (chunk, head g,
    // group): part_o[.., n, d] (coalesced over d), part_ml[.., n] = (m, l)
    const size_t slot = (static_cast<size_t>(grp) * p.nkv + g) * p.chunks + chunk;
    float* po = p.part_o + slot * static_cast<size_t>(n_pad) * kAttnHeadDim;
    for (int c0 = 0; c0 < n_pad; c0 += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + lane_addr + static_cast<uint32_t>(p.nb * n_pad + c0), v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j)
        po[static_cast<size_t>(c0 + j) * kAttnHeadDim + r] = ok ? __uint_as_float(v[j]) : 0.0f;
    }
    if (et < n_pad) {
      float* pml = p.part_ml + slot * static_cast<size_t>(n_pad) * 2;
      pml[2 * et] = ok ? m_s[et] : neg_inf();
      pml[2 * et + 1] = ok ? l_s[et] : 0.0f;
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

// One warp per (token i, query head h): merge the chunk partials of head h in
// chunk order.  M = max_c m_c; ctx = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c,
// one bf16 rounding.  Lane l owns d = 4 l .. 4 l + 3.
__global__ void attn_combine_kernel(const float* __restrict__ part_o,
                                    const float* __restrict__ part_ml, int T, int nq, int nkv,
                                    int G, int Tq, int n_pad, int chunks,
                                    uint16_t* __restrict__ ctx) {
  grid_dependency_wait();
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= T * nq) return;
  const int i = wid / nq;
  const int h = wid % nq;
  const int g = h / G;
  const int grp = i / Tq;
  const int n = (i - grp * Tq) * G + (h - g * G);
  const size_t base = (static_cast<size_t>(grp) * nkv + g) * chunks;
  float M = neg_inf();
  for (int c = 0; c < chunks; ++c)
    M = fmaxf(M, part_ml[((base + c) * n_pad + n) * 2]);
  float L = 0.0f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c = 0; c < chunks; ++c) {
    const float m = part_ml[((base + c) * n_pad + n) * 2];
    const float w = m == neg_inf() ? 0.0f : exp2f(m - M);
    L += w * part_ml[((base + c) * n_pad + n) * 2 + 1];
    const float4 o = *reinterpret_cast<const float4*>(
        part_o + ((base + c) * n_pad + n) * kAttnHeadDim + 4 * lane);
    acc.x += w * o.x;
    acc.y += w * o.y;
    acc.z += w * o.z;
    acc.w += w * o.w;
  }
  const float inv = 1.0f / L;
  uint2 packed;
  packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  *reinterpret_cast<uint2*>(ctx + static_cast<size_t>(i) * nq * kAttnHeadDim +
                            static_cast<size_t>(h) * kAttnHeadDim + 4 * lane) = packed;
}

}  // namespace tpb
