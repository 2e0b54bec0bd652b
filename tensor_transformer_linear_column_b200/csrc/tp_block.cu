// tp_block.cu -- the C ABI of include/tp_block.h: argument checks, path
// choice (weight-streaming kernel for few tokens, persistent tiled kernel for
// many), TMA descriptor encoding and kernel launches.  See the header for the
// contract of each entry point.
#include "tp_block.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "attn_kernel.cuh"
#include "attn_prefill_kernel.cuh"
#include "colsum_kernel.cuh"
#include "diag_kernel.cuh"
#include "norm_kernel.cuh"
#include "pair_kernel.cuh"
#include "ptx.cuh"
#include "stream_kernel.cuh"
#include "tiled_kernel.cuh"

namespace {

using tpb::StreamParams;
using tpb::TiledParams;

// up to 128 tokens the weight-streaming kernel is faster than the tiled one on
// the 70B MLP (96 tokens: 0.240 vs 0.261 ms per block; 128: 0.257 vs 0.264):
// the tiled kernel's grid is N / 256 CTAs, 32 for an 8192-wide output
std::atomic<int> g_decode_max_tokens{128};
thread_local cudaError_t g_last_cuda_error = cudaSuccess;
thread_local const char* g_last_cuda_call = "";

// Returns true on success; otherwise remembers the error for tp_last_cuda_error().
inline bool cuda_ok(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return true;
  g_last_cuda_error = e;
  g_last_cuda_call = what;
  return false;
}
std::atomic<unsigned int> g_launch_options{TP_OPT_PDL};

constexpr int kMaxDevices = 64;
constexpr int kStreamMaxTokens = 128;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int max_smem = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Per-device facts and one-time kernel attributes.  Returns nullptr on failure.
using StreamKernel = void (*)(const CUtensorMap, const CUtensorMap, const tpb::StreamParams);

// Largest dynamic shared memory, and all of the unified L1 / shared storage
// as shared memory, for one instantiation of the streaming kernel.
bool stream_attrs(StreamKernel k, int smem) {
  return cuda_ok(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                 "cudaFuncSetAttribute") &&
         cuda_ok(cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                      cudaSharedmemCarveoutMaxShared),
                 "cudaFuncSetAttribute");
}

// The CTA-pair kernel's instantiations: (epilogue, A MN-major, B MN-major).
using PairKernel = void (*)(const CUtensorMap, const CUtensorMap, const tpb::TiledParams);
constexpr PairKernel kPairKernels[] = {
    tpb::pair_gemm_kernel<tpb::kEpiAct, false, false>,     // forward column-parallel
    tpb::pair_gemm_kernel<tpb::kEpiRowpar, false, false>,  // forward row-parallel + sum
    tpb::pair_gemm_kernel<tpb::kEpiDact, false, true>,     // dy W2, times act'(z)
    tpb::pair_gemm_kernel<tpb::kEpiRowpar, false, true>,   // sum_s dz_s W1_s
    tpb::pair_gemm_kernel<tpb::kEpiAct, true, true>,       // weight gradients (K = tokens)
};

PairKernel pair_kernel_for(int epi, bool a_mn, bool b_mn) {
  if (!a_mn && !b_mn) return epi == tpb::kEpiAct ? kPairKernels[0]
                             : epi == tpb::kEpiRowpar ? kPairKernels[1] : nullptr;
  if (!a_mn && b_mn) return epi == tpb::kEpiDact ? kPairKernels[2]
                            : epi == tpb::kEpiRowpar ? kPairKernels[3] : nullptr;
  if (a_mn && b_mn && epi == tpb::kEpiAct) return kPairKernels[4];
  return nullptr;
}

const DeviceInfo* device_info() {
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev), "cudaGetDevice") || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.ready) return &d;
  int sms = 0, smem = 0;
  if (!cuda_ok(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "cudaDeviceGetAttribute"))
    return nullptr;
  if (!cuda_ok(cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev),
               "cudaDeviceGetAttribute"))
    return nullptr;
  if (smem < tpb::kTiledSmemBytes) return nullptr;
  // all of the unified L1 / shared storage as shared memory, so three ~65 KB
  // streaming CTAs fit on an SM (the driver's default carveout allows two)
  if (!stream_attrs(tpb::stream_gemm_kernel<false, false>, smem) ||
      !stream_attrs(tpb::stream_gemm_kernel<true, false>, smem) ||
      !stream_attrs(tpb::stream_gemm_kernel<false, true>, smem) ||
      !stream_attrs(tpb::stream_gemm_kernel<true, true>, smem))
    return nullptr;
  if (!cuda_ok(cudaFuncSetAttribute(tpb::tiled_gemm_kernel<false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           tpb::kTiledSmemBytes), "cudaFuncSetAttribute"))
    return nullptr;
  if (!cuda_ok(cudaFuncSetAttribute(tpb::tiled_gemm_kernel<true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           tpb::kTiledSmemBytes), "cudaFuncSetAttribute"))
    return nullptr;
  for (PairKernel k : kPairKernels)
    if (!cuda_ok(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      tpb::kPairSmemBytes),
                 "cudaFuncSetAttribute"))
      return nullptr;
  if (!cuda_ok(cudaFuncSetAttribute(tpb::attn_prefill2_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    tpb::prefill2_smem_bytes()),
               "cudaFuncSetAttribute") ||
      !cuda_ok(cudaFuncSetAttribute(tpb::attn_prefill_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    tpb::prefill_smem_bytes()),
               "cudaFuncSetAttribute") ||
      !cuda_ok(cudaFuncSetAttribute(tpb::attn_prefill_kernel,
                                    cudaFuncAttributePreferredSharedMemoryCarveout,
                                    cudaSharedmemCarveoutMaxShared),
               "cudaFuncSetAttribute"))
    return nullptr;
  if (!cuda_ok(cudaFuncSetAttribute(tpb::attn_decode_kernel<16>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
               "cudaFuncSetAttribute") ||
      !cuda_ok(cudaFuncSetAttribute(tpb::attn_decode_kernel<32>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
               "cudaFuncSetAttribute"))
    return nullptr;
  d.sms = sms;
  d.max_smem = smem;
  d.ready = true;
  return &d;
}

// Row-major bf16 [rows, cols] viewed as 64-column x box_rows tiles with
// 128-byte swizzling; reads outside the tensor return zeros.
bool make_tmap(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
               uint32_t box_rows, uint32_t box_cols = 64, bool swizzle = true) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cuda_ok(cudaErrorSymbolNotFound, "cuTensorMapEncodeTiled lookup");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const bool ok = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  if (!ok) cuda_ok(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
  return ok;
}

// 3-D view of a row-major [rows, cols] bf16 matrix as (column within a
// 64-column block, row, block): a box {64, box_rows, blocks} lands in shared
// memory as `blocks` consecutive 128-byte-swizzled [box_rows][64] tiles.
bool make_tmap_blocks(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows, uint32_t blocks) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cuda_ok(cudaErrorSymbolNotFound, "cuTensorMapEncodeTiled lookup");
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {cols * 2, 128};
  cuuint32_t box[3] = {64, box_rows, blocks};
  cuuint32_t estr[3] = {1, 1, 1};
  const bool ok = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  if (!ok) cuda_ok(cudaErrorInvalidValue, "cuTensorMapEncodeTiled (blocks)");
  return ok;
}

// Same view of a row-major [rows, cols] 8-bit matrix with 64-byte swizzling:
// a box {64, box_rows, 1} lands as [box_rows][64] bytes, 16-byte chunk c of
// row r stored at chunk c ^ ((r / 2) % 4).
bool make_tmap_blocks_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                         uint32_t box_rows, uint32_t blocks) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cuda_ok(cudaErrorSymbolNotFound, "cuTensorMapEncodeTiled lookup");
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {cols, 64};
  cuuint32_t box[3] = {64, box_rows, blocks};
  cuuint32_t estr[3] = {1, 1, 1};
  const bool ok = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  if (!ok) cuda_ok(cudaErrorInvalidValue, "cuTensorMapEncodeTiled (8-bit blocks)");
  return ok;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool feat_ok(int n) { return n > 0 && n % 64 == 0; }
inline int next_pow2(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

// ------------------------------------------------------------------ launches

// Attributes shared by every launch: programmatic dependent launch (when
// enabled) lets a kernel's set-up overlap the tail of the previous kernel on
// the stream; the kernels wait for that kernel before touching activations or
// outputs.
int launch_attrs(cudaLaunchAttribute* attr, int n) {
  if (g_launch_options.load(std::memory_order_relaxed) & TP_OPT_PDL) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  return n;
}

inline int prefetch_weights() {
  const unsigned int o = g_launch_options.load(std::memory_order_relaxed);
  return ((o & TP_OPT_PDL) && (o & TP_OPT_STATIC_WEIGHTS)) ? 1 : 0;
}

struct StreamGeometry {
  int csize = 0, jsplit = 0, spc = 0;
};

// Cluster shape of the streaming kernel for an N x K weight in 128-row tiles:
// the largest cluster (1, 2, 4 or 8 CTAs along K) that keeps the grid within
// two CTAs per SM, so every CTA is resident from the start.  Either a shard is
// split over jsplit CTAs or a CTA owns spc whole shards (register running sum:
// t_pad <= 64).  csize == 0 when no shape fits.
StreamGeometry stream_geometry(int N, int kb_total, int shards, int t_pad, int sms) {
  const int n_tiles = (N + tpb::kStreamTileM - 1) / tpb::kStreamTileM;
  StreamGeometry fallback;
  const int kbs = kb_total / shards;
  for (int csize = 8; csize >= 1; csize >>= 1) {
    StreamGeometry g;
    g.csize = csize;
    if (csize >= shards) {
      if (csize % shards != 0) continue;
      g.jsplit = csize / shards;
      g.spc = 1;
      if (kbs / g.jsplit < 1) continue;
    } else {
      if (shards % csize != 0 || t_pad > tpb::kStreamRunCols) continue;
      g.jsplit = 1;
      g.spc = shards / csize;
    }
    if (n_tiles * csize <= 2 * sms) return g;
    fallback = g;
  }
  return fallback;
}

// Shared memory per SM (B200: 228 KB) and the 1 KB the hardware reserves per
// CTA: the least dynamic shared memory per CTA that lets at most `ctas` CTAs
// share an SM.
constexpr int kSmemPerSm = 228 * 1024;
constexpr int kSmemReservedPerCta = 1024;
inline int stream_smem_for_ctas(int ctas) {
  return kSmemPerSm / (ctas + 1) - kSmemReservedPerCta + 1;
}

// The sizes of a streaming launch (everything but pointers and options):
// geometry, ring depth, box size, shared memory.  Host arithmetic only; the
// device enters through max_smem.  TP_ERR_UNSUPPORTED if it does not fit.
tp_status plan_stream(int max_smem, const StreamGeometry& geo, bool w8, int T, int K, int N,
                      int shards, StreamParams& p, int& smem) {
  if (geo.csize == 0 || (w8 && geo.spc > 2)) return TP_ERR_UNSUPPORTED;
  p = StreamParams{};
  p.T = T;
  p.K = K;
  p.N = N;
  p.kb_total = K / tpb::kStreamTileK;
  p.t_pad = (T + 15) / 16 * 16;
  p.tmem_cols = next_pow2(p.t_pad < 32 ? 32 : p.t_pad);
  // one k-block of W (16 KB of bf16, or 8 KB of E4M3 codes) and of x
  p.stage_bytes = (w8 ? tpb::kStreamW8Bytes : tpb::kStreamTileM * tpb::kStreamTileK * 2) +
                  p.t_pad * tpb::kStreamTileK * 2;
  p.shards = shards;
  p.csize = geo.csize;
  p.jsplit = geo.jsplit;
  p.spc = geo.spc;
  // Ring depth: CTAs that stream >= 256 KB of weights get ~110 KB (two CTAs
  // per SM, deep ring); short streams get ~72 KB so three CTAs fit on an SM
  // and the next kernel's CTAs can start while this one drains.  At least 3
  // k-blocks in flight.  Two k-blocks per TMA box where every CTA's range is
  // even and three such stages fit the budget: a CTA's boxes complete one
  // after another, so larger boxes stream faster, but only a ring that still
  // holds three of them keeps enough in flight.
  {
    int lo, hi;
    tpb::stream_cta_range(p, 0, lo, hi);
    const long w_cta =
        static_cast<long>(hi - lo) * tpb::kStreamTileM * tpb::kStreamTileK * (w8 ? 1 : 2);
    const int budget = (w_cta >= 256 * 1024 ? 110 : 72) * 1024 -
                       tpb::stream_recv_bytes(p.T, p.csize);
    const int kb_bytes = p.stage_bytes;
    bool even = p.spc == 1;
    for (int r = 0; even && r < p.csize; ++r) {
      tpb::stream_cta_range(p, r, lo, hi);
      even = lo % 2 == 0 && hi % 2 == 0;
    }
    // 8-bit weights: two k-blocks per box (16 KB of codes per request) where
    // four such stages fit; each TMA request carries a fixed cost, and 8 KB
    // requests left the ring waiting on the copies
    p.kpb = (even && (w8 ? 8 * kb_bytes : 6 * kb_bytes) <= budget) ? 2 : 1;
    int kbs = budget / kb_bytes;
    kbs = kbs < 3 ? 3 : kbs;
    int stages = kbs / p.kpb;
    const int max_stages = w8 ? tpb::kStreamMaxStagesW8 : tpb::kStreamMaxStages;
    stages = stages < 2 ? 2 : (stages > max_stages ? max_stages : stages);
    p.stages = stages;
    p.stage_bytes = p.kpb * kb_bytes;
    // short streams: two more boxes into L2 before the grid wait (measured
    // best of 0-4 on the 4096 x 4096 decode step); long streams keep HBM busy
    // on their own
    p.l2_ahead = w_cta >= 256 * 1024 ? 0 : 2;
  }
  // large T: the receive buffer leaves room for two stages only
  while (p.stages > 2 &&
         tpb::stream_smem_bytes(p.stages, p.stage_bytes, p.T, p.csize, w8) > max_smem)
    --p.stages;
  smem = tpb::stream_smem_bytes(p.stages, p.stage_bytes, p.T, p.csize, w8);
  // The CTAs that share an SM must fit their TMEM allocations together: a CTA
  // whose allocation waited for a cluster peer on the same SM to finish would
  // wait for ever (the peer waits for it at the cluster barrier).  Shared
  // memory caps the CTAs per SM, so ask for enough of it.
  {
    const int alloc = tpb::stream_tmem_alloc_cols(p.tmem_cols, w8);
    const int max_ctas = 512 / alloc;
    const int floor_smem = stream_smem_for_ctas(max_ctas);
    if (smem < floor_smem) smem = floor_smem;
  }
  return smem > max_smem ? TP_ERR_UNSUPPORTED : TP_OK;
}

// Weight-streaming kernel.  `shards` groups the reduction for the row-parallel
// sum (1 for the column-parallel layer).  Requires T <= 128 and a geometry
// from stream_geometry().  With `w_scale` non-null the weight is 8-bit (E4M3
// bytes, [N, K]) and w_scale[n] scales row n; the geometry must then keep
// spc <= 2 (both shard regions are drained after all tiles are converted).
tp_status launch_stream(const DeviceInfo& dev, const StreamGeometry& geo, const tp_bf16* x,
                        const void* w, const float* w_scale, const tp_bf16* b, int T, int K,
                        int N, int shards, int act, tp_bf16* out, cudaStream_t stream) {
  const bool w8 = w_scale != nullptr;
  StreamParams p;
  int smem = 0;
  const tp_status planned = plan_stream(dev.max_smem, geo, w8, T, K, N, shards, p, smem);
  if (planned != TP_OK) return planned;
  p.act = act;
  p.prefetch_w = prefetch_weights();
  p.bias = b;
  p.w_scale = w_scale;
  p.out = out;
  const int n_tiles = (N + tpb::kStreamTileM - 1) / tpb::kStreamTileM;

  CUtensorMap tw, tx;
  const bool tw_ok =
      w8 ? make_tmap_blocks_u8(&tw, w, static_cast<uint64_t>(N), static_cast<uint64_t>(K),
                               static_cast<uint32_t>(tpb::kStreamTileM), static_cast<uint32_t>(p.kpb))
         : make_tmap_blocks(&tw, w, static_cast<uint64_t>(N), static_cast<uint64_t>(K),
                            static_cast<uint32_t>(tpb::kStreamTileM), static_cast<uint32_t>(p.kpb));
  if (!tw_ok) return TP_ERR_CUDA;
  if (!make_tmap_blocks(&tx, x, static_cast<uint64_t>(T), static_cast<uint64_t>(K),
                        static_cast<uint32_t>(p.t_pad), static_cast<uint32_t>(p.kpb)))
    return TP_ERR_CUDA;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(n_tiles), static_cast<unsigned>(p.csize), 1);
  cfg.blockDim = dim3(tpb::kStreamThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(p.csize);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = static_cast<unsigned>(launch_attrs(attr, 1));
  StreamKernel k = p.spc > 1 ? (w8 ? tpb::stream_gemm_kernel<true, true>
                                   : tpb::stream_gemm_kernel<true, false>)
                             : (w8 ? tpb::stream_gemm_kernel<false, true>
                                   : tpb::stream_gemm_kernel<false, false>);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, tw, tx, p);
  if (!cuda_ok(e, "launch stream_gemm_kernel")) return TP_ERR_CUDA;
  return TP_OK;
}

// One operand of the CTA-pair kernel as it is stored: K-major ([rows, K],
// K contiguous) or MN-major ([K, rows], the rows' index contiguous).
struct PairOperand {
  const tp_bf16* ptr;
  bool mn;
};

// Persistent CTA-pair kernel (256 x 256 tiles on two SMs): out[M, N] =
// epilogue(A[M, K] B[N, K]^T).  K need not be a multiple of 64: the loads
// past K read zeros.  `prefetch` allows B's first k-blocks to be requested
// before the preceding grid completes (B is a weight that no kernel writes).
tp_status launch_pair_ex(const DeviceInfo& dev, PairOperand a, PairOperand bop, const tp_bf16* bias,
                         int M, int K, int N, int segs, int epi, int act, tp_bf16* out,
                         const tp_bf16* aux, tp_bf16* out2, bool prefetch, cudaStream_t stream) {
  const PairKernel kernel = pair_kernel_for(epi, a.mn, bop.mn);
  if (kernel == nullptr) return TP_ERR_UNSUPPORTED;
  TiledParams p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.kb_total = (K + tpb::kPairBK - 1) / tpb::kPairBK;
  p.segs = segs;
  p.m_tiles = (M + tpb::kPairBM - 1) / tpb::kPairBM;
  p.n_tiles = (N + tpb::kPairBN - 1) / tpb::kPairBN;
  p.tiles = p.m_tiles * p.n_tiles;
  p.group_m = p.m_tiles < 8 ? p.m_tiles : 8;
  p.act = act;
  p.prefetch_w = prefetch ? prefetch_weights() : 0;
  p.bias = bias;
  p.out = out;
  p.aux = aux;
  p.out2 = out2;

  // K-major: box {64 K, 128 rows} of [rows, K]; MN-major: box {64 rows, 64 K} of [K, rows]
  CUtensorMap ta, tb;
  const bool ta_ok = a.mn ? make_tmap(&ta, a.ptr, static_cast<uint64_t>(K), static_cast<uint64_t>(M), 64)
                          : make_tmap(&ta, a.ptr, static_cast<uint64_t>(M), static_cast<uint64_t>(K), 128);
  if (!ta_ok) return TP_ERR_CUDA;
  const bool tb_ok = bop.mn ? make_tmap(&tb, bop.ptr, static_cast<uint64_t>(K), static_cast<uint64_t>(N), 64)
                            : make_tmap(&tb, bop.ptr, static_cast<uint64_t>(N), static_cast<uint64_t>(K), 128);
  if (!tb_ok) return TP_ERR_CUDA;

  const int pairs = p.tiles < dev.sms / 2 ? p.tiles : dev.sms / 2;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
  cfg.blockDim = dim3(tpb::kPairThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(tpb::kPairSmemBytes);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = static_cast<unsigned>(launch_attrs(attr, 1));
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, ta, tb, p);
  return cuda_ok(e, "launch pair_gemm_kernel") ? TP_OK : TP_ERR_CUDA;
}

// The forward pass's use of it: K-major activations and weights.
tp_status launch_pair(const DeviceInfo& dev, const tp_bf16* a, const tp_bf16* w,
                      const tp_bf16* b, int M, int K, int N, int segs, int act, tp_bf16* out,
                      cudaStream_t stream) {
  return launch_pair_ex(dev, PairOperand{a, false}, PairOperand{w, false}, b, M, K, N, segs,
                        segs > 1 ? tpb::kEpiRowpar : tpb::kEpiAct, act, out, nullptr, nullptr,
                        true, stream);
}

// Persistent tiled kernel.  segs = t accumulation segments in row-parallel
// mode (each from zero, summed in the epilogue), 1 otherwise.  More than 128
// rows go to the CTA-pair kernel.
tp_status launch_tiled(const DeviceInfo& dev, const tp_bf16* a, const tp_bf16* w,
                       const tp_bf16* b, int M, int K, int N, int segs, int act, tp_bf16* out,
                       cudaStream_t stream) {
  if (M > tpb::kTiledBM)
    return launch_pair(dev, a, w, b, M, K, N, segs, act, out, stream);
  TiledParams p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.kb_total = K / tpb::kTiledBK;
  p.segs = segs;
  p.m_tiles = (M + tpb::kTiledBM - 1) / tpb::kTiledBM;
  p.n_tiles = (N + tpb::kTiledBN - 1) / tpb::kTiledBN;
  p.tiles = p.m_tiles * p.n_tiles;
  p.group_m = p.m_tiles < 16 ? p.m_tiles : 16;
  p.act = act;
  p.prefetch_w = prefetch_weights();
  p.bias = b;
  p.out = out;

  CUtensorMap ta, tb;
  if (!make_tmap(&ta, a, static_cast<uint64_t>(M), static_cast<uint64_t>(K), tpb::kTiledBM))
    return TP_ERR_CUDA;
  if (!make_tmap(&tb, w, static_cast<uint64_t>(N), static_cast<uint64_t>(K), tpb::kTiledBN))
    return TP_ERR_CUDA;

  const int grid = p.tiles < dev.sms ? p.tiles : dev.sms;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(tpb::kTiledThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(tpb::kTiledSmemBytes);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  cfg.attrs = attr;
  cfg.numAttrs = static_cast<unsigned>(launch_attrs(attr, 0));
  cudaError_t e;
  if (segs > 1)
    e = cudaLaunchKernelEx(&cfg, tpb::tiled_gemm_kernel<true>, ta, tb, p);
  else
    e = cudaLaunchKernelEx(&cfg, tpb::tiled_gemm_kernel<false>, ta, tb, p);
  return cuda_ok(e, "launch tiled_gemm_kernel") ? TP_OK : TP_ERR_CUDA;
}

// Weight streaming for few tokens (decode), the tiled kernel otherwise.
bool use_stream(const DeviceInfo& dev, int T, int N) {
  (void)dev;
  (void)N;
  return T <= g_decode_max_tokens.load(std::memory_order_relaxed) && T <= kStreamMaxTokens;
}

tp_status run_colpar(const tp_bf16* x, const tp_bf16* w, const tp_bf16* b, int T, int K, int N,
                     int act, tp_bf16* out, cudaStream_t stream) {
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return TP_ERR_CUDA;
  if (use_stream(*dev, T, N)) {
    const int t_pad = (T + 15) / 16 * 16;
    const StreamGeometry g = stream_geometry(N, K / 64, 1, t_pad, dev->sms);
    if (g.csize > 0) return launch_stream(*dev, g, x, w, nullptr, b, T, K, N, 1, act, out, stream);
  }
  return launch_tiled(*dev, x, w, b, T, K, N, 1, act, out, stream);
}

tp_status run_rowpar(const tp_bf16* h, const tp_bf16* w, const tp_bf16* b, int T, int K, int N,
                     int t, tp_bf16* out, cudaStream_t stream) {
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return TP_ERR_CUDA;
  if (use_stream(*dev, T, N)) {
    const int t_pad = (T + 15) / 16 * 16;
    const StreamGeometry g = stream_geometry(N, K / 64, t, t_pad, dev->sms);
    if (g.csize > 0) return launch_stream(*dev, g, h, w, nullptr, b, T, K, N, t, 0, out, stream);
  }
  return launch_tiled(*dev, h, w, b, T, K, N, t, 0, out, stream);
}

// Geometry of an 8-bit streaming launch: csize == 0 when the split is not
// supported (no cluster shape, or more than two shards per CTA).
StreamGeometry w8_geometry(const DeviceInfo& dev, int T, int K, int N, int shards) {
  const int t_pad = (T + 15) / 16 * 16;
  StreamGeometry g = stream_geometry(N, K / 64, shards, t_pad, dev.sms);
  if (g.spc > 2) g.csize = 0;
  return g;
}

// 8-bit weights: the streaming kernel only (T <= kStreamMaxTokens).
tp_status run_linear_w8(const tp_bf16* x, const uint8_t* w8, const float* w_scale,
                        const tp_bf16* b, int T, int K, int N, int shards, int act, tp_bf16* out,
                        cudaStream_t stream) {
  if (T > kStreamMaxTokens) return TP_ERR_UNSUPPORTED;
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return TP_ERR_CUDA;
  const StreamGeometry g = w8_geometry(*dev, T, K, N, shards);
  if (g.csize == 0) return TP_ERR_UNSUPPORTED;
  return launch_stream(*dev, g, x, w8, w_scale, b, T, K, N, shards, act, out, stream);
}

// ------------------------------------------------------------------ attention core (decode)

// The launch of the decode attention core for a shape; a function of the shape
// only (not of the device), so the chunking and therefore the order of the
// sums are the same on every GPU.  TP_ERR_UNSUPPORTED if G is not 1, 2, 4, 8
// or 16.
constexpr int kAttnTargetCtas = 296;  // two waves' worth of CTAs on 148 SMs

tp_status plan_attn(int T, int past, int nq, int nkv, tpb::AttnParams& p, int& groups,
                    size_t& part_o_bytes, size_t& part_ml_bytes) {
  const int G = nq / nkv;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return TP_ERR_UNSUPPORTED;
  p = tpb::AttnParams{};
  p.T = T;
  p.past = past;
  p.L = past + T;
  p.nq = nq;
  p.nkv = nkv;
  p.G = G;
  // At most 32 query rows per CTA: the scores of a whole chunk (up to 8 key
  // blocks) then fit in TMEM, so the chunk maximum is known before any P V
  // product and no accumulator is rescaled.  More tokens form token groups
  // (grid z), each of which reads the chunk's keys and values again.
  const int tq_step = G >= 16 ? 1 : 16 / G;   // tokens that make 16 query rows
  const int tq_max = 32 / G;
  if (T <= tq_max) {
    p.Tq = (T + tq_step - 1) / tq_step * tq_step;
    groups = 1;
  } else {
    p.Tq = tq_max;
    groups = (T + tq_max - 1) / tq_max;
  }
  p.n_pad = p.Tq * G;
  p.nblk = (p.L + tpb::kAttnBlockKeys - 1) / tpb::kAttnBlockKeys;
  // chunks per key-value head so the grid is about kAttnTargetCtas CTAs (two
  // per SM, one wave); every chunk streams nb blocks with a running softmax
  const int per_chunk = nkv * groups;  // CTAs per chunk index
  int chunks = (kAttnTargetCtas + per_chunk - 1) / per_chunk;
  chunks = chunks < 1 ? 1 : (chunks > p.nblk ? p.nblk : chunks);
  p.nb = (p.nblk + chunks - 1) / chunks;
  p.chunks = (p.nblk + p.nb - 1) / p.nb;
  // a 2-deep ring of 32 KB stages: in the load order K_0, K_1, V_0, K_2,
  // V_1, ... the two MMA issuers (scores, P V) then each take their stage's
  // fills in order (see attn_decode_kernel); TMEM: two score slots and two
  // accumulators
  p.stages = 2;
  p.tmem_cols = next_pow2(4 * p.n_pad < 32 ? 32 : 4 * p.n_pad);  // 2 score slots, 2 O's
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(tpb::kAttnHeadDim));
  const size_t rows = static_cast<size_t>(groups) * nkv * p.chunks * p.n_pad;
  part_o_bytes = (rows * tpb::kAttnHeadDim * 4 + 255) / 256 * 256;
  part_ml_bytes = (rows * 2 * 4 + 255) / 256 * 256;
  return TP_OK;
}

// 3-D view {d, rows, outer} of a bf16 tensor whose rows are d = 128 elements
// apart and whose outer index is `outer_stride` elements apart; a box
// {64, box_rows, box_outer} lands as box_outer * box_rows 128-byte rows with
// 128-byte swizzling.  Reads outside [0, rows) return zeros.
bool make_tmap_rows3(CUtensorMap* map, const void* base, uint64_t rows, uint64_t outer,
                     uint64_t row_stride, uint64_t outer_stride, uint32_t box_rows,
                     uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cuda_ok(cudaErrorSymbolNotFound, "cuTensorMapEncodeTiled lookup");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(tpb::kAttnHeadDim), rows, outer};
  cuuint64_t strides[2] = {row_stride * 2, outer_stride * 2};
  cuuint32_t box[3] = {64, box_rows, box_outer};
  cuuint32_t estr[3] = {1, 1, 1};
  const bool ok = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  if (!ok) cuda_ok(cudaErrorInvalidValue, "cuTensorMapEncodeTiled (rows3)");
  return ok;
}

// ------------------------------------------------------------------ checks

tp_status check_linear(const void* x, const void* w, const void* b, const void* out, int T, int K,
                       int N, int act) {
  if (x == nullptr || w == nullptr || out == nullptr) return TP_ERR_NULL;
  if (!aligned16(x) || !aligned16(w) || !aligned16(out) || (b != nullptr && !aligned16(b)))
    return TP_ERR_ALIGN;
  if (T < 1 || !feat_ok(K) || !feat_ok(N)) return TP_ERR_SHAPE;
  if (act != TP_ACT_NONE && act != TP_ACT_GELU_TANH) return TP_ERR_UNSUPPORTED;
  return TP_OK;
}

}  // namespace

extern "C" {

tp_status tp_colpar_gemm_gelu(const tp_bf16* x, const tp_bf16* w, const tp_bf16* b, int T, int K,
                              int N, int tp_degree, int act, tp_bf16* out, tp_stream_t stream) {
  tp_status s = check_linear(x, w, b, out, T, K, N, act);
  if (s != TP_OK) return s;
  if (tp_degree < 1 || N % tp_degree != 0) return TP_ERR_TP_DEGREE;
  return run_colpar(x, w, b, T, K, N, act, out, reinterpret_cast<cudaStream_t>(stream));
}

tp_status tp_rowpar_gemm_reduce(const tp_bf16* h, const tp_bf16* w, const tp_bf16* b, int T, int K,
                                int N, int tp_degree, tp_bf16* out, tp_stream_t stream) {
  tp_status s = check_linear(h, w, b, out, T, K, N, TP_ACT_NONE);
  if (s != TP_OK) return s;
  if (tp_degree < 1 || K % tp_degree != 0 || (K / tp_degree) % 64 != 0) return TP_ERR_TP_DEGREE;
  return run_rowpar(h, w, b, T, K, N, tp_degree, out, reinterpret_cast<cudaStream_t>(stream));
}

size_t tp_mlp_workspace_bytes(int T, int F) {
  if (T < 1 || F < 1) return 0;
  const size_t raw = static_cast<size_t>(T) * static_cast<size_t>(F) * 2u;
  return (raw + 255u) / 256u * 256u;
}

tp_status tp_mlp_forward(const tp_bf16* x, const tp_bf16* w1, const tp_bf16* b1,
                         const tp_bf16* w2, const tp_bf16* b2, int T, int H, int F, int tp_degree,
                         int act, tp_bf16* out, void* workspace, size_t workspace_bytes,
                         tp_stream_t stream) {
  if (x == nullptr || w1 == nullptr || w2 == nullptr || out == nullptr) return TP_ERR_NULL;
  if (!aligned16(x) || !aligned16(w1) || !aligned16(w2) || !aligned16(out) ||
      (b1 != nullptr && !aligned16(b1)) || (b2 != nullptr && !aligned16(b2)))
    return TP_ERR_ALIGN;
  if (T < 1 || !feat_ok(H) || !feat_ok(F)) return TP_ERR_SHAPE;
  if (act != TP_ACT_NONE && act != TP_ACT_GELU_TANH) return TP_ERR_UNSUPPORTED;
  if (tp_degree < 1 || F % tp_degree != 0 || (F / tp_degree) % 64 != 0) return TP_ERR_TP_DEGREE;
  if (workspace == nullptr || workspace_bytes < tp_mlp_workspace_bytes(T, F))
    return TP_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TP_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  tp_bf16* h = static_cast<tp_bf16*>(workspace);
  tp_status s = run_colpar(x, w1, b1, T, H, F, act, h, st);
  if (s != TP_OK) return s;
  return run_rowpar(h, w2, b2, T, F, H, tp_degree, out, st);
}

tp_status tp_attn_proj_forward(const tp_bf16* x, const tp_bf16* w_qkv, const tp_bf16* b_qkv,
                               const tp_bf16* ctx, const tp_bf16* w_o, const tp_bf16* b_o, int T,
                               int H, int n_q_heads, int n_kv_heads, int head_dim, int tp_degree,
                               tp_bf16* qkv_out, tp_bf16* out, tp_stream_t stream) {
  if (x == nullptr || w_qkv == nullptr || ctx == nullptr || w_o == nullptr ||
      qkv_out == nullptr || out == nullptr)
    return TP_ERR_NULL;
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(ctx) || !aligned16(w_o) ||
      !aligned16(qkv_out) || !aligned16(out) || (b_qkv != nullptr && !aligned16(b_qkv)) ||
      (b_o != nullptr && !aligned16(b_o)))
    return TP_ERR_ALIGN;
  if (T < 1 || !feat_ok(H) || n_q_heads < 1 || n_kv_heads < 1 || head_dim < 1)
    return TP_ERR_SHAPE;
  const long long nqkv = static_cast<long long>(n_q_heads + 2 * n_kv_heads) * head_dim;
  const long long nctx = static_cast<long long>(n_q_heads) * head_dim;
  if (nqkv > (1ll << 30) || nqkv % 64 != 0 || nctx % 64 != 0) return TP_ERR_SHAPE;
  if (tp_degree < 1 || n_q_heads % tp_degree != 0 || n_kv_heads % tp_degree != 0 ||
      ((n_q_heads / tp_degree) * head_dim) % 64 != 0)
    return TP_ERR_TP_DEGREE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  tp_status s = run_colpar(x, w_qkv, b_qkv, T, H, static_cast<int>(nqkv), TP_ACT_NONE, qkv_out, st);
  if (s != TP_OK) return s;
  return run_rowpar(ctx, w_o, b_o, T, static_cast<int>(nctx), H, tp_degree, out, st);
}

size_t tp_mlp_backward_workspace_bytes(int T, int F) {
  if (T < 1 || F < 1) return 0;
  return 3u * tp_mlp_workspace_bytes(T, F);
}

tp_status tp_mlp_backward(const tp_bf16* x, const tp_bf16* w1, const tp_bf16* b1,
                          const tp_bf16* w2, const tp_bf16* dy, int T, int H, int F,
                          int tp_degree, int act, tp_bf16* dx, tp_bf16* dw1, tp_bf16* db1,
                          tp_bf16* dw2, tp_bf16* db2, void* workspace, size_t workspace_bytes,
                          tp_stream_t stream) {
  if (x == nullptr || w1 == nullptr || w2 == nullptr || dy == nullptr || dx == nullptr ||
      dw1 == nullptr || dw2 == nullptr)
    return TP_ERR_NULL;
  if (!aligned16(x) || !aligned16(w1) || !aligned16(w2) || !aligned16(dy) || !aligned16(dx) ||
      !aligned16(dw1) || !aligned16(dw2) || (b1 != nullptr && !aligned16(b1)) ||
      (db1 != nullptr && !aligned16(db1)) || (db2 != nullptr && !aligned16(db2)))
    return TP_ERR_ALIGN;
  if (T < 1 || !feat_ok(H) || !feat_ok(F)) return TP_ERR_SHAPE;
  if (act != TP_ACT_NONE && act != TP_ACT_GELU_TANH) return TP_ERR_UNSUPPORTED;
  if (tp_degree < 1 || F % tp_degree != 0 || (F / tp_degree) % 64 != 0) return TP_ERR_TP_DEGREE;
  if (workspace == nullptr || workspace_bytes < tp_mlp_backward_workspace_bytes(T, F))
    return TP_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TP_ERR_ALIGN;
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return TP_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t slot = tp_mlp_workspace_bytes(T, F);
  tp_bf16* z = static_cast<tp_bf16*>(workspace);
  tp_bf16* dz = reinterpret_cast<tp_bf16*>(static_cast<uint8_t*>(workspace) + slot);
  tp_bf16* h = reinterpret_cast<tp_bf16*>(static_cast<uint8_t*>(workspace) + 2 * slot);
  // z = x W1^T + b1, the forward pre-activation (column-parallel, no activation)
  tp_status s = run_colpar(x, w1, b1, T, H, F, TP_ACT_NONE, z, st);
  if (s != TP_OK) return s;
  // dz = (dy W2) * act'(z) and h = act(z); W2 [H, F] is read with F as N (MN-major).
  // Shard s's columns F_s need nothing from other shards: dy reaches every shard whole.
  s = launch_pair_ex(*dev, PairOperand{dy, false}, PairOperand{w2, true}, nullptr, T, H, F, 1,
                     tpb::kEpiDact, act, dz, z, h, true, st);
  if (s != TP_OK) return s;
  // dx = sum_s dz[:, F_s] W1[F_s, :]: the backward all-reduce, each shard's
  // partial from zero, summed in ascending shard order in the epilogue
  s = launch_pair_ex(*dev, PairOperand{dz, false}, PairOperand{w1, true}, nullptr, T, F, H,
                     tp_degree, tpb::kEpiRowpar, TP_ACT_NONE, dx, nullptr, nullptr, true, st);
  if (s != TP_OK) return s;
  // weight gradients stay on their shards: dW1 = dz^T x [F, H], dW2 = dy^T h [H, F],
  // contractions over the tokens (both operands read MN-major)
  s = launch_pair_ex(*dev, PairOperand{dz, true}, PairOperand{x, true}, nullptr, F, T, H, 1,
                     tpb::kEpiAct, TP_ACT_NONE, dw1, nullptr, nullptr, false, st);
  if (s != TP_OK) return s;
  s = launch_pair_ex(*dev, PairOperand{dy, true}, PairOperand{h, true}, nullptr, H, T, F, 1,
                     tpb::kEpiAct, TP_ACT_NONE, dw2, nullptr, nullptr, false, st);
  if (s != TP_OK) return s;
  if (db1 != nullptr) {
    tpb::colsum_kernel<<<(F + 63) / 64, tpb::kColsumWarps * 32, 0, st>>>(dz, T, F, db1);
    if (!cuda_ok(cudaGetLastError(), "launch colsum_kernel")) return TP_ERR_CUDA;
  }
  if (db2 != nullptr) {
    tpb::colsum_kernel<<<(H + 63) / 64, tpb::kColsumWarps * 32, 0, st>>>(dy, T, H, db2);
    if (!cuda_ok(cudaGetLastError(), "launch colsum_kernel")) return TP_ERR_CUDA;
  }
  return TP_OK;
}

size_t tp_attn_decode_workspace_bytes(int T, int past, int n_q_heads, int n_kv_heads,
                                      int head_dim) {
  if (T < 1 || past < 0 || n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads != 0 ||
      head_dim != tpb::kAttnHeadDim)
    return 0;
  tpb::AttnParams p;
  int groups = 0;
  size_t po = 0, pml = 0;
  if (plan_attn(T, past, n_q_heads, n_kv_heads, p, groups, po, pml) != TP_OK) return 0;
  return po + pml;
}

tp_status tp_attn_decode(const tp_bf16* qkv, tp_bf16* k_cache, tp_bf16* v_cache, int T, int past,
                         int max_len, int n_q_heads, int n_kv_heads, int head_dim, int tp_degree,
                         tp_bf16* ctx, void* workspace, size_t workspace_bytes,
                         tp_stream_t stream) {
  if (qkv == nullptr || k_cache == nullptr || v_cache == nullptr || ctx == nullptr)
    return TP_ERR_NULL;
  if (!aligned16(qkv) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(ctx))
    return TP_ERR_ALIGN;
  if (T < 1 || past < 0 || n_q_heads < 1 || n_kv_heads < 1 || head_dim < 1 ||
      n_q_heads % n_kv_heads != 0 || max_len < 1 || static_cast<long long>(past) + T > max_len ||
      static_cast<long long>(n_kv_heads) * max_len * head_dim > (1ll << 40))
    return TP_ERR_SHAPE;
  if (head_dim != tpb::kAttnHeadDim) return TP_ERR_UNSUPPORTED;
  if (tp_degree < 1 || n_q_heads % tp_degree != 0 || n_kv_heads % tp_degree != 0)
    return TP_ERR_TP_DEGREE;
  tpb::AttnParams p;
  int groups = 0;
  size_t po = 0, pml = 0;
  const tp_status planned = plan_attn(T, past, n_q_heads, n_kv_heads, p, groups, po, pml);
  if (planned != TP_OK) return planned;
  if (workspace == nullptr || workspace_bytes < po + pml) return TP_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TP_ERR_ALIGN;
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return TP_ERR_CUDA;
  const int smem = tpb::attn_smem_bytes(p.stages, p.n_pad);
  if (smem > dev->max_smem) return TP_ERR_UNSUPPORTED;
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + po);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int nqkv = (n_q_heads + 2 * n_kv_heads) * head_dim;

  // Q: {d, heads, tokens}; K, V: {d, keys 0 .. L - 1, key-value heads}
  CUtensorMap tq, tk, tv;
  if (!make_tmap_rows3(&tq, qkv, static_cast<uint64_t>(n_q_heads), static_cast<uint64_t>(T),
                       static_cast<uint64_t>(head_dim), static_cast<uint64_t>(nqkv),
                       static_cast<uint32_t>(p.G), static_cast<uint32_t>(p.Tq)) ||
      !make_tmap_rows3(&tk, k_cache, static_cast<uint64_t>(p.L), static_cast<uint64_t>(n_kv_heads),
                       static_cast<uint64_t>(head_dim),
                       static_cast<uint64_t>(max_len) * head_dim, tpb::kAttnBlockKeys, 1) ||
      !make_tmap_rows3(&tv, v_cache, static_cast<uint64_t>(p.L), static_cast<uint64_t>(n_kv_heads),
                       static_cast<uint64_t>(head_dim),
                       static_cast<uint64_t>(max_len) * head_dim, tpb::kAttnBlockKeys, 1))
    return TP_ERR_CUDA;

  p.qkv = qkv;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.max_len = max_len;
  cudaLaunchAttribute attr[1];
  const int nattr = launch_attrs(attr, 0);
  // 1. chunk partials: grid (chunks, key-value heads, token groups); the CTAs
  //    holding rows [past, past + T) write the new keys and values first
  {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(p.chunks), static_cast<unsigned>(n_kv_heads),
                       static_cast<unsigned>(groups));
    cfg.blockDim = dim3(tpb::kAttnThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = static_cast<unsigned>(nattr);
    const cudaError_t e = p.n_pad <= 16
                              ? cudaLaunchKernelEx(&cfg, tpb::attn_decode_kernel<16>, tq, tk, tv, p)
                              : cudaLaunchKernelEx(&cfg, tpb::attn_decode_kernel<32>, tq, tk, tv, p);
    if (!cuda_ok(e, "launch attn_decode_kernel")) return TP_ERR_CUDA;
  }
  // 2. merge the chunks of every (token, query head): one CTA each
  {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(T * n_q_heads), 1, 1);
    cfg.blockDim = dim3(tpb::kCombineWarps * 32, 1, 1);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = static_cast<unsigned>(nattr);
    if (!cuda_ok(cudaLaunchKernelEx(&cfg, tpb::attn_combine_kernel,
                                    static_cast<const float*>(p.part_o),
                                    static_cast<const float*>(p.part_ml), T, n_q_heads,
                                    n_kv_heads, p.G, p.Tq, p.n_pad, p.chunks, ctx),
                 "launch attn_combine_kernel"))
      return TP_ERR_CUDA;
  }
  return TP_OK;
}

tp_status tp_attn_prefill(const tp_bf16* qkv, tp_bf16* k_cache, tp_bf16* v_cache, int T,
                          int past, int max_len, int n_q_heads, int n_kv_heads, int head_dim,
                          int tp_degree, tp_bf16* ctx, tp_stream_t stream) {
  if (qkv == nullptr || k_cache == nullptr || v_cache == nullptr || ctx == nullptr)
    return TP_ERR_NULL;
  if (!aligned16(qkv) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(ctx))
    return TP_ERR_ALIGN;
  if (T < 1 || past < 0 || n_q_heads < 1 || n_kv_heads < 1 || head_dim < 1 ||
      n_q_heads % n_kv_heads != 0 || max_len < 1 || static_cast<long long>(past) + T > max_len ||
      static_cast<long long>(n_kv_heads) * max_len * head_dim > (1ll << 40) ||
      (T + tpb::kPrefillRows - 1) / tpb::kPrefillRows > 65535)
    return TP_ERR_SHAPE;
  if (head_dim != tpb::kAttnHeadDim) return TP_ERR_UNSUPPORTED;
  if (tp_degree < 1 || n_q_heads % tp_degree != 0 || n_kv_heads % tp_degree != 0)
    return TP_ERR_TP_DEGREE;
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return TP_ERR_CUDA;
  // an even number of query heads per key-value head: two heads per CTA
  const bool pairs = (n_q_heads / n_kv_heads) % 2 == 0;
  if ((pairs ? tpb::prefill2_smem_bytes() : tpb::prefill_smem_bytes()) > dev->max_smem)
    return TP_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int nqkv = (n_q_heads + 2 * n_kv_heads) * head_dim;
  tpb::PrefillParams p{};
  p.T = T;
  p.past = past;
  p.L = past + T;
  p.nq = n_q_heads;
  p.G = n_q_heads / n_kv_heads;
  p.ntiles = (T + tpb::kPrefillRows - 1) / tpb::kPrefillRows;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(tpb::kAttnHeadDim));
  p.ctx = ctx;
  // Q: qkv as [T, nqkv] in 64-column x 128-row boxes; K, V: {d, keys 0 .. L - 1,
  // key-value heads} in 128-key boxes (keys at or past L read as zeros)
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, qkv, static_cast<uint64_t>(T), static_cast<uint64_t>(nqkv),
                 tpb::kPrefillRows) ||
      !make_tmap_rows3(&tk, k_cache, static_cast<uint64_t>(p.L), static_cast<uint64_t>(n_kv_heads),
                       static_cast<uint64_t>(head_dim),
                       static_cast<uint64_t>(max_len) * head_dim, tpb::kAttnBlockKeys, 1) ||
      !make_tmap_rows3(&tv, v_cache, static_cast<uint64_t>(p.L), static_cast<uint64_t>(n_kv_heads),
                       static_cast<uint64_t>(head_dim),
                       static_cast<uint64_t>(max_len) * head_dim, tpb::kAttnBlockKeys, 1))
    return TP_ERR_CUDA;
  cudaLaunchAttribute attr[1];
  const int nattr = launch_attrs(attr, 0);
  // 1. the new keys and values into the caches
  {
    const long long pieces = static_cast<long long>(T) * n_kv_heads * 2 * (head_dim / 8);
    long long blocks = (pieces + 255) / 256;
    if (blocks > 16ll * dev->sms) blocks = 16ll * dev->sms;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = static_cast<unsigned>(nattr);
    if (!cuda_ok(cudaLaunchKernelEx(&cfg, tpb::kv_append_kernel, static_cast<const uint16_t*>(qkv),
                                    T, past, n_q_heads, n_kv_heads, max_len,
                                    static_cast<uint16_t*>(k_cache),
                                    static_cast<uint16_t*>(v_cache)),
                 "launch kv_append_kernel"))
      return TP_ERR_CUDA;
  }
  // 2. the attention kernel: heads fastest, longest tiles first
  {
    cudaLaunchConfig_t cfg{};
    // two heads per CTA: a persistent grid, one CTA per SM, over (head pair,
    // tile) items; one head per CTA: CTA (head, tile)
    const long long items = static_cast<long long>(n_q_heads / 2) * p.ntiles;
    cfg.gridDim = pairs ? dim3(static_cast<unsigned>(items < dev->sms ? items : dev->sms), 1, 1)
                        : dim3(static_cast<unsigned>(n_q_heads), static_cast<unsigned>(p.ntiles), 1);
    cfg.blockDim = dim3(pairs ? tpb::kPrefill2Threads : tpb::kPrefillThreads, 1, 1);
    cfg.dynamicSmemBytes =
        static_cast<size_t>(pairs ? tpb::prefill2_smem_bytes() : tpb::prefill_smem_bytes());
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = static_cast<unsigned>(nattr);
    const cudaError_t e = pairs ? cudaLaunchKernelEx(&cfg, tpb::attn_prefill2_kernel, tq, tk, tv, p)
                                : cudaLaunchKernelEx(&cfg, tpb::attn_prefill_kernel, tq, tk, tv, p);
    if (!cuda_ok(e, "launch attn_prefill_kernel")) return TP_ERR_CUDA;
  }
  return TP_OK;
}

tp_status tp_sp_add_rmsnorm(const tp_bf16* y, const tp_bf16* residual, const tp_bf16* gamma,
                            int T, int H, int tp_degree, float eps, tp_bf16* r_out,
                            tp_bf16* n_out, tp_stream_t stream) {
  if (y == nullptr || residual == nullptr || gamma == nullptr || r_out == nullptr ||
      n_out == nullptr)
    return TP_ERR_NULL;
  if (!aligned16(y) || !aligned16(residual) || !aligned16(gamma) || !aligned16(r_out) ||
      !aligned16(n_out))
    return TP_ERR_ALIGN;
  if (T < 1 || !feat_ok(H) || !(eps >= 0.0f)) return TP_ERR_SHAPE;
  if (tp_degree < 1 || T % tp_degree != 0) return TP_ERR_TP_DEGREE;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(T), 1, 1);  // token shard s: rows [s T/t, (s+1) T/t)
  cfg.blockDim = dim3(tpb::kNormThreads, 1, 1);
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cfg.attrs = attr;
  cfg.numAttrs = static_cast<unsigned>(launch_attrs(attr, 0));
  const bool in_regs = H <= tpb::kNormThreads * tpb::kNormVecPerThread * 8;
  const cudaError_t e =
      in_regs ? cudaLaunchKernelEx(&cfg, tpb::add_rmsnorm_kernel<true>, y, residual, gamma, H, eps,
                                   r_out, n_out)
              : cudaLaunchKernelEx(&cfg, tpb::add_rmsnorm_kernel<false>, y, residual, gamma, H, eps,
                                   r_out, n_out);
  return cuda_ok(e, "launch add_rmsnorm_kernel") ? TP_OK : TP_ERR_CUDA;
}

tp_status tp_colpar_gemm_gelu_w8(const tp_bf16* x, const uint8_t* w8, const float* w_scale,
                                 const tp_bf16* b, int T, int K, int N, int tp_degree, int act,
                                 tp_bf16* out, tp_stream_t stream) {
  tp_status s = check_linear(x, w8, b, out, T, K, N, act);
  if (s != TP_OK) return s;
  if (w_scale == nullptr) return TP_ERR_NULL;
  if (!aligned16(w_scale)) return TP_ERR_ALIGN;
  if (tp_degree < 1 || N % tp_degree != 0) return TP_ERR_TP_DEGREE;
  return run_linear_w8(x, w8, w_scale, b, T, K, N, 1, act, out,
                       reinterpret_cast<cudaStream_t>(stream));
}

tp_status tp_rowpar_gemm_reduce_w8(const tp_bf16* h, const uint8_t* w8, const float* w_scale,
                                   const tp_bf16* b, int T, int K, int N, int tp_degree,
                                   tp_bf16* out, tp_stream_t stream) {
  tp_status s = check_linear(h, w8, b, out, T, K, N, TP_ACT_NONE);
  if (s != TP_OK) return s;
  if (w_scale == nullptr) return TP_ERR_NULL;
  if (!aligned16(w_scale)) return TP_ERR_ALIGN;
  if (tp_degree < 1 || K % tp_degree != 0 || (K / tp_degree) % 64 != 0) return TP_ERR_TP_DEGREE;
  return run_linear_w8(h, w8, w_scale, b, T, K, N, tp_degree, TP_ACT_NONE, out,
                       reinterpret_cast<cudaStream_t>(stream));
}

tp_status tp_mlp_forward_w8(const tp_bf16* x, const uint8_t* w1, const float* s1,
                            const tp_bf16* b1, const uint8_t* w2, const float* s2,
                            const tp_bf16* b2, int T, int H, int F, int tp_degree, int act,
                            tp_bf16* out, void* workspace, size_t workspace_bytes,
                            tp_stream_t stream) {
  if (x == nullptr || w1 == nullptr || s1 == nullptr || w2 == nullptr || s2 == nullptr ||
      out == nullptr)
    return TP_ERR_NULL;
  if (!aligned16(x) || !aligned16(w1) || !aligned16(s1) || !aligned16(w2) || !aligned16(s2) ||
      !aligned16(out) || (b1 != nullptr && !aligned16(b1)) || (b2 != nullptr && !aligned16(b2)))
    return TP_ERR_ALIGN;
  if (T < 1 || !feat_ok(H) || !feat_ok(F)) return TP_ERR_SHAPE;
  if (act != TP_ACT_NONE && act != TP_ACT_GELU_TANH) return TP_ERR_UNSUPPORTED;
  if (tp_degree < 1 || F % tp_degree != 0 || (F / tp_degree) % 64 != 0) return TP_ERR_TP_DEGREE;
  if (T > kStreamMaxTokens) return TP_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < tp_mlp_workspace_bytes(T, F))
    return TP_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TP_ERR_ALIGN;
  // both layers' splits are checked before the first launch, so an
  // unsupported split leaves the workspace untouched
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return TP_ERR_CUDA;
  if (w8_geometry(*dev, T, H, F, 1).csize == 0 || w8_geometry(*dev, T, F, H, tp_degree).csize == 0)
    return TP_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  tp_bf16* h = static_cast<tp_bf16*>(workspace);
  tp_status s = run_linear_w8(x, w1, s1, b1, T, H, F, 1, act, h, st);
  if (s != TP_OK) return s;
  return run_linear_w8(h, w2, s2, b2, T, F, H, tp_degree, TP_ACT_NONE, out, st);
}

tp_status tp_stream_plan(int T, int K, int N, int row_shards, int w8, int sms, int max_smem,
                         tp_stream_plan_t* plan) {
  if (plan == nullptr) return TP_ERR_NULL;
  if (T < 1 || !feat_ok(K) || !feat_ok(N) || sms < 1 || max_smem < 1) return TP_ERR_SHAPE;
  if (row_shards < 1 || K % row_shards != 0 || (K / row_shards) % 64 != 0)
    return TP_ERR_TP_DEGREE;
  if (T > kStreamMaxTokens) return TP_ERR_UNSUPPORTED;
  const int t_pad = (T + 15) / 16 * 16;
  const StreamGeometry g = stream_geometry(N, K / 64, row_shards, t_pad, sms);
  StreamParams p;
  int smem = 0;
  const tp_status s = plan_stream(max_smem, g, w8 != 0, T, K, N, row_shards, p, smem);
  if (s != TP_OK) return s;
  plan->grid_x = (N + tpb::kStreamTileM - 1) / tpb::kStreamTileM;
  plan->cluster = p.csize;
  plan->jsplit = p.jsplit;
  plan->shards_per_cta = p.spc;
  plan->stages = p.stages;
  plan->kblocks_per_box = p.kpb;
  plan->stage_bytes = p.stage_bytes;
  plan->smem_bytes = smem;
  plan->l2_ahead = p.l2_ahead;
  return TP_OK;
}

const char* tp_status_string(tp_status status) {
  switch (status) {
    case TP_OK: return "ok";
    case TP_ERR_NULL: return "a required pointer is NULL";
    case TP_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case TP_ERR_SHAPE: return "a size is out of range (T >= 1, feature sizes positive multiples of 64)";
    case TP_ERR_TP_DEGREE: return "tp_degree does not divide the dimension or head counts it splits";
    case TP_ERR_WORKSPACE: return "workspace missing or too small";
    case TP_ERR_UNSUPPORTED: return "unsupported option";
    case TP_ERR_CUDA: return "a CUDA call failed";
    case TP_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait ran out";
  }
  return "unknown status";
}

const char* tp_last_cuda_error(void) {
  static thread_local char buf[256];
  if (g_last_cuda_error == cudaSuccess) return "no CUDA error recorded";
  snprintf(buf, sizeof(buf), "%s: %s (%d)", g_last_cuda_call, cudaGetErrorString(g_last_cuda_error),
           static_cast<int>(g_last_cuda_error));
  return buf;
}

tp_status tp_device_error_check(void) {
  if (!cuda_ok(cudaDeviceSynchronize(), "cudaDeviceSynchronize")) return TP_ERR_CUDA;
  unsigned int v = 0;
  if (!cuda_ok(cudaMemcpyFromSymbol(&v, tpb::g_tp_device_error, sizeof(v)), "cudaMemcpyFromSymbol"))
    return TP_ERR_CUDA;
  if (v != 0u) {
    const unsigned int zero = 0u;
    if (!cuda_ok(cudaMemcpyToSymbol(tpb::g_tp_device_error, &zero, sizeof(zero)),
                 "cudaMemcpyToSymbol"))
      return TP_ERR_CUDA;
    return TP_ERR_DEVICE_TIMEOUT;
  }
  return TP_OK;
}

tp_status tp_diag_bounded_wait(unsigned int limit_us, int* result, tp_stream_t stream) {
  if (result == nullptr) return TP_ERR_NULL;
  if (!aligned16(result)) return TP_ERR_ALIGN;
  if (limit_us < 1u || limit_us > 1000000u) return TP_ERR_UNSUPPORTED;
  tpb::bounded_wait_probe_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_us) * 1000ull, result);
  return cuda_ok(cudaGetLastError(), "launch bounded_wait_probe_kernel") ? TP_OK : TP_ERR_CUDA;
}

tp_status tp_set_decode_max_tokens(int max_tokens) {
  if (max_tokens < 0 || max_tokens > kStreamMaxTokens) return TP_ERR_UNSUPPORTED;
  g_decode_max_tokens.store(max_tokens, std::memory_order_relaxed);
  return TP_OK;
}

int tp_get_decode_max_tokens(void) { return g_decode_max_tokens.load(std::memory_order_relaxed); }

tp_status tp_set_launch_options(unsigned int flags) {
  if ((flags & ~(TP_OPT_PDL | TP_OPT_STATIC_WEIGHTS)) != 0u) return TP_ERR_UNSUPPORTED;
  g_launch_options.store(flags, std::memory_order_relaxed);
  return TP_OK;
}

unsigned int tp_get_launch_options(void) {
  return g_launch_options.load(std::memory_order_relaxed);
}

}  // extern "C"

// ------------------------------------------------------------------ allocation-free MLP call
//
// h for tp_mlp_forward_noalloc, in the library's own device memory.  In host
// code this name is only a host-side stand-in for the array: the device
// address is looked up with cudaGetSymbolAddress, once per device, and cached.
static __device__ __align__(256) unsigned char g_tp_noalloc_scratch[TP_NOALLOC_SCRATCH_BYTES];

namespace {

void* g_noalloc_addr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of g_tp_noalloc_scratch on the current device, or nullptr.
void* noalloc_scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_tp_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_addr[dev] = p;
  }
  return g_noalloc_addr[dev];
}

}  // namespace

extern "C" tp_status tp_mlp_forward_noalloc(const tp_bf16* x, const tp_bf16* w1,
                                            const tp_bf16* b1, const tp_bf16* w2,
                                            const tp_bf16* b2, int T, int H, int F,
                                            int tp_degree, int act, tp_bf16* out,
                                            tp_stream_t stream) {
  // every argument check comes before the first CUDA call
  if (x == nullptr || w1 == nullptr || w2 == nullptr || out == nullptr) return TP_ERR_NULL;
  if (!aligned16(x) || !aligned16(w1) || !aligned16(w2) || !aligned16(out) ||
      (b1 != nullptr && !aligned16(b1)) || (b2 != nullptr && !aligned16(b2)))
    return TP_ERR_ALIGN;
  if (T < 1 || !feat_ok(H) || !feat_ok(F)) return TP_ERR_SHAPE;
  if (act != TP_ACT_NONE && act != TP_ACT_GELU_TANH) return TP_ERR_UNSUPPORTED;
  if (tp_degree < 1 || F % tp_degree != 0 || (F / tp_degree) % 64 != 0) return TP_ERR_TP_DEGREE;
  const size_t need = static_cast<size_t>(T) * static_cast<size_t>(F) * 2u;
  if (need > static_cast<size_t>(TP_NOALLOC_SCRATCH_BYTES)) return TP_ERR_WORKSPACE;
  void* scratch = noalloc_scratch_address();
  if (scratch == nullptr) return TP_ERR_CUDA;
  return tp_mlp_forward(x, w1, b1, w2, b2, T, H, F, tp_degree, act, out, scratch,
                        static_cast<size_t>(TP_NOALLOC_SCRATCH_BYTES), stream);
}
