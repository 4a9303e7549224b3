// loza_ssa.cu - host side of the C ABI declared in include/loza_ssa.h:
// argument validation, TMA descriptor construction, kernel selection and
// launch on the caller's stream. All arithmetic runs in the kernels included
// below; nothing here touches tensor data.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "loza_ssa.h"
#include "prefill.cuh"
#include "prefill_pair.cuh"
#include "prefill_mha2.cuh"
#include "prefill_mla.cuh"
#include "decode.cuh"
#include "decode_mla.cuh"
#include "decode_mla_hb.cuh"
#include "merge.cuh"
#include "backward.cuh"
#include "hi_index.cuh"

namespace loza {
namespace {

std::atomic<uint64_t> g_launches{0};

// cuTensorMapEncodeTiled, fetched from the driver at first use (no libcuda link).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 3-D bf16 map over [rows, heads, dim] with 128-byte swizzle and a
// {64, 1, box_rows} box: one [box_rows x 64 columns] tile of one head per load.
bool make_map_3d(CUtensorMap* m, const void* base, int64_t dim, int64_t heads, int64_t rows,
                 int64_t head_stride_elems, int64_t row_stride_elems, uint32_t box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)dim, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)(head_stride_elems * 2), (cuuint64_t)(row_stride_elems * 2)};
  cuuint32_t box[3] = {64, 1, box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool stride_ok(int64_t s) { return s > 0 && (s * 2) % 16 == 0 && s * 2 < (int64_t(1) << 40); }

// A window the prefill and decode kernels take: b a power of two from 1 to
// 65,536 tokens per block; s >= 0 sink blocks and l >= 1 local blocks, or the
// unbounded window (l = LOZA_UNBOUNDED: every earlier key; s is then unused).
bool window_ok(const loza_ssa_params& p) {
  const int b = p.block_size;
  if (b < 1 || b > 65536 || (b & (b - 1)) != 0) return false;
  if (p.n_local == LOZA_UNBOUNDED) return true;
  if (p.n_local < 1 || p.n_sink < 0) return false;
  if ((int64_t)p.n_sink * b > (int64_t(1) << 30) || (int64_t)p.n_local * b > (int64_t(1) << 30)) return false;
  return true;
}

SsaWindow host_window(const loza_ssa_params& p) {
  const bool unb = p.n_local == LOZA_UNBOUNDED;
  return SsaWindow{p.block_size, unb ? 0 : p.n_sink * p.block_size, unb ? -1 : p.n_local};
}

// Most units of `unit` keys (RowWalk) that a query at any position below
// max_seqlen reads. Once the window is full the count repeats with period
// max(b, unit) (both powers of two), so the positions of the first window and
// the last few periods before max_seqlen cover every value it takes.
int max_row_units(const loza_ssa_params& p, int32_t max_seqlen, int unit) {
  const SsaWindow w = host_window(p);
  if (w.n_local < 0) return (max_seqlen - 1) / unit + 1;
  const int64_t period = std::max(p.block_size, unit);
  const int64_t span = std::min<int64_t>(max_seqlen, (int64_t)(p.n_sink + p.n_local + 2) * p.block_size + 4 * period);
  int best = 0;
  for (int64_t i = 0; i < span; ++i) best = std::max(best, RowWalk(w, (int)i, unit).count);
  for (int64_t i = std::max<int64_t>(span, max_seqlen - 4 * period - unit); i < max_seqlen; ++i)
    best = std::max(best, RowWalk(w, (int)i, unit).count);
  return best;
}

// Most key tiles (BlockWalk) a query tile of a sequence of max_seqlen reads.
int max_tiles(const loza_ssa_params& p, int32_t max_seqlen) {
  const int nq = (max_seqlen + kTile - 1) / kTile;
  const SsaWindow w = host_window(p);
  if (w.n_local < 0) return nq;
  const int n_sink = p.n_sink, b = p.block_size;
  const int64_t period = std::max(1, b / kTile);
  const int64_t span = std::min<int64_t>(nq, ((int64_t)(n_sink + p.n_local + 2) * b) / kTile + 4 * period + 2);
  int best = 0;
  for (int64_t q = 0; q < span; ++q) best = std::max(best, BlockWalk((int)q, n_sink, w.n_local, b).count);
  for (int64_t q = std::max<int64_t>(span, nq - 4 * period - 2); q < nq; ++q)
    best = std::max(best, BlockWalk((int)q, n_sink, w.n_local, b).count);
  return best;
}

int sm_count() {
  static const int n = [] {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
      return v;
    return 148;
  }();
  return n;
}

// Split-KV plan of the absorbed decode: CTAs per sequence (nsplit) and selected
// blocks (or half blocks) per CTA (bps), sized so that batch * nsplit CTAs fill
// the GPU in one wave.
//   - a few sequences with long windows (more than 8 blocks, batch * 16 <= SMs):
//     the block kernel, many splits, merged through the workspace;
//   - windows of at most 24 blocks while two CTAs per sequence fit (batch * 2
//     <= SMs): the half-block kernel, up to 4 splits per sequence in a
//     cluster, merged on chip;
//   - otherwise the block kernel with up to 4 splits per sequence in a
//     cluster (one CTA per sequence for large batches), merged on chip.
// Measured kernel times (64 heads, 8-block window, contexts of 64K-128K;
// half-block vs the best alternative measured: the block kernel, or at 64
// sequences a kernel splitting the heads over two CTAs per sequence):
// 1 sequence 21.8 vs 25.4 us, 8: 22.2 vs 24.5, 64: 32.5 vs 34.3,
// 96: 47.2 vs 43.6, 128: 49.0 vs 47.6. With the whole context selected (the dense decode of
// 64 sequences of 64K-128K) the block kernel took 1.74 ms, the half-block one
// 2.22 ms.
struct DecodePlan {
  int bps, nsplit;  // half_block: half blocks per split
  bool cluster;     // the splits of a sequence form a cluster and merge on chip
  bool half_block;  // 64-row units resident for both MMAs (decode_mla_hb.cuh)
};
DecodePlan decode_plan(const loza_ssa_params& p, int32_t max_seqlen, int32_t batch) {
  const int count = max_row_units(p, max_seqlen, kTile);  // selected 128-row blocks
  const int sms = sm_count();
  if (count > 8 && (int64_t)batch * 16 <= sms) {
    int ns = (sms + batch - 1) / batch;
    if (ns > count) ns = count;
    const int bps = (count + ns - 1) / ns;
    return {bps, (count + bps - 1) / bps, false, false};
  }
  if (count <= 24 && (int64_t)batch * 2 <= sms) {
    // half blocks: up to 4 CTAs per sequence in one cluster, each pulling
    // its share of the rows once
    // (the on-chip merge splits the 512 value columns evenly: nsplit is 1, 2
    // or 4, and a split may get no half block)
    const int nh = max_row_units(p, max_seqlen, kHbRows);
    int ns = 1;
    while (ns < kHbMaxSplit && ns * 2 <= nh && (int64_t)batch * ns * 2 <= sms) ns *= 2;
    return {(nh + ns - 1) / ns, ns, true, true};
  }
  int ns = 1;
  while (ns < 4 && ns * 2 <= count && (int64_t)batch * ns * 2 <= sms) ns *= 2;
  return {(count + ns - 1) / ns, ns, true, false};
}

struct DecodeWorkspace {
  size_t o_off, ml_off, ticket_off, total;
};
DecodeWorkspace decode_workspace(int32_t batch, const DecodePlan& plan) {
  DecodeWorkspace w{0, 0, 0, 0};
  if (plan.cluster) return w;
  const size_t parts = (size_t)batch * plan.nsplit * kDecHeads;
  w.o_off = 0;
  w.ml_off = parts * 512 * sizeof(float);
  w.ticket_off = w.ml_off + parts * sizeof(float4);
  w.total = w.ticket_off + ((size_t)batch * sizeof(int) + 255) / 256 * 256;
  return w;
}

// 4-D bf16 map {64 columns, rows, ntiles, 1}: column tile i of row r at
// base + r * row_stride + i * tile_stride_bytes (128-byte swizzle); a box
// {64, box_rows, box_tiles, 1} lands as box_tiles consecutive [box_rows x 64]
// tiles.
bool make_map_tiles4(CUtensorMap* m, const void* base, int64_t rows, int ntiles, int64_t row_stride,
                     int64_t tile_stride_bytes, uint32_t box_rows, uint32_t box_tiles) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {64, (cuuint64_t)rows, (cuuint64_t)ntiles, 1};
  cuuint64_t strides[3] = {(cuuint64_t)row_stride * 2, (cuuint64_t)tile_stride_bytes,
                           (cuuint64_t)row_stride * 2 * (cuuint64_t)rows};
  cuuint32_t box[4] = {64, box_rows, box_tiles, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D bf16 map {64 columns, rows, 9 column tiles, batch} over a latent tensor
// [batch][rows][576] with the given row and batch strides (elements): the
// tile dimension's stride is 128 bytes, so a box {64, box_rows, 3, 1} lands as
// three consecutive [box_rows x 64] 128-byte-swizzled tiles.
bool make_map_latent3(CUtensorMap* m, const void* base, int64_t rows, int64_t batch, int64_t row_stride,
                      int64_t batch_stride, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {64, (cuuint64_t)rows, 9, (cuuint64_t)batch};
  cuuint64_t strides[3] = {(cuuint64_t)row_stride * 2, 128, (cuuint64_t)batch_stride * 2};
  cuuint32_t box[4] = {64, box_rows, 3, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Validate an absorbed-MLA decode call and build its kernel parameters
// (everything except the workspace pointers).
loza_status setup_decode_mla(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                             int32_t batch, int32_t max_seqlen, int64_t cache_batch_stride,
                             int64_t cache_row_stride, int32_t n_heads, const loza_ssa_params& p, void* out,
                             float* lse, DecodeParams* prm, DecodePlan* plan) {
  if (!q || !k_cache || !seqlens || !out || !lse) return LOZA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(out)) return LOZA_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || max_seqlen < 1) return LOZA_ERR_INVALID_ARG;
  if (!stride_ok(cache_row_stride) || !stride_ok(cache_batch_stride) ||
      cache_batch_stride < (int64_t)max_seqlen * cache_row_stride || cache_row_stride < 576)
    return LOZA_ERR_INVALID_ARG;
  if (!window_ok(p)) return LOZA_ERR_UNSUPPORTED;
  if (n_heads != kDecHeads) return LOZA_ERR_UNSUPPORTED;
  if (v_cache && v_cache != k_cache) return LOZA_ERR_UNSUPPORTED;
  *plan = decode_plan(p, max_seqlen, batch);
  std::memset(prm, 0, sizeof(*prm));
  EncodeTiledFn fn = encode_fn();
  if (!fn) return LOZA_ERR_CUDA;
  {
    cuuint64_t dims[3] = {576, (cuuint64_t)n_heads, (cuuint64_t)batch};
    cuuint64_t strides[2] = {576 * 2, (cuuint64_t)n_heads * 576 * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kDecHeads, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (fn(&prm->tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return LOZA_ERR_CUDA;
  }
  {
    cuuint64_t dims[3] = {576, (cuuint64_t)max_seqlen, (cuuint64_t)batch};
    cuuint64_t strides[2] = {(cuuint64_t)cache_row_stride * 2, (cuuint64_t)cache_batch_stride * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t box64[3] = {64, 64, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (fn(&prm->tm_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(k_cache), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        fn(&prm->tm_kv64, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(k_cache), dims, strides, box64,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return LOZA_ERR_CUDA;
  }
  if (!make_map_latent3(&prm->tm_q3, q, n_heads, batch, 576, (int64_t)n_heads * 576, (uint32_t)kDecHeads) ||
      !make_map_latent3(&prm->tm_kv3, k_cache, max_seqlen, batch, cache_row_stride, cache_batch_stride, 64))
    return LOZA_ERR_CUDA;
  prm->seqlens = seqlens;
  prm->out = reinterpret_cast<__nv_bfloat16*>(out);
  prm->lse = lse;
  prm->nsplit = plan->nsplit;
  prm->bps = plan->bps;
  prm->n_sink = p.n_local == LOZA_UNBOUNDED ? 0 : p.n_sink;
  prm->n_local = p.n_local == LOZA_UNBOUNDED ? -1 : p.n_local;
  prm->block = p.block_size;
  prm->scale_log2 = p.scale * 1.4426950408889634f;
  return LOZA_OK;
}

// Point the kernel at its workspace (unless the plan merges on chip) and launch.
loza_status launch_decode_mla(DecodeParams& prm, const DecodePlan& plan, int32_t batch, uint8_t* ws,
                              cudaStream_t st, bool after = false) {
  // after: launched with programmatic stream serialization behind the kernel
  // that produced its rows and lengths (the kernels wait for it first)
  if (plan.half_block) {
    // the kernel's merge gives each split 512 / nsplit whole value columns
    if (plan.nsplit != 1 && plan.nsplit != 2 && plan.nsplit != 4) return LOZA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(ssa_decode_mla_hb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecodeHbLayout::SMEM_BYTES) != cudaSuccess)
      return LOZA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.nsplit, batch, 1);
    cfg.blockDim = dim3(kHbThreads, 1, 1);
    cfg.dynamicSmemBytes = DecodeHbLayout::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = plan.nsplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, ssa_decode_mla_hb_kernel, prm) != cudaSuccess) return LOZA_ERR_CUDA;
  } else if (!plan.cluster) {
    const DecodeWorkspace wl = decode_workspace(batch, plan);
    prm.ws_o = reinterpret_cast<float*>(ws + wl.o_off);
    prm.ws_ml = reinterpret_cast<float4*>(ws + wl.ml_off);
    prm.ws_ticket = reinterpret_cast<int*>(ws + wl.ticket_off);
    // the arrival counters must start at zero; the partials are fully rewritten
    if (cudaMemsetAsync(prm.ws_ticket, 0, (size_t)batch * sizeof(int), st) != cudaSuccess) return LOZA_ERR_CUDA;
    if (cudaFuncSetAttribute(ssa_decode_mla_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecodeLayout::SMEM_BYTES) != cudaSuccess)
      return LOZA_ERR_CUDA;
    ssa_decode_mla_kernel<false><<<dim3(plan.nsplit, batch), kDecThreads, DecodeLayout::SMEM_BYTES, st>>>(prm);
  } else {
    // the cluster merge gives each split 512 / nsplit whole value columns
    if (plan.nsplit != 1 && plan.nsplit != 2 && plan.nsplit != 4) return LOZA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(ssa_decode_mla_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecodeLayout::SMEM_BYTES) != cudaSuccess)
      return LOZA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.nsplit, batch, 1);
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = DecodeLayout::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = plan.nsplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, ssa_decode_mla_kernel<true>, prm) != cudaSuccess) return LOZA_ERR_CUDA;
  }
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? LOZA_OK : LOZA_ERR_CUDA;
}

// Backward workspace: D [T*H] fp32, then the sink partials
// [B][s][H][nslots][128][DQK+DV] fp32.
struct BwdWorkspace {
  size_t d_off, part_off, total;
  int nslots;
};
// 128-key tiles that hold a sink key.
int bwd_sink_tiles(const loza_ssa_params& p) {
  return (int)(((int64_t)p.n_sink * p.block_size + kTile - 1) / kTile);
}
BwdWorkspace bwd_workspace(int32_t batch, int64_t total_tokens, int32_t max_seqlen, int32_t n_heads, int d_qk,
                           int d_v, const loza_ssa_params& p) {
  BwdWorkspace w;
  const int nq_max = (max_seqlen + kTile - 1) / kTile;
  // sink tile 0 has the most "far" query tiles: those past its local range
  const int far = std::max(0, nq_max - bwd_local_end(0, p.block_size, p.n_local));
  w.nslots = 1 + (far + kSinkChunk - 1) / kSinkChunk;
  w.d_off = 0;
  w.part_off = ((size_t)total_tokens * n_heads * sizeof(float) + 255) / 256 * 256;
  w.total = w.part_off +
            (size_t)batch * bwd_sink_tiles(p) * n_heads * w.nslots * kTile * (d_qk + d_v) * sizeof(float);
  return w;
}

template <int DQK, int DV>
loza_status launch_backward(BwdParams& prm, const void* out, const void* dout, int64_t rows, int nq_max, int batch,
                            cudaStream_t st) {
  {
    const int64_t threads = rows * (DV / 8);
    ssa_bwd_preprocess<DV><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), const_cast<float*>(prm.dvec),
        rows);
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  using LQ = BwdDqLayout<DQK, DV>;
  using LK = BwdDkvLayout<DQK, DV>;
  if (cudaFuncSetAttribute(ssa_bwd_dq_kernel<DQK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           LQ::SMEM_BYTES) != cudaSuccess ||
      cudaFuncSetAttribute(ssa_bwd_dkdv_kernel<DQK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           LK::SMEM_BYTES) != cudaSuccess)
    return LOZA_ERR_CUDA;
  prm.far_mode = 0;
  ssa_bwd_dq_kernel<DQK, DV><<<dim3(nq_max, prm.n_heads, batch), kBwdDqThreads, LQ::SMEM_BYTES, st>>>(prm);
  ssa_bwd_dkdv_kernel<DQK, DV><<<dim3(nq_max, prm.n_heads, batch), kBwdDkvThreads, LK::SMEM_BYTES, st>>>(prm);
  g_launches.fetch_add(2, std::memory_order_relaxed);
  if (prm.n_sink_tiles > 0) {
    if (prm.nslots > 1) {
      prm.far_mode = 1;
      ssa_bwd_dkdv_kernel<DQK, DV><<<dim3(prm.nslots - 1, prm.n_heads * prm.n_sink_tiles, batch), kBwdDkvThreads,
                                     LK::SMEM_BYTES, st>>>(prm);
      g_launches.fetch_add(1, std::memory_order_relaxed);
    }
    ssa_bwd_sink_reduce<DQK, DV><<<dim3(kTile, prm.n_heads * prm.n_sink_tiles, batch), DQK + DV, 0, st>>>(prm);
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  return cudaGetLastError() == cudaSuccess ? LOZA_OK : LOZA_ERR_CUDA;
}

template <int DQK, int DVT, int NSTAGE>
loza_status launch_prefill(const PrefillParams& prm, int max_seqlen, int batch, cudaStream_t stream) {
  using LY = PrefillLayout<DQK, DVT, NSTAGE>;
  auto kern = ssa_prefill_kernel<DQK, DVT, NSTAGE>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::SMEM_BYTES) != cudaSuccess)
    return LOZA_ERR_CUDA;
  dim3 grid((max_seqlen + kTile - 1) / kTile, prm.n_heads * prm.dv_slices, batch);
  kern<<<grid, kPrefillThreads, LY::SMEM_BYTES, stream>>>(prm);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? LOZA_OK : LOZA_ERR_CUDA;
}

// Per-head 192 / 128 prefill, two query tiles per CTA: grid (tile pairs, heads, sequences).
loza_status launch_prefill_mha2(const PrefillParams& prm, int max_seqlen, int batch, cudaStream_t stream) {
  using LY = PrefillMha2Layout<192, 128>;
  auto kern = ssa_prefill_mha2_kernel<192, 128>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::SMEM_BYTES) != cudaSuccess)
    return LOZA_ERR_CUDA;
  const int tiles = (max_seqlen + kTile - 1) / kTile;
  dim3 grid((tiles + 1) / 2, prm.n_heads, batch);
  kern<<<grid, kMha2Threads, LY::SMEM_BYTES, stream>>>(prm);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? LOZA_OK : LOZA_ERR_CUDA;
}

// Absorbed-MLA prefill on CTA pairs: grid x = (head pair, value slice, CTA of
// the pair), y = query tile, z = sequence; clusters of 2 along x.
loza_status launch_prefill_pair(const PrefillPairParams& prm, int max_seqlen, int batch, cudaStream_t stream) {
  using LY = PrefillPairLayout;
  if (cudaFuncSetAttribute(ssa_prefill_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::SMEM_BYTES) !=
      cudaSuccess)
    return LOZA_ERR_CUDA;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  const int pairs = std::max(1, std::min(sm_count() / 2, prm.total_tiles));
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kPairThreads, 1, 1);
  cfg.dynamicSmemBytes = LY::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, ssa_prefill_pair_kernel, prm) != cudaSuccess) return LOZA_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? LOZA_OK : LOZA_ERR_CUDA;
}

// Two-pass absorbed prefill: scratch per CTA of the persistent grid (at most
// one CTA per SM): P of every key block of a tile, and the rescale factors.
size_t mla_scratch_per_cta(int max_blocks) {
  return (size_t)max_blocks * (kTile * kTile * 2 + 256 * 4);
}
size_t mla_workspace_bytes(int max_blocks) { return (size_t)sm_count() * mla_scratch_per_cta(max_blocks); }
// The two-pass kernel keeps one bit per key tile of a query tile.
bool mla_window_ok(const loza_ssa_params& p, int32_t max_seqlen) {
  return p.n_local != LOZA_UNBOUNDED && max_tiles(p, max_seqlen) <= kMlaMaxBlocks;
}

loza_status launch_prefill_mla(PrefillMlaParams& prm, void* workspace, cudaStream_t stream) {
  using LY = PrefillMlaLayout;
  if (cudaFuncSetAttribute(ssa_prefill_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::SMEM_BYTES) !=
      cudaSuccess)
    return LOZA_ERR_CUDA;
  const int pairs = std::max(1, std::min(sm_count() / 2, prm.total_tiles));
  const int ctas = 2 * pairs;
  // scratch: P as 16 KB images of [8 key chunks][128 rows][8 keys] bf16, two
  // per key block (keys 0-63, 64-127), max_blocks blocks per CTA; then the factors.
  // The map reads one image as 128 lines of 128 bytes, copied unswizzled.
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  prm.p_ws = reinterpret_cast<__nv_bfloat16*>(ws);
  prm.a_ws = reinterpret_cast<float*>(ws + (size_t)sm_count() * prm.max_blocks * kTile * kTile * 2);
  {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return LOZA_ERR_CUDA;
    cuuint64_t dims[2] = {64, (cuuint64_t)ctas * prm.max_blocks * 2 * kTile};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {64, (cuuint32_t)kTile};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&prm.tm_p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, prm.p_ws, dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return LOZA_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(ctas, 1, 1);
  cfg.blockDim = dim3(kMlaThreads, 1, 1);
  cfg.dynamicSmemBytes = LY::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, ssa_prefill_mla_kernel, prm) != cudaSuccess) return LOZA_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? LOZA_OK : LOZA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Built-in scratch for loza_ssa_decode_noalloc.
//
// The absorbed decode keeps one partial result per (sequence, split, head)
// between its split CTAs and the CTA that merges them. Callers that cannot
// allocate device memory get this fixed array instead of a caller-provided
// workspace. It is ordinary device memory of this module: every GPU that loads
// the library reserves kNoAllocScratchBytes for it until the process exits.
// Host code must not use the name g_decode_scratch as a pointer; the device
// address comes from cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) uint8_t g_decode_scratch[kNoAllocScratchBytes];

// Devices of one process for which per-device host state is kept.
constexpr int kMaxDevices = 64;

// Device address of g_decode_scratch on the current device, looked up on
// every call: the lookup is cheap once the module is loaded, and a module
// loaded again after cudaDeviceReset may place the array elsewhere. Returns
// nullptr if the lookup fails.
void* decode_scratch_address() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return nullptr;
  return p;
}

// Grid for a grid-stride pass over n 16-byte vectors: at most a few waves.
unsigned stream_grid(int64_t n) {
  const int64_t per = (int64_t)kMergeThreads;
  const int64_t cap = (int64_t)sm_count() * 8;
  return (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + per - 1) / per, cap));
}

// Hierarchical index (page 4): the window part and the selected tokens are
// packed per sequence (hi_gather_kernel) and attended by the absorbed decode
// with the unbounded window: every packed row is visible.
constexpr int64_t kHiMaxWindowRows = 65536;  // rows of a bounded window the packed block holds at most

loza_ssa_params hi_packed_params(float scale) {
  loza_ssa_params q;
  q.block_size = kTile;
  q.n_sink = 0;
  q.n_local = LOZA_UNBOUNDED;
  q.scale = scale;
  return q;
}

bool hi_window_ok(const loza_ssa_params& p) {
  if (!window_ok(p)) return false;
  return p.n_local == LOZA_UNBOUNDED ||
         ((int64_t)p.n_sink + p.n_local) * p.block_size <= kHiMaxWindowRows;
}

struct HiWorkspace {
  size_t page_scored, sel_pages, n_pages, zeroed, zeroed_bytes, page_hist, hist1, counters, page_cand, tok_keys,
      tok_cand, selected, n_sel, counts, packed, dec, total;
  int cap_rows;  // packed rows per sequence (0: the unbounded window, decoded in place)
};
size_t hi_align(size_t x) { return (x + 255) / 256 * 256; }
HiWorkspace hi_workspace(int32_t batch, int32_t max_seqlen, int32_t top_pages, int32_t top_k,
                         const loza_ssa_params& p) {
  HiWorkspace w;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = hi_align(off + bytes);
    return at;
  };
  const int64_t pages = std::max<int64_t>(max_seqlen / kHiPage, 1);
  w.page_scored = take((size_t)batch * pages * 8);
  w.sel_pages = take((size_t)batch * top_pages * 4);
  w.n_pages = take((size_t)batch * 4);
  // histograms and list counters, cleared by one memset per call
  w.zeroed_bytes = (size_t)batch * (2 * kHiBins + 4) * 4;
  w.zeroed = take(w.zeroed_bytes);
  w.page_hist = w.zeroed;
  w.hist1 = w.page_hist + (size_t)batch * kHiBins * 4;
  w.counters = w.hist1 + (size_t)batch * kHiBins * 4;
  w.page_cand = take((size_t)batch * pages * 8);
  w.tok_keys = take((size_t)batch * top_pages * kHiPage * 8);
  w.tok_cand = take((size_t)batch * top_pages * kHiPage * 8);
  w.selected = take((size_t)batch * std::max(top_k, 1) * 4);
  w.n_sel = take((size_t)batch * 4);
  w.counts = take((size_t)batch * 4);
  if (p.n_local == LOZA_UNBOUNDED) {
    w.cap_rows = 0;
    w.packed = take(0);
    w.dec = take(decode_workspace(batch, decode_plan(p, max_seqlen, batch)).total);
  } else {
    const int64_t rows = std::min<int64_t>(max_seqlen, ((int64_t)p.n_sink + p.n_local) * p.block_size + top_k);
    w.cap_rows = (int)((rows + kTile - 1) / kTile * kTile);
    w.packed = take((size_t)batch * w.cap_rows * 576 * 2);
    w.dec = take(decode_workspace(batch, decode_plan(hi_packed_params(p.scale), w.cap_rows, batch)).total);
  }
  w.total = off;
  return w;
}

bool hi_args_ok(const void* k_index, int64_t index_batch_stride, int64_t index_row_stride, int32_t batch,
                int32_t max_seqlen, int32_t d_index) {
  if (!k_index || !aligned16(k_index)) return false;
  if (batch < 1 || batch > 65535 || max_seqlen < 1) return false;
  if (d_index < kHiDimStep || d_index > kHiMaxDim || d_index % kHiDimStep != 0) return false;
  if (!stride_ok(index_row_stride) || !stride_ok(index_batch_stride) || index_row_stride < d_index ||
      index_batch_stride < (int64_t)max_seqlen * index_row_stride)
    return false;
  return true;
}

// Launch with programmatic stream serialization: the kernel may start while
// the kernel before it in the stream finishes (it calls griddep_wait before
// reading that kernel's results), hiding the launch gap of a chain.
template <typename... KArgs, typename... Args>
cudaError_t launch_after(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                         Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Index keys as a 3-D tensor {d, rows, batch}: 128-row x 64-column tiles with
// the 128-byte swizzle.
bool make_map_index(CUtensorMap* m, const void* k_index, int32_t d, int32_t rows, int32_t batch,
                    int64_t row_stride, int64_t batch_stride) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)row_stride * 2, (cuuint64_t)batch_stride * 2};
  cuuint32_t box[3] = {(cuuint32_t)kHiDimStep, (cuuint32_t)kHiPage, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(k_index), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The bounded-wait self-test: one thread waits on an mbarrier that nothing
// completes, gives up after limit_ns and records the timeout like every
// kernel's waits do. No TMA, MMA or other thread is involved.
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    mbar_wait_for(smem_u32(&bar), 0, nullptr, limit_ns);
  }
}

}  // namespace
}  // namespace loza

#include "prefill_host.cuh"

using namespace loza;

extern "C" {

loza_status loza_ssa_decode_paged(const void* q, const void* kv_pool, int32_t num_pages, int64_t pool_row_stride,
                                  const int32_t* block_table, int32_t bt_stride, const int32_t* seqlens,
                                  int32_t batch, int32_t max_seqlen, int32_t n_heads, loza_ssa_params p, void* out,
                                  float* lse, void* workspace, size_t workspace_bytes, loza_stream_t stream) {
  if (!block_table || !kv_pool) return LOZA_ERR_INVALID_ARG;
  if (num_pages < 1 || (int64_t)num_pages * kTile > INT32_MAX) return LOZA_ERR_INVALID_ARG;
  if (max_seqlen < 1 || bt_stride < (max_seqlen + kTile - 1) / kTile) return LOZA_ERR_INVALID_ARG;
  if (!stride_ok(pool_row_stride) || pool_row_stride < 576) return LOZA_ERR_INVALID_ARG;
  DecodeParams prm;
  DecodePlan plan;
  // validation and the query map as for a contiguous cache of max_seqlen rows per sequence ...
  const loza_status rc = setup_decode_mla(q, kv_pool, nullptr, seqlens, batch, max_seqlen,
                                          (int64_t)max_seqlen * pool_row_stride, pool_row_stride, n_heads, p, out,
                                          lse, &prm, &plan);
  if (rc != LOZA_OK) return rc;
  // ... then the cache map over the whole pool, addressed through the block table
  EncodeTiledFn fn = encode_fn();
  if (!fn) return LOZA_ERR_CUDA;
  cuuint64_t dims[3] = {576, (cuuint64_t)num_pages * kTile, 1};
  cuuint64_t strides[2] = {(cuuint64_t)pool_row_stride * 2, (cuuint64_t)num_pages * kTile * pool_row_stride * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  if (strides[1] >= (cuuint64_t(1) << 40)) return LOZA_ERR_INVALID_ARG;
  cuuint32_t box64[3] = {64, 64, 1};
  if (fn(&prm.tm_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kv_pool), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
      fn(&prm.tm_kv64, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kv_pool), dims, strides, box64, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return LOZA_ERR_CUDA;
  if (!make_map_latent3(&prm.tm_kv3, kv_pool, (int64_t)num_pages * kTile, 1, pool_row_stride,
                        (int64_t)num_pages * kTile * pool_row_stride, 64))
    return LOZA_ERR_CUDA;
  prm.block_table = block_table;
  prm.bt_stride = bt_stride;
  const DecodeWorkspace wl = decode_workspace(batch, plan);
  if (wl.total > 0) {
    if (!workspace || !aligned16(workspace)) return LOZA_ERR_INVALID_ARG;
    if (workspace_bytes < wl.total) return LOZA_ERR_WORKSPACE;
  }
  return launch_decode_mla(prm, plan, batch, static_cast<uint8_t*>(workspace), reinterpret_cast<cudaStream_t>(stream));
}

loza_status loza_ssa_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b, int64_t rows,
                           int32_t d_v, void* out, float* lse_out, loza_stream_t stream) {
  if (rows < 0 || d_v < 8 || d_v % 8 != 0) return LOZA_ERR_INVALID_ARG;
  if (rows == 0) return LOZA_OK;
  if (!o_a || !o_b || !out || !lse_a || !lse_b || !lse_out) return LOZA_ERR_INVALID_ARG;
  if (!aligned16(o_a) || !aligned16(o_b) || !aligned16(out)) return LOZA_ERR_INVALID_ARG;
  if (rows > (int64_t(1) << 40) / d_v) return LOZA_ERR_INVALID_ARG;
  const int vec8 = d_v / 8;
  ssa_merge_kernel<<<stream_grid(rows * vec8), kMergeThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(o_a), lse_a, static_cast<const uint4*>(o_b), lse_b, static_cast<uint4*>(out),
      lse_out, rows, vec8);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? LOZA_OK : LOZA_ERR_CUDA;
}

loza_status loza_ssa_mix(const void* o_full, const void* o_ssa, int64_t n, float alpha, void* out,
                         loza_stream_t stream) {
  if (n < 0 || n % 8 != 0) return LOZA_ERR_INVALID_ARG;
  if (n == 0) return LOZA_OK;
  if (!o_full || !o_ssa || !out) return LOZA_ERR_INVALID_ARG;
  if (!aligned16(o_full) || !aligned16(o_ssa) || !aligned16(out)) return LOZA_ERR_INVALID_ARG;
  ssa_mix_kernel<<<stream_grid(n / 8), kMergeThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(o_full), static_cast<const uint4*>(o_ssa), static_cast<uint4*>(out), n / 8, alpha);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? LOZA_OK : LOZA_ERR_CUDA;
}

const char* loza_status_string(loza_status s) {
  switch (s) {
    case LOZA_OK: return "ok";
    case LOZA_ERR_INVALID_ARG: return "invalid argument";
    case LOZA_ERR_UNSUPPORTED: return "unsupported shape or window";
    case LOZA_ERR_WORKSPACE: return "workspace too small";
    case LOZA_ERR_CUDA: return "CUDA error";
    case LOZA_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

uint64_t loza_launch_count(void) { return g_launches.load(); }

loza_status loza_wait_selftest(uint32_t limit_us, loza_stream_t stream) {
  if (limit_us < 1 || limit_us > 2000000) return LOZA_ERR_INVALID_ARG;
  wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>((unsigned long long)limit_us * 1000ull);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? LOZA_OK : LOZA_ERR_CUDA;
}

loza_status loza_device_status(loza_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return LOZA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return LOZA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return LOZA_ERR_CUDA;
    return LOZA_ERR_TIMEOUT;
  }
  return LOZA_OK;
}

size_t loza_ssa_workspace_size(int op, int32_t batch, int64_t total_tokens, int32_t max_seqlen,
                               int32_t n_heads, int32_t n_kv_heads, int32_t d_qk, int32_t d_v,
                               loza_ssa_params p) {
  (void)total_tokens;
  if (batch < 1 || max_seqlen < 1 || !window_ok(p)) return 0;
  if (op == LOZA_OP_DECODE) {
    if (n_kv_heads == 1 && n_heads == kDecHeads && d_qk == 576 && d_v == 512)
      return decode_workspace(batch, decode_plan(p, max_seqlen, batch)).total;
    return 0;
  }
  if (op == LOZA_OP_PREFILL) {
    if (n_kv_heads == 1 && d_qk == 576 && d_v == 512 && n_heads % 2 == 0 && mla_window_ok(p, max_seqlen))
      return mla_workspace_bytes(max_tiles(p, max_seqlen));
    return 0;
  }
  if (op == LOZA_OP_PREFILL_HOST) {
    if (!window_ok(p)) return 0;
    if (total_tokens < max_seqlen || total_tokens > INT32_MAX || !host_shape_ok(n_heads, n_kv_heads, d_qk, d_v))
      return 0;
    const HostChunkPlan h = host_chunk_plan(max_seqlen, p);
    const size_t pf = loza_ssa_workspace_size(LOZA_OP_PREFILL, 1, h.rows_max, (int32_t)h.rows_max, n_heads,
                                              n_kv_heads, d_qk, d_v, p);
    return host_layout(h, host_chunk_cap(batch, total_tokens), pf, n_heads, n_kv_heads, d_qk, d_v).total;
  }
  if (op == LOZA_OP_BACKWARD) {
    if (!window_ok(p)) return 0;
    if (n_kv_heads != n_heads || p.n_local == LOZA_UNBOUNDED || total_tokens < 1) return 0;
    if (!((d_qk == 64 && d_v == 64) || (d_qk == 192 && d_v == 128))) return 0;
    return bwd_workspace(batch, total_tokens, max_seqlen, n_heads, d_qk, d_v, p).total;
  }
  return 0;
}

loza_status loza_ssa_prefill(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                             int32_t batch, int64_t total_tokens, int32_t max_seqlen, int32_t n_heads,
                             int32_t n_kv_heads, int32_t d_qk, int32_t d_v, int64_t q_row_stride,
                             int64_t k_row_stride, int64_t v_row_stride, loza_ssa_params p, void* out,
                             float* lse, void* workspace, size_t workspace_bytes, loza_stream_t stream) {
  if (!q || !k || !v || !cu_seqlens || !out || !lse) return LOZA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LOZA_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || total_tokens < 1 || total_tokens > INT32_MAX || max_seqlen < 1 ||
      max_seqlen > total_tokens)
    return LOZA_ERR_INVALID_ARG;
  if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads != 0) return LOZA_ERR_INVALID_ARG;
  if (!stride_ok(q_row_stride) || !stride_ok(k_row_stride) || !stride_ok(v_row_stride))
    return LOZA_ERR_INVALID_ARG;
  if (q_row_stride < (int64_t)n_heads * d_qk || k_row_stride < (int64_t)n_kv_heads * d_qk)
    return LOZA_ERR_INVALID_ARG;
  const bool latent_v = (v == k);
  if (latent_v ? (d_v > d_qk || v_row_stride != k_row_stride) : v_row_stride < (int64_t)n_kv_heads * d_v)
    return LOZA_ERR_INVALID_ARG;
  if (!window_ok(p)) return LOZA_ERR_UNSUPPORTED;
  if (!(n_kv_heads == 1 || n_kv_heads == n_heads)) return LOZA_ERR_UNSUPPORTED;

  PrefillParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.cu_seqlens = cu_seqlens;
  prm.out = reinterpret_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.n_heads = n_heads;
  prm.n_kv_heads = n_kv_heads;
  prm.d_v = d_v;
  prm.n_sink = p.n_local == LOZA_UNBOUNDED ? 0 : p.n_sink;
  prm.n_local = p.n_local == LOZA_UNBOUNDED ? -1 : p.n_local;
  prm.block = p.block_size;
  prm.scale_log2 = p.scale * 1.4426950408889634f;

  int dvt;
  if (d_qk == 64 && d_v == 64) dvt = 64;
  else if (d_qk == 192 && d_v == 128) dvt = 128;
  else if (d_qk == 576 && d_v == 512) dvt = 256;
  else return LOZA_ERR_UNSUPPORTED;
  prm.dv_slices = d_v / dvt;
  if ((int64_t)n_heads * prm.dv_slices > 65535) return LOZA_ERR_UNSUPPORTED;

  const int64_t v_head_stride = latent_v ? d_qk : d_v;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dvt == 256 && n_kv_heads == 1 && n_heads % 2 == 0 && mla_window_ok(p, max_seqlen) && workspace != nullptr &&
      aligned16(workspace) && workspace_bytes >= mla_workspace_bytes(max_tiles(p, max_seqlen))) {
    // absorbed MLA, bounded window: S once, the value dimension in two passes
    PrefillMlaParams mp;
    std::memset(&mp, 0, sizeof(mp));
    mp.cu_seqlens = cu_seqlens;
    mp.out = prm.out;
    mp.lse = lse;
    mp.max_blocks = max_tiles(p, max_seqlen);
    mp.n_heads = n_heads;
    mp.n_qtiles = (max_seqlen + kTile - 1) / kTile;
    if ((int64_t)batch * mp.n_qtiles * (n_heads / 2) > INT32_MAX) return LOZA_ERR_UNSUPPORTED;
    mp.total_tiles = batch * mp.n_qtiles * (n_heads / 2);
    mp.n_sink = prm.n_sink;
    mp.n_local = prm.n_local;
    mp.block = prm.block;
    mp.scale_log2 = prm.scale_log2;
    if (!make_map_3d(&mp.tm_q, q, d_qk, n_heads, total_tokens, d_qk, q_row_stride) ||
        !make_map_3d(&mp.tm_k, k, d_qk, 1, total_tokens, d_qk, k_row_stride, 64) ||
        !make_map_3d(&mp.tm_v, v, d_v, 1, total_tokens, v_head_stride, v_row_stride) ||
        !make_map_3d(&mp.tm_v64, v, d_v, 1, total_tokens, v_head_stride, v_row_stride, 64) ||
        !make_map_tiles4(&mp.tm_k2, k, total_tokens, 9, k_row_stride, 128, 64, 2) ||
        !make_map_tiles4(&mp.tm_v2[0], static_cast<const uint16_t*>(v) + 256, total_tokens, 2, v_row_stride, 256, 64,
                         2) ||
        !make_map_tiles4(&mp.tm_v2[1], static_cast<const uint16_t*>(v) + 320, total_tokens, 2, v_row_stride, 256, 64,
                         2))
      return LOZA_ERR_CUDA;
    return launch_prefill_mla(mp, workspace, st);
  }
  if (dvt == 256 && n_kv_heads == 1 && n_heads % 2 == 0) {
    // absorbed MLA: two heads share every key block, so pairs of CTAs split the B operands
    PrefillPairParams pp;
    std::memset(&pp, 0, sizeof(pp));
    pp.cu_seqlens = cu_seqlens;
    pp.out = prm.out;
    pp.lse = lse;
    pp.n_heads = n_heads;
    pp.n_qtiles = (max_seqlen + kTile - 1) / kTile;
    if ((int64_t)batch * pp.n_qtiles * n_heads > INT32_MAX) return LOZA_ERR_UNSUPPORTED;
    pp.total_tiles = batch * pp.n_qtiles * n_heads;
    pp.n_sink = prm.n_sink;
    pp.n_local = prm.n_local;
    pp.block = prm.block;
    pp.scale_log2 = prm.scale_log2;
    if (!make_map_3d(&pp.tm_q, q, d_qk, n_heads, total_tokens, d_qk, q_row_stride) ||
        !make_map_3d(&pp.tm_k, k, d_qk, 1, total_tokens, d_qk, k_row_stride, 64) ||
        !make_map_3d(&pp.tm_v, v, d_v, 1, total_tokens, v_head_stride, v_row_stride))
      return LOZA_ERR_CUDA;
    return launch_prefill_pair(pp, max_seqlen, batch, st);
  }
  if (!make_map_3d(&prm.tm_q, q, d_qk, n_heads, total_tokens, d_qk, q_row_stride) ||
      !make_map_3d(&prm.tm_k, k, d_qk, n_kv_heads, total_tokens, d_qk, k_row_stride) ||
      !make_map_3d(&prm.tm_v, v, d_v, n_kv_heads, total_tokens, v_head_stride, v_row_stride))
    return LOZA_ERR_CUDA;

  switch (dvt) {
    case 64: return launch_prefill<64, 64, 8>(prm, max_seqlen, batch, st);
    case 128:
      // the two-tile kernel's union walk assumes blocks of 128 tokens
      return p.block_size == kTile ? launch_prefill_mha2(prm, max_seqlen, batch, st)
                                   : launch_prefill<192, 128, 8>(prm, max_seqlen, batch, st);
    default: return launch_prefill<576, 256, 5>(prm, max_seqlen, batch, st);
  }
}

loza_status loza_ssa_prefill_host(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                                  int32_t batch, int64_t total_tokens, int32_t max_seqlen, int32_t n_heads,
                                  int32_t n_kv_heads, int32_t d_qk, int32_t d_v, loza_ssa_params p, void* out,
                                  float* lse, void* workspace, size_t workspace_bytes, loza_stream_t stream) {
  if (!q || !k || !v || !cu_seqlens || !out || !lse) return LOZA_ERR_INVALID_ARG;
  if (batch < 1 || total_tokens < 1 || total_tokens > INT32_MAX || max_seqlen < 1 || max_seqlen > total_tokens)
    return LOZA_ERR_INVALID_ARG;
  // cu_seqlens is host memory: {0, ..., total_tokens}, non-decreasing, no sequence longer than max_seqlen
  if (cu_seqlens[0] != 0 || cu_seqlens[batch] != total_tokens) return LOZA_ERR_INVALID_ARG;
  for (int32_t n = 0; n < batch; ++n)
    if (cu_seqlens[n + 1] < cu_seqlens[n] || cu_seqlens[n + 1] - cu_seqlens[n] > max_seqlen)
      return LOZA_ERR_INVALID_ARG;
  if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads != 0) return LOZA_ERR_INVALID_ARG;
  if (!window_ok(p) || !host_shape_ok(n_heads, n_kv_heads, d_qk, d_v)) return LOZA_ERR_UNSUPPORTED;
  const bool latent_v = (v == k);
  if (latent_v && d_v > d_qk) return LOZA_ERR_INVALID_ARG;
  const size_t need = loza_ssa_workspace_size(LOZA_OP_PREFILL_HOST, batch, total_tokens, max_seqlen, n_heads,
                                              n_kv_heads, d_qk, d_v, p);
  if (need == 0) return LOZA_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LOZA_ERR_INVALID_ARG;
  if (workspace_bytes < need) return LOZA_ERR_WORKSPACE;

  // every chunk of every sequence, in order
  struct Work {
    int64_t row0;  // the sequence's first packed row
    HostChunk ck;
  };
  std::vector<Work> work;
  for (int32_t n = 0; n < batch; ++n) {
    const int64_t L = cu_seqlens[n + 1] - cu_seqlens[n];
    if (L == 0) continue;
    const HostChunkPlan hn = host_chunk_plan(L, p);
    for (int64_t c = 0; c < hn.n_chunks; ++c) work.push_back({(int64_t)cu_seqlens[n], host_chunk(hn, c, L, p)});
  }
  const HostChunkPlan h = host_chunk_plan(max_seqlen, p);
  const int64_t cap = host_chunk_cap(batch, total_tokens);
  if ((int64_t)work.size() > cap) return LOZA_ERR_UNSUPPORTED;  // cannot happen: the cap bounds every plan

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LOZA_ERR_CUDA;
  HostPipe& hp = g_host_pipes[dev];
  std::lock_guard<std::mutex> lock(hp.mu);
  if (!host_pipe_init(hp)) return LOZA_ERR_CUDA;

  const size_t pf = loza_ssa_workspace_size(LOZA_OP_PREFILL, 1, h.rows_max, (int32_t)h.rows_max, n_heads,
                                            n_kv_heads, d_qk, d_v, p);
  const HostLayout w = host_layout(h, cap, pf, n_heads, n_kv_heads, d_qk, d_v);
  const int slots = (int)std::min<int64_t>(w.slots, (int64_t)work.size());
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t q_row = (size_t)n_heads * d_qk * 2, k_row = (size_t)n_kv_heads * d_qk * 2;
  const size_t v_row = (size_t)n_kv_heads * d_v * 2, o_row = (size_t)n_heads * d_v * 2;
  const size_t l_row = (size_t)n_heads * sizeof(float);
  const uint8_t* qh = static_cast<const uint8_t*>(q);
  const uint8_t* kh = static_cast<const uint8_t*>(k);
  const uint8_t* vh = static_cast<const uint8_t*>(v);
  uint8_t* oh = static_cast<uint8_t*>(out);
  uint8_t* lh = reinterpret_cast<uint8_t*>(lse);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (work.empty()) return LOZA_OK;  // only empty sequences
#define LOZA_CU(x) \
  do {                                  \
    if ((x) != cudaSuccess) return LOZA_ERR_CUDA; \
  } while (0)

  // the local cu_seqlens {0, local length} of every chunk, staged from pageable memory
  std::vector<int32_t> cu(work.size() * 2);
  for (size_t g = 0; g < work.size(); ++g) {
    cu[2 * g] = 0;
    cu[2 * g + 1] = (int32_t)work[g].ck.local_len();
  }
  // the copy streams start after the caller's earlier work on `stream`
  LOZA_CU(cudaEventRecord(hp.start, st));
  LOZA_CU(cudaStreamWaitEvent(hp.h2d, hp.start, 0));
  LOZA_CU(cudaStreamWaitEvent(hp.d2h, hp.start, 0));
  int32_t* cu_dev = reinterpret_cast<int32_t*>(ws + w.cu_off);
  LOZA_CU(cudaMemcpyAsync(cu_dev, cu.data(), cu.size() * sizeof(int32_t), cudaMemcpyHostToDevice, hp.h2d));

  for (size_t g = 0; g < work.size(); ++g) {
    const int sl = (int)(g % slots);
    const HostChunk& ck = work[g].ck;
    const int64_t r0 = work[g].row0;  // sequence-relative rows + r0 = packed rows
    uint8_t* slot = ws + w.slot_off + (size_t)sl * w.slot_bytes;
    uint8_t* qd = slot + w.q_off;
    uint8_t* kd = slot + w.k_off;
    uint8_t* vd = latent_v ? kd : slot + w.v_off;
    uint8_t* od = slot + w.o_off;
    float* ld = reinterpret_cast<float*>(slot + w.l_off);
    const int64_t pre_rows = ck.pre, own = ck.q1 - ck.q0;

    // copy in: the slot's inputs are free once the chunk that used them ran
    if (g >= (size_t)slots) LOZA_CU(cudaStreamWaitEvent(hp.h2d, hp.run_done[sl], 0));
    if (pre_rows > 0) LOZA_CU(cudaMemsetAsync(qd, 0, (size_t)pre_rows * q_row, hp.h2d));
    LOZA_CU(cudaMemcpyAsync(qd + (size_t)pre_rows * q_row, qh + (size_t)(r0 + ck.q0) * q_row, (size_t)own * q_row,
                            cudaMemcpyDefault, hp.h2d));
    // K (and V) rows: run 0, the gap as zero rows (read with the tiles around it
    // and masked, so they must be finite), run 1
    const int64_t at1 = ck.n0 + ck.gap;
    LOZA_CU(cudaMemcpyAsync(kd, kh + (size_t)(r0 + ck.src0) * k_row, (size_t)ck.n0 * k_row, cudaMemcpyDefault,
                            hp.h2d));
    if (ck.gap > 0) LOZA_CU(cudaMemsetAsync(kd + (size_t)ck.n0 * k_row, 0, (size_t)ck.gap * k_row, hp.h2d));
    if (ck.n1 > 0)
      LOZA_CU(cudaMemcpyAsync(kd + (size_t)at1 * k_row, kh + (size_t)(r0 + ck.src1) * k_row, (size_t)ck.n1 * k_row,
                              cudaMemcpyDefault, hp.h2d));
    if (!latent_v) {
      LOZA_CU(cudaMemcpyAsync(vd, vh + (size_t)(r0 + ck.src0) * v_row, (size_t)ck.n0 * v_row, cudaMemcpyDefault,
                              hp.h2d));
      if (ck.gap > 0) LOZA_CU(cudaMemsetAsync(vd + (size_t)ck.n0 * v_row, 0, (size_t)ck.gap * v_row, hp.h2d));
      if (ck.n1 > 0)
        LOZA_CU(cudaMemcpyAsync(vd + (size_t)at1 * v_row, vh + (size_t)(r0 + ck.src1) * v_row,
                                (size_t)ck.n1 * v_row, cudaMemcpyDefault, hp.h2d));
    }
    LOZA_CU(cudaEventRecord(hp.in_done[sl], hp.h2d));

    // compute on the caller's stream: the slot's outputs are free once copied out
    LOZA_CU(cudaStreamWaitEvent(st, hp.in_done[sl], 0));
    if (g >= (size_t)slots) LOZA_CU(cudaStreamWaitEvent(st, hp.out_done[sl], 0));
    const int32_t len = (int32_t)ck.local_len();
    const loza_status rc = loza_ssa_prefill(
        qd, kd, vd, cu_dev + 2 * g, 1, len, len, n_heads, n_kv_heads, d_qk, d_v, (int64_t)n_heads * d_qk,
        (int64_t)n_kv_heads * d_qk, latent_v ? (int64_t)n_kv_heads * d_qk : (int64_t)n_kv_heads * d_v, p, od, ld,
        pf > 0 ? ws + w.pf_off : nullptr, pf, stream);
    if (rc != LOZA_OK) return rc;
    LOZA_CU(cudaEventRecord(hp.run_done[sl], st));

    // copy out the own rows
    LOZA_CU(cudaStreamWaitEvent(hp.d2h, hp.run_done[sl], 0));
    LOZA_CU(cudaMemcpyAsync(oh + (size_t)(r0 + ck.q0) * o_row, od + (size_t)pre_rows * o_row, (size_t)own * o_row,
                            cudaMemcpyDefault, hp.d2h));
    LOZA_CU(cudaMemcpyAsync(lh + (size_t)(r0 + ck.q0) * l_row,
                            reinterpret_cast<uint8_t*>(ld) + (size_t)pre_rows * l_row, (size_t)own * l_row,
                            cudaMemcpyDefault, hp.d2h));
    LOZA_CU(cudaEventRecord(hp.out_done[sl], hp.d2h));
  }
  // the caller's stream completes when the last rows have reached the host
  LOZA_CU(cudaStreamWaitEvent(st, hp.out_done[(work.size() - 1) % slots], 0));
#undef LOZA_CU
  return LOZA_OK;
}

loza_status loza_ssa_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                            int32_t batch, int32_t max_seqlen, int64_t cache_batch_stride,
                            int64_t cache_row_stride, int32_t n_heads, int32_t n_kv_heads, int32_t d_qk,
                            int32_t d_v, loza_ssa_params p, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, loza_stream_t stream) {
  if (!q || !k_cache || !seqlens || !out || !lse) return LOZA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(out) || (v_cache && !aligned16(v_cache)))
    return LOZA_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || max_seqlen < 1) return LOZA_ERR_INVALID_ARG;
  if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads != 0) return LOZA_ERR_INVALID_ARG;
  if (!stride_ok(cache_row_stride) || !stride_ok(cache_batch_stride) ||
      cache_batch_stride < (int64_t)max_seqlen * cache_row_stride || cache_row_stride < (int64_t)n_kv_heads * d_qk)
    return LOZA_ERR_INVALID_ARG;
  if (!window_ok(p)) return LOZA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int n_sink = p.n_local == LOZA_UNBOUNDED ? 0 : p.n_sink;
  const int n_local = p.n_local == LOZA_UNBOUNDED ? -1 : p.n_local;
  const float scale_log2 = p.scale * 1.4426950408889634f;

  if (n_kv_heads == 1 && d_qk == 576 && d_v == 512) {
    // absorbed MLA: shared latent cache, V = first 512 columns
    DecodeParams prm;
    DecodePlan plan;
    const loza_status rc = setup_decode_mla(q, k_cache, v_cache, seqlens, batch, max_seqlen, cache_batch_stride,
                                            cache_row_stride, n_heads, p, out, lse, &prm, &plan);
    if (rc != LOZA_OK) return rc;
    const DecodeWorkspace wl = decode_workspace(batch, plan);
    if (wl.total > 0) {
      if (!workspace || !aligned16(workspace)) return LOZA_ERR_INVALID_ARG;
      if (workspace_bytes < wl.total) return LOZA_ERR_WORKSPACE;
    }
    return launch_decode_mla(prm, plan, batch, static_cast<uint8_t*>(workspace), st);
  }

  // per-head K/V on CUDA cores
  if (!(n_kv_heads == n_heads || n_kv_heads == 1)) return LOZA_ERR_UNSUPPORTED;
  if (!v_cache) return LOZA_ERR_INVALID_ARG;
  if (n_heads > 65535) return LOZA_ERR_UNSUPPORTED;
  DecodeMhaParams prm;
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.k = static_cast<const __nv_bfloat16*>(k_cache);
  prm.v = static_cast<const __nv_bfloat16*>(v_cache);
  prm.k_batch_stride = cache_batch_stride;
  prm.k_row_stride = cache_row_stride;
  prm.v_batch_stride = cache_batch_stride / d_qk * d_v;
  prm.v_row_stride = cache_row_stride / d_qk * d_v;
  prm.seqlens = seqlens;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.n_heads = n_heads;
  prm.n_kv_heads = n_kv_heads;
  prm.n_sink = n_sink;
  prm.n_local = n_local;
  prm.block = p.block_size;
  prm.scale_log2 = scale_log2;
  if (cache_batch_stride % d_qk != 0 || cache_row_stride % d_qk != 0) return LOZA_ERR_INVALID_ARG;
  const dim3 grid(n_heads, batch);
  if (d_qk == 64 && d_v == 64) ssa_decode_mha_kernel<64, 64><<<grid, 128, 0, st>>>(prm);
  else if (d_qk == 192 && d_v == 128) ssa_decode_mha_kernel<192, 128><<<grid, 128, 0, st>>>(prm);
  else return LOZA_ERR_UNSUPPORTED;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? LOZA_OK : LOZA_ERR_CUDA;
}

loza_status loza_ssa_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                              const float* lse, const int32_t* cu_seqlens, int32_t batch, int64_t total_tokens,
                              int32_t max_seqlen, int32_t n_heads, int32_t n_kv_heads, int32_t d_qk,
                              int32_t d_v, loza_ssa_params p, void* dq, void* dk, void* dv, void* workspace,
                              size_t workspace_bytes, loza_stream_t stream) {
  if (!q || !k || !v || !out || !dout || !lse || !cu_seqlens || !dq || !dk || !dv) return LOZA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv))
    return LOZA_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || total_tokens < 1 || total_tokens > INT32_MAX || max_seqlen < 1 ||
      max_seqlen > total_tokens)
    return LOZA_ERR_INVALID_ARG;
  if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads != 0) return LOZA_ERR_INVALID_ARG;
  if (!window_ok(p)) return LOZA_ERR_UNSUPPORTED;
  if (p.n_local == LOZA_UNBOUNDED) return LOZA_ERR_UNSUPPORTED;
  const int sink_tiles = bwd_sink_tiles(p);
  if (n_kv_heads != n_heads || n_heads > 65535 / std::max(sink_tiles, 1)) return LOZA_ERR_UNSUPPORTED;
  const bool d64 = (d_qk == 64 && d_v == 64), d192 = (d_qk == 192 && d_v == 128);
  if (!d64 && !d192) return LOZA_ERR_UNSUPPORTED;
  const BwdWorkspace wl = bwd_workspace(batch, total_tokens, max_seqlen, n_heads, d_qk, d_v, p);
  if (!workspace || !aligned16(workspace)) return LOZA_ERR_INVALID_ARG;
  if (workspace_bytes < wl.total) return LOZA_ERR_WORKSPACE;

  BwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  const int64_t T = total_tokens;
  if (!make_map_3d(&prm.tm_q, q, d_qk, n_heads, T, d_qk, (int64_t)n_heads * d_qk) ||
      !make_map_3d(&prm.tm_k, k, d_qk, n_heads, T, d_qk, (int64_t)n_heads * d_qk) ||
      !make_map_3d(&prm.tm_v, v, d_v, n_heads, T, d_v, (int64_t)n_heads * d_v) ||
      !make_map_3d(&prm.tm_do, dout, d_v, n_heads, T, d_v, (int64_t)n_heads * d_v))
    return LOZA_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  prm.cu_seqlens = cu_seqlens;
  prm.lse = lse;
  prm.dvec = reinterpret_cast<float*>(ws + wl.d_off);
  prm.dq = static_cast<__nv_bfloat16*>(dq);
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.partial = reinterpret_cast<float*>(ws + wl.part_off);
  prm.n_heads = n_heads;
  prm.n_sink = p.n_sink;
  prm.n_local = p.n_local;
  prm.block = p.block_size;
  prm.sink_end = p.n_sink * p.block_size;
  prm.n_sink_tiles = sink_tiles;
  prm.nslots = wl.nslots;
  prm.scale = p.scale;
  prm.scale_log2 = p.scale * 1.4426950408889634f;
  const int nq_max = (max_seqlen + kTile - 1) / kTile;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d64) return launch_backward<64, 64>(prm, out, dout, T * n_heads, nq_max, batch, st);
  return launch_backward<192, 128>(prm, out, dout, T * n_heads, nq_max, batch, st);
}

loza_status loza_hi_page_keys(const void* k_index, int64_t index_batch_stride, int64_t index_row_stride,
                              const int32_t* seqlens, int32_t batch, int32_t max_seqlen, int32_t d_index,
                              float* page_keys, loza_stream_t stream) {
  if (!seqlens || !page_keys) return LOZA_ERR_INVALID_ARG;
  if (!hi_args_ok(k_index, index_batch_stride, index_row_stride, batch, max_seqlen, d_index))
    return LOZA_ERR_INVALID_ARG;
  const int64_t pages = max_seqlen / kHiPage;
  if (pages < 1) return LOZA_OK;
  hi_page_keys_kernel<<<dim3((unsigned)((pages + 31) / 32), d_index / 64, batch), 256, 0,
                        reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<const __nv_bfloat16*>(k_index),
                                                                  index_batch_stride, index_row_stride, seqlens,
                                                                  d_index, pages, page_keys);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? LOZA_OK : LOZA_ERR_CUDA;
}

size_t loza_hi_workspace_size(int32_t batch, int32_t max_seqlen, int32_t top_pages, int32_t top_k,
                              loza_ssa_params p) {
  if (batch < 1 || batch > 65535 || max_seqlen < 1 || top_pages < 1 || top_k < 0 || top_k > kHiMaxTopK ||
      !hi_window_ok(p))
    return 0;
  return hi_workspace(batch, max_seqlen, top_pages, top_k, p).total;
}

}  // extern "C"

namespace loza {
namespace {
// Enqueue the selection (validated by the caller) into `selected`.
loza_status hi_select_launch(const void* q_index, const void* k_index, int64_t index_batch_stride,
                             int64_t index_row_stride, const float* page_keys, const int32_t* seqlens,
                             int32_t batch, int32_t max_seqlen, int32_t d_index, const loza_ssa_params& p,
                             int32_t top_pages, int32_t top_k, int32_t* selected, uint8_t* ws, const HiWorkspace& w,
                             cudaStream_t st) {
  HiParams hp;
  std::memset(&hp, 0, sizeof(hp));
  if (!make_map_index(&hp.tm_index, k_index, d_index, max_seqlen, batch, index_row_stride, index_batch_stride))
    return LOZA_ERR_CUDA;
  hp.q_index = static_cast<const __nv_bfloat16*>(q_index);
  hp.page_keys = page_keys;
  hp.pages_per_seq = max_seqlen / kHiPage;
  hp.seqlens = seqlens;
  hp.batch = batch;
  hp.d = d_index;
  hp.block = p.block_size;
  hp.n_sink = p.n_local == LOZA_UNBOUNDED ? 0 : p.n_sink;
  hp.n_local = p.n_local == LOZA_UNBOUNDED ? -1 : p.n_local;
  hp.top_pages = top_pages;
  hp.top_k = top_k;
  hp.page_scored = reinterpret_cast<unsigned long long*>(ws + w.page_scored);
  hp.sel_pages = reinterpret_cast<int32_t*>(ws + w.sel_pages);
  hp.n_pages = reinterpret_cast<int32_t*>(ws + w.n_pages);
  hp.page_hist = reinterpret_cast<int32_t*>(ws + w.page_hist);
  hp.hist1 = reinterpret_cast<int32_t*>(ws + w.hist1);
  hp.counters = reinterpret_cast<int32_t*>(ws + w.counters);
  hp.page_cand = reinterpret_cast<unsigned long long*>(ws + w.page_cand);
  hp.tok_keys = reinterpret_cast<unsigned long long*>(ws + w.tok_keys);
  hp.tok_cand = reinterpret_cast<unsigned long long*>(ws + w.tok_cand);
  hp.selected = selected;
  hp.n_sel = reinterpret_cast<int32_t*>(ws + w.n_sel);
  if (cudaFuncSetAttribute(hi_tokens_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           HiTokLayout::SMEM_ALLOC) != cudaSuccess ||
      cudaFuncSetAttribute(hi_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           HiTopkLayout::bytes(hp.pages_per_seq)) != cudaSuccess)
    return LOZA_ERR_CUDA;
  if (cudaMemsetAsync(ws + w.zeroed, 0, w.zeroed_bytes, st) != cudaSuccess) return LOZA_ERR_CUDA;
  int launches = 4;
  if (hp.pages_per_seq >= 1) {
    hi_page_scores_kernel<<<dim3((unsigned)((hp.pages_per_seq + 255) / 256), batch), 256, 0, st>>>(hp);
    ++launches;
  }
  // each kernel after the first waits (griddep_wait) for the one before it
  const int64_t items = (int64_t)batch * ((top_pages + kHiTokPages - 1) / kHiTokPages);
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(items, 3 * (int64_t)sm_count()));
  const int64_t slices = ((int64_t)top_pages * kHiPage + kHiCollectKeys - 1) / kHiCollectKeys;
  const bool chained = hp.pages_per_seq >= 1;  // page selection follows the page scores
  auto launch = [&](auto kernel, dim3 g, dim3 b, size_t sm, bool after) {
    if (after) return launch_after(kernel, g, b, sm, st, hp);
    kernel<<<g, b, sm, st>>>(hp);
    return cudaGetLastError();
  };
  if (launch(hi_page_select_kernel, dim3(batch), dim3(1024), 0, chained) != cudaSuccess ||
      launch(hi_tokens_kernel, dim3(grid), dim3(kHiTokThreads), HiTokLayout::SMEM_ALLOC, true) != cudaSuccess ||
      launch(hi_topk_collect_kernel, dim3((unsigned)slices, batch), dim3(256), 0, true) != cudaSuccess ||
      launch(hi_topk_kernel, dim3(batch), dim3(1024), HiTopkLayout::bytes(hp.pages_per_seq), true) != cudaSuccess)
    return LOZA_ERR_CUDA;
  g_launches.fetch_add(launches, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? LOZA_OK : LOZA_ERR_CUDA;
}

// Validate the attention part of loza_ssa_decode_selected / loza_hi_decode and
// prepare its decode: over the packed rows (bounded window) or over the cache
// itself (unbounded window: the selection adds no token).
loza_status hi_attend_setup(const void* q, const void* kv_cache, int64_t cache_batch_stride,
                            int64_t cache_row_stride, const int32_t* seqlens, int32_t batch, int32_t max_seqlen,
                            const loza_ssa_params& p, void* out, float* lse, uint8_t* ws, const HiWorkspace& w,
                            DecodeParams* prm, DecodePlan* plan) {
  // the cache and the outputs, as loza_ssa_decode checks them
  loza_status rc = setup_decode_mla(q, kv_cache, nullptr, seqlens, batch, max_seqlen, cache_batch_stride,
                                    cache_row_stride, kDecHeads, p, out, lse, prm, plan);
  if (rc != LOZA_OK || w.cap_rows == 0) return rc;
  return setup_decode_mla(q, ws + w.packed, nullptr, reinterpret_cast<const int32_t*>(ws + w.counts), batch,
                          w.cap_rows, (int64_t)w.cap_rows * 576, 576, kDecHeads, hi_packed_params(p.scale), out,
                          lse, prm, plan);
}

// Pack the window and the selection (list: compact, n_sel entries per
// sequence) and run the decode prepared by hi_attend_setup.
loza_status hi_attend_launch(const void* kv_cache, int64_t cache_batch_stride, int64_t cache_row_stride,
                             const int32_t* seqlens, int32_t batch, const loza_ssa_params& p, const int32_t* list,
                             int32_t top_k, uint8_t* ws, const HiWorkspace& w, DecodeParams& prm,
                             const DecodePlan& plan, cudaStream_t st) {
  if (w.cap_rows > 0) {
    const SsaWindow win{p.block_size, p.n_sink * p.block_size, p.n_local};
    // after the selection or the compaction of a caller's list
    if (launch_after(hi_gather_kernel, dim3(w.cap_rows / 32, batch), dim3(256), 0, st,
                     static_cast<const __nv_bfloat16*>(kv_cache), cache_batch_stride, cache_row_stride, seqlens, win,
                     list, std::max(top_k, 1), reinterpret_cast<const int32_t*>(ws + w.n_sel), w.cap_rows,
                     reinterpret_cast<__nv_bfloat16*>(ws + w.packed),
                     reinterpret_cast<int32_t*>(ws + w.counts)) != cudaSuccess)
      return LOZA_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return launch_decode_mla(prm, plan, batch, ws + w.dec, st, /*after=*/true);
  }
  return launch_decode_mla(prm, plan, batch, ws + w.dec, st);
}
}  // namespace
}  // namespace loza

extern "C" {

loza_status loza_hi_select(const void* q_index, const void* k_index, int64_t index_batch_stride,
                           int64_t index_row_stride, const float* page_keys, const int32_t* seqlens, int32_t batch,
                           int32_t max_seqlen, int32_t d_index, loza_ssa_params p, int32_t top_pages, int32_t top_k,
                           int32_t* selected, void* workspace, size_t workspace_bytes, loza_stream_t stream) {
  if (!q_index || !page_keys || !seqlens || !selected || !aligned16(q_index)) return LOZA_ERR_INVALID_ARG;
  if (!hi_args_ok(k_index, index_batch_stride, index_row_stride, batch, max_seqlen, d_index))
    return LOZA_ERR_INVALID_ARG;
  if (top_pages < 1 || top_k < 1 || top_k > kHiMaxTopK) return LOZA_ERR_INVALID_ARG;
  if (!hi_window_ok(p) || max_seqlen / kHiPage > kHiMaxPages) return LOZA_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LOZA_ERR_INVALID_ARG;
  const HiWorkspace w = hi_workspace(batch, max_seqlen, top_pages, top_k, p);
  if (workspace_bytes < w.total) return LOZA_ERR_WORKSPACE;
  return hi_select_launch(q_index, k_index, index_batch_stride, index_row_stride, page_keys, seqlens, batch,
                          max_seqlen, d_index, p, top_pages, top_k, selected, static_cast<uint8_t*>(workspace), w,
                          reinterpret_cast<cudaStream_t>(stream));
}

loza_status loza_ssa_decode_selected(const void* q, const void* kv_cache, int64_t cache_batch_stride,
                                     int64_t cache_row_stride, const int32_t* seqlens, int32_t batch,
                                     int32_t max_seqlen, loza_ssa_params p, const int32_t* selected, int32_t top_k,
                                     void* out, float* lse, void* workspace, size_t workspace_bytes,
                                     loza_stream_t stream) {
  if (top_k < 0 || top_k > kHiMaxTopK || (top_k > 0 && !selected)) return LOZA_ERR_INVALID_ARG;
  if (!hi_window_ok(p)) return LOZA_ERR_UNSUPPORTED;
  if (batch < 1 || batch > 65535 || max_seqlen < 1) return LOZA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LOZA_ERR_INVALID_ARG;
  const HiWorkspace w = hi_workspace(batch, max_seqlen, 1, top_k, p);
  if (workspace_bytes < w.total) return LOZA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeParams prm;
  DecodePlan plan;
  loza_status rc = hi_attend_setup(q, kv_cache, cache_batch_stride, cache_row_stride, seqlens, batch, max_seqlen,
                                   p, out, lse, ws, w, &prm, &plan);
  if (rc != LOZA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t* list = reinterpret_cast<int32_t*>(ws + w.selected);
  if (w.cap_rows > 0) {
    const SsaWindow win{p.block_size, p.n_sink * p.block_size, p.n_local};
    hi_compact_kernel<<<batch, 1024, 0, st>>>(selected, top_k, seqlens, win, list,
                                               reinterpret_cast<int32_t*>(ws + w.n_sel));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (cudaGetLastError() != cudaSuccess) return LOZA_ERR_CUDA;
  }
  return hi_attend_launch(kv_cache, cache_batch_stride, cache_row_stride, seqlens, batch, p, list, top_k, ws, w,
                          prm, plan, st);
}

loza_status loza_hi_decode(const void* q, const void* kv_cache, int64_t cache_batch_stride, int64_t cache_row_stride,
                           const void* q_index, const void* k_index, int64_t index_batch_stride,
                           int64_t index_row_stride, const float* page_keys, const int32_t* seqlens, int32_t batch,
                           int32_t max_seqlen, int32_t d_index, loza_ssa_params p, int32_t top_pages, int32_t top_k,
                           void* out, float* lse, void* workspace, size_t workspace_bytes, loza_stream_t stream) {
  if (!q_index || !page_keys || !seqlens || !aligned16(q_index)) return LOZA_ERR_INVALID_ARG;
  if (!hi_args_ok(k_index, index_batch_stride, index_row_stride, batch, max_seqlen, d_index))
    return LOZA_ERR_INVALID_ARG;
  if (top_pages < 1 || top_k < 1 || top_k > kHiMaxTopK) return LOZA_ERR_INVALID_ARG;
  if (max_seqlen / kHiPage > kHiMaxPages || !hi_window_ok(p)) return LOZA_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LOZA_ERR_INVALID_ARG;
  const HiWorkspace w = hi_workspace(batch, max_seqlen, top_pages, top_k, p);
  if (workspace_bytes < w.total) return LOZA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeParams prm;
  DecodePlan plan;
  loza_status rc = hi_attend_setup(q, kv_cache, cache_batch_stride, cache_row_stride, seqlens, batch, max_seqlen,
                                   p, out, lse, ws, w, &prm, &plan);
  if (rc != LOZA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t* sel = reinterpret_cast<int32_t*>(ws + w.selected);
  if (w.cap_rows > 0) {  // an unbounded window leaves no token to select
    rc = hi_select_launch(q_index, k_index, index_batch_stride, index_row_stride, page_keys, seqlens, batch,
                          max_seqlen, d_index, p, top_pages, top_k, sel, ws, w, st);
    if (rc != LOZA_OK) return rc;
  }
  return hi_attend_launch(kv_cache, cache_batch_stride, cache_row_stride, seqlens, batch, p, sel, top_k, ws, w, prm,
                          plan, st);
}

loza_status loza_ssa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                    const int32_t* seqlens, int32_t batch, int32_t max_seqlen,
                                    int64_t cache_batch_stride, int64_t cache_row_stride, int32_t n_heads,
                                    int32_t n_kv_heads, int32_t d_qk, int32_t d_v, loza_ssa_params p, void* out,
                                    float* lse, loza_stream_t stream) {
  // Per-head K/V decode needs no scratch at all: same call, no workspace.
  if (!(n_kv_heads == 1 && d_qk == 576 && d_v == 512))
    return loza_ssa_decode(q, k_cache, v_cache, seqlens, batch, max_seqlen, cache_batch_stride, cache_row_stride,
                           n_heads, n_kv_heads, d_qk, d_v, p, out, lse, nullptr, 0, stream);
  // batch too large for the built-in scratch: refuse before touching the driver
  if (batch >= 1 && max_seqlen >= 1 && window_ok(p) &&
      decode_workspace(batch, decode_plan(p, max_seqlen, batch)).total > kNoAllocScratchBytes)
    return LOZA_ERR_WORKSPACE;
  DecodeParams prm;
  DecodePlan plan;
  const loza_status rc = setup_decode_mla(q, k_cache, v_cache, seqlens, batch, max_seqlen, cache_batch_stride,
                                          cache_row_stride, n_heads, p, out, lse, &prm, &plan);
  if (rc != LOZA_OK) return rc;
  const DecodeWorkspace wl = decode_workspace(batch, plan);
  uint8_t* ws = nullptr;
  if (wl.total > 0) {
    ws = static_cast<uint8_t*>(decode_scratch_address());
    if (!ws) return LOZA_ERR_CUDA;
  }
  return launch_decode_mla(prm, plan, batch, ws, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
