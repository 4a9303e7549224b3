// hi_index.cuh - hierarchical index for the decode, and the gather that feeds
// the attention over the window and the selected tokens.
//
// Page 4 of the LoZA pages ("LongCat Sparse Attention: Taming the Lightning
// via Streaming-aware Hierarchical Cross-Layer Indexing") splits a decode
// query's attention budget into fixed sink and window tokens (the SSA window
// of this library) and dynamically selected tokens, chosen by a hierarchical
// index in two stages: a coarse pass over pages of 128 tokens recalls the top
// pages, then only the tokens of those pages are scored and the best kept.
//
// Readings (the pages give no scoring function): the index score of a key is
// the dot product of the sequence's index query with the key's index key
// (both supplied by the caller); a page is represented by the mean of its 128
// index keys; only whole pages that hold a token outside the fixed window are
// candidates, and only tokens outside it are selected, so the parts are
// disjoint; ties go to the lower page or token index. The scores decide a
// selection, so they are formed in one fixed order: fp32 fused multiply-adds
// over the index dimension in order (page means: fp32 sums in token order,
// times 1/128); the result is a unique set.
//
// A (score, index) pair is one 64-bit key (larger score first, then lower
// index), so every selection is "the k largest keys", found by radix select
// on 11-bit digits. Kernels, in the order a decode runs them:
//   hi_page_keys_kernel     mean index key of every whole page (maintained as
//                           the cache fills; not part of a decode step)
//   hi_page_scores_kernel   a thread per page: its key (0 for a non-candidate)
//   hi_page_select_kernel   a CTA per sequence: the top pages (radix select)
//   hi_tokens_kernel        persistent; the index keys of the recalled pages
//                           arrive by TMA in 128-row x 64-column tiles and a
//                           thread per token forms its score; writes the keys
//                           and a histogram of their top digit per sequence
//   hi_topk_kernel          a CTA per sequence: the top_k tokens, starting
//                           from that histogram; sorted by position
//   hi_compact_kernel       (caller-given lists only) the valid entries
//   hi_gather_kernel        the latent rows of the window and the selection,
//                           packed per sequence for the tensor-core decode
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "prefill.cuh"
#include "sm100.cuh"

namespace loza {

constexpr int kHiPage = 128;        // tokens per page
constexpr int kHiMaxPages = 8192;   // pages per sequence (1,048,576 tokens)
constexpr int kHiMaxTopK = 2048;    // selected tokens per sequence at most
constexpr int kHiMaxDim = 512;      // index dimension at most
constexpr int kHiDimStep = 64;      // the index dimension is a multiple of this (one TMA column tile)
constexpr int kHiBits = 11;         // radix digit
constexpr int kHiBins = 1 << kHiBits;
constexpr int kHiTopShift = 64 - kHiBits;  // the first digit: bits 53..63
constexpr int kHiCand = 4096;       // keys sharing the threshold's first digit that the top-k sorts on chip

struct HiParams {
  CUtensorMap tm_index;           // index keys {d, rows, batch}, box {64, 128, 1}, 128-byte swizzle
  const __nv_bfloat16* q_index;   // [B, d]
  const float* page_keys;         // [B, d, pages_per_seq] (the page dimension innermost)
  int64_t pages_per_seq;
  const int32_t* seqlens;
  int batch, d;
  int block, n_sink, n_local;     // the fixed window (n_local < 0: unbounded)
  int top_pages, top_k;
  unsigned long long* page_scored;  // [B, pages_per_seq] page keys, 0 = not a candidate
  int32_t* sel_pages;             // [B, top_pages] recalled pages (any order)
  int32_t* n_pages;               // [B] recalled page count
  int32_t* hist1;                 // [B, kHiBins] top-digit histogram of the token keys
  unsigned long long* tok_keys;   // [B, top_pages * 128] token keys, 0 = none
  int32_t* selected;              // [B, top_k] selected tokens, ascending, then -1
  int32_t* n_sel;                 // [B] selected count
};

// (score, index) as one unsigned key: larger for a larger score, then for a
// smaller index. The score's bits are made monotone (negative values
// flipped); -0 is first turned into +0 so that equal scores compare equal.
// A real key is never 0 (its index half would have to be 2^32 - 1).
__device__ __forceinline__ unsigned long long hi_key(float s, int64_t index) {
  s = s + 0.0f;
  uint32_t u = __float_as_uint(s);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)index);
}
__device__ __forceinline__ uint32_t hi_key_index(unsigned long long key) {
  return 0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull);
}

// Whether token t, at or before the query i, lies outside the fixed window.
__device__ __forceinline__ bool hi_outside(const SsaWindow& w, int64_t t, int i) {
  return w.n_local >= 0 && t >= w.sink_end && t < w.lo(i);
}

__device__ __forceinline__ SsaWindow hi_window(const HiParams& p) {
  return SsaWindow{p.block, p.n_sink * p.block, p.n_local};
}

// Add 1 to hist[bin] for every lane with bin >= 0, one shared-memory atomic
// per distinct bin of the warp (scores crowd into few top digits). Whole warp.
__device__ __forceinline__ void hi_hist_add(int* hist, int bin) {
  const unsigned peers = __match_any_sync(0xffffffffu, bin);
  if (bin >= 0 && (threadIdx.x & 31) == (unsigned)(__ffs(peers) - 1)) atomicAdd(&hist[bin], __popc(peers));
}

// A slot in a shared list for every lane with `take`: one atomic per warp.
// Whole warp; returns the lane's slot (meaningless where !take).
__device__ __forceinline__ int hi_warp_slot(int* counter, bool take) {
  const unsigned m = __ballot_sync(0xffffffffu, take);
  const int lane = threadIdx.x & 31;
  const int leader = m ? __ffs(m) - 1 : 0;
  int base = 0;
  if (m && lane == leader) base = atomicAdd(counter, __popc(m));
  base = __shfl_sync(0xffffffffu, base, leader);
  return base + __popc(m & ((1u << lane) - 1u));
}

// Block-wide: the rank-th largest non-zero key of keys[0, N) among those
// equal to `prefix` on the bits `mask` already fixed, deciding the digits
// from bit `shift` down (1 <= rank <= that count). `hist` holds kHiBins
// ints, `sh` two ints.
__device__ unsigned long long hi_radix_kth(const unsigned long long* keys, int64_t N, int rank,
                                           unsigned long long prefix, unsigned long long mask, int shift, int* hist,
                                           int* sh) {
  const int64_t n_iter = (N + blockDim.x - 1) / blockDim.x * blockDim.x;  // warp-uniform trip count
  for (; shift > -kHiBits; shift -= kHiBits) {
    const int s0 = max(shift, 0);
    const int width = shift >= 0 ? kHiBits : kHiBits + shift;  // the last digit holds the remaining bits
    const unsigned long long dmask = ((1ull << width) - 1ull) << s0;
    for (int b = threadIdx.x; b < kHiBins; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    for (int64_t t = threadIdx.x; t < n_iter; t += blockDim.x) {
      const unsigned long long k = t < N ? keys[t] : 0ull;
      const bool in = k != 0ull && (k & mask) == prefix;
      hi_hist_add(hist, in ? (int)((k & dmask) >> s0) : -1);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // the digit holding the rank-th largest key, counted from the top: lane
      // j sums bins [64j, 64j + 64), a suffix scan over the lanes gives the
      // count above each lane's bins, and the lane where the rank falls scans
      const int lane = threadIdx.x;
      int own = 0;
      for (int b = 64 * lane; b < 64 * lane + 64; ++b) own += hist[b];
      int above = 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_down_sync(0xffffffffu, above + own, o);
        if (lane + o < 32) above += x;
      }
      if (above < rank && above + own >= rank) {
        int r = rank - above, dg = 64 * lane + 63;
        for (; dg > 64 * lane && hist[dg] < r; --dg) r -= hist[dg];
        sh[0] = r;
        sh[1] = dg;
      }
    }
    __syncthreads();
    rank = sh[0];
    prefix |= (unsigned long long)sh[1] << s0;
    mask |= dmask;
    __syncthreads();
  }
  return prefix;
}

// Bitonic sort of n (a power of two) keys in shared memory, largest first.
__device__ void hi_sort_desc(unsigned long long* keys, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < n; t += blockDim.x) {
        const int u = t ^ j;
        if (u > t) {
          const unsigned long long a = keys[t], b = keys[u];
          const bool desc = (t & k) == 0;
          if (desc ? a < b : a > b) {
            keys[t] = b;
            keys[u] = a;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Block-wide sum of one int per thread; `scratch` holds 33 ints.
__device__ __forceinline__ int hi_block_sum(int v, int* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x < 32) {
    int t = threadIdx.x < (blockDim.x >> 5) ? scratch[threadIdx.x] : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (threadIdx.x == 0) scratch[32] = t;
  }
  __syncthreads();
  const int r = scratch[32];
  __syncthreads();
  return r;
}

// ---------------------------------------------------------------------------
// Page keys: grid (ceil(pages / 32), d / 64, B), 256 threads. Thread (column
// c, page lane) sums its column over the 128 rows of a page in token order;
// a shared tile turns the [page][column] results into the [column][page]
// layout (pages innermost) that the page scoring reads coalesced.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) hi_page_keys_kernel(const __nv_bfloat16* __restrict__ k, int64_t batch_stride,
                                                           int64_t row_stride, const int32_t* __restrict__ seqlens,
                                                           int d, int64_t pages_per_seq, float* __restrict__ out) {
  __shared__ float tile[64][33];
  const int n = blockIdx.z;
  const int64_t full = min((int64_t)seqlens[n] / kHiPage, pages_per_seq);
  const int64_t pg0 = (int64_t)blockIdx.x * 32;
  const int c0 = blockIdx.y * 64;
  const int c = threadIdx.x & 63;
  for (int pp = threadIdx.x >> 6; pp < 32; pp += 4) {
    const int64_t pg = pg0 + pp;
    if (pg < full) {
      const __nv_bfloat16* col = k + n * batch_stride + pg * kHiPage * row_stride + c0 + c;
      float sum = 0.f;
#pragma unroll 16
      for (int r = 0; r < kHiPage; ++r) sum += __bfloat162float(col[r * row_stride]);
      tile[c][pp] = sum * (1.0f / kHiPage);
    }
  }
  __syncthreads();
  const int pp = threadIdx.x & 31;
  if (pg0 + pp < full)
    for (int cc = threadIdx.x >> 5; cc < 64; cc += 8)
      out[((int64_t)n * d + c0 + cc) * pages_per_seq + pg0 + pp] = tile[cc][pp];
}

// ---------------------------------------------------------------------------
// Page scores: grid (ceil(pages / 256), B), 256 threads, a thread per page.
// A page is a candidate if it is whole and meets [sink_end, lo(i)).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) hi_page_scores_kernel(const __grid_constant__ HiParams p) {
  __shared__ float q[kHiMaxDim];
  const int n = blockIdx.y;
  const int L = p.seqlens[n];
  const int i = L - 1;
  const SsaWindow w = hi_window(p);
  const int64_t full = min((int64_t)max(L, 0) / kHiPage, p.pages_per_seq);
  for (int c = threadIdx.x; c < p.d; c += blockDim.x) q[c] = __bfloat162float(p.q_index[(int64_t)n * p.d + c]);
  __syncthreads();
  const int64_t pg = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (pg >= p.pages_per_seq) return;
  unsigned long long key = 0;
  if (pg < full && w.n_local >= 0 && pg * kHiPage + kHiPage - 1 >= w.sink_end && pg * kHiPage < w.lo(i)) {
    const float* pk = p.page_keys + (int64_t)n * p.d * p.pages_per_seq + pg;
    float s = 0.f;
    for (int c = 0; c < p.d; ++c) s = __fmaf_rn(q[c], pk[(int64_t)c * p.pages_per_seq], s);
    key = hi_key(s, pg);
  }
  p.page_scored[(int64_t)n * p.pages_per_seq + pg] = key;
}

// ---------------------------------------------------------------------------
// Page selection: a CTA (1024 threads) per sequence. The top_pages largest
// page keys (all candidates if fewer); also clears the sequence's token-key
// histogram for the token stage.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) hi_page_select_kernel(const __grid_constant__ HiParams p) {
  __shared__ int hist[kHiBins];
  __shared__ int sh[34];
  __shared__ int n_out;
  const int n = blockIdx.x;
  for (int b = threadIdx.x; b < kHiBins; b += blockDim.x) p.hist1[(int64_t)n * kHiBins + b] = 0;
  const unsigned long long* keys = p.page_scored + (int64_t)n * p.pages_per_seq;
  const int64_t N = p.pages_per_seq;
  int v = 0;
  for (int64_t t = threadIdx.x; t < N; t += blockDim.x) v += keys[t] != 0ull;
  const int n_valid = hi_block_sum(v, sh);
  const int m = min(n_valid, p.top_pages);
  unsigned long long thr = 1ull;  // every real key is >= 1
  if (m > 0 && m < n_valid) thr = hi_radix_kth(keys, N, m, 0ull, 0ull, kHiTopShift, hist, sh);
  if (threadIdx.x == 0) n_out = 0;
  __syncthreads();
  if (m > 0) {
    const int64_t n_iter = (N + blockDim.x - 1) / blockDim.x * blockDim.x;
    for (int64_t t = threadIdx.x; t < n_iter; t += blockDim.x) {
      const unsigned long long k = t < N ? keys[t] : 0ull;
      const bool take = k != 0ull && k >= thr;
      const int slot = hi_warp_slot(&n_out, take);
      if (take && slot < p.top_pages) p.sel_pages[(int64_t)n * p.top_pages + slot] = (int32_t)hi_key_index(k);
    }
  }
  if (threadIdx.x == 0) p.n_pages[n] = m;
}

// ---------------------------------------------------------------------------
// Token scores: persistent CTAs, 4 consumer warps (a thread per token of a
// page) and 1 producer warp. Work item = up to kHiTokPages recalled pages of
// one sequence; unit = one page x 64 index columns, a 16 KB tile that TMA
// brings in (128-byte swizzle: 16-byte unit u of row r at unit u ^ (r & 7), so
// the 8 threads of a shared-memory phase, reading rows r..r+7 at the same
// logical unit, hit 8 different bank groups).
// ---------------------------------------------------------------------------
constexpr int kHiTokStages = 3;
constexpr int kHiTokPages = 8;
constexpr int kHiTokThreads = 160;
constexpr int kHiTokTile = kHiPage * 128;  // bytes of one unit
struct HiTokLayout {
  static constexpr int STAGE_OFF = 0;
  static constexpr int Q_OFF = kHiTokStages * kHiTokTile;
  static constexpr int HIST_OFF = Q_OFF + kHiMaxDim * 4;
  static constexpr int BAR_OFF = HIST_OFF + kHiBins * 4;  // full[S], empty[S]
  static constexpr int ABORT_OFF = BAR_OFF + 2 * kHiTokStages * 8;
  static constexpr int SMEM_BYTES = ABORT_OFF + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;  // room to align the tiles to 1 KB
};

__global__ void __launch_bounds__(kHiTokThreads) hi_tokens_kernel(const __grid_constant__ HiParams p) {
  using LY = HiTokLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* q = reinterpret_cast<float*>(smem + LY::Q_OFF);
  int* hist = reinterpret_cast<int*>(smem + LY::HIST_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::ABORT_OFF);
  const uint32_t bar0 = smem_u32(smem + LY::BAR_OFF);
  auto full = [bar0](int s) { return bar0 + 8u * s; };
  auto empty = [bar0](int s) { return bar0 + 8u * (kHiTokStages + s); };
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kHiTokStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  for (int b = threadIdx.x; b < kHiBins; b += blockDim.x) hist[b] = 0;
  __syncthreads();
  const int n_ch = p.d / kHiDimStep;
  const int groups = (p.top_pages + kHiTokPages - 1) / kHiTokPages;
  const int64_t items = (int64_t)p.batch * groups;
  const SsaWindow w = hi_window(p);
  if (warp == 4) {
    // producer: one lane issues a 16 KB tile per unit once its stage is free
    if (elect_one()) tma_prefetch_desc(&p.tm_index);
    uint32_t it = 0;
    bool ok = true;
    for (int64_t item = blockIdx.x; item < items && ok; item += gridDim.x) {
      const int n = (int)(item / groups);
      const int a0 = (int)(item % groups) * kHiTokPages;
      const int a1 = min(p.n_pages[n], a0 + kHiTokPages);
      for (int a = a0; a < a1 && ok; ++a) {
        const int pg = p.sel_pages[(int64_t)n * p.top_pages + a];
        for (int ch = 0; ch < n_ch; ++ch) {
          const int s = it % kHiTokStages;
          if (__any_sync(0xffffffffu, *abort_flag != 0) ||
              (it >= kHiTokStages && !warp_wait(empty(s), ((it / kHiTokStages) - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          if (elect_one()) {
            mbar_arrive_expect_tx(full(s), kHiTokTile);
            tma_load_3d(smem_u32(smem + LY::STAGE_OFF + s * kHiTokTile), &p.tm_index, full(s), kHiDimStep * ch,
                        pg * kHiPage, n);
          }
          __syncwarp();
          ++it;
        }
      }
    }
    if (!ok) {
      // after an abort, the tiles still in flight land before the CTA leaves
      for (uint32_t j = it > (uint32_t)kHiTokStages ? it - kHiTokStages : 0; j < it; ++j)
        mbar_wait(full(j % kHiTokStages), (j / kHiTokStages) & 1, nullptr);
    }
    return;
  }
  // consumers: thread t scores token t of each page
  const int t = threadIdx.x;
  uint32_t it = 0;
  bool ok = true;
  int q_seq = -1;
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
    const int n = (int)(item / groups);
    const int a0 = (int)(item % groups) * kHiTokPages;
    const int a1 = min(p.n_pages[n], a0 + kHiTokPages);
    if (a0 >= a1) continue;
    if (n != q_seq) {
      named_barrier_sync(1, 128);  // the previous sequence's q is no longer read
      for (int c = t; c < p.d; c += 128) q[c] = __bfloat162float(p.q_index[(int64_t)n * p.d + c]);
      named_barrier_sync(1, 128);
      q_seq = n;
    }
    const int i = p.seqlens[n] - 1;
    for (int a = a0; a < a1; ++a) {
      const int64_t tok = (int64_t)p.sel_pages[(int64_t)n * p.top_pages + a] * kHiPage + t;
      float sc = 0.f;
      for (int ch = 0; ch < n_ch; ++ch, ++it) {
        const int s = it % kHiTokStages;
        ok = ok && warp_wait(full(s), (it / kHiTokStages) & 1, abort_flag);
        if (ok) {
          const uint8_t* row = smem + LY::STAGE_OFF + s * kHiTokTile + t * 128;
          const float* qc = q + kHiDimStep * ch;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint4 v = *reinterpret_cast<const uint4*>(row + ((u ^ (t & 7)) << 4));
            const float4 qa = *reinterpret_cast<const float4*>(qc + 8 * u);
            const float4 qb = *reinterpret_cast<const float4*>(qc + 8 * u + 4);
            sc = __fmaf_rn(qa.x, __uint_as_float(v.x << 16), sc);
            sc = __fmaf_rn(qa.y, __uint_as_float(v.x & 0xFFFF0000u), sc);
            sc = __fmaf_rn(qa.z, __uint_as_float(v.y << 16), sc);
            sc = __fmaf_rn(qa.w, __uint_as_float(v.y & 0xFFFF0000u), sc);
            sc = __fmaf_rn(qb.x, __uint_as_float(v.z << 16), sc);
            sc = __fmaf_rn(qb.y, __uint_as_float(v.z & 0xFFFF0000u), sc);
            sc = __fmaf_rn(qb.z, __uint_as_float(v.w << 16), sc);
            sc = __fmaf_rn(qb.w, __uint_as_float(v.w & 0xFFFF0000u), sc);
          }
        }
        __syncwarp();
        if ((t & 31) == 0) mbar_arrive(empty(s));
      }
      const unsigned long long key = hi_outside(w, tok, i) ? hi_key(sc, tok) : 0ull;
      p.tok_keys[(int64_t)n * p.top_pages * kHiPage + (int64_t)a * kHiPage + t] = key;
      hi_hist_add(hist, key ? (int)(key >> kHiTopShift) : -1);
    }
    // this item's digits into the sequence's histogram
    named_barrier_sync(1, 128);
    for (int b = t; b < kHiBins; b += 128) {
      const int c = hist[b];
      if (c) {
        atomicAdd(&p.hist1[(int64_t)n * kHiBins + b], c);
        hist[b] = 0;
      }
    }
    named_barrier_sync(1, 128);
  }
}

// ---------------------------------------------------------------------------
// Token selection: a CTA (1024 threads) per sequence. The histogram of the
// keys' top digits gives the digit d1 of the top_k-th largest key: keys with
// a larger top digit are selected outright, those with digit d1 are the
// candidates, sorted out on chip by the remaining digits (or, if more than
// kHiCand share d1, by passes over the keys). The selection is then sorted by
// position. Dynamic shared memory: HiTopkLayout::SMEM_BYTES.
// ---------------------------------------------------------------------------
struct HiTopkLayout {
  static constexpr int SEL_OFF = 0;                          // [kHiMaxTopK] u64
  static constexpr int CAND_OFF = SEL_OFF + kHiMaxTopK * 8;  // [kHiCand] u64
  static constexpr int HIST_OFF = CAND_OFF + kHiCand * 8;    // [kHiBins] int
  static constexpr int SH_OFF = HIST_OFF + kHiBins * 4;      // [40] int
  static constexpr int SMEM_BYTES = SH_OFF + 40 * 4;
};

__global__ void __launch_bounds__(1024) hi_topk_kernel(const __grid_constant__ HiParams p) {
  using LY = HiTopkLayout;
  extern __shared__ __align__(16) uint8_t smem[];
  unsigned long long* sel = reinterpret_cast<unsigned long long*>(smem + LY::SEL_OFF);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem + LY::CAND_OFF);
  int* hist = reinterpret_cast<int*>(smem + LY::HIST_OFF);
  int* sh = reinterpret_cast<int*>(smem + LY::SH_OFF);  // [0..32] sums, [34..35] digit search, [36..37] counters
  const int n = blockIdx.x;
  const int64_t N = (int64_t)p.n_pages[n] * kHiPage;
  const unsigned long long* keys = p.tok_keys + (int64_t)n * p.top_pages * kHiPage;
  int v = 0;
  for (int b = threadIdx.x; b < kHiBins; b += blockDim.x) {
    hist[b] = p.hist1[(int64_t)n * kHiBins + b];
    v += hist[b];
  }
  if (threadIdx.x == 0) {
    sh[34] = 1;
    sh[35] = 0;
    sh[36] = 0;
    sh[37] = 0;
  }
  const int n_valid = hi_block_sum(v, sh);
  const int k_eff = min(n_valid, p.top_k);
  if (k_eff > 0) {
    if (threadIdx.x < 32) {
      // the top digit d1 of the k_eff-th largest key and its rank r1 among the keys of that digit
      const int lane = threadIdx.x;
      int own = 0;
      for (int b = 64 * lane; b < 64 * lane + 64; ++b) own += hist[b];
      int above = 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_down_sync(0xffffffffu, above + own, o);
        if (lane + o < 32) above += x;
      }
      if (above < k_eff && above + own >= k_eff) {
        int r = k_eff - above, dg = 64 * lane + 63;
        for (; dg > 64 * lane && hist[dg] < r; --dg) r -= hist[dg];
        sh[34] = r;
        sh[35] = dg;
      }
    }
    __syncthreads();
    const int r1 = sh[34], d1 = sh[35] & (kHiBins - 1);
    const int c1 = hist[d1];
    const bool on_chip = c1 <= kHiCand;
    const int64_t n_iter = (N + blockDim.x - 1) / blockDim.x * blockDim.x;
    for (int64_t t = threadIdx.x; t < n_iter; t += blockDim.x) {
      const unsigned long long k = t < N ? keys[t] : 0ull;
      const int dg = k ? (int)(k >> kHiTopShift) : -1;
      const bool take = dg > d1;
      const int s = hi_warp_slot(&sh[36], take);
      if (take && s < kHiMaxTopK) sel[s] = k;
      const bool keep = on_chip && dg == d1;
      const int c = hi_warp_slot(&sh[37], keep);
      if (keep && c < kHiCand) cand[c] = k;
    }
    __syncthreads();
    const unsigned long long pre = (unsigned long long)d1 << kHiTopShift;
    const unsigned long long msk = (unsigned long long)(kHiBins - 1) << kHiTopShift;
    const unsigned long long* src = on_chip ? cand : keys;
    const int64_t n_src = on_chip ? c1 : N;
    // the r1-th largest key of digit d1, by the digits below it
    const unsigned long long thr = hi_radix_kth(src, n_src, r1, pre, msk, kHiTopShift - kHiBits, hist, sh + 34);
    const int64_t n_iter2 = (n_src + blockDim.x - 1) / blockDim.x * blockDim.x;
    for (int64_t t = threadIdx.x; t < n_iter2; t += blockDim.x) {
      const unsigned long long k = t < n_src ? src[t] : 0ull;
      const bool take = k != 0ull && (k & msk) == pre && k >= thr;
      const int s = hi_warp_slot(&sh[36], take);
      if (take && s < kHiMaxTopK) sel[s] = k;
    }
  }
  __syncthreads();
  // by position: keys whose value is 2^32 - 1 - position, sorted largest first
  int npow2 = 1;
  while (npow2 < k_eff) npow2 <<= 1;
  for (int t = threadIdx.x; t < npow2; t += blockDim.x)
    sel[t] = t < k_eff ? (unsigned long long)(0xFFFFFFFFu - hi_key_index(sel[t])) : 0ull;
  __syncthreads();
  if (k_eff > 1) hi_sort_desc(sel, npow2);
  for (int t = threadIdx.x; t < p.top_k; t += blockDim.x)
    p.selected[(int64_t)n * p.top_k + t] = t < k_eff ? (int32_t)(0xFFFFFFFFu - (uint32_t)sel[t]) : -1;
  if (threadIdx.x == 0) p.n_sel[n] = k_eff;
}

// ---------------------------------------------------------------------------
// Caller-given selections: a CTA (1024 threads) per sequence keeps, in list
// order, the entries that name a token at or before the query and outside
// the window (stable compaction), and counts them.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) hi_compact_kernel(const int32_t* __restrict__ list, int top_k,
                                                          const int32_t* __restrict__ seqlens, SsaWindow w,
                                                          int32_t* __restrict__ out, int32_t* __restrict__ n_out) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  const int n = blockIdx.x;
  const int i = seqlens[n] - 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < top_k; base += blockDim.x) {
    const int j = base + threadIdx.x;
    const int e = j < top_k ? list[(int64_t)n * top_k + j] : -1;
    const bool keep = e >= 0 && e <= i && hi_outside(w, e, i);
    const unsigned m = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) warp_sums[warp] = __popc(m);
    __syncthreads();
    int before = carry;
    for (int x = 0; x < warp; ++x) before += warp_sums[x];
    if (keep) out[(int64_t)n * top_k + before + __popc(m & ((1u << lane) - 1u))] = e;
    __syncthreads();
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int x = 0; x < (int)(blockDim.x >> 5); ++x) tot += warp_sums[x];
      carry += tot;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) n_out[n] = carry;
}

// ---------------------------------------------------------------------------
// Gather: grid (cap_rows / 32, B), 256 threads. Row j of sequence n's packed
// block is, in order, the window's sink rows [0, min(s*b, L)), the selected
// tokens, and the window's local rows [max(lo, s*b), L). The three sets are
// disjoint, so attention over the packed rows (every row visible) is the
// attention over the window and the selection. counts[n] = rows packed.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) hi_gather_kernel(const __nv_bfloat16* __restrict__ kv, int64_t batch_stride,
                                                        int64_t row_stride, const int32_t* __restrict__ seqlens,
                                                        SsaWindow w, const int32_t* __restrict__ sel, int top_k,
                                                        const int32_t* __restrict__ n_sel, int cap_rows,
                                                        __nv_bfloat16* __restrict__ packed,
                                                        int32_t* __restrict__ counts) {
  const int n = blockIdx.y;
  const int L = seqlens[n];
  const int i = L - 1;
  const int sink_rows = (int)min((int64_t)w.sink_end, (int64_t)L);
  const int lo = (int)max((int64_t)w.lo(i), (int64_t)sink_rows);
  const int local_rows = max(L - lo, 0);
  const int ns = min(n_sel[n], top_k);
  const int count = min(sink_rows + ns + local_rows, cap_rows);
  if (blockIdx.x == 0 && threadIdx.x == 0) counts[n] = count;
  const int j0 = blockIdx.x * 32;
  for (int e = threadIdx.x; e < 32 * 72; e += blockDim.x) {
    const int j = j0 + e / 72, c = e % 72;
    if (j >= count) continue;
    int64_t tok;
    if (j < sink_rows) tok = j;
    else if (j < sink_rows + ns) tok = sel[(int64_t)n * top_k + (j - sink_rows)];
    else tok = lo + (j - sink_rows - ns);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (tok >= 0 && tok < L) v = reinterpret_cast<const uint4*>(kv + n * batch_stride + tok * row_stride)[c];
    reinterpret_cast<uint4*>(packed + ((int64_t)n * cap_rows + j) * 576)[c] = v;
  }
}

}  // namespace loza
