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
//                           and a histogram of the keys' top digit
//   hi_page_select_kernel   a CTA per sequence: the top pages (one pass over
//                           the keys from that histogram, radix select among
//                           the keys sharing the threshold's top digit)
//   hi_tokens_kernel        persistent; the index keys of the recalled pages
//                           arrive by TMA in 128-row x 64-column tiles and a
//                           thread per token forms its score; writes the keys
//                           and a histogram of their top digit per sequence
//   hi_topk_collect_kernel  many CTAs per sequence: from that histogram, the
//                           keys at or above the threshold's top digit
//   hi_topk_kernel          a CTA per sequence: the top_k tokens (radix
//                           select among the threshold's digit), in order of
//                           position through a bitmap
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
constexpr int kHiCand = 4096;       // keys sharing the threshold's first digit that are sorted out on chip
constexpr int kHiTiny = 64;         // a digit shared by at most this many keys is resolved by direct ranking

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
  // zero on entry (one memset per call): histograms of top digits and list counters
  int32_t* page_hist;             // [B, kHiBins] of the page keys
  int32_t* hist1;                 // [B, kHiBins] of the token keys
  int32_t* counters;              // [B, 4]: [3] the length of the sequence's tok_cand list
  unsigned long long* page_cand;  // [B, pages_per_seq] page keys at or above the threshold's top digit
  unsigned long long* tok_keys;   // [B, top_pages * 128] token keys, 0 = none
  unsigned long long* tok_cand;   // [B, top_pages * 128] token keys at or above the threshold's top digit
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
  if (!__any_sync(0xffffffffu, bin >= 0)) return;
  const unsigned peers = __match_any_sync(0xffffffffu, bin);
  if (bin >= 0 && (threadIdx.x & 31) == (unsigned)(__ffs(peers) - 1)) atomicAdd(&hist[bin], __popc(peers));
}

// A slot in a shared list for every lane with `take`: one atomic per warp.
// Whole warp; returns the lane's slot (meaningless where !take).
__device__ __forceinline__ int hi_warp_slot(int* counter, bool take) {
  const unsigned m = __ballot_sync(0xffffffffu, take);
  if (!m) return 0;
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(m) - 1;
  int base = 0;
  if (lane == leader) base = atomicAdd(counter, __popc(m));
  base = __shfl_sync(0xffffffffu, base, leader);
  return base + __popc(m & ((1u << lane) - 1u));
}

// Warp 0 of a block (all 32 lanes): the bin of hist[0, kHiBins) holding the
// rank-th largest element, counting from the top bin, the element's rank
// within that bin and the bin's count, into sh[0] (rank), sh[1] (bin) and
// sh[2] (count); sh is left as it was
// if the counts hold fewer than rank elements. Lane j first sums bins
// [64j, 64j + 64) (hist 16-byte aligned), a suffix scan over the lanes finds
// the lane whose bins hold the rank, and its 64 bins, two per lane, are
// resolved the same way.
__device__ __forceinline__ void hi_find_bin(const int* hist, int rank, int* sh) {
  const int lane = threadIdx.x & 31;
  const int4* h4 = reinterpret_cast<const int4*>(hist + 64 * lane);
  int own = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int4 v = h4[j];
    own += v.x + v.y + v.z + v.w;
  }
  int above = 0;  // elements in the bins of the lanes above this one
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_down_sync(0xffffffffu, above + own, o);
    if (lane + o < 32) above += x;
  }
  const unsigned hit = __ballot_sync(0xffffffffu, above < rank && above + own >= rank);
  if (!hit) return;
  const int L = __ffs(hit) - 1;
  const int r = rank - __shfl_sync(0xffffffffu, above, L);  // rank among lane L's bins
  const int b0 = hist[64 * L + 2 * lane], b1 = hist[64 * L + 2 * lane + 1];
  const int own2 = b0 + b1;
  int above2 = 0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_down_sync(0xffffffffu, above2 + own2, o);
    if (lane + o < 32) above2 += x;
  }
  if (above2 < r && above2 + own2 >= r) {
    const int rr = r - above2;  // the higher bin of the pair first
    if (b1 >= rr) {
      sh[0] = rr;
      sh[1] = 64 * L + 2 * lane + 1;
      sh[2] = b1;
    } else {
      sh[0] = rr - b1;
      sh[1] = 64 * L + 2 * lane;
      sh[2] = b0;
    }
  }
}

// Block-wide pass over keys[0, N): f(key) on every thread, the same number
// of times on every lane (0 past the end), with kHiScanDepth loads in flight
// per thread so that a pass over global memory is not one round trip per key.
constexpr int kHiScanDepth = 8;
template <typename F>
__device__ __forceinline__ void hi_for_keys(const unsigned long long* keys, int64_t N, F&& f) {
  const int64_t step = (int64_t)blockDim.x * kHiScanDepth;
  for (int64_t base = 0; base < N; base += step) {
    unsigned long long kk[kHiScanDepth];
#pragma unroll
    for (int j = 0; j < kHiScanDepth; ++j) {
      const int64_t t = base + (int64_t)j * blockDim.x + threadIdx.x;
      kk[j] = t < N ? keys[t] : 0ull;
    }
#pragma unroll
    for (int j = 0; j < kHiScanDepth; ++j)
      if (base + (int64_t)j * blockDim.x < N) f(kk[j]);  // block-uniform: rows past the end are skipped
  }
}

// Block-wide: the rank-th largest non-zero key of keys[0, N) among those
// equal to `prefix` on the bits `mask` already fixed, deciding the digits
// from bit `shift` down (1 <= rank <= that count). Once the digits so far
// leave at most kHiTiny keys, those are gathered and ranked directly. `hist`
// holds kHiBins ints (16-byte aligned), `sh` four ints, `tiny` kHiTiny + 1
// keys, all in shared memory.
__device__ unsigned long long hi_radix_kth(const unsigned long long* keys, int64_t N, int rank,
                                           unsigned long long prefix, unsigned long long mask, int shift, int* hist,
                                           int* sh, unsigned long long* tiny) {
  for (; shift > -kHiBits; shift -= kHiBits) {
    const int s0 = max(shift, 0);
    const int width = shift >= 0 ? kHiBits : kHiBits + shift;  // the last digit holds the remaining bits
    const unsigned long long dmask = ((1ull << width) - 1ull) << s0;
    for (int b = threadIdx.x; b < kHiBins; b += blockDim.x) hist[b] = 0;
    if (threadIdx.x == 0) sh[2] = kHiTiny + 1;
    __syncthreads();
    hi_for_keys(keys, N, [&](unsigned long long k) {
      const bool in = k != 0ull && (k & mask) == prefix;
      hi_hist_add(hist, in ? (int)((k & dmask) >> s0) : -1);
    });
    __syncthreads();
    if (threadIdx.x < 32) hi_find_bin(hist, rank, sh);
    __syncthreads();
    rank = sh[0];
    prefix |= (unsigned long long)sh[1] << s0;
    mask |= dmask;
    const int cnt = sh[2];
    __syncthreads();
    if (s0 == 0) break;  // every bit decided
    if (cnt <= kHiTiny) {
      // the few keys with this prefix: the one with rank - 1 larger keys among them
      if (threadIdx.x == 0) {
        sh[3] = 0;
        tiny[kHiTiny] = prefix;
      }
      __syncthreads();
      hi_for_keys(keys, N, [&](unsigned long long k) {
        const bool in = k != 0ull && (k & mask) == prefix;
        const int slot = hi_warp_slot(&sh[3], in);
        if (in && slot < kHiTiny) tiny[slot] = k;
      });
      __syncthreads();
      const int c = min(sh[3], kHiTiny);
      if ((int)threadIdx.x < c) {
        const unsigned long long k = tiny[threadIdx.x];
        int larger = 0;
        for (int j = 0; j < c; ++j) larger += tiny[j] > k;
        if (larger == rank - 1) tiny[kHiTiny] = k;
      }
      __syncthreads();
      const unsigned long long r = tiny[kHiTiny];
      __syncthreads();
      return r;
    }
  }
  return prefix;
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
// A page is a candidate if it is whole and meets [sink_end, lo(i)). Also the
// histogram of the keys' top digits per sequence (page_hist, zero on entry).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) hi_page_scores_kernel(const __grid_constant__ HiParams p) {
  __shared__ float q[kHiMaxDim];
  __shared__ int hist[kHiBins];
  const int n = blockIdx.y;
  const int L = p.seqlens[n];
  const int i = L - 1;
  const SsaWindow w = hi_window(p);
  const int64_t full = min((int64_t)max(L, 0) / kHiPage, p.pages_per_seq);
  for (int c = threadIdx.x; c < p.d; c += blockDim.x) q[c] = __bfloat162float(p.q_index[(int64_t)n * p.d + c]);
  for (int b = threadIdx.x; b < kHiBins; b += blockDim.x) hist[b] = 0;
  __syncthreads();
  const int64_t pg = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  unsigned long long key = 0;
  if (pg < full && w.n_local >= 0 && pg * kHiPage + kHiPage - 1 >= w.sink_end && pg * kHiPage < w.lo(i)) {
    const float* pk = p.page_keys + (int64_t)n * p.d * p.pages_per_seq + pg;
    float s = 0.f;
#pragma unroll 16
    for (int c = 0; c < p.d; ++c) s = __fmaf_rn(q[c], pk[(int64_t)c * p.pages_per_seq], s);
    key = hi_key(s, pg);
  }
  if (pg < p.pages_per_seq) p.page_scored[(int64_t)n * p.pages_per_seq + pg] = key;
  hi_hist_add(hist, key ? (int)(key >> kHiTopShift) : -1);
  __syncthreads();
  for (int b = threadIdx.x; b < kHiBins; b += blockDim.x)
    if (hist[b]) atomicAdd(&p.page_hist[(int64_t)n * kHiBins + b], hist[b]);
  griddep_launch_dependents();
}

// Top-k by the histogram of top digits: the digit d1 of the k-th largest key
// and its rank r1 among the keys of that digit (warp 0 writes sh[0..2]:
// r1, d1, count of d1; defaults r1 = 1, d1 = 0). Block-wide; hist in shared
// memory (16-byte aligned) holds the histogram.
__device__ __forceinline__ void hi_first_digit(const int* hist, int k, int* sh) {
  if (threadIdx.x < 32) hi_find_bin(hist, k, sh);
  __syncthreads();
}

// ---------------------------------------------------------------------------
// Page selection: a CTA (1024 threads) per sequence. From the histogram of
// the page keys' top digits, the digit d1 of the top_pages-th key: the keys
// with top digit >= d1 are listed (on chip, or in the workspace if many), the
// r1-th largest of digit d1 found among them by the remaining digits, and
// every listed key at or above it is recalled.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) hi_page_select_kernel(const __grid_constant__ HiParams p) {
  __shared__ __align__(16) int hist[kHiBins];
  __shared__ __align__(16) unsigned long long list_s[kHiCand];
  __shared__ unsigned long long tiny[kHiTiny + 1];
  __shared__ int sh[40];
  const int n = blockIdx.x;
  const unsigned long long* keys = p.page_scored + (int64_t)n * p.pages_per_seq;
  const int64_t N = p.pages_per_seq;
  griddep_wait();  // the page keys and their histogram
  int v = 0;
  for (int b = threadIdx.x; b < kHiBins; b += blockDim.x) {
    hist[b] = p.page_hist[(int64_t)n * kHiBins + b];
    v += hist[b];
  }
  if (threadIdx.x == 0) {
    sh[34] = 1;
    sh[35] = 0;
    sh[38] = 0;  // listed
    sh[39] = 0;  // recalled
  }
  const int n_valid = hi_block_sum(v, sh);
  const int m = min(n_valid, p.top_pages);
  if (m > 0) {
    hi_first_digit(hist, m, sh + 34);
    const int r1 = sh[34], d1 = sh[35] & (kHiBins - 1);
    const int n_list = m - r1 + hist[d1];
    const bool on_chip = n_list <= kHiCand;
    unsigned long long* list = on_chip ? list_s : p.page_cand + (int64_t)n * p.pages_per_seq;
    hi_for_keys(keys, N, [&](unsigned long long k) {
      const bool in = k != 0ull && (int)(k >> kHiTopShift) >= d1;
      const int s = hi_warp_slot(&sh[38], in);
      if (in && s < n_list) list[s] = k;
    });
    __syncthreads();
    const unsigned long long pre = (unsigned long long)d1 << kHiTopShift;
    const unsigned long long msk = (unsigned long long)(kHiBins - 1) << kHiTopShift;
    const unsigned long long thr = hi_radix_kth(list, n_list, r1, pre, msk, kHiTopShift - kHiBits, hist, sh, tiny);
    int32_t* out = p.sel_pages + (int64_t)n * p.top_pages;
    hi_for_keys(list, n_list, [&](unsigned long long k) {
      const bool take = k != 0ull && k >= thr;
      const int s = hi_warp_slot(&sh[39], take);
      if (take && s < p.top_pages) out[s] = (int32_t)hi_key_index(k);
    });
  }
  if (threadIdx.x == 0) p.n_pages[n] = m;
  griddep_launch_dependents();
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
  griddep_wait();  // the recalled pages
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
    griddep_launch_dependents();
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
  griddep_launch_dependents();
}

// ---------------------------------------------------------------------------
// Token selection, first pass: grid (ceil(top_pages * 128 / kHiCollectKeys),
// B), 256 threads. From the histogram of the token keys' top digits every
// CTA derives the digit d1 of the top_k-th largest key, lists the keys of its
// slice with top digit >= d1 on chip and appends them to the sequence's list
// tok_cand (its length in counters[n * 4 + 3], zero on entry).
// ---------------------------------------------------------------------------
constexpr int kHiCollectKeys = 8192;
constexpr int kHiCollectList = 2048;
__global__ void __launch_bounds__(256) hi_topk_collect_kernel(const __grid_constant__ HiParams p) {
  __shared__ __align__(16) int hist[kHiBins];
  __shared__ unsigned long long list_s[kHiCollectList];
  __shared__ int sh[40];
  const int n = blockIdx.y;
  griddep_wait();  // the token keys and their histogram
  const int64_t N = (int64_t)p.n_pages[n] * kHiPage;
  const int64_t t0 = (int64_t)blockIdx.x * kHiCollectKeys;
  if (t0 >= N) {
    griddep_launch_dependents();
    return;
  }
  int v = 0;
  for (int b = threadIdx.x; b < kHiBins; b += blockDim.x) {
    hist[b] = p.hist1[(int64_t)n * kHiBins + b];
    v += hist[b];
  }
  if (threadIdx.x == 0) {
    sh[34] = 1;
    sh[35] = 0;
    sh[38] = 0;
  }
  const int k_eff = min(hi_block_sum(v, sh), p.top_k);
  if (k_eff <= 0) {
    griddep_launch_dependents();
    return;
  }
  hi_first_digit(hist, k_eff, sh + 34);
  const int d1 = sh[35] & (kHiBins - 1);
  int32_t* cnt = p.counters + (int64_t)n * 4;
  unsigned long long* list = p.tok_cand + (int64_t)n * p.top_pages * kHiPage;
  const int64_t cap = (int64_t)p.top_pages * kHiPage;
  hi_for_keys(p.tok_keys + (int64_t)n * p.top_pages * kHiPage + t0, min((int64_t)kHiCollectKeys, N - t0),
              [&](unsigned long long k) {
                const bool in = k != 0ull && (int)(k >> kHiTopShift) >= d1;
                const int s = hi_warp_slot(&sh[38], in);
                if (in && s < kHiCollectList) list_s[s] = k;
                const bool spill = in && s >= kHiCollectList;  // a crowded slice: straight to the list
                const int g = hi_warp_slot(&cnt[3], spill);
                if (spill && g < cap) list[g] = k;
              });
  __syncthreads();
  const int nl = min(sh[38], kHiCollectList);
  if (threadIdx.x == 0) sh[0] = nl ? atomicAdd(&cnt[3], nl) : 0;
  __syncthreads();
  const int base = sh[0];
  for (int t = threadIdx.x; t < nl; t += blockDim.x)
    if (base + t < cap) list[base + t] = list_s[t];
  griddep_launch_dependents();
}

// ---------------------------------------------------------------------------
// Token selection, second pass: a CTA (1024 threads) per sequence. Among the
// listed keys (top digit >= d1; on chip when at most kHiCand), the r1-th
// largest of digit d1 by the remaining digits is the threshold; the listed
// keys at or above it are the selection. Their positions go into a bitmap of
// the sequence's whole pages, read back in order. Dynamic shared memory:
// HiTopkLayout::bytes(pages_per_seq).
// ---------------------------------------------------------------------------
struct HiTopkLayout {
  static constexpr int LIST_OFF = 0;                            // [kHiCand] u64
  static constexpr int TINY_OFF = LIST_OFF + kHiCand * 8;       // [kHiTiny + 1] u64
  static constexpr int HIST_OFF = TINY_OFF + (kHiTiny + 2) * 8;  // [kHiBins] int
  static constexpr int SH_OFF = HIST_OFF + kHiBins * 4;         // [64] int
  static constexpr int BITS_OFF = SH_OFF + 64 * 4;              // [pages * 4] u32 bitmap
  static constexpr int bytes(int64_t pages) { return BITS_OFF + (int)(pages * 4 * 4); }
};

__global__ void __launch_bounds__(1024) hi_topk_kernel(const __grid_constant__ HiParams p) {
  using LY = HiTopkLayout;
  extern __shared__ __align__(1024) uint8_t smem[];
  unsigned long long* list_s = reinterpret_cast<unsigned long long*>(smem + LY::LIST_OFF);
  unsigned long long* tiny = reinterpret_cast<unsigned long long*>(smem + LY::TINY_OFF);
  int* hist = reinterpret_cast<int*>(smem + LY::HIST_OFF);
  int* sh = reinterpret_cast<int*>(smem + LY::SH_OFF);  // [0..32] sums, [34..36] first digit, [40..43] radix
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem + LY::BITS_OFF);
  const int n = blockIdx.x;
  const int nwords = (int)(p.pages_per_seq * 4);
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) bits[w] = 0u;
  griddep_wait();  // the lists of the first pass
  int v = 0;
  for (int b = threadIdx.x; b < kHiBins; b += blockDim.x) {
    hist[b] = p.hist1[(int64_t)n * kHiBins + b];
    v += hist[b];
  }
  if (threadIdx.x == 0) {
    sh[34] = 1;
    sh[35] = 0;
  }
  const int k_eff = min(hi_block_sum(v, sh), p.top_k);
  if (k_eff > 0) {
    hi_first_digit(hist, k_eff, sh + 34);
    const int r1 = sh[34], d1 = sh[35] & (kHiBins - 1);
    const int n_list = min((int64_t)p.counters[(int64_t)n * 4 + 3], (int64_t)p.top_pages * kHiPage);
    const unsigned long long* list_g = p.tok_cand + (int64_t)n * p.top_pages * kHiPage;
    const bool on_chip = n_list <= kHiCand;
    if (on_chip)
      for (int t = threadIdx.x; t < n_list; t += blockDim.x) list_s[t] = list_g[t];
    __syncthreads();
    const unsigned long long* list = on_chip ? list_s : list_g;
    const unsigned long long pre = (unsigned long long)d1 << kHiTopShift;
    const unsigned long long msk = (unsigned long long)(kHiBins - 1) << kHiTopShift;
    const unsigned long long thr =
        hi_radix_kth(list, n_list, r1, pre, msk, kHiTopShift - kHiBits, hist, sh + 40, tiny);
    hi_for_keys(list, n_list, [&](unsigned long long k) {
      if (k != 0ull && k >= thr) {
        const uint32_t pos = hi_key_index(k);
        if (pos < (uint32_t)nwords * 32u) atomicOr(&bits[pos >> 5], 1u << (pos & 31));
      }
    });
  }
  __syncthreads();
  // positions in order: warp w reads the words [w * per, (w + 1) * per), 32
  // consecutive words at a time (lane = word)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, n_warps = blockDim.x >> 5;
  const int per = (nwords + n_warps - 1) / n_warps;
  const int wb = warp * per, we = min(wb + per, nwords);
  int cnt = 0;
  for (int w = wb + lane; w < we; w += 32) cnt += __popc(bits[w]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) sh[warp] = cnt;
  __syncthreads();
  if (warp == 0) {
    const int wv = lane < n_warps ? sh[lane] : 0;
    int wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += x;
    }
    sh[lane] = wi - wv;  // positions before this warp's words
  }
  __syncthreads();
  int at = sh[warp];
  int32_t* out = p.selected + (int64_t)n * p.top_k;
  for (int w0 = wb; w0 < we; w0 += 32) {
    const int w = w0 + lane;
    uint32_t b = w < we ? bits[w] : 0u;
    const int c = __popc(b);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    int q = at + incl - c;
    while (b) {
      const int j = __ffs(b) - 1;
      b &= b - 1;
      if (q < p.top_k) out[q] = w * 32 + j;
      ++q;
    }
    at += __shfl_sync(0xffffffffu, incl, 31);
  }
  for (int t = k_eff + threadIdx.x; t < p.top_k; t += blockDim.x) out[t] = -1;
  if (threadIdx.x == 0) p.n_sel[n] = k_eff;
  griddep_launch_dependents();
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
  griddep_wait();  // the selection
  const int L = seqlens[n];
  const int i = L - 1;
  const int sink_rows = (int)min((int64_t)w.sink_end, (int64_t)L);
  const int lo = (int)max((int64_t)w.lo(i), (int64_t)sink_rows);
  const int local_rows = max(L - lo, 0);
  const int ns = min(n_sel[n], top_k);
  const int count = min(sink_rows + ns + local_rows, cap_rows);
  if (blockIdx.x == 0 && threadIdx.x == 0) counts[n] = count;
  // the 32 rows' tokens first (-1: past the packed rows, not written; -2: an
  // entry that names no row of the sequence, written as zeros), then all 9
  // copies of each thread in flight at once
  __shared__ int64_t src[32];
  const int j0 = blockIdx.x * 32;
  if (threadIdx.x < 32) {
    const int j = j0 + threadIdx.x;
    int64_t tok = -1;
    if (j < count) {
      if (j < sink_rows) tok = j;
      else if (j < sink_rows + ns) tok = sel[(int64_t)n * top_k + (j - sink_rows)];
      else tok = lo + (j - sink_rows - ns);
      if (tok >= L) tok = -1;
    }
    src[threadIdx.x] = j < count ? (tok < 0 ? -2 : tok) : -1;
  }
  __syncthreads();
  static_assert(32 * 72 % 256 == 0, "whole copies per thread");
  uint4 v[32 * 72 / 256];
#pragma unroll
  for (int it = 0; it < 32 * 72 / 256; ++it) {
    const int e = threadIdx.x + it * 256, r = e / 72, c = e % 72;
    const int64_t tok = src[r];
    v[it] = tok >= 0 ? reinterpret_cast<const uint4*>(kv + n * batch_stride + tok * row_stride)[c]
                     : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int it = 0; it < 32 * 72 / 256; ++it) {
    const int e = threadIdx.x + it * 256, r = e / 72, c = e % 72;
    if (src[r] != -1) reinterpret_cast<uint4*>(packed + ((int64_t)n * cap_rows + j0 + r) * 576)[c] = v[it];
  }
  griddep_launch_dependents();
}

}  // namespace loza
