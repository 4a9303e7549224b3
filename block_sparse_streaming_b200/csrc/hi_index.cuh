// hi_index.cuh - hierarchical index for the decode, and attention over the
// tokens it selects.
//
// Page 4 of the LoZA pages ("LongCat Sparse Attention: Taming the Lightning
// via Streaming-aware Hierarchical Cross-Layer Indexing") splits a decode
// query's attention budget into fixed sink and window tokens (the SSA window
// of this library) and dynamically selected tokens, chosen by a hierarchical
// index in two stages: a coarse pass over pages of 128 tokens recalls the top
// pages, then only the tokens of those pages are scored and the best kept.
// The two parts are attended separately and merged by their log-sum-exp.
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
// Kernels:
//   hi_page_keys_kernel   mean index key per whole page (a thread per column)
//   hi_pages_kernel       one CTA per sequence: coarse scores of its pages,
//                         one bitonic sort of (score, page) keys in shared
//                         memory, the top pages
//   hi_tokens_kernel      a thread per token of a recalled page: its score
//   hi_topk_kernel        one CTA per sequence: radix select of the k-th
//                         largest (score, token) key, the tokens at or above
//                         it, sorted by position
//   hi_attend_kernel      softmax attention of the 64 heads over the selected
//                         latent rows (CUDA cores, fp32); optionally merged
//                         with the window part's fp32 O and LSE in its epilogue
#pragma once

#include <cuda_bf16.h>

#include "prefill.cuh"
#include "sm100.cuh"

namespace loza {

constexpr int kHiPage = 128;        // tokens per page
constexpr int kHiMaxPages = 8192;   // pages per sequence the one-CTA page sort holds
constexpr int kHiMaxTopK = 2048;    // selected tokens per sequence at most
constexpr int kHiMaxDim = 512;      // index dimension at most

struct HiParams {
  const __nv_bfloat16* q_index;  // [B, d]
  const __nv_bfloat16* k_index;  // token t of sequence n at n * batch_stride + t * row_stride (elements)
  int64_t batch_stride, row_stride;
  const float* page_keys;        // [B, pages_per_seq, d]
  int64_t pages_per_seq;
  const int32_t* seqlens;
  int d;
  int block, n_sink, n_local;    // the fixed window
  int top_pages, top_k;
  int32_t* sel_pages;            // [B, top_pages] recalled pages, best first
  int32_t* n_pages;              // [B] recalled page count
  unsigned long long* tok_keys;  // [B, top_pages * 128] (score, token) keys, 0 = none
  int32_t* selected;             // [B, top_k] selected tokens, ascending, then -1
};

// (score, index) as one unsigned key: larger for a larger score, then for a
// smaller index. The score's bits are made monotone (negative values
// flipped); -0 is first turned into +0 so that equal scores compare equal.
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

__global__ void __launch_bounds__(256) hi_page_keys_kernel(const __nv_bfloat16* __restrict__ k, int64_t batch_stride,
                                                           int64_t row_stride, const int32_t* __restrict__ seqlens,
                                                           int d, int64_t pages_per_seq, float* __restrict__ out) {
  const int n = blockIdx.y;
  const int64_t full = min((int64_t)seqlens[n] / kHiPage, pages_per_seq);
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < full * d;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t pg = idx / d;
    const int c = (int)(idx % d);
    const __nv_bfloat16* col = k + n * batch_stride + pg * kHiPage * row_stride + c;
    float sum = 0.f;
    for (int r = 0; r < kHiPage; ++r) sum += __bfloat162float(col[r * row_stride]);
    out[((int64_t)n * pages_per_seq + pg) * d + c] = sum * (1.0f / kHiPage);
  }
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

// One CTA (1024 threads) per sequence: the recalled pages.
__global__ void __launch_bounds__(1024) hi_pages_kernel(const HiParams p) {
  extern __shared__ __align__(16) unsigned long long hkeys[];  // [npow2]
  __shared__ float q[kHiMaxDim];
  const int n = blockIdx.x;
  const int L = p.seqlens[n];
  const int i = L - 1;
  const SsaWindow w{p.block, p.n_sink * p.block, p.n_local};
  const int full = (int)min((int64_t)max(L, 0) / kHiPage, p.pages_per_seq);
  int npow2 = 1;
  while (npow2 < full) npow2 <<= 1;
  for (int c = threadIdx.x; c < p.d; c += blockDim.x) q[c] = __bfloat162float(p.q_index[(int64_t)n * p.d + c]);
  __syncthreads();
  for (int pg = threadIdx.x; pg < npow2; pg += blockDim.x) {
    unsigned long long key = 0;
    // a whole page with a token outside the window: [128pg, 128pg+127] meets [sink_end, lo(i))
    if (pg < full && w.n_local >= 0 && (int64_t)pg * kHiPage + kHiPage - 1 >= w.sink_end &&
        (int64_t)pg * kHiPage < w.lo(i)) {
      const float* pk = p.page_keys + ((int64_t)n * p.pages_per_seq + pg) * p.d;
      float s = 0.f;
      for (int c = 0; c < p.d; ++c) s = __fmaf_rn(q[c], pk[c], s);
      key = hi_key(s, pg);
    }
    hkeys[pg] = key;
  }
  __syncthreads();
  hi_sort_desc(hkeys, npow2);
  // candidates are the non-zero keys, all at the front after the sort
  __shared__ int n_cand;
  if (threadIdx.x == 0) n_cand = 0;
  __syncthreads();
  int mine = 0;
  for (int t = threadIdx.x; t < npow2; t += blockDim.x) mine += hkeys[t] != 0ull;
  atomicAdd(&n_cand, mine);
  __syncthreads();
  const int m = min(n_cand, p.top_pages);
  for (int t = threadIdx.x; t < m; t += blockDim.x) p.sel_pages[(int64_t)n * p.top_pages + t] = (int32_t)hi_key_index(hkeys[t]);
  if (threadIdx.x == 0) p.n_pages[n] = m;
}

// A thread per token of a recalled page: its (score, token) key, 0 for a
// token inside the window. Grid (ceil(top_pages / pages_per_cta), B).
constexpr int kHiTokPagesPerCta = 8;
__global__ void __launch_bounds__(kHiPage) hi_tokens_kernel(const HiParams p) {
  __shared__ float q[kHiMaxDim];
  const int n = blockIdx.y;
  const int m = p.n_pages[n];
  const int a0 = blockIdx.x * kHiTokPagesPerCta;
  if (a0 >= m) return;
  const int i = p.seqlens[n] - 1;
  const SsaWindow w{p.block, p.n_sink * p.block, p.n_local};
  for (int c = threadIdx.x; c < p.d; c += blockDim.x) q[c] = __bfloat162float(p.q_index[(int64_t)n * p.d + c]);
  __syncthreads();
  for (int a = a0; a < min(m, a0 + kHiTokPagesPerCta); ++a) {
    const int64_t t = (int64_t)p.sel_pages[(int64_t)n * p.top_pages + a] * kHiPage + threadIdx.x;
    unsigned long long key = 0;
    if (hi_outside(w, t, i)) {
      const uint4* kr = reinterpret_cast<const uint4*>(p.k_index + n * p.batch_stride + t * p.row_stride);
      float s = 0.f;
      for (int c8 = 0; c8 < p.d / 8; ++c8) {
        const uint4 v = kr[c8];
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          s = __fmaf_rn(q[8 * c8 + 2 * e], __uint_as_float(wv[e] << 16), s);
          s = __fmaf_rn(q[8 * c8 + 2 * e + 1], __uint_as_float(wv[e] & 0xFFFF0000u), s);
        }
      }
      key = hi_key(s, t);
    }
    p.tok_keys[(int64_t)n * p.top_pages * kHiPage + (int64_t)a * kHiPage + threadIdx.x] = key;
  }
}

// One CTA (1024 threads) per sequence: the top_k tokens by key, by radix
// select of the k-th largest key (keys are distinct: the index is in them),
// then sorted by position.
__global__ void __launch_bounds__(1024) hi_topk_kernel(const HiParams p) {
  constexpr int kBits = 11, kBins = 1 << kBits;
  __shared__ int hist[kBins];
  __shared__ unsigned long long sel[kHiMaxTopK];
  __shared__ int n_valid, n_out;
  __shared__ int rank_s, digit_s;
  const int n = blockIdx.x;
  const int64_t N = (int64_t)p.n_pages[n] * kHiPage;
  const unsigned long long* keys = p.tok_keys + (int64_t)n * p.top_pages * kHiPage;
  if (threadIdx.x == 0) {
    n_valid = 0;
    n_out = 0;
  }
  __syncthreads();
  int v = 0;
  for (int64_t t = threadIdx.x; t < N; t += blockDim.x) v += keys[t] != 0ull;
  atomicAdd(&n_valid, v);
  __syncthreads();
  const int k_eff = min(n_valid, p.top_k);
  unsigned long long thr = 0;  // the k-th largest key
  if (k_eff > 0) {
    unsigned long long prefix = 0, mask = 0;
    int rank = k_eff;  // the rank of the wanted key among those matching the prefix, from the top
    for (int shift = 64 - kBits; shift > -kBits; shift -= kBits) {
      const int sh = max(shift, 0);
      const int width = shift >= 0 ? kBits : kBits + shift;  // the last digit has the remaining bits
      const unsigned long long dmask = ((1ull << width) - 1ull) << sh;
      for (int b = threadIdx.x; b < kBins; b += blockDim.x) hist[b] = 0;
      __syncthreads();
      for (int64_t t = threadIdx.x; t < N; t += blockDim.x) {
        const unsigned long long k = keys[t];
        if (k != 0ull && (k & mask) == prefix) atomicAdd(&hist[(int)((k & dmask) >> sh)], 1);
      }
      __syncthreads();
      if (threadIdx.x < 32) {
        // the digit holding the rank-th largest key, counted from the top:
        // lane j sums bins [64j, 64j+64), the lanes above it give the count
        // of larger digits, and the lane where the rank falls scans its bins
        const int lane = threadIdx.x;
        int own = 0;
        for (int b = 64 * lane; b < 64 * lane + 64; ++b) own += hist[b];
        int above = 0;  // bins of the lanes above this one
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int x = __shfl_down_sync(0xffffffffu, above + own, o);
          if (lane + o < 32) above += x;
        }
        // inclusive suffix sums: above + own counts the bins from 64*lane upward
        if (above < rank && above + own >= rank) {
          int r = rank - above, dgt = 64 * lane + 63;
          for (; dgt > 64 * lane && hist[dgt] < r; --dgt) r -= hist[dgt];
          rank_s = r;
          digit_s = dgt;
        }
      }
      __syncthreads();
      rank = rank_s;
      prefix |= (unsigned long long)digit_s << sh;
      mask |= dmask;
      __syncthreads();
    }
    thr = prefix;
    for (int64_t t = threadIdx.x; t < N; t += blockDim.x) {
      const unsigned long long k = keys[t];
      if (k != 0ull && k >= thr) {
        const int slot = atomicAdd(&n_out, 1);  // < k_eff: the keys are distinct
        if (slot < kHiMaxTopK) sel[slot] = k;
      }
    }
  }
  __syncthreads();
  // by position: sort the indices (as keys whose upper half is the position)
  int npow2 = 1;
  while (npow2 < k_eff) npow2 <<= 1;
  for (int t = threadIdx.x; t < npow2; t += blockDim.x)
    sel[t] = t < k_eff ? (unsigned long long)(0xFFFFFFFFu - hi_key_index(sel[t])) : 0ull;
  __syncthreads();
  if (k_eff > 1) hi_sort_desc(sel, npow2);  // largest 0xFFFFFFFF - t first: ascending t
  for (int t = threadIdx.x; t < p.top_k; t += blockDim.x)
    p.selected[(int64_t)n * p.top_k + t] = t < k_eff ? (int32_t)(0xFFFFFFFFu - (uint32_t)sel[t]) : -1;
}

// Attention of the 64 heads of the decode query over its selected latent rows
// (absorbed MLA: K = the 576-wide row, V = its first 512 columns), fp32 on
// CUDA cores. Grid (B, 8 groups of 8 heads), 256 threads: warp h of a group
// owns head h's softmax; thread (h, lane) accumulates 16 value columns.
constexpr int kHiAttnChunk = 64;
constexpr int kHiAttnRowBytes = 576 * 2 + 16;  // padded shared-memory row
struct HiAttnLayout {
  static constexpr int Q_OFF = 0;                                  // [8][576] fp32
  static constexpr int K_OFF = Q_OFF + 8 * 576 * 4;                // [64][kHiAttnRowBytes]
  static constexpr int P_OFF = K_OFF + kHiAttnChunk * kHiAttnRowBytes;  // [8][64] fp32
  static constexpr int A_OFF = P_OFF + 8 * kHiAttnChunk * 4;       // [8] rescale factors
  static constexpr int SMEM_BYTES = A_OFF + 8 * 4;
};

__global__ void __launch_bounds__(256) hi_attend_kernel(const __nv_bfloat16* __restrict__ q,
                                                        const __nv_bfloat16* __restrict__ kv, int64_t batch_stride,
                                                        int64_t row_stride, const int32_t* __restrict__ selected,
                                                        int top_k, float scale_log2,
                                                        const float* __restrict__ o_win,
                                                        const float* __restrict__ lse_win,
                                                        __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  using LY = HiAttnLayout;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int n = blockIdx.x, g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = 8 * g + warp;
  float* qs = reinterpret_cast<float*>(smem + LY::Q_OFF);
  float* ps = reinterpret_cast<float*>(smem + LY::P_OFF);
  float* as = reinterpret_cast<float*>(smem + LY::A_OFF);
  for (int e = threadIdx.x; e < 8 * 576; e += blockDim.x)
    qs[e] = __bfloat162float(q[((int64_t)n * 64 + 8 * g) * 576 + e]);
  const int32_t* sel = selected + (int64_t)n * top_k;
  float m = -INFINITY, l = 0.f;  // of this warp's head (every lane holds them)
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  for (int c0 = 0; c0 < top_k; c0 += kHiAttnChunk) {
    __syncthreads();  // the previous chunk's rows and P are consumed
    // rows of this chunk: 64 x 72 sixteen-byte vectors
    for (int e = threadIdx.x; e < kHiAttnChunk * 72; e += blockDim.x) {
      const int r = e / 72, c = e % 72;
      const int t = c0 + r < top_k ? sel[c0 + r] : -1;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t >= 0) v = reinterpret_cast<const uint4*>(kv + n * batch_stride + (int64_t)t * row_stride)[c];
      *reinterpret_cast<uint4*>(smem + LY::K_OFF + r * kHiAttnRowBytes + 16 * c) = v;
    }
    __syncthreads();
    // logits of tokens lane and lane + 32 for this warp's head (log2 units)
    float z[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = lane + 32 * half;
      const uint4* kr = reinterpret_cast<const uint4*>(smem + LY::K_OFF + r * kHiAttnRowBytes);
      const float* qh = qs + warp * 576;
      float s = 0.f;
      for (int c = 0; c < 72; ++c) {
        const uint4 v = kr[c];
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          s = fmaf(qh[8 * c + 2 * e], __uint_as_float(wv[e] << 16), s);
          s = fmaf(qh[8 * c + 2 * e + 1], __uint_as_float(wv[e] & 0xFFFF0000u), s);
        }
      }
      const bool valid = c0 + r < top_k && sel[c0 + r] >= 0;
      z[half] = valid ? s * scale_log2 : -INFINITY;
    }
    float mx = fmaxf(z[0], z[1]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float mn = fmaxf(m, mx);
    const float alpha = mn == -INFINITY ? 1.f : exp2f(m - mn);
    const float p0 = mn == -INFINITY ? 0.f : exp2f(z[0] - mn);
    const float p1 = mn == -INFINITY ? 0.f : exp2f(z[1] - mn);
    float sp = p0 + p1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sp += __shfl_xor_sync(0xffffffffu, sp, o);
    l = l * alpha + sp;
    m = mn;
    ps[warp * kHiAttnChunk + lane] = p0;
    ps[warp * kHiAttnChunk + lane + 32] = p1;
    if (lane == 0) as[warp] = alpha;
    __syncwarp();
    // O(head, 16 columns of this lane) = O * alpha + sum_t P[t] V[t, columns]
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] *= alpha;
    for (int r = 0; r < kHiAttnChunk; ++r) {
      const float pr = ps[warp * kHiAttnChunk + r];
      const uint4* vr = reinterpret_cast<const uint4*>(smem + LY::K_OFF + r * kHiAttnRowBytes + 32 * lane);
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const uint4 v = vr[h2];
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[8 * h2 + 2 * e] = fmaf(pr, __uint_as_float(wv[e] << 16), acc[8 * h2 + 2 * e]);
          acc[8 * h2 + 2 * e + 1] = fmaf(pr, __uint_as_float(wv[e] & 0xFFFF0000u), acc[8 * h2 + 2 * e + 1]);
        }
      }
    }
  }
  // This part alone (no selected token: O = 0, LSE = -inf), or, given the
  // window part's unrounded O and its LSE, the log-sum-exp merge of the two
  // (weights exp(LSE_part - LSE), LSE = log(exp(LSE_win) + exp(LSE_sel))).
  const int64_t row = (int64_t)n * 64 + head;
  float w_sel = l > 0.f ? 1.f / l : 0.f;  // multiplies acc
  float w_win = 0.f;
  float lse2 = l > 0.f ? m + log2f(l) : -INFINITY;  // log2 units
  if (o_win) {
    const float a = lse_win[row] * 1.4426950408889634f;
    const float mx = fmaxf(a, lse2);
    if (mx == -INFINITY) {
      w_sel = 0.f;
    } else {
      const float ea = exp2f(a - mx), eb = exp2f(lse2 - mx);
      const float inv = 1.f / (ea + eb);
      w_win = ea * inv;
      w_sel = l > 0.f ? exp2f(m - mx) * inv : 0.f;  // eb / l
      lse2 = mx + log2f(ea + eb);
    }
  }
  __nv_bfloat16* o = out + row * 512 + 16 * lane;
  if (o_win) {
    const float4* ow = reinterpret_cast<const float4*>(o_win + row * 512 + 16 * lane);
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) {
      const float4 v = ow[e4];
      acc[4 * e4] = fmaf(w_win, v.x, acc[4 * e4] * w_sel);
      acc[4 * e4 + 1] = fmaf(w_win, v.y, acc[4 * e4 + 1] * w_sel);
      acc[4 * e4 + 2] = fmaf(w_win, v.z, acc[4 * e4 + 2] * w_sel);
      acc[4 * e4 + 3] = fmaf(w_win, v.w, acc[4 * e4 + 3] * w_sel);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] *= w_sel;
  }
#pragma unroll
  for (int e = 0; e < 16; e += 2)
    *reinterpret_cast<__nv_bfloat162*>(o + e) = __floats2bfloat162_rn(acc[e], acc[e + 1]);
  if (lane == 0) lse[row] = lse2 == -INFINITY ? -INFINITY : lse2 * 0.69314718055994530942f;
}

}  // namespace loza
