// decode.cuh - SSA decode for per-head K/V on sm_100a.
//
// Decode runs one new query token per sequence: the token at position
// i = L-1 attends to the keys its window selects (sink blocks plus the l most
// recent blocks, causal inside its own block; page 1 section 01 of the LoZA
// pages, and section 02 for the decode use of the streaming kernel).
// With per-head K/V (d = 64, or 192/128) one query vector per head against
// <= 1024 keys is a matrix-vector product, so it runs on CUDA cores: 4 warps
// per (sequence, head), online softmax per warp, merged through shared memory.
// The absorbed-MLA decode, where all heads share one latent row and the
// product is a real GEMM, is in decode_mla.cuh.
#pragma once

#include "sm100.cuh"
#include "prefill.cuh"

namespace loza {

// ---------------------------------------------------------------------------
// Per-head K/V decode on CUDA cores.
// ---------------------------------------------------------------------------
struct DecodeMhaParams {
  const __nv_bfloat16* q;      // [B, H, DQK]
  const __nv_bfloat16* k;      // cache rows: k + n*batch_stride + t*row_stride + hk*DQK
  const __nv_bfloat16* v;      // same with DV
  int64_t k_batch_stride, k_row_stride, v_batch_stride, v_row_stride;
  const int32_t* seqlens;
  __nv_bfloat16* out;          // [B, H, DV]
  float* lse;                  // [B, H]
  int n_heads, n_kv_heads;
  int n_sink, n_local;
  int block;  // b, tokens per block of the window
  float scale_log2;
};

template <int DQK, int DV>
__global__ void __launch_bounds__(128) ssa_decode_mha_kernel(const DecodeMhaParams p) {
  constexpr int QPL = DQK / 32;  // q elements per lane
  constexpr int VPL = DV / 32;
  const int h = blockIdx.x, seq = blockIdx.y;
  const int hk = h / (p.n_heads / p.n_kv_heads);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = p.seqlens[seq];
  const int i_q = L - 1;
  // the window of the query: keys [0, sink_end) and [lo, i_q], each once
  const SsaWindow win{p.block, p.n_sink * p.block, p.n_local};
  const int r0_end = min(win.sink_end, i_q + 1);
  const int r1_lo = max(win.lo(i_q), r0_end);
  float qv[QPL];
  const __nv_bfloat16* qp = p.q + ((int64_t)seq * p.n_heads + h) * DQK;
#pragma unroll
  for (int e = 0; e < QPL; ++e) qv[e] = __bfloat162float(qp[lane + 32 * e]);
  float m = -INFINITY, l = 0.f, acc[VPL];
#pragma unroll
  for (int e = 0; e < VPL; ++e) acc[e] = 0.f;
  // keys of the window (the sink range, then the local range), warp w takes every 4th key
  for (int range = 0; range < 2; ++range) {
    const int t_lo = range == 0 ? 0 : r1_lo;
    const int t_end = range == 0 ? r0_end : i_q + 1;
    for (int t = t_lo + warp; t < t_end; t += 4) {
      const __nv_bfloat16* kp = p.k + seq * p.k_batch_stride + (int64_t)t * p.k_row_stride + (int64_t)hk * DQK;
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < QPL; ++e) s += qv[e] * __bfloat162float(kp[lane + 32 * e]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      s *= p.scale_log2;
      const float mn = fmaxf(m, s);
      const float a = exp2f(m - mn);
      const float pw = exp2f(s - mn);
      const __nv_bfloat16* vp = p.v + seq * p.v_batch_stride + (int64_t)t * p.v_row_stride + (int64_t)hk * DV;
#pragma unroll
      for (int e = 0; e < VPL; ++e) acc[e] = acc[e] * a + pw * __bfloat162float(vp[lane + 32 * e]);
      l = l * a + pw;
      m = mn;
    }
  }
  __shared__ float sm_m[4], sm_l[4], sm_o[4][DV];
  if (lane == 0) { sm_m[warp] = m; sm_l[warp] = l; }
#pragma unroll
  for (int e = 0; e < VPL; ++e) sm_o[warp][lane + 32 * e] = acc[e];
  __syncthreads();
  const float mm = fmaxf(fmaxf(sm_m[0], sm_m[1]), fmaxf(sm_m[2], sm_m[3]));
  float w[4], lt = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[i] = sm_l[i] > 0.f ? exp2f(sm_m[i] - mm) : 0.f;
    lt += sm_l[i] * w[i];
  }
  for (int d = threadIdx.x; d < DV; d += 128) {
    float o = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) o += sm_o[i][d] * w[i];
    p.out[((int64_t)seq * p.n_heads + h) * DV + d] = __float2bfloat16_rn(o / lt);
  }
  if (threadIdx.x == 0) p.lse[(int64_t)seq * p.n_heads + h] = (mm + log2f(lt)) * 0.69314718055994530942f;
}

}  // namespace loza
