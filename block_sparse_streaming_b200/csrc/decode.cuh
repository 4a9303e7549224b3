// decode.cuh - SSA decode on sm_100a.
//
// Decode runs one new query token per sequence: the token at position
// i = L-1 attends to the keys its window selects (sink blocks plus the l most
// recent blocks, causal inside its own block; page 1 section 01 of the LoZA
// pages, and section 02 for the decode use of the streaming kernel).
//
// (1) ssa_decode_mla_kernel - absorbed MLA: every head reads the same latent
//     row (576 = 512 + 64 rope; V = first 512 columns), so one key block
//     against all heads is a real GEMM and runs on tcgen05 with keys on M:
//       S^T [128 keys x H] = K_blk [128 x 576] . Q^T          (K-major A and B)
//       O^T [512 x H]     += V_blk^T [512 x 128] . P^T        (MN-major A = the
//                                                              same K_blk tiles)
//     A CTA owns `bps` consecutive selected blocks of one sequence (split-KV);
//     each block is loaded whole into shared memory (9 TMA tiles), S^T is
//     computed as the tiles land, the softmax over keys is a column reduction
//     (shuffle reduce-scatter + a 4-warp combine in shared memory), P^T goes to
//     shared memory and O^T stays in TMEM. The partials (O, m, l) of a
//     sequence's splits are merged with the log-sum-exp rule:
//       - sink + local window (<= 8 blocks, one per CTA): the 8 CTAs of a
//         sequence form a thread-block cluster; each stages its partial O in
//         its own shared memory and then merges one 64-column slice of the
//         output by reading all 8 partials over distributed shared memory, so
//         no partial ever leaves the chip;
//       - unbounded window (dense baseline, up to 32 splits of many blocks):
//         partials go to the workspace and the last CTA of a sequence (atomic
//         ticket, no waiting) merges them.
// (2) ssa_decode_mha_kernel - per-head K/V (d = 64 or 192/128): one query
//     vector per head against <= 1024 keys is a matrix-vector product, so it
//     runs on CUDA cores: 4 warps per (sequence, head), online softmax per
//     warp, merged through shared memory.
#pragma once

#include <cuda.h>

#include "sm100.cuh"

namespace loza {

constexpr int kDecHeads = 64;          // N of the decode MMAs (query heads)
constexpr int kDecThreads = 192;
constexpr int kDecQChunk = 64 * 64 * 2;  // [64 heads x 64 dims] bf16
constexpr int kDecQBytes = 9 * kDecQChunk;
constexpr int kDecKvBytes = 9 * kChunkBytes;

struct DecodeParams {
  CUtensorMap tm_q;    // q [B, H, 576]       box {64, 64, 1}
  CUtensorMap tm_kv;   // cache [B, rows, 576] box {64, 128, 1}
  const int32_t* seqlens;
  float* ws_o;         // [B, nsplit, H, 512] partial O (unnormalised)
  float2* ws_ml;       // [B, nsplit, H] partial (m in log2 units, l)
  int* ws_ticket;      // [B] arrival counters (zero on entry)
  __nv_bfloat16* out;  // [B, H, 512]
  float* lse;          // [B, H]
  int nsplit;
  int bps;             // selected blocks per split
  int n_sink;
  int n_local;         // < 0: unbounded
  float scale_log2;
};

struct DecodeLayout {
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = kDecQBytes;                 // 73728, 1024-aligned
  static constexpr int P_OFF = KV_OFF + 8 * kChunkBytes;    // P^T reuses the rope tile
  static constexpr int RED_OFF = KV_OFF + kDecKvBytes;      // [8][64] floats (reductions, merge weights)
  static constexpr int STAT_OFF = RED_OFF + 8 * 64 * 4;     // m_run[64], l_run[64], alpha[64]
  static constexpr int BAR_OFF = STAT_OFF + 3 * 64 * 4;
  // barriers: q_full, kv_full[9], s_full, p_ready, pv_done
  static constexpr int BAR_Q = 0, BAR_KV = 1, BAR_S = 10, BAR_P = 11, BAR_PV = 12, NBAR = 13;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem base, abort, last-CTA flag
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Reduce 64 per-thread values across the 32 lanes of a warp by halving
// exchanges (reduce-scatter): returns the two column results this lane ends
// up owning, for columns col0 and col0 + 1.
template <bool IS_MAX>
__device__ __forceinline__ void warp_reduce_scatter64(const float (&v)[64], float& r0, float& r1, int& col0) {
  const int lane = threadIdx.x & 31;
  float a[32];
  {
    const bool hi = lane & 16;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float send = hi ? v[i] : v[32 + i];
      const float keep = hi ? v[32 + i] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
      a[i] = IS_MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  float b[16];
  {
    const bool hi = lane & 8;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float send = hi ? a[i] : a[16 + i];
      const float keep = hi ? a[16 + i] : a[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 8);
      b[i] = IS_MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  float c[8];
  {
    const bool hi = lane & 4;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float send = hi ? b[i] : b[8 + i];
      const float keep = hi ? b[8 + i] : b[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 4);
      c[i] = IS_MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  float d[4];
  {
    const bool hi = lane & 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float send = hi ? c[i] : c[4 + i];
      const float keep = hi ? c[4 + i] : c[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 2);
      d[i] = IS_MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  {
    const bool hi = lane & 1;
    float e[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float send = hi ? d[i] : d[2 + i];
      const float keep = hi ? d[2 + i] : d[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
      e[i] = IS_MAX ? fmaxf(keep, recv) : keep + recv;
    }
    r0 = e[0];
    r1 = e[1];
  }
  col0 = ((lane >> 4) & 1) * 32 + ((lane >> 3) & 1) * 16 + ((lane >> 2) & 1) * 8 + ((lane >> 1) & 1) * 4 +
         (lane & 1) * 2;
}

template <bool CLUSTER>
__global__ void __launch_bounds__(kDecThreads, 1) ssa_decode_mla_kernel(const __grid_constant__ DecodeParams p) {
  using LY = DecodeLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int split = blockIdx.x;
  const int seq = blockIdx.y;
  const int L = p.seqlens[seq];
  const int i_q = L - 1;                 // decode query position
  const int jq = i_q / kTile;            // its block
  const BlockWalk walk(jq, p.n_sink, p.n_local);
  const int b_lo = split * p.bps;
  const int b_hi = min(walk.count, b_lo + p.bps);
  const int nb = max(0, b_hi - b_lo);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + LY::BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 4);
  int* last_flag = reinterpret_cast<int*>(smem + LY::MISC_OFF + 8);
  float* red = reinterpret_cast<float*>(smem + LY::RED_OFF);
  float* m_run = reinterpret_cast<float*>(smem + LY::STAT_OFF);
  float* l_run = m_run + 64;
  float* alpha = m_run + 128;
  const int64_t part = (int64_t)seq * p.nsplit + split;

  if (threadIdx.x == 0) {
    mbar_init(bar(LY::BAR_Q), 1);
    for (int c = 0; c < 9; ++c) mbar_init(bar(LY::BAR_KV + c), 1);
    mbar_init(bar(LY::BAR_S), 1);
    mbar_init(bar(LY::BAR_P), 128);
    mbar_init(bar(LY::BAR_PV), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 64) {
    m_run[threadIdx.x] = -INFINITY;
    l_run[threadIdx.x] = 0.f;
  }
  if (warp == 1 && nb > 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = nb > 0 ? *tmem_slot : 0;

  if (nb > 0) {
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_kv);
        mbar_arrive_expect_tx(bar(LY::BAR_Q), kDecQBytes);
        for (int c = 0; c < 9; ++c)
          tma_load_3d(sbase + LY::Q_OFF + c * kDecQChunk, &p.tm_q, bar(LY::BAR_Q), c * 64, 0, seq);
        bool ok = true;
        for (int b = 0; b < nb && ok; ++b) {
          if (b > 0) ok = mbar_wait(bar(LY::BAR_PV), (b - 1) & 1, abort_flag);  // block b-1 fully consumed
          if (!ok) break;
          const int krow = walk.block(b_lo + b) * kTile;
          for (int c = 0; c < 9; ++c) {
            mbar_arrive_expect_tx(bar(LY::BAR_KV + c), kChunkBytes);
            tma_load_3d(sbase + LY::KV_OFF + c * kChunkBytes, &p.tm_kv, bar(LY::BAR_KV + c), c * 64, krow, seq);
          }
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc_s = idesc_bf16(128, kDecHeads, false, false);
        constexpr uint32_t idesc_o = idesc_bf16(128, kDecHeads, true, false);
        const uint32_t tmem_s = tmem;          // S^T: 64 columns
        const uint32_t tmem_o = tmem + 64;     // O^T: 4 x 64 columns
        bool ok = mbar_wait(bar(LY::BAR_Q), 0, abort_flag);
        for (int b = 0; b < nb && ok; ++b) {
          for (int c = 0; c < 9; ++c) {
            ok = mbar_wait(bar(LY::BAR_KV + c), b & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const uint32_t ka = sbase + LY::KV_OFF + c * kChunkBytes;
            const uint32_t qb = sbase + LY::Q_OFF + c * kDecQChunk;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem_s, sdesc_sw128(ka + 32 * kk, 16, 1024), sdesc_sw128(qb + 32 * kk, 16, 1024), idesc_s,
                     (c | kk) != 0);
          }
          if (!ok) break;
          mma_commit(bar(LY::BAR_S));
          ok = mbar_wait(bar(LY::BAR_P), b & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          // O^T[dv chunk c] += V^T (dims 128c..128c+127 = K tiles 2c, 2c+1) . P^T
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            const uint32_t va = sbase + LY::KV_OFF + (2 * c) * kChunkBytes;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t pb = sbase + LY::P_OFF + (kk >> 2) * kDecQChunk + (kk & 3) * 32;
              mma_ss(tmem_o + 64 * c, sdesc_sw128(va + 2048 * kk, kChunkBytes, 1024), sdesc_sw128(pb, 16, 1024),
                     idesc_o, (b > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(bar(LY::BAR_PV));
        }
      }
    } else {
      // ---------------------------------------------------------- softmax over keys
      const int quarter = warp & 3;
      const int key = quarter * 32 + lane;  // TMEM lane == key row of the block
      const int tid = threadIdx.x - 64;      // 0..127
      const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
      bool ok = true;
      for (int b = 0; b < nb && ok; ++b) {
        ok = mbar_wait(bar(LY::BAR_S), b & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        float x[64];
        {
          float t[32];
          tmem_ld32(lane_addr + 0, t);
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = t[i];
          tmem_ld32(lane_addr + 32, t);
#pragma unroll
          for (int i = 0; i < 32; ++i) x[32 + i] = t[i];
        }
        const int kb = walk.block(b_lo + b);
        const int tpos = kb * kTile + key;
        const bool valid = tpos <= i_q;
#pragma unroll
        for (int h = 0; h < 64; ++h) x[h] = valid ? x[h] * p.scale_log2 : -INFINITY;
        // column (head) maxima over the 128 keys
        {
          float r0, r1;
          int col0;
          warp_reduce_scatter64<true>(x, r0, r1, col0);
          red[quarter * 64 + col0] = r0;
          red[quarter * 64 + col0 + 1] = r1;
        }
        // keys past the sequence end: zero their V rows (the cache may hold
        // anything there) so that 0 * garbage cannot reach the accumulator
        if (!valid) {
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4* row = reinterpret_cast<uint4*>(smem + LY::KV_OFF + c * kChunkBytes + key * 128);
#pragma unroll
            for (int u = 0; u < 8; ++u) row[u] = z;
          }
        }
        named_barrier_sync(1, 128);
        if (b > 0) {
          ok = mbar_wait(bar(LY::BAR_PV), (b - 1) & 1, abort_flag);  // P^T and O^T free
          if (!ok) break;
          tc_fence_after();
        }
        if (tid < 64) {
          const float mb = fmaxf(fmaxf(red[tid], red[64 + tid]), fmaxf(red[128 + tid], red[192 + tid]));
          const float mo = m_run[tid];
          float a = 1.f, mn = mo;
          if (b == 0) {
            mn = mb;
          } else if (mb > mo + (float)kRescaleThreshold) {
            a = exp2f(mo - mb);
            mn = mb;
          }
          m_run[tid] = mn;
          alpha[tid] = a;
        }
        named_barrier_sync(1, 128);
        // P^T = 2^(x - m) into shared memory as the K-major B operand [64 heads x 128 keys]
        {
          uint8_t* pbase = smem + LY::P_OFF + (key >> 6) * kDecQChunk;
          const uint32_t col = key & 63;
#pragma unroll
          for (int h = 0; h < 64; ++h) {
            const float pv = exp2f(x[h] - m_run[h]);
            x[h] = pv;
            *reinterpret_cast<__nv_bfloat16*>(pbase + sw128_offset(h, col)) = __float2bfloat16_rn(pv);
          }
        }
        {
          float r0, r1;
          int col0;
          warp_reduce_scatter64<false>(x, r0, r1, col0);
          red[quarter * 64 + col0] = r0;
          red[quarter * 64 + col0 + 1] = r1;
        }
        // O^T rescale where a head's running max moved (rare): lane = dv row
        bool any_rescale = false;
#pragma unroll 1
        for (int h = 0; h < 64; ++h) any_rescale |= (alpha[h] != 1.f);
        if (b > 0 && any_rescale) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
              float o[32];
              tmem_ld32(lane_addr + 64 + 64 * c + 32 * hh, o);
              uint32_t w[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(o[i] * alpha[32 * hh + i]);
              tmem_st32(lane_addr + 64 + 64 * c + 32 * hh, w);
            }
          }
          tmem_st_wait();
        }
        named_barrier_sync(1, 128);
        if (tid < 64)
          l_run[tid] = l_run[tid] * alpha[tid] + (red[tid] + red[64 + tid] + red[128 + tid] + red[192 + tid]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(LY::BAR_P));
      }
      // ---------------------------------------------------------- partial epilogue
      if (ok) ok = mbar_wait(bar(LY::BAR_PV), (nb - 1) & 1, abort_flag);
      if (ok) {
        tc_fence_after();
        named_barrier_sync(1, 128);  // l_run complete
        // CLUSTER: stage O^T as [head][512] fp32 over the (now idle) K/V tiles;
        // otherwise write it to this split's workspace slot.
        float* so = reinterpret_cast<float*>(smem + LY::KV_OFF);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const int dv = 128 * c + key;
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            float o[32];
            tmem_ld32(lane_addr + 64 + 64 * c + 32 * hh, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (CLUSTER)
                so[(32 * hh + i) * 512 + dv] = o[i];
              else
                p.ws_o[(part * kDecHeads + 32 * hh + i) * 512 + dv] = o[i];
            }
          }
        }
        if (!CLUSTER && tid < 64) p.ws_ml[part * kDecHeads + tid] = make_float2(m_run[tid], l_run[tid]);
      }
    }
  } else if (!CLUSTER && threadIdx.x < 64) {
    // no block for this split: an empty partial
    p.ws_ml[part * kDecHeads + threadIdx.x] = make_float2(-INFINITY, 0.f);
  }

  if (CLUSTER) {
    // ---------------------------------------------------------- on-chip merge
    // Split r of the cluster merges output columns [r*W, (r+1)*W) of every head,
    // W = 512 / nsplit, reading the partials of all splits over DSMEM. Splits
    // without a block have l = 0 and weight 0 (their staging area is not read).
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    const int r = (int)cluster_rank();
    constexpr int NS = 8;  // splits per cluster (== cluster size)
    float* wgt = red;      // [NS][64] merge weights
    float* mls = reinterpret_cast<float*>(smem + LY::Q_OFF);  // [2][NS][64] peers' m, l (Q tiles are idle now)
    for (int idx = threadIdx.x; idx < NS * 64; idx += blockDim.x) {
      const int s2 = idx >> 6, h = idx & 63;
      const float* pm = static_cast<const float*>(__cluster_map_shared_rank(m_run + h, s2));
      const float* pl = static_cast<const float*>(__cluster_map_shared_rank(l_run + h, s2));
      mls[idx] = *pm;
      mls[NS * 64 + idx] = *pl;
    }
    __syncthreads();
    if (threadIdx.x < 64) {
      const int h = threadIdx.x;
      float M = -INFINITY;
#pragma unroll
      for (int s2 = 0; s2 < NS; ++s2)
        if (mls[NS * 64 + s2 * 64 + h] > 0.f) M = fmaxf(M, mls[s2 * 64 + h]);
      float Ls = 0.f, w[NS];
#pragma unroll
      for (int s2 = 0; s2 < NS; ++s2) {
        const float l = mls[NS * 64 + s2 * 64 + h];
        w[s2] = l > 0.f ? exp2f(mls[s2 * 64 + h] - M) : 0.f;
        Ls += l * w[s2];
      }
      const float inv = 1.f / Ls;
#pragma unroll
      for (int s2 = 0; s2 < NS; ++s2) wgt[s2 * 64 + h] = w[s2] * inv;
      if (r == 0) p.lse[(int64_t)seq * kDecHeads + h] = (M + log2f(Ls)) * 0.69314718055994530942f;
    }
    __syncthreads();
    constexpr int W = 512 / NS;  // output columns this split merges
    const float* so = reinterpret_cast<const float*>(smem + LY::KV_OFF);
    for (int idx = threadIdx.x; idx < kDecHeads * (W / 4); idx += blockDim.x) {
      const int h = idx / (W / 4);
      const int d = r * W + (idx % (W / 4)) * 4;
      float4 o[NS];
#pragma unroll
      for (int s2 = 0; s2 < NS; ++s2) {
        // a split without a block has weight 0 and an unwritten staging area: do not read it
        o[s2] = wgt[s2 * 64 + h] != 0.f
                    ? *static_cast<const float4*>(__cluster_map_shared_rank(so + h * 512 + d, s2))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int s2 = 0; s2 < NS; ++s2) {
        const float w = wgt[s2 * 64 + h];
        acc.x += o[s2].x * w;
        acc.y += o[s2].y * w;
        acc.z += o[s2].z * w;
        acc.w += o[s2].w * w;
      }
      __nv_bfloat16* dst = p.out + ((int64_t)seq * kDecHeads + h) * 512 + d;
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
    }
    cluster_sync_all();  // peers may still read this CTA's shared memory until here
    if (warp == 1 && nb > 0) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
    return;
  }

  // ------------------------------------------------------------ last CTA merges
  __threadfence();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) *last_flag = (atomicAdd(&p.ws_ticket[seq], 1) == p.nsplit - 1);
  __syncthreads();
  if (*last_flag) {
    __threadfence();
    // merge weights per (split, head) once, then stream the partials
    float* wgt = reinterpret_cast<float*>(smem + LY::KV_OFF);  // [nsplit][64], K/V tiles are idle now
    if (threadIdx.x < 64) {
      const int h = threadIdx.x;
      float M = -INFINITY;
      for (int s2 = 0; s2 < p.nsplit; ++s2) {
        const float2 ml = p.ws_ml[((int64_t)seq * p.nsplit + s2) * kDecHeads + h];
        if (ml.y > 0.f) M = fmaxf(M, ml.x);
      }
      float Ls = 0.f;
      for (int s2 = 0; s2 < p.nsplit; ++s2) {
        const float2 ml = p.ws_ml[((int64_t)seq * p.nsplit + s2) * kDecHeads + h];
        const float w = ml.y > 0.f ? exp2f(ml.x - M) : 0.f;
        wgt[s2 * 64 + h] = w;
        Ls += ml.y * w;
      }
      const float inv = 1.f / Ls;
      for (int s2 = 0; s2 < p.nsplit; ++s2) wgt[s2 * 64 + h] *= inv;
      p.lse[(int64_t)seq * kDecHeads + h] = (M + log2f(Ls)) * 0.69314718055994530942f;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < kDecHeads * 128; idx += blockDim.x) {
      const int h = idx >> 7;
      const int d4 = (idx & 127) * 4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
      for (int s2 = 0; s2 < p.nsplit; ++s2) {
        const float w = wgt[s2 * 64 + h];
        const float4 o = *reinterpret_cast<const float4*>(p.ws_o + (((int64_t)seq * p.nsplit + s2) * kDecHeads + h) * 512 + d4);
        if (w != 0.f) {
          acc.x += o.x * w;
          acc.y += o.y * w;
          acc.z += o.z * w;
          acc.w += o.w * w;
        }
      }
      __nv_bfloat16* dst = p.out + ((int64_t)seq * kDecHeads + h) * 512 + d4;
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
    }
    if (threadIdx.x == 0) p.ws_ticket[seq] = 0;  // ready for the next call
  }
  if (warp == 1 && nb > 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

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
  const BlockWalk walk(i_q / kTile, p.n_sink, p.n_local);
  float qv[QPL];
  const __nv_bfloat16* qp = p.q + ((int64_t)seq * p.n_heads + h) * DQK;
#pragma unroll
  for (int e = 0; e < QPL; ++e) qv[e] = __bfloat162float(qp[lane + 32 * e]);
  float m = -INFINITY, l = 0.f, acc[VPL];
#pragma unroll
  for (int e = 0; e < VPL; ++e) acc[e] = 0.f;
  // keys of the window, warp w takes every 4th key
  for (int b = 0; b < walk.count; ++b) {
    const int kb = walk.block(b);
    const int t_end = min(kb * kTile + kTile, i_q + 1);
    for (int t = kb * kTile + warp; t < t_end; t += 4) {
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
