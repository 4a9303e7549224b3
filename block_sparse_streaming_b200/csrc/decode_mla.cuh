// decode_mla.cuh - absorbed-MLA SSA decode on sm_100a (tcgen05 + TMA), streaming.
//
// One new query token per sequence, at position i = L-1, attends to the keys
// its window selects (sink blocks plus the l most recent blocks, causal inside
// its own block; page 1 section 01 of the LoZA pages, and section 02 for the
// streaming kernel in decode). In absorbed MLA every head reads the same
// 576-wide latent row (V = its first 512 columns), so one key block against
// all 64 heads is a real GEMM; it runs on tcgen05 with the 128 keys of a
// block on M and the 64 heads on N:
//     S^T [128 keys x 64] = K_blk [128 x 576] . Q^T       (K-major A and B)
//     O^T [512 x 64]     += V_blk^T [512 x 128] . P^T     (MN-major A)
//
// Work split: the selected blocks of a sequence are divided among `nsplit`
// CTAs (`bps` consecutive blocks each) so that batch * nsplit CTAs fill the
// GPU in one wave. A CTA streams its blocks through a 4-unit TMA ring (one
// unit = 128 rows x 128 latent columns, 32 KB) in the order
//     K(0) K(1) V(0) K(2) V(1) ...        (K = 5 units, V = 4 units per block)
// so that S^T of the next block is computed while the softmax of this one
// runs. V units are the first 512 columns of the same rows, re-read from L2.
// The softmax over keys is a column reduction done by 8 warps (two per TMEM
// lane quarter, 32 heads each): a shuffle reduce-scatter per warp plus a
// 4-quarter combine in shared memory. O^T accumulates across the CTA's blocks
// in TMEM with an online softmax (rescaled only when a head's maximum grows
// by more than 2^8).
//
// Merge of the splits of a sequence (log-sum-exp rule):
//   CLUSTER  = true : the nsplit (<= 4) CTAs of a sequence form a thread-block
//                     cluster; after exchanging (m, l), each stages its
//                     weighted partial O (from TMEM) for the columns the other
//                     CTAs own in its shared memory and moves each part with
//                     one DSMEM bulk copy, and each CTA sums its 512/nsplit
//                     columns. The decode plan uses it with one CTA per
//                     sequence (large batches), which writes all columns.
//   CLUSTER  = false: partials go to the workspace and the last CTA of the
//                     sequence (atomic ticket, no waiting) merges them; used
//                     when a few long sequences need more than 8 splits.
// Batches of at most half as many sequences as SMs use the half-block kernel
// (decode_mla_hb.cuh) instead, which reads every selected row once; this
// kernel then runs either as one CTA per sequence (no merge) or with many
// splits merged through the workspace.
#pragma once

#include <cuda.h>

#include "sm100.cuh"

namespace loza {

constexpr int kDecHeads = 64;            // N of the decode MMAs (query heads)
constexpr int kDecThreads = 320;         // producer, MMA, 8 softmax warps
constexpr int kDecQTile = 64 * 64 * 2;   // [64 heads x 64 dims] bf16
constexpr int kDecUnit = 2 * kChunkBytes;  // [128 rows x 128 dims] bf16 as two [128 x 64] tiles
constexpr int kDecStages = 4;
constexpr int kDecKUnits = 5;            // 576 columns: 4 full units + the 64-column rope part
constexpr int kDecVUnits = 4;            // 512 columns

struct DecodeParams {
  CUtensorMap tm_q;    // q [B, H, 576]       box {64, 64, 1}
  CUtensorMap tm_kv;   // cache [B, rows, 576] box {64, 128, 1}; paged: the pool [1, pages * 128, 576]
  CUtensorMap tm_kv64; // the same tensor with box {64, 64, 1} (half blocks)
  // 4-D views {64 columns, rows, 9 column tiles, batch} (tile stride 128 B):
  CUtensorMap tm_q3;   // q, box {64, 64 heads, 3, 1}: three Q tiles per request
  CUtensorMap tm_kv3;  // cache, box {64, 64 rows, 3, 1}: three half-block tiles per request
  const int32_t* seqlens;
  const int32_t* block_table;  // paged cache: [B, bt_stride] pool page of each logical block; nullptr: contiguous
  int bt_stride;
  float* ws_o;         // workspace mode: [B, nsplit, H, 512] partial O (unnormalised)
  float4* ws_ml;       // workspace mode: [B, nsplit, H] partial (m in log2 units, l exact, l of bf16 P, -)
  int* ws_ticket;      // workspace mode: [B] arrival counters (zero on entry)
  __nv_bfloat16* out;  // [B, H, 512]
  float* lse;          // [B, H]
  int nsplit;
  int bps;             // selected blocks per split
  int n_sink;
  int n_local;         // < 0: unbounded
  int block;           // b, tokens per block of the window
  float scale_log2;
};

// TMA coordinates (row, batch) of logical block kb of sequence seq: in the
// sequence's own cache, or on its page of a paged pool (pages of 128 rows).
__device__ __forceinline__ int2 dec_block_rows(const DecodeParams& p, int seq, int kb) {
  if (p.block_table) return make_int2(p.block_table[(int64_t)seq * p.bt_stride + kb] * kTile, 0);
  return make_int2(kb * kTile, seq);
}

struct DecodeLayout {
  static constexpr int Q_OFF = 0;                                   // 9 Q tiles, 72 KB
  static constexpr int RING_OFF = 9 * kDecQTile;                    // 73728 (1024-aligned)
  static constexpr int P_OFF = RING_OFF + kDecStages * kDecUnit;    // P^T: [128 keys x 64 heads], heads contiguous
  static constexpr int RED_OFF = P_OFF + 2 * kDecQTile;             // redmax, redsum, redrsum [4][64] each
  static constexpr int STAT_OFF = RED_OFF + 3 * 4 * 64 * 4;         // m_run, l_run, alpha, r_run [64] each
  static constexpr int BAR_OFF = STAT_OFF + 4 * 64 * 4;
  // barriers: q_full, full[4], empty[4], s_full[2], p_ready, pv_done, vtail (the block holding
  // the query's own, possibly partial, block has all its V units resident)
  static constexpr int BAR_Q = 0, BAR_FULL = 1, BAR_EMPTY = 1 + kDecStages, BAR_S = 1 + 2 * kDecStages,
                       BAR_P = BAR_S + 2, BAR_PV = BAR_P + 1, BAR_VT = BAR_PV + 1,
                       BAR_MRG = BAR_VT + 1,  // on-chip merge: the other splits' parts have arrived
                       NBAR = BAR_MRG + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem base, abort, last-CTA flag
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(kDecStages * kDecUnit >= kDecHeads * 512 * 4, "partial-O staging reuses the ring");
};

// Sum / max of 32 per-lane values across a warp by halving exchanges
// (reduce-scatter): lane j returns the reduction of column j.
template <bool IS_MAX>
__device__ __forceinline__ float warp_reduce_scatter32(const float (&v)[32]) {
  const int lane = threadIdx.x & 31;
  float a[16];
  {
    const bool hi = lane & 16;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float send = hi ? v[i] : v[16 + i];
      const float keep = hi ? v[16 + i] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
      a[i] = IS_MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  float b[8];
  {
    const bool hi = lane & 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float send = hi ? a[i] : a[8 + i];
      const float keep = hi ? a[8 + i] : a[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 8);
      b[i] = IS_MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  float c[4];
  {
    const bool hi = lane & 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float send = hi ? b[i] : b[4 + i];
      const float keep = hi ? b[4 + i] : b[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 4);
      c[i] = IS_MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  float d[2];
  {
    const bool hi = lane & 2;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float send = hi ? c[i] : c[2 + i];
      const float keep = hi ? c[2 + i] : c[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 2);
      d[i] = IS_MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  const bool hi = lane & 1;
  const float send = hi ? d[0] : d[1];
  const float keep = hi ? d[1] : d[0];
  const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
  return IS_MAX ? fmaxf(keep, recv) : keep + recv;
}

// Ring position (in units) of V unit u of CTA-local block b, given nb blocks:
// K units of blocks 0 .. min(b+1, nb-1) and V units of blocks 0 .. b-1 precede it.
__device__ __forceinline__ int dec_v_pos(int b, int u, int nb) {
  return kDecKUnits * min(b + 2, nb) + kDecVUnits * b + u;
}

template <bool CLUSTER>
__global__ void __launch_bounds__(kDecThreads, 1) ssa_decode_mla_kernel(const __grid_constant__ DecodeParams p) {
  using LY = DecodeLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int split = blockIdx.x;
  const int seq = blockIdx.y;
  griddep_wait();  // in a chain of launches, the sequence lengths and cache rows may come from the kernel before
  const int L = p.seqlens[seq];
  const int i_q = L - 1;                 // decode query position
  const int jq = i_q / kTile;            // its block
  // the 128-row units of the window of position i_q (the own block last)
  const SsaWindow win{p.block, p.n_sink * p.block, p.n_local};
  const RowWalk walk(win, i_q, kTile);
  const int lo_q = win.lo(i_q);
  const int b_lo = split * p.bps;
  const int nb = max(0, min(walk.count, b_lo + p.bps) - b_lo);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + LY::BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 4);
  int* last_flag = reinterpret_cast<int*>(smem + LY::MISC_OFF + 8);
  float* redmax = reinterpret_cast<float*>(smem + LY::RED_OFF);  // [4 quarters][64]
  float* redsum = redmax + 4 * 64;   // sums of exact P (for the LSE)
  float* redrsum = redsum + 4 * 64;  // sums of bf16-rounded P (for normalising O)
  float* m_run = reinterpret_cast<float*>(smem + LY::STAT_OFF);
  float* l_run = m_run + 64;
  float* r_run = m_run + 192;
  float* alpha = m_run + 128;
  const int64_t part = (int64_t)seq * p.nsplit + split;

  if (threadIdx.x == 0) {
    mbar_init(bar(LY::BAR_Q), 1);
    for (int i = 0; i < kDecStages; ++i) {
      mbar_init(bar(LY::BAR_FULL + i), 1);
      mbar_init(bar(LY::BAR_EMPTY + i), 1);
    }
    mbar_init(bar(LY::BAR_S + 0), 1);
    mbar_init(bar(LY::BAR_S + 1), 1);
    mbar_init(bar(LY::BAR_P), 8);  // one arrival per softmax warp
    mbar_init(bar(LY::BAR_PV), 1);
    mbar_init(bar(LY::BAR_VT), 1);
    mbar_init(bar(LY::BAR_MRG), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 64) {
    m_run[threadIdx.x] = -INFINITY;
    l_run[threadIdx.x] = 0.f;
    r_run[threadIdx.x] = 0.f;
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
      // whole warp walks the schedule; one elected lane issues the TMA loads
      if (elect_one()) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_kv);
        mbar_arrive_expect_tx(bar(LY::BAR_Q), 9 * kDecQTile);
        for (int c = 0; c < 9; ++c)
          tma_load_3d(sbase + LY::Q_OFF + c * kDecQTile, &p.tm_q, bar(LY::BAR_Q), c * 64, 0, seq);
      }
      __syncwarp();
      int slot = 0;
      uint32_t phase = 0;
      bool ok = true;
      auto load_unit = [&](int2 rz, int u) {
        ok = warp_wait(bar(LY::BAR_EMPTY + slot), phase ^ 1, abort_flag);
        if (!ok) return;
        if (elect_one()) {
          const uint32_t dst = sbase + LY::RING_OFF + slot * kDecUnit;
          const int ntile = (u < 4) ? 2 : 1;
          mbar_arrive_expect_tx(bar(LY::BAR_FULL + slot), ntile * kChunkBytes);
          for (int t = 0; t < ntile; ++t)
            tma_load_3d(dst + t * kChunkBytes, &p.tm_kv, bar(LY::BAR_FULL + slot), 128 * u + 64 * t, rz.x, rz.y);
        }
        __syncwarp();
        if (++slot == kDecStages) { slot = 0; phase ^= 1; }
      };
      for (int it = 0; it <= nb && ok; ++it) {
        if (it < nb) {
          const int2 krow = dec_block_rows(p, seq, walk.unit_at(b_lo + it));
          for (int u = 0; u < kDecKUnits && ok; ++u) load_unit(krow, u);
        }
        if (it >= 1) {
          const int2 vrow = dec_block_rows(p, seq, walk.unit_at(b_lo + it - 1));
          for (int u = 0; u < kDecVUnits && ok; ++u) load_unit(vrow, u);
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      // whole warp walks the schedule with warp-uniform descriptors; one
      // elected lane issues each tcgen05 instruction
      constexpr uint32_t idesc_s = idesc_bf16(128, kDecHeads, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(128, kDecHeads, true, true);
      const uint32_t tmem_o = tmem + 128;  // O^T: 4 x 64 columns after the two S^T buffers
      const uint64_t dk0 = sdesc_sw128(sbase + LY::RING_OFF, 16, 1024);           // K tiles, K-major
      const uint64_t dq0 = sdesc_sw128(sbase + LY::Q_OFF, 16, 1024);              // Q tiles, K-major
      const uint64_t dv0 = sdesc_sw128(sbase + LY::RING_OFF, kChunkBytes, 1024);  // V unit, MN-major
      const uint64_t dp0 = sdesc_sw128(sbase + LY::P_OFF, 8192, 1024);            // P^T, MN-major (heads contiguous)
      int slot = 0;
      uint32_t phase = 0;
      bool ok = warp_wait(bar(LY::BAR_Q), 0, abort_flag);
      for (int it = 0; it <= nb && ok; ++it) {
        if (it < nb) {
          // S^T(it) = K . Q^T over 9 column tiles
          const uint32_t tmem_s = tmem + 64 * (it & 1);
          for (int u = 0; u < kDecKUnits && ok; ++u) {
            ok = warp_wait(bar(LY::BAR_FULL + slot), phase, abort_flag);
            if (!ok) break;
            tc_fence_after();
            if (elect_one()) {
              for (int t = 0; t < ((u < 4) ? 2 : 1); ++t) {
                const int c = 2 * u + t;
                const uint64_t da = desc_add(dk0, slot * kDecUnit + t * kChunkBytes);
                const uint64_t db = desc_add(dq0, c * kDecQTile);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_ss(tmem_s, desc_add(da, 32 * kk), desc_add(db, 32 * kk), idesc_s, (c | kk) != 0);
              }
              mma_commit(bar(LY::BAR_EMPTY + slot));
            }
            __syncwarp();
            if (++slot == kDecStages) { slot = 0; phase ^= 1; }
          }
          if (!ok) break;
          if (elect_one()) mma_commit(bar(LY::BAR_S + (it & 1)));
          __syncwarp();
        }
        if (it >= 1) {
          // O^T += V^T . P^T(b), V unit u = latent columns 128u .. 128u+127
          const int b = it - 1;
          if (walk.unit_at(b_lo + b) == jq) {
            // the query's own block may end inside the block: once its V units
            // are resident, let the softmax warps zero the rows past the end
            for (int u = 0; u < kDecVUnits && ok; ++u) {
              const int su = slot + u;
              ok = warp_wait(bar(LY::BAR_FULL + su % kDecStages), phase ^ (su >= kDecStages ? 1u : 0u), abort_flag);
            }
            if (!ok) break;
            if (elect_one()) mbar_arrive(bar(LY::BAR_VT));
            __syncwarp();
          }
          ok = warp_wait(bar(LY::BAR_P), b & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          for (int u = 0; u < kDecVUnits && ok; ++u) {
            ok = warp_wait(bar(LY::BAR_FULL + slot), phase, abort_flag);
            if (!ok) break;
            tc_fence_after();
            if (elect_one()) {
              const uint64_t da = desc_add(dv0, slot * kDecUnit);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma_ss(tmem_o + 64 * u, desc_add(da, 2048 * kk), desc_add(dp0, 2048 * kk), idesc_o,
                       (b > 0 || kk > 0) ? 1u : 0u);
              mma_commit(bar(LY::BAR_EMPTY + slot));
            }
            __syncwarp();
            if (++slot == kDecStages) { slot = 0; phase ^= 1; }
          }
          if (!ok) break;
          if (elect_one()) mma_commit(bar(LY::BAR_PV));
          __syncwarp();
        }
      }
    } else {
      // ---------------------------------------------------------- softmax over keys
      const int quarter = warp & 3;
      const int grp = (warp - 2) >> 2;       // heads 32*grp .. 32*grp+31
      const int key = quarter * 32 + lane;   // TMEM lane == key row of the block
      const int tid = threadIdx.x - 64;      // 0..255
      const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
      const float cs = p.scale_log2;
      bool ok = true;
      volatile int* rescale_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 12);
      for (int b = 0; b < nb && ok; ++b) {
        ok = warp_wait(bar(LY::BAR_S + (b & 1)), (b >> 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (tid == 0) *rescale_flag = 0;  // read by all only after the next two barriers
        float x[32];
        tmem_ld32(lane_addr + 64 * (b & 1) + 32 * grp, x);
        const int kb = walk.unit_at(b_lo + b);
        const int tpos = kb * kTile + key;
        const bool valid = tpos <= i_q && (tpos < win.sink_end || tpos >= lo_q);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = valid ? x[i] : -INFINITY;
        redmax[quarter * 64 + grp * 32 + lane] = warp_reduce_scatter32<true>(x);
        named_barrier_sync(1, 256);
        if (b > 0) {
          // PV(b-1) done: P^T buffer free and O^T stable (phases waited in order)
          ok = warp_wait(bar(LY::BAR_PV), (b - 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
        }
        if (tid < 64) {
          const float mb = fmaxf(fmaxf(redmax[tid], redmax[64 + tid]), fmaxf(redmax[128 + tid], redmax[192 + tid])) * cs;
          const float mo = m_run[tid];
          float a = 1.f, mn = mo;
          if (b == 0) {
            mn = mb;
          } else if (mb > mo + (float)kRescaleThreshold) {
            a = ex2_approx(mo - mb);
            mn = mb;
          }
          m_run[tid] = mn;
          alpha[tid] = a;
          if (a != 1.f) *rescale_flag = 1;
        }
        named_barrier_sync(1, 256);
        // P^T = 2^(cs*s - m) as the MN-major B operand: row = key, its 64
        // heads contiguous (128-byte swizzled rows); this thread writes the
        // 32 heads of its group as four 16-byte chunks
        float xr[32];
        {
          const float4* m4 = reinterpret_cast<const float4*>(m_run + 32 * grp);
          uint32_t pk[16];
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const float4 mm = m4[i4];
            const float mv[4] = {mm.x, mm.y, mm.z, mm.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) x[4 * i4 + j] = ex2_approx(fmaf(x[4 * i4 + j], cs, -mv[j]));
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            pk[i] = pack_bf16(x[2 * i], x[2 * i + 1]);
            xr[2 * i] = __uint_as_float(pk[i] << 16);
            xr[2 * i + 1] = __uint_as_float(pk[i] & 0xFFFF0000u);
          }
          uint8_t* prow = smem + LY::P_OFF + key * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(prow + (((4 * grp + j) ^ (key & 7)) << 4)) =
                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
        redsum[quarter * 64 + grp * 32 + lane] = warp_reduce_scatter32<false>(x);
        redrsum[quarter * 64 + grp * 32 + lane] = warp_reduce_scatter32<false>(xr);
        // O^T rescale where a head's running maximum moved (lane = latent column)
        if (b > 0 && *rescale_flag) {
          float av[32];
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const float4 a4 = reinterpret_cast<const float4*>(alpha + 32 * grp)[i4];
            av[4 * i4] = a4.x;
            av[4 * i4 + 1] = a4.y;
            av[4 * i4 + 2] = a4.z;
            av[4 * i4 + 3] = a4.w;
          }
#pragma unroll 1
          for (int u = 0; u < 4; ++u) {
            float o[32];
            tmem_ld32(lane_addr + 128 + 64 * u + 32 * grp, o);
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(o[i] * av[i]);
            tmem_st32(lane_addr + 128 + 64 * u + 32 * grp, w);
          }
          tmem_st_wait();
        }
        named_barrier_sync(1, 256);
        if (tid < 64) {
          l_run[tid] = l_run[tid] * alpha[tid] + ((redsum[tid] + redsum[64 + tid]) + (redsum[128 + tid] + redsum[192 + tid]));
          r_run[tid] = r_run[tid] * alpha[tid] + ((redrsum[tid] + redrsum[64 + tid]) + (redrsum[128 + tid] + redrsum[192 + tid]));
        }
        if (kb == jq) {
          // rows past the sequence end: zero them in the V units (the cache may
          // hold anything there) so that 0 * garbage cannot reach O
          ok = warp_wait(bar(LY::BAR_VT), 0, abort_flag);
          if (!ok) break;
          if (tpos > i_q) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            for (int u = 2 * grp; u < 2 * grp + 2; ++u) {
              const int slot_u = dec_v_pos(b, u, nb) % kDecStages;
#pragma unroll
              for (int t = 0; t < 2; ++t) {
                uint4* row = reinterpret_cast<uint4*>(smem + LY::RING_OFF + slot_u * kDecUnit + t * kChunkBytes + key * 128);
#pragma unroll
                for (int q8 = 0; q8 < 8; ++q8) row[(q8 + lane) & 7] = z;  // lanes spread over the banks
              }
            }
          }
        }
        // one arrival per warp, after every lane's shared-memory writes are
        // made visible to the tensor core
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(LY::BAR_P));
      }
      // ---------------------------------------------------------- partial epilogue
      if (ok) ok = warp_wait(bar(LY::BAR_PV), (nb - 1) & 1, abort_flag);
      if (ok) {
        tc_fence_after();
        named_barrier_sync(1, 256);  // l_run complete
        if (!CLUSTER) {
#pragma unroll 1
          for (int u = 0; u < 4; ++u) {
            const int dv = 128 * u + key;
            float o[32];
            tmem_ld32(lane_addr + 128 + 64 * u + 32 * grp, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) p.ws_o[(part * kDecHeads + 32 * grp + i) * 512 + dv] = o[i];
          }
        }
        if (!CLUSTER && tid < 64) p.ws_ml[part * kDecHeads + tid] = make_float4(m_run[tid], l_run[tid], r_run[tid], 0.f);
      }
    }
  } else if (!CLUSTER && threadIdx.x < 64) {
    p.ws_ml[part * kDecHeads + threadIdx.x] = make_float4(-INFINITY, 0.f, 0.f, 0.f);  // a split without blocks
  }

  if (CLUSTER) {
    // ---------------------------------------------------------- on-chip merge
    // Split r owns output columns [r*W, (r+1)*W), W = 512 / nsplit.
    // 1. every CTA reads all splits' (m, l) over DSMEM and computes the same
    //    merge weights; 2. each thread scales the O^T values it holds in TMEM
    //    that belong to other splits' columns and stores them to a staging
    //    area in this CTA's shared memory, laid out as the owner's receive
    //    slot; 3. one bulk copy per owner moves the slot into the owner's
    //    shared memory; 4. each CTA adds its own scaled part (from TMEM) and
    //    the received parts and writes its columns.
    const int r = (int)cluster_rank();
    const int ns = p.nsplit;
    const int W = 512 / ns;
    const uint32_t part_bytes = 64u * (uint32_t)W * 4u;
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && ns > 1) mbar_arrive_expect_tx(bar(LY::BAR_MRG), (uint32_t)(ns - 1) * part_bytes);
    cluster_sync_all();  // (m, l) of every split visible; every receive barrier armed
    // staging [ns-1][64][W] and receive [ns-1][64][W] buffers over the idle Q
    // tiles and ring; slot of split s in either: s < r ? s : s - 1
    float* stg = reinterpret_cast<float*>(smem + LY::Q_OFF);
    float* recv = stg + (size_t)(ns - 1) * 64 * W;
    float* wgt = reinterpret_cast<float*>(smem + LY::P_OFF);  // [8][64]; P^T is idle now
    float* mls = wgt + 8 * 64;                                 // [3][8][64] all splits' m, l, r
    for (int idx = threadIdx.x; idx < ns * 64; idx += blockDim.x) {
      const int s2 = idx >> 6, h = idx & 63;
      mls[idx] = *static_cast<const float*>(__cluster_map_shared_rank(m_run + h, s2));
      mls[8 * 64 + idx] = *static_cast<const float*>(__cluster_map_shared_rank(l_run + h, s2));
      mls[16 * 64 + idx] = *static_cast<const float*>(__cluster_map_shared_rank(r_run + h, s2));
    }
    __syncthreads();
    if (threadIdx.x < 64) {
      const int h = threadIdx.x;
      float M = -INFINITY;
      for (int s2 = 0; s2 < ns; ++s2)
        if (mls[8 * 64 + s2 * 64 + h] > 0.f) M = fmaxf(M, mls[s2 * 64 + h]);
      // O is normalised by the merged sum of the bf16 P that multiplied V,
      // the LSE by the merged exact sum
      float Ls = 0.f, Rs = 0.f;
      for (int s2 = 0; s2 < ns; ++s2) {
        const float l = mls[8 * 64 + s2 * 64 + h];
        const float w = l > 0.f ? ex2_approx(mls[s2 * 64 + h] - M) : 0.f;
        wgt[s2 * 64 + h] = w;
        Ls += l * w;
        Rs += mls[16 * 64 + s2 * 64 + h] * w;
      }
      const float inv = 1.f / Rs;
      for (int s2 = 0; s2 < ns; ++s2) wgt[s2 * 64 + h] *= inv;
      if (r == 0) p.lse[(int64_t)seq * kDecHeads + h] = (M + log2f(Ls)) * 0.69314718055994530942f;
    }
    __syncthreads();
    const int quarter = warp & 3, grp = (warp - 2) >> 2, key = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    if (nb > 0 && warp >= 2) {
#pragma unroll 1
      for (int u = 0; u < 4; ++u) {
        const int d = 128 * u + key;  // latent column of this lane
        const int owner = d / W;
        if (owner == r) continue;
        float* dst = stg + (size_t)(owner < r ? owner : owner - 1) * 64 * W + (d - owner * W);
        float o[32];
        tmem_ld32(lane_addr + 128 + 64 * u + 32 * grp, o);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int h = 32 * grp + i;
          dst[(size_t)h * W] = o[i] * wgt[r * 64 + h];
        }
      }
    }
    fence_proxy_async_smem();  // staging written by threads, read by the bulk copies
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int s2 = 0; s2 < ns; ++s2) {
        if (s2 == r) continue;
        const uint32_t src = smem_u32(stg + (size_t)(s2 < r ? s2 : s2 - 1) * 64 * W);
        const uint32_t dst = peer_addr(smem_u32(recv + (size_t)(r < s2 ? r : r - 1) * 64 * W), (uint32_t)s2);
        bulk_copy_to_peer(dst, src, part_bytes, peer_addr(bar(LY::BAR_MRG), (uint32_t)s2));
      }
    }
    const bool arrived = ns == 1 || mbar_wait(bar(LY::BAR_MRG), 0, nullptr);
    if (arrived && warp >= 2) {
#pragma unroll 1
      for (int u = 0; u < 4; ++u) {
        const int d = 128 * u + key;
        if (d / W != r) continue;
        float acc[32];
        if (nb > 0) {
          tmem_ld32(lane_addr + 128 + 64 * u + 32 * grp, acc);
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] *= wgt[r * 64 + 32 * grp + i];
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = 0.f;
        }
        for (int s2 = 0; s2 < ns; ++s2) {
          if (s2 == r) continue;
          const float* src = recv + (size_t)(s2 < r ? s2 : s2 - 1) * 64 * W + (d - r * W);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int h = 32 * grp + i;
            if (wgt[s2 * 64 + h] != 0.f) acc[i] += src[(size_t)h * W];  // a split without blocks sent no data
          }
        }
        __nv_bfloat16* dst = p.out + (int64_t)seq * kDecHeads * 512 + d;
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[(int64_t)(32 * grp + i) * 512] = __float2bfloat16_rn(acc[i]);
      }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // every bulk copy has finished reading its source before any CTA exits
  } else {
    // ---------------------------------------------------------- last CTA merges
    __threadfence();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) *last_flag = (atomicAdd(&p.ws_ticket[seq], 1) == p.nsplit - 1);
    __syncthreads();
    if (*last_flag) {
      __threadfence();
      float* wgt = reinterpret_cast<float*>(smem + LY::RING_OFF);  // [nsplit][64]; the ring is idle now
      if (threadIdx.x < 64) {
        const int h = threadIdx.x;
        float M = -INFINITY;
        for (int s2 = 0; s2 < p.nsplit; ++s2) {
          const float4 ml = p.ws_ml[((int64_t)seq * p.nsplit + s2) * kDecHeads + h];
          if (ml.y > 0.f) M = fmaxf(M, ml.x);
        }
        float Ls = 0.f, Rs = 0.f;
        for (int s2 = 0; s2 < p.nsplit; ++s2) {
          const float4 ml = p.ws_ml[((int64_t)seq * p.nsplit + s2) * kDecHeads + h];
          const float w = ml.y > 0.f ? ex2_approx(ml.x - M) : 0.f;
          wgt[s2 * 64 + h] = w;
          Ls += ml.y * w;
          Rs += ml.z * w;
        }
        const float inv = 1.f / Rs;
        for (int s2 = 0; s2 < p.nsplit; ++s2) wgt[s2 * 64 + h] *= inv;
        p.lse[(int64_t)seq * kDecHeads + h] = (M + log2f(Ls)) * 0.69314718055994530942f;
      }
      __syncthreads();
      for (int idx = threadIdx.x; idx < kDecHeads * 128; idx += blockDim.x) {
        const int h = idx >> 7;
        const int d4 = (idx & 127) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int s2 = 0; s2 < p.nsplit; ++s2) {
          const float w = wgt[s2 * 64 + h];
          if (w != 0.f) {
            const float4 o =
                *reinterpret_cast<const float4*>(p.ws_o + (((int64_t)seq * p.nsplit + s2) * kDecHeads + h) * 512 + d4);
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
  }
  if (warp == 1 && nb > 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace loza
