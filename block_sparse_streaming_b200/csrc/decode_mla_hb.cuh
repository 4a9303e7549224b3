// decode_mla_hb.cuh - absorbed-MLA SSA decode that reads every selected latent
// row into shared memory once: half-block streaming.
//
// The operation is that of decode_mla.cuh (one query token per sequence
// against the sink and local blocks of its window, LongCat ZigZag Attention
// page 1 sections 01-02; 64 heads share one 576-wide latent row, V = its first
// 512 columns). The difference is the unit of streaming. The block kernel
// streams 128-row blocks through a ring too small to hold one, so the 512 V
// columns of every row are fetched a second time after its S. Here the unit is
// a half block of 64 rows: its 576 columns (nine [64 x 64] tiles, 72 KB) stay
// resident from the S MMA through the P.V MMA, two of them double-buffered
// next to the 64 heads' Q (72 KB), so every selected row is read once.
//     S^T [64 keys x 64 heads]  = K_hb [64 x 576] . Q^T      (M = 64, K-major A and B)
//     O^T [512 x 64 heads]     += V_hb^T [512 x 64] . P^T    (MN-major A: the same tiles)
// P^T (bf16, [64 keys x 64 heads]) is written into the half block's rope tile
// (columns 512..575), which no MMA reads after S. An M = 64 accumulator
// occupies TMEM lanes 0-15 of each 32-lane quarter (row r at lane
// r % 16 + 32 * (r / 16)), so each softmax warp holds 16 keys.
//
// Roles: a TMA producer warp, an S^T issuer, a P.V issuer (separate, so that
// P.V of one half block never waits for the load of the next; the slot it
// frees is what the load after that needs) and 8 softmax warps, which wait
// for the previous P.V only when a running maximum moved and O^T must be
// rescaled.
//
// The selected half blocks of a sequence (2 per selected block; the query's
// own block contributes only the halves that reach its position) are split
// among nsplit <= 4 CTAs of a thread-block cluster. They merge on chip by the
// log-sum-exp rule: after a cluster barrier each pushes its (m, l) and its
// unscaled partial O^T for the columns the others own straight into their
// shared memory (plain DSMEM stores); after a second barrier each weights,
// sums and writes its own columns.
#pragma once

#include <cuda.h>

#include "decode_mla.cuh"
#include "sm100.cuh"

namespace loza {

constexpr int kHbRows = 64;                 // keys per half block (M of S^T)
constexpr int kHbTile = kHbRows * 64 * 2;   // [64 rows x 64 columns] bf16, 8 KB
constexpr int kHbSlot = 9 * kHbTile;        // one half block: 576 columns
constexpr int kHbThreads = 352;             // producer, S issuer, P.V issuer, 8 softmax warps
constexpr int kHbMaxSplit = 4;

struct DecodeHbLayout {
  static constexpr int Q_OFF = 0;                                  // 9 Q tiles [64 heads x 64], 72 KB
  static constexpr int SLOT_OFF = 9 * kDecQTile;                   // 2 half-block slots, 144 KB
  static constexpr int RED_OFF = SLOT_OFF + 2 * kHbSlot;           // redmax, redsum, redrsum [4][64]
  static constexpr int STAT_OFF = RED_OFF + 3 * 4 * 64 * 4;        // m_run, l_run, alpha, r_run [64]
  static constexpr int BAR_OFF = STAT_OFF + 4 * 64 * 4;
  // barriers: q_full, full[2], empty[2], s_full[2], p_ready, pv_done[2] (P.V of even / odd
  // half blocks), s_free[2] (the softmax warps have read an S^T buffer)
  static constexpr int BAR_Q = 0, BAR_FULL = 1, BAR_EMPTY = 3, BAR_S = 5, BAR_P = 7, BAR_PV = 8, BAR_SFREE = 10,
                       NBAR = 12;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;              // tmem base, abort, rescale flag
  static constexpr int SMEM_BYTES = MISC_OFF + 16;
  // merge, once every split of the cluster is done with its shared memory:
  // receive buffer [nsplit][64 heads][512 / nsplit] fp32 over Q and the
  // slots, the splits' (m, l, r) [nsplit][3][64] over RED, weights
  // [nsplit][64] over slot 1's rope tile
  static constexpr int WGT_OFF = SLOT_OFF + kHbSlot + 8 * kHbTile;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(64 * 512 * 4 <= WGT_OFF, "merge receive buffer");
  static_assert(kHbMaxSplit * 3 * 64 * 4 <= STAT_OFF - RED_OFF, "merge statistics");
  static_assert(WGT_OFF + kHbMaxSplit * 64 * 4 <= RED_OFF, "merge weights");
};

__global__ void __launch_bounds__(kHbThreads, 1) ssa_decode_mla_hb_kernel(const __grid_constant__ DecodeParams p) {
  using LY = DecodeHbLayout;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // the same in every CTA of the cluster: all leave before any barrier
    if (threadIdx.x == 0) atomicOr(&g_device_status, kErrLayout);
    return;
  }
  const int split = blockIdx.x;
  const int seq = blockIdx.y;
  const int L = p.seqlens[seq];
  const int i_q = L - 1;                  // decode query position
  const int jq = i_q / kTile;             // its block
  const int hq = (i_q % kTile) / kHbRows; // the half of its block that holds it
  const BlockWalk walk(jq, p.n_sink, p.n_local);
  // half blocks in walk order (the own block is last; its second half only if hq == 1)
  const int nh_total = 2 * walk.count - (hq == 0 ? 1 : 0);
  const int h_lo = split * p.bps;
  const int nh = max(0, min(nh_total, h_lo + p.bps) - h_lo);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + LY::BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 4);
  volatile int* rescale_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 8);
  float* redmax = reinterpret_cast<float*>(smem + LY::RED_OFF);  // [4 quarters][64]
  float* redsum = redmax + 4 * 64;   // sums of exact P (for the LSE)
  float* redrsum = redsum + 4 * 64;  // sums of bf16-rounded P (for normalising O)
  float* m_run = reinterpret_cast<float*>(smem + LY::STAT_OFF);
  float* l_run = m_run + 64;
  float* alpha = m_run + 128;
  float* r_run = m_run + 192;

  if (threadIdx.x == 0) {
    mbar_init(bar(LY::BAR_Q), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(LY::BAR_FULL + i), 1);
      mbar_init(bar(LY::BAR_EMPTY + i), 1);
      mbar_init(bar(LY::BAR_S + i), 1);
      mbar_init(bar(LY::BAR_SFREE + i), 8);  // one arrival per softmax warp
    }
    mbar_init(bar(LY::BAR_P), 8);  // one arrival per softmax warp
    mbar_init(bar(LY::BAR_PV + 0), 1);
    mbar_init(bar(LY::BAR_PV + 1), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 64) {
    m_run[threadIdx.x] = -INFINITY;
    l_run[threadIdx.x] = 0.f;
    r_run[threadIdx.x] = 0.f;
  }
  if (warp == 1 && nh > 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = nh > 0 ? *tmem_slot : 0;

  if (nh > 0) {
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (elect_one()) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_kv64);
        mbar_arrive_expect_tx(bar(LY::BAR_Q), 9 * kDecQTile);
        for (int c = 0; c < 9; ++c)
          tma_load_3d(sbase + LY::Q_OFF + c * kDecQTile, &p.tm_q, bar(LY::BAR_Q), c * 64, 0, seq);
      }
      __syncwarp();
      bool ok = true;
      for (int it = 0; it < nh && ok; ++it) {
        const int slot = it & 1;
        // the slot is free once the P.V of the half block two back completed
        ok = warp_wait(bar(LY::BAR_EMPTY + slot), ((it >> 1) & 1) ^ 1, abort_flag);
        if (!ok) break;
        if (elect_one()) {
          const int h = h_lo + it;
          const int2 rz = dec_block_rows(p, seq, walk.block(h >> 1));
          const uint32_t dst = sbase + LY::SLOT_OFF + slot * kHbSlot;
          mbar_arrive_expect_tx(bar(LY::BAR_FULL + slot), kHbSlot);
          for (int t = 0; t < 9; ++t)
            tma_load_3d(dst + t * kHbTile, &p.tm_kv64, bar(LY::BAR_FULL + slot), 64 * t, rz.x + kHbRows * (h & 1),
                        rz.y);
        }
        __syncwarp();
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- S^T issuer
      // S^T of half block `it` as soon as its slot is loaded and the softmax
      // warps have read the S^T buffer it reuses (that of `it - 2`)
      constexpr uint32_t idesc_s = idesc_bf16(kHbRows, kDecHeads, false, false);
      const uint64_t dk0 = sdesc_sw128(sbase + LY::SLOT_OFF, 16, 1024);  // K tiles, K-major
      const uint64_t dq0 = sdesc_sw128(sbase + LY::Q_OFF, 16, 1024);     // Q tiles, K-major
      bool ok = warp_wait(bar(LY::BAR_Q), 0, abort_flag);
      for (int it = 0; it < nh && ok; ++it) {
        const int slot = it & 1;
        if (it >= 2) {
          ok = warp_wait(bar(LY::BAR_SFREE + slot), ((it >> 1) & 1) ^ 1, abort_flag);
          if (!ok) break;
        }
        ok = warp_wait(bar(LY::BAR_FULL + slot), (it >> 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t tmem_s = tmem + 64 * slot;
          for (int t = 0; t < 9; ++t) {
            const uint64_t da = desc_add(dk0, slot * kHbSlot + t * kHbTile);
            const uint64_t db = desc_add(dq0, t * kDecQTile);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem_s, desc_add(da, 32 * kk), desc_add(db, 32 * kk), idesc_s, (t | kk) != 0);
          }
          mma_commit(bar(LY::BAR_S + slot));
        }
        __syncwarp();
      }
    } else if (warp == 2) {
      // ---------------------------------------------------------- P.V issuer
      // a separate warp, so that P.V of half block b never waits for the
      // load of b + 1 (the slot it frees is what the load of b + 2 needs)
      constexpr uint32_t idesc_o = idesc_bf16(128, kDecHeads, true, true);
      const uint32_t tmem_o = tmem + 128;  // O^T: 4 x 64 columns after the two S^T buffers
      const uint64_t dv0 = sdesc_sw128(sbase + LY::SLOT_OFF, kHbTile, 1024);             // V tiles, MN-major
      const uint64_t dp0 = sdesc_sw128(sbase + LY::SLOT_OFF + 8 * kHbTile, 8192, 1024);  // P^T, MN-major
      bool ok = true;
      for (int b = 0; b < nh && ok; ++b) {
        // O^T += V^T . P^T(b): column chunk u = latent columns 128u .. 128u+127 (tiles 2u, 2u+1)
        const int slot = b & 1;
        ok = warp_wait(bar(LY::BAR_P), b & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          const uint64_t dp = desc_add(dp0, slot * kHbSlot);
          for (int u = 0; u < 4; ++u) {
            const uint64_t da = desc_add(dv0, slot * kHbSlot + 2 * u * kHbTile);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem_o + 64 * u, desc_add(da, 2048 * kk), desc_add(dp, 2048 * kk), idesc_o,
                     (b > 0 || kk > 0) ? 1u : 0u);
          }
          // S^T(b) read the slot too; it completed before P(b) was written.
          // pv_done first: a reload of the slot implies P.V(b) is signalled
          mma_commit(bar(LY::BAR_PV + (b & 1)));
          mma_commit(bar(LY::BAR_EMPTY + slot));
        }
        __syncwarp();
      }
    } else {
      // ---------------------------------------------------------- softmax over keys
      const int quarter = warp & 3;
      const int grp = (warp - 3) >> 2;         // heads 32*grp .. 32*grp+31
      const bool row_lane = lane < 16;         // an M = 64 accumulator uses lanes 0-15 of each quarter
      const int key = quarter * 16 + (lane & 15);
      const int tid = threadIdx.x - 96;        // 0..255
      const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
      const float cs = p.scale_log2;
      bool ok = true;
      for (int b = 0; b < nh && ok; ++b) {
        const int slot = b & 1;
        ok = warp_wait(bar(LY::BAR_S + slot), (b >> 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (tid == 0) *rescale_flag = 0;  // read by all only after the next two barriers
        float x[32];
        tmem_ld32(lane_addr + 64 * slot + 32 * grp, x);
        // this S^T buffer may be overwritten (by S^T of b + 2) from now on
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(LY::BAR_SFREE + slot));
        const int h = h_lo + b;
        const int kb = walk.block(h >> 1);
        const int pos = kb * kTile + kHbRows * (h & 1) + key;
        const bool valid = row_lane && pos <= i_q;
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = valid ? x[i] : -INFINITY;
        redmax[quarter * 64 + grp * 32 + lane] = warp_reduce_scatter32<true>(x);
        named_barrier_sync(1, 256);
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
        // P^T = 2^(cs*s - m) into the rope tile of this half block's slot
        // (S^T has completed, so no MMA reads that tile any more): row = key,
        // its 64 heads contiguous in a 128-byte swizzled row; this thread
        // writes the 32 heads of its group as four 16-byte chunks
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
          if (row_lane) {
            uint8_t* prow = smem + LY::SLOT_OFF + slot * kHbSlot + 8 * kHbTile + key * 128;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              *reinterpret_cast<uint4*>(prow + (((4 * grp + j) ^ (key & 7)) << 4)) =
                  make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
        redsum[quarter * 64 + grp * 32 + lane] = warp_reduce_scatter32<false>(x);
        redrsum[quarter * 64 + grp * 32 + lane] = warp_reduce_scatter32<false>(xr);
        // O^T rescale where a head's running maximum moved (lane = latent column),
        // once P.V(b-1) has completed. Only then is O^T waited for: P(b) goes to
        // this half block's own slot, so it never waits for P.V(b-1). The wait
        // is unambiguous: P.V(b-3), of the same parity, completed before the
        // slot of b-1 was reloaded, and P.V(b+1) needs P(b+1).
        if (b > 0 && *rescale_flag) {
          ok = warp_wait(bar(LY::BAR_PV + ((b - 1) & 1)), ((b - 1) >> 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
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
        if (kb == jq && row_lane && !valid) {
          // rows past the sequence end: zero them in the V tiles (the cache may
          // hold anything there) so that 0 * garbage cannot reach O; group g
          // clears tiles 4g .. 4g+3 of the row
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int t = 4 * grp; t < 4 * grp + 4; ++t) {
            uint4* row = reinterpret_cast<uint4*>(smem + LY::SLOT_OFF + slot * kHbSlot + t * kHbTile + key * 128);
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8) row[(q8 + lane) & 7] = z;  // lanes spread over the banks
          }
        }
        // one arrival per warp, after every lane's shared-memory writes are
        // made visible to the tensor core
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(LY::BAR_P));
      }
      // the last P.V's signal covers every earlier MMA of its issuing thread
      if (ok) ok = warp_wait(bar(LY::BAR_PV + ((nh - 1) & 1)), ((nh - 1) >> 1) & 1, abort_flag);
      if (ok) tc_fence_after();
    }
  }

  // ---------------------------------------------------------- on-chip merge
  // Split r owns output columns [r*W, (r+1)*W), W = 512 / nsplit. After one
  // cluster barrier (every split is done with its shared memory) each split
  // pushes, with plain DSMEM stores, its (m, l, r) and its unscaled partial
  // O^T for the columns other splits own into the owners' receive buffers;
  // after a second barrier (every push has landed, and nothing crosses CTAs
  // after it) each split weights and sums its columns by the log-sum-exp
  // rule and writes them. A single split (nsplit 1) writes all columns.
  const int r = (int)cluster_rank();
  const int ns = p.nsplit;
  const int W = 512 / ns;
  float* recv = reinterpret_cast<float*>(smem + LY::Q_OFF);     // [ns][64][W]; slot r unused
  float* stats = reinterpret_cast<float*>(smem + LY::RED_OFF);  // [ns][3][64]; slot r unused
  float* wgt = reinterpret_cast<float*>(smem + LY::WGT_OFF);    // [ns][64]
  const int quarter = warp & 3, grp = (warp - 3) >> 2, col = quarter * 32 + lane;
  const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
  tc_fence_before();
  __syncthreads();
  if (ns > 1) {
    cluster_sync_all();
    if (threadIdx.x < 64) {
      const int h = threadIdx.x;
      for (int s2 = 0; s2 < ns; ++s2) {
        if (s2 == r) continue;
        const uint32_t dst = peer_addr(smem_u32(stats + r * 192 + h), (uint32_t)s2);
        st_cluster_u32(dst, __float_as_uint(m_run[h]));
        st_cluster_u32(dst + 256, __float_as_uint(l_run[h]));
        st_cluster_u32(dst + 512, __float_as_uint(r_run[h]));
      }
    }
    if (nh > 0 && warp >= 3) {
      tc_fence_after();
#pragma unroll 1
      for (int u = 0; u < 4; ++u) {
        const int d = 128 * u + col;  // latent column of this lane
        const int owner = d / W;
        if (owner == r) continue;
        float o[32];
        tmem_ld32(lane_addr + 128 + 64 * u + 32 * grp, o);
        const uint32_t dst =
            peer_addr(smem_u32(recv + ((size_t)r * 64 + 32 * grp) * W + (d - owner * W)), (uint32_t)owner);
#pragma unroll
        for (int i = 0; i < 32; ++i) st_cluster_u32(dst + 4u * (uint32_t)(i * W), __float_as_uint(o[i]));
      }
    }
    cluster_sync_all();
  }
  if (threadIdx.x < 64) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int s2 = 0; s2 < ns; ++s2) {
      const float l = s2 == r ? l_run[h] : stats[s2 * 192 + 64 + h];
      if (l > 0.f) M = fmaxf(M, s2 == r ? m_run[h] : stats[s2 * 192 + h]);
    }
    // O is normalised by the merged sum of the bf16 P that multiplied V,
    // the LSE by the merged exact sum
    float Ls = 0.f, Rs = 0.f;
    for (int s2 = 0; s2 < ns; ++s2) {
      const float m = s2 == r ? m_run[h] : stats[s2 * 192 + h];
      const float l = s2 == r ? l_run[h] : stats[s2 * 192 + 64 + h];
      const float rr = s2 == r ? r_run[h] : stats[s2 * 192 + 128 + h];
      const float w = l > 0.f ? ex2_approx(m - M) : 0.f;
      wgt[s2 * 64 + h] = w;
      Ls += l * w;
      Rs += rr * w;
    }
    const float inv = 1.f / Rs;
    for (int s2 = 0; s2 < ns; ++s2) wgt[s2 * 64 + h] *= inv;
    if (r == 0) p.lse[(int64_t)seq * kDecHeads + h] = (M + log2f(Ls)) * 0.69314718055994530942f;
  }
  __syncthreads();
  if (warp >= 3) {
    if (nh > 0) tc_fence_after();
#pragma unroll 1
    for (int u = 0; u < 4; ++u) {
      const int d = 128 * u + col;
      if (d / W != r) continue;
      float acc[32];
      if (nh > 0) {
        tmem_ld32(lane_addr + 128 + 64 * u + 32 * grp, acc);
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] *= wgt[r * 64 + 32 * grp + i];
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = 0.f;
      }
      for (int s2 = 0; s2 < ns; ++s2) {
        if (s2 == r) continue;
        const float* src = recv + (size_t)s2 * 64 * W + (d - r * W);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int h = 32 * grp + i;
          const float w = wgt[s2 * 64 + h];
          if (w != 0.f) acc[i] += src[(size_t)h * W] * w;  // a split without half blocks pushed no O
        }
      }
      __nv_bfloat16* dst = p.out + (int64_t)seq * kDecHeads * 512 + d;
#pragma unroll
      for (int i = 0; i < 32; ++i) dst[(int64_t)(32 * grp + i) * 512] = __float2bfloat16_rn(acc[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1 && nh > 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace loza
