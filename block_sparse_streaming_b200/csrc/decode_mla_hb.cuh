// decode_mla_hb.cuh - absorbed-MLA SSA decode that reads every selected latent
// row into shared memory once: half-block streaming with the heads on M.
//
// The operation is that of decode_mla.cuh (one query token per sequence
// against the sink and local blocks of its window, LongCat ZigZag Attention
// page 1 sections 01-02; 64 heads share one 576-wide latent row, V = its first
// 512 columns). The unit of streaming is a half block of 64 rows: its 576
// columns (nine [64 x 64] tiles, 72 KB) stay resident from the S MMA through
// the P.V MMA, two of them double-buffered next to the 64 heads' Q (72 KB), so
// every selected row is read once.
//     S    [64 heads x 64 keys] = Q [64 x 576] . K_hb^T        (M = 64, K-major A and B)
//     O^T [512 x 64 heads]    += V_hb^T [512 x 64] . P^T       (MN-major A: the same tiles)
// With the heads on M, each head's logits sit in one TMEM lane (an M = 64
// accumulator occupies lanes 0-15 of each 32-lane quarter: head h at lane
// h % 16 + 32 (h / 16)), so the softmax of a head needs no exchange between
// warps: the two softmax warps of a quarter each take the whole row for the
// maximum and half of the keys for P, and a head's running maximum and sums
// live in the registers of the four threads that share its lane. P (bf16,
// [64 heads x 64 keys], K-major) replaces the half block's rope tile (columns
// 512..575), which no MMA reads after S.
//
// Roles: a TMA producer warp, an S issuer (one MMA group per tile as the tile
// lands), a P.V issuer (separate, so that P.V of one half block never waits
// for the load of the next; each 128-column chunk of P.V frees its two tiles
// for the load after next) and 8 softmax warps. O^T is rescaled only when a
// head's maximum grows by more than 2^8; the softmax warps agree on that once
// per half block at one named barrier.
//
// The selected half blocks of a sequence (2 per selected block; the query's
// own block contributes only the halves that reach its position) are split
// among nsplit <= 4 CTAs of a thread-block cluster. They merge on chip by the
// log-sum-exp rule: split r owns output columns [r W, (r+1) W), W = 512 /
// nsplit. When its own MMAs are done, each split tells the others that its
// shared memory is free; each then pushes its (m, l, r) and its unscaled
// partial O^T for the columns the others own straight into their shared
// memory (16-byte DSMEM stores, no multicast) and arrives on their mbarrier;
// each owner weights, sums and writes its columns.
#pragma once

#include <cuda.h>

#include "decode_mla.cuh"
#include "sm100.cuh"

namespace loza {

constexpr int kHbRows = 64;                 // keys per half block (N of S)
constexpr int kHbTile = kHbRows * 64 * 2;   // [64 rows x 64 columns] bf16, 8 KB
constexpr int kHbSlot = 9 * kHbTile;        // one half block: 576 columns
constexpr int kHbThreads = 352;             // producer, S issuer, P.V issuer, 8 softmax warps
constexpr int kHbMaxSplit = 4;
constexpr int kHbRecvPitch = 64 * 4 + 16;   // one received latent column: 64 heads fp32, padded

struct DecodeHbLayout {
  static constexpr int Q_OFF = 0;                                   // 9 Q tiles [64 heads x 64], 72 KB
  static constexpr int SLOT_OFF = 9 * kDecQTile;                    // 2 half-block slots, 144 KB
  static constexpr int STAT_OFF = SLOT_OFF + 2 * kHbSlot;           // (m, l, r) [kHbMaxSplit][3][64]
  static constexpr int WGT_OFF = STAT_OFF + kHbMaxSplit * 3 * 64 * 4;  // merge weights [kHbMaxSplit][64]
  static constexpr int ALPHA_OFF = WGT_OFF + kHbMaxSplit * 64 * 4;  // O^T rescale factors [2][64]
  static constexpr int LPART_OFF = ALPHA_OFF + 2 * 64 * 4;          // second key group's (l, r) [2][64]
  static constexpr int FLAG_OFF = LPART_OFF + 2 * 64 * 4;           // rescale flags [2]
  static constexpr int BAR_OFF = FLAG_OFF + 16;
  // barriers: q[9] (Q tile t), full[2][9] (slot, tile), empty[2][4] (slot, 128-column
  // chunk of P.V: tiles 2c, 2c+1, and the P tile with the last chunk), s_full[2],
  // s_free[2] (the softmax warps have read an S buffer), p_ready, pv_done[2]
  // (P.V of even / odd half blocks), ready (the other splits' shared memory is
  // free for the merge), data (the other splits' parts have landed)
  static constexpr int BAR_Q = 0, BAR_FULL = 9, BAR_EMPTY = 27, BAR_S = 35, BAR_SFREE = 37, BAR_P = 39,
                       BAR_PV = 40, BAR_READY = 42, BAR_DATA = 43, NBAR = 44;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;               // tmem base, abort
  static constexpr int SMEM_BYTES = MISC_OFF + 16;
  // merge receive buffer over Q and the slots: [nsplit - 1][W][kHbRecvPitch]
  static constexpr int RECV_OFF = 0;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(BAR_OFF % 8 == 0, "mbarrier alignment");
  static_assert((kHbMaxSplit - 1) * (512 / kHbMaxSplit) * kHbRecvPitch <= STAT_OFF, "merge receive buffer");
  static_assert(1 * 256 * kHbRecvPitch <= STAT_OFF, "merge receive buffer");
};

__global__ void __launch_bounds__(kHbThreads, 1) ssa_decode_mla_hb_kernel(const __grid_constant__ DecodeParams p) {
  using LY = DecodeHbLayout;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // the same in every CTA of the cluster: all leave before any barrier
    if (threadIdx.x == 0) atomicOr(&g_device_status, kErrLayout);
    return;
  }
  const int split = blockIdx.x;  // == rank in the cluster
  const int seq = blockIdx.y;
  const int ns = p.nsplit;
  const int L = p.seqlens[seq];
  const int i_q = L - 1;                                 // decode query position
  const int jq = i_q >= 0 ? i_q / kTile : 0;             // its block
  const int hq = i_q >= 0 ? (i_q % kTile) / kHbRows : 0; // the half of its block that holds it
  const BlockWalk walk(jq, p.n_sink, p.n_local);
  // half blocks in walk order (the own block is last; its second half only if hq == 1)
  const int nh_total = i_q >= 0 ? 2 * walk.count - (hq == 0 ? 1 : 0) : 0;
  const int h_lo = split * p.bps;
  const int nh = max(0, min(nh_total, h_lo + p.bps) - h_lo);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + LY::BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 4);
  float* stats = reinterpret_cast<float*>(smem + LY::STAT_OFF);   // [split][m, l, r][64]
  float* wgt = reinterpret_cast<float*>(smem + LY::WGT_OFF);      // [split][64]
  float* alpha = reinterpret_cast<float*>(smem + LY::ALPHA_OFF);  // [b & 1][64]
  float* lpart = reinterpret_cast<float*>(smem + LY::LPART_OFF);  // [l, r][64]
  volatile int* rflag = reinterpret_cast<volatile int*>(smem + LY::FLAG_OFF);

  if (threadIdx.x == 0) {
    for (int t = 0; t < 9; ++t) {
      mbar_init(bar(LY::BAR_Q + t), 1);
      mbar_init(bar(LY::BAR_FULL + t), 1);
      mbar_init(bar(LY::BAR_FULL + 9 + t), 1);
    }
    for (int c = 0; c < 8; ++c) mbar_init(bar(LY::BAR_EMPTY + c), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(LY::BAR_S + i), 1);
      mbar_init(bar(LY::BAR_SFREE + i), 8);  // one arrival per softmax warp
      mbar_init(bar(LY::BAR_PV + i), 1);
    }
    mbar_init(bar(LY::BAR_P), 8);  // one arrival per softmax warp
    mbar_init(bar(LY::BAR_READY), ns > 1 ? ns - 1 : 1);          // one arrival per other split
    mbar_init(bar(LY::BAR_DATA), ns > 1 ? 8 * (ns - 1) : 1);     // one per softmax warp of each other split
    *abort_flag = 0;
    rflag[0] = -1;
    rflag[1] = -1;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the other splits may signal this CTA's barriers only after they were
  // initialised: the matching wait comes before the first remote access
  if (ns > 1) cluster_arrive();

  if (nh > 0 && warp == 0) {
    // ---------------------------------------------------------- producer
    // Q tile t just before the first half block's tile t, so that S starts on
    // the first tiles while the rest land
    if (elect_one()) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_kv64);
    }
    __syncwarp();
    bool ok = true;
    for (int it = 0; it < nh && ok; ++it) {
      const int slot = it & 1;
      const int h = h_lo + it;
      const int2 rz = dec_block_rows(p, seq, walk.block(h >> 1));
      const uint32_t dst = sbase + LY::SLOT_OFF + slot * kHbSlot;
      for (int t = 0; t < 9 && ok; ++t) {
        // tiles 2c, 2c+1 are free once chunk c of the P.V two half blocks back
        // completed; the P tile (8) with the last chunk
        if (it >= 2 && (t & 1) == 0 && t < 8) {
          ok = warp_wait(bar(LY::BAR_EMPTY + 4 * slot + t / 2), ((it >> 1) & 1) ^ 1, abort_flag);
          if (!ok) break;
        }
        if (elect_one()) {
          if (it == 0) {
            mbar_arrive_expect_tx(bar(LY::BAR_Q + t), kDecQTile);
            tma_load_3d(sbase + LY::Q_OFF + t * kDecQTile, &p.tm_q, bar(LY::BAR_Q + t), t * 64, 0, seq);
          }
          mbar_arrive_expect_tx(bar(LY::BAR_FULL + 9 * slot + t), kHbTile);
          tma_load_3d(dst + t * kHbTile, &p.tm_kv64, bar(LY::BAR_FULL + 9 * slot + t), 64 * t,
                      rz.x + kHbRows * (h & 1), rz.y);
        }
        __syncwarp();
      }
    }
  } else if (nh > 0 && warp == 1) {
    // ---------------------------------------------------------- S issuer
    // S of half block `it`, one group of four MMAs per tile as it lands, once
    // the softmax warps have read the S buffer it reuses (that of `it - 2`)
    constexpr uint32_t idesc_s = idesc_bf16(kDecHeads, kHbRows, false, false);
    const uint64_t dq0 = sdesc_sw128(sbase + LY::Q_OFF, 16, 1024);     // Q tiles, K-major
    const uint64_t dk0 = sdesc_sw128(sbase + LY::SLOT_OFF, 16, 1024);  // K tiles, K-major
    bool ok = true;
    for (int it = 0; it < nh && ok; ++it) {
      const int slot = it & 1;
      if (it >= 2) {
        ok = warp_wait(bar(LY::BAR_SFREE + slot), ((it >> 1) & 1) ^ 1, abort_flag);
        if (!ok) break;
      }
      const uint32_t tmem_s = tmem + 64 * slot;
      for (int t = 0; t < 9 && ok; ++t) {
        if (it == 0) ok = warp_wait(bar(LY::BAR_Q + t), 0, abort_flag);
        if (ok) ok = warp_wait(bar(LY::BAR_FULL + 9 * slot + t), (it >> 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          const uint64_t da = desc_add(dq0, t * kDecQTile);
          const uint64_t db = desc_add(dk0, slot * kHbSlot + t * kHbTile);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem_s, desc_add(da, 32 * kk), desc_add(db, 32 * kk), idesc_s, (t | kk) != 0);
          if (t == 8) mma_commit(bar(LY::BAR_S + slot));
        }
        __syncwarp();
      }
    }
  } else if (nh > 0 && warp == 2) {
    // ---------------------------------------------------------- P.V issuer
    constexpr uint32_t idesc_o = idesc_bf16(128, kDecHeads, true, false);
    const uint32_t tmem_o = tmem + 128;  // O^T: 4 x 64 columns after the two S buffers
    const uint64_t dv0 = sdesc_sw128(sbase + LY::SLOT_OFF, kHbTile, 1024);         // V tiles, MN-major
    const uint64_t dp0 = sdesc_sw128(sbase + LY::SLOT_OFF + 8 * kHbTile, 16, 1024);  // P, K-major
    bool ok = true;
    for (int b = 0; b < nh && ok; ++b) {
      // O^T += V^T . P^T(b): chunk u = latent columns 128u .. 128u+127 (tiles 2u, 2u+1)
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
            mma_ss(tmem_o + 64 * u, desc_add(da, 2048 * kk), desc_add(dp, 32 * kk), idesc_o,
                   (b > 0 || kk > 0) ? 1u : 0u);
          // pv_done before the last chunk's empty: a reload of the P tile
          // implies P.V(b) is signalled
          if (u == 3) mma_commit(bar(LY::BAR_PV + (b & 1)));
          mma_commit(bar(LY::BAR_EMPTY + 4 * slot + u));
        }
      }
      __syncwarp();
    }
  }

  // ---------------------------------------------------------- softmax over the keys of each head
  // warp w >= 3: lane quarter w % 4 (heads 16q .. 16q+15 of S, latent
  // columns 32q .. 32q+31 of each O^T chunk); key group g = (w - 3) / 4
  // (keys 32g .. 32g+31 of each half block for P; heads 32g .. 32g+31 of O^T).
  // Thread t holds heads ha = 16q + t/4 and hb = ha + 8 (16x256b shape).
  const bool smx = warp >= 3;
  const int quarter = warp & 3;
  const int grp = (warp - 3) >> 2;
  const int t4 = lane & 3;
  const int ha = 16 * quarter + (lane >> 2), hb2 = ha + 8;
  const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
  const int tid = threadIdx.x - 96;  // 0..255 in the softmax warps
  float m_a = -INFINITY, m_b = -INFINITY;  // running maxima (scaled logits, log2 units)
  float l_a = 0.f, l_b = 0.f;              // sums of exact P
  float r_a = 0.f, r_b = 0.f;              // sums of bf16-rounded P (normalise O)
  bool ok = true;
  if (smx && nh > 0) {
    const float cs = p.scale_log2;
    for (int b = 0; b < nh; ++b) {
      const int slot = b & 1;
      if (ok) ok = warp_wait(bar(LY::BAR_S + slot), (b >> 1) & 1, abort_flag);
      float x[32];
      if (ok) {
        tc_fence_after();
        tmem_ld16x256b_x8(lane_addr + 64 * slot, x);
        // this S buffer may be overwritten (by S of b + 2) from now on
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(LY::BAR_SFREE + slot));
      const int h = h_lo + b;
      const int kb = walk.block(h >> 1);
      const int base_pos = kb * kTile + kHbRows * (h & 1);
      const int cut = i_q - base_pos;  // keys c <= cut are visible (>= 63: all)
      if (cut < 63) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int c = 8 * k + 2 * t4;
          if (c > cut) { x[4 * k] = -INFINITY; x[4 * k + 2] = -INFINITY; }
          if (c + 1 > cut) { x[4 * k + 1] = -INFINITY; x[4 * k + 3] = -INFINITY; }
        }
      }
      // row maxima over all 64 keys (both key groups compute the same)
      float ma = fmaxf(x[0], x[1]), mb = fmaxf(x[2], x[3]);
#pragma unroll
      for (int k = 1; k < 8; ++k) {
        ma = fmax3(ma, x[4 * k], x[4 * k + 1]);
        mb = fmax3(mb, x[4 * k + 2], x[4 * k + 3]);
      }
      ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, 1));
      mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
      ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, 2));
      mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
      ma *= cs;
      mb *= cs;
      // lazy rescale: keep the running maximum unless it grows by more than 2^8
      float aa = 1.f, ab = 1.f;
      if (b == 0) {
        m_a = ma;
        m_b = mb;
      } else {
        if (ma > m_a + (float)kRescaleThreshold) { aa = ex2_approx(m_a - ma); m_a = ma; }
        if (mb > m_b + (float)kRescaleThreshold) { ab = ex2_approx(m_b - mb); m_b = mb; }
      }
      const bool resc = __any_sync(0xffffffffu, aa != 1.f || ab != 1.f);
      if (grp == 0 && t4 == 0) {
        alpha[64 * slot + ha] = aa;
        alpha[64 * slot + hb2] = ab;
      }
      if (resc && lane == 0) rflag[slot] = b;
      l_a *= aa; r_a *= aa;
      l_b *= ab; r_b *= ab;
      // P = 2^(cs*s - m) for this group's 32 keys, into the P tile (the slot's
      // rope tile): row = head, keys contiguous (K-major, 128-byte swizzle)
      {
        uint8_t* ptile = smem + LY::SLOT_OFF + slot * kHbSlot + 8 * kHbTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if ((k >> 2) != grp) continue;  // static register indices, a warp-uniform branch
          const float pa0 = ex2_approx(fmaf(x[4 * k], cs, -m_a));
          const float pa1 = ex2_approx(fmaf(x[4 * k + 1], cs, -m_a));
          const float pb0 = ex2_approx(fmaf(x[4 * k + 2], cs, -m_b));
          const float pb1 = ex2_approx(fmaf(x[4 * k + 3], cs, -m_b));
          const uint32_t wa = pack_bf16(pa0, pa1), wb = pack_bf16(pb0, pb1);
          l_a += pa0 + pa1;
          l_b += pb0 + pb1;
          r_a += __uint_as_float(wa << 16) + __uint_as_float(wa & 0xFFFF0000u);
          r_b += __uint_as_float(wb << 16) + __uint_as_float(wb & 0xFFFF0000u);
          *reinterpret_cast<uint32_t*>(ptile + ha * 128 + ((k ^ (ha & 7)) << 4) + 4 * t4) = wa;
          *reinterpret_cast<uint32_t*>(ptile + hb2 * 128 + ((k ^ (hb2 & 7)) << 4) + 4 * t4) = wb;
        }
      }
      if (cut < 63) {
        // rows past the sequence end: zero them in the V tiles (the cache may
        // hold anything there) so that 0 * garbage cannot reach O^T
        const int r0 = cut + 1;
        const int n16 = (64 - r0) * 64;  // 16-byte units: rows x 8 tiles x 8 units
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int i = tid; i < n16; i += 256) {
          const int row = r0 + i / 64, tile = (i / 8) & 7, u = i & 7;
          *reinterpret_cast<uint4*>(smem + LY::SLOT_OFF + slot * kHbSlot + tile * kHbTile + row * 128 + u * 16) = z;
        }
      }
      // every lane's shared-memory writes visible to the tensor core, then
      // one barrier: whether any head of any quarter moved its maximum
      fence_proxy_async_smem();
      named_barrier_sync(1, 256);
      if (b > 0 && rflag[slot] == b) {
        // O^T columns of the heads whose maximum moved, times their factor,
        // once P.V(b-1) completed (P.V(b-3), of the same parity, completed
        // before the slot of b-1 was reloaded; P.V(b+1) needs P(b+1))
        if (ok) ok = warp_wait(bar(LY::BAR_PV + ((b - 1) & 1)), ((b - 1) >> 1) & 1, abort_flag);
        if (ok) {
          tc_fence_after();
          float av[32];
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const float4 a4 = reinterpret_cast<const float4*>(alpha + 64 * slot + 32 * grp)[i4];
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
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(LY::BAR_P));
    }
    // the last P.V's signal covers every earlier MMA of its issuing thread
    if (ok) ok = warp_wait(bar(LY::BAR_PV + ((nh - 1) & 1)), ((nh - 1) >> 1) & 1, abort_flag);
    if (ok) tc_fence_after();
  }

  // ---------------------------------------------------------- this split's (m, l, r)
  if (smx) {
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    r_a += __shfl_xor_sync(0xffffffffu, r_a, 1);
    r_b += __shfl_xor_sync(0xffffffffu, r_b, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    r_a += __shfl_xor_sync(0xffffffffu, r_a, 2);
    r_b += __shfl_xor_sync(0xffffffffu, r_b, 2);
    if (grp == 1 && t4 == 0) {
      lpart[ha] = l_a;
      lpart[hb2] = l_b;
      lpart[64 + ha] = r_a;
      lpart[64 + hb2] = r_b;
    }
    named_barrier_sync(1, 256);
    if (grp == 0 && t4 == 0) {
      float* st = stats + split * 192;
      st[ha] = m_a;
      st[hb2] = m_b;
      st[64 + ha] = nh > 0 ? l_a + lpart[ha] : 0.f;
      st[64 + hb2] = nh > 0 ? l_b + lpart[hb2] : 0.f;
      st[128 + ha] = nh > 0 ? r_a + lpart[64 + ha] : 0.f;
      st[128 + hb2] = nh > 0 ? r_b + lpart[64 + hb2] : 0.f;
    }
    named_barrier_sync(1, 256);
  }

  // ---------------------------------------------------------- on-chip merge of the splits
  const int W = 512 / ns;
  float* recv = reinterpret_cast<float*>(smem + LY::RECV_OFF);
  if (ns > 1) {
    cluster_wait();  // every split's barriers are initialised
    if (smx) {
      // this CTA's MMAs are done (or it had none): its shared memory may
      // receive; then wait until every other split's may
      if (tid == 0) {
        for (int s2 = 0; s2 < ns; ++s2)
          if (s2 != split) mbar_arrive_cluster_release(peer_addr(bar(LY::BAR_READY), (uint32_t)s2));
      }
      const bool rdy = warp_wait_cluster(bar(LY::BAR_READY), 0, abort_flag);
      if (rdy) {
        if (tid < 64) {
          const float* st = stats + split * 192;
          for (int s2 = 0; s2 < ns; ++s2) {
            if (s2 == split) continue;
            const uint32_t dst = peer_addr(smem_u32(stats + split * 192 + tid), (uint32_t)s2);
            st_cluster_u32(dst, __float_as_uint(st[tid]));
            st_cluster_u32(dst + 256, __float_as_uint(st[64 + tid]));
            st_cluster_u32(dst + 512, __float_as_uint(st[128 + tid]));
          }
        }
        if (nh > 0 && ok) {
          // the unscaled partial O^T of the columns other splits own: lane =
          // latent column, 32 heads per thread as eight 16-byte stores
#pragma unroll 1
          for (int u = 0; u < 4; ++u) {
            const int d = 128 * u + 32 * quarter + lane;
            const int owner = d / W;
            if (owner == split) continue;
            float o[32];
            tmem_ld32(lane_addr + 128 + 64 * u + 32 * grp, o);
            const int slot_in = split < owner ? split : split - 1;
            const uint32_t dst = peer_addr(
                smem_u32(reinterpret_cast<uint8_t*>(recv) + (size_t)(slot_in * W + (d - owner * W)) * kHbRecvPitch +
                         grp * 128),
                (uint32_t)owner);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              st_cluster_v4(dst + 16 * j, __float_as_uint(o[4 * j]), __float_as_uint(o[4 * j + 1]),
                            __float_as_uint(o[4 * j + 2]), __float_as_uint(o[4 * j + 3]));
          }
        }
      }
      fence_acq_rel_cluster();
      __syncwarp();
      if (lane == 0) {
        for (int s2 = 0; s2 < ns; ++s2)
          if (s2 != split) mbar_arrive_cluster_release(peer_addr(bar(LY::BAR_DATA), (uint32_t)s2));
      }
      ok = warp_wait_cluster(bar(LY::BAR_DATA), 0, abort_flag) && ok && rdy;
    }
  }
  if (smx) {
    if (tid < 64) {
      const int h = tid;
      float M = -INFINITY;
      for (int s2 = 0; s2 < ns; ++s2)
        if (stats[s2 * 192 + 64 + h] > 0.f) M = fmaxf(M, stats[s2 * 192 + h]);
      // O is normalised by the merged sum of the bf16 P that multiplied V,
      // the LSE by the merged exact sum
      float Ls = 0.f, Rs = 0.f;
      for (int s2 = 0; s2 < ns; ++s2) {
        const float l = stats[s2 * 192 + 64 + h];
        const float w = l > 0.f ? ex2_approx(stats[s2 * 192 + h] - M) : 0.f;
        wgt[s2 * 64 + h] = w;
        Ls += l * w;
        Rs += stats[s2 * 192 + 128 + h] * w;
      }
      const float inv = Rs > 0.f ? 1.f / Rs : 0.f;
      for (int s2 = 0; s2 < ns; ++s2) wgt[s2 * 64 + h] *= inv;
      if (split == 0) p.lse[(int64_t)seq * kDecHeads + h] = Ls > 0.f ? (M + log2f(Ls)) * 0.69314718055994530942f : -INFINITY;
    }
    named_barrier_sync(1, 256);
#pragma unroll 1
    for (int u = 0; u < 4; ++u) {
      const int d = 128 * u + 32 * quarter + lane;  // latent column of this lane
      if (d / W != split) continue;
      float acc[32];
      if (nh > 0 && ok) {
        tmem_ld32(lane_addr + 128 + 64 * u + 32 * grp, acc);
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] *= wgt[split * 64 + 32 * grp + i];
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = 0.f;
      }
      for (int s2 = 0; s2 < ns; ++s2) {
        if (s2 == split) continue;
        const int slot_in = s2 < split ? s2 : s2 - 1;
        const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const uint8_t*>(recv) +
                                                            (size_t)(slot_in * W + (d - split * W)) * kHbRecvPitch +
                                                            grp * 128);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 v = src[j];
          const float* w = wgt + s2 * 64 + 32 * grp + 4 * j;
          // a split without keys pushed no O (its weight is 0)
          if (w[0] != 0.f) acc[4 * j] += v.x * w[0];
          if (w[1] != 0.f) acc[4 * j + 1] += v.y * w[1];
          if (w[2] != 0.f) acc[4 * j + 2] += v.z * w[2];
          if (w[3] != 0.f) acc[4 * j + 3] += v.w * w[3];
        }
      }
      __nv_bfloat16* dst = p.out + (int64_t)seq * kDecHeads * 512 + d;
#pragma unroll
      for (int i = 0; i < 32; ++i) dst[(int64_t)(32 * grp + i) * 512] = __float2bfloat16_rn(acc[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace loza
