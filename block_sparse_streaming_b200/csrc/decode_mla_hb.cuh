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
// Roles: a TMA producer warp (three 24 KB boxes per half block), an S issuer
// (one MMA group per box as it lands), a P.V issuer (separate, so that P.V of
// one half block never waits for the load of the next; its 128-column chunks
// free the tiles for the load after next box by box) and 8 softmax warps. O^T is rescaled only when a
// head's maximum grows by more than 2^8; the softmax warps agree on that once
// per half block at one named barrier.
//
// The selected half blocks of a sequence (2 per selected block; the query's
// own block contributes only the halves that reach its position) are split
// among nsplit <= 4 CTAs of a thread-block cluster. They merge on chip by the
// log-sum-exp rule: split r owns output columns [r W, (r+1) W), W = 512 /
// nsplit. When its own MMAs are done, each split tells the others that its
// shared memory is free, stages its (m, l, r) and its unscaled partial O^T
// for the columns each other split owns in its own shared memory, and moves
// each part with one bulk copy (no multicast) into the owner's receive area,
// where it completes as transaction bytes on the owner's mbarrier; each owner
// weights, sums and writes its columns. The L2 is asked for the half blocks
// after the first two of each split at the start, so HBM keeps streaming
// while the two slots turn over.
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
  static constexpr int STAT_OFF = SLOT_OFF + 2 * kHbSlot;           // (m, l0, l1, r0, r1) [5][64]
  static constexpr int WGT_OFF = STAT_OFF + 5 * 64 * 4;             // merge weights [kHbMaxSplit][64]
  static constexpr int ALPHA_OFF = WGT_OFF + kHbMaxSplit * 64 * 4;  // O^T rescale factors [2][64]
  static constexpr int FLAG_OFF = ALPHA_OFF + 2 * 64 * 4;           // rescale flags [2]
  static constexpr int BAR_OFF = FLAG_OFF + 16;
  // barriers: q[3] (Q tiles 3g .. 3g+2), full[2][3] (slot, tiles 3g .. 3g+2),
  // empty[2][3] (slot, tiles 3g .. 3g+2 free: after 128-column chunk g+1 of
  // P.V; the P tile, 8, with the last chunk), s_full[2], s_free[2] (the
  // softmax warps have read an S buffer), p_ready, pv_done[2] (P.V of even /
  // odd half blocks), ready (the other splits' shared memory is free for the
  // merge), data (the other splits' parts have landed), sent (the other
  // splits have received this split's parts: its shared memory may go)
  static constexpr int BAR_Q = 0, BAR_FULL = 3, BAR_EMPTY = 9, BAR_S = 15, BAR_SFREE = 17, BAR_P = 19,
                       BAR_PV = 20, BAR_READY = 22, BAR_DATA = 23, BAR_SENT = 24, NBAR = 25;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;               // tmem base, abort
  static constexpr int SMEM_BYTES = MISC_OFF + 16;
  // merge, over Q and the slots once the MMAs are done: the parts this split
  // sends (stage) and receives, [nsplit - 1] parts each of
  // [(m, l0, l1, r0, r1) x 64][W = 512 / nsplit latent columns x kHbRecvPitch]
  static constexpr int kPartHead = 5 * 64 * 4;
  static constexpr __host__ __device__ int part_bytes(int ns) { return kPartHead + (512 / ns) * kHbRecvPitch; }
  static constexpr int STAGE_OFF = 0;
  static constexpr int RECV_OFF = 110592;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(BAR_OFF % 8 == 0, "mbarrier alignment");
};
static_assert(DecodeHbLayout::part_bytes(2) % 16 == 0 && DecodeHbLayout::part_bytes(4) % 16 == 0, "bulk copy sizes");
static_assert(DecodeHbLayout::STAGE_OFF + 3 * DecodeHbLayout::part_bytes(4) <= DecodeHbLayout::RECV_OFF &&
                  DecodeHbLayout::STAGE_OFF + DecodeHbLayout::part_bytes(2) <= DecodeHbLayout::RECV_OFF,
              "merge stage");
static_assert(DecodeHbLayout::RECV_OFF + 3 * DecodeHbLayout::part_bytes(4) <= DecodeHbLayout::STAT_OFF &&
                  DecodeHbLayout::RECV_OFF + DecodeHbLayout::part_bytes(2) <= DecodeHbLayout::STAT_OFF,
              "merge receive");

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
  griddep_wait();  // in a chain of launches, the sequence lengths and cache rows may come from the kernel before
  const int L = p.seqlens[seq];
  const int i_q = L - 1;                                 // decode query position
  // the half blocks (64-row units) of the window of position i_q, sinks
  // first, the unit holding i_q last; each holds at least one visible key
  const SsaWindow win{p.block, p.n_sink * p.block, p.n_local};
  const RowWalk walk(win, max(i_q, 0), kHbRows);
  const int lo_q = win.lo(max(i_q, 0));
  const int nh_total = i_q >= 0 ? walk.count : 0;
  const int h_lo = split * p.bps;
  const int nh = max(0, min(nh_total, h_lo + p.bps) - h_lo);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + LY::BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 4);
  float* stats = reinterpret_cast<float*>(smem + LY::STAT_OFF);   // [m, l0, l1, r0, r1][64]
  float* wgt = reinterpret_cast<float*>(smem + LY::WGT_OFF);      // [split][64]
  float* alpha = reinterpret_cast<float*>(smem + LY::ALPHA_OFF);  // [b & 1][64]
  volatile int* rflag = reinterpret_cast<volatile int*>(smem + LY::FLAG_OFF);

  if (threadIdx.x == 0) {
    for (int g = 0; g < 3; ++g) mbar_init(bar(LY::BAR_Q + g), 1);
    for (int g = 0; g < 6; ++g) {
      mbar_init(bar(LY::BAR_FULL + g), 1);
      mbar_init(bar(LY::BAR_EMPTY + g), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(LY::BAR_S + i), 1);
      mbar_init(bar(LY::BAR_SFREE + i), 8);  // one arrival per softmax warp
      mbar_init(bar(LY::BAR_PV + i), 1);
    }
    mbar_init(bar(LY::BAR_P), 8);  // one arrival per softmax warp
    mbar_init(bar(LY::BAR_READY), ns > 1 ? ns - 1 : 1);          // one arrival per other split
    mbar_init(bar(LY::BAR_DATA), 1);
    mbar_init(bar(LY::BAR_SENT), ns > 1 ? ns - 1 : 1);
    // every other split's part arrives by a bulk copy as transaction bytes
    if (ns > 1) mbar_arrive_expect_tx(bar(LY::BAR_DATA), (uint32_t)((ns - 1) * LY::part_bytes(ns)));
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
  // initialised: the softmax warps, which make every remote access, wait for
  // that before their main loop; the other warps before they leave
  if (ns > 1) cluster_arrive();

  if (nh > 0 && warp == 0) {
    // ---------------------------------------------------------- producer
    // three requests per half block (tiles 3g .. 3g+2 each, 24 KB: a TMA
    // request has a fixed cost, so few large boxes keep more bytes in flight
    // than nine 8 KB tiles); Q's three groups just before the first half
    // block's, so that S starts on the first tiles while the rest land
    if (elect_one()) {
      tma_prefetch_desc(&p.tm_q3);
      tma_prefetch_desc(&p.tm_kv3);
    }
    __syncwarp();
    bool ok = true;
    for (int it = 0; it < nh && ok; ++it) {
      const int slot = it & 1;
      const int h = walk.unit_at(h_lo + it);  // rows 64h .. 64h+63 of the context
      const int2 rz = dec_block_rows(p, seq, h >> 1);
      const uint32_t dst = sbase + LY::SLOT_OFF + slot * kHbSlot;
      for (int g = 0; g < 3 && ok; ++g) {
        // tiles 3g .. 3g+2 are free once P.V of the half block two back has
        // completed the chunks that read them
        if (it >= 2) {
          ok = warp_wait(bar(LY::BAR_EMPTY + 3 * slot + g), ((it >> 1) & 1) ^ 1, abort_flag);
          if (!ok) break;
        }
        if (elect_one()) {
          if (it == 0) {
            mbar_arrive_expect_tx(bar(LY::BAR_Q + g), 3 * kDecQTile);
            tma_load_4d(sbase + LY::Q_OFF + 3 * g * kDecQTile, &p.tm_q3, bar(LY::BAR_Q + g), 0, 0, 3 * g, seq);
          }
          mbar_arrive_expect_tx(bar(LY::BAR_FULL + 3 * slot + g), 3 * kHbTile);
          tma_load_4d(dst + 3 * g * kHbTile, &p.tm_kv3, bar(LY::BAR_FULL + 3 * slot + g), 0,
                      rz.x + kHbRows * (h & 1), 3 * g, rz.y);
        }
        __syncwarp();
      }
      if (it == 1 && elect_one()) {
        // the half blocks after the first two into L2 now, so that HBM streams
        // while the slots turn over; their loads into the slots then hit L2
        for (int i2 = h_lo + 2; i2 < h_lo + nh; ++i2) {
          const int h2 = walk.unit_at(i2);
          const int2 r2 = dec_block_rows(p, seq, h2 >> 1);
          for (int g = 0; g < 3; ++g) tma_prefetch_l2_4d(&p.tm_kv3, 0, r2.x + kHbRows * (h2 & 1), 3 * g, r2.y);
        }
      }
      __syncwarp();
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
      for (int g = 0; g < 3 && ok; ++g) {
        if (it == 0) ok = warp_wait(bar(LY::BAR_Q + g), 0, abort_flag);
        if (ok) ok = warp_wait(bar(LY::BAR_FULL + 3 * slot + g), (it >> 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          for (int t = 3 * g; t < 3 * g + 3; ++t) {
            const uint64_t da = desc_add(dq0, t * kDecQTile);
            const uint64_t db = desc_add(dk0, slot * kHbSlot + t * kHbTile);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem_s, desc_add(da, 32 * kk), desc_add(db, 32 * kk), idesc_s, (t | kk) != 0);
          }
          if (g == 2) mma_commit(bar(LY::BAR_S + slot));
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
          // implies P.V(b) is signalled. Chunk u >= 1 frees tiles 3(u-1) ..
          // 3(u-1)+2 (chunks complete in order; the last also frees the P tile)
          if (u == 3) mma_commit(bar(LY::BAR_PV + (b & 1)));
          if (u >= 1) mma_commit(bar(LY::BAR_EMPTY + 3 * slot + (u - 1)));
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
  if (smx && ns > 1) cluster_wait();
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
      const int base_pos = kHbRows * walk.unit_at(h_lo + b);
      const int cut = i_q - base_pos;         // keys c <= cut exist (>= 63: all)
      const int e = win.sink_end - base_pos;  // c < e: sink keys
      const int f = lo_q - base_pos;          // c >= f: the local range
      if (cut < 63 || (e < 64 && f > 0)) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int c = 8 * k + 2 * t4;
          if (!(c <= cut && (c < e || c >= f))) { x[4 * k] = -INFINITY; x[4 * k + 2] = -INFINITY; }
          if (!(c + 1 <= cut && (c + 1 < e || c + 1 >= f))) { x[4 * k + 1] = -INFINITY; x[4 * k + 3] = -INFINITY; }
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
  // m, and the sums of each key group kept apart (the owner adds them):
  // [m, l of group 0, l of group 1, r of group 0, r of group 1][64 heads],
  // here and at the head of every part staged for another split
  if (smx) {
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    r_a += __shfl_xor_sync(0xffffffffu, r_a, 1);
    r_b += __shfl_xor_sync(0xffffffffu, r_b, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    r_a += __shfl_xor_sync(0xffffffffu, r_a, 2);
    r_b += __shfl_xor_sync(0xffffffffu, r_b, 2);
    if (t4 == 0) {
      for (int j = -1; j < ns - 1; ++j) {
        float* st = j < 0 ? stats : reinterpret_cast<float*>(smem + LY::STAGE_OFF + j * LY::part_bytes(ns));
        if (grp == 0) {
          st[ha] = m_a;
          st[hb2] = m_b;
        }
        st[64 * (1 + grp) + ha] = l_a;
        st[64 * (1 + grp) + hb2] = l_b;
        st[64 * (3 + grp) + ha] = r_a;
        st[64 * (3 + grp) + hb2] = r_b;
      }
    }
  }

  // ---------------------------------------------------------- on-chip merge of the splits
  // Each split stages, for every other split, its (m, l, r) and its unscaled
  // partial O^T of that split's columns in its own shared memory (free once
  // its MMAs are done), and moves each part with one bulk copy into the
  // owner's receive area once the owner has said that area is free. The
  // copies complete as transaction bytes on the owner's data barrier.
  const int W = 512 / ns;
  const int DB = LY::part_bytes(ns);
  if (ns > 1) {
    if (smx) {
      if (tid == 32) {
        // this CTA's MMAs are done (or it had none): its receive area is free
        // (a plain arrive: the MMAs that read the area have completed)
        for (int s2 = 0; s2 < ns; ++s2)
          if (s2 != split) mbar_arrive_cluster(peer_addr(bar(LY::BAR_READY), (uint32_t)s2));
      }
      {
        // lane = latent column, 32 heads per thread as eight 16-byte stores
        // (zeros from a split without keys, so the owner needs no test)
#pragma unroll 1
        for (int u = 0; u < 4; ++u) {
          const int d = 128 * u + 32 * quarter + lane;
          const int owner = d / W;
          if (owner == split) continue;
          float o[32];
          if (nh > 0 && ok) {
            tmem_ld32(lane_addr + 128 + 64 * u + 32 * grp, o);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
          }
          const int j = owner < split ? owner : owner - 1;
          uint4* dst = reinterpret_cast<uint4*>(smem + LY::STAGE_OFF + j * DB + LY::kPartHead +
                                                (d - owner * W) * kHbRecvPitch + grp * 128);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            dst[q4] = make_uint4(__float_as_uint(o[4 * q4]), __float_as_uint(o[4 * q4 + 1]),
                                 __float_as_uint(o[4 * q4 + 2]), __float_as_uint(o[4 * q4 + 3]));
        }
      }
      fence_proxy_async_smem();  // the staged parts are read by the bulk copies
      named_barrier_sync(1, 256);
      // every other split's receive area is free: one bulk copy per owner
      if (warp_wait_cluster(bar(LY::BAR_READY), 0, abort_flag) && tid == 0) {
        for (int o2 = 0; o2 < ns; ++o2) {
          if (o2 == split) continue;
          const int j = o2 < split ? o2 : o2 - 1;       // the part for o2 in this split's stage
          const int jr = split < o2 ? split : split - 1; // this split's part in o2's receive area
          bulk_copy_to_peer(peer_addr(sbase + LY::RECV_OFF + jr * DB, (uint32_t)o2), sbase + LY::STAGE_OFF + j * DB,
                            DB, peer_addr(bar(LY::BAR_DATA), (uint32_t)o2));
        }
      }
      ok = warp_wait(bar(LY::BAR_DATA), 0, abort_flag) && ok;
      // every part copied into this CTA has landed: tell each sender that it
      // may leave (its copies have read their source)
      if (tid == 0) {
        for (int s2 = 0; s2 < ns; ++s2)
          if (s2 != split) mbar_arrive_cluster(peer_addr(bar(LY::BAR_SENT), (uint32_t)s2));
      }
    }
  }
  if (smx) {
    // weights of the splits' partial O by the log-sum-exp rule
    if (ns == 1) named_barrier_sync(1, 256);  // the statistics above are complete
    // [m, l0, l1, r0, r1] of split s2: this split's own, or the head of its received part
    auto part = [&](int s2) -> const float* {
      if (s2 == split) return stats;
      return reinterpret_cast<const float*>(smem + LY::RECV_OFF + (s2 < split ? s2 : s2 - 1) * DB);
    };
    if (tid < 64) {
      const int h = tid;
      float M = -INFINITY;
      for (int s2 = 0; s2 < ns; ++s2) {
        const float* st = part(s2);
        if (st[64 + h] + st[128 + h] > 0.f) M = fmaxf(M, st[h]);
      }
      // O is normalised by the merged sum of the bf16 P that multiplied V,
      // the LSE by the merged exact sum
      float Ls = 0.f, Rs = 0.f;
      for (int s2 = 0; s2 < ns; ++s2) {
        const float* st = part(s2);
        const float l = st[64 + h] + st[128 + h];
        const float w = l > 0.f ? ex2_approx(st[h] - M) : 0.f;
        wgt[s2 * 64 + h] = w;
        Ls += l * w;
        Rs += (st[192 + h] + st[256 + h]) * w;
      }
      const float inv = Rs > 0.f ? rcp_approx(Rs) : 0.f;
      for (int s2 = 0; s2 < ns; ++s2) wgt[s2 * 64 + h] *= inv;
      if (split == 0)
        p.lse[(int64_t)seq * kDecHeads + h] = Ls > 0.f ? (M + lg2_approx(Ls)) * 0.69314718055994530942f : -INFINITY;
    }
    named_barrier_sync(1, 256);
#pragma unroll 1
    for (int u = 0; u < 4; ++u) {
      const int d = 128 * u + 32 * quarter + lane;  // latent column of this lane
      if (d / W != split) continue;
      float acc[32];
      if (nh > 0 && ok) {
        tmem_ld32(lane_addr + 128 + 64 * u + 32 * grp, acc);
        const float4* w4 = reinterpret_cast<const float4*>(wgt + split * 64 + 32 * grp);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 w = w4[q4];
          acc[4 * q4] *= w.x;
          acc[4 * q4 + 1] *= w.y;
          acc[4 * q4 + 2] *= w.z;
          acc[4 * q4 + 3] *= w.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = 0.f;
      }
      for (int s2 = 0; s2 < ns; ++s2) {
        if (s2 == split) continue;
        const int j = s2 < split ? s2 : s2 - 1;
        const float4* src = reinterpret_cast<const float4*>(smem + LY::RECV_OFF + j * DB + LY::kPartHead +
                                                            (d - split * W) * kHbRecvPitch + grp * 128);
        const float4* w4 = reinterpret_cast<const float4*>(wgt + s2 * 64 + 32 * grp);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 v = src[q4], w = w4[q4];
          acc[4 * q4] = fmaf(v.x, w.x, acc[4 * q4]);
          acc[4 * q4 + 1] = fmaf(v.y, w.y, acc[4 * q4 + 1]);
          acc[4 * q4 + 2] = fmaf(v.z, w.z, acc[4 * q4 + 2]);
          acc[4 * q4 + 3] = fmaf(v.w, w.w, acc[4 * q4 + 3]);
        }
      }
      __nv_bfloat16* dst = p.out + (int64_t)seq * kDecHeads * 512 + d;
#pragma unroll
      for (int i = 0; i < 32; ++i) dst[(int64_t)(32 * grp + i) * 512] = __float2bfloat16_rn(acc[i]);
    }
  }
  // no split leaves while a bulk copy out of its shared memory may still run
  if (ns > 1 && smx) ok = warp_wait_cluster(bar(LY::BAR_SENT), 0, abort_flag) && ok;
  if (ns > 1 && !smx) cluster_wait();  // the other warps' half of the barrier at the start
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace loza
