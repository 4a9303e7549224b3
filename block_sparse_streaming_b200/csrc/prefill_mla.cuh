// prefill_mla.cuh - absorbed-MLA SSA prefill on CTA pairs in two passes over
// the value dimension, computing S once.
//
// Operation: O, LSE of the streaming sparse attention of the LoZA pages (page
// 1 section 01: per query block j the sink blocks and the local blocks
// j-l+1 .. j of b = 128 tokens, token-causal inside block j) for the absorbed
// MLA shapes: 576-wide latent K shared by all heads, V = its first 512 columns.
//
// O of 128 rows x 512 value columns in fp32 fills all of an SM's TMEM, so the
// value dimension is done in two passes of 256 columns by the same CTA pair
// (two heads of one 128-query tile, one 256-row tcgen05 cta_group::2 MMA per
// step, B operands split between the two CTAs as in ssa_prefill_pair_kernel):
//   pass 1: S_b = Q K_b^T, online softmax, O[:, 0:256] += P_b V_b[:, 0:256];
//           every P_b (bf16, exactly the values the MMA used) and the factor
//           by which O was rescaled before it are also written to a
//           per-CTA scratch area in global memory (it stays in L2).
//   pass 2: O[:, 256:512] is accumulated from the stored P_b, with the same
//           rescale factors, and normalised by the same row sums.
// S (576-wide) is computed once instead of once per value half.
//
// Roles (10 warps per CTA), persistent over tiles (one pair per two SMs):
//   warp 0     TMA producer: Q, K halves, V halves (pass 1); stored P and the
//              second-half V halves (pass 2).
//   warp 1     TMEM allocation; in the even CTA the MMA issuer.
//   warps 2-9  softmax / P store / rescale / epilogues, two warps per row.
#pragma once

#include <cuda.h>

#include "prefill.cuh"
#include "sm100.cuh"

namespace loza {

struct PrefillMlaParams {
  CUtensorMap tm_q;    // q [T, H, 576]              box {64, 1, 128}
  CUtensorMap tm_k;    // latent [T, 1, 576]         box {64, 1, 64}
  CUtensorMap tm_v;    // value [T, 1, 512]          box {64, 1, 128}
  CUtensorMap tm_v64;  // value [T, 1, 512]          box {64, 1, 64}
  CUtensorMap tm_p;    // P scratch as lines of 64 bf16  box {64, 128}, unswizzled
  // 4-D views {64 columns, rows, column tile, 1}: two [64 x 64] tiles per request
  CUtensorMap tm_k2;   // latent, tiles of 64 columns (stride 128 B), box {64, 64, 2, 1}
  CUtensorMap tm_v2[2];  // value columns 256 + 64r + 128m (m = 0, 1; r = CTA rank), box {64, 64, 2, 1}
  const int32_t* cu_seqlens;
  __nv_bfloat16* out;  // [T, H, 512]
  float* lse;          // [T, H]
  __nv_bfloat16* p_ws; // [grid CTAs][max_blocks][2 key halves][8 key chunks][128 rows][8 keys]
  float* a_ws;         // [grid CTAs][max_blocks][2 halves][128 rows] rescale factors
  int max_blocks;      // key blocks per tile at most (the window's s + l)
  int n_heads;         // even
  int n_qtiles;
  int total_tiles;     // batch * n_qtiles * n_heads / 2
  int n_sink;
  int n_local;
  int block;           // b, tokens per block of the window
  float scale_log2;
};

constexpr int kMlaStages = 5;
constexpr int kMlaMaxBlocks = 32;  // key blocks per query tile
constexpr int kMlaThreads = 320;
constexpr int kMlaHalfK = 64 * 64 * 2;  // [64 keys x 64 dims]

struct PrefillMlaLayout {
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = 9 * kChunkBytes;
  static constexpr int XCH_OFF = RING_OFF + kMlaStages * kChunkBytes;  // [2][2][128] f32 row sums
  static constexpr int BAR_OFF = XCH_OFF + 2 * 2 * 128 * 4;
  static constexpr int BAR_Q = 0, BAR_QE = 1, BAR_FULL = 2, BAR_EMPTY = 2 + kMlaStages,
                       BAR_S = 2 + 2 * kMlaStages,  // [2]
                       BAR_P = BAR_S + 2,           // [2] pass-1 P ready, by block parity (even CTA)
                       BAR_PV = BAR_P + 2,          // pass-1 P.V done (both)
                       BAR_PG = BAR_PV + 1,         // [kMlaMaxBlocks] P of block b stored to global (this CTA)
                       BAR_E1 = BAR_PG + kMlaMaxBlocks,  // pass-1 O read out by both CTAs (even CTA)
                       BAR_RS = BAR_E1 + 1,         // pass-2 O ready for a rescale (this CTA)
                       BAR_R2 = BAR_RS + 1,         // [2] pass-2 rescale done, per CTA rank (even CTA)
                       BAR_PV2 = BAR_R2 + 2,        // pass-2 P.V done (both)
                       BAR_ROW = BAR_PV2 + 1,       // [4] the two softmax warps of a lane quarter
                       NBAR = BAR_ROW + 4;
  // rescale masks: bit b set if block b rescaled O in some row of a warp;
  // [2 ranks][8 warps] in the even CTA (for the MMA issuer), then [8 warps]
  // of this CTA (for its own softmax warps)
  static constexpr int MASK_OFF = BAR_OFF + NBAR * 8;
  static constexpr int MISC_OFF = MASK_OFF + 24 * 4;
  static constexpr int SMEM_BYTES = MISC_OFF + 16;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct MlaTile {
  int seq, qb, hp, seq_start, seq_len;
  __device__ __forceinline__ bool load(const PrefillMlaParams& p, int t) {
    const int hpairs = p.n_heads >> 1;
    hp = t % hpairs;
    const int r = t / hpairs;
    qb = r % p.n_qtiles;
    seq = r / p.n_qtiles;
    seq_start = p.cu_seqlens[seq];
    seq_len = p.cu_seqlens[seq + 1] - seq_start;
    return qb * kTile < seq_len;
  }
};

__host__ __device__ constexpr uint32_t mla_k_slot_bytes(int k) { return (2 * k + 1 < 9 ? 2u : 1u) * kMlaHalfK; }

__global__ void __launch_bounds__(kMlaThreads, 1)
ssa_prefill_mla_kernel(const __grid_constant__ PrefillMlaParams p) {
  using LY = PrefillMlaLayout;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // same in both CTAs: both leave before any cluster barrier
    if (threadIdx.x == 0) atomicOr(&g_device_status, kErrLayout);
    return;
  }
  const uint32_t rank = cluster_rank();  // 0: the CTA that issues the pair's MMAs
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + LY::BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  const uint32_t lead_bar0 = peer_addr(bar0, 0);
  auto lead_bar = [&](int i) { return lead_bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 4);
  // this CTA's scratch: rows [blockIdx.x * max_blocks * 128, +max_blocks * 128) of P
  const int p_row0 = blockIdx.x * p.max_blocks * kTile;

  if (threadIdx.x == 0) {
    mbar_init(bar(LY::BAR_Q), 1);
    mbar_init(bar(LY::BAR_QE), 1);
    for (int i = 0; i < kMlaStages; ++i) {
      mbar_init(bar(LY::BAR_FULL + i), 1);
      mbar_init(bar(LY::BAR_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(LY::BAR_S + i), 1);
      mbar_init(bar(LY::BAR_P + i), 16);   // one arrival per softmax warp of each CTA
      mbar_init(bar(LY::BAR_R2 + i), 8);   // the softmax warps of CTA rank i
    }
    mbar_init(bar(LY::BAR_PV), 1);
    mbar_init(bar(LY::BAR_PV2), 1);
    for (int i = 0; i < kMlaMaxBlocks; ++i) mbar_init(bar(LY::BAR_PG + i), 8);  // this CTA's softmax warps
    mbar_init(bar(LY::BAR_E1), 16);
    mbar_init(bar(LY::BAR_RS), 1);
    for (int i = 0; i < 4; ++i) mbar_init(bar(LY::BAR_ROW + i), 2);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (elect_one()) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      tma_prefetch_desc(&p.tm_v64);
      tma_prefetch_desc(&p.tm_p);
      tma_prefetch_desc(&p.tm_k2);
      tma_prefetch_desc(&p.tm_v2[rank]);
    }
    __syncwarp();
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    auto acquire = [&](uint32_t bytes) {
      ok = warp_wait(bar(LY::BAR_EMPTY + slot), phase ^ 1, abort_flag);
      if (ok && rank == 0 && elect_one()) mbar_arrive_expect_tx(bar(LY::BAR_FULL + slot), 2u * bytes);
      __syncwarp();
      return ok;
    };
    auto advance = [&]() {
      if (++slot == kMlaStages) { slot = 0; phase ^= 1; }
    };
    int ntile = 0;
    MlaTile tl;
    auto next_tile = [&](int t, MlaTile& x) {
      while (t < p.total_tiles && !x.load(p, t)) t += npairs;
      return t;
    };
    auto load_q = [&](const MlaTile& x) {
      if (elect_one()) {
        if (rank == 0) mbar_arrive_expect_tx(bar(LY::BAR_Q), 2u * 9 * kChunkBytes);
        const int row0 = x.seq_start + x.qb * kTile;
        for (int c = 0; c < 9; ++c)
          tma_load_3d_pair(sbase + LY::Q_OFF + c * kChunkBytes, &p.tm_q, lead_bar(LY::BAR_Q), c * 64,
                           2 * x.hp + (int)rank, row0);
      }
      __syncwarp();
    };
    uint32_t pg_parity = 0;  // bit b: parity of the next phase of PG[b]
    int t = next_tile(pair, tl);
    if (t < p.total_tiles) load_q(tl);
    while (t < p.total_tiles && ok) {
      const BlockWalk walk(tl.qb, p.n_sink, p.n_local, p.block);
      const int nb = walk.count;
      // pass 1: K halves of every block, value columns [0, 256)
      for (int it = 0; it <= nb && ok; ++it) {
        if (it < nb) {
          const int krow = tl.seq_start + walk.block(it) * kTile + 64 * (int)rank;
          for (int k = 0; k < 5 && ok; ++k) {
            if (!acquire(mla_k_slot_bytes(k))) break;
            if (elect_one()) {
              // column tiles 2k and 2k+1 in one request (a TMA request has a
              // fixed cost); the rope tile 8 alone
              const uint32_t dst = sbase + LY::RING_OFF + slot * kChunkBytes;
              if (2 * k + 1 < 9)
                tma_load_4d_pair(dst, &p.tm_k2, lead_bar(LY::BAR_FULL + slot), 0, krow, 2 * k, 0);
              else
                tma_load_3d_pair(dst, &p.tm_k, lead_bar(LY::BAR_FULL + slot), 128 * k, 0, krow);
            }
            __syncwarp();
            advance();
          }
        }
        if (it >= 1) {
          const int vrow = tl.seq_start + walk.block(it - 1) * kTile;
          for (int m = 0; m < 2 && ok; ++m) {
            if (!acquire(kChunkBytes)) break;
            if (elect_one())
              tma_load_3d_pair(sbase + LY::RING_OFF + slot * kChunkBytes, &p.tm_v, lead_bar(LY::BAR_FULL + slot),
                               128 * m + 64 * (int)rank, 0, vrow);
            __syncwarp();
            advance();
          }
        }
      }
      // the next tile's Q, as soon as this tile's S no longer read Q
      MlaTile tn;
      const int t_next = next_tile(t + npairs, tn);
      if (ok && t_next < p.total_tiles) {
        ok = warp_wait(bar(LY::BAR_QE), ntile & 1, abort_flag);
        if (ok) load_q(tn);
      }
      // pass 2: the stored P of every block (once it is in global memory) and
      // value columns [256, 512); per block and key half kh: P[:, 64kh .. +64]
      // (one slot), then this CTA's value columns of both 128-column groups
      // for those keys (one slot)
      for (int b = 0; b < nb && ok; ++b) {
        // PG[b] completes once per tile that has a block b
        ok = warp_wait(bar(LY::BAR_PG + b), (pg_parity >> b) & 1u, abort_flag);
        pg_parity ^= 1u << b;
        if (!ok) break;
        const int vrow = tl.seq_start + walk.block(b) * kTile;
        for (int kh = 0; kh < 2 && ok; ++kh) {
          if (!acquire(kChunkBytes)) break;
          if (elect_one())
            tma_load_2d_pair(sbase + LY::RING_OFF + slot * kChunkBytes, &p.tm_p, lead_bar(LY::BAR_FULL + slot), 0,
                             2 * p_row0 + (2 * b + kh) * kTile);
          __syncwarp();
          advance();
          if (!acquire(kChunkBytes)) break;
          if (elect_one())  // this CTA's columns of both 128-column groups, one request
            tma_load_4d_pair(sbase + LY::RING_OFF + slot * kChunkBytes, &p.tm_v2[rank], lead_bar(LY::BAR_FULL + slot),
                             0, vrow + 64 * kh, 0, 0);
          __syncwarp();
          advance();
        }
      }
      ++ntile;
      t = t_next;
      tl = tn;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    // TMEM columns: the tile's S double buffer and later its pass-2 O share
    // one half (ra); its pass-1 O is the other half. ra alternates between
    // tiles, so pass 2 runs while the softmax warps read out pass-1 O, and the
    // next tile's first S while they read out pass-2 O.
    if (rank == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(256, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(256, 128, false, true);
      constexpr uint16_t kBoth = 0x3;
      const uint64_t dq0 = sdesc_sw128(sbase + LY::Q_OFF, 16, 1024);       // Q column tile (K-major)
      const uint64_t dk0 = sdesc_sw128(sbase + LY::RING_OFF, 16, 1024);    // [64 keys x 64] K-major
      const uint64_t dp0 = sdesc_interleave(sbase + LY::RING_OFF, 2048, 128);  // P [128 x 64 keys] K-major, unswizzled
      const uint64_t dv0 = sdesc_sw128(sbase + LY::RING_OFF, 8192, 1024);  // [128 or 64 keys x 64 values] MN-major
      const volatile uint32_t* masks = reinterpret_cast<const volatile uint32_t*>(smem + LY::MASK_OFF);
      int slot = 0;
      uint32_t phase = 0;
      bool ok = true;
      int ntile = 0, g = 0;
      int ev[2] = {0, 0};  // rescale events so far, per CTA rank
      MlaTile tl;
      auto next_full = [&]() {
        ok = warp_wait(bar(LY::BAR_FULL + slot), phase, abort_flag);
        if (ok) tc_fence_after();
        return ok;
      };
      auto advance = [&]() {
        if (++slot == kMlaStages) { slot = 0; phase ^= 1; }
      };
      for (int t = pair; t < p.total_tiles && ok; t += npairs) {
        if (!tl.load(p, t)) continue;
        const int nb = BlockWalk(tl.qb, p.n_sink, p.n_local, p.block).count;
        const uint32_t ra = (uint32_t)(ntile & 1) * 256;
        const uint32_t tmem_o1 = tmem + (256 - ra);
        const uint32_t tmem_o2 = tmem + ra;
        ok = warp_wait(bar(LY::BAR_Q), ntile & 1, abort_flag);
        // S overwrites the columns of the previous tile's pass-1 O
        if (ok && ntile > 0) ok = warp_wait(bar(LY::BAR_E1), (ntile - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        // ---------------- pass 1: S and the first 256 value columns
        for (int it = 0; it <= nb && ok; ++it) {
          if (it < nb) {
            const int gs = g + it;
            const uint32_t tmem_s = tmem + ra + (gs & 1) * 128;
            for (int k = 0; k < 5; ++k) {
              if (!next_full()) break;
              if (elect_one()) {
                const int nc = 2 * k + 1 < 9 ? 2 : 1;
                for (int cc = 0; cc < nc; ++cc) {
                  const int c = 2 * k + cc;
                  const uint64_t da = desc_add(dq0, c * kChunkBytes);
                  const uint64_t db = desc_add(dk0, slot * kChunkBytes + cc * kMlaHalfK);
#pragma unroll
                  for (int kk = 0; kk < 4; ++kk)
                    mma_ss_pair(tmem_s, desc_add(da, 32 * kk), desc_add(db, 32 * kk), idesc_s, (c | kk) != 0);
                }
                mma_commit_pair(bar(LY::BAR_EMPTY + slot), kBoth);
              }
              __syncwarp();
              advance();
            }
            if (!ok) break;
            if (elect_one()) {
              mma_commit_pair(bar(LY::BAR_S + (gs & 1)), kBoth);
              if (it == nb - 1) mma_commit_pair(bar(LY::BAR_QE), kBoth);  // Q no longer read
            }
            __syncwarp();
          }
          if (it >= 1) {
            const int b = it - 1;
            const int gb = g + b;
            // the last block's arrivals also publish the warps' rescale masks
            ok = b == nb - 1 ? warp_wait_cluster(bar(LY::BAR_P + (gb & 1)), (gb >> 1) & 1, abort_flag)
                             : warp_wait(bar(LY::BAR_P + (gb & 1)), (gb >> 1) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tmem_p = tmem + ra + (gb & 1) * 128;
            for (int m = 0; m < 2; ++m) {
              if (!next_full()) break;
              if (elect_one()) {
                const uint64_t dv = desc_add(dv0, slot * kChunkBytes);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                  mma_ts_pair(tmem_o1 + 128 * m, tmem_p + kk * 8, desc_add(dv, 2048 * kk), idesc_pv,
                              (b > 0 || kk > 0) ? 1u : 0u);
                mma_commit_pair(bar(LY::BAR_EMPTY + slot), kBoth);
              }
              __syncwarp();
              advance();
            }
            if (!ok) break;
            if (elect_one()) mma_commit_pair(bar(LY::BAR_PV), kBoth);
            __syncwarp();
          }
        }
        if (!ok) break;
        // ---------------- pass 2: the stored P against value columns [256, 512);
        // O is rescaled only at the blocks where some row of a CTA rescaled in pass 1
        uint32_t rmask[2] = {0u, 0u};
        for (int w = 0; w < 8; ++w) {
          rmask[0] |= masks[w];
          rmask[1] |= masks[8 + w];
        }
        for (int b = 0; b < nb && ok; ++b) {
          for (int c = 0; c < 2 && ok; ++c) {
            if ((rmask[c] >> b) & 1u) {
              ok = warp_wait(bar(LY::BAR_R2 + c), ev[c] & 1, abort_flag);
              ++ev[c];
            }
          }
          if (!ok) break;
          tc_fence_after();
          for (int kh = 0; kh < 2; ++kh) {
            if (!next_full()) break;
            const int pslot = slot;
            advance();
            if (!next_full()) break;
            if (elect_one()) {
              const uint64_t da = desc_add(dp0, pslot * kChunkBytes);
              const uint64_t dv = desc_add(dv0, slot * kChunkBytes);
              for (int m = 0; m < 2; ++m) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_ss_pair(tmem_o2 + 128 * m, desc_add(da, 4096 * kk), desc_add(dv, m * kMlaHalfK + 2048 * kk),
                              idesc_pv, (b > 0 || kh > 0 || kk > 0) ? 1u : 0u);
              }
              mma_commit_pair(bar(LY::BAR_EMPTY + pslot), kBoth);
              mma_commit_pair(bar(LY::BAR_EMPTY + slot), kBoth);
            }
            __syncwarp();
            advance();
          }
          if (!ok) break;
          // O holds blocks 0 .. b once these complete: a CTA that rescales at b + 1 may start
          if (elect_one()) {
            for (int c = 0; c < 2; ++c)
              if (b + 1 < nb && ((rmask[c] >> (b + 1)) & 1u)) mma_commit_pair(bar(LY::BAR_RS), (uint16_t)(1u << c));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) mma_commit_pair(bar(LY::BAR_PV2), kBoth);
        __syncwarp();
        g += nb;
        ++ntile;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogues (both CTAs)
    // Warps w and w+4 share TMEM lane quarter w & 3; `half` picks the keys
    // [64*half, +64) whose exponentials this warp computes and the O columns
    // [128*half, +128) it rescales and writes, in both passes.
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    float* xl = reinterpret_cast<float*>(smem + LY::XCH_OFF);  // [2][128] exact row sums
    float* xr = xl + 256;                                       // [2][128] sums of bf16 P
    __nv_bfloat16* p_mine = p.p_ws + (size_t)p_row0 * kTile;    // this CTA's stored P
    float* a_mine = p.a_ws + (size_t)blockIdx.x * p.max_blocks * 256;  // this CTA's rescale factors
    const float c = p.scale_log2;
    // this warp's rescale mask: its slot in the even CTA, and in this CTA
    const uint32_t mask_lead = peer_addr(sbase + LY::MASK_OFF, 0) + 4u * (rank * 8 + (warp - 2));
    volatile uint32_t* mask_own = reinterpret_cast<volatile uint32_t*>(smem + LY::MASK_OFF + 64);
    bool ok = true;
    int g = 0, n_row = 0, ntile = 0, n_ev = 0;
    MlaTile tl;
    auto arrive_lead = [&](int i) {
      if (rank == 0)
        mbar_arrive(bar(i));
      else
        mbar_arrive_cluster(lead_bar(i));
    };
    // multiply this warp's 128 columns of the O at TMEM column o_col by alpha (per row)
    auto rescale_o = [&](uint32_t o_col, float alpha) {
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        const uint32_t o_addr = lane_addr + o_col + 128 * half + 32 * cc;
        float o[32];
        tmem_ld32(o_addr, o);
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(o[i] * alpha);
        tmem_st32(o_addr, w);
      }
      tmem_st_wait();
    };
    // write this warp's 128 O columns, normalised, to value columns col0 ..;
    // rows [0, n_valid) of the tile exist. Each 8-lane group transposes its
    // 8 rows x 8 chunks of 16 bytes, so that every store of the warp writes
    // four whole 128-byte row segments.
    const int j8 = lane & 7;
    const int r8 = quarter * 32 + (lane & ~7);  // first row of this lane's group
    auto store_o = [&](uint32_t o_col, float inv, int64_t grow0, int n_valid, int head, int col0) {
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        float o[32], o2[32];
        tmem_ld32(lane_addr + o_col + 128 * half + 64 * cc, o);
        tmem_ld32(lane_addr + o_col + 128 * half + 64 * cc + 32, o2);
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          w[i] = pack_bf16(o[2 * i] * inv, o[2 * i + 1] * inv);
          w[16 + i] = pack_bf16(o2[2 * i] * inv, o2[2 * i + 1] * inv);
        }
        transpose8x8_u4(w, lane);  // now chunk j8 of rows r8 .. r8 + 7
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (r8 + k < n_valid) {
            __nv_bfloat16* dst =
                p.out + ((grow0 + r8 + k) * p.n_heads + head) * (int64_t)512 + col0 + 128 * half + 64 * cc + 8 * j8;
            *reinterpret_cast<uint4*>(dst) = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
          }
        }
      }
    };
    for (int t = pair; t < p.total_tiles && ok; t += npairs) {
      if (!tl.load(p, t)) continue;
      const BlockWalk walk(tl.qb, p.n_sink, p.n_local, p.block);
      const int nb = walk.count;
      const int head = 2 * tl.hp + (int)rank;
      // m_run: running row maximum of scale*log2(e)*s (the reference of P);
      // l_run / r_run: this warp's share of the exact / bf16-rounded sums of P
      float m_run = -INFINITY, l_run = 0.f, r_run = 0.f;
      const uint32_t ra = (uint32_t)(ntile & 1) * 256;  // S and pass-2 O; pass-1 O at 256 - ra
      uint32_t wmask = 0;  // blocks at which some row of this warp rescaled O
      // ---------------- pass 1
      for (int b = 0; b < nb && ok; ++b) {
        const int gb = g + b;
        ok = warp_wait(bar(LY::BAR_S + (gb & 1)), (gb >> 1) & 1, abort_flag);
        if (!ok) break;
        if (b > 0) {
          // the previous block's P (stored a block ago) is visible to the TMA loads of pass 2
          fence_proxy_async_global();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(LY::BAR_PG + b - 1));
        }
        tc_fence_after();
        const uint32_t s_addr = lane_addr + ra + (gb & 1) * 128;
        float so[64], s[64];  // the other warp's keys (maximum only) and this warp's keys
        tmem_ld64x2(s_addr + 64 * (half ^ 1), s_addr + 64 * half, so, s);
        // P is stored over S columns holding keys of both warps of the row:
        // neither stores before its partner warp has loaded S
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(LY::BAR_ROW + quarter));
        ok = warp_wait(bar(LY::BAR_ROW + quarter), n_row & 1, abort_flag);
        ++n_row;
        if (!ok) break;
        if (walk.masked(walk.block(b), tl.qb)) {
          // keys this row does not see: after its query (the diagonal tile), or
          // between the sinks and its local range (tiles at the window's edges)
          const SsaWindow win{p.block, walk.sink_end, p.n_local};
          const RowMask rm(win, tl.qb * kTile + row, walk.block(b) * kTile);
          const uint64_t vo = rm.bits64(64 * (half ^ 1)), vs = rm.bits64(64 * half);
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            if (!((vo >> j) & 1ull)) so[j] = -INFINITY;
            if (!((vs >> j) & 1ull)) s[j] = -INFINITY;
          }
        }
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < 32; ++j) m4[j & 3] = fmax3(m4[j & 3], so[2 * j], so[2 * j + 1]);
#pragma unroll
        for (int j = 0; j < 32; ++j) m4[j & 3] = fmax3(m4[j & 3], s[2 * j], s[2 * j + 1]);
        const float mx = c * fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        // keep the stale maximum unless this block raises it by more than 2^8
        float alpha = 1.f;
        if (b == 0) {
          m_run = mx;
        } else if (mx > m_run + (float)kRescaleThreshold) {
          alpha = ex2_approx(m_run - mx);
          m_run = mx;
        }
        const float2 c2 = make_float2(c, c);
        // a row that has seen no key yet (all masked so far) takes P = 0
        const float nm = m_run == -INFINITY ? 0.f : -m_run;
        const float2 nm2 = make_float2(nm, nm);
        float2 l2[4], r2[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) l2[i] = r2[i] = make_float2(0.f, 0.f);
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 x = ffma2(make_float2(s[2 * i], s[2 * i + 1]), c2, nm2);
          const float p0 = ex2_approx(x.x);
          const float p1 = ex2_approx(x.y);
          pk[i] = pack_bf16(p0, p1);
          l2[i & 3] = fadd2(l2[i & 3], make_float2(p0, p1));
          r2[i & 3] = fadd2(r2[i & 3], make_float2(__uint_as_float(pk[i] << 16), __uint_as_float(pk[i] & 0xFFFF0000u)));
        }
        tmem_st32(s_addr + 32 * half, pk);  // P for pass 1's P.V, over the first 64 columns of S
        {
          // the same P and the rescale factor, for pass 2: chunk i of 8 keys of
          // every row is contiguous, so each store of a warp fills 512 bytes
          uint4* dst = reinterpret_cast<uint4*>(p_mine + (size_t)(b * 2 + half) * (8 * kTile * 8)) + row;
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i * kTile] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          a_mine[(b * 2 + half) * 128 + row] = alpha;
        }
        l_run = l_run * alpha + (((l2[0].x + l2[0].y) + (l2[1].x + l2[1].y)) + ((l2[2].x + l2[2].y) + (l2[3].x + l2[3].y)));
        r_run = r_run * alpha + (((r2[0].x + r2[0].y) + (r2[1].x + r2[1].y)) + ((r2[2].x + r2[2].y) + (r2[3].x + r2[3].y)));
        tmem_st_wait();
        // PV(b-1) is waited every block (parity waits in order); O is then
        // rescaled, if the maximum moved, before PV(b) runs
        const bool rescale = __any_sync(0xffffffffu, alpha != 1.f);  // never at b == 0
        if (b > 0) {
          ok = warp_wait(bar(LY::BAR_PV), (gb - 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          if (rescale) {
            rescale_o(256 - ra, alpha);
            wmask |= 1u << b;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (b == nb - 1) {
            // publish the mask: to the MMA issuer with this arrival, and to this CTA's warps
            mask_own[warp - 2] = wmask;
            if (rank == 0) {
              *reinterpret_cast<volatile uint32_t*>(smem + LY::MASK_OFF + 4 * (warp - 2)) = wmask;
              mbar_arrive(bar(LY::BAR_P + (gb & 1)));
            } else {
              st_cluster_u32(mask_lead, wmask);
              mbar_arrive_cluster_release(lead_bar(LY::BAR_P + (gb & 1)));
            }
          } else {
            arrive_lead(LY::BAR_P + (gb & 1));
          }
        }
      }
      // the last block's P
      fence_proxy_async_global();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(LY::BAR_PG + nb - 1));
      // ---------------- epilogue 1: value columns [0, 256)
      if (ok) ok = warp_wait(bar(LY::BAR_PV), (g + nb - 1) & 1, abort_flag);
      if (ok) {
        xl[half * 128 + row] = l_run;
        xr[half * 128 + row] = r_run;
      }
      named_barrier_sync(1, 256);
      const float l_tot = xl[row] + xl[128 + row];
      const float r_tot = xr[row] + xr[128 + row];
      const float inv = 1.f / r_tot;
      uint32_t cmask = 0;  // blocks at which some row of this CTA rescaled O
      for (int w = 0; w < 8; ++w) cmask |= mask_own[w];
      const int qpos = tl.qb * kTile + row;
      const bool valid = qpos < tl.seq_len;
      const int64_t grow = (int64_t)tl.seq_start + qpos;
      const int64_t grow0 = (int64_t)tl.seq_start + tl.qb * kTile;
      const int n_valid = min(kTile, tl.seq_len - tl.qb * kTile);
      if (ok) {
        tc_fence_after();
        store_o(256 - ra, inv, grow0, n_valid, head, 0);
        if (valid && half == 0) p.lse[grow * p.n_heads + head] = (m_run + log2f(l_tot)) * 0.69314718055994530942f;
      }
      // pass-1 O has been read: the next tile's S may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_lead(LY::BAR_E1);
      // ---------------- pass 2: repeat pass 1's rescales on value columns [256, 512),
      // at the blocks where some row of this CTA rescaled
      for (int b = 1; b < nb && ok; ++b) {
        if (!((cmask >> b) & 1u)) continue;
        const float alpha = a_mine[(b * 2 + half) * 128 + row];  // this thread's own pass-1 write
        ok = warp_wait(bar(LY::BAR_RS), n_ev & 1, abort_flag);
        ++n_ev;
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) rescale_o(ra, alpha);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_lead(LY::BAR_R2 + (int)rank);
      }
      // ---------------- epilogue 2: value columns [256, 512)
      if (ok) ok = warp_wait(bar(LY::BAR_PV2), ntile & 1, abort_flag);
      if (ok) {
        tc_fence_after();
        store_o(ra, inv, grow0, n_valid, head, 256);
      }
      // the sums buffer is rewritten only after every warp has read it, and
      // all softmax warps leave together once any role gave up
      named_barrier_sync(1, 256);
      ok = ok && *abort_flag == 0;
      g += nb;
      ++ntile;
    }
  }

  // Neither CTA releases TMEM or shared memory while the other may still use
  // them: the even CTA's MMAs read the odd CTA's shared memory and write its TMEM.
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace loza
