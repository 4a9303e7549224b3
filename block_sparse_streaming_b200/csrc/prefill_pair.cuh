// prefill_pair.cuh - absorbed-MLA SSA prefill on CTA pairs (tcgen05 cta_group::2).
//
// Same operation as ssa_prefill_kernel for the absorbed shapes (576-wide
// shared latent as K, its first 512 columns as V, 64 query heads), but the
// tensor-core work of two heads of the same 128-query tile is issued as one
// 256-row MMA shared by a cluster pair of CTAs on two SMs:
//   CTA rank r (r = 0, 1) owns head 2*hp + r: its 128 query rows of Q stay in
//   its own shared memory (A rows), its S and O accumulators in its own TMEM.
//   Both heads read the same key blocks (MLA heads share the latent), so the
//   B operands are split between the two CTAs: for S = Q K^T each CTA stages
//   64 of the block's 128 keys, for O += P V each CTA stages 64 of every 128
//   value columns. Every CTA therefore loads half of the K/V bytes per block
//   that a single-CTA tile would, and every MMA reads half as much B from its
//   own shared memory, while each SM still runs full 128-row MMAs.
//
// The key-block walk, masking, online softmax (base 2, lazy rescale) and the
// epilogue are those of the single-CTA kernel (sink blocks then local blocks,
// page 1 section 01 of the LoZA pages; token-causal inside the diagonal
// block). The value dimension is split into two 256-column slices (two pairs
// per tile), each recomputing S, because O for 128 rows x 512 columns would
// fill all of TMEM.
//
// Persistent schedule: one cluster pair per two SMs walks the tiles
// (sequence, query tile, head pair, value slice) pair, pair + npairs, ...;
// consecutive tiles of a wave share their key blocks in L2. Across tiles the
// pipelines do not drain: Q of the next tile streams in as soon as the last
// S MMA of the current tile has read Q, and the next tile's first S MMAs run
// while the softmax warps write the current tile's output.
//
// Roles (10 warps in each CTA):
//   warp 0     TMA producer, in both CTAs: own Q rows per tile, then own
//              halves of the K and V tiles of every selected block, in MMA
//              order. All loads of the pair complete on the even CTA's ring
//              barriers.
//   warp 1     TMEM allocation in both CTAs; in the even CTA also the single
//              thread that issues every MMA of the pair and commits them to
//              the barriers of both CTAs.
//   warps 2-9  softmax / correction / epilogue on the CTA's own 128 rows, two
//              warps per row (each takes half of the keys and half of O); the
//              odd CTA reports P ready to the even CTA's barrier remotely.
#pragma once

#include <cuda.h>

#include "prefill.cuh"
#include "sm100.cuh"

namespace loza {

struct PrefillPairParams {
  CUtensorMap tm_q;    // q [T, H, 576]        box {64, 1, 128}
  CUtensorMap tm_k;    // latent [T, 1, 576]   box {64, 1, 64}   (half a key block)
  CUtensorMap tm_v;    // value [T, 1, 512]    box {64, 1, 128}
  const int32_t* cu_seqlens;
  __nv_bfloat16* out;  // [T, H, 512]
  float* lse;          // [T, H]
  int n_heads;         // even
  int n_qtiles;        // query tiles of the longest sequence
  int total_tiles;     // batch * n_qtiles * n_heads (head pairs x 2 value slices)
  int n_sink;
  int n_local;         // < 0: unbounded
  int block;           // b, tokens per block of the window
  float scale_log2;
};

constexpr int kPairDqk = 576;
constexpr int kPairDv = 512;
constexpr int kPairSlice = 256;               // value columns per pair (O in TMEM)
constexpr int kPairStages = 5;
constexpr int kPairThreads = 320;           // producer, MMA, 8 softmax warps
constexpr int kPairHalfKBytes = 64 * 64 * 2;  // [64 keys x 64 dims] bf16
constexpr int kPairKSlots = 5;                // 9 dim chunks, two per slot
constexpr int kPairVSlots = 2;                // 128 of the slice's columns per CTA

struct PrefillPairLayout {
  static constexpr int NQC = kPairDqk / 64;
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = NQC * kChunkBytes;
  static constexpr int XCH_OFF = RING_OFF + kPairStages * kChunkBytes;  // [2][2][128] f32 row sums
  static constexpr int BAR_OFF = XCH_OFF + 2 * 2 * 128 * 4;
  // q_full, q_empty, ring_full[NSTAGE], ring_empty[NSTAGE], s_full[2], p_full[2], pv_done
  // (P-ready alternates between two barriers by block parity: a warp that has
  // already finished block b+1 must not count towards block b)
  static constexpr int BAR_Q = 0;
  static constexpr int BAR_QE = 1;
  static constexpr int BAR_FULL = 2;
  static constexpr int BAR_EMPTY = 2 + kPairStages;
  static constexpr int BAR_S = 2 + 2 * kPairStages;
  static constexpr int BAR_P = BAR_S + 2;
  static constexpr int BAR_PV = BAR_P + 2;
  static constexpr int NBAR = BAR_PV + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  // No alignment slack: the kernel checks that dynamic shared memory starts
  // on a 1024-byte boundary (128-byte swizzle atoms) and reports otherwise.
  static constexpr int SMEM_BYTES = MISC_OFF + 16;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Tile t of the persistent walk: value slice fastest, then head pair, query
// tile and sequence. Returns false for query tiles past the sequence's end.
struct PairTile {
  int seq, qb, hp, slice, seq_start, seq_len;
  __device__ __forceinline__ bool load(const PrefillPairParams& p, int t) {
    slice = t & 1;
    int r = t >> 1;
    const int hpairs = p.n_heads >> 1;
    hp = r % hpairs;
    r /= hpairs;
    qb = r % p.n_qtiles;
    seq = r / p.n_qtiles;
    seq_start = p.cu_seqlens[seq];
    seq_len = p.cu_seqlens[seq + 1] - seq_start;
    return qb * kTile < seq_len;
  }
};

// Bytes one CTA stages into ring slot k of a key block's K part.
__host__ __device__ constexpr uint32_t pair_k_slot_bytes(int k) {
  return (2 * k + 1 < kPairDqk / 64 ? 2u : 1u) * kPairHalfKBytes;
}

__global__ void __launch_bounds__(kPairThreads, 1)
ssa_prefill_pair_kernel(const __grid_constant__ PrefillPairParams p) {
  using LY = PrefillPairLayout;
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
  const uint32_t lead_bar0 = peer_addr(bar0, 0);  // the even CTA's barriers, cluster address
  auto lead_bar = [&](int i) { return lead_bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar(LY::BAR_Q), 1);
    mbar_init(bar(LY::BAR_QE), 1);
    for (int i = 0; i < kPairStages; ++i) {
      mbar_init(bar(LY::BAR_FULL + i), 1);
      mbar_init(bar(LY::BAR_EMPTY + i), 1);
    }
    mbar_init(bar(LY::BAR_S + 0), 1);
    mbar_init(bar(LY::BAR_S + 1), 1);
    mbar_init(bar(LY::BAR_P + 0), 16);  // one arrival per softmax warp of each CTA
    mbar_init(bar(LY::BAR_P + 1), 16);
    mbar_init(bar(LY::BAR_PV), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (elect_one()) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
    }
    __syncwarp();
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    // Wait until this CTA's copy of the slot is free; the even CTA then
    // announces the bytes both CTAs will deliver to its barrier.
    auto acquire = [&](uint32_t bytes) {
      ok = warp_wait(bar(LY::BAR_EMPTY + slot), phase ^ 1, abort_flag);
      if (ok && rank == 0 && elect_one()) mbar_arrive_expect_tx(bar(LY::BAR_FULL + slot), 2u * bytes);
      __syncwarp();
      return ok;
    };
    auto advance = [&]() {
      if (++slot == kPairStages) { slot = 0; phase ^= 1; }
    };
    int ntile = 0;
    PairTile tl;
    for (int t = pair; t < p.total_tiles && ok; t += npairs) {
      if (!tl.load(p, t)) continue;
      const BlockWalk walk(tl.qb, p.n_sink, p.n_local, p.block);
      const int nb = walk.count;
      const int head = 2 * tl.hp + (int)rank;
      // Q of this tile once the previous tile's last S MMA has read Q
      if (ntile > 0) ok = warp_wait(bar(LY::BAR_QE), (ntile - 1) & 1, abort_flag);
      if (!ok) break;
      if (elect_one()) {
        if (rank == 0) mbar_arrive_expect_tx(bar(LY::BAR_Q), 2u * LY::NQC * kChunkBytes);
        const int row0 = tl.seq_start + tl.qb * kTile;
        for (int c = 0; c < LY::NQC; ++c)
          tma_load_3d_pair(sbase + LY::Q_OFF + c * kChunkBytes, &p.tm_q, lead_bar(LY::BAR_Q), c * 64, head, row0);
      }
      __syncwarp();
      for (int it = 0; it <= nb && ok; ++it) {
        if (it < nb) {
          const int krow = tl.seq_start + walk.block(it) * kTile + 64 * (int)rank;  // this CTA's 64 keys
          for (int k = 0; k < kPairKSlots && ok; ++k) {
            if (!acquire(pair_k_slot_bytes(k))) break;
            if (elect_one()) {
              const uint32_t dst = sbase + LY::RING_OFF + slot * kChunkBytes;
              tma_load_3d_pair(dst, &p.tm_k, lead_bar(LY::BAR_FULL + slot), 128 * k, 0, krow);
              if (2 * k + 1 < LY::NQC)
                tma_load_3d_pair(dst + kPairHalfKBytes, &p.tm_k, lead_bar(LY::BAR_FULL + slot), 128 * k + 64, 0, krow);
            }
            __syncwarp();
            advance();
          }
        }
        if (it >= 1) {
          const int vrow = tl.seq_start + walk.block(it - 1) * kTile;
          for (int m = 0; m < kPairVSlots && ok; ++m) {
            if (!acquire(kChunkBytes)) break;
            if (elect_one())
              tma_load_3d_pair(sbase + LY::RING_OFF + slot * kChunkBytes, &p.tm_v, lead_bar(LY::BAR_FULL + slot),
                               tl.slice * kPairSlice + 128 * m + 64 * (int)rank, 0, vrow);
            __syncwarp();
            advance();
          }
        }
      }
      ++ntile;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (rank == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(256, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(256, 128, false, true);
      constexpr uint16_t kBoth = 0x3;
      const uint32_t tmem_o = tmem + 256;
      const uint64_t dq0 = sdesc_sw128(sbase + LY::Q_OFF, 16, 1024);       // Q chunk 0 (K-major)
      const uint64_t dk0 = sdesc_sw128(sbase + LY::RING_OFF, 16, 1024);    // [64 keys x 64] K-major
      const uint64_t dv0 = sdesc_sw128(sbase + LY::RING_OFF, 8192, 1024);  // [128 keys x 64] MN-major
      int slot = 0;
      uint32_t phase = 0;
      bool ok = true;
      int ntile = 0, g = 0;  // tiles and key blocks done (barrier phases run across tiles)
      PairTile tl;
      for (int t = pair; t < p.total_tiles && ok; t += npairs) {
        if (!tl.load(p, t)) continue;
        const int nb = BlockWalk(tl.qb, p.n_sink, p.n_local, p.block).count;
        ok = warp_wait(bar(LY::BAR_Q), ntile & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        for (int it = 0; it <= nb && ok; ++it) {
          if (it < nb) {
            const int gs = g + it;
            const uint32_t tmem_s = tmem + (gs & 1) * 128;
            for (int k = 0; k < kPairKSlots; ++k) {
              ok = warp_wait(bar(LY::BAR_FULL + slot), phase, abort_flag);
              if (!ok) break;
              tc_fence_after();
              if (elect_one()) {
                const int nc = 2 * k + 1 < LY::NQC ? 2 : 1;
                for (int cc = 0; cc < nc; ++cc) {
                  const int c = 2 * k + cc;
                  const uint64_t da = desc_add(dq0, c * kChunkBytes);
                  const uint64_t db = desc_add(dk0, slot * kChunkBytes + cc * kPairHalfKBytes);
#pragma unroll
                  for (int kk = 0; kk < 4; ++kk)
                    mma_ss_pair(tmem_s, desc_add(da, 32 * kk), desc_add(db, 32 * kk), idesc_s, (c | kk) != 0);
                }
                mma_commit_pair(bar(LY::BAR_EMPTY + slot), kBoth);
              }
              __syncwarp();
              if (++slot == kPairStages) { slot = 0; phase ^= 1; }
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
            ok = warp_wait(bar(LY::BAR_P + (gb & 1)), (gb >> 1) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tmem_p = tmem + (gb & 1) * 128;
            for (int m = 0; m < kPairVSlots; ++m) {
              ok = warp_wait(bar(LY::BAR_FULL + slot), phase, abort_flag);
              if (!ok) break;
              tc_fence_after();
              if (elect_one()) {
                const uint64_t dv = desc_add(dv0, slot * kChunkBytes);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                  mma_ts_pair(tmem_o + 128 * m, tmem_p + kk * 8, desc_add(dv, 2048 * kk), idesc_pv,
                              (b > 0 || kk > 0) ? 1u : 0u);
                mma_commit_pair(bar(LY::BAR_EMPTY + slot), kBoth);
              }
              __syncwarp();
              if (++slot == kPairStages) { slot = 0; phase ^= 1; }
            }
            if (!ok) break;
            if (elect_one()) mma_commit_pair(bar(LY::BAR_PV), kBoth);
            __syncwarp();
          }
        }
        g += nb;
        ++ntile;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue (both CTAs)
    // Eight warps: warps w and w+4 share TMEM lane quarter w & 3 (rows
    // 32*(w&3) .. +31); `half` picks the keys [64*half, +64) whose
    // exponentials this warp computes and the O columns [128*half, +128) it
    // rescales and writes. Both warps of a row take the row maximum over all
    // 128 keys themselves, so they agree on it without exchanging anything.
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    float* xl = reinterpret_cast<float*>(smem + LY::XCH_OFF);  // [2][128] exact row sums
    float* xr = xl + 256;                                       // [2][128] sums of bf16 P
    const float c = p.scale_log2;  // > 0, so max(c*s) = c*max(s)
    bool ok = true;
    int g = 0;  // key blocks done (barrier phases run across tiles)
    PairTile tl;
    for (int t = pair; t < p.total_tiles && ok; t += npairs) {
      if (!tl.load(p, t)) continue;
      const BlockWalk walk(tl.qb, p.n_sink, p.n_local, p.block);
      const int nb = walk.count;
      // m_run: running row maximum of scale*log2(e)*s (the reference of P);
      // l_run: this warp's share of the running sum of 2^(x - m_run) (exact,
      //        for the LSE); r_run: its share of the sum of the bf16-rounded P
      //        values that enter P.V, which normalises O.
      float m_run = -INFINITY, l_run = 0.f, r_run = 0.f;
      for (int b = 0; b < nb && ok; ++b) {
        const int gb = g + b;
        ok = warp_wait(bar(LY::BAR_S + (gb & 1)), (gb >> 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t s_addr = lane_addr + (gb & 1) * 128;
        float so[64], s[64];  // the other warp's keys (maximum only) and this warp's keys
        tmem_ld64x2(s_addr + 64 * (half ^ 1), s_addr + 64 * half, so, s);
        // P is written over the first 64 columns of this S buffer, which hold
        // keys of both warps of the row: neither warp may store P before its
        // partner has loaded all of S.
        named_barrier_sync(2 + quarter, 64);
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
        tmem_st32(s_addr + 32 * half, pk);  // P (bf16 pairs) over the first 64 columns of this S buffer
        const float sum = ((l2[0].x + l2[0].y) + (l2[1].x + l2[1].y)) + ((l2[2].x + l2[2].y) + (l2[3].x + l2[3].y));
        const float rsum = ((r2[0].x + r2[0].y) + (r2[1].x + r2[1].y)) + ((r2[2].x + r2[2].y) + (r2[3].x + r2[3].y));
        l_run = l_run * alpha + sum;
        r_run = r_run * alpha + rsum;
        tmem_st_wait();
        // PV(b-1) is waited every block, after the exponentials (by then it
        // has normally finished): O may then be rescaled before PV(b) runs.
        // The waits are taken in order (PV(b-2) in the previous block, the
        // previous tile's last PV in its epilogue) and PV(b) cannot complete
        // before this warp's P(b) arrival, so each parity wait is exact.
        const bool rescale = __any_sync(0xffffffffu, alpha != 1.f);
        if (b > 0) {
          ok = warp_wait(bar(LY::BAR_PV), (gb - 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          if (rescale) {
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
              const uint32_t o_addr = lane_addr + 256 + 128 * half + 32 * cc;
              float o[32];
              tmem_ld32(o_addr, o);
              uint32_t w[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(o[i] * alpha);
              tmem_st32(o_addr, w);
            }
            tmem_st_wait();
          }
        }
        // one arrival per warp: every lane's TMEM stores have completed
        // (tcgen05.wait::st) and are ordered before lane 0's arrive
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0)
            mbar_arrive(bar(LY::BAR_P + (gb & 1)));
          else
            mbar_arrive_cluster(lead_bar(LY::BAR_P + (gb & 1)));
        }
      }
      if (ok) ok = warp_wait(bar(LY::BAR_PV), (g + nb - 1) & 1, abort_flag);
      // Combine the two warps' sums of each row (fixed order, so both agree).
      // The buffer is rewritten only in the next tile's epilogue, after every
      // softmax warp has passed its next P arrival (which follows these reads).
      if (ok) {
        xl[half * 128 + row] = l_run;
        xr[half * 128 + row] = r_run;
      }
      named_barrier_sync(1, 256);
      if (ok) {
        tc_fence_after();
        const float l_tot = xl[row] + xl[128 + row];
        const float r_tot = xr[row] + xr[128 + row];
        const float inv = 1.f / r_tot;
        const int head = 2 * tl.hp + (int)rank;
        const int qpos = tl.qb * kTile + row;
        const bool valid = qpos < tl.seq_len;
        const int64_t grow = (int64_t)tl.seq_start + qpos;
        __nv_bfloat16* orow =
            p.out + (grow * p.n_heads + head) * (int64_t)kPairDv + tl.slice * kPairSlice + 128 * half;
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          float o[32], o2[32];
          tmem_ld32(lane_addr + 256 + 128 * half + 64 * cc, o);
          tmem_ld32(lane_addr + 256 + 128 * half + 64 * cc + 32, o2);
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            w[i] = pack_bf16(o[2 * i] * inv, o[2 * i + 1] * inv);
            w[16 + i] = pack_bf16(o2[2 * i] * inv, o2[2 * i + 1] * inv);
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 64 * cc);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
        if (valid && tl.slice == 0 && half == 0)
          p.lse[grow * p.n_heads + head] = (m_run + log2f(l_tot)) * 0.69314718055994530942f;
      }
      g += nb;
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
