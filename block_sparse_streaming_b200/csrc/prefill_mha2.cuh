// prefill_mha2.cuh - SSA prefill / training forward with per-head K and V
// (the 192 / 128 shape), two query tiles per CTA.
//
// Operation: O, LSE of the streaming sparse attention of the LoZA pages (page
// 1 section 01: per query block j the sink blocks and the local blocks
// j-l+1 .. j of b = 128 tokens, token-causal inside block j).
//
// With a K and V per head, a 128-query tile moves 80 KB of K and V per key
// block for 10.5 MFLOP of MMA work, more than one SM's TMA engine delivers in
// the time the tensor cores need for it. A CTA here takes two consecutive
// query tiles qb0 = 2t, qb1 = 2t+1 of one head: every key block of the union of
// their windows is loaded once and multiplied against both tiles, halving the
// bytes per FLOP. Each tile has its own S (single-buffered) and O in TMEM and
// its own softmax warpgroup, and the two tiles alternate on the tensor pipe:
//   S0(i) S1(i) | PV0(i) S0(i+1) | PV1(i) S1(i+1) | ...
// so warpgroup 0 works on S0(i+1) while the MMAs of tile 1 run, and the
// other way round. A block only one tile sees (the oldest local block of
// tile 0, the diagonal block of tile 1) is multiplied against that tile only.
//
// Roles (10 warps): warp 0 TMA producer (Q of both tiles, then K and V
// [128 x 64] tiles of every block of the union, into an 8-slot ring; a slot is
// released after the last MMA that reads it); warp 1 TMEM allocation and MMA
// issuer; warps 2-5 softmax of tile 0, warps 6-9 softmax of tile 1 (one query
// row per thread, online softmax in base 2, lazy rescale above 2^8).
//
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
#pragma once

#include <cuda.h>

#include "prefill.cuh"
#include "sm100.cuh"

namespace loza {

constexpr int kMha2Threads = 320;
constexpr int kMha2Stages = 8;

template <int DQK, int DV>
struct PrefillMha2Layout {
  static constexpr int NQC = DQK / 64;
  static constexpr int NVC = DV / 64;
  static constexpr int Q_OFF = 0;                                    // [2 tiles][NQC] tiles
  static constexpr int RING_OFF = 2 * NQC * kChunkBytes;
  static constexpr int BAR_OFF = RING_OFF + kMha2Stages * kChunkBytes;
  // barriers: q_full, ring_full[8], ring_empty[8], s_full[2], p_full[2], pv_done[2] (per tile)
  static constexpr int BAR_Q = 0, BAR_FULL = 1, BAR_EMPTY = 1 + kMha2Stages, BAR_S = 1 + 2 * kMha2Stages,
                       BAR_P = BAR_S + 2, BAR_PV = BAR_P + 2, NBAR = BAR_PV + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem base (u32), abort (int)
  static constexpr int SMEM_BYTES = MISC_OFF + 16;
  static_assert(DQK % 64 == 0 && DV == 128, "tile shape");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// The key blocks of the union of the windows of query blocks qb0 and qb1 =
// qb0 + 1 (sinks first, then the local blocks in increasing order), and which
// of the two tiles sees each of them.
struct PairWalk {
  int sinks, lo, count, qb0, lo0, lo1, sinks0, sinks1;
  bool has1;
  __device__ __forceinline__ PairWalk(int qb0_, bool has1_, int n_sink, int n_local) {
    qb0 = qb0_;
    has1 = has1_;
    const int qb_last = has1 ? qb0 + 1 : qb0;
    sinks = min(n_sink, qb_last + 1);
    lo = n_local < 0 ? sinks : max(n_sink, qb0 - n_local + 1);
    count = sinks + max(0, qb_last - lo + 1);
    sinks0 = min(n_sink, qb0 + 1);
    lo0 = n_local < 0 ? sinks0 : max(n_sink, qb0 - n_local + 1);
    sinks1 = min(n_sink, qb0 + 2);
    lo1 = n_local < 0 ? sinks1 : max(n_sink, qb0 + 1 - n_local + 1);
  }
  __device__ __forceinline__ int block(int i) const { return i < sinks ? i : lo + (i - sinks); }
  __device__ __forceinline__ bool vis0(int kb) const { return kb <= qb0 && (kb < sinks0 || kb >= lo0); }
  __device__ __forceinline__ bool vis1(int kb) const { return has1 && kb <= qb0 + 1 && (kb < sinks1 || kb >= lo1); }
};

template <int DQK, int DV>
__global__ void __launch_bounds__(kMha2Threads, 1)
ssa_prefill_mha2_kernel(const __grid_constant__ PrefillParams p) {
  using LY = PrefillMha2Layout<DQK, DV>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(&g_device_status, kErrLayout);
    return;
  }
  const int qb0 = 2 * blockIdx.x;
  const int head = blockIdx.y;
  const int seq = blockIdx.z;
  const int seq_start = p.cu_seqlens[seq];
  const int seq_len = p.cu_seqlens[seq + 1] - seq_start;
  if (qb0 * kTile >= seq_len) return;  // whole CTA leaves before any setup
  const bool has1 = (qb0 + 1) * kTile < seq_len;
  const int hk = head / (p.n_heads / p.n_kv_heads);
  const PairWalk walk(qb0, has1, p.n_sink, p.n_local);
  const int nb = walk.count;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + LY::BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar(LY::BAR_Q), 1);
    for (int i = 0; i < kMha2Stages; ++i) {
      mbar_init(bar(LY::BAR_FULL + i), 1);
      mbar_init(bar(LY::BAR_EMPTY + i), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(LY::BAR_S + t), 1);
      mbar_init(bar(LY::BAR_P + t), 4);  // one arrival per softmax warp of the tile
      mbar_init(bar(LY::BAR_PV + t), 1);
    }
    *abort_flag = 0;
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

  // ring position of chunk c of the K or V tiles of union block i (load order)
  auto kpos = [&](int i, int c) { return i * (LY::NQC + LY::NVC) + c; };
  auto vpos = [&](int i, int c) { return i * (LY::NQC + LY::NVC) + LY::NQC + c; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      const int ntq = has1 ? 2 : 1;
      mbar_arrive_expect_tx(bar(LY::BAR_Q), ntq * LY::NQC * kChunkBytes);
      for (int t = 0; t < ntq; ++t)
        for (int c = 0; c < LY::NQC; ++c)
          tma_load_3d(sbase + LY::Q_OFF + (t * LY::NQC + c) * kChunkBytes, &p.tm_q, bar(LY::BAR_Q), c * 64, head,
                      seq_start + (qb0 + t) * kTile);
    }
    __syncwarp();
    bool ok = true;
    auto load_tile = [&](int n, const CUtensorMap* map, int col, int row) {
      const int slot = n % kMha2Stages;
      ok = warp_wait(bar(LY::BAR_EMPTY + slot), ((n / kMha2Stages) & 1) ^ 1, abort_flag);
      if (!ok) return;
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(LY::BAR_FULL + slot), kChunkBytes);
        tma_load_3d(sbase + LY::RING_OFF + slot * kChunkBytes, map, bar(LY::BAR_FULL + slot), col, hk, row);
      }
      __syncwarp();
    };
    for (int i = 0; i < nb && ok; ++i) {
      const int row = seq_start + walk.block(i) * kTile;
      for (int c = 0; c < LY::NQC && ok; ++c) load_tile(kpos(i, c), &p.tm_k, c * 64, row);
      for (int c = 0; c < LY::NVC && ok; ++c) load_tile(vpos(i, c), &p.tm_v, c * 64, row);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16(128, 64, false, true);
    const uint64_t dq0 = sdesc_sw128(sbase + LY::Q_OFF, 16, 1024);       // Q tiles (K-major)
    const uint64_t dk0 = sdesc_sw128(sbase + LY::RING_OFF, 16, 1024);    // ring slot 0 read K-major
    const uint64_t dv0 = sdesc_sw128(sbase + LY::RING_OFF, 8192, 1024);  // ring slot 0 read MN-major
    bool ok = warp_wait(bar(LY::BAR_Q), 0, abort_flag);
    tc_fence_after();
    int np[2] = {0, 0};  // PV issued per tile (phases of P_t waited)
    auto wait_full = [&](int n) {
      ok = warp_wait(bar(LY::BAR_FULL + n % kMha2Stages), (n / kMha2Stages) & 1, abort_flag);
      if (ok) tc_fence_after();
    };
    // S_t of union block i; `first` / `last`: this is the first / last MMA group reading K(i)
    auto issue_s = [&](int t, int i, bool first, bool last) {
      for (int c = 0; c < LY::NQC && ok; ++c) {
        const int n = kpos(i, c);
        if (first) wait_full(n);
        if (!ok) break;
        if (elect_one()) {
          const uint64_t da = desc_add(dq0, (t * LY::NQC + c) * kChunkBytes);
          const uint64_t db = desc_add(dk0, (n % kMha2Stages) * kChunkBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + 128 * t, desc_add(da, 32 * kk), desc_add(db, 32 * kk), idesc_s, (c | kk) != 0);
          if (last) mma_commit(bar(LY::BAR_EMPTY + n % kMha2Stages));
        }
        __syncwarp();
      }
      if (ok && elect_one()) mma_commit(bar(LY::BAR_S + t));
      __syncwarp();
    };
    auto issue_pv = [&](int t, int i, bool first, bool last) {
      ok = warp_wait(bar(LY::BAR_P + t), np[t] & 1, abort_flag);
      if (!ok) return;
      tc_fence_after();
      for (int c = 0; c < LY::NVC && ok; ++c) {
        const int n = vpos(i, c);
        if (first) wait_full(n);
        if (!ok) break;
        if (elect_one()) {
          const uint64_t dv = desc_add(dv0, (n % kMha2Stages) * kChunkBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + 256 + 128 * t + c * 64, tmem + 128 * t + kk * 8, desc_add(dv, 2048 * kk), idesc_pv,
                   (np[t] > 0 || kk > 0) ? 1u : 0u);
          if (last) mma_commit(bar(LY::BAR_EMPTY + n % kMha2Stages));
        }
        __syncwarp();
      }
      if (ok && elect_one()) mma_commit(bar(LY::BAR_PV + t));
      __syncwarp();
      ++np[t];
    };
    // PV0(i-1), S0(i), PV1(i-1), S1(i): softmax warpgroup 0 works on S0(i)
    // while tile 1's MMAs run, and the other way round
    bool pv0 = false, pv1 = false;  // visibility of block i-1
    for (int i = 0; i <= nb && ok; ++i) {
      bool s0 = false, s1 = false;
      if (i < nb) {
        const int kb = walk.block(i);
        s0 = walk.vis0(kb);
        s1 = walk.vis1(kb);
      }
      if (pv0) issue_pv(0, i - 1, true, !pv1);
      if (ok && s0) issue_s(0, i, true, !s1);
      if (ok && pv1) issue_pv(1, i - 1, !pv0, true);
      if (ok && s1) issue_s(1, i, !s0, true);
      pv0 = s0;
      pv1 = s1;
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue of tile t
    const int t = (warp - 2) >> 2;
    const int qb = qb0 + t;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // row of the tile == TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t s_addr = lane_addr + 128 * t;
    const uint32_t o_addr = lane_addr + 256 + 128 * t;
    // m_run: running row maximum of scale*log2(e)*s (the reference of P);
    // l_run: running sum of 2^(x - m_run) (exact, for the LSE);
    // r_run: running sum of the bf16-rounded P values that enter P.V, so that
    //        O is normalised by exactly the weights it was accumulated with.
    float m_run = -INFINITY, l_run = 0.f, r_run = 0.f;
    const float c = p.scale_log2;  // > 0, so max(c*s) = c*max(s)
    bool ok = t == 0 || has1;
    int k = 0;  // blocks of this tile so far
    for (int i = 0; i < nb && ok; ++i) {
      const int kb = walk.block(i);
      if (!(t == 0 ? walk.vis0(kb) : walk.vis1(kb))) continue;
      ok = warp_wait(bar(LY::BAR_S + t), k & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      float s[128];
      tmem_ld128(s_addr, s);
      // the diagonal block is token-causal: keys after this row's query do not exist
      if (kb == qb) {
#pragma unroll
        for (int j = 0; j < 128; ++j)
          if (j > row) s[j] = -INFINITY;
      }
      float mx;
      {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < 64; ++j) m4[j & 3] = fmax3(m4[j & 3], s[2 * j], s[2 * j + 1]);
        mx = c * fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      }
      // keep the stale maximum unless this block raises it by more than 2^8
      float alpha = 1.f;
      if (k == 0) {
        m_run = mx;
      } else if (mx > m_run + (float)kRescaleThreshold) {
        alpha = ex2_approx(m_run - mx);
        m_run = mx;
      }
      const float2 c2 = make_float2(c, c);
      const float2 nm2 = make_float2(-m_run, -m_run);
      float2 l2[4], r2[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) l2[q] = r2[q] = make_float2(0.f, 0.f);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const float2 x = ffma2(make_float2(s[64 * h + 2 * q], s[64 * h + 2 * q + 1]), c2, nm2);
          const float p0 = ex2_approx(x.x);
          const float p1 = ex2_approx(x.y);
          pk[q] = pack_bf16(p0, p1);
          l2[q & 3] = fadd2(l2[q & 3], make_float2(p0, p1));
          r2[q & 3] = fadd2(r2[q & 3], make_float2(__uint_as_float(pk[q] << 16), __uint_as_float(pk[q] & 0xFFFF0000u)));
        }
        tmem_st32(s_addr + 32 * h, pk);  // P over the first 64 columns of S
      }
      l_run = l_run * alpha + (((l2[0].x + l2[0].y) + (l2[1].x + l2[1].y)) + ((l2[2].x + l2[2].y) + (l2[3].x + l2[3].y)));
      r_run = r_run * alpha + (((r2[0].x + r2[0].y) + (r2[1].x + r2[1].y)) + ((r2[2].x + r2[2].y) + (r2[3].x + r2[3].y)));
      tmem_st_wait();
      // PV(k-1) of this tile is waited every block (phases in order; PV(k)
      // cannot complete before this warp's P(k) arrival): O may then be
      // rescaled before PV(k) runs
      const bool rescale = __any_sync(0xffffffffu, alpha != 1.f);
      if (k > 0) {
        ok = warp_wait(bar(LY::BAR_PV + t), (k - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (rescale) {
#pragma unroll 1
          for (int cc = 0; cc < DV / 32; ++cc) {
            float o[32];
            tmem_ld32(o_addr + 32 * cc, o);
            uint32_t w[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) w[q] = __float_as_uint(o[q] * alpha);
            tmem_st32(o_addr + 32 * cc, w);
          }
          tmem_st_wait();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(LY::BAR_P + t));
      ++k;
    }
    if (ok && k > 0) ok = warp_wait(bar(LY::BAR_PV + t), (k - 1) & 1, abort_flag);
    if (ok && k > 0) {
      tc_fence_after();
      const float inv = 1.f / r_run;
      const int64_t grow0 = (int64_t)seq_start + qb * kTile;
      const int n_valid = min(kTile, seq_len - qb * kTile);
      // each 8-lane group transposes its 8 rows x 8 chunks of 16 bytes so that
      // every store of the warp writes four whole 128-byte row segments
      const int j8 = lane & 7;
      const int r8 = quarter * 32 + (lane & ~7);  // first row of this lane's group
#pragma unroll 1
      for (int g = 0; g < DV / 64; ++g) {
        float o[32], o2[32];
        tmem_ld32(o_addr + 64 * g, o);
        tmem_ld32(o_addr + 64 * g + 32, o2);
        uint32_t w[32];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          w[q] = pack_bf16(o[2 * q] * inv, o[2 * q + 1] * inv);
          w[16 + q] = pack_bf16(o2[2 * q] * inv, o2[2 * q + 1] * inv);
        }
        transpose8x8_u4(w, lane);  // now chunk j8 of rows r8 .. r8 + 7
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          if (r8 + kk < n_valid) {
            __nv_bfloat16* dst = p.out + ((grow0 + r8 + kk) * p.n_heads + head) * (int64_t)p.d_v + 64 * g + 8 * j8;
            *reinterpret_cast<uint4*>(dst) = make_uint4(w[4 * kk], w[4 * kk + 1], w[4 * kk + 2], w[4 * kk + 3]);
          }
        }
      }
      if (row < n_valid) p.lse[(grow0 + row) * p.n_heads + head] = (m_run + log2f(l_run)) * 0.69314718055994530942f;
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
