// prefill.cuh - SSA prefill / training forward on sm_100a (tcgen05 + TMA).
//
// One CTA computes a 128-query tile (128 consecutive tokens of one sequence,
// one head) against the key blocks the window selects, for one slice of the
// value dimension:
//   key blocks of query block j:  sink blocks 0 .. min(s, j+1)-1, then local
//   blocks max(s, j-l+1) .. j (page 1 section 01 (1)-(2) of the LoZA pages:
//   sink + local blocks of b = 128 tokens, s = 1, l = 7), diagonal block last;
//   token-causal inside block j.
//
// Pipeline (warp-specialised, 6 warps):
//   warp 0      TMA producer: Q tile once, then K chunks / V chunks of every
//               selected block into a ring of 16 KB [128 x 64] bf16 tiles
//               (128-byte swizzle), in exactly the order the MMA consumes them.
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer:
//                 S_b  = Q K_b^T      (A = Q smem, B = K smem, both K-major)
//                 O   += P_b V_b      (A = P in TMEM, B = V smem, MN-major)
//               S is double-buffered in TMEM so S_{b+1} runs while the
//               softmax works on S_b; P_b overwrites the first half of S_b.
//   warps 2..9  softmax / correction / epilogue, two warps per TMEM lane
//               quarter (one query row per lane): warp half h computes the
//               exponentials of keys [64h, 64h+64) and rescales / writes half of
//               the O columns; both read the whole row of S for the maximum, so
//               only the row sums are combined (once, at the end). Online
//               softmax in base 2; O is rescaled in TMEM only when the running
//               max grows by more than 2^8 (otherwise the stale max is kept,
//               which is exact).
//
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+DVT).
// The value dimension is split into slices of DVT <= 256 columns so that O
// fits next to the two S buffers; the d_v = 512 (absorbed MLA) case runs two
// slices, each recomputing S.
#pragma once

#include <cuda.h>

#include "sm100.cuh"

namespace loza {

struct PrefillParams {
  CUtensorMap tm_q;   // [T, H, DQK]   box {64, 1, 128}
  CUtensorMap tm_k;   // [T, Hkv, DQK] box {64, 1, 128}
  CUtensorMap tm_v;   // [T, Hkv, DV]  box {64, 1, 128}
  const int32_t* cu_seqlens;
  __nv_bfloat16* out;  // [T, H, DV]
  float* lse;          // [T, H]
  int n_heads;
  int n_kv_heads;
  int d_v;             // full value width (row length of out)
  int dv_slices;       // d_v / DVT
  int n_sink;          // already 0 for the unbounded window
  int n_local;         // < 0: unbounded (full causal)
  int block;           // b, tokens per block of the window
  float scale_log2;    // scale * log2(e)
};

constexpr int kTile = 128;               // queries per tile == keys per block
constexpr int kChunkBytes = 128 * 64 * 2;  // one [128 x 64] bf16 tile
constexpr int kPrefillThreads = 320;
constexpr uint32_t kRescaleThreshold = 8;  // log2 units

template <int DQK, int DVT, int NSTAGE>
struct PrefillLayout {
  static constexpr int NQC = DQK / 64;
  static constexpr int NVC = DVT / 64;
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = NQC * kChunkBytes;
  static constexpr int XCH_OFF = RING_OFF + NSTAGE * kChunkBytes;  // [2][2][128] f32 row sums
  static constexpr int BAR_OFF = XCH_OFF + 2 * 2 * 128 * 4;
  // barriers: q_full, ring_full[NSTAGE], ring_empty[NSTAGE], s_full[2], p_full[2], pv_done,
  // row[4] (the two softmax warps of a lane quarter)
  // (P-ready alternates between two barriers by block parity: a warp that has
  // already finished block b+1 must not count towards block b)
  static constexpr int BAR_Q = 0;
  static constexpr int BAR_FULL = 1;
  static constexpr int BAR_EMPTY = 1 + NSTAGE;
  static constexpr int BAR_S = 1 + 2 * NSTAGE;
  static constexpr int BAR_P = BAR_S + 2;
  static constexpr int BAR_PV = BAR_P + 2;
  static constexpr int BAR_ROW = BAR_PV + 1;
  static constexpr int NBAR = BAR_ROW + 4;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem base (u32), abort (int)
  static constexpr int SMEM_BYTES = MISC_OFF + 16;
  static_assert(DQK % 64 == 0 && DVT % 64 == 0 && DVT <= 256, "tile shape");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// The keys query position i sees (LoZA page 1 section 01 (1): the sink
// blocks and the l most recent blocks of b tokens, token-causal):
//   A(i) = {t <= i : t < sink_end or t >= lo(i)},  sink_end = s * b,
//   lo(i) = max(0, (floor(i / b) - l + 1) * b)   (l < 0: unbounded, lo = 0).
// b = 128, s = 1, l = 7 is the pages' configuration; b = 1 makes every token
// a block, which is page 4's fixed part of the streaming-aware index (s = 16
// sink tokens and an l = 1,024-token sliding window).
struct SsaWindow {
  int b, sink_end, n_local;
  __host__ __device__ __forceinline__ int lo(int i) const {
    return n_local < 0 ? 0 : max(0, (i / b - n_local + 1) * b);
  }
};

// Key tiles (kTile = 128 keys) that query tile qb reads, sinks first, then
// the local tiles in order (the diagonal last), each tile once. A tile needs
// the per-row mask (visible(i, t) of SsaWindow) if it is the diagonal or if
// some of its keys are neither sinks for every row nor inside every row's
// local range; with b = 128 only the diagonal does.
struct BlockWalk {
  int sinks, local_lo, count;
  int sink_end, lo_last;  // lo() of the tile's last row
  __host__ __device__ __forceinline__ BlockWalk(int qb, int n_sink, int n_local, int b = kTile) {
    const SsaWindow w{b, n_sink * b, n_local};
    sink_end = w.sink_end;
    sinks = min((sink_end + kTile - 1) / kTile, qb + 1);
    local_lo = max(sinks, w.lo(qb * kTile) / kTile);
    lo_last = w.lo(qb * kTile + kTile - 1);
    count = sinks + max(0, qb - local_lo + 1);
  }
  __host__ __device__ __forceinline__ int block(int it) const { return it < sinks ? it : local_lo + (it - sinks); }
  __host__ __device__ __forceinline__ bool masked(int kb, int qb) const {
    return kb == qb || !(kb * kTile + kTile <= sink_end || kb * kTile >= lo_last);
  }
};

// Whether key t (relative to the tile start `base`, as j = t - base) is
// visible from query position i: j <= i - base and (j < sink_end - base or
// j >= lo(i) - base). The three bounds are per row; the test is per key.
struct RowMask {
  int a, e, f;
  __device__ __forceinline__ RowMask(const SsaWindow& w, int i, int base)
      : a(i - base), e(w.sink_end - base), f(w.lo(i) - base) {}
  __device__ __forceinline__ bool visible(int j) const { return j <= a && (j < e || j >= f); }
  // bit j of the result: visible(j0 + j), for j = 0 .. 63
  __device__ __forceinline__ uint64_t bits64(int j0) const {
    auto below = [](int x) -> uint64_t {  // bits j with j < x
      return x <= 0 ? 0ull : (x >= 64 ? ~0ull : ((1ull << x) - 1ull));
    };
    return below(a - j0 + 1) & (below(e - j0) | ~below(f - j0));
  }
};

// The units (of `unit` keys) that a single query position i reads, sinks
// first, then the local range in order, each unit once; each holds at least
// one visible key. Used by the decode kernels.
struct RowWalk {
  int sinks, local_lo, count;
  __host__ __device__ __forceinline__ RowWalk(const SsaWindow& w, int i, int unit) {
    const int last = i / unit;
    sinks = min((w.sink_end + unit - 1) / unit, last + 1);
    local_lo = max(sinks, w.lo(i) / unit);
    count = sinks + max(0, last - local_lo + 1);
  }
  __host__ __device__ __forceinline__ int unit_at(int it) const { return it < sinks ? it : local_lo + (it - sinks); }
};

template <int DQK, int DVT, int NSTAGE>
__global__ void __launch_bounds__(kPrefillThreads, 1)
ssa_prefill_kernel(const __grid_constant__ PrefillParams p) {
  using LY = PrefillLayout<DQK, DVT, NSTAGE>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(&g_device_status, kErrLayout);
    return;
  }

  const int qb = blockIdx.x;
  const int head = blockIdx.y / p.dv_slices;
  const int slice = blockIdx.y % p.dv_slices;
  const int seq = blockIdx.z;
  const int seq_start = p.cu_seqlens[seq];
  const int seq_len = p.cu_seqlens[seq + 1] - seq_start;
  if (qb * kTile >= seq_len) return;  // whole CTA leaves before any setup
  const int hk = head / (p.n_heads / p.n_kv_heads);
  const BlockWalk walk(qb, p.n_sink, p.n_local, p.block);
  const SsaWindow win{p.block, walk.sink_end, p.n_local};
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
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(bar(LY::BAR_FULL + i), 1);
      mbar_init(bar(LY::BAR_EMPTY + i), 1);
    }
    mbar_init(bar(LY::BAR_S + 0), 1);
    mbar_init(bar(LY::BAR_S + 1), 1);
    mbar_init(bar(LY::BAR_P + 0), 8);  // one arrival per softmax warp
    mbar_init(bar(LY::BAR_P + 1), 8);
    mbar_init(bar(LY::BAR_PV), 1);
    for (int i = 0; i < 4; ++i) mbar_init(bar(LY::BAR_ROW + i), 2);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // whole warp walks the schedule; one elected lane issues the TMA loads
    if (elect_one()) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      const int row0 = seq_start + qb * kTile;
      mbar_arrive_expect_tx(bar(LY::BAR_Q), LY::NQC * kChunkBytes);
      for (int c = 0; c < LY::NQC; ++c)
        tma_load_3d(sbase + LY::Q_OFF + c * kChunkBytes, &p.tm_q, bar(LY::BAR_Q), c * 64, head, row0);
    }
    __syncwarp();
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    auto load_tile = [&](const CUtensorMap* map, int col, int row) {
      ok = warp_wait(bar(LY::BAR_EMPTY + slot), phase ^ 1, abort_flag);
      if (!ok) return;
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(LY::BAR_FULL + slot), kChunkBytes);
        tma_load_3d(sbase + LY::RING_OFF + slot * kChunkBytes, map, bar(LY::BAR_FULL + slot), col, hk, row);
      }
      __syncwarp();
      if (++slot == NSTAGE) { slot = 0; phase ^= 1; }
    };
    for (int it = 0; it <= nb && ok; ++it) {
      if (it < nb) {
        const int krow = seq_start + walk.block(it) * kTile;
        for (int c = 0; c < LY::NQC && ok; ++c) load_tile(&p.tm_k, c * 64, krow);
      }
      if (it >= 1) {
        const int vrow = seq_start + walk.block(it - 1) * kTile;
        for (int c = 0; c < LY::NVC && ok; ++c) load_tile(&p.tm_v, slice * DVT + c * 64, vrow);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the schedule (warp-uniform descriptors); one
    // elected lane issues each tcgen05 instruction.
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16(128, 64, false, true);
    const uint32_t tmem_o = tmem + 256;
    const uint64_t dq0 = sdesc_sw128(sbase + LY::Q_OFF, 16, 1024);       // Q tile 0 (K-major)
    const uint64_t dk0 = sdesc_sw128(sbase + LY::RING_OFF, 16, 1024);    // ring slot 0 read K-major
    const uint64_t dv0 = sdesc_sw128(sbase + LY::RING_OFF, 8192, 1024);  // ring slot 0 read MN-major
    int slot = 0;
    uint32_t phase = 0;
    bool ok = warp_wait(bar(LY::BAR_Q), 0, abort_flag);
    tc_fence_after();
    for (int it = 0; it <= nb && ok; ++it) {
      if (it < nb) {
        const uint32_t tmem_s = tmem + (it & 1) * 128;
        for (int c = 0; c < LY::NQC; ++c) {
          ok = warp_wait(bar(LY::BAR_FULL + slot), phase, abort_flag);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            const uint64_t da = desc_add(dq0, c * kChunkBytes);
            const uint64_t db = desc_add(dk0, slot * kChunkBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem_s, desc_add(da, 32 * kk), desc_add(db, 32 * kk), idesc_s, (c | kk) != 0);
            mma_commit(bar(LY::BAR_EMPTY + slot));
          }
          __syncwarp();
          if (++slot == NSTAGE) { slot = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (elect_one()) mma_commit(bar(LY::BAR_S + (it & 1)));
        __syncwarp();
      }
      if (it >= 1) {
        const int b = it - 1;
        ok = warp_wait(bar(LY::BAR_P + (b & 1)), (b >> 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tmem_p = tmem + (b & 1) * 128;
        for (int c = 0; c < LY::NVC; ++c) {
          ok = warp_wait(bar(LY::BAR_FULL + slot), phase, abort_flag);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            const uint64_t dv = desc_add(dv0, slot * kChunkBytes);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem_o + c * 64, tmem_p + kk * 8, desc_add(dv, 2048 * kk), idesc_pv, (b > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar(LY::BAR_EMPTY + slot));
          }
          __syncwarp();
          if (++slot == NSTAGE) { slot = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (elect_one()) mma_commit(bar(LY::BAR_PV));
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;                  // keys [64*half, +64) of every block
    const int row = quarter * 32 + lane;               // row of the tile == TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const int qpos = qb * kTile + row;                  // position inside the sequence
    float* xl = reinterpret_cast<float*>(smem + LY::XCH_OFF);  // [2][128] exact row sums
    float* xr = xl + 256;                                       // [2][128] sums of bf16 P
    // m_run: running row maximum of scale*log2(e)*s (the reference of P);
    // l_run: this warp's share of the running sum of 2^(x - m_run) (exact, for the LSE);
    // r_run: its share of the running sum of the bf16-rounded P values that enter
    //        P.V, so that O is normalised by exactly the weights it was accumulated with.
    float m_run = -INFINITY, l_run = 0.f, r_run = 0.f;
    const float c = p.scale_log2;  // > 0, so max(c*s) = c*max(s)
    bool ok = true;
    for (int b = 0; b < nb && ok; ++b) {
      ok = warp_wait(bar(LY::BAR_S + (b & 1)), (b >> 1) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_addr = lane_addr + (b & 1) * 128;
      float so[64], s[64];  // the other warp's keys (maximum only) and this warp's keys
      tmem_ld64x2(s_addr + 64 * (half ^ 1), s_addr + 64 * half, so, s);
      // P is stored over S columns holding keys of both warps of the row:
      // neither stores before its partner warp has loaded S
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(LY::BAR_ROW + quarter));
      ok = warp_wait(bar(LY::BAR_ROW + quarter), b & 1, abort_flag);
      if (!ok) break;
      // keys this row does not see: after its query (the diagonal tile), or
      // between the sinks and its local range (tiles at the window's edges)
      if (walk.masked(walk.block(b), qb)) {
        const RowMask rm(win, qpos, walk.block(b) * kTile);
        const uint64_t vo = rm.bits64(64 * (half ^ 1)), vs = rm.bits64(64 * half);
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          if (!((vo >> j) & 1ull)) so[j] = -INFINITY;
          if (!((vs >> j) & 1ull)) s[j] = -INFINITY;
        }
      }
      float mx;
      {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < 32; ++j) m4[j & 3] = fmax3(m4[j & 3], so[2 * j], so[2 * j + 1]);
#pragma unroll
        for (int j = 0; j < 32; ++j) m4[j & 3] = fmax3(m4[j & 3], s[2 * j], s[2 * j + 1]);
        mx = c * fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      }
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
      tmem_st32(s_addr + 32 * half, pk);  // P over the first 64 columns of S
      l_run = l_run * alpha + (((l2[0].x + l2[0].y) + (l2[1].x + l2[1].y)) + ((l2[2].x + l2[2].y) + (l2[3].x + l2[3].y)));
      r_run = r_run * alpha + (((r2[0].x + r2[0].y) + (r2[1].x + r2[1].y)) + ((r2[2].x + r2[2].y) + (r2[3].x + r2[3].y)));
      tmem_st_wait();
      // PV(b-1) is waited every block, after the exponentials (by then it has
      // normally finished): O may then be rescaled before PV(b) runs. The
      // waits are taken in order and PV(b) cannot complete before this warp's
      // P(b) arrival, so each parity wait is exact.
      const bool rescale = __any_sync(0xffffffffu, alpha != 1.f);
      if (b > 0) {
        ok = warp_wait(bar(LY::BAR_PV), (b - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (rescale) {
          // this warp's 32-column units of O: u = half, half + 2, ...
#pragma unroll 1
          for (int cc = half; cc < DVT / 32; cc += 2) {
            float o[32];
            tmem_ld32(lane_addr + 256 + 32 * cc, o);
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(o[i] * alpha);
            tmem_st32(lane_addr + 256 + 32 * cc, w);
          }
          tmem_st_wait();
        }
      }
      // one arrival per warp: every lane's TMEM stores have completed
      // (tcgen05.wait::st) and are ordered before lane 0's release-arrive
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(LY::BAR_P + (b & 1)));
    }
    if (ok) ok = warp_wait(bar(LY::BAR_PV), (nb - 1) & 1, abort_flag);
    if (ok) {
      xl[half * 128 + row] = l_run;
      xr[half * 128 + row] = r_run;
    }
    named_barrier_sync(1, 256);
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / (xr[row] + xr[128 + row]);
      const int64_t grow0 = (int64_t)seq_start + qb * kTile;
      const int n_valid = min(kTile, seq_len - qb * kTile);
      // O in 64-column groups g = half, half + 2, ...: each 8-lane group
      // transposes its 8 rows x 8 chunks of 16 bytes so that every store of
      // the warp writes four whole 128-byte row segments
      const int j8 = lane & 7;
      const int r8 = quarter * 32 + (lane & ~7);  // first row of this lane's group
#pragma unroll 1
      for (int g = half; g < DVT / 64; g += 2) {
        float o[32], o2[32];
        tmem_ld32(lane_addr + 256 + 64 * g, o);
        tmem_ld32(lane_addr + 256 + 64 * g + 32, o2);
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
            __nv_bfloat16* dst = p.out + ((grow0 + r8 + k) * p.n_heads + head) * (int64_t)p.d_v + slice * DVT +
                                 64 * g + 8 * j8;
            *reinterpret_cast<uint4*>(dst) = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
          }
        }
      }
      if (half == 0 && qpos < seq_len && slice == 0)
        p.lse[(grow0 + row) * p.n_heads + head] = (m_run + log2f(xl[row] + xl[128 + row])) * 0.69314718055994530942f;
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
