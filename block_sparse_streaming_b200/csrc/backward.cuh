// backward.cuh - SSA training backward on sm_100a (tcgen05 + TMA).
//
// The model is mid-trained with SSA in place (page 1 section 01 "training" of
// the LoZA pages), so the operator needs dQ, dK, dV. With P = softmax over the
// selected keys (recomputed from the forward LSE), D_i = dO_i . O_i,
// dP = dO V^T, dS = P o (dP - D):
//     dQ = scale dS K,   dK = scale dS^T Q,   dV = P^T dO.
// Gradients are written by exactly one owner CTA per output tile (no atomics).
// Tiles are 128 tokens; the window (any power-of-two block size b) is applied
// per element where a tile is only partly visible:
//   ssa_bwd_dq_kernel     owner of a 128-query tile; walks the key tiles its
//                         window reads (S, dP, dQ += dS K).
//   ssa_bwd_dkdv_kernel   owner of a 128-key tile; walks the query tiles that
//                         see it through the local window: k .. (with b = 128,
//                         l tiles; bwd_local_end in general). A tile holding a
//                         sink key is also seen by every later query tile;
//                         those "far" query tiles are handled by extra CTAs in
//                         fixed chunks, and every contribution to such a tile
//                         goes to an fp32 partial in the workspace.
//   ssa_bwd_sink_reduce   adds a sink tile's partials in a fixed order
//                         (deterministic) and writes its dK, dV.
//   ssa_bwd_preprocess    D = rowsum(dO o O), bandwidth bound.
#pragma once

#include <cuda.h>

#include "prefill.cuh"
#include "sm100.cuh"

namespace loza {

constexpr int kBwdDkvThreads = 320;  // producer, MMA, 8 elementwise warps
constexpr int kSinkChunk = 256;  // far query blocks per sink-partial CTA

struct BwdParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;  // [T, H, d] maps, box {64, 1, 128}
  const int32_t* cu_seqlens;
  const float* lse;    // [T, H] natural log
  const float* dvec;   // [T, H] D = rowsum(dO o O)
  __nv_bfloat16* dq;   // [T, H, DQK]
  __nv_bfloat16* dk;   // [T, H, DQK]
  __nv_bfloat16* dv;   // [T, H, DV]
  float* partial;      // sink partials [B][s][H][nslots][128][DQK + DV]
  int n_heads;
  int n_sink, n_local;
  int block;           // b, tokens per block of the window (a power of two)
  int sink_end;        // s * b: keys below it are sinks
  int n_sink_tiles;    // 128-key tiles holding a sink key: ceil(s * b / 128)
  int nslots;          // partial slots per (sequence, sink tile, head)
  int far_mode;        // dK/dV kernel: 0 = owners, 1 = far sink chunks
  float scale;         // softmax scale
  float scale_log2;    // scale * log2(e)
};

// Query tiles [k, bwd_local_end(k)) see key tile k through the local part of
// the window: the last query that does is the last i with lo(i) <= 128k + 127,
// i.e. i < (floor((128k + 127) / b) + l) * b. Beyond it only sink keys are seen.
__host__ __device__ __forceinline__ int bwd_local_end(int k, int b, int n_local) {
  const int64_t i_end = ((int64_t)(k * kTile + kTile - 1) / b + n_local) * b;  // first query past the range
  return (int)((i_end - 1) / kTile + 1);
}

// Bits q = 0 .. 63 of the queries i0 + q that see key t: t <= i and (t is a
// sink or i < (floor(t / b) + l) * b).
__device__ __forceinline__ uint64_t bwd_key_mask(int64_t t, int64_t i0, int b, int sink_end, int n_local) {
  const int64_t lo = t - i0;
  const int64_t hi = t < sink_end ? 64 : ((t / b + n_local) * b - i0);
  auto below = [](int64_t x) -> uint64_t { return x <= 0 ? 0ull : (x >= 64 ? ~0ull : ((1ull << x) - 1ull)); };
  return below(hi) & ~below(lo);
}

// ---------------------------------------------------------------------------
// D = rowsum(dO o O) over DV columns; one half-warp per (token, head) row.
// ---------------------------------------------------------------------------
template <int DV>
__global__ void __launch_bounds__(256) ssa_bwd_preprocess(const __nv_bfloat16* __restrict__ out,
                                                          const __nv_bfloat16* __restrict__ dout,
                                                          float* __restrict__ dvec, int64_t rows) {
  constexpr int LANES = DV / 8;  // 16-byte vectors per row
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = gid / LANES;
  const int l = (int)(gid % LANES);
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = reinterpret_cast<const uint4*>(out + row * DV)[l];
    const uint4 b = reinterpret_cast<const uint4*>(dout + row * DV)[l];
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(pa[i]);
      const float2 y = __bfloat1622float2(pb[i]);
      acc += x.x * y.x + x.y * y.y;
    }
  }
#pragma unroll
  for (int o = LANES / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o, LANES);
  if (row < rows && l == 0) dvec[row] = acc;
}

// ---------------------------------------------------------------------------
// dQ: one CTA per (query tile, head, sequence).
// TMEM: S [0,128), dP [128,256), dQ [256, 256+DQK), dS (bf16, packed) [448,512).
// dS has columns of its own, so the MMAs of block b+1 (S, dP) are issued as
// soon as the elementwise warps have read S(b) and dP(b), and run while they
// compute dS(b); dQ(b) follows. Ring order: K(0) V(0), then per block b:
// K(b+1) V(b+1) (for S, dP) and K(b) again (for dQ), as the MMAs consume them.
// Warps: 0 TMA producer, 1 TMEM allocation + MMA issuer, 2-9 elementwise
// (two per TMEM lane quarter, 64 keys each).
// ---------------------------------------------------------------------------
constexpr int kBwdDqThreads = 320;

template <int DQK, int DV>
struct BwdDqLayout {
  static constexpr int NQC = DQK / 64, NVC = DV / 64, NSTAGE = 8;
  static constexpr int Q_OFF = 0;
  static constexpr int DO_OFF = NQC * kChunkBytes;
  static constexpr int RING_OFF = DO_OFF + NVC * kChunkBytes;
  static constexpr int BAR_OFF = RING_OFF + NSTAGE * kChunkBytes;
  static constexpr int BAR_IN = 0, BAR_FULL = 1, BAR_EMPTY = 1 + NSTAGE, BAR_DP = 1 + 2 * NSTAGE,
                       BAR_FREE = BAR_DP + 1, BAR_DS = BAR_FREE + 1, BAR_DQ = BAR_DS + 1, NBAR = BAR_DQ + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16;
  static constexpr int T_DS = 448;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(256 + DQK <= T_DS, "TMEM budget");
};

template <int DQK, int DV>
__global__ void __launch_bounds__(kBwdDqThreads, 1) ssa_bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  using LY = BwdDqLayout<DQK, DV>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(&g_device_status, kErrLayout);
    return;
  }
  const int qb = blockIdx.x, head = blockIdx.y, seq = blockIdx.z;
  const int seq_start = p.cu_seqlens[seq];
  const int seq_len = p.cu_seqlens[seq + 1] - seq_start;
  if (qb * kTile >= seq_len) return;
  const BlockWalk walk(qb, p.n_sink, p.n_local, p.block);
  const SsaWindow win{p.block, walk.sink_end, p.n_local};
  const int nb = walk.count;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + LY::BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar(LY::BAR_IN), 1);
    for (int i = 0; i < LY::NSTAGE; ++i) {
      mbar_init(bar(LY::BAR_FULL + i), 1);
      mbar_init(bar(LY::BAR_EMPTY + i), 1);
    }
    mbar_init(bar(LY::BAR_DP), 1);
    mbar_init(bar(LY::BAR_FREE), 8);  // one arrival per elementwise warp
    mbar_init(bar(LY::BAR_DS), 8);
    mbar_init(bar(LY::BAR_DQ), 1);
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
    if (lane == 0) {
      const int row0 = seq_start + qb * kTile;
      mbar_arrive_expect_tx(bar(LY::BAR_IN), (LY::NQC + LY::NVC) * kChunkBytes);
      for (int c = 0; c < LY::NQC; ++c)
        tma_load_3d(sbase + LY::Q_OFF + c * kChunkBytes, &p.tm_q, bar(LY::BAR_IN), c * 64, head, row0);
      for (int c = 0; c < LY::NVC; ++c)
        tma_load_3d(sbase + LY::DO_OFF + c * kChunkBytes, &p.tm_do, bar(LY::BAR_IN), c * 64, head, row0);
      int slot = 0;
      uint32_t phase = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* map, int col, int row) {
        ok = mbar_wait(bar(LY::BAR_EMPTY + slot), phase ^ 1, abort_flag);
        if (!ok) return;
        mbar_arrive_expect_tx(bar(LY::BAR_FULL + slot), kChunkBytes);
        tma_load_3d(sbase + LY::RING_OFF + slot * kChunkBytes, map, bar(LY::BAR_FULL + slot), col, head, row);
        if (++slot == LY::NSTAGE) { slot = 0; phase ^= 1; }
      };
      for (int b = 0; b <= nb && ok; ++b) {
        if (b < nb) {
          const int krow = seq_start + walk.block(b) * kTile;
          for (int c = 0; c < LY::NQC && ok; ++c) load(&p.tm_k, c * 64, krow);
          for (int c = 0; c < LY::NVC && ok; ++c) load(&p.tm_v, c * 64, krow);
        }
        if (b >= 1) {
          const int krow = seq_start + walk.block(b - 1) * kTile;
          for (int c = 0; c < LY::NQC && ok; ++c) load(&p.tm_k, c * 64, krow);
        }
      }
    }
  } else if (warp == 1) {
    // whole warp walks the schedule; one elected lane issues each tcgen05 instruction
    constexpr uint32_t idesc_ss = idesc_bf16(128, 128, false, false);
    constexpr uint32_t idesc_dq = idesc_bf16(128, 64, false, true);
    const uint32_t t_s = tmem, t_dp = tmem + 128, t_dq = tmem + 256, t_ds = tmem + LY::T_DS;
    int slot = 0;
    uint32_t phase = 0;
    bool ok = warp_wait(bar(LY::BAR_IN), 0, abort_flag);
    tc_fence_after();
    auto next_full = [&]() {
      ok = warp_wait(bar(LY::BAR_FULL + slot), phase, abort_flag);
      if (ok) tc_fence_after();
      return ok;
    };
    auto advance = [&]() {
      if (++slot == LY::NSTAGE) { slot = 0; phase ^= 1; }
    };
    // S = Q K^T and dP = dO V^T of the next block
    auto issue_s_dp = [&]() {
      for (int c = 0; c < LY::NQC && ok; ++c) {
        if (!next_full()) break;
        if (elect_one()) {
          const uint32_t a = sbase + LY::Q_OFF + c * kChunkBytes, bb = sbase + LY::RING_OFF + slot * kChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(t_s, sdesc_sw128(a + 32 * kk, 16, 1024), sdesc_sw128(bb + 32 * kk, 16, 1024), idesc_ss,
                   (c | kk) != 0);
          mma_commit(bar(LY::BAR_EMPTY + slot));
        }
        __syncwarp();
        advance();
      }
      for (int c = 0; c < LY::NVC && ok; ++c) {
        if (!next_full()) break;
        if (elect_one()) {
          const uint32_t a = sbase + LY::DO_OFF + c * kChunkBytes, bb = sbase + LY::RING_OFF + slot * kChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(t_dp, sdesc_sw128(a + 32 * kk, 16, 1024), sdesc_sw128(bb + 32 * kk, 16, 1024), idesc_ss,
                   (c | kk) != 0);
          mma_commit(bar(LY::BAR_EMPTY + slot));
        }
        __syncwarp();
        advance();
      }
      if (ok && elect_one()) mma_commit(bar(LY::BAR_DP));
      __syncwarp();
    };
    if (ok) issue_s_dp();
    for (int b = 0; b < nb && ok; ++b) {
      if (b + 1 < nb) {
        // S(b), dP(b) have been read: the next block's products may overwrite them
        ok = warp_wait(bar(LY::BAR_FREE), b & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_s_dp();
        if (!ok) break;
      }
      ok = warp_wait(bar(LY::BAR_DS), b & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      // dQ += dS K  (A = dS in TMEM, B = K tiles MN-major)
      for (int c = 0; c < LY::NQC && ok; ++c) {
        if (!next_full()) break;
        if (elect_one()) {
          const uint32_t bb = sbase + LY::RING_OFF + slot * kChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(t_dq + 64 * c, t_ds + 8 * kk, sdesc_sw128(bb + 2048 * kk, 8192, 1024), idesc_dq,
                   (b > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(LY::BAR_EMPTY + slot));
        }
        __syncwarp();
        advance();
      }
      if (!ok) break;
      if (elect_one()) mma_commit(bar(LY::BAR_DQ));
      __syncwarp();
    }
  } else {
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;  // keys [64*half, +64)
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const int qpos = qb * kTile + row;
    const bool valid = qpos < seq_len;
    const int64_t grow = (int64_t)seq_start + qpos;
    const float lse2 = valid ? p.lse[grow * p.n_heads + head] * 1.4426950408889634f : 0.f;
    const float dd = valid ? p.dvec[grow * p.n_heads + head] : 0.f;
    const float c2 = p.scale_log2;
    bool ok = true;
    for (int b = 0; b < nb && ok; ++b) {
      ok = warp_wait(bar(LY::BAR_DP), b & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      float s[64], dp[64];
      tmem_ld64x2(lane_addr + 64 * half, lane_addr + 128 + 64 * half, s, dp);
      // S(b) and dP(b) are in registers: the MMAs of the next block may start
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(LY::BAR_FREE));
      // keys of this tile the row does not see (the diagonal, and tiles at
      // the window's edges when b < 128): bit j for key 64 * half + j
      const int kb = walk.block(b);
      const uint64_t vis = walk.masked(kb, qb) ? RowMask(win, qpos, kb * kTile).bits64(64 * half) : ~0ull;
      uint32_t pk[2][16];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float ds2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float pr = ex2_approx(fmaf(s[2 * i + e], c2, -lse2));
          if (!((vis >> (2 * i + e)) & 1ull)) pr = 0.f;
          ds2[e] = pr * (dp[2 * i + e] - dd);
        }
        pk[i >> 4][i & 15] = pack_bf16(ds2[0], ds2[1]);
      }
      // dQ(b-1) has read dS(b-1) (phases waited in order)
      if (b > 0) {
        ok = warp_wait(bar(LY::BAR_DQ), (b - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st16(lane_addr + LY::T_DS + 32 * half, pk[0]);
      tmem_st16(lane_addr + LY::T_DS + 32 * half + 16, pk[1]);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(LY::BAR_DS));  // one arrival per warp
    }
    if (ok) ok = warp_wait(bar(LY::BAR_DQ), (nb - 1) & 1, abort_flag);
    if (ok) {
      tc_fence_after();
      const int64_t grow0 = (int64_t)seq_start + qb * kTile;
      const int n_valid = min(kTile, seq_len - qb * kTile);
      // dQ in 64-column groups g = half, half + 2, ...: each 8-lane group
      // transposes its 8 rows x 8 chunks of 16 bytes so that every store of
      // the warp writes four whole 128-byte row segments
      const int j8 = lane & 7;
      const int r8 = quarter * 32 + (lane & ~7);
#pragma unroll 1
      for (int g = half; g < DQK / 64; g += 2) {
        float o[32], o2[32];
        tmem_ld32(lane_addr + 256 + 64 * g, o);
        tmem_ld32(lane_addr + 256 + 64 * g + 32, o2);
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          w[i] = pack_bf16(o[2 * i] * p.scale, o[2 * i + 1] * p.scale);
          w[16 + i] = pack_bf16(o2[2 * i] * p.scale, o2[2 * i + 1] * p.scale);
        }
        transpose8x8_u4(w, lane);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (r8 + k < n_valid) {
            __nv_bfloat16* dst = p.dq + ((grow0 + r8 + k) * p.n_heads + head) * (int64_t)DQK + 64 * g + 8 * j8;
            *reinterpret_cast<uint4*>(dst) = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// dK / dV: one CTA per (key tile, head, sequence) in owner mode, or per
// (far chunk, sink tile x head, sequence) in far mode.
// TMEM: S^T [0,128) (P^T and later dS^T packed into [0,64)), dP^T [64,192),
//       dV [192, 192+DV), dK [192+DV, 192+DV+DQK).
// ---------------------------------------------------------------------------
template <int DQK, int DV>
struct BwdDkvLayout {
  static constexpr int NQC = DQK / 64, NVC = DV / 64;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = NQC * kChunkBytes;
  static constexpr int Q_OFF = V_OFF + NVC * kChunkBytes;       // [2 buffers][NQC] tiles
  static constexpr int DO_OFF = Q_OFF + 2 * NQC * kChunkBytes;
  static constexpr int STAT_OFF = DO_OFF + NVC * kChunkBytes;  // lse2[128], d[128]
  static constexpr int BAR_OFF = STAT_OFF + 2 * 128 * 4;
  // Q of query block j goes to buffer j & 1 and is released after dK(j); dO
  // is single-buffered and released after dV(j) and dP^T(j) have read it
  static constexpr int BAR_KV = 0, BAR_Q = 1 /* [2] */, BAR_QE = 3 /* [2] */, BAR_DO = 5, BAR_DOE = 6, BAR_S = 7,
                       BAR_P = 8, BAR_DP = 9, BAR_DS = 10, BAR_ROW = 11 /* [4] */, NBAR = 15;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static constexpr int T_DV = 192, T_DK = 192 + DV;
  static_assert(T_DK + DQK <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int DQK, int DV>
__global__ void __launch_bounds__(kBwdDkvThreads, 1) ssa_bwd_dkdv_kernel(const __grid_constant__ BwdParams p) {
  using LY = BwdDkvLayout<DQK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int seq = blockIdx.z;
  const int seq_start = p.cu_seqlens[seq];
  const int seq_len = p.cu_seqlens[seq + 1] - seq_start;
  const int nq = (seq_len + kTile - 1) / kTile;
  int kblk, head, j_lo, j_hi, slot = -1;
  if (!p.far_mode) {
    kblk = blockIdx.x;
    head = blockIdx.y;
    if (kblk >= nq) return;
    j_lo = kblk;
    j_hi = min(nq, bwd_local_end(kblk, p.block, p.n_local));
    if (kblk < p.n_sink_tiles) slot = 0;
  } else {
    kblk = blockIdx.y % p.n_sink_tiles;
    head = blockIdx.y / p.n_sink_tiles;
    if (kblk >= nq) return;  // no such sink tile: its partial slots are never read
    j_lo = bwd_local_end(kblk, p.block, p.n_local) + blockIdx.x * kSinkChunk;
    j_hi = min(nq, j_lo + kSinkChunk);
    slot = 1 + blockIdx.x;
  }
  const int nj = max(0, j_hi - j_lo);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // sink partial destination: [seq][kblk][head][slot][128][DQK+DV]
  float* part = nullptr;
  if (slot >= 0)
    part = p.partial + ((((int64_t)seq * p.n_sink_tiles + kblk) * p.n_heads + head) * p.nslots + slot) *
                           (int64_t)(kTile * (DQK + DV));
  if (nj == 0) {
    // empty far chunk: its partial contributes zero
    for (int i = threadIdx.x; i < kTile * (DQK + DV) / 4; i += blockDim.x)
      reinterpret_cast<float4*>(part)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }

  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + LY::BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 4);
  float* s_lse2 = reinterpret_cast<float*>(smem + LY::STAT_OFF);
  float* s_d = s_lse2 + 128;

  if (threadIdx.x == 0) {
    mbar_init(bar(LY::BAR_KV), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(LY::BAR_Q + i), 1);
      mbar_init(bar(LY::BAR_QE + i), 1);
    }
    mbar_init(bar(LY::BAR_DO), 1);
    mbar_init(bar(LY::BAR_DOE), 1);
    mbar_init(bar(LY::BAR_S), 1);
    mbar_init(bar(LY::BAR_P), 8);  // one arrival per elementwise warp
    mbar_init(bar(LY::BAR_DP), 1);
    mbar_init(bar(LY::BAR_DS), 8);
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
  const int krow = seq_start + kblk * kTile;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(LY::BAR_KV), (LY::NQC + LY::NVC) * kChunkBytes);
      for (int c = 0; c < LY::NQC; ++c)
        tma_load_3d(sbase + LY::K_OFF + c * kChunkBytes, &p.tm_k, bar(LY::BAR_KV), c * 64, head, krow);
      for (int c = 0; c < LY::NVC; ++c)
        tma_load_3d(sbase + LY::V_OFF + c * kChunkBytes, &p.tm_v, bar(LY::BAR_KV), c * 64, head, krow);
      bool ok = true;
      for (int jj = 0; jj < nj && ok; ++jj) {
        const int qrow = seq_start + (j_lo + jj) * kTile;
        const int qbuf = jj & 1;
        ok = mbar_wait(bar(LY::BAR_QE + qbuf), ((jj >> 1) & 1) ^ 1, abort_flag);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(LY::BAR_Q + qbuf), LY::NQC * kChunkBytes);
        for (int c = 0; c < LY::NQC; ++c)
          tma_load_3d(sbase + LY::Q_OFF + (qbuf * LY::NQC + c) * kChunkBytes, &p.tm_q, bar(LY::BAR_Q + qbuf), c * 64,
                      head, qrow);
        ok = mbar_wait(bar(LY::BAR_DOE), (jj & 1) ^ 1, abort_flag);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(LY::BAR_DO), LY::NVC * kChunkBytes);
        for (int c = 0; c < LY::NVC; ++c)
          tma_load_3d(sbase + LY::DO_OFF + c * kChunkBytes, &p.tm_do, bar(LY::BAR_DO), c * 64, head, qrow);
      }
    }
  } else if (warp == 1) {
    // whole warp walks the schedule; one elected lane issues each tcgen05 instruction
    constexpr uint32_t idesc_ss = idesc_bf16(128, 128, false, false);
    constexpr uint32_t idesc_ts = idesc_bf16(128, 64, false, true);
    const uint32_t t_s = tmem, t_dp = tmem + 64, t_dv = tmem + LY::T_DV, t_dk = tmem + LY::T_DK;
    bool ok = warp_wait(bar(LY::BAR_KV), 0, abort_flag);
    for (int jj = 0; jj < nj && ok; ++jj) {
      const int qbuf = jj & 1;
      const uint32_t q_off = sbase + LY::Q_OFF + qbuf * LY::NQC * kChunkBytes;
      ok = warp_wait(bar(LY::BAR_Q + qbuf), (jj >> 1) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      // S^T = K Q^T
      if (elect_one()) {
      for (int c = 0; c < LY::NQC; ++c) {
        const uint32_t a = sbase + LY::K_OFF + c * kChunkBytes, bb = q_off + c * kChunkBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(t_s, sdesc_sw128(a + 32 * kk, 16, 1024), sdesc_sw128(bb + 32 * kk, 16, 1024), idesc_ss,
                 (c | kk) != 0);
      }
      mma_commit(bar(LY::BAR_S));
      }
      __syncwarp();
      ok = warp_wait(bar(LY::BAR_P), jj & 1, abort_flag) && warp_wait(bar(LY::BAR_DO), jj & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      // dV += P^T dO   (A = P^T in TMEM, B = dO tiles MN-major)
      if (elect_one()) {
      for (int c = 0; c < LY::NVC; ++c) {
        const uint32_t bb = sbase + LY::DO_OFF + c * kChunkBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(t_dv + 64 * c, t_s + 8 * kk, sdesc_sw128(bb + 2048 * kk, 8192, 1024), idesc_ts,
                 (jj > 0 || kk > 0) ? 1u : 0u);
      }
      // dP^T = V dO^T
      for (int c = 0; c < LY::NVC; ++c) {
        const uint32_t a = sbase + LY::V_OFF + c * kChunkBytes, bb = sbase + LY::DO_OFF + c * kChunkBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(t_dp, sdesc_sw128(a + 32 * kk, 16, 1024), sdesc_sw128(bb + 32 * kk, 16, 1024), idesc_ss,
                 (c | kk) != 0);
      }
      mma_commit(bar(LY::BAR_DP));
      mma_commit(bar(LY::BAR_DOE));  // dO read by dV and dP^T
      }
      __syncwarp();
      ok = warp_wait(bar(LY::BAR_DS), jj & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      // dK += dS^T Q   (A = dS^T in TMEM, B = Q tiles MN-major)
      if (elect_one()) {
      for (int c = 0; c < LY::NQC; ++c) {
        const uint32_t bb = q_off + c * kChunkBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(t_dk + 64 * c, t_s + 8 * kk, sdesc_sw128(bb + 2048 * kk, 8192, 1024), idesc_ts,
                 (jj > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(bar(LY::BAR_QE + qbuf));  // Q(j) no longer read
      }
      __syncwarp();
    }
  } else {
    // elementwise: two warps per TMEM lane quarter, warp half h takes the
    // queries [64h, 64h+64) of every key row
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int tid = threadIdx.x - 64;     // 0..255
    const int key = quarter * 32 + lane;  // TMEM lane == key row of the block
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    bool ok = true;
    for (int jj = 0; jj < nj && ok; ++jj) {
      const int j = j_lo + jj;
      if (tid < 128) {
        // per-query statistics of block j (invalid rows: P = 0, D = 0)
        const int qpos = j * kTile + tid;
        const bool v = qpos < seq_len;
        const int64_t g = (int64_t)seq_start + qpos;
        s_lse2[tid] = v ? p.lse[g * p.n_heads + head] * 1.4426950408889634f : INFINITY;
        s_d[tid] = v ? p.dvec[g * p.n_heads + head] : 0.f;
      }
      named_barrier_sync(1, 256);
      ok = warp_wait(bar(LY::BAR_S), jj & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      // queries of block j that see this row's key (causality, and the
      // window's end for a key that is not a sink): bit q for query 64 * half + q
      const uint64_t vis = bwd_key_mask((int64_t)kblk * kTile + key, (int64_t)j * kTile + 64 * half, p.block,
                                        p.sink_end, p.n_local);
      float pr[64];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float sx[32];
        tmem_ld32(lane_addr + 64 * half + 32 * c, sx);
        const float4* l4 = reinterpret_cast<const float4*>(s_lse2 + 64 * half + 32 * c);
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 l = l4[i4];
          const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 32 * c + 4 * i4 + e;
            float v = ex2_approx(fmaf(sx[4 * i4 + e], p.scale_log2, -lv[e]));
            if (!((vis >> i) & 1ull)) v = 0.f;
            pr[i] = v;
          }
        }
      }
      // P^T is stored over S^T columns holding queries of both warps of the
      // row: neither stores before its partner has loaded S^T
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(LY::BAR_ROW + quarter));
      ok = warp_wait(bar(LY::BAR_ROW + quarter), jj & 1, abort_flag);
      if (!ok) break;
      {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16(pr[2 * i], pr[2 * i + 1]);
        tmem_st32(lane_addr + 32 * half, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(LY::BAR_P));  // one arrival per warp
      ok = warp_wait(bar(LY::BAR_DP), jj & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float dx[32];
        tmem_ld32(lane_addr + 64 + 64 * half + 32 * c, dx);
        const float4* d4 = reinterpret_cast<const float4*>(s_d + 64 * half + 32 * c);
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 d = d4[i4];
          const float dv4[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) pr[32 * c + 4 * i4 + e] *= dx[4 * i4 + e] - dv4[e];
        }
      }
      {
        // dS^T over this warp's own P^T columns (dV and dP^T have read P^T)
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16(pr[2 * i], pr[2 * i + 1]);
        tmem_st32(lane_addr + 32 * half, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(LY::BAR_DS));  // one arrival per warp
      named_barrier_sync(1, 256);  // statistics of block j no longer read
    }
    if (ok) ok = warp_wait(bar(LY::BAR_QE + ((nj - 1) & 1)), ((nj - 1) >> 1) & 1, abort_flag);  // last dK done
    if (ok) {
      tc_fence_after();
      const int64_t g0 = (int64_t)seq_start + kblk * kTile;
      const int n_valid = min(kTile, seq_len - kblk * kTile);
      if (part) {
        // fp32 partials, row `key`: dK columns [0, DQK), dV columns [DQK, DQK+DV);
        // this warp takes the 32-column units u = half, half + 2, ...
        float* prow = part + (int64_t)key * (DQK + DV);
#pragma unroll 1
        for (int u = half; u < (DQK + DV) / 32; u += 2) {
          float o[32];
          const bool is_k = u < DQK / 32;
          tmem_ld32(lane_addr + (is_k ? LY::T_DK + 32 * u : LY::T_DV + 32 * u - DQK), o);
          const float sc = is_k ? p.scale : 1.f;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(prow + 32 * u + i) =
                make_float4(o[i] * sc, o[i + 1] * sc, o[i + 2] * sc, o[i + 3] * sc);
        }
      } else {
        // bf16 dK, dV in 64-column groups (dK groups, then dV groups; this warp
        // takes g = half, half + 2, ...): each 8-lane group transposes its 8
        // rows x 8 chunks of 16 bytes so every store writes whole 128-byte segments
        const int j8 = lane & 7;
        const int r8 = quarter * 32 + (lane & ~7);
#pragma unroll 1
        for (int gi = half; gi < (DQK + DV) / 64; gi += 2) {
          const bool is_k = gi < DQK / 64;
          const int g = is_k ? gi : gi - DQK / 64;
          const uint32_t col = is_k ? LY::T_DK + 64 * g : LY::T_DV + 64 * g;
          const float sc = is_k ? p.scale : 1.f;
          float o[32], o2[32];
          tmem_ld32(lane_addr + col, o);
          tmem_ld32(lane_addr + col + 32, o2);
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            w[i] = pack_bf16(o[2 * i] * sc, o[2 * i + 1] * sc);
            w[16 + i] = pack_bf16(o2[2 * i] * sc, o2[2 * i + 1] * sc);
          }
          transpose8x8_u4(w, lane);
          __nv_bfloat16* base = is_k ? p.dk : p.dv;
          const int width = is_k ? DQK : DV;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if (r8 + k < n_valid) {
              __nv_bfloat16* dst = base + ((g0 + r8 + k) * p.n_heads + head) * (int64_t)width + 64 * g + 8 * j8;
              *reinterpret_cast<uint4*>(dst) = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Sink tiles (the 128-key tiles holding a sink key): dK, dV = sum of the
// partial slots, in slot order. grid (128 key rows, sink tiles * H, B);
// thread = column of [DQK | DV].
// ---------------------------------------------------------------------------
template <int DQK, int DV>
__global__ void __launch_bounds__(DQK + DV) ssa_bwd_sink_reduce(const BwdParams p) {
  const int key = blockIdx.x;
  const int kblk = blockIdx.y % p.n_sink_tiles, head = blockIdx.y / p.n_sink_tiles, seq = blockIdx.z;
  const int seq_start = p.cu_seqlens[seq];
  const int seq_len = p.cu_seqlens[seq + 1] - seq_start;
  const int nq = (seq_len + kTile - 1) / kTile;
  const int kpos = kblk * kTile + key;
  if (kblk >= nq || kpos >= seq_len) return;
  const int col = threadIdx.x;
  // slots that received work: 0 (local) and the far chunks that start inside the sequence
  const int far = max(0, nq - bwd_local_end(kblk, p.block, p.n_local));
  const int used = min(p.nslots, 1 + (far + kSinkChunk - 1) / kSinkChunk);
  const float* base = p.partial + (((int64_t)seq * p.n_sink_tiles + kblk) * p.n_heads + head) * p.nslots *
                                      (int64_t)(kTile * (DQK + DV));
  float acc = 0.f;
  for (int s = 0; s < used; ++s) acc += base[(int64_t)s * kTile * (DQK + DV) + (int64_t)key * (DQK + DV) + col];
  const int64_t g = (int64_t)seq_start + kpos;
  if (col < DQK)
    p.dk[(g * p.n_heads + head) * DQK + col] = __float2bfloat16_rn(acc);
  else
    p.dv[(g * p.n_heads + head) * DV + (col - DQK)] = __float2bfloat16_rn(acc);
}

}  // namespace loza
