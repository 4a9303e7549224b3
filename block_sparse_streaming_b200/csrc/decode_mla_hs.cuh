// decode_mla_hs.cuh - absorbed-MLA SSA decode, heads split between CTAs.
//
// Same operation as ssa_decode_mla_kernel (one query token per sequence at
// position i = L-1 against the blocks its window selects; page 1 section 01
// of the LoZA pages, section 02 for decode), with another division of the
// work: each sequence gets 64 / kHsHeads CTAs, one per group of kHsHeads query
// heads, and every CTA walks all of the sequence's selected blocks. A CTA
// therefore owns complete output rows and writes them directly: there is no
// merge of partial results. The CTAs of a sequence read the same latent rows
// at the same time, so DRAM sees each row about once (the others hit L2); what
// grows is the traffic from L2 into each SM.
//
//     S^T [128 keys x 32] = K_blk [128 x 576] . Q_g^T        (K-major A and B)
//     O^T [512 x 32]     += V_blk^T [512 x 128] . P^T         (MN-major A and B)
//
// The query's own block is processed first. Streaming as in
// ssa_decode_mla_kernel: a 5-unit TMA ring (unit = 128 rows x
// 128 latent columns, 32 KB) in the order K(0) K(1) V(0) K(2) V(1) ..., V units
// being the first 512 columns of the same rows (re-read from L2). One
// producer warp, one MMA warp, four softmax warps (one per TMEM lane quarter,
// 32 keys x 32 heads each).
#pragma once

#include <cuda.h>

#include "decode_mla.cuh"
#include "sm100.cuh"

namespace loza {

constexpr int kHsHeads = 32;                 // query heads per CTA (N of the MMAs)
constexpr int kHsThreads = 192;              // producer, MMA, 4 softmax warps
constexpr int kHsQTile = kHsHeads * 64 * 2;  // [32 heads x 64 dims] bf16
constexpr int kHsStages = 5;

struct DecodeHsLayout {
  static constexpr int Q_OFF = 0;                                 // 9 Q tiles, 36 KB
  static constexpr int RING_OFF = 9 * kHsQTile;                   // 36864 (1024-aligned)
  static constexpr int P_OFF = RING_OFF + kHsStages * kDecUnit;   // P^T: [128 keys] x 128-byte rows (32 heads used)
  static constexpr int RED_OFF = P_OFF + kChunkBytes;             // redmax, redsum, redrsum [4][32] each
  static constexpr int STAT_OFF = RED_OFF + 3 * 4 * kHsHeads * 4;  // m_run, l_run, alpha, r_run [32] each
  static constexpr int BAR_OFF = STAT_OFF + 4 * kHsHeads * 4;
  // barriers: q_full, full[5], empty[5], s_full[2], p_ready, pv_done, vtail
  static constexpr int BAR_Q = 0, BAR_FULL = 1, BAR_EMPTY = 1 + kHsStages, BAR_S = 1 + 2 * kHsStages,
                       BAR_P = BAR_S + 2, BAR_PV = BAR_P + 1, BAR_VT = BAR_PV + 1, NBAR = BAR_VT + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem base, abort flag, rescale flag
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(RING_OFF % 1024 == 0 && P_OFF % 1024 == 0, "swizzled tiles need 1024-byte alignment");
};

// Ring position (in units) of V unit u of block b (of nb): the K units of
// blocks 0 .. min(b+1, nb-1) and the V units of blocks 0 .. b-1 precede it.
__device__ __forceinline__ int hs_v_pos(int b, int u, int nb) {
  return kDecKUnits * min(b + 2, nb) + kDecVUnits * b + u;
}

// Grid: (64 / kHsHeads, batch). p.tm_q has a box of kHsHeads heads.
__global__ void __launch_bounds__(kHsThreads, 1) ssa_decode_mla_hs_kernel(const __grid_constant__ DecodeParams p) {
  using LY = DecodeHsLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int head0 = blockIdx.x * kHsHeads;
  const int seq = blockIdx.y;
  const int L = p.seqlens[seq];
  const int i_q = L - 1;       // decode query position
  const int jq = i_q / kTile;  // its block
  const BlockWalk walk(jq, p.n_sink, p.n_local);
  const int nb = walk.count;   // >= 1: the query's own block is always selected
  // processing order: the query's own block first (its rows past the end are
  // zeroed once its V units arrive, early in the stream), then the walk's others
  auto blk = [&](int b) { return walk.block(b == 0 ? nb - 1 : b - 1); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + LY::BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 4);
  volatile int* rescale_flag = reinterpret_cast<volatile int*>(smem + LY::MISC_OFF + 8);
  float* redmax = reinterpret_cast<float*>(smem + LY::RED_OFF);  // [4 quarters][32]
  float* redsum = redmax + 4 * kHsHeads;   // sums of exact P (for the LSE)
  float* redrsum = redsum + 4 * kHsHeads;  // sums of bf16-rounded P (for normalising O)
  float* m_run = reinterpret_cast<float*>(smem + LY::STAT_OFF);
  float* l_run = m_run + kHsHeads;
  float* alpha = m_run + 2 * kHsHeads;
  float* r_run = m_run + 3 * kHsHeads;

  if (threadIdx.x == 0) {
    mbar_init(bar(LY::BAR_Q), 1);
    for (int i = 0; i < kHsStages; ++i) {
      mbar_init(bar(LY::BAR_FULL + i), 1);
      mbar_init(bar(LY::BAR_EMPTY + i), 1);
    }
    mbar_init(bar(LY::BAR_S + 0), 1);
    mbar_init(bar(LY::BAR_S + 1), 1);
    mbar_init(bar(LY::BAR_P), 4);  // one arrival per softmax warp
    mbar_init(bar(LY::BAR_PV), 1);
    mbar_init(bar(LY::BAR_VT), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < kHsHeads) {
    m_run[threadIdx.x] = -INFINITY;
    l_run[threadIdx.x] = 0.f;
    r_run[threadIdx.x] = 0.f;
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S^T double buffer at 0 and 32; O^T unit u at 64 + 32u
  const uint32_t tmem_o = tmem + 2 * kHsHeads;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_kv);
      mbar_arrive_expect_tx(bar(LY::BAR_Q), 9 * kHsQTile);
      for (int c = 0; c < 9; ++c)
        tma_load_3d(sbase + LY::Q_OFF + c * kHsQTile, &p.tm_q, bar(LY::BAR_Q), c * 64, head0, seq);
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
      if (++slot == kHsStages) { slot = 0; phase ^= 1; }
    };
    for (int it = 0; it <= nb && ok; ++it) {
      if (it < nb) {
        const int2 krow = dec_block_rows(p, seq, blk(it));
        for (int u = 0; u < kDecKUnits && ok; ++u) load_unit(krow, u);
      }
      if (it >= 1) {
        const int2 vrow = dec_block_rows(p, seq, blk(it - 1));
        for (int u = 0; u < kDecVUnits && ok; ++u) load_unit(vrow, u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16(128, kHsHeads, false, false);
    constexpr uint32_t idesc_o = idesc_bf16(128, kHsHeads, true, true);
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
        const uint32_t tmem_s = tmem + kHsHeads * (it & 1);
        for (int u = 0; u < kDecKUnits && ok; ++u) {
          ok = warp_wait(bar(LY::BAR_FULL + slot), phase, abort_flag);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            for (int t = 0; t < ((u < 4) ? 2 : 1); ++t) {
              const int c = 2 * u + t;
              const uint64_t da = desc_add(dk0, slot * kDecUnit + t * kChunkBytes);
              const uint64_t db = desc_add(dq0, c * kHsQTile);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss(tmem_s, desc_add(da, 32 * kk), desc_add(db, 32 * kk), idesc_s, (c | kk) != 0);
            }
            mma_commit(bar(LY::BAR_EMPTY + slot));
          }
          __syncwarp();
          if (++slot == kHsStages) { slot = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (elect_one()) mma_commit(bar(LY::BAR_S + (it & 1)));
        __syncwarp();
      }
      if (it >= 1) {
        // O^T += V^T . P^T(b), V unit u = latent columns 128u .. 128u+127
        const int b = it - 1;
        if (blk(b) == jq) {
          // the query's own block may end inside the block: once its V units
          // are resident, let the softmax warps zero the rows past the end
          for (int u = 0; u < kDecVUnits && ok; ++u) {
            const int su = slot + u;
            ok = warp_wait(bar(LY::BAR_FULL + su % kHsStages), phase ^ (su >= kHsStages ? 1u : 0u), abort_flag);
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
              mma_ss(tmem_o + kHsHeads * u, desc_add(da, 2048 * kk), desc_add(dp0, 2048 * kk), idesc_o,
                     (b > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar(LY::BAR_EMPTY + slot));
          }
          __syncwarp();
          if (++slot == kHsStages) { slot = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (elect_one()) mma_commit(bar(LY::BAR_PV));
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------------------ softmax over keys
    const int quarter = warp & 3;
    const int key = quarter * 32 + lane;  // TMEM lane == key row of the block
    const int tid = threadIdx.x - 64;     // 0..127
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float cs = p.scale_log2;
    bool ok = true;
    for (int b = 0; b < nb && ok; ++b) {
      ok = warp_wait(bar(LY::BAR_S + (b & 1)), (b >> 1) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      if (tid == 0) *rescale_flag = 0;  // read by all only after the next two barriers
      float x[32];
      tmem_ld32(lane_addr + kHsHeads * (b & 1), x);
      const int kb = blk(b);
      const bool valid = kb * kTile + key <= i_q;
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] = valid ? x[i] : -INFINITY;
      redmax[quarter * kHsHeads + lane] = warp_reduce_scatter32<true>(x);
      named_barrier_sync(1, 128);
      if (b > 0) {
        // PV(b-1) done: P^T buffer free and O^T stable (phases waited in order)
        ok = warp_wait(bar(LY::BAR_PV), (b - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
      }
      if (tid < kHsHeads) {
        const float mb = fmaxf(fmaxf(redmax[tid], redmax[32 + tid]), fmaxf(redmax[64 + tid], redmax[96 + tid])) * cs;
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
      named_barrier_sync(1, 128);
      // P^T = 2^(cs*s - m) as the MN-major B operand: row = key, its 32 heads
      // contiguous in the first half of a 128-byte swizzled row
      float xr[32];
      {
        const float4* m4 = reinterpret_cast<const float4*>(m_run);
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
          *reinterpret_cast<uint4*>(prow + ((j ^ (key & 7)) << 4)) =
              make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      }
      redsum[quarter * kHsHeads + lane] = warp_reduce_scatter32<false>(x);
      redrsum[quarter * kHsHeads + lane] = warp_reduce_scatter32<false>(xr);
      // O^T rescale where a head's running maximum moved (lane = latent column)
      if (b > 0 && *rescale_flag) {
        float av[32];
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 a4 = reinterpret_cast<const float4*>(alpha)[i4];
          av[4 * i4] = a4.x;
          av[4 * i4 + 1] = a4.y;
          av[4 * i4 + 2] = a4.z;
          av[4 * i4 + 3] = a4.w;
        }
#pragma unroll 1
        for (int u = 0; u < 4; ++u) {
          float o[32];
          tmem_ld32(lane_addr + 2 * kHsHeads + kHsHeads * u, o);
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(o[i] * av[i]);
          tmem_st32(lane_addr + 2 * kHsHeads + kHsHeads * u, w);
        }
        tmem_st_wait();
      }
      named_barrier_sync(1, 128);
      if (tid < kHsHeads) {
        l_run[tid] = l_run[tid] * alpha[tid] + ((redsum[tid] + redsum[32 + tid]) + (redsum[64 + tid] + redsum[96 + tid]));
        r_run[tid] = r_run[tid] * alpha[tid] + ((redrsum[tid] + redrsum[32 + tid]) + (redrsum[64 + tid] + redrsum[96 + tid]));
      }
      if (kb == jq) {
        // rows past the sequence end: zero them in the V units (the cache may
        // hold anything there) so that 0 * garbage cannot reach O
        ok = warp_wait(bar(LY::BAR_VT), 0, abort_flag);
        if (!ok) break;
        if (!valid) {
          const uint4 z = make_uint4(0, 0, 0, 0);
          for (int u = 0; u < kDecVUnits; ++u) {
            const int slot_u = hs_v_pos(b, u, nb) % kHsStages;
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
    // ------------------------------------------------------------ epilogue
    if (ok) ok = warp_wait(bar(LY::BAR_PV), (nb - 1) & 1, abort_flag);
    named_barrier_sync(1, 128);  // l_run, r_run complete
    if (ok) {
      tc_fence_after();
      float inv[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) inv[i] = 1.f / r_run[i];
      __nv_bfloat16* orow = p.out + ((int64_t)seq * kDecHeads + head0) * 512;
#pragma unroll 1
      for (int u = 0; u < 4; ++u) {
        const int d = 128 * u + key;  // latent column of this lane
        float o[32];
        tmem_ld32(lane_addr + 2 * kHsHeads + kHsHeads * u, o);
#pragma unroll
        for (int i = 0; i < 32; ++i) orow[(int64_t)i * 512 + d] = __float2bfloat16_rn(o[i] * inv[i]);
      }
      if (tid < kHsHeads)
        p.lse[(int64_t)seq * kDecHeads + head0 + tid] = (m_run[tid] + log2f(l_run[tid])) * 0.69314718055994530942f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace loza
