// merge.cuh - combining two attention branches of the same queries.
//
// ssa_merge_kernel: branches a and b are softmax attention of each (token,
// head) row over two disjoint key sets (for example the sink + local blocks
// of SSA and a second set of selected blocks); from their (O, LSE) it writes
// attention over the union:
//     LSE = ln(e^LSE_a + e^LSE_b),  O = e^(LSE_a - LSE) O_a + e^(LSE_b - LSE) O_b
// with LSE = -inf for a branch without keys (weight 0; both empty: O = 0).
//
// ssa_mix_kernel: O = alpha O_full + (1 - alpha) O_ssa, the mix of a module's
// full-attention and sparse branches during calibration (page 1 section 01
// (1) of the LoZA pages; the formula is lost in the page text, this is its
// plain reading).
//
// Both are one pass over HBM: every thread moves 16-byte vectors (8 bf16) of
// one row, grid-stride over rows x vectors.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace loza {

constexpr int kMergeThreads = 256;

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
}

// vec8 = d_v / 8 vectors per row
__global__ void __launch_bounds__(kMergeThreads) ssa_merge_kernel(const uint4* __restrict__ o_a,
                                                                  const float* __restrict__ lse_a,
                                                                  const uint4* __restrict__ o_b,
                                                                  const float* __restrict__ lse_b,
                                                                  uint4* __restrict__ out, float* __restrict__ lse_out,
                                                                  int64_t rows, int vec8) {
  const int64_t total = rows * vec8;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = idx / vec8;
    const float la = lse_a[r], lb = lse_b[r];
    float wa = 0.f, wb = 0.f, l = -INFINITY;
    if (la != -INFINITY || lb != -INFINITY) {
      const float m = fmaxf(la, lb);
      const float ea = expf(la - m), eb = expf(lb - m);
      const float inv = 1.f / (ea + eb);
      wa = ea * inv;
      wb = eb * inv;
      l = m + logf(ea + eb);
    }
    float fa[8], fb[8], fo[8];
    unpack8(o_a[idx], fa);
    unpack8(o_b[idx], fb);
#pragma unroll
    for (int i = 0; i < 8; ++i) fo[i] = wa * fa[i] + wb * fb[i];
    out[idx] = pack8(fo);
    if (idx - r * vec8 == 0) lse_out[r] = l;
  }
}

__global__ void __launch_bounds__(kMergeThreads) ssa_mix_kernel(const uint4* __restrict__ o_full,
                                                                const uint4* __restrict__ o_ssa,
                                                                uint4* __restrict__ out, int64_t n8, float alpha) {
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n8;
       idx += (int64_t)gridDim.x * blockDim.x) {
    float fa[8], fb[8], fo[8];
    unpack8(o_full[idx], fa);
    unpack8(o_ssa[idx], fb);
#pragma unroll
    for (int i = 0; i < 8; ++i) fo[i] = fmaf(alpha, fa[i], (1.f - alpha) * fb[i]);
    out[idx] = pack8(fo);
  }
}

}  // namespace loza
