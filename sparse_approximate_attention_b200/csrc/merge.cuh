// Merge of the per-host partial query results by log-sum-exp.
//
// "APB-V ..." (pith.science review), Axiom & Free-Parameter Ledger: merging
// partial attention results through their FlashAttention lse is exact;
// "Technische Samenvatting: APB-V" (gist.science, nl), fused context and
// query forward: the partial query results are merged with the lse outputs.
//   lse = log sum_h exp(lse_h),  O = sum_h exp(lse_h - lse) O_h
#pragma once
#include <cuda_bf16.h>

#include "plan.hpp"

namespace spava {

// One warp per (query row, head), rows in output order: lane h < V loads
// partial h's lse, the maximum and the sum go round the warp by shuffles,
// then every lane combines its D/32 columns over the V partials (four loads
// in flight) and writes them as bf16; lane 0 writes the lse.
template <int D>
__global__ void __launch_bounds__(256)
    merge_kernel(const float* __restrict__ O_part, const float* __restrict__ lse_part,
                 __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int V, int lq, int Hq,
                 int64_t qs, int64_t n) {
  constexpr int kPer = D / 32;   // columns per lane: 4 (d = 128) or 2 (d = 64)
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t total = static_cast<int64_t>(lq) * Hq;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); t < total;
       t += warps) {
    const int g = static_cast<int>(t % Hq);
    const int i = static_cast<int>(t / Hq);
    const float lp = lane < V ? lse_part[(static_cast<int64_t>(lane) * Hq + g) * lq + i] : -INFINITY;
    float mx = lp;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float e = lane < V ? expf(lp - mx) : 0.f;
    float sum = e;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float w_mine = e / sum;   // weight of partial `lane`
    float acc[kPer];
#pragma unroll
    for (int c = 0; c < kPer; ++c) acc[c] = 0.f;
    const float* src = O_part + (static_cast<int64_t>(i) * Hq + g) * D + lane * kPer;
    const int64_t hstride = static_cast<int64_t>(lq) * Hq * D;
#pragma unroll 4
    for (int h = 0; h < V; ++h) {
      const float w = __shfl_sync(0xffffffffu, w_mine, h);
      if (kPer == 4) {
        const float4 o = *reinterpret_cast<const float4*>(src + h * hstride);
        acc[0] = fmaf(w, o.x, acc[0]);
        acc[1] = fmaf(w, o.y, acc[1]);
        acc[2] = fmaf(w, o.z, acc[2]);
        acc[3] = fmaf(w, o.w, acc[3]);
      } else {
        const float2 o = *reinterpret_cast<const float2*>(src + h * hstride);
        acc[0] = fmaf(w, o.x, acc[0]);
        acc[1] = fmaf(w, o.y, acc[1]);
      }
    }
    __nv_bfloat16* dst = O + ((qs + i) * Hq + g) * D + lane * kPer;
    if (kPer == 4) {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0], acc[1]);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2], acc[3]);
      *reinterpret_cast<uint2*>(dst) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
    } else {
      const __nv_bfloat162 v = __floats2bfloat162_rn(acc[0], acc[1]);
      *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(&v);
    }
    if (lane == 0) lse[static_cast<int64_t>(g) * n + qs + i] = mx + logf(sum);
  }
}

}  // namespace spava
