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

template <int D>
__global__ void __launch_bounds__(256)
    merge_kernel(const float* __restrict__ O_part, const float* __restrict__ lse_part,
                 __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int V, int lq, int Hq,
                 int64_t qs, int64_t n) {
  constexpr int kQuads = D / 4;
  const int64_t total = static_cast<int64_t>(lq) * Hq * kQuads;
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < total;
       c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int qd = static_cast<int>(c % kQuads);
    const int64_t t = c / kQuads;
    const int g = static_cast<int>(t % Hq);
    const int i = static_cast<int>(t / Hq);
    float mx = -INFINITY;
    for (int h = 0; h < V; ++h) mx = fmaxf(mx, lse_part[(static_cast<int64_t>(h) * Hq + g) * lq + i]);
    float sum = 0.f;
    for (int h = 0; h < V; ++h) sum += expf(lse_part[(static_cast<int64_t>(h) * Hq + g) * lq + i] - mx);
    const float lse_tot = mx + logf(sum);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int h = 0; h < V; ++h) {
      const float w = expf(lse_part[(static_cast<int64_t>(h) * Hq + g) * lq + i] - lse_tot);
      const float4 o = *reinterpret_cast<const float4*>(
          O_part + ((static_cast<int64_t>(h) * lq + i) * Hq + g) * D + qd * 4);
      acc.x = fmaf(w, o.x, acc.x);
      acc.y = fmaf(w, o.y, acc.y);
      acc.z = fmaf(w, o.z, acc.z);
      acc.w = fmaf(w, o.w, acc.w);
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 packed = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
    *reinterpret_cast<uint2*>(O + ((qs + i) * Hq + g) * D + qd * 4) = packed;
    if (qd == 0) lse[static_cast<int64_t>(g) * n + qs + i] = lse_tot;
  }
}

}  // namespace spava
