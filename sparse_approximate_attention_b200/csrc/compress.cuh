// Compression stage: query-block sum, KV importance scores, top-lp selection
// and the passing-buffer gather.  All four are HBM- or latency-bound; none of
// them is a dense contraction once the score is written in its linear form.
//
// "Spava ..." (sciencestack.ai), Fig. 5 caption: Q_qr K^(h)T estimates KV
// importance and B_c^(h) are the essential KVs; "APB-V ..." (pith.science
// review), "What carries the argument": each context block is compressed to
// its top-lp key-value pairs ranked by Q_qr K^T and gathered by later hosts.
#pragma once
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "plan.hpp"
#include "ptx.cuh"

namespace spava {

namespace cg = cooperative_groups;

// ---------------------------------------------------------------------------
// qsum[kv][c] = scale * sum over query rows i and heads g of KV head kv of
// Q[qs+i, g, c].  One cluster of kQsumSplit CTAs per KV head: each CTA sums a
// slice of the (row, head) pairs (kQsumUnroll 16-byte loads per thread in
// flight), pushes its slice sum into CTA 0 through distributed shared
// memory, and CTA 0 adds the slices in rank order (deterministic, one
// launch).  The order of every addition is fixed by the problem's sizes
// alone, so the scoring stage and the fused compression, which both start
// with this kernel, see the same qsum bits.
// ---------------------------------------------------------------------------
constexpr int kQsumSplit = 8;
constexpr int kQsumThreads = 512;
constexpr int kQsumUnroll = 8;

template <int D>
__global__ void __cluster_dims__(kQsumSplit, 1, 1) __launch_bounds__(kQsumThreads, 1)
    qsum_kernel(const __nv_bfloat16* __restrict__ Q, float* __restrict__ qsum, int64_t qs, int lq,
                int Hq, int G, float scale) {
  constexpr int kParts = D / 8;                    // 16-byte chunks per row
  constexpr int kRows = kQsumThreads / kParts;     // rows per pass of the CTA
  constexpr int kWarps = kQsumThreads / 32;
  __shared__ float part[kWarps][D];
  __shared__ float gathered[kQsumSplit][D];
  // A kernel launched after this one as its programmatic dependent (the fused
  // compression) may start now; it waits for this grid before reading qsum.
  if (threadIdx.x == 0) grid_dependents_launch();
  cg::cluster_group cluster = cg::this_cluster();
  const int kv = blockIdx.y;
  const int rank = static_cast<int>(cluster.block_rank());
  const int total = lq * G;
  const int r0 = static_cast<int>((static_cast<int64_t>(total) * rank) / kQsumSplit);
  const int r1 = static_cast<int>((static_cast<int64_t>(total) * (rank + 1)) / kQsumSplit);
  const int tid = threadIdx.x, pc = tid % kParts, lr = tid / kParts;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int rb = r0 + lr; rb < r1; rb += kQsumUnroll * kRows) {
    uint4 raw[kQsumUnroll];
#pragma unroll
    for (int u = 0; u < kQsumUnroll; ++u) {
      const int rr = rb + u * kRows;
      const int i = rr / G, g = kv * G + rr % G;
      raw[u] = rr < r1 ? *reinterpret_cast<const uint4*>(Q + ((qs + i) * Hq + g) * D + pc * 8)
                       : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kQsumUnroll; ++u) {
      const __nv_bfloat16* v = reinterpret_cast<const __nv_bfloat16*>(&raw[u]);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __bfloat162float(v[e]);
    }
  }
  // lanes l and l ^ 16 hold the same column chunk (for D = 128): add them
#pragma unroll
  for (int off = kParts; off < 32; off <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  if ((tid & 31) < kParts)
#pragma unroll
    for (int e = 0; e < 8; ++e) part[tid >> 5][pc * 8 + e] = acc[e];
  __syncthreads();
  for (int c = tid; c < D; c += kQsumThreads) {
    float s = 0.f;
    for (int w = 0; w < kWarps; ++w) s += part[w][c];
    cluster.map_shared_rank(&gathered[rank][0], 0)[c] = s;
  }
  cluster.sync();   // CTA 0 holds every slice; no CTA touches another's memory after this
  if (rank == 0) {
    for (int c = tid; c < D; c += kQsumThreads) {
      float s = 0.f;
      for (int r = 0; r < kQsumSplit; ++r) s += gathered[r][c];
      qsum[kv * D + c] = s * scale;
    }
  }
}

// ---------------------------------------------------------------------------
// scores[kv][j] = <qsum[kv], K[key0 + j, kv, :]> for j < nkeys.  The rows
// [key0, key0 + nkeys) of K are one contiguous region (all KV heads); each
// CTA streams an equal share of it through a ring in shared memory:
// kScoreSlots 16-byte cp.async copies per thread in flight, each thread
// reading back only its own cells; the first copies are issued before the
// wait for the query sum (the kernel is qsum_kernel's programmatic dependent).  The D/8 lanes that hold one (key, head)
// row reduce with shuffles, in the same order as the fused compression, so
// both give the same bits.
// ---------------------------------------------------------------------------
constexpr int kScoreThreads = 512;
constexpr int kScoreSlots = 8;
constexpr int kScoreChunk = kScoreThreads * 16;   // bytes of one ring slot

__host__ __device__ constexpr int score_smem_bytes(int Hkv, int D) {
  return kScoreSlots * kScoreChunk + Hkv * D * 4;
}

template <int D>
__global__ void __launch_bounds__(kScoreThreads, 2)
    score_kernel(const __nv_bfloat16* __restrict__ K, const float* __restrict__ qsum,
                 float* __restrict__ scores, int64_t key0, int64_t nkeys, int Hkv) {
  constexpr int kParts = D / 8;
  extern __shared__ __align__(16) uint8_t dsm[];
  float* sq = reinterpret_cast<float*>(dsm + kScoreSlots * kScoreChunk);
  const int tid = threadIdx.x, pc = tid % kParts;
  const int64_t total = nkeys * Hkv * kParts;   // 16-byte chunks
  const int64_t items = (total + kScoreThreads - 1) / kScoreThreads;
  const int64_t it0 = items * blockIdx.x / gridDim.x, it1 = items * (blockIdx.x + 1) / gridDim.x;
  const int n = static_cast<int>(it1 - it0);
  const uint4* src = reinterpret_cast<const uint4*>(K + key0 * Hkv * D);
  const uint32_t cell = smem_u32(dsm) + tid * 16;
  auto issue = [&](int i) {
    if (i < n) {
      const int64_t c = (it0 + i) * kScoreThreads + tid;
      if (c < total) cp_async16(cell + (i % kScoreSlots) * kScoreChunk, src + c);
    }
    cp_async_commit();
  };
  // this thread's (key, head) row, advanced by kScoreThreads / kParts rows per item
  // without a division per item
  constexpr int kStep = kScoreThreads / kParts;
  const int64_t rh0 = (it0 * kScoreThreads + tid) / kParts;
  int64_t j = rh0 / Hkv;
  int kv = static_cast<int>(rh0 % Hkv);
  const int step_j = kStep / Hkv, step_kv = kStep % Hkv;
#pragma unroll 1
  for (int i = 0; i < kScoreSlots; ++i) issue(i);
  grid_dependency_wait();   // launched as qsum_kernel's programmatic dependent
  for (int c = tid; c < Hkv * D; c += kScoreThreads) sq[c] = __ldcg(qsum + c);
  __syncthreads();
#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    cp_async_wait<kScoreSlots - 1>();
    const uint4 raw = ld_shared_v4(cell + (i % kScoreSlots) * kScoreChunk);
    const __nv_bfloat16* v = reinterpret_cast<const __nv_bfloat16*>(&raw);
    const float* q = sq + kv * D + pc * 8;
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) dot = fmaf(__bfloat162float(v[e]), q[e], dot);
    issue(i + kScoreSlots);   // the slot's value is consumed
#pragma unroll
    for (int off = kParts / 2; off >= 1; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    if (pc == 0 && j < nkeys) scores[kv * nkeys + j] = dot;
    j += step_j;
    kv += step_kv;
    if (kv >= Hkv) {
      kv -= Hkv;
      ++j;
    }
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// top-lp per (block h < V-1, KV head): MSB-first radix select on
// order-preserving 32-bit keys finds the lp-th largest key T and how many
// copies of T to keep; a block-wide scan in index order then writes the kept
// indices ascending (ties at T keep the lowest indices).
// ---------------------------------------------------------------------------
constexpr int kTopkThreads = 1024;

struct TopkParams {
  int32_t start[kMaxV];   // first score column of block h
  int32_t L[kMaxV];
  int32_t k[kMaxV];       // lp_eff(h)
  int32_t Hkv, lp;
  int64_t score_cols;
};

__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;   // -0.0 ranks as +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t block_exclusive_scan_u64(uint64_t v, uint64_t* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    uint64_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    uint64_t t = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      uint64_t y = __shfl_up_sync(0xffffffffu, t, off);
      if (lane >= off) t += y;
    }
    if (lane < nw) warp_tot[lane] = t;   // inclusive
  }
  __syncthreads();
  const uint64_t before = warp ? warp_tot[warp - 1] : 0;
  return before + x - v;
}

__global__ void __launch_bounds__(kTopkThreads)
    topk_kernel(const float* __restrict__ scores, int32_t* __restrict__ idx, TopkParams p) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_k;
  __shared__ uint64_t warp_tot[32];
  const int h = blockIdx.x / p.Hkv, kv = blockIdx.x % p.Hkv;
  const int L = p.L[h], k = p.k[h];
  const float* s = scores + kv * p.score_cols + p.start[h];
  int32_t* out = idx + (static_cast<int64_t>(h) * p.Hkv + kv) * p.lp;
  const int tid = threadIdx.x;
  for (int t = k + tid; t < p.lp; t += blockDim.x) out[t] = -1;
  if (k <= 0) return;
  if (tid == 0) {
    s_prefix = 0;
    s_k = static_cast<uint32_t>(k);
  }
  uint32_t mask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    for (int i = tid; i < L; i += blockDim.x) {
      const uint32_t key = order_key(s[i]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        c[b] = hist[tid * 8 + b];
        tot += c[b];
      }
      uint32_t x = tot;   // inclusive suffix sum over lanes
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        uint32_t y = __shfl_down_sync(0xffffffffu, x, off);
        if (tid + off < 32) x += y;
      }
      uint32_t running = x - tot;   // count in higher bins
      const uint32_t kk = s_k;
#pragma unroll
      for (int b = 7; b >= 0; --b) {
        if (running < kk && running + c[b] >= kk) {
          s_prefix = prefix | (static_cast<uint32_t>(tid * 8 + b) << shift);
          s_k = kk - running;
        }
        running += c[b];
      }
    }
    __syncthreads();
    mask |= 0xFFu << shift;
  }
  const uint32_t T = s_prefix;
  const uint32_t keq = s_k;   // copies of T to keep (>= 1)
  const int chunk = (L + blockDim.x - 1) / blockDim.x;
  const int i0 = min(L, tid * chunk), i1 = min(L, i0 + chunk);
  uint32_t gt = 0, eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = order_key(s[i]);
    gt += key > T;
    eq += key == T;
  }
  const uint64_t pre = block_exclusive_scan_u64((static_cast<uint64_t>(eq) << 32) | gt, warp_tot);
  uint32_t gt_pre = static_cast<uint32_t>(pre), eq_pre = static_cast<uint32_t>(pre >> 32);
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = order_key(s[i]);
    if (key > T) {
      out[gt_pre + min(eq_pre, keq)] = i;
      ++gt_pre;
    } else if (key == T) {
      if (eq_pre < keq) out[gt_pre + eq_pre] = i;
      ++eq_pre;
    }
  }
}

// ---------------------------------------------------------------------------
// Kp/Vp[off_h + t, kv, :] = K/V[start_h + idx[h][kv][t], kv, :].  One thread
// per 16-byte chunk; an index outside its block writes zeros and raises bit 1
// of the device error word instead of reading out of bounds.
// ---------------------------------------------------------------------------
constexpr unsigned int kErrBadIndex = 2u;

struct GatherParams {
  int32_t start[kMaxV];
  int32_t L[kMaxV];
  int32_t poff[kMaxV + 1];
  int32_t nblocks;   // V - 1
  int32_t Hkv, lp;
  int64_t rows;      // passing rows
};

template <int D>
__global__ void __launch_bounds__(256)
    gather_kernel(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
                  const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ Kp,
                  __nv_bfloat16* __restrict__ Vp, GatherParams p) {
  constexpr int kParts = D / 8;
  const int64_t per = p.rows * p.Hkv * kParts;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < 2 * per;
       c += stride) {
    const int which = c >= per;
    const int64_t cc = c - which * per;
    const int pc = static_cast<int>(cc % kParts);
    const int64_t t2 = cc / kParts;
    const int kv = static_cast<int>(t2 % p.Hkv);
    const int64_t prow = t2 / p.Hkv;
    int h = 0;
    while (h + 1 < p.nblocks && p.poff[h + 1] <= prow) ++h;
    const int t = static_cast<int>(prow - p.poff[h]);
    const int32_t j = idx[(static_cast<int64_t>(h) * p.Hkv + kv) * p.lp + t];
    uint4 val = make_uint4(0, 0, 0, 0);
    if (j >= 0 && j < p.L[h]) {
      const __nv_bfloat16* src = (which ? V : K) +
                                 ((static_cast<int64_t>(p.start[h]) + j) * p.Hkv + kv) * D + pc * 8;
      val = *reinterpret_cast<const uint4*>(src);
    } else if (pc == 0) {
      atomicOr(&g_device_error, kErrBadIndex);
    }
    __nv_bfloat16* dst = (which ? Vp : Kp) + (prow * p.Hkv + kv) * D + pc * 8;
    *reinterpret_cast<uint4*>(dst) = val;
  }
}

}  // namespace spava
