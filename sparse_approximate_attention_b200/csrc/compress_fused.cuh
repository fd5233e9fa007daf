// Fused compression: KV importance scores, top-lp selection and the
// passing-buffer gather in one launch, after the query-block sum
// (qsum_kernel, whose programmatic dependent it is).
//
// "Spava ..." (sciencestack.ai), Fig. 5 caption: Q_qr K^(h)T estimates KV
// importance and B_c^(h) are the essential KVs; "APB-V ..." (pith.science
// review), "What carries the argument": each context block is compressed to
// its top-lp key-value pairs ranked by Q_qr K^T and gathered by later hosts.
//
// One thread-block cluster of nc CTAs (4 or 8, chosen at launch so that the
// grid fits the GPU in one wave when it can) per (block h < V-1, KV head) (all
// such blocks, or those a host mask selects), for blocks of up to
// kCompressMaxBlock keys.  CTA r of the cluster owns slice r of the block's
// keys.
//   1. The K rows of the slice stream through a ring in shared memory,
//      16-byte cp.async copies per thread.  The first ring's worth is issued
//      before the kernel waits for the query-block sum qsum = scale * sum q;
//      each K row then gives its score, written out and kept in shared
//      memory as an order-preserving 32-bit key.
//   2. MSB-first radix select over the cluster: four 8-bit passes; each CTA
//      counts its own slice (warp-aggregated shared atomics) and pushes the
//      256 counts into every CTA of the cluster, so all CTAs pick the same
//      digit from the same totals.  The counts of the earlier slices give
//      each CTA how many kept keys precede its slice.
//   3. Each CTA ranks its own kept keys in index order (ballots) and writes
//      their indices (ascending over the block; ties at the threshold keep
//      the lower indices).
//   4. After one more cluster barrier (which publishes the indices), CTA r
//      copies kept ranks [r*k/nc, (r+1)*k/nc) of K and V into the passing
//      buffer, so the copy is balanced whatever slices the kept keys fall in.
// After step 4's barrier no CTA touches another's shared memory, so CTAs
// leave independently.
//
// kSelectOnly: the stage entry spava_select_topk.  Step 1 reads the scores
// (written by spava_score) instead of computing them, and step 4 is skipped.
#pragma once
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "compress.cuh"
#include "plan.hpp"
#include "ptx.cuh"

namespace spava {

constexpr int kCompressMinCtas = 4;    // cluster sizes: 4 or 8 (16, a non-portable size, was
constexpr int kCompressMaxCtas = 8;    // measured slower on small problems: 31 us against 27)
constexpr int kCompressThreads = 512;
constexpr int kCompressWarps = kCompressThreads / 32;
constexpr int kCompressMaxBlock = 24576;   // keys per block
// The copy ring: kRingSlots slots of 16 bytes per thread.  The K stream keeps
// every slot in flight; the gather uses slot pairs (K and V).
constexpr int kRingChunk = kCompressThreads * 16;
constexpr int kRingSlots = 8;
constexpr int kRingBytes = kRingSlots * kRingChunk;

__host__ __device__ constexpr int compress_slice_cap(int lmax, int nc) {
  return ((lmax + nc - 1) / nc + 3) / 4 * 4;
}

// Dynamic shared memory of a launch with clusters of nc CTAs whose longest
// compressed block has lmax keys: the ring, then the keys of one slice (later
// the CTA's share of the kept indices).
__host__ __device__ constexpr int compress_smem_bytes(int lmax, int nc) {
  return kRingBytes + 4 * compress_slice_cap(lmax, nc);
}
// The same for the select-only form: no ring.
__host__ __device__ constexpr int select_smem_bytes(int lmax, int nc) { return 4 * compress_slice_cap(lmax, nc); }

struct CompressParams {
  int32_t start[kMaxV];   // first sequence row of block h
  int32_t L[kMaxV];
  int32_t k[kMaxV];       // lp_eff(h)
  int32_t poff[kMaxV + 1];
  int32_t Hkv, lp;
  int32_t lmax;           // longest compressed block (sizes the shared key array)
  int64_t la, score_cols;
  // merge counters of the attention launch that follows (zeroed here so that
  // no separate launch is needed); null when called on its own
  int32_t* merge_count;
  int32_t n_merge;
  int32_t blk[kMaxV];     // the compressed blocks, one per grid row (all h < V-1, or a host mask's)
};

template <int D, bool kSelectOnly = false>
__global__ void __launch_bounds__(kCompressThreads, 2)
    compress_kernel(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
                    const float* __restrict__ qsum,
                    float* __restrict__ scores, int32_t* __restrict__ idx,
                    __nv_bfloat16* __restrict__ Kp, __nv_bfloat16* __restrict__ Vp,
                    const __grid_constant__ CompressParams p) {
  constexpr int kParts = D / 8;                           // 16-byte chunks per row
  constexpr int kRowsPerIter = kCompressThreads / kParts;  // rows per ring slot
  extern __shared__ __align__(16) uint8_t dsm[];
  const int nc = static_cast<int>(gridDim.x);   // the cluster: one per (block, KV head)
  uint32_t* keys = reinterpret_cast<uint32_t*>(dsm + (kSelectOnly ? 0 : kRingBytes));   // [slice] keys, then kept indices
  __shared__ uint32_t hx[2][kCompressMaxCtas][256];   // every CTA's counts of a radix pass
  __shared__ uint32_t hist[256], tot[256], low[256];
  __shared__ uint64_t warp_tot[32];
  __shared__ uint32_t s_digit, s_k, s_gt_before, s_eq_before;

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int h = p.blk[blockIdx.y], kv = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // The attention launch that follows may start on the SMs this grid leaves
  // free; it reads nothing written here before its griddepcontrol.wait.
  if (tid == 0) grid_dependents_launch();
  if (p.merge_count != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && kv == 0)
    for (int i = tid; i < p.n_merge; i += kCompressThreads) p.merge_count[i] = 0;
  const int L = p.L[h], kk = p.k[h];
  const bool all = kk >= L;
  const int j0 = static_cast<int>((static_cast<int64_t>(L) * rank) / nc);
  const int j1 = static_cast<int>((static_cast<int64_t>(L) * (rank + 1)) / nc);
  const int n = j1 - j0;   // keys of this CTA's slice
  const int pc = tid % kParts, lr = tid / kParts;
  const uint32_t cell = smem_u32(dsm) + tid * 16;   // this thread's cell of ring slot 0

  float* srow = scores + static_cast<int64_t>(kv) * p.score_cols + (p.start[h] - p.la) + j0;
  if constexpr (kSelectOnly) {
    // ---- 1. this slice's scores into keys
    for (int i = tid; i < n; i += kCompressThreads) keys[i] = order_key(srow[i]);
  } else {
    // ---- 1. K rows of the slice through the ring; scores and keys
    const int nItems = (n + kRowsPerIter - 1) / kRowsPerIter;
    const int64_t row0 = p.start[h] + j0;
    auto issue = [&](int it) {
      if (it < nItems) {
        const int jj = it * kRowsPerIter + lr;
        if (jj < n) cp_async16(cell + (it % kRingSlots) * kRingChunk, K + ((row0 + jj) * p.Hkv + kv) * D + pc * 8);
      }
      cp_async_commit();   // one group per item (empty past the end), so the waits count items
    };
#pragma unroll 1
    for (int it = 0; it < kRingSlots; ++it) issue(it);
    grid_dependency_wait();   // qsum is complete and visible
    float q8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) q8[e] = __ldcg(qsum + kv * D + pc * 8 + e);
#pragma unroll 1
    for (int it = 0; it < nItems; ++it) {
      cp_async_wait<kRingSlots - 1>();   // this thread's copy of item it has landed
      const uint4 raw = ld_shared_v4(cell + (it % kRingSlots) * kRingChunk);
      const __nv_bfloat16* v = reinterpret_cast<const __nv_bfloat16*>(&raw);
      const int jj = it * kRowsPerIter + lr;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(__bfloat162float(v[e]), q8[e], dot);
      issue(it + kRingSlots);   // the slot's value is consumed
#pragma unroll
      for (int off = kParts / 2; off >= 1; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      if (pc == 0 && jj < n) {
        srow[jj] = dot;
        keys[jj] = order_key(dot);
      }
    }
  }
  __syncthreads();

  // ---- 2. radix select of the kk largest keys of the block, over the cluster
  uint32_t T = 0, keq = 0, gt_before = 0, eq_before = 0;
  if (!all && kk > 0) {
    if (tid == 0) s_gt_before = 0;
    uint32_t prefix = 0, mask = 0, need = static_cast<uint32_t>(kk);
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass, buf = pass & 1;
      if (tid < 256) hist[tid] = 0;
      __syncthreads();
      for (int base = 0; base < n; base += kCompressThreads) {   // CTA-uniform trip count
        const int i = base + tid;
        uint32_t bin = 0xFFFFFFFFu;
        if (i < n) {
          const uint32_t key = keys[i];
          if ((key & mask) == prefix) bin = (key >> shift) & 255u;
        }
        const uint32_t same = __match_any_sync(0xffffffffu, bin);
        if (bin != 0xFFFFFFFFu && lane == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
      }
      __syncthreads();
      if (tid < 256) {
        const uint32_t c = hist[tid];
        for (int r = 0; r < nc; ++r) cluster.map_shared_rank(&hx[buf][rank][0], r)[tid] = c;
      }
      cluster.sync();   // every CTA's counts of this pass are in every CTA
      if (tid < 256) {
        uint32_t t = 0, lo = 0;
        for (int r = 0; r < nc; ++r) {
          const uint32_t c = hx[buf][r][tid];
          t += c;
          if (r < rank) lo += c;
        }
        tot[tid] = t;
        low[tid] = lo;
      }
      __syncthreads();
      if (warp == 0) {
        uint32_t c[8], t8 = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          c[b] = tot[lane * 8 + b];
          t8 += c[b];
        }
        uint32_t x = t8;   // inclusive suffix sum over lanes
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t y = __shfl_down_sync(0xffffffffu, x, off);
          if (lane + off < 32) x += y;
        }
        uint32_t running = x - t8;   // count in higher bins
#pragma unroll
        for (int b = 7; b >= 0; --b) {
          if (running < need && running + c[b] >= need) {
            s_digit = static_cast<uint32_t>(lane * 8 + b);
            s_k = need - running;
          }
          running += c[b];
        }
        __syncwarp();
        // keys of earlier slices in bins above the digit are kept and precede this slice
        const uint32_t d = s_digit;
        uint32_t lo = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b)
          if (static_cast<uint32_t>(lane * 8 + b) > d) lo += low[lane * 8 + b];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) lo += __shfl_xor_sync(0xffffffffu, lo, off);
        if (lane == 0) {
          s_gt_before += lo;
          if (pass == 3) s_eq_before = low[d];
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      need = s_k;
      mask |= 0xFFu << shift;
    }
    T = prefix;
    keq = need;
    gt_before = s_gt_before;
    eq_before = s_eq_before;
  }

  // ---- 3. this slice's kept keys: positions in index order, indices out
  int32_t* out = idx + (static_cast<int64_t>(h) * p.Hkv + kv) * p.lp;
  if (all) {
    for (int i = tid; i < n; i += kCompressThreads) out[j0 + i] = j0 + i;
  } else if (kk > 0) {
    // warp w takes a contiguous run of the slice, 32 keys per ballot
    const int per = (n + kCompressWarps * 32 - 1) / (kCompressWarps * 32) * 32;
    const int w0 = min(n, warp * per), w1 = min(n, w0 + per);
    uint32_t g = 0, e = 0;
    for (int b = w0; b < w1; b += 32) {
      const int i = b + lane;
      const uint32_t key = i < w1 ? keys[i] : 0u;
      g += __popc(__ballot_sync(0xffffffffu, i < w1 && key > T));
      e += __popc(__ballot_sync(0xffffffffu, i < w1 && key == T));
    }
    const uint64_t wsum = lane == 0 ? (static_cast<uint64_t>(e) << 32) | g : 0ull;
    const uint64_t pre = __shfl_sync(0xffffffffu, block_exclusive_scan_u64(wsum, warp_tot), 0);
    uint32_t G = gt_before + static_cast<uint32_t>(pre);
    uint32_t E = eq_before + static_cast<uint32_t>(pre >> 32);
    const uint32_t lt = (1u << lane) - 1u;
    for (int b = w0; b < w1; b += 32) {
      const int i = b + lane;
      const uint32_t key = i < w1 ? keys[i] : 0u;
      const bool isg = i < w1 && key > T, ise = i < w1 && key == T;
      const uint32_t gb = __ballot_sync(0xffffffffu, isg), eb = __ballot_sync(0xffffffffu, ise);
      const uint32_t Gi = G + __popc(gb & lt), Ei = E + __popc(eb & lt);
      if (isg || (ise && Ei < keq)) out[Gi + min(Ei, keq)] = j0 + i;
      G += __popc(gb);
      E += __popc(eb);
    }
  }
  if (rank == 0)
    for (int t = kk + tid; t < p.lp; t += kCompressThreads) out[t] = -1;
  cluster.sync();   // the indices of every slice are written; the last access to peer shared memory
  if constexpr (kSelectOnly) return;

  // ---- 4. kept ranks [g0, g1) of the block: K and V rows into the passing buffer
  if (kk > 0) {
    const int g0 = static_cast<int>((static_cast<int64_t>(kk) * rank) / nc);
    const int g1 = static_cast<int>((static_cast<int64_t>(kk) * (rank + 1)) / nc);
    const int cnt = g1 - g0;   // <= compress_slice_cap(p.lmax, nc)
    int32_t* gidx = reinterpret_cast<int32_t*>(keys);
    for (int t = tid; t < cnt; t += kCompressThreads) gidx[t] = all ? g0 + t : __ldcg(out + g0 + t);
    __syncthreads();
    constexpr int kPairs = kRingSlots / 2;
    const int nG = (cnt + kRowsPerIter - 1) / kRowsPerIter;
    const int64_t src0 = p.start[h], dst0 = static_cast<int64_t>(p.poff[h]) + g0;
    auto issue_g = [&](int it) {
      if (it < nG) {
        const int s = it * kRowsPerIter + lr;
        if (s < cnt) {
          const int64_t src = ((src0 + gidx[s]) * p.Hkv + kv) * D + pc * 8;
          const uint32_t dst = cell + (it % kPairs) * 2 * kRingChunk;
          cp_async16(dst, K + src);
          cp_async16(dst + kRingChunk, V + src);
        }
      }
      cp_async_commit();
    };
#pragma unroll 1
    for (int it = 0; it < kPairs; ++it) issue_g(it);
#pragma unroll 1
    for (int it = 0; it < nG; ++it) {
      cp_async_wait<kPairs - 1>();
      const int s = it * kRowsPerIter + lr;
      if (s < cnt) {
        const uint32_t a = cell + (it % kPairs) * 2 * kRingChunk;
        const uint4 kx = ld_shared_v4(a), vx = ld_shared_v4(a + kRingChunk);
        const int64_t dst = ((dst0 + s) * p.Hkv + kv) * D + pc * 8;
        *reinterpret_cast<uint4*>(Kp + dst) = kx;
        *reinterpret_cast<uint4*>(Vp + dst) = vx;
      }
      issue_g(it + kPairs);   // the slot pair's values are consumed
    }
  }
  cp_async_wait<0>();
}

}  // namespace spava
