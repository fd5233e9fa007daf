// Fused compression: query-block sum, KV importance scores, top-lp selection
// and the passing-buffer gather in one launch.
//
// "Spava ..." (sciencestack.ai), Fig. 5 caption: Q_qr K^(h)T estimates KV
// importance and B_c^(h) are the essential KVs; "APB-V ..." (pith.science
// review), "What carries the argument": each context block is compressed to
// its top-lp key-value pairs ranked by Q_qr K^T and gathered by later hosts.
//
// One thread-block cluster of nc CTAs (4 or 8, chosen at launch so that the
// grid fits the GPU in one wave when it can) per (block h < V-1, KV head) (all such
// blocks, or those a host mask selects),
// for blocks of up to kCompressMaxBlock keys:
//   1. each CTA sums a slice of the query block's (row, head) pairs of the KV
//      group; the slices are added in rank order through distributed shared
//      memory, so every CTA holds the same qsum = scale * sum q;
//   2. each CTA streams its 1/nc slice of K^(h) once (16-byte
//      loads, the first ones issued before step 1) and turns the scores into
//      order-preserving 32-bit keys (the scores are also written out); it
//      then copies its slice's keys into every CTA of the cluster, so that
//      after one cluster barrier each CTA holds the whole block's keys;
//   3. each CTA runs the same MSB-first radix select over the block's keys
//      locally (block barriers only): the threshold key T and the number of
//      copies of T to keep (lower indices first);
//   4. the keys of earlier slices give the CTA its starting rank; a scan in
//      index order ranks its own kept keys; it writes their indices and
//      copies their K and V rows to the passing buffer.
// After step 2's barrier no CTA touches another's shared memory, so CTAs
// leave independently.
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
static_assert(kCompressMaxBlock <= 65536, "kept keys pack their block index and rank in 16 bits each");

// Scratch shared by two phases: the query sum's per-warp partials (step 1,
// kCompressWarps x 128 floats at most) and the radix select's per-warp
// histograms (step 3, kCompressWarps x 256 counts).
constexpr int kCompressScratchBytes = kCompressWarps * 256 * 4;

// Dynamic shared memory of a launch with clusters of nc CTAs whose longest
// compressed block has lmax keys: every key of the block, this CTA's kept
// keys (block index and rank packed in 32 bits; at most one slice), then the
// scratch.
__host__ __device__ constexpr int compress_smem_bytes(int lmax, int nc) {
  return 4 * ((lmax + 3) / 4 * 4) + 4 * (((lmax + nc - 1) / nc + 3) / 4 * 4) + kCompressScratchBytes;
}

struct CompressParams {
  int32_t start[kMaxV];   // first sequence row of block h
  int32_t L[kMaxV];
  int32_t k[kMaxV];       // lp_eff(h)
  int32_t poff[kMaxV + 1];
  int32_t Hq, Hkv, G, lq, lp;
  int32_t lmax;           // longest compressed block (sizes the shared key array)
  int64_t qs, la, score_cols;
  float scale;
  // merge counters of the attention launch that follows (zeroed here so that
  // no separate launch is needed); null when called on its own
  int32_t* merge_count;
  int32_t n_merge;
  int32_t blk[kMaxV];     // the compressed blocks, one per grid row (all h < V-1, or a host mask's)
};

template <int D>
__global__ void __launch_bounds__(kCompressThreads, 2)
    compress_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                    const __nv_bfloat16* __restrict__ V, float* __restrict__ qsum_out,
                    float* __restrict__ scores, int32_t* __restrict__ idx,
                    __nv_bfloat16* __restrict__ Kp, __nv_bfloat16* __restrict__ Vp,
                    const __grid_constant__ CompressParams p) {
  constexpr int kParts = D / 8;                           // 16-byte chunks per row
  constexpr int kRowsPerIter = kCompressThreads / kParts;
  extern __shared__ uint8_t dsm[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(dsm);                                  // [L] whole block
  uint32_t* sel = reinterpret_cast<uint32_t*>(dsm + 4 * ((p.lmax + 3) / 4 * 4));    // [slice]: (rank << 16) | j
  const int nc = static_cast<int>(gridDim.x);   // the cluster: one per (block, KV head)
  uint8_t* scratch = reinterpret_cast<uint8_t*>(sel + ((p.lmax + nc - 1) / nc + 3) / 4 * 4);
  float (*part_q)[D] = reinterpret_cast<float (*)[D]>(scratch);              // step 1
  uint32_t (*hist)[256] = reinterpret_cast<uint32_t (*)[256]>(scratch);     // step 3, one per warp
  __shared__ float slice_q[D];
  __shared__ float qs_full[D];
  __shared__ uint32_t tot[256];
  __shared__ uint64_t warp_tot[32];
  __shared__ uint32_t s_prefix, s_k;
  __shared__ uint64_t s_before;
  __shared__ int s_nsel;

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
  const int j0 = static_cast<int>((static_cast<int64_t>(L) * rank) / nc);
  const int j1 = static_cast<int>((static_cast<int64_t>(L) * (rank + 1)) / nc);
  const int n = j1 - j0;   // keys of this CTA's slice
  const int pc = tid % kParts, lr = tid / kParts;

  // K loads of the slice, four rows per thread in flight; the first group is
  // issued before the query sum so that its latency overlaps step 1
  constexpr int kU = 4;
  constexpr int kStep = kRowsPerIter * kU;
  const int64_t row0 = p.start[h] + j0;
  auto load = [&](int base, uint4 (&raw)[kU]) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int jj = base + u * kRowsPerIter + lr;
      raw[u] = jj < n ? __ldcs(reinterpret_cast<const uint4*>(K + ((row0 + jj) * p.Hkv + kv) * D + pc * 8))
                      : make_uint4(0, 0, 0, 0);
    }
  };
  uint4 cur[kU], nxt[kU];
  load(0, nxt);

  // ---- 1. qsum for this KV group
  {
    const int total = p.lq * p.G;
    const int r0 = static_cast<int>((static_cast<int64_t>(total) * rank) / nc);
    const int r1 = static_cast<int>((static_cast<int64_t>(total) * (rank + 1)) / nc);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    // four (row, head) pairs per thread in flight at once
    for (int rb = r0 + lr; rb < r1; rb += 4 * kRowsPerIter) {
      uint4 raw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int rr = rb + u * kRowsPerIter;
        const int i = rr / p.G, g = kv * p.G + rr % p.G;
        raw[u] = rr < r1 ? *reinterpret_cast<const uint4*>(Q + ((p.qs + i) * p.Hq + g) * D + pc * 8)
                         : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const __nv_bfloat16* v = reinterpret_cast<const __nv_bfloat16*>(&raw[u]);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += __bfloat162float(v[e]);
      }
    }
    // lanes l and l ^ 16 hold the same column chunk (for D = 128); add them,
    // then the warps' sums in warp order
#pragma unroll
    for (int off = kParts; off < 32; off <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    if (lane < kParts)
#pragma unroll
      for (int e = 0; e < 8; ++e) part_q[warp][pc * 8 + e] = acc[e];
    __syncthreads();
    for (int c = tid; c < D; c += kCompressThreads) {
      float s = 0.f;
      for (int w = 0; w < kCompressWarps; ++w) s += part_q[w][c];
      slice_q[c] = s;
    }
    cluster.sync();
    for (int c = tid; c < D; c += kCompressThreads) {
      float s = 0.f;
      for (int r = 0; r < nc; ++r) s += cluster.map_shared_rank(slice_q, r)[c];
      qs_full[c] = s * p.scale;
      if (h == 0 && rank == 0) qsum_out[kv * D + c] = s * p.scale;
    }
    __syncthreads();
  }

  // ---- 2. scores of this slice (one pass over K), then every CTA gets them
  {
    float q8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) q8[e] = qs_full[pc * 8 + e];
    float* srow = scores + static_cast<int64_t>(kv) * p.score_cols + (p.start[h] - p.la) + j0;
    for (int base = 0; base < n; base += kStep) {
#pragma unroll
      for (int u = 0; u < kU; ++u) cur[u] = nxt[u];
      if (base + kStep < n) load(base + kStep, nxt);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int jj = base + u * kRowsPerIter + lr;
        const __nv_bfloat16* v = reinterpret_cast<const __nv_bfloat16*>(&cur[u]);
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) dot = fmaf(__bfloat162float(v[e]), q8[e], dot);
#pragma unroll
        for (int off = kParts / 2; off >= 1; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        if (pc == 0 && jj < n) {
          srow[jj] = dot;
          keys[j0 + jj] = order_key(dot);
        }
      }
    }
  }
  __syncthreads();
  for (int r = 1; r < nc; ++r) {   // this slice's keys into every other CTA
    uint32_t* dst = cluster.map_shared_rank(keys, (rank + r) % nc);
    for (int i = tid; i < n; i += kCompressThreads) dst[j0 + i] = keys[j0 + i];
  }
  cluster.sync();   // every CTA holds the block's keys; the last access to peer shared memory

  // ---- 3. radix select of the kk largest keys, locally
  uint32_t T = 0, keq = 0;
  const bool all = kk >= L;
  if (!all && kk > 0) {
    if (tid == 0) {
      s_prefix = 0;
      s_k = static_cast<uint32_t>(kk);
    }
    uint32_t mask = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < kCompressWarps * 256; i += kCompressThreads) (&hist[0][0])[i] = 0;
      __syncthreads();
      const uint32_t prefix = s_prefix;
      for (int i = tid; i < L; i += kCompressThreads) {
        const uint32_t key = keys[i];
        if ((key & mask) == prefix) atomicAdd(&hist[warp][(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      for (int b = tid; b < 256; b += kCompressThreads) {
        uint32_t sum = 0;
#pragma unroll
        for (int w = 0; w < kCompressWarps; ++w) sum += hist[w][b];
        tot[b] = sum;
      }
      __syncthreads();
      if (tid < 32) {
        uint32_t c[8], t8 = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          c[b] = tot[tid * 8 + b];
          t8 += c[b];
        }
        uint32_t x = t8;   // inclusive suffix sum over lanes
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t y = __shfl_down_sync(0xffffffffu, x, off);
          if (tid + off < 32) x += y;
        }
        uint32_t running = x - t8;   // count in higher bins
        const uint32_t need = s_k;
#pragma unroll
        for (int b = 7; b >= 0; --b) {
          if (running < need && running + c[b] >= need) {
            s_prefix = prefix | (static_cast<uint32_t>(tid * 8 + b) << shift);
            s_k = need - running;
          }
          running += c[b];
        }
      }
      __syncthreads();
      mask |= 0xFFu << shift;
    }
    T = s_prefix;
    keq = s_k;
  }

  // ---- 4. ranks in index order; write idx; gather rows
  // (eq << 32) | gt counted over the keys of earlier slices
  if (!all && kk > 0) {
    uint32_t gt = 0, eq = 0;
    for (int i = tid; i < j0; i += kCompressThreads) {
      gt += keys[i] > T;
      eq += keys[i] == T;
    }
    const uint64_t part = block_exclusive_scan_u64((static_cast<uint64_t>(eq) << 32) | gt, warp_tot);
    if (tid == kCompressThreads - 1) s_before = part + ((static_cast<uint64_t>(eq) << 32) | gt);
    __syncthreads();
  }
  const uint64_t before = (!all && kk > 0) ? s_before : 0;
  const int chunk = (n + kCompressThreads - 1) / kCompressThreads;
  const int i0 = min(n, tid * chunk), i1 = min(n, i0 + chunk);
  uint32_t gt = 0, eq = 0;
  if (!all && kk > 0) {
    for (int i = j0 + i0; i < j0 + i1; ++i) {
      gt += keys[i] > T;
      eq += keys[i] == T;
    }
  }
  const uint64_t pre = block_exclusive_scan_u64((static_cast<uint64_t>(eq) << 32) | gt, warp_tot);
  // counts before this thread's chunk over the whole block, and this thread's
  // first slot in the CTA's list of kept keys
  uint32_t gt_pre = static_cast<uint32_t>(before + pre);
  uint32_t eq_pre = static_cast<uint32_t>((before + pre) >> 32);
  const uint32_t eq_cta0 = static_cast<uint32_t>(before >> 32);     // T-copies in earlier slices
  const uint32_t eq_keep_cta = keq > eq_cta0 ? keq - eq_cta0 : 0u;  // still to keep from here on
  uint32_t lsel = all ? static_cast<uint32_t>(i0)
                      : static_cast<uint32_t>(pre) + min(static_cast<uint32_t>(pre >> 32), eq_keep_cta);
  int32_t* out = idx + (static_cast<int64_t>(h) * p.Hkv + kv) * p.lp;
  if (kk > 0) {
    for (int i = i0; i < i1; ++i) {
      const uint32_t key = keys[j0 + i];
      int pos = -1;
      if (all) {
        pos = j0 + i;
      } else if (key > T) {
        pos = static_cast<int>(gt_pre + min(eq_pre, keq));
        ++gt_pre;
      } else if (key == T) {
        if (eq_pre < keq) pos = static_cast<int>(gt_pre + eq_pre);
        ++eq_pre;
      }
      if (pos >= 0) {
        out[pos] = j0 + i;
        sel[lsel] = (static_cast<uint32_t>(pos) << 16) | static_cast<uint32_t>(j0 + i);
        ++lsel;
      }
    }
  }
  if (rank == 0)
    for (int t = kk + tid; t < p.lp; t += kCompressThreads) out[t] = -1;
  if (tid == kCompressThreads - 1) s_nsel = static_cast<int>(lsel);   // = the CTA's kept keys
  __syncthreads();
  const int nsel = s_nsel;
  // gather: kParts lanes per row (16 lanes x 16 B = 256 B for d = 128)
  {
    const int64_t off = p.poff[h];
    // four rows per thread group in flight at once
    for (int sb = lr; sb < nsel; sb += 4 * kRowsPerIter) {
      uint4 kx[4], vx[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int s = sb + u * kRowsPerIter;
        if (s < nsel) {
          const int64_t src = static_cast<int64_t>(p.start[h]) + (sel[s] & 0xFFFFu);
          kx[u] = *reinterpret_cast<const uint4*>(K + (src * p.Hkv + kv) * D + pc * 8);
          vx[u] = *reinterpret_cast<const uint4*>(V + (src * p.Hkv + kv) * D + pc * 8);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int s = sb + u * kRowsPerIter;
        if (s < nsel) {
          const int64_t dst = off + (sel[s] >> 16);
          *reinterpret_cast<uint4*>(Kp + (dst * p.Hkv + kv) * D + pc * 8) = kx[u];
          *reinterpret_cast<uint4*>(Vp + (dst * p.Hkv + kv) * D + pc * 8) = vx[u];
        }
      }
    }
  }
}

}  // namespace spava
