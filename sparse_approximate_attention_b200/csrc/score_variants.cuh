// Selector variants, second pass: per key, the sum over a set of scoring rows
// of softmax probabilities whose normalisers (lse) the first pass computed.
//   softmax: rows = the query block's rows (all query heads of the KV head),
//            normalised over block h's keys;
//   context: rows = block h's own rows, causal within the block (a row sees
//            the block's keys up to itself) -- the review's oracle selector
//            ("APB-V ..." pith.science review, major comment 1 and "What would
//            settle it": cumulative attention from all tokens of the block).
// score_j = sum_{rows r, heads g of the KV head} exp(scale <q_rg, k_j> - lse_rg).
//
// One CTA per (128-key tile of a block h < V-1, KV head).  S^T = K_tile Q^T
// is computed on the tensor cores (M = 128 keys, N = 128 rows per row tile,
// K = head_dim) into one of two TMEM buffers while the four consumer warps,
// one thread per key (its TMEM lane), turn the previous row tile into
// probabilities and add them up.  256 threads: warp 0 TMA producer, warp 1
// MMA issuer and TMEM owner, warps 4-7 consumers.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "plan.hpp"
#include "ptx.cuh"

namespace spava {

enum : int32_t { kScoreLinear = 0, kScoreSoftmax = 1, kScoreContext = 2 };

struct ColsumParams {
  CUtensorMap tm_q, tm_k;   // [rows, heads, d] bf16, boxes of 128 rows x 64 columns
  float* scores;            // [Hkv, score_cols]
  const float* lse;         // softmax: [V, Hq, lq] (block h's query partials); context: [Hq, n]
  int32_t kind, Hq, G, lq, qs, n, la, V;
  int64_t score_cols;
  float scale_log2;
  int32_t nblocks;                 // V - 1
  int32_t start[kMaxV], L[kMaxV];  // blocks
  int32_t tile0[kMaxV + 1];        // first key tile of each block in the grid's x dimension
};

template <int D>
struct ColsumCfg {
  static constexpr int kSlabs = D / 64;
  static constexpr int kSlabBytes = 128 * 128;
  static constexpr int kTileBytes = kSlabs * kSlabBytes;
  static constexpr int kStages = 2;   // Q row tiles in flight
  static constexpr int kOffK = 0;
  static constexpr int kOffQ = kTileBytes;
  static constexpr int kOffLse = kOffQ + kStages * kTileBytes;   // [2][128] f32
  static constexpr int kOffBar = kOffLse + 2 * 128 * 4;
  // barriers: Kfull, Qfull[2], Qempty[2], Sfull[2], Sfree[2], Fin
  static constexpr int kNumBars = 1 + 2 * kStages + 4 + 1;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 32 + 1024;   // tmem slot, abort flag, status[4]
  static constexpr int kThreads = 256;
};

template <int D>
__global__ void __launch_bounds__(ColsumCfg<D>::kThreads, 1) colsum_kernel(const __grid_constant__ ColsumParams p) {
  using C = ColsumCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t sbase = (raw_base + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_base);
  const uint32_t sK = sbase + C::kOffK, sQ = sbase + C::kOffQ;
  float* lse_s = reinterpret_cast<float*>(smem + C::kOffLse);
  const uint32_t bar0 = sbase + C::kOffBar;
  const uint32_t BAR_K = bar0;
  auto BAR_QF = [&](int s) { return bar0 + 8u * (1 + s); };
  auto BAR_QE = [&](int s) { return bar0 + 8u * (3 + s); };
  auto BAR_SF = [&](int b) { return bar0 + 8u * (5 + b); };
  auto BAR_SE = [&](int b) { return bar0 + 8u * (7 + b); };
  const uint32_t BAR_FIN = bar0 + 8u * 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kv = blockIdx.y;
  int h = 0;
  while (h + 1 < p.nblocks && p.tile0[h + 1] <= static_cast<int>(blockIdx.x)) ++h;
  const int kt = static_cast<int>(blockIdx.x) - p.tile0[h];
  const int Lh = p.L[h], s0 = p.start[h];
  const int key0 = s0 + kt * 128;                 // first key (sequence row) of the tile
  // scoring rows: softmax -> the query block; context -> block h from this tile on
  const bool ctx = p.kind == kScoreContext;
  const int rbase = ctx ? key0 : p.qs;
  const int rend = ctx ? s0 + Lh : p.qs + p.lq;
  const int nrt = (rend - rbase + 127) / 128;     // row tiles per query head
  const int ntiles = nrt * p.G;                   // row tiles over the KV head's query heads
  auto tile_rows = [&](int t, int* g, int* r0) {
    *g = kv * p.G + t / nrt;
    *r0 = rbase + (t % nrt) * 128;
  };

  if (threadIdx.x == 0) {
    mbar_init(BAR_K, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR_QF(s), 1);
      mbar_init(BAR_QE(s), 1);
      mbar_init(BAR_SF(s), 1);
      mbar_init(BAR_SE(s), 4);   // the four consumer warps
    }
    mbar_init(BAR_FIN, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(BAR_K, C::kTileBytes);
      for (int sl = 0; sl < C::kSlabs; ++sl)
        tma_load_3d(sK + sl * C::kSlabBytes, &p.tm_k, BAR_K, sl * 64, kv, key0);
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int st = t & 1;
        if (t >= 2 && !mbar_wait(BAR_QE(st), ((t >> 1) - 1) & 1, abort_flag)) break;
        int g, r0;
        tile_rows(t, &g, &r0);
        mbar_arrive_expect_tx(BAR_QF(st), C::kTileBytes);
        for (int sl = 0; sl < C::kSlabs; ++sl)
          tma_load_3d(sQ + st * C::kTileBytes + sl * C::kSlabBytes, &p.tm_q, BAR_QF(st), sl * 64, g, r0);
        issued = t + 1;
      }
      if (*abort_flag) {   // let copies already in flight land before the CTA exits
        mbar_wait_drain(BAR_K, 0);
        for (int t = max(0, issued - 2); t < issued; ++t) mbar_wait_drain(BAR_QF(t & 1), (t >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
      auto desc = [](uint32_t lo) -> uint64_t { return (static_cast<uint64_t>(kDescHi) << 32) | lo; };
      const uint32_t k_lo = (sK >> 4) | (1u << 16);
      const uint32_t q_lo = (sQ >> 4) | (1u << 16);
      bool ok = mbar_wait(BAR_K, 0, abort_flag);
      for (int t = 0; ok && t < ntiles; ++t) {
        const int st = t & 1;
        ok = mbar_wait(BAR_QF(st), (t >> 1) & 1, abort_flag);
        if (ok && t >= 2) ok = mbar_wait(BAR_SE(st), ((t >> 1) - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qb = q_lo + ((st * C::kTileBytes) >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * C::kSlabBytes + (k & 3) * 32) >> 4;
          mma_ss(tmem + 128u * st, desc(k_lo + off), desc(qb + off), kIdesc, k > 0 ? 1u : 0u);
        }
        mma_commit(BAR_SF(st));
        mma_commit(BAR_QE(st));
      }
      mma_commit(BAR_FIN);
      mbar_wait_drain(BAR_FIN, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ consumers: one thread per key
    const int q = warp & 3;
    const int key = q * 32 + lane;                 // TMEM lane = key within the tile
    const int kpos = key0 + key;                   // its sequence position
    const int c = threadIdx.x - 128;               // 0..127: the row this thread stages an lse for
    const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16);
    float acc = 0.f;
    volatile int* okx = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);   // [4] per-warp status
    // The four consumer warps meet at a named barrier (no timeout): they
    // leave the loop only together, on the status all four wrote before it.
    bool ok = true;
    for (int t = 0; t < ntiles; ++t) {
      const int b = t & 1;
      int g, r0;
      tile_rows(t, &g, &r0);
      {   // lse of this tile's rows, log2 units; rows past the end contribute nothing
        const int r = r0 + c;
        float v = INFINITY;
        if (r < rend) v = (ctx ? p.lse[static_cast<int64_t>(g) * p.n + r]
                               : p.lse[(static_cast<int64_t>(h) * p.Hq + g) * p.lq + (r - p.qs)]) *
                          1.44269504088896340736f;
        lse_s[b * 128 + c] = v;
      }
      const bool okw = __all_sync(0xffffffffu, mbar_wait(BAR_SF(b), (t >> 1) & 1, abort_flag));
      if (lane == 0) okx[q] = okw ? 1 : 0;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      ok = okx[0] && okx[1] && okx[2] && okx[3];
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        tmem_ld32(tq + 128u * b + cc * 32, r);
        tmem_wait_ld();
        if (cc == 3) {   // S^T of this buffer is in registers: let the MMA reuse it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR_SE(b));
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = cc * 32 + e;
          // causal (context rows): row r0 + col sees this key only from its own position on
          const bool vis = !ctx || r0 + col >= kpos;
          const float x = __uint_as_float(r[e]) * p.scale_log2 - lse_s[b * 128 + col];
          acc += vis ? ex2_approx(x) : 0.f;
        }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");   // lse_s and the status are rewritten next
    }
    if (ok && key < Lh - kt * 128) p.scores[static_cast<int64_t>(kv) * p.score_cols + (s0 - p.la) + kt * 128 + key] = acc;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace spava
