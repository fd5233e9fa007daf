// Variable-segment causal attention on tcgen05 / TMEM with TMA-fed tiles.
//
// One CTA computes one 128-row tile of one query head.  Its keys are a list
// of up to three segments (rows of K/V or of the passing buffer Kp/Vp), which
// covers every row kind of the layer in a single launch:
//   anchor rows            : causal over B_a
//   context rows of host h : B_a, Kp rows of hosts < h, causal B^(h)
//                            ("APB-V ..." pith.science review, minor comment
//                            2: Eq. 4 key list [K_a, K_p, K^(h)])
//   query rows, host h     : B^(h) (host 0 also B_a and causal B_qr); written
//                            as a partial with its lse for the merge
//                            ("Spava ..." sciencestack.ai, Fig. 3 fused
//                            context and query forward).
// The launch's CTAs are ordered longest key list first (Fig. 4, attention
// load balancing).
//
// Warp roles (192 threads):
//   warp 0     TMA producer: Q once, then K and V tiles into a ring of stages
//   warp 1     TMEM owner and MMA issuer: S = Q K^T into one of two TMEM
//              buffers, then O += P V with P read from TMEM
//   warps 2-5  softmax: one thread per query row, online softmax in the
//              exp2 domain with a lazy rescale of O (only when the running
//              max grows by more than 2^8), P written back to TMEM as bf16
// TMEM columns: O [0, D), S/P buffer b at [128 + 128 b, 256 + 128 b).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "plan.hpp"
#include "ptx.cuh"

namespace spava {

struct AttnParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_kp, tm_vp;
  __nv_bfloat16* O;
  float* lse;
  float* O_part;
  float* lse_part;
  int32_t n, Hq, G, lq, qs;
  float scale_log2;
  int32_t nregions, nitems;
  Region regions[kMaxRegions];
  uint32_t items[kMaxItems];
};
static_assert(sizeof(AttnParams) <= 32764, "kernel parameter block too large");

template <int D>
struct AttnCfg {
  static constexpr int kSlabs = D / 64;                  // 128-byte-wide column slabs
  static constexpr int kSlabBytes = 128 * 128;           // 128 rows x 128 B
  static constexpr int kTileBytes = kSlabs * kSlabBytes;
  static constexpr int kKStages = (D == 128) ? 3 : 4;    // K ring (released after S = Q K^T)
  static constexpr int kVStages = (D == 128) ? 2 : 4;    // V ring (released after O += P V)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  // barriers: Q, Kfull[KS], Kempty[KS], Vfull[VS], Vempty[VS], Sfull[2], Pfull[2], Odone, Fin
  static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 2 + 2 + 1 + 1;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;   // + slack for 1 KB alignment
  static constexpr int kThreads = 192;
  static constexpr uint32_t kTmemCols = 512;
};
static_assert(AttnCfg<128>::kSmemBytes <= 232448, "shared memory budget");
static_assert(AttnCfg<64>::kSmemBytes <= 232448, "shared memory budget");

template <int D>
__global__ void __launch_bounds__(AttnCfg<D>::kThreads, 1)
    attn_kernel(const __grid_constant__ AttnParams p) {
  using C = AttnCfg<D>;
  constexpr int KS = C::kKStages, VS = C::kVStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t sbase = (raw_base + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_base);
  const uint32_t sQ = sbase + C::kOffQ, sK = sbase + C::kOffK, sV = sbase + C::kOffV;
  const uint32_t bar0 = sbase + C::kOffBar;
  const uint32_t BAR_Q = bar0;
  auto BAR_KF = [&](int s) { return bar0 + 8u * (1 + s); };
  auto BAR_KE = [&](int s) { return bar0 + 8u * (1 + KS + s); };
  auto BAR_VF = [&](int s) { return bar0 + 8u * (1 + 2 * KS + s); };
  auto BAR_VE = [&](int s) { return bar0 + 8u * (1 + 2 * KS + VS + s); };
  auto BAR_SF = [&](int b) { return bar0 + 8u * (1 + 2 * KS + 2 * VS + b); };
  auto BAR_PF = [&](int b) { return bar0 + 8u * (3 + 2 * KS + 2 * VS + b); };
  const uint32_t BAR_OD = bar0 + 8u * (5 + 2 * KS + 2 * VS);
  const uint32_t BAR_FIN = bar0 + 8u * (6 + 2 * KS + 2 * VS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t item = p.items[blockIdx.x / p.Hq];
  const int head = blockIdx.x % p.Hq;
  const Region& R = p.regions[item >> 20];
  const int tile = static_cast<int>(item & 0xFFFFFu);
  const int kv = head / p.G;
  const int row0 = R.row_start + tile * kBM;
  const int rows_valid = min(kBM, R.nrows - tile * kBM);
  const int r_last = row0 + rows_valid - 1;
  const int nseg = R.nseg;
  int nt[kMaxSegs];
  int ntiles = 0;
#pragma unroll
  for (int s = 0; s < kMaxSegs; ++s) {
    int vis = 0;
    if (s < nseg) {
      const Seg& sg = R.seg[s];
      vis = sg.causal ? max(0, min(sg.len, r_last - sg.start + 1)) : sg.len;
    }
    nt[s] = (vis + kBN - 1) / kBN;
    ntiles += nt[s];
  }
  // Walks the key tiles in order: segment s, tile kt within it.
  struct TileIter {
    int s, kt;
  };
  auto iter_begin = [&]() {
    TileIter it{0, 0};
    while (it.s < nseg && nt[it.s] == 0) ++it.s;
    return it;
  };
  auto iter_next = [&](TileIter& it) {
    if (++it.kt == nt[it.s]) {
      it.kt = 0;
      ++it.s;
      while (it.s < nseg && nt[it.s] == 0) ++it.s;
    }
  };

  if (threadIdx.x == 0) {
    mbar_init(BAR_Q, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(BAR_KF(s), 1);
      mbar_init(BAR_KE(s), 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(BAR_VF(s), 1);
      mbar_init(BAR_VE(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR_SF(b), 1);
      mbar_init(BAR_PF(b), 128);
    }
    mbar_init(BAR_OD, 1);
    mbar_init(BAR_FIN, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // K runs one tile ahead of V, matching the order the MMA consumes them
    // (S_j = Q K_j^T is issued before O += P_{j-1} V_{j-1}).
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(BAR_Q, C::kTileBytes);
      for (int sl = 0; sl < C::kSlabs; ++sl)
        tma_load_3d(sQ + sl * C::kSlabBytes, &p.tm_q, BAR_Q, sl * 64, head, row0);
      int k_issued = 0, v_issued = 0;
      TileIter ik = iter_begin(), iv = iter_begin();
      for (int j = 0; j <= ntiles; ++j) {
        if (j < ntiles) {
          const int st = j % KS;
          if (j >= KS && !mbar_wait(BAR_KE(st), ((j / KS) - 1) & 1, abort_flag)) break;
          const Seg& sg = R.seg[ik.s];
          const CUtensorMap* tk = sg.src == kSrcMain ? &p.tm_k : &p.tm_kp;
          const int krow = sg.start + ik.kt * kBN;
          mbar_arrive_expect_tx(BAR_KF(st), C::kTileBytes);
          for (int sl = 0; sl < C::kSlabs; ++sl)
            tma_load_3d(sK + st * C::kTileBytes + sl * C::kSlabBytes, tk, BAR_KF(st), sl * 64, kv, krow);
          k_issued = j + 1;
          iter_next(ik);
        }
        if (j >= 1) {
          const int i = j - 1, st = i % VS;
          if (i >= VS && !mbar_wait(BAR_VE(st), ((i / VS) - 1) & 1, abort_flag)) break;
          const Seg& sg = R.seg[iv.s];
          const CUtensorMap* tv = sg.src == kSrcMain ? &p.tm_v : &p.tm_vp;
          const int krow = sg.start + iv.kt * kBN;
          mbar_arrive_expect_tx(BAR_VF(st), C::kTileBytes);
          for (int sl = 0; sl < C::kSlabs; ++sl)
            tma_load_3d(sV + st * C::kTileBytes + sl * C::kSlabBytes, tv, BAR_VF(st), sl * 64, kv, krow);
          v_issued = i + 1;
          iter_next(iv);
        }
      }
      if (*abort_flag) {   // let copies already in flight land before the CTA exits
        mbar_wait_drain(BAR_Q, 0);
        for (int j = max(0, k_issued - KS); j < k_issued; ++j) mbar_wait_drain(BAR_KF(j % KS), (j / KS) & 1);
        for (int j = max(0, v_issued - VS); j < v_issued; ++j) mbar_wait_drain(BAR_VF(j % VS), (j / VS) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kBN, false, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
      const uint32_t tO = tmem;
      auto issue_pv = [&](int i) -> bool {
        const int st = i % VS, b = i & 1;
        if (!mbar_wait(BAR_PF(b), (i >> 1) & 1, abort_flag)) return false;
        if (!mbar_wait(BAR_VF(st), (i / VS) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t tP = tmem + 128u + 128u * b;
#pragma unroll
        for (int k = 0; k < kBN / 16; ++k) {
          const uint64_t bdesc = sw128_desc(sV + st * C::kTileBytes + k * 2048, C::kSlabBytes, 1024);
          mma_ts(tO, tP + k * 8, bdesc, kIdescPV, (i > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(BAR_OD);
        mma_commit(BAR_VE(st));
        return true;
      };
      bool ok = mbar_wait(BAR_Q, 0, abort_flag);
      for (int j = 0; ok && j < ntiles; ++j) {
        const int st = j % KS, b = j & 1;
        ok = mbar_wait(BAR_KF(st), (j / KS) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tmem + 128u + 128u * b;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const int sl = k >> 2, off = (k & 3) * 32;
          const uint64_t adesc = sw128_desc(sQ + sl * C::kSlabBytes + off, 16, 1024);
          const uint64_t bdesc = sw128_desc(sK + st * C::kTileBytes + sl * C::kSlabBytes + off, 16, 1024);
          mma_ss(tS, adesc, bdesc, kIdescQK, k > 0 ? 1u : 0u);
        }
        mma_commit(BAR_SF(b));
        mma_commit(BAR_KE(st));
        if (j > 0) ok = issue_pv(j - 1);
      }
      if (ok && ntiles > 0) issue_pv(ntiles - 1);
      mma_commit(BAR_FIN);   // every MMA issued above has finished once this lands
      mbar_wait_drain(BAR_FIN, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int rit = q * 32 + lane;          // row in tile
    const int row = row0 + rit;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const float sl2 = p.scale_log2;
    float m = -INFINITY;   // running max of the scaled logits, log2 units
    float l = 0.f;
    bool ok = true;
    int s = 0, kt = 0;
    while (s < nseg && nt[s] == 0) ++s;
    for (int j = 0; j < ntiles; ++j) {
      const int b = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(BAR_SF(b), (j >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float x[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + 128u + 128u * b + c * 32, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(r[e]);
      }
      tmem_wait_ld();
      const Seg& sg = R.seg[s];
      int lim = sg.len;
      if (sg.causal) lim = min(lim, row - sg.start + 1);
      const int nvalid = lim - kt * kBN;
      if (nvalid < kBN) {
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c >= nvalid) x[c] = -INFINITY;
      }
      float mx = x[0];
#pragma unroll
      for (int c = 1; c < kBN; ++c) mx = fmaxf(mx, x[c]);
      mx *= sl2;
      const bool grow = mx > m + 8.0f;
      const float m_new = grow ? mx : m;
      const float alpha = grow ? ex2_approx(m - m_new) : 1.0f;
      const float neg = -m_new;
      uint32_t pk[kBN / 2];
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < kBN; c += 2) {
        const float p0 = ex2_approx(fmaf(x[c], sl2, neg));
        const float p1 = ex2_approx(fmaf(x[c + 1], sl2, neg));
        sum += p0 + p1;
        pk[c / 2] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + sum;
      m = m_new;
      if (j > 0) {
        // O += P_{j-1} V_{j-1} must be complete before O is rescaled and
        // before P_j may be consumed; waiting every tile keeps the barrier
        // within one phase of this waiter.
        ok = __all_sync(0xffffffffu, mbar_wait(BAR_OD, (j - 1) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(taddr + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(taddr + c * 32, r);
          }
        }
      }
      {
        uint32_t r0[32], r1[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          r0[e] = pk[e];
          r1[e] = pk[32 + e];
        }
        tmem_st32(taddr + 128u + 128u * b, r0);
        tmem_st32(taddr + 128u + 128u * b + 32, r1);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR_PF(b));
      if (++kt == nt[s]) {
        kt = 0;
        ++s;
        while (s < nseg && nt[s] == 0) ++s;
      }
    }
    if (ok && ntiles > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(BAR_OD, (ntiles - 1) & 1, abort_flag));
    }
    if (ok) {
      tc_fence_after();
      const bool valid = rit < rows_valid;
      const float inv_l = 1.0f / l;
      const float lse_nat = (m + __log2f(l)) * 0.69314718055994530942f;
      if (R.out_kind == kOutRows) {
        __nv_bfloat16* dst = p.O + (static_cast<int64_t>(row) * p.Hq + head) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(r[e + 0]) * inv_l, __uint_as_float(r[e + 1]) * inv_l);
              v.y = pack_bf16x2(__uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
              v.z = pack_bf16x2(__uint_as_float(r[e + 4]) * inv_l, __uint_as_float(r[e + 5]) * inv_l);
              v.w = pack_bf16x2(__uint_as_float(r[e + 6]) * inv_l, __uint_as_float(r[e + 7]) * inv_l);
              *reinterpret_cast<uint4*>(dst + c * 32 + e) = v;
            }
          }
        }
        if (valid) p.lse[static_cast<int64_t>(head) * p.n + row] = lse_nat;
      } else {
        const int qi = row - p.qs;
        float* dst = p.O_part + ((static_cast<int64_t>(R.host) * p.lq + qi) * p.Hq + head) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              float4 v = make_float4(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l,
                                     __uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
              *reinterpret_cast<float4*>(dst + c * 32 + e) = v;
            }
          }
        }
        if (valid) p.lse_part[(static_cast<int64_t>(R.host) * p.Hq + head) * p.lq + qi] = lse_nat;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace spava
