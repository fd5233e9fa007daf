// Variable-segment causal attention on tcgen05 / TMEM with TMA-fed tiles.
//
// One CTA computes two consecutive 128-row tiles (Q0, Q1) of one query head
// that share one key list.  The key list is up to three segments (rows of
// K/V or of the passing buffer Kp/Vp), which covers every row kind of the
// layer in a single launch:
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
// Warp roles (384 threads, three warpgroups; the first gives registers to the
// other two with setmaxnreg):
//   warp 0     TMA producer: Q0 and Q1 once, then K and V tiles into separate
//              rings (K runs one tile ahead of V, the order the MMAs use them)
//   warp 1     TMEM owner and MMA issuer (warp-wide loop, one elected lane
//              issues).  Per key tile j:
//              S0 = Q0 K_j^T, O1 += P1 V_{j-1}, S1 = Q1 K_j^T, O0 += P0 V_j,
//              so the tensor pipe works on one tile while the other tile's
//              softmax runs
//   warps 2-3  idle (they complete warpgroup 0)
//   warps 4-7  softmax of Q0, warps 8-11 softmax of Q1: one thread per row,
//              online softmax in the exp2 domain (exponentials on MUFU,
//              packed f32x2 arithmetic elsewhere), lazy rescale of O (only
//              when the row max grows by more than 2^8), P written back to
//              TMEM as bf16 over S
// TMEM columns: O0 [0, D), O1 [128, 128 + D), S0/P0 [256, 384), S1/P1 [384, 512).
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
  // Fused merge of the query partials: one arrival counter per (query tile
  // pair, query head), zero before the launch; the last of the V partial
  // CTAs of a pair merges it into the query rows of O and lse.  Null: the
  // partials are left for a separate merge.
  int32_t* merge_count;
  int32_t V;
  // 1 when launched as a programmatic dependent of the compression kernel:
  // the passing buffer and the merge counters are read only after
  // griddepcontrol.wait.
  int32_t pdl_wait;
  // Bounded waits: every wait gives up after wait_limit_ns (4 s in the
  // layer).  skip_k_tile >= 0 (a test hook, -1 in the layer): the producer
  // does not load that key tile, so the waits for it run out and the CTA
  // takes its abort path.
  int32_t skip_k_tile;
  uint64_t wait_limit_ns;
  Region regions[kMaxRegions];
  uint32_t items[kMaxItems];   // (region << 20) | pair of 128-row tiles
};
static_assert(sizeof(AttnParams) <= 32764, "kernel parameter block too large");

template <int D>
struct AttnCfg {
  static constexpr int kSlabs = D / 64;                  // 128-byte-wide column slabs
  static constexpr int kSlabBytes = 128 * 128;           // 128 rows x 128 B
  static constexpr int kTileBytes = kSlabs * kSlabBytes;
  static constexpr int kKStages = (D == 128) ? 3 : 4;    // K ring (released after both S MMAs)
  static constexpr int kVStages = (D == 128) ? 2 : 4;    // V ring (released after both PV MMAs)
  static constexpr int kOffQ = 0;                        // Q0, Q1
  static constexpr int kOffK = 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  // barriers: Q, Kfull[KS], Kempty[KS], Vfull[VS], Vempty[VS], Sfull[2], Pfull[2][2 halves],
  // Odone[2], Fin
  static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 2 + 4 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;   // tmem slot, abort flag, merge flag; + 1 KB alignment slack
  static constexpr int kThreads = 384;
  static constexpr uint32_t kRegsLow = 56;     // warpgroup 0: producer, MMA issuer
  static constexpr uint32_t kRegsHigh = 224;   // warpgroups 1, 2: softmax
  static constexpr uint32_t kTmemCols = 512;
};
static_assert(AttnCfg<128>::kSmemBytes <= 232448, "shared memory budget");
static_assert(AttnCfg<64>::kSmemBytes <= 232448, "shared memory budget");

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Merge query rows [q0, q0 + nrows) of head g from the V partials:
// lse = log sum_h exp(lse_h), O = sum_h exp(lse_h - lse) O_h.  Eight warps,
// one row per warp at a time, D/32 columns per lane; the partials were written
// by other CTAs of this launch, so they are read from L2 (no L1 copies).
template <int D>
__device__ __forceinline__ void merge_rows(const AttnParams& p, int q0, int nrows, int g, int w8, int lane) {
  constexpr int kPer = D / 32;
  for (int r = w8; r < nrows; r += 8) {
    const int qi = q0 + r;
    const float lp = lane < p.V ? __ldcg(p.lse_part + (static_cast<int64_t>(lane) * p.Hq + g) * p.lq + qi) : -INFINITY;
    float mx = lp;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float e = lane < p.V ? __expf(lp - mx) : 0.f;
    float sum = e;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float lse_tot = mx + __logf(sum);
    const float w_mine = e / sum;          // weight of partial `lane`
    float acc[kPer];
#pragma unroll
    for (int c = 0; c < kPer; ++c) acc[c] = 0.f;
    for (int hh = 0; hh < p.V; ++hh) {
      const float w = __shfl_sync(0xffffffffu, w_mine, hh);
      const float* src = p.O_part + ((static_cast<int64_t>(hh) * p.lq + qi) * p.Hq + g) * D + lane * kPer;
      if (kPer == 4) {
        const float4 o = __ldcg(reinterpret_cast<const float4*>(src));
        acc[0] = fmaf(w, o.x, acc[0]);
        acc[1] = fmaf(w, o.y, acc[1]);
        acc[2] = fmaf(w, o.z, acc[2]);
        acc[3] = fmaf(w, o.w, acc[3]);
      } else {
        const float2 o = __ldcg(reinterpret_cast<const float2*>(src));
        acc[0] = fmaf(w, o.x, acc[0]);
        acc[1] = fmaf(w, o.y, acc[1]);
      }
    }
    __nv_bfloat16* dst = p.O + (static_cast<int64_t>(p.qs + qi) * p.Hq + g) * D + lane * kPer;
    if (kPer == 4) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
    } else {
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0], acc[1]);
    }
    if (lane == 0) p.lse[static_cast<int64_t>(g) * p.n + p.qs + qi] = lse_tot;
  }
}

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
  auto BAR_SF = [&](int t) { return bar0 + 8u * (1 + 2 * KS + 2 * VS + t); };
  auto BAR_PF = [&](int t, int half) { return bar0 + 8u * (3 + 2 * KS + 2 * VS + 2 * t + half); };
  auto BAR_OD = [&](int t) { return bar0 + 8u * (7 + 2 * KS + 2 * VS + t); };
  const uint32_t BAR_FIN = bar0 + 8u * (9 + 2 * KS + 2 * VS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t item = p.items[blockIdx.x / p.Hq];
  const int head = blockIdx.x % p.Hq;
  const Region& R = p.regions[item >> 20];
  const int pair = static_cast<int>(item & 0xFFFFFu);
  const int kv = head / p.G;
  const int row0 = R.row_start + pair * 2 * kBM;               // first row of Q0
  const int rv0 = min(kBM, R.nrows - pair * 2 * kBM);          // valid rows of Q0 (>= 1)
  const int rv1 = min(kBM, R.nrows - (pair * 2 + 1) * kBM);    // valid rows of Q1 (<= 0: none)
  const bool has1 = rv1 > 0;
  const int nseg = R.nseg;
  // Key tiles per segment.  Q0's key tiles are a prefix of Q1's: only the
  // trailing causal segment can reach further for Q1's later rows.
  int ntks[kMaxSegs];
  int nt0 = 0, ntk = 0;
#pragma unroll
  for (int s = 0; s < kMaxSegs; ++s) {
    int v0 = 0, v1 = 0;
    if (s < nseg) {
      const Seg& sg = R.seg[s];
      const int rl0 = row0 + rv0 - 1;
      const int rl1 = has1 ? row0 + kBM + rv1 - 1 : rl0;
      v0 = sg.causal ? max(0, min(sg.len, rl0 - sg.start + 1)) : sg.len;
      v1 = sg.causal ? max(0, min(sg.len, rl1 - sg.start + 1)) : sg.len;
    }
    nt0 += (v0 + kBN - 1) / kBN;
    ntks[s] = (v1 + kBN - 1) / kBN;
    ntk += ntks[s];
  }
  const int nt1 = has1 ? ntk : 0;      // key tiles of Q1 (all loaded tiles)
  // Walks the loaded key tiles in order: segment s, tile kt within it.
  struct TileIter {
    int s, kt;
  };
  auto iter_begin = [&]() {
    TileIter it{0, 0};
    while (it.s < nseg && ntks[it.s] == 0) ++it.s;
    return it;
  };
  auto iter_next = [&](TileIter& it) {
    if (++it.kt == ntks[it.s]) {
      it.kt = 0;
      ++it.s;
      while (it.s < nseg && ntks[it.s] == 0) ++it.s;
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
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR_SF(t), 1);
      mbar_init(BAR_PF(t, 0), 4);   // one arrival per softmax warp
      mbar_init(BAR_PF(t, 1), 4);
      mbar_init(BAR_OD(t), 1);
    }
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

  if (warp < 4) setmaxnreg_dec<C::kRegsLow>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      const int nq = has1 ? 2 : 1;
      mbar_arrive_expect_tx(BAR_Q, nq * C::kTileBytes);
      for (int t = 0; t < nq; ++t)
        for (int sl = 0; sl < C::kSlabs; ++sl)
          tma_load_3d(sQ + t * C::kTileBytes + sl * C::kSlabBytes, &p.tm_q, BAR_Q, sl * 64, head,
                      row0 + t * kBM);
      int k_issued = 0, v_issued = 0;
      bool waited = !p.pdl_wait;
      TileIter ik = iter_begin(), iv = iter_begin();
      for (int j = 0; j <= ntk; ++j) {
        if (j < ntk) {
          const int st = j % KS;
          if (j >= KS && !mbar_wait(BAR_KE(st), ((j / KS) - 1) & 1, abort_flag, p.wait_limit_ns)) break;
          const Seg& sg = R.seg[ik.s];
          if (sg.src == kSrcPass && !waited) {   // the passing buffer is written by the preceding grid
            grid_dependency_wait();
            waited = true;
          }
          const CUtensorMap* tk = sg.src == kSrcMain ? &p.tm_k : &p.tm_kp;
          const int krow = sg.start + ik.kt * kBN;
          if (j != p.skip_k_tile) {
            mbar_arrive_expect_tx(BAR_KF(st), C::kTileBytes);
            for (int sl = 0; sl < C::kSlabs; ++sl)
              tma_load_3d(sK + st * C::kTileBytes + sl * C::kSlabBytes, tk, BAR_KF(st), sl * 64, kv, krow);
          }
          k_issued = j + 1;
          iter_next(ik);
        }
        if (j >= 1) {
          const int i = j - 1, st = i % VS;
          if (i >= VS && !mbar_wait(BAR_VE(st), ((i / VS) - 1) & 1, abort_flag, p.wait_limit_ns)) break;
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
        const uint64_t dl = p.wait_limit_ns / 4;
        mbar_wait_drain(BAR_Q, 0, dl);
        for (int j = max(0, k_issued - KS); j < k_issued; ++j)
          if (j != p.skip_k_tile) mbar_wait_drain(BAR_KF(j % KS), (j / KS) & 1, dl);
        for (int j = max(0, v_issued - VS); j < v_issued; ++j) mbar_wait_drain(BAR_VF(j % VS), (j / VS) & 1, dl);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop; elect.sync picks the lane that issues
    // each MMA and commit (ptx.cuh: mma_*_warp), and the waits are taken by
    // every lane and voted, so control flow stays warp-uniform.
    {
      constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kBN, false, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
      // Descriptor high words are constant (SBO 1024 B, version 1, 128-B
      // swizzle); the low word is (address >> 4) | (LBO >> 4) << 16, so
      // stepping through a tile only adds to the low word.
      constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
      auto desc = [](uint32_t lo) -> uint64_t { return (static_cast<uint64_t>(kDescHi) << 32) | lo; };
      const uint32_t q_lo = (sQ >> 4) | (1u << 16);
      const uint32_t k_lo = (sK >> 4) | (1u << 16);
      const uint32_t v_lo = (sV >> 4) | ((static_cast<uint32_t>(C::kSlabBytes) >> 4) << 16);
      auto wait = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.wait_limit_ns));
      };
      // S_t = Q_t K_j^T into TMEM buffer t
      auto issue_s = [&](int t, int j) {
        const uint32_t tS = tmem + 256u + 128u * t;
        const uint32_t qa = q_lo + ((t * C::kTileBytes) >> 4);
        const uint32_t kb = k_lo + (((j % KS) * C::kTileBytes) >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * C::kSlabBytes + (k & 3) * 32) >> 4;
          mma_ss_warp(tS, desc(qa + off), desc(kb + off), kIdescQK, k > 0 ? 1u : 0u);
        }
        mma_commit_warp(BAR_SF(t));
      };
      // O_t += P_t V_j once P_t (softmax of tile t) is ready; V_j's arrival
      // is awaited by the caller beforehand, off the P-ready path.
      auto issue_pv = [&](int t, int j, bool release_v, bool last) -> bool {
        const int st = j % VS;
        const uint32_t tP = tmem + 256u + 128u * t;
        const uint32_t tO = tmem + 128u * t;
        const uint32_t vb = v_lo + ((st * C::kTileBytes) >> 4);
        // P arrives in two halves of 64 keys; the first four MMAs run while
        // the softmax still computes the second half
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!wait(BAR_PF(t, half), j & 1)) return false;
          tc_fence_after();
#pragma unroll
          for (int k = 4 * half; k < 4 * half + 4; ++k)
            mma_ts_warp(tO, tP + k * 8, desc(vb + ((k * 2048) >> 4)), kIdescPV, (j > 0 || k > 0) ? 1u : 0u);
        }
        if (last) mma_commit_warp(BAR_OD(t));   // single phase: O_t is final
        if (release_v) mma_commit_warp(BAR_VE(st));
        return true;
      };
      bool ok = wait(BAR_Q, 0);
      for (int j = 0; ok && j < ntk; ++j) {
        ok = wait(BAR_KF(j % KS), (j / KS) & 1);
        if (!ok) break;
        tc_fence_after();
        if (j < nt0) issue_s(0, j);
        if (j >= 1 && j - 1 < nt1) {
          ok = issue_pv(1, j - 1, true, j - 1 == nt1 - 1);   // V_{j-1} arrived before O0 += P0 V_{j-1}
          if (!ok) break;
        }
        if (j < nt1) issue_s(1, j);
        mma_commit_warp(BAR_KE(j % KS));
        ok = wait(BAR_VF(j % VS), (j / VS) & 1);   // V_j is needed by O0 (now) or O1 (next)
        if (!ok) break;
        if (j < nt0) {
          ok = issue_pv(0, j, j >= nt1, j == nt0 - 1);   // V_j is Q0's alone when Q1 does not read it
          if (!ok) break;
        }
      }
      if (ok && nt1 > 0) issue_pv(1, nt1 - 1, true, true);
      mma_commit_warp(BAR_FIN);   // every MMA issued above has finished once this lands
      mbar_wait_drain(BAR_FIN, 0, p.wait_limit_ns / 4);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    setmaxnreg_inc<C::kRegsHigh>();
    const int qt = warp >= 8 ? 1 : 0;       // which Q tile this warpgroup owns
    const int nt = qt ? nt1 : nt0;
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int rit = q * 32 + lane;          // row in tile
    const int row = row0 + qt * kBM + rit;
    const int rows_valid = qt ? rv1 : rv0;
    const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t tS = tq + 256u + 128u * qt;
    const uint32_t tO = tq + 128u * qt;
    const float sl2 = p.scale_log2;
    float m = -INFINITY;   // running max of the scaled logits, log2 units
    float l = 0.f;
    bool ok = true;
    // Keys of each segment this row sees, computed once (the loop below then
    // reads no segment descriptors from parameter memory).
    int seg_lim[kMaxSegs];
#pragma unroll
    for (int s = 0; s < kMaxSegs; ++s) {
      seg_lim[s] = 0;
      if (s < nseg) {
        const Seg& sg = R.seg[s];
        seg_lim[s] = sg.causal ? min(sg.len, row - sg.start + 1) : sg.len;
      }
    }
    TileIter it = iter_begin();
    for (int j = 0; j < nt; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(BAR_SF(qt), j & 1, abort_flag, p.wait_limit_ns));
      if (!ok) break;
      tc_fence_after();
      float2 x[kBN / 2];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + c * 32, r);
#pragma unroll
        for (int e = 0; e < 16; ++e)
          x[c * 16 + e] = make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
      }
      tmem_wait_ld();
      const int lim = it.s == 0 ? seg_lim[0] : it.s == 1 ? seg_lim[1] : seg_lim[2];
      const int nvalid = lim - it.kt * kBN;
      if (nvalid < kBN) {
#pragma unroll
        for (int i = 0; i < kBN / 2; ++i) {
          if (2 * i >= nvalid) x[i].x = -INFINITY;
          if (2 * i + 1 >= nvalid) x[i].y = -INFINITY;
        }
      }
      float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < kBN / 2; i += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) mq[u] = fmax3(mq[u], x[i + u].x, x[i + u].y);
      }
      const float mx = fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3])) * sl2;
      const bool grow = mx > m + 8.0f;
      const float m_new = grow ? mx : m;
      const float alpha = grow ? ex2_approx(m - m_new) : 1.0f;
      const float2 sl22 = make_float2(sl2, sl2);
      const float2 neg2 = make_float2(-m_new, -m_new);
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // O_t += P V of the previous key tile is complete here: that MMA was
        // issued before the one that produced this S, the commit tracked by
        // BAR_SF covers every MMA issued before it, and MMAs complete in issue
        // order.  So O_t can be rescaled without another wait.
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 v = __fmul2_rn(make_float2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), a2);
            r[e] = __float_as_uint(v.x);
            r[e + 1] = __float_as_uint(v.y);
          }
          tmem_st32(tO + c * 32, r);
        }
      }
      // P in two halves of 64 keys (32 packed columns each), each published
      // as soon as it is in TMEM
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const int i = 32 * half + u;
          const float2 y = __ffma2_rn(x[i], sl22, neg2);
          const float2 pe = make_float2(ex2_approx(y.x), ex2_approx(y.y));
          acc[i & 3] = __fadd2_rn(acc[i & 3], pe);
          pk[u] = pack_bf16x2(pe.x, pe.y);
        }
        tmem_st32(tS + 32 * half, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR_PF(qt, half));   // one arrival per warp
      }
      const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
      const float2 a4 = __fadd2_rn(a01, a23);
      l = l * alpha + (a4.x + a4.y);
      m = m_new;
      iter_next(it);
    }
    if (ok && nt > 0) {   // BAR_OD(t) completes once, after the last O_t += P V
      ok = __all_sync(0xffffffffu, mbar_wait(BAR_OD(qt), 0, abort_flag, p.wait_limit_ns));
    }
    if (ok && nt > 0) {
      tc_fence_after();
      const bool valid = rit < rows_valid;
      const float inv_l = 1.0f / l;
      const float lse_nat = (m + __log2f(l)) * 0.69314718055994530942f;
      if (R.out_kind == kOutRows) {
        __nv_bfloat16* dst = p.O + (static_cast<int64_t>(row) * p.Hq + head) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
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
          tmem_ld32(tO + c * 32, r);
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
    if (p.merge_count != nullptr && R.out_kind == kOutPartial) {
      // Last-arriver merge ("APB-V ..." pith.science review, ledger: merging
      // partial results through their lse is exact).  Every softmax thread
      // of the CTA takes part, whatever happened above, so the named barrier
      // always completes.
      __threadfence();                       // this CTA's partial rows are visible device-wide
      named_barrier_sync(1, 256);
      int32_t* s_last = reinterpret_cast<int32_t*>(smem + C::kOffMisc + 8);
      if (threadIdx.x == 128) {
        if (p.pdl_wait) grid_dependency_wait();   // the counters were zeroed by the preceding grid
        const int qpair = (row0 - p.qs) / (2 * kBM);
        const int old = atomicAdd(p.merge_count + qpair * p.Hq + head, 1);
        *s_last = old == p.V - 1 ? 1 : 0;
      }
      named_barrier_sync(1, 256);
      if (*s_last) {
        __threadfence();                     // every other partial of these rows is visible
        merge_rows<D>(p, row0 - p.qs, rv0 + max(rv1, 0), head, warp - 4, lane);
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
