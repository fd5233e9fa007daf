// Host-side problem plan: validation, context splitting, passing-buffer
// offsets, workspace carving and the attention launch's work list.
//
// Context splitting follows "Spava: Accelerating Long-Video Understanding via
// Sequence-Parallelism-aware Approximate Attention" (sciencestack.ai), Fig. 2
// caption: anchor block, 2H context blocks on virtual hosts, query block.
// The attention work list follows its Fig. 4 (attention load balancing): the
// pages pair virtual hosts h and 2H-1-h on one physical host so that cheap
// (early) and expensive (late) blocks even out; on one GPU the same goal is
// met by ordering every 128-row tile by its key count, longest first, with
// ZigZag pairs adjacent among equal costs.
#pragma once
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/spava.h"

namespace spava {

constexpr int kMaxV = 2 * SPAVA_MAX_HOSTS;
constexpr int kBM = 128;   // query rows per attention tile
constexpr int kBN = 128;   // keys per attention tile
constexpr int kMaxSegs = 3;
constexpr int kMaxRegions = 2 + 2 * kMaxV;
constexpr int kMaxItems = 6144;

enum : int32_t { kSrcMain = 0, kSrcPass = 1 };
enum : int32_t { kOutRows = 0, kOutPartial = 1 };

// A contiguous run of keys: rows [start, start+len) of K/V (src main) or of
// Kp/Vp (src pass).  causal: main-sequence key p is visible to row r iff p <= r.
struct Seg {
  int32_t src, start, len, causal;
};

// Rows [row_start, row_start+nrows) of the sequence that share one key list.
struct Region {
  int32_t row_start, nrows, out_kind, host, nseg;
  Seg seg[kMaxSegs];
};

struct Plan {
  int H = 0, V = 0, la = 0, lq = 0, lp = 0, Hq = 0, Hkv = 0, d = 0, G = 0;
  int score_kind = 0;   // SPAVA_SCORE_*
  uint64_t hmask = 0;   // selected virtual hosts (all V bits when the problem's mask is 0)
  bool partial = false; // some virtual host is not selected
  int ncblk = 0;        // selected compressed blocks (h < V-1)
  int32_t cblk[kMaxV] = {};
  float scale = 0.f;
  int64_t n = 0, qs = 0, score_cols = 0, passing_rows = 0;
  int32_t L[kMaxV] = {}, start[kMaxV] = {}, lpe[kMaxV] = {}, poff[kMaxV + 1] = {};
  int nregions = 0;
  Region regions[kMaxRegions];
  int64_t pairs = 0;
  int64_t tiles = 0;
  int64_t items = 0;   // attention work items (pairs of 128-row tiles)
  int n_merge = 0;   // merge counters: one per (pair of 128-row query tiles, query head)
  // workspace carving (bytes from the workspace base)
  size_t ws_qsum = 0, ws_scores = 0, ws_idx = 0, ws_kp = 0, ws_vp = 0, ws_opart = 0,
         ws_lsepart = 0, ws_count = 0, ws_vo = 0, ws_vlse = 0, ws_total = 0;
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// sum over rows r in [r0, r1) of clamp(r - s + 1, 0, len)
inline int64_t causal_pairs(int64_t r0, int64_t r1, int64_t s, int64_t len) {
  int64_t x0 = r0 - s + 1, x1 = r1 - s;   // x runs over [x0, x1]
  if (x1 < 1 || len <= 0 || r1 <= r0) return 0;
  int64_t lo = std::max<int64_t>(x0, 1), hi = std::min<int64_t>(x1, len);
  int64_t total = 0;
  if (hi >= lo) total += (lo + hi) * (hi - lo + 1) / 2;
  int64_t over_lo = std::max<int64_t>(x0, len + 1);
  if (x1 >= over_lo) total += len * (x1 - over_lo + 1);
  return total;
}

inline int64_t seg_pairs(const Seg& sg, int64_t r0, int64_t r1) {
  if (!sg.causal) return static_cast<int64_t>(sg.len) * (r1 - r0);
  return causal_pairs(r0, r1, sg.start, sg.len);
}

// Keys of segment sg that the last row of a tile can see (tile rows end at r_last).
inline int64_t seg_visible_len(const Seg& sg, int64_t r_last) {
  if (!sg.causal) return sg.len;
  return std::max<int64_t>(0, std::min<int64_t>(sg.len, r_last - sg.start + 1));
}

inline spava_status_t make_plan(const spava_problem_t* p, Plan* pl) {
  if (!p || !pl) return SPAVA_ERR_INVALID_ARG;
  if (p->num_hosts < 1 || p->num_hosts > SPAVA_MAX_HOSTS) return SPAVA_ERR_INVALID_ARG;
  if (!p->block_lens) return SPAVA_ERR_INVALID_ARG;
  if (p->anchor_len < 0 || p->query_len < 1 || p->lp < 0) return SPAVA_ERR_INVALID_ARG;
  if (p->num_q_heads < 1 || p->num_kv_heads < 1) return SPAVA_ERR_INVALID_ARG;
  if (p->num_q_heads % p->num_kv_heads) return SPAVA_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return SPAVA_ERR_UNSUPPORTED;
  if (!(p->softmax_scale == p->softmax_scale)) return SPAVA_ERR_INVALID_ARG;  // NaN
  if (p->score_kind < SPAVA_SCORE_LINEAR || p->score_kind > SPAVA_SCORE_CONTEXT) return SPAVA_ERR_INVALID_ARG;
  Plan& P = *pl;
  P = Plan();
  P.H = p->num_hosts;
  P.V = 2 * p->num_hosts;
  P.la = p->anchor_len;
  P.lq = p->query_len;
  P.lp = p->lp;
  P.Hq = p->num_q_heads;
  P.Hkv = p->num_kv_heads;
  P.d = p->head_dim;
  P.G = P.Hq / P.Hkv;
  P.score_kind = p->score_kind;
  P.scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(P.d));
  const uint64_t all = (uint64_t(1) << P.V) - 1;
  if (static_cast<uint64_t>(p->host_mask) & ~all) return SPAVA_ERR_INVALID_ARG;
  P.hmask = p->host_mask ? static_cast<uint64_t>(p->host_mask) : all;
  P.partial = P.hmask != all;
  auto sel = [&](int h) { return ((P.hmask >> h) & 1u) != 0; };
  for (int h = 0; h < P.V - 1; ++h)
    if (sel(h)) P.cblk[P.ncblk++] = h;
  int64_t pos = P.la;
  for (int h = 0; h < P.V; ++h) {
    int32_t L = p->block_lens[h];
    if (L < 1) return SPAVA_ERR_INVALID_ARG;
    P.L[h] = L;
    P.start[h] = static_cast<int32_t>(pos);
    P.lpe[h] = std::min(P.lp, L);
    pos += L;
    if (pos > (int64_t(1) << 30)) return SPAVA_ERR_UNSUPPORTED;
  }
  P.qs = pos;
  P.n = pos + P.lq;
  if (P.n > (int64_t(1) << 30)) return SPAVA_ERR_UNSUPPORTED;
  P.poff[0] = 0;
  for (int h = 0; h < P.V; ++h) {
    P.poff[h + 1] = P.poff[h] + (h < P.V - 1 ? P.lpe[h] : 0);
    if (h < P.V - 1) P.score_cols += P.L[h];
  }
  P.passing_rows = P.poff[P.V - 1];

  // regions: query partials, context blocks, anchor
  auto add = [&](int32_t r0, int32_t nr, int32_t kind, int32_t host) -> Region& {
    Region& R = P.regions[P.nregions++];
    R.row_start = r0;
    R.nrows = nr;
    R.out_kind = kind;
    R.host = host;
    R.nseg = 0;
    return R;
  };
  auto seg = [](Region& R, int32_t src, int32_t s, int32_t len, int32_t causal) {
    if (len <= 0) return;
    R.seg[R.nseg++] = Seg{src, s, len, causal};
  };
  for (int h = 0; h < P.V; ++h) {   // query rows, partial of host h
    if (!sel(h)) continue;
    Region& R = add(static_cast<int32_t>(P.qs), P.lq, kOutPartial, h);
    if (h == 0) {
      seg(R, kSrcMain, 0, P.la + P.L[0], 0);       // A and B^(0), contiguous
      seg(R, kSrcMain, static_cast<int32_t>(P.qs), P.lq, 1);
    } else {
      seg(R, kSrcMain, P.start[h], P.L[h], 0);
    }
  }
  for (int i = 0; i < P.V; ++i) {   // context rows, ZigZag order 0, V-1, 1, V-2, ...
    int h = (i % 2 == 0) ? i / 2 : P.V - 1 - i / 2;
    if (!sel(h)) continue;
    Region& R = add(P.start[h], P.L[h], kOutRows, h);
    if (h == 0) {
      seg(R, kSrcMain, 0, P.la + P.L[0], 1);       // A then causal B^(0): plain causal
    } else {
      seg(R, kSrcMain, 0, P.la, 0);
      seg(R, kSrcPass, 0, P.poff[h], 0);
      seg(R, kSrcMain, P.start[h], P.L[h], 1);
    }
  }
  if (P.la > 0 && sel(0)) {   // the anchor rows go with virtual host 0
    Region& R = add(0, P.la, kOutRows, -1);
    seg(R, kSrcMain, 0, P.la, 1);
  }
  for (int r = 0; r < P.nregions; ++r) {
    const Region& R = P.regions[r];
    for (int s = 0; s < R.nseg; ++s) P.pairs += seg_pairs(R.seg[s], R.row_start, R.row_start + R.nrows);
    P.tiles += (R.nrows + kBM - 1) / kBM;
    P.items += ((R.nrows + kBM - 1) / kBM + 1) / 2;
  }

  // workspace carving for the fused layer
  size_t off = 0;
  auto carve = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  P.ws_qsum = carve(sizeof(float) * P.Hkv * P.d);
  P.ws_scores = carve(sizeof(float) * P.Hkv * static_cast<size_t>(P.score_cols));
  P.ws_idx = carve(sizeof(int32_t) * static_cast<size_t>(P.V - 1) * P.Hkv * P.lp);
  P.ws_kp = carve(2ull * static_cast<size_t>(P.passing_rows) * P.Hkv * P.d);
  P.ws_vp = carve(2ull * static_cast<size_t>(P.passing_rows) * P.Hkv * P.d);
  P.ws_opart = carve(sizeof(float) * static_cast<size_t>(P.V) * P.lq * P.Hq * P.d);
  P.ws_lsepart = carve(sizeof(float) * static_cast<size_t>(P.V) * P.Hq * P.lq);
  P.n_merge = ((P.lq + 2 * kBM - 1) / (2 * kBM)) * P.Hq;
  P.ws_count = carve(sizeof(int32_t) * static_cast<size_t>(P.n_merge));
  if (P.score_kind == SPAVA_SCORE_CONTEXT) {   // first pass of the context selector: O and lse of the block rows
    P.ws_vo = carve(2ull * static_cast<size_t>(P.n) * P.Hq * P.d);
    P.ws_vlse = carve(sizeof(float) * static_cast<size_t>(P.Hq) * P.n);
  }
  P.ws_total = off;
  return SPAVA_OK;
}

// The first pass of a selector variant as attention regions over the blocks
// h < V-1: softmax -> the query block's rows over block h's keys (written as
// host h's query partial); context -> block h's rows causally over its own
// keys (written as rows).  Replaces the plan's regions, tiles and items.
inline void make_variant_regions(Plan* pl) {
  Plan& P = *pl;
  P.nregions = 0;
  P.tiles = 0;
  P.items = 0;
  P.passing_rows = 0;   // no region reads the passing buffer
  for (int h = 0; h < P.V - 1; ++h) {
    Region& R = P.regions[P.nregions++];
    const bool ctx = P.score_kind == SPAVA_SCORE_CONTEXT;
    R.row_start = ctx ? P.start[h] : static_cast<int32_t>(P.qs);
    R.nrows = ctx ? P.L[h] : P.lq;
    R.out_kind = ctx ? kOutRows : kOutPartial;
    R.host = h;
    R.nseg = 1;
    R.seg[0] = Seg{kSrcMain, P.start[h], P.L[h], ctx ? 1 : 0};
    const int nt = (R.nrows + kBM - 1) / kBM;
    P.tiles += nt;
    P.items += (nt + 1) / 2;
  }
}

// Cost-ordered work items: (region << 20) | pair, one CTA per pair of
// consecutive 128-row tiles of a region, longest key list first.  A pair
// without its second tile costs about two thirds of a full one per key tile
// (the softmax of one tile is then exposed).
inline spava_status_t make_items(const Plan& P, std::vector<uint32_t>* items) {
  struct It {
    int64_t cost;
    uint32_t code;
  };
  std::vector<It> v;
  v.reserve(static_cast<size_t>(P.tiles / 2 + P.nregions));
  for (int r = 0; r < P.nregions; ++r) {
    const Region& R = P.regions[r];
    const int nt = (R.nrows + kBM - 1) / kBM;
    const int np = (nt + 1) / 2;
    for (int q = np - 1; q >= 0; --q) {
      const bool two = 2 * q + 1 < nt;
      const int64_t r_last = R.row_start + std::min(R.nrows, (2 * q + (two ? 2 : 1)) * kBM) - 1;
      int64_t ktiles = 0;
      for (int s = 0; s < R.nseg; ++s) ktiles += (seg_visible_len(R.seg[s], r_last) + kBN - 1) / kBN;
      v.push_back(It{ktiles * (two ? 3 : 2), (static_cast<uint32_t>(r) << 20) | static_cast<uint32_t>(q)});
    }
  }
  if (v.size() > static_cast<size_t>(kMaxItems)) return SPAVA_ERR_UNSUPPORTED;
  std::stable_sort(v.begin(), v.end(), [](const It& a, const It& b) { return a.cost > b.cost; });
  items->resize(v.size());
  for (size_t i = 0; i < v.size(); ++i) (*items)[i] = v[i].code;
  return SPAVA_OK;
}

}  // namespace spava
