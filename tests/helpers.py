"""Shared helpers for the parity tests (not collected as tests)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_approximate_attention_b200 import workloads as W

# Tolerances of the layer (bf16 inputs, fp32 accumulation): outputs within
# 2e-2 max-abs, lse within 1e-3; top-lp sets exact except near-ties whose
# oracle score gap is below 1e-4 of the block's largest |score|.
O_TOL = 2e-2
LSE_TOL = 1e-3
TIE_REL = 1e-4


def layout_of(wl: W.Workload) -> oracle.Layout:
    return oracle.make_layout(wl.num_hosts, wl.anchor_len, wl.block_lens, wl.query_len, wl.lp,
                              wl.num_q_heads, wl.num_kv_heads, wl.head_dim)


def small_workload(name, la, blocks, lq, lp, hq, hkv, d, gen="gaussian", seed=5):
    return W.Workload(name, num_hosts=len(blocks) // 2, anchor_len=la, block_lens=list(blocks),
                      query_len=lq, lp=lp, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                      generator=gen, seed=seed)


def compare_selection(lay: oracle.Layout, ref_scores: dict, ref_idx: dict, gpu_idx: np.ndarray,
                      tie_rel: float = TIE_REL):
    """Compare GPU passing indices [V-1, Hkv, lp] with the oracle's.  Returns
    (tolerated_swaps, affected) where affected[h][kv] is True when the sets
    differ (only at near-ties within tie_rel of the block's largest |score|,
    else AssertionError)."""
    swaps = 0
    affected = {}
    for h in range(lay.V - 1):
        e = lay.lp_eff(h)
        affected[h] = {}
        for kv in range(lay.num_kv_heads):
            g = gpu_idx[h, kv]
            assert np.all(g[e:] == -1), f"block {h} kv {kv}: padding not -1"
            gs = g[:e]
            assert np.all(np.diff(gs) > 0), f"block {h} kv {kv}: indices not ascending/unique"
            rs = np.asarray(ref_idx[h][kv])
            diff = set(gs.tolist()) ^ set(rs.tolist())
            if diff:
                s = np.asarray(ref_scores[h][kv], dtype=np.float64)
                tau = np.sort(s)[::-1][e - 1]
                tol = tie_rel * np.abs(s).max()
                bad = [j for j in diff if abs(s[j] - tau) > tol]
                assert not bad, f"block {h} kv {kv}: non-tie mismatches at {bad[:8]}"
                swaps += len(set(gs.tolist()) - set(rs.tolist()))
            affected[h][kv] = bool(diff)
    return swaps, affected


def host_affected(lay, affected, h, kv) -> bool:
    return any(affected[j][kv] for j in range(min(h, lay.V - 1)))


def max_err(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.abs(a - b).max()) if a.size else 0.0


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


def idx_dict(lay: oracle.Layout, idx_arr: np.ndarray) -> dict:
    """[V-1, Hkv, lp] index array (-1 padded) -> the oracle's {h: [Hkv, lp_eff]} form."""
    return {h: np.stack([np.asarray(idx_arr[h, kv, :lay.lp_eff(h)], dtype=np.int64)
                         for kv in range(lay.num_kv_heads)])
            for h in range(lay.V - 1)}


def check_rows(lay: oracle.Layout, inp: dict, sel_idx: np.ndarray, affected: dict,
               rows, heads, O_rows: np.ndarray, lse_rows: np.ndarray, ref_O: np.ndarray,
               ref_lse: np.ndarray) -> int:
    """Compare output rows with the oracle at O_TOL / LSE_TOL.

    ``O_rows`` [len(rows), len(heads), d] and ``lse_rows`` [len(heads), len(rows)]
    are the rows under test; ``ref_O`` / ``ref_lse`` the oracle's rows (same
    shapes) computed with the oracle's own selection.  A context
    row of a host whose passing keys differ from the oracle's only at
    tolerated near-ties (``affected``, from compare_selection) is instead
    compared with the oracle recomputed on the selection under test
    ``sel_idx`` ([V-1, Hkv, lp]), since both selections are valid there.
    Returns the number of (row, head) pairs recomputed that way."""
    rows = [int(r) for r in rows]
    redo = []
    for i, r in enumerate(rows):
        kind, h = lay.host_of_row(r)
        for hi, g in enumerate(heads):
            kv = g // lay.group
            if kind == "context" and host_affected(lay, affected, h, kv):
                redo.append((i, hi))
                continue
            assert np.abs(O_rows[i, hi] - ref_O[i, hi]).max() <= O_TOL, (r, g)
            assert abs(lse_rows[hi, i] - ref_lse[hi, i]) <= LSE_TOL, (r, g)
    if redo:
        sel = idx_dict(lay, sel_idx)
        rr = sorted({rows[i] for i, _ in redo})
        hh = sorted({heads[hi] for _, hi in redo})
        got_rows, o2, l2 = oracle.rows_fwd(lay, inp["Q"], inp["K"], inp["V"], sel, rr, hh)
        pos_r = {int(r): k for k, r in enumerate(got_rows)}
        pos_h = {g: k for k, g in enumerate(hh)}
        for i, hi in redo:
            r, g = rows[i], heads[hi]
            assert np.abs(O_rows[i, hi] - o2[pos_r[r], pos_h[g]]).max() <= O_TOL, ("reselected", r, g)
            assert abs(lse_rows[hi, i] - l2[pos_h[g], pos_r[r]]) <= LSE_TOL, ("reselected", r, g)
    return len(redo)
