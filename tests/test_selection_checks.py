"""CPU checks of the parity tests' own selection logic.

When the layer's top-lp set differs from the oracle's only at a near-tie
(the oracle's score gap to the lp-th score within 1e-4 of the block's largest
|score|), both sets are valid; the GPU tests then compare the affected hosts'
rows with the oracle recomputed on the layer's selection.  These tests force
such a swap on the CPU, with the 'layer' played by the oracle run on the
swapped selection, and check that the comparison runs, accepts correct rows
and rejects wrong ones."""
import numpy as np
import pytest
import torch

import oracle

from helpers import check_rows, compare_selection, idx_dict


def _near_tie_case():
    """A small layout whose block 0 has two keys whose scores differ by far
    less than the tie tolerance, sitting exactly at the lp-th place."""
    H, la, blocks, lq, lp, hq, hkv, d = 2, 8, [16, 16, 16, 16], 4, 4, 2, 1, 16
    lay = oracle.make_layout(H, la, blocks, lq, lp, hq, hkv, d)
    g = torch.Generator().manual_seed(21)
    n = lay.n
    Q = torch.randn(n, hq, d, generator=g, dtype=torch.float64)
    K = torch.randn(n, hkv, d, generator=g, dtype=torch.float64)
    V = torch.randn(n, hkv, d, generator=g, dtype=torch.float64)
    s0 = lay.block_starts[0]
    s = oracle.importance_scores(lay, Q, K, 0)[0]
    order = np.argsort(-s, kind="stable")
    a, b = int(order[lp - 1]), int(order[lp])          # lp-th and (lp+1)-th keys of block 0
    K[s0 + b, 0] = K[s0 + a, 0] * (1.0 + 1e-7)          # b now ties with a to ~1e-7
    return lay, {"Q": Q, "K": K, "V": V}, a, b


def test_forced_near_tie_swap_is_tolerated_and_rows_are_recomputed():
    lay, inp, a, b = _near_tie_case()
    ref = oracle.layer_fwd(lay, inp["Q"], inp["K"], inp["V"])
    kept = set(ref["idx"][0][0].tolist())
    assert (a in kept) != (b in kept)                   # exactly one of the tied pair is kept
    out, inn = (a, b) if a in kept else (b, a)
    # the selection under test keeps the other key of the tied pair
    sel = np.full((lay.V - 1, lay.num_kv_heads, lay.lp), -1, dtype=np.int32)
    for h in range(lay.V - 1):
        sel[h, 0, :lay.lp_eff(h)] = ref["idx"][h][0]
    sel[0, 0, :lay.lp_eff(0)] = np.sort([j for j in ref["idx"][0][0] if j != out] + [inn])
    swaps, affected = compare_selection(lay, ref["scores"], ref["idx"], sel)
    assert swaps == 1 and affected[0][0]
    # 'layer' outputs: the oracle on the swapped selection
    sw = idx_dict(lay, sel)
    rows = list(range(lay.n))
    heads = list(range(lay.num_q_heads))
    _, O_sw, l_sw = oracle.rows_fwd(lay, inp["Q"], inp["K"], inp["V"], sw, rows, heads)
    # the swap really changes later hosts' rows (else the test would prove nothing)
    s1 = lay.block_starts[1]
    assert np.abs(O_sw[s1:s1 + 16] - ref["O"][s1:s1 + 16]).max() > 1e-6
    n_redo = check_rows(lay, inp, sel, affected, rows, heads, O_sw, l_sw, ref["O"], ref["lse"])
    assert n_redo == sum(lay.block_lens[1:]) * len(heads)   # every row of hosts 1..V-1
    # and wrong rows on an affected host are caught (no finite-only pass)
    bad = O_sw.copy()
    bad[s1 + 3, 1] += 0.05
    with pytest.raises(AssertionError):
        check_rows(lay, inp, sel, affected, rows, heads, bad, l_sw, ref["O"], ref["lse"])


def test_non_tie_mismatch_is_rejected():
    lay, inp, a, b = _near_tie_case()
    ref = oracle.layer_fwd(lay, inp["Q"], inp["K"], inp["V"])
    sel = np.full((lay.V - 1, lay.num_kv_heads, lay.lp), -1, dtype=np.int32)
    for h in range(lay.V - 1):
        sel[h, 0, :lay.lp_eff(h)] = ref["idx"][h][0]
    kept = ref["idx"][1][0].tolist()
    s = ref["scores"][1][0]
    worst = int(np.argmin(s))                           # far below the lp-th score
    sel[1, 0, :lay.lp_eff(1)] = np.sort(kept[1:] + [worst])
    with pytest.raises(AssertionError):
        compare_selection(lay, ref["scores"], ref["idx"], sel)
