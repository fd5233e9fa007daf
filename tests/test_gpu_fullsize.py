"""Parity at the full long-video sizes, in the launch configuration the bench
times (the fused spava_layer_fwd): every score and every passing index is
checked, and output rows are checked on samples the oracle computes one by
one -- for every virtual host the first, the last and one seeded-random
128-row tile, the anchor's first tile and all query rows, for two query heads
(one in the first and one in the last KV group)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_approximate_attention_b200 as spava
from sparse_approximate_attention_b200 import workloads as W

from helpers import check_rows, compare_selection, layout_of, max_err, to_np

pytestmark = pytest.mark.gpu

FULL = ["qwen25vl3b_64f", "qwen25vl7b_128k", "longvideo_256k_lp512", "longvideo_256k_lp2048",
        "longvideo_256k_lp4096", "exact_dense_3b", "exact_dense_3b_unequal", "ruler_llama31_8b_128k"]


def _sample_rows(lay, rng):
    rows = list(range(min(128, lay.anchor_len)))
    for h in range(lay.V):
        s0, L = lay.block_starts[h], lay.block_lens[h]
        ntile = -(-L // 128)
        picks = {0, ntile - 1, int(rng.integers(0, ntile))}
        for t in picks:
            rows += list(range(s0 + 128 * t, min(s0 + L, s0 + 128 * (t + 1))))
    rows += list(range(lay.query_start, lay.n))
    return rows


@pytest.mark.parametrize("name", FULL)
def test_full_size_layer(name):
    wl = W.workloads()[name]
    lay = layout_of(wl)
    inp = W.make_inputs(wl)
    p = spava.Problem.from_workload(wl)
    dev = {k: inp[k].cuda() for k in ("Q", "K", "V")}
    O, lse = spava.layer_fwd(p, dev["Q"], dev["K"], dev["V"])
    _, scores, idx, _, _ = spava.compress(p, dev["Q"], dev["K"], dev["V"])   # the layer's selection
    idx = to_np(idx)
    torch.cuda.synchronize()
    assert spava.device_error() == 0
    s_gpu = to_np(scores)
    del dev, scores

    ref_scores, ref_idx = oracle.compress(lay, inp["Q"], inp["K"])
    col = 0
    for h in range(lay.V - 1):
        r = ref_scores[h]
        L = lay.block_lens[h]
        assert max_err(s_gpu[:, col:col + L], r) <= 1e-5 * np.abs(r).max() + 1e-4, f"scores block {h}"
        col += L
    swaps, affected = compare_selection(lay, ref_scores, ref_idx, idx)
    print(f"{name}: tolerated near-tie swaps = {swaps}")

    rng = np.random.default_rng(1234)
    heads = [0, wl.num_q_heads - 1]
    rows, o_ref, l_ref = oracle.rows_fwd(lay, inp["Q"], inp["K"], inp["V"], ref_idx,
                                         _sample_rows(lay, rng), heads)
    On = O[torch.as_tensor(rows).cuda()][:, heads].float().cpu().numpy()
    Ln = lse[heads][:, torch.as_tensor(rows).cuda()].cpu().numpy()
    On = On.astype(np.float64)
    recomputed = check_rows(lay, inp, idx, affected, rows, heads, On, Ln, o_ref, l_ref)
    print(f"{name}: rows recomputed on the layer's own selection = {recomputed}")
