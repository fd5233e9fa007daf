"""The pages' split of the layer over GPUs (host masks, hosts.py) with the
library's kernels.  One GPU stands in for the ranks: each rank's compression
and attention run one after another into one shared set of buffers, which is
exactly what the all-gathers leave on every rank.  Every output must equal,
bit for bit, the single-GPU stage path (compress, attention over all hosts,
merge), which the other parity tests pin to the oracle."""
import pytest
import torch

import sparse_approximate_attention_b200 as spava
from sparse_approximate_attention_b200 import hosts
from sparse_approximate_attention_b200 import workloads as W

from helpers import small_workload

pytestmark = pytest.mark.gpu

CASES = {
    "ragged_d128": (small_workload("ragged_d128", 64, (300, 129, 77, 511), 37, 50, 4, 2, 128), (2,)),
    "unequal_h3_d128": (small_workload("unequal_h3", 100, (250, 90, 333, 17, 128, 129), 64, 80, 4, 2, 128),
                        (2, 3)),
    "no_anchor_h4_d64": (small_workload("no_anchor_h4", 0, (129, 255, 64, 300, 1, 77, 200, 130), 19, 33,
                                        4, 4, 64), (2, 3, 4)),
    "frames_h4": (small_workload("frames_h4", 256, (1024,) * 8, 128, 256, 8, 2, 128, gen="frames"), (4,)),
    "lp0": (small_workload("lp0", 32, (130, 200, 64, 90), 17, 0, 2, 1, 128), (2,)),
}


def _stage_path(p, Q, K, V):
    qsum, scores, idx, Kp, Vp = spava.compress(p, Q, K, V)
    if p.lp == 0:
        Kp = Vp = None
    O, lse, O_part, lse_part = spava.attn_fwd(p, Q, K, V, Kp, Vp)
    spava.lse_merge(p, O_part, lse_part, O, lse)
    return scores, idx, Kp, Vp, O, lse


@pytest.mark.parametrize("name", list(CASES))
def test_ranks_on_one_gpu_reproduce_the_stage_path(name):
    wl, worlds = CASES[name]
    inp = W.make_inputs(wl)
    Q, K, V = (inp[k].cuda() for k in ("Q", "K", "V"))
    p = spava.Problem.from_workload(wl)
    ref = _stage_path(p, Q, K, V)
    torch.cuda.synchronize()
    assert spava.device_error() == 0
    sz = p.sizes()
    n, hq, hkv, d, Vh = sz["seq_len"], wl.num_q_heads, wl.num_kv_heads, wl.head_dim, p.V
    for world in worlds:
        qsum = torch.empty(hkv, d, dtype=torch.float32, device="cuda")
        scores = torch.full((hkv, sz["score_cols"]), float("nan"), dtype=torch.float32, device="cuda")
        idx = torch.full((Vh - 1, hkv, wl.lp), -7, dtype=torch.int32, device="cuda")
        rows = sz["passing_rows"]
        Kp = torch.zeros(max(1, rows), hkv, d, dtype=torch.bfloat16, device="cuda")[:rows]
        Vp = torch.zeros_like(Kp)
        O = torch.full((n, hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((hq, n), float("nan"), dtype=torch.float32, device="cuda")
        O_part = torch.full((Vh, wl.query_len, hq, d), float("nan"), dtype=torch.float32, device="cuda")
        lse_part = torch.full((Vh, hq, wl.query_len), float("nan"), dtype=torch.float32, device="cuda")
        qs = [p.with_hosts(hosts.host_mask(wl.num_hosts, world, r)) for r in range(world)]
        if wl.lp:
            for q in qs:
                spava.compress(q, Q, K, V, qsum, scores, idx, Kp, Vp)
        for q in qs:
            spava.attn_fwd(q, Q, K, V, Kp if wl.lp else None, Vp if wl.lp else None, O, lse, O_part, lse_part)
        spava.lse_merge(p, O_part, lse_part, O, lse)
        torch.cuda.synchronize()
        assert spava.device_error() == 0
        r_scores, r_idx, r_Kp, r_Vp, r_O, r_lse = ref
        if wl.lp:
            assert torch.equal(scores, r_scores), f"world {world}: scores"
            assert torch.equal(idx, r_idx), f"world {world}: idx"
            assert torch.equal(Kp, r_Kp) and torch.equal(Vp, r_Vp), f"world {world}: passing rows"
        assert torch.equal(O, r_O), f"world {world}: O"
        assert torch.equal(lse, r_lse), f"world {world}: lse"


def test_sharded_layer_object_on_one_rank_matches_the_stage_path():
    """HostShardedLayer with world 1 (no collective): the library's kernels
    through the split's code path."""
    wl = CASES["frames_h4"][0]
    inp = W.make_inputs(wl)
    Q, K, V = (inp[k].cuda() for k in ("Q", "K", "V"))
    p = spava.Problem.from_workload(wl)
    ref = _stage_path(p, Q, K, V)
    layer = hosts.HostShardedLayer(p, 1, 0, "cuda")
    n, hq, d = p.sizes()["seq_len"], wl.num_q_heads, wl.head_dim
    O = torch.empty(n, hq, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(hq, n, dtype=torch.float32, device="cuda")
    layer.forward(Q, K, V, O, lse)
    torch.cuda.synchronize()
    assert spava.device_error() == 0
    assert torch.equal(O, ref[4]) and torch.equal(lse, ref[5])


def test_partial_masks_are_refused_where_all_hosts_are_needed():
    wl = CASES["ragged_d128"][0]
    inp = W.make_inputs(wl)
    Q, K, V = (inp[k].cuda() for k in ("Q", "K", "V"))
    q = spava.Problem.from_workload(wl, host_mask=0b1001)
    with pytest.raises(spava.SpavaError) as e:
        spava.layer_fwd(q, Q, K, V)
    assert e.value.code == 2   # SPAVA_ERR_UNSUPPORTED
    with pytest.raises(spava.SpavaError) as e:
        spava.score(q, Q, K)
    assert e.value.code == 2
