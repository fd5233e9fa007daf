"""GPU parity of every stage and of the fused layer against the CPU oracle,
through the C ABI, on small seeded cases that span several tiles and ragged
tails (partial anchor / block / query tiles, unequal blocks, la = 0, lp = 0,
lp >= L_h, G = 1, lq = 1, d = 64 and 128)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_approximate_attention_b200 as spava
from sparse_approximate_attention_b200 import workloads as W

from helpers import (LSE_TOL, O_TOL, check_rows, compare_selection, layout_of, max_err,
                     small_workload, to_np)

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": W.workloads()["tiny"],
    "ragged_d128": small_workload("ragged_d128", 64, (300, 129, 77, 511), 37, 50, 4, 2, 128),
    "no_anchor_no_passing": small_workload("no_anchor_no_passing", 0, (130, 200), 5, 0, 2, 1, 128),
    "dense_unequal_g1": small_workload("dense_unequal_g1", 100, (250, 90, 333, 17, 128, 129), 64,
                                       400, 2, 2, 128),
    "pair_lq1_d64": small_workload("pair_lq1_d64", 128, (256, 384), 1, 64, 3, 1, 64),
    "frames_multi": small_workload("frames_multi", 256, (1024,) * 4, 128, 256, 8, 2, 128,
                                   gen="frames"),
    "no_anchor_d64": small_workload("no_anchor_d64", 0, (129, 255, 64, 300, 1, 77), 19, 33, 4, 4, 64),
    # three KV heads: (row, head) strides and head steps that are not powers of two
    "kv3_d128": small_workload("kv3_d128", 40, (333, 130, 257, 96), 45, 70, 6, 3, 128),
}

_cache = {}


def _case(name):
    if name not in _cache:
        wl = CASES[name]
        inp = W.make_inputs(wl)
        lay = layout_of(wl)
        ref = oracle.layer_fwd(lay, inp["Q"], inp["K"], inp["V"])
        _cache[name] = (wl, lay, inp, ref)
    return _cache[name]


def _dev(inp):
    return {k: inp[k].cuda() for k in ("Q", "K", "V")}


def _no_device_error():
    assert spava.device_error() == 0


@pytest.mark.parametrize("name", list(CASES))
def test_score_stage(name):
    wl, lay, inp, ref = _case(name)
    p = spava.Problem.from_workload(wl)
    d = _dev(inp)
    qsum, scores = spava.score(p, d["Q"], d["K"])
    torch.cuda.synchronize()
    s = to_np(scores)
    col = 0
    for h in range(lay.V - 1):
        r = ref["scores"][h]
        L = lay.block_lens[h]
        tol = 1e-5 * np.abs(r).max() + 1e-4
        assert max_err(s[:, col:col + L], r) <= tol, f"block {h}"
        col += L
    assert col == s.shape[1]
    _no_device_error()


@pytest.mark.parametrize("name", list(CASES))
def test_topk_stage_on_oracle_scores_is_exact(name):
    """Both sides decide on the same fp32 scores, so the sets are bit-exact."""
    wl, lay, inp, ref = _case(name)
    if wl.lp == 0:
        pytest.skip("lp = 0 selects nothing")
    p = spava.Problem.from_workload(wl)
    s32 = np.concatenate([np.asarray(ref["scores"][h], dtype=np.float32) for h in range(lay.V - 1)], axis=1)
    idx = to_np(spava.select_topk(p, torch.from_numpy(np.ascontiguousarray(s32)).cuda()))
    for h in range(lay.V - 1):
        e = lay.lp_eff(h)
        for kv in range(lay.num_kv_heads):
            assert np.array_equal(idx[h, kv, :e], ref["idx"][h][kv]), f"block {h} kv {kv}"
            assert np.all(idx[h, kv, e:] == -1)
    _no_device_error()


@pytest.mark.parametrize("L,lp,seed", [(1, 1, 0), (7, 3, 1), (1000, 1, 2), (1000, 999, 3),
                                        (4096, 512, 4), (16384, 2048, 5), (5000, 6000, 6),
                                        (3000, 64, 7)])
def test_topk_ties_signed_zero_and_clamp(L, lp, seed):
    """Planted ties, repeated maxima and +-0.0 against the oracle's rule."""
    s = W.random_scores(L, 2, seed)
    p = spava.Problem(1, 0, [L, 1], 1, lp, 2, 2, 64)
    idx = to_np(spava.select_topk(p, s.cuda().contiguous()))
    for kv in range(2):
        want = oracle.top_lp(s[kv].numpy(), lp)
        e = min(lp, L)
        assert np.array_equal(idx[0, kv, :e], want)
        assert np.all(idx[0, kv, e:] == -1)
    _no_device_error()


@pytest.mark.parametrize("name", list(CASES))
def test_gather_stage_exact(name):
    wl, lay, inp, ref = _case(name)
    if wl.lp == 0:
        pytest.skip("lp = 0 gathers nothing")
    p = spava.Problem.from_workload(wl)
    d = _dev(inp)
    idx = np.full((lay.V - 1, lay.num_kv_heads, wl.lp), -1, dtype=np.int32)
    for h in range(lay.V - 1):
        for kv in range(lay.num_kv_heads):
            idx[h, kv, :lay.lp_eff(h)] = ref["idx"][h][kv]
    Kp, Vp = spava.gather_passing(p, d["K"], d["V"], torch.from_numpy(idx).cuda())
    Kr, Vr = oracle.gather_passing(lay, inp["K"], inp["V"], ref["idx"])
    assert np.array_equal(to_np(Kp), Kr) and np.array_equal(to_np(Vp), Vr)
    _no_device_error()


def _oracle_passing_dev(lay, inp, ref, hkv, d):
    Kr, Vr = oracle.gather_passing(lay, inp["K"], inp["V"], ref["idx"])
    if Kr.shape[0] == 0:
        return None, None
    return (torch.from_numpy(Kr).to(torch.bfloat16).cuda().contiguous(),
            torch.from_numpy(Vr).to(torch.bfloat16).cuda().contiguous())


@pytest.mark.parametrize("name", list(CASES))
def test_fused_compress_stage(name):
    """Scores, top-lp indices and the passing buffer from the fused
    compression against the oracle (indices exact up to near-ties; passing
    rows exact wherever the selection is)."""
    wl, lay, inp, ref = _case(name)
    if wl.lp == 0:
        pytest.skip("lp = 0 compresses nothing")
    p = spava.Problem.from_workload(wl)
    d = _dev(inp)
    qsum, scores, idx, Kp, Vp = spava.compress(p, d["Q"], d["K"], d["V"])
    torch.cuda.synchronize()
    _no_device_error()
    s = to_np(scores)
    col = 0
    for h in range(lay.V - 1):
        r = ref["scores"][h]
        L = lay.block_lens[h]
        assert max_err(s[:, col:col + L], r) <= 1e-5 * np.abs(r).max() + 1e-4, f"block {h}"
        col += L
    swaps, affected = compare_selection(lay, ref["scores"], ref["idx"], to_np(idx))
    Kr, Vr = oracle.gather_passing(lay, inp["K"], inp["V"], ref["idx"])
    Kn, Vn = to_np(Kp), to_np(Vp)
    off = 0
    for h in range(lay.V - 1):
        e = lay.lp_eff(h)
        for kv in range(lay.num_kv_heads):
            if not affected[h][kv]:
                assert np.array_equal(Kn[off:off + e, kv], Kr[off:off + e, kv]), (h, kv)
                assert np.array_equal(Vn[off:off + e, kv], Vr[off:off + e, kv]), (h, kv)
        off += e


@pytest.mark.parametrize("name", list(CASES))
def test_fused_compress_scores_equal_the_scoring_stage(name):
    """Both paths start with the same query-sum kernel and reduce each dot
    product in the same order, so qsum and the scores agree bit for bit (and
    with them the selection)."""
    wl, lay, inp, ref = _case(name)
    if wl.lp == 0:
        pytest.skip("lp = 0 compresses nothing")
    p = spava.Problem.from_workload(wl)
    d = _dev(inp)
    qsum_s, scores_s = spava.score(p, d["Q"], d["K"])
    idx_s = spava.select_topk(p, scores_s)
    qsum_f, scores_f, idx_f, _, _ = spava.compress(p, d["Q"], d["K"], d["V"])
    torch.cuda.synchronize()
    _no_device_error()
    assert torch.equal(qsum_s, qsum_f)
    assert torch.equal(scores_s, scores_f)
    assert torch.equal(idx_s, idx_f)


@pytest.mark.parametrize("L,lp,seed", [(5, 2, 0), (1000, 37, 1), (4096, 512, 2), (8191, 1, 3),
                                        (20000, 3000, 4), (12288, 12287, 5)])
def test_fused_compress_ties_and_sizes(L, lp, seed):
    """Keys engineered to tie exactly (only four distinct key rows, repeated
    across every CTA slice), odd lengths and lp near L: the fused selection
    equals the oracle's rule on the oracle's own scores (identical rows tie
    exactly on both sides; distinct rows are far apart)."""
    g = torch.Generator().manual_seed(seed)
    hq, hkv, d, lq = 2, 1, 128, 3
    la = 8
    blocks = [L, 7]
    n = la + sum(blocks) + lq
    Q = torch.randn(n, hq, d, generator=g).to(torch.bfloat16)
    K = torch.randn(n, hkv, d, generator=g).to(torch.bfloat16)
    V = torch.randn(n, hkv, d, generator=g).to(torch.bfloat16)
    rows = torch.randint(0, 4, (L,), generator=g)
    K[la:la + L] = K[la:la + 4][rows]
    lay = oracle.make_layout(1, la, blocks, lq, lp, hq, hkv, d)
    ref_s = oracle.importance_scores(lay, Q, K, 0)[0]
    want = oracle.top_lp(ref_s.astype(np.float32), lp)
    p = spava.Problem(1, la, blocks, lq, lp, hq, hkv, d)
    _, scores, idx, Kp, Vp = spava.compress(p, Q.cuda(), K.cuda(), V.cuda())
    assert max_err(to_np(scores)[0], ref_s) <= 1e-5 * np.abs(ref_s).max() + 1e-4
    got = to_np(idx)[0, 0]
    e = min(lp, L)
    assert np.array_equal(got[:e], want)
    assert np.all(got[e:] == -1)
    assert np.array_equal(to_np(Kp)[:e, 0], K[la + want, 0].float().numpy())
    assert np.array_equal(to_np(Vp)[:e, 0], V[la + want, 0].float().numpy())
    _no_device_error()


@pytest.mark.parametrize("name", list(CASES))
def test_attention_stage(name):
    """Attention on the oracle's passing buffer: context/anchor rows and the
    per-host query partials."""
    wl, lay, inp, ref = _case(name)
    p = spava.Problem.from_workload(wl)
    d = _dev(inp)
    Kp, Vp = _oracle_passing_dev(lay, inp, ref, wl.num_kv_heads, wl.head_dim)
    O, lse, O_part, lse_part = spava.attn_fwd(p, d["Q"], d["K"], d["V"], Kp, Vp)
    torch.cuda.synchronize()
    _no_device_error()
    qs = lay.query_start
    assert max_err(to_np(O)[:qs], ref["O"][:qs]) <= O_TOL
    assert max_err(to_np(lse)[:, :qs], ref["lse"][:, :qs]) <= LSE_TOL
    assert max_err(to_np(O_part), ref["o_part"]) <= O_TOL
    assert max_err(to_np(lse_part), ref["lse_part"]) <= LSE_TOL


@pytest.mark.parametrize("name", list(CASES))
def test_merge_stage(name):
    wl, lay, inp, ref = _case(name)
    p = spava.Problem.from_workload(wl)
    n = lay.n
    O = torch.zeros(n, wl.num_q_heads, wl.head_dim, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(wl.num_q_heads, n, dtype=torch.float32, device="cuda")
    op = torch.from_numpy(ref["o_part"].astype(np.float32)).cuda().contiguous()
    lp_ = torch.from_numpy(ref["lse_part"].astype(np.float32)).cuda().contiguous()
    spava.lse_merge(p, op, lp_, O, lse)
    torch.cuda.synchronize()
    qs = lay.query_start
    assert max_err(to_np(O)[qs:], ref["O"][qs:]) <= O_TOL
    assert max_err(to_np(lse)[:, qs:], ref["lse"][:, qs:]) <= LSE_TOL
    assert np.all(to_np(O)[:qs] == 0)            # rows outside the query block untouched
    _no_device_error()


@pytest.mark.parametrize("name", list(CASES))
def test_layer_fwd(name):
    """The whole layer against the oracle, every row and head.  Where the
    layer's top-lp set differs from the oracle's only at tolerated near-ties,
    the affected hosts' rows are compared with the oracle recomputed on the
    layer's own selection (both selections are valid there)."""
    wl, lay, inp, ref = _case(name)
    p = spava.Problem.from_workload(wl)
    d = _dev(inp)
    O, lse = spava.layer_fwd(p, d["Q"], d["K"], d["V"])
    torch.cuda.synchronize()
    _no_device_error()
    On, ln = to_np(O), to_np(lse)
    affected = {h: {kv: False for kv in range(lay.num_kv_heads)} for h in range(lay.V - 1)}
    sel = np.zeros((lay.V - 1, lay.num_kv_heads, wl.lp), dtype=np.int32)
    if wl.lp > 0:
        # the layer's own selection (the fused compression it runs)
        _, scores, idx, _, _ = spava.compress(p, d["Q"], d["K"], d["V"])
        sel = to_np(idx)
        swaps, affected = compare_selection(lay, ref["scores"], ref["idx"], sel)
    check_rows(lay, inp, sel, affected, range(lay.n), list(range(wl.num_q_heads)),
               On, ln, ref["O"], ref["lse"])


def test_layer_is_deterministic_and_stream_ordered():
    wl, lay, inp, ref = _case("frames_multi")
    p = spava.Problem.from_workload(wl)
    d = _dev(inp)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        O1, l1 = spava.layer_fwd(p, d["Q"], d["K"], d["V"], stream=s)
        O2, l2 = spava.layer_fwd(p, d["Q"], d["K"], d["V"], stream=s)
    s.synchronize()
    assert torch.equal(O1, O2) and torch.equal(l1, l2)
    _no_device_error()


def test_bad_arguments_are_rejected_before_launch():
    wl, lay, inp, ref = _case("tiny")
    p = spava.Problem.from_workload(wl)
    d = _dev(inp)
    with pytest.raises(spava.SpavaError) as e:
        spava.layer_fwd(p, d["Q"], d["K"], d["V"],
                        workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.code == 3   # SPAVA_ERR_WORKSPACE
    lib = spava.lib()
    import ctypes
    r = lib.spava_layer_fwd(p.ref, None, ctypes.c_void_p(d["K"].data_ptr()), ctypes.c_void_p(d["V"].data_ptr()),
                            None, None, None, ctypes.c_size_t(0), None)
    assert r == 1              # SPAVA_ERR_INVALID_ARG
    mis = ctypes.c_void_p(d["Q"].data_ptr() + 2)
    ws = torch.empty(spava.workspace_size(p), dtype=torch.uint8, device="cuda")
    O = torch.empty_like(d["Q"])
    lse = torch.empty(wl.num_q_heads, lay.n, device="cuda")
    r = lib.spava_attn_fwd(p.ref, mis, ctypes.c_void_p(d["K"].data_ptr()), ctypes.c_void_p(d["V"].data_ptr()),
                           ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                           ctypes.c_void_p(O.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
                           ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(ws.data_ptr()), None)
    assert r == 1              # misaligned Q
    _no_device_error()


def test_layer_long_block_fallback():
    """A context block longer than the fused compression takes (24576
    keys): the layer runs the three stage kernels for steps 1-3 instead, then
    the same attention launch.  Scores and indices are checked in full, rows
    on samples the oracle computes one by one."""
    wl = small_workload("long_block", 16, (100000, 64), 8, 128, 2, 1, 64, seed=9)
    lay = layout_of(wl)
    inp = W.make_inputs(wl)
    p = spava.Problem.from_workload(wl)
    d = _dev(inp)
    O, lse = spava.layer_fwd(p, d["Q"], d["K"], d["V"])
    _, scores = spava.score(p, d["Q"], d["K"])              # the stage kernels the layer ran
    idx = to_np(spava.select_topk(p, scores))
    torch.cuda.synchronize()
    _no_device_error()
    ref_scores, ref_idx = oracle.compress(lay, inp["Q"], inp["K"])
    s = to_np(scores)
    assert max_err(s[:, :100000], ref_scores[0]) <= 1e-5 * np.abs(ref_scores[0]).max() + 1e-4
    swaps, affected = compare_selection(lay, ref_scores, ref_idx, idx)
    s0 = lay.block_starts[0]
    rng = np.random.default_rng(3)
    rows = list(range(16)) + list(range(s0, s0 + 16)) + list(range(s0 + 100000 - 16, s0 + 100000)) + \
        sorted(set(int(x) for x in rng.integers(s0, s0 + 100000, 16))) + \
        list(range(lay.block_starts[1], lay.block_starts[1] + 64)) + list(range(lay.query_start, lay.n))
    heads = [0, 1]
    got_rows, o_ref, l_ref = oracle.rows_fwd(lay, inp["Q"], inp["K"], inp["V"], ref_idx, rows, heads)
    r = torch.as_tensor(got_rows).cuda()
    On = O[r][:, heads].float().cpu().numpy().astype(np.float64)
    Ln = lse[heads][:, r].cpu().numpy()
    check_rows(lay, inp, idx, affected, got_rows, heads, On, Ln, o_ref, l_ref)


# ---------------------------------------------------------------- selector variants
# The variants' scores come from two passes on the GPU (the attention kernel's
# lse over the block, then exp(logit - lse) summed per key), both with fp32
# exp2 approximations: scores agree with the oracle to 1e-3 of the block's
# largest score, and selections differ at most at near-ties within that bound.
VARIANT_TIE_REL = 1e-3
VARIANT_CASES = ["ragged_d128", "frames_multi", "no_anchor_d64", "dense_unequal_g1"]


@pytest.mark.parametrize("kind", ["softmax", "context"])
@pytest.mark.parametrize("name", VARIANT_CASES)
def test_score_variant_against_oracle(name, kind):
    wl, lay, inp, ref = _case(name)
    p = spava.Problem.from_workload(wl, score_kind=kind)
    d = _dev(inp)
    scores = spava.score_variant(p, d["Q"], d["K"])
    idx = to_np(spava.select_topk(p, scores))
    torch.cuda.synchronize()
    _no_device_error()
    s = to_np(scores)
    ref_scores, ref_idx = oracle.compress_with(lay, inp["Q"], inp["K"], kind)
    col = 0
    for h in range(lay.V - 1):
        r = ref_scores[h]
        L = lay.block_lens[h]
        assert max_err(s[:, col:col + L], r) <= VARIANT_TIE_REL * np.abs(r).max(), (kind, h)
        col += L
    compare_selection(lay, ref_scores, ref_idx, idx, tie_rel=VARIANT_TIE_REL)


@pytest.mark.parametrize("kind", ["softmax", "context"])
def test_layer_with_score_variant(kind):
    """The whole layer under a selector variant: every row and head against the
    oracle run with the same selector (rows of hosts whose selection differs at
    a near-tie are recomputed on the layer's own selection)."""
    wl, lay, inp, _ = _case("frames_multi")
    p = spava.Problem.from_workload(wl, score_kind=kind)
    d = _dev(inp)
    O, lse = spava.layer_fwd(p, d["Q"], d["K"], d["V"])
    scores = spava.score_variant(p, d["Q"], d["K"])
    sel = to_np(spava.select_topk(p, scores))
    torch.cuda.synchronize()
    _no_device_error()
    ref_scores, ref_idx = oracle.compress_with(lay, inp["Q"], inp["K"], kind)
    _, affected = compare_selection(lay, ref_scores, ref_idx, sel, tie_rel=VARIANT_TIE_REL)
    rows = list(range(lay.n))
    heads = list(range(wl.num_q_heads))
    got_rows, o_ref, l_ref = oracle.rows_fwd(lay, inp["Q"], inp["K"], inp["V"], ref_idx, rows, heads)
    check_rows(lay, inp, sel, affected, got_rows, heads, to_np(O).astype(np.float64), to_np(lse), o_ref, l_ref)


def test_bounded_wait_gives_up_reports_and_leaves_the_context_usable():
    """A wait on an mbarrier that nothing completes (the kernels' own bounded
    waits, with a 2 ms limit) gives up, raises the abort flag and sets the
    device error word; the next device_error() reads it and clears it, and the
    layer then still runs correctly."""
    assert spava.device_error() == 0
    w, ab, dr, ns = spava.debug_wait_timeout(2_000_000)
    assert (w, ab, dr) == (0, 1, 0)
    assert 3_000_000 <= ns < 1_000_000_000
    assert spava.device_error() == 1
    assert spava.device_error() == 0
    wl, lay, inp, ref = _case("tiny")
    d = _dev(inp)
    O, lse = spava.layer_fwd(spava.Problem.from_workload(wl), d["Q"], d["K"], d["V"])
    torch.cuda.synchronize()
    _no_device_error()
    assert max_err(to_np(O).astype(np.float64), ref["O"]) <= O_TOL
    assert max_err(to_np(lse), ref["lse"]) <= LSE_TOL


@pytest.mark.parametrize("name", ["frames_multi", "pair_lq1_d64"])
def test_attention_abort_path_drains_and_leaves_the_context_usable(name):
    """The attention kernel's own abort path: with key tile 1 left unloaded
    and every wait limited to 50 ms, the CTAs that reach the tile give up,
    drain what is in flight, free TMEM and set the device error word; the
    same attention then runs correctly on the same context."""
    wl, lay, inp, ref = _case(name)
    p = spava.Problem.from_workload(wl)
    d = _dev(inp)
    Kp, Vp = _oracle_passing_dev(lay, inp, ref, wl.num_kv_heads, wl.head_dim)
    _no_device_error()
    spava.debug_attn_abort(p, d["Q"], d["K"], d["V"], Kp, Vp, skip_k_tile=1, limit_ns=50_000_000)
    torch.cuda.synchronize()
    assert spava.device_error() == 1
    O, lse, O_part, lse_part = spava.attn_fwd(p, d["Q"], d["K"], d["V"], Kp, Vp)
    torch.cuda.synchronize()
    _no_device_error()
    qs = lay.query_start
    assert max_err(to_np(O)[:qs], ref["O"][:qs]) <= O_TOL
    assert max_err(to_np(lse)[:, :qs], ref["lse"][:, :qs]) <= LSE_TOL
    assert max_err(to_np(O_part), ref["o_part"]) <= O_TOL
