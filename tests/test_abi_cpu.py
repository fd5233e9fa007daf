"""CPU-side checks of the C ABI: the library loads without a GPU, exports
every entry point the header declares, and its host logic (validation,
context splitting, FLOP count, workspace size) agrees with the oracle."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import sparse_approximate_attention_b200 as spava
from sparse_approximate_attention_b200 import build as B
from sparse_approximate_attention_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def _declared():
    txt = open(os.path.join(ROOT, "include", "spava.h")).read()
    return sorted(set(re.findall(r"^\s*(?:spava_status_t|const char\*)\s+(spava_\w+)\s*\(", txt, re.M)))


def test_header_declares_the_entry_points():
    names = _declared()
    for must in ("spava_score", "spava_select_topk", "spava_gather_passing", "spava_attn_fwd",
                 "spava_lse_merge", "spava_layer_fwd", "spava_workspace_size",
                 "spava_problem_sizes", "spava_device_error", "spava_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(B.LIB)
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings():
    lib = spava.lib()
    for code, name in spava.spava.STATUS.items():
        assert lib.spava_status_string(code).decode() == name


@pytest.mark.parametrize("name", list(W.workloads()))
def test_sizes_match_oracle(name):
    wl = W.workloads()[name]
    lay = oracle.make_layout(wl.num_hosts, wl.anchor_len, wl.block_lens, wl.query_len, wl.lp,
                             wl.num_q_heads, wl.num_kv_heads, wl.head_dim)
    sz = spava.Problem.from_workload(wl).sizes()
    assert sz["seq_len"] == lay.n
    assert sz["query_start"] == lay.query_start
    assert sz["score_cols"] == sum(lay.block_lens[:-1])
    assert sz["passing_rows"] == sum(lay.lp_eff(h) for h in range(lay.V - 1))
    assert int(sz["attn_flops"]) == oracle.flops(lay)
    assert sz["workspace_bytes"] > 0


def test_sizes_random_layouts_match_oracle_count():
    rng = np.random.default_rng(1)
    for _ in range(200):
        H = int(rng.integers(1, 5))
        blocks = [int(x) for x in rng.integers(1, 400, size=2 * H)]
        la, lq, lp = int(rng.integers(0, 300)), int(rng.integers(1, 300)), int(rng.integers(0, 500))
        hkv = int(rng.integers(1, 4))
        hq = hkv * int(rng.integers(1, 4))
        d = int(rng.choice([64, 128]))
        lay = oracle.make_layout(H, la, blocks, lq, lp, hq, hkv, d)
        sz = spava.Problem(H, la, blocks, lq, lp, hq, hkv, d).sizes()
        assert int(sz["attn_flops"]) == oracle.flops(lay)
        assert sz["attn_tiles"] == sum(-(-L // 128) for L in blocks) + (-(-la // 128)) + 2 * H * (-(-lq // 128))


@pytest.mark.parametrize("kw,code", [
    (dict(num_hosts=0), 1), (dict(num_hosts=17), 1), (dict(anchor_len=-1), 1),
    (dict(query_len=0), 1), (dict(lp=-1), 1), (dict(num_q_heads=3, num_kv_heads=2), 1),
    (dict(head_dim=96), 2), (dict(block_lens=[4, 0]), 1),
])
def test_invalid_problems_rejected(kw, code):
    base = dict(num_hosts=1, anchor_len=4, block_lens=[4, 4], query_len=2, lp=2, num_q_heads=2,
                num_kv_heads=1, head_dim=64)
    base.update(kw)
    if "num_hosts" in kw and kw["num_hosts"] > 0:
        base["block_lens"] = [4] * (2 * kw["num_hosts"])
    p = spava.Problem(**base)
    with pytest.raises(spava.SpavaError) as e:
        p.sizes()
    assert e.value.code == code


def test_null_problem_and_null_block_lens():
    lib = spava.lib()
    s = spava.spava._Sizes()
    assert lib.spava_problem_sizes(None, ctypes.byref(s)) == 1
    p = spava.Problem(1, 4, [4, 4], 2, 2, 2, 1, 64)
    p._c.block_lens = ctypes.POINTER(ctypes.c_int32)()
    assert lib.spava_problem_sizes(p.ref, ctypes.byref(s)) == 1


def test_too_many_tiles_is_unsupported_not_a_crash():
    """A layer whose attention work list exceeds the launch's capacity is
    refused before anything is launched or dereferenced (the pointers below
    are never touched; no GPU is needed)."""
    p = spava.Problem(16, 0, [65536] * 32, 16, 16, 2, 1, 128)   # ~2M rows -> > 6144 work items
    sz = p.sizes()
    assert sz["attn_tiles"] > 2 * 6144
    fake = ctypes.c_void_p(1 << 20)   # 256-byte aligned, never dereferenced
    r = spava.lib().spava_layer_fwd(p.ref, fake, fake, fake, fake, fake, fake,
                                    ctypes.c_size_t(sz["workspace_bytes"]), None)
    assert r == 2   # SPAVA_ERR_UNSUPPORTED
