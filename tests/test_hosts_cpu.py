"""The pages' split of the layer over GPUs (hosts.py), on CPU: which ranks
hold which virtual hosts, the per-rank attention work, and the two collective
steps (passing rows, query partials) between gloo ranks.  The kernels are
stood in for by the fp64 oracle, restricted to each rank's hosts, so what is
checked is the plumbing: every rank ends with the whole passing buffer and
the merged query rows of the single-process layer."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import spava_oracle as oracle
from sparse_approximate_attention_b200 import hosts, spava


@pytest.mark.parametrize("H", range(1, 9))
def test_ranks_partition_the_virtual_hosts_in_zigzag_pairs(H):
    V = 2 * H
    for world in range(1, H + 1):
        seen = []
        for r in range(world):
            hs = hosts.rank_virtual_hosts(H, world, r)
            for h in hs:   # every host comes with its ZigZag partner
                assert V - 1 - h in hs
            seen += hs
            assert hosts.host_mask(H, world, r) == sum(1 << h for h in hs)
        assert sorted(seen) == list(range(V))


def test_rank_masks_split_the_attention_work_exactly():
    """The selected rows' FLOPs (spava_problem_sizes, no CUDA call) of the
    ranks add up to the whole layer's, and ZigZag pairs balance them."""
    p = spava.Problem(4, 96, [300, 257, 512, 128, 640, 333, 256, 700], 77, 40, 8, 2, 128)
    full = p.sizes()["attn_flops"]
    for world in (1, 2, 4):
        parts = [p.with_hosts(hosts.host_mask(4, world, r)).sizes()["attn_flops"] for r in range(world)]
        assert sum(parts) == full
    eq = spava.Problem(4, 1024, [8192] * 8, 128, 1024, 16, 2, 128)
    parts = [eq.with_hosts(hosts.host_mask(4, 4, r)).sizes()["attn_flops"] for r in range(4)]
    assert max(parts) / min(parts) < 1.01


def test_masks_beyond_the_hosts_are_rejected():
    p = spava.Problem(2, 16, [32, 32, 32, 32], 8, 4, 2, 1, 64, host_mask=1 << 4)
    with pytest.raises(spava.SpavaError):
        p.sizes()


class OracleKernels:
    """compress / attn_fwd / lse_merge with the library's host-mask semantics,
    computed by the oracle on the full problem and written only where the
    mask says."""

    def __init__(self, lay, Q, K, V):
        self.lay = lay
        self.full = oracle.layer_fwd(lay, Q, K, V)
        self.Kp, self.Vp = oracle.gather_passing(lay, K, V, self.full["idx"])
        self.off = np.cumsum([0] + [lay.lp_eff(h) for h in range(lay.V - 1)])

    def compress(self, q, Q, K, V, qsum, scores, idx, Kp, Vp, stream=None):
        for h in range(self.lay.V - 1):
            if q.host_mask >> h & 1:
                a, b = self.off[h], self.off[h + 1]
                Kp[a:b] = torch.from_numpy(self.Kp[a:b])
                Vp[a:b] = torch.from_numpy(self.Vp[a:b])

    def attn_fwd(self, q, Q, K, V, Kp, Vp, O, lse, O_part, lse_part, stream=None):
        lay = self.lay
        for h in range(lay.V):
            if not (q.host_mask >> h & 1):
                continue
            s0 = lay.block_starts[h]
            rows = slice(s0, s0 + lay.block_lens[h])
            O[rows] = torch.from_numpy(self.full["O"][rows])
            lse[:, rows] = torch.from_numpy(self.full["lse"][:, rows])
            O_part[h] = torch.from_numpy(self.full["o_part"][h])
            lse_part[h] = torch.from_numpy(self.full["lse_part"][h])
        if lay.anchor_len and (q.host_mask & 1):
            O[: lay.anchor_len] = torch.from_numpy(self.full["O"][: lay.anchor_len])
            lse[:, : lay.anchor_len] = torch.from_numpy(self.full["lse"][:, : lay.anchor_len])

    def lse_merge(self, p, O_part, lse_part, O, lse, stream=None):
        qo, ql = oracle.lse_merge(O_part.numpy(), lse_part.numpy().transpose(0, 2, 1))
        qs = self.lay.query_start
        O[qs:] = torch.from_numpy(qo)
        lse[:, qs:] = torch.from_numpy(ql.T)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASE = dict(num_hosts=4, anchor_len=12, block_lens=[40, 23, 37, 31, 29, 44, 26, 35], query_len=9,
            lp=6, num_q_heads=4, num_kv_heads=2, head_dim=64)


def _inputs():
    g = torch.Generator().manual_seed(77)
    n = CASE["anchor_len"] + sum(CASE["block_lens"]) + CASE["query_len"]
    mk = lambda h: torch.randn(n, h, CASE["head_dim"], generator=g, dtype=torch.float64)
    return mk(CASE["num_q_heads"]), mk(CASE["num_kv_heads"]), mk(CASE["num_kv_heads"])


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lay = oracle.make_layout(**CASE)
        Q, K, V = _inputs()
        p = spava.Problem(**CASE)
        kern = OracleKernels(lay, Q, K, V)
        layer = hosts.HostShardedLayer(p, world, rank, "cpu", kernels=kern,
                                       dtypes=(torch.float64, torch.float64))
        n, hq, d = lay.n, lay.num_q_heads, lay.head_dim
        O = torch.full((n, hq, d), float("nan"), dtype=torch.float64)
        lse = torch.full((hq, n), float("nan"), dtype=torch.float64)
        layer.forward(Q, K, V, O, lse)
        ok_kp = np.array_equal(layer.Kp.numpy(), kern.Kp) and np.array_equal(layer.Vp.numpy(), kern.Vp)
        rows = [r for rg in layer.owned_rows() for r in rg] + list(range(lay.query_start, n))
        err_o = float(np.abs(O.numpy()[rows] - kern.full["O"][rows]).max())
        err_l = float(np.abs(lse.numpy()[:, rows] - kern.full["lse"][:, rows]).max())
        out[rank] = (ok_kp, err_o, err_l, len(rows))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 5])
def test_gloo_ranks_exchange_passing_rows_and_query_partials(world):
    """world 5 > H = 4: rank 4 holds no host, computes nothing and still takes
    part in both all-gathers."""
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    lay = oracle.make_layout(**CASE)
    total = 0
    for r in range(world):
        ok_kp, err_o, err_l, nrows = out[r]
        assert ok_kp, f"rank {r}: passing buffer differs from the single-process gather"
        assert err_o < 1e-12 and err_l < 1e-12, (r, err_o, err_l)
        total += nrows - lay.query_len
    assert total == lay.n - lay.query_len   # the ranks' own rows cover the sequence once
