"""The layer split over GPUs the way the pages deploy it.

"Spava ..." (sciencestack.ai), Fig. 2 and Fig. 4 captions: the context is
cut into 2H blocks on virtual hosts, and physical host p holds virtual hosts
p and 2H-1-p (the ZigZag pairing that evens out early, cheap blocks and late,
expensive ones).  "APB-V ..." (pith.science review), "What carries the
argument": each host compresses its block to its passing block, and the
passing blocks are all-gathered, so that host h attends to those of the hosts
before it; the query block's partial results of all hosts are merged through
their log-sum-exp ("Axiom & Free-Parameter Ledger": the merge is exact).

One process per GPU (torch.distributed; NCCL between GPUs, gloo on CPU).  The
physical hosts are dealt to the ranks round-robin (p % world == rank), so a
rank holds whole ZigZag pairs; with more ranks than physical hosts the extra
ranks hold none and only take part in the collectives.  Per layer every rank
  1. compresses its own context blocks (spava_compress with its host mask):
     their scores, indices and passing rows, at their offsets of the full
     passing buffer;
  2. all-gathers the passing rows of every rank into its passing buffer;
  3. runs the attention of its own hosts (spava_attn_fwd with its mask): its
     context rows (and the anchor rows on the rank holding host 0) and its
     hosts' query partials;
  4. all-gathers the query partials;
  5. merges all 2H partials into the query rows (spava_lse_merge), so every
     rank ends with the query rows; the other rows of O and lse are valid on
     the rank that owns them.
The collectives move only what the pages exchange: passing rows and query
partials.  This module is plumbing (packing, collectives, unpacking); every
arithmetic step runs in the library's kernels.
"""
from __future__ import annotations

from typing import List, Optional

import torch
import torch.distributed as dist

from . import spava


def rank_physical_hosts(num_hosts: int, world: int, rank: int) -> List[int]:
    """Physical hosts held by `rank`: p with p % world == rank."""
    return [p for p in range(num_hosts) if p % world == rank]


def rank_virtual_hosts(num_hosts: int, world: int, rank: int) -> List[int]:
    """Virtual hosts held by `rank`, ascending: p and 2H-1-p for each of its
    physical hosts p."""
    V = 2 * num_hosts
    return sorted(h for p in rank_physical_hosts(num_hosts, world, rank) for h in (p, V - 1 - p))


def host_mask(num_hosts: int, world: int, rank: int) -> int:
    """spava_problem_t.host_mask of `rank`."""
    m = 0
    for h in rank_virtual_hosts(num_hosts, world, rank):
        m |= 1 << h
    return m


class HostExchange:
    """The two collective steps of the split, for one problem and one process
    group: the all-gather of the passing rows and of the query partials.
    Every rank calls both, in the same order."""

    def __init__(self, p: "spava.Problem", world: int, rank: int, group=None):
        self.p, self.world, self.rank, self.group = p, world, rank, group
        V, lp = p.V, p.lp
        lens = p.block_lens
        lpe = [min(lp, L) for L in lens]
        off = [0]
        for h in range(V - 1):
            off.append(off[-1] + lpe[h])
        self.passing_rows = off[-1]
        # rows of the passing buffer each rank fills: its compressed blocks in ascending order
        self.rows_of = []
        for r in range(world):
            rows = []
            for h in rank_virtual_hosts(p.num_hosts, world, r):
                if h < V - 1:
                    rows.extend(range(off[h], off[h] + lpe[h]))
            self.rows_of.append(rows)
        self.chunk_rows = max(1, max(len(x) for x in self.rows_of))
        self.hosts_of = [rank_virtual_hosts(p.num_hosts, world, r) for r in range(world)]
        self.chunk_hosts = max(len(x) for x in self.hosts_of)
        self._idx = {}

    def _index(self, name, rows, device):
        key = (name, device)
        if key not in self._idx:
            self._idx[key] = torch.as_tensor(rows, dtype=torch.long, device=device)
        return self._idx[key]

    def _all_gather(self, chunk: torch.Tensor) -> torch.Tensor:
        """[world, *chunk.shape]: every rank's chunk, in rank order (gathered
        as one concatenation along dim 0, the form both NCCL and gloo take)."""
        if self.world == 1:
            return chunk.unsqueeze(0)
        out = torch.empty((self.world * chunk.shape[0],) + tuple(chunk.shape[1:]), dtype=chunk.dtype,
                          device=chunk.device)
        dist.all_gather_into_tensor(out, chunk.contiguous(), group=self.group)
        return out.view((self.world,) + tuple(chunk.shape))

    def exchange_passing(self, Kp: torch.Tensor, Vp: torch.Tensor) -> None:
        """Fill every rank's rows of Kp and Vp ([P, Hkv, d], this rank's own
        rows already written) with the rows the other ranks computed."""
        if self.passing_rows == 0:
            return
        dev = Kp.device
        mine = self.rows_of[self.rank]
        for buf in (Kp, Vp):
            chunk = torch.zeros((self.chunk_rows,) + tuple(buf.shape[1:]), dtype=buf.dtype, device=dev)
            if mine:
                chunk[: len(mine)] = buf.index_select(0, self._index(("own", self.rank), mine, dev))
            got = self._all_gather(chunk)
            for r in range(self.world):
                rows = self.rows_of[r]
                if r == self.rank or not rows:
                    continue
                buf.index_copy_(0, self._index(("dst", r), rows, dev), got[r, : len(rows)])

    def exchange_partials(self, O_part: torch.Tensor, lse_part: torch.Tensor) -> None:
        """Fill every host's query partial (O_part [V, lq, Hq, d], lse_part
        [V, Hq, lq]) from the rank that computed it."""
        dev = O_part.device
        mine = self.hosts_of[self.rank]
        for buf in (O_part, lse_part):
            chunk = torch.zeros((self.chunk_hosts,) + tuple(buf.shape[1:]), dtype=buf.dtype, device=dev)
            chunk[: len(mine)] = buf.index_select(0, self._index(("hown", self.rank), mine, dev))
            got = self._all_gather(chunk)
            for r in range(self.world):
                hs = self.hosts_of[r]
                if r == self.rank or not hs:
                    continue
                buf.index_copy_(0, self._index(("hdst", r), hs, dev), got[r, : len(hs)])


class HostShardedLayer:
    """The layer on `world` GPUs (one rank each): rank r computes the virtual
    hosts of host_mask(H, world, r).  `kernels` defaults to the library
    (spava.compress, spava.attn_fwd, spava.lse_merge); the buffers are
    allocated once on `device`, in the library's types (bf16 passing rows,
    fp32 partials) unless `dtypes` says otherwise."""

    def __init__(self, p: "spava.Problem", world: int, rank: int, device, group=None, kernels=None,
                 dtypes=(torch.bfloat16, torch.float32)):
        self.p, self.world, self.rank = p, world, rank
        self.mask = host_mask(p.num_hosts, world, rank)
        # a rank without hosts (world > H) computes nothing: host_mask 0 would mean "every host"
        self.idle = self.mask == 0
        self.q = p.with_hosts(self.mask)
        self.ex = HostExchange(p, world, rank, group)
        self.k = kernels if kernels is not None else spava
        sz = p.sizes()
        V, hq, hkv, d, lq, lp = p.V, p.num_q_heads, p.num_kv_heads, p.head_dim, p.query_len, p.lp
        bf, f32 = dtypes
        self.qsum = torch.empty(hkv, d, dtype=f32, device=device)
        self.scores = torch.empty(hkv, sz["score_cols"], dtype=f32, device=device)
        self.idx = torch.empty(V - 1, hkv, lp, dtype=torch.int32, device=device)
        rows = sz["passing_rows"]
        self.Kp = torch.empty(max(1, rows), hkv, d, dtype=bf, device=device)[:rows]
        self.Vp = torch.empty(max(1, rows), hkv, d, dtype=bf, device=device)[:rows]
        self.O_part = torch.empty(V, lq, hq, d, dtype=f32, device=device)
        self.lse_part = torch.empty(V, hq, lq, dtype=f32, device=device)

    def forward(self, Q, K, V, O, lse, stream=None) -> None:
        """O and lse: this rank's rows (its hosts' context rows, the anchor rows
        on the rank of host 0) and, on every rank, the query rows."""
        if self.p.lp > 0 and not self.idle:
            self.k.compress(self.q, Q, K, V, self.qsum, self.scores, self.idx, self.Kp, self.Vp, stream=stream)
        self.ex.exchange_passing(self.Kp, self.Vp)
        if not self.idle:
            self.k.attn_fwd(self.q, Q, K, V, self.Kp if self.p.lp else None, self.Vp if self.p.lp else None,
                            O, lse, self.O_part, self.lse_part, stream=stream)
        self.ex.exchange_partials(self.O_part, self.lse_part)
        self.k.lse_merge(self.p, self.O_part, self.lse_part, O, lse, stream=stream)

    def owned_rows(self) -> List[range]:
        """Row ranges of O / lse this rank computes (besides the query rows)."""
        p = self.p
        starts = [p.anchor_len]
        for L in p.block_lens:
            starts.append(starts[-1] + L)
        out = []
        if p.anchor_len and (self.mask & 1):
            out.append(range(0, p.anchor_len))
        for h in rank_virtual_hosts(p.num_hosts, self.world, self.rank):
            out.append(range(starts[h], starts[h + 1]))
        return out
