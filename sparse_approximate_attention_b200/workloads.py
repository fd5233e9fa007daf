"""Seeded synthetic inputs for the approximate-attention prefill layer.

This module only draws random tensors in the shapes of the long-video
workloads the Spava / APB-V pages describe (Qwen2.5-VL-3B/7B-shaped attention
layers, anchor + 2H context blocks + a short text query).  It holds none of
the layer's arithmetic: no scores, no selection, no attention.  Both the
CUDA path's tests/bench and the CPU oracle take their inputs from here.

Layouts (token-major, sequence order ``A | B^0 .. B^{V-1} | B_qr``):
    Q : [n, Hq,  d] bf16
    K : [n, Hkv, d] bf16
    V : [n, Hkv, d] bf16

Every tensor is produced on the CPU from a ``torch.Generator`` seeded with the
workload's seed, so the same seed gives the same bytes on any machine with the
same torch build.
"""
from __future__ import annotations

from dataclasses import dataclass, field, asdict
from typing import Dict, List, Optional

import torch

FRAME_TOKENS = 1024   # tokens per video frame in the long-video generator
FRAME_RANK = 16       # rank of the per-frame key/value embedding
NOISE = 0.3           # isotropic noise added to the low-rank frame part
QR_HIT_FRACTION = 0.02  # fraction of context keys the text query correlates with
TEXT_NEEDLES = 16       # needle keys per KV head in the text generator


@dataclass
class Workload:
    """One synthetic prefill-layer problem.

    num_hosts   H physical hosts; V = 2H virtual hosts = context blocks
    anchor_len  la, tokens in the anchor block B_a
    block_lens  L_h for the 2H context blocks B^(h)
    query_len   lq, tokens in the query block B_qr
    lp          passing length (top-lp keys kept per block and KV head)
    """
    name: str
    num_hosts: int
    anchor_len: int
    block_lens: List[int]
    query_len: int
    lp: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    generator: str = "gaussian"       # "gaussian" | "needles" | "frames" | "text"
    seed: int = 0
    description: str = ""
    extra: Dict = field(default_factory=dict)

    @property
    def num_virtual(self) -> int:
        return 2 * self.num_hosts

    @property
    def seq_len(self) -> int:
        return self.anchor_len + sum(self.block_lens) + self.query_len

    def with_(self, **kw) -> "Workload":
        d = asdict(self)
        d.update(kw)
        return Workload(**d)


def _unequal_blocks(seed: int, count: int, total: int, lo: int, hi: int) -> List[int]:
    """Block lengths drawn uniformly in [lo, hi] with a fixed total; the last
    block takes the remainder and the draw repeats until it lands in range."""
    g = torch.Generator().manual_seed(seed)
    for _ in range(10000):
        head = torch.randint(lo, hi + 1, (count - 1,), generator=g).tolist()
        last = total - sum(head)
        if lo <= last <= hi:
            return head + [last]
    raise RuntimeError("could not draw block lengths")


def workloads() -> Dict[str, Workload]:
    """The named synthetic workloads (sizes from the long-video settings)."""
    w = {}
    w["tiny"] = Workload(
        "tiny", num_hosts=2, anchor_len=64, block_lens=[256] * 4, query_len=32,
        lp=32, num_q_heads=2, num_kv_heads=1, head_dim=64, generator="needles",
        seed=1235, description="H=2/V=4, 2 q heads / 1 kv head, d=64, "
        "anchor 64 + 4x256 + query 32, lp=32, 8 planted needle keys per block")
    w["qwen25vl3b_64f"] = Workload(
        "qwen25vl3b_64f", num_hosts=4, anchor_len=1024, block_lens=[8192] * 8,
        query_len=128, lp=1024, num_q_heads=16, num_kv_heads=2, head_dim=128,
        generator="frames", seed=1236,
        description="Qwen2.5-VL-3B-shaped layer, 64 frames x 1024 tokens, "
        "H=4/V=8, anchor 1024 + 8x8192 + query 128, lp=1024")
    w["qwen25vl7b_128k"] = Workload(
        "qwen25vl7b_128k", num_hosts=4, anchor_len=2048, block_lens=[16384] * 8,
        query_len=256, lp=2048, num_q_heads=28, num_kv_heads=4, head_dim=128,
        generator="frames", seed=1237,
        description="Qwen2.5-VL-7B-shaped layer, ~128K tokens, H=4/V=8, "
        "anchor 2048 + 8x16384 + query 256, lp=2048")
    for lp in (512, 2048, 4096):
        nm = f"longvideo_256k_lp{lp}"
        w[nm] = Workload(
            nm, num_hosts=8, anchor_len=2048, block_lens=[16384] * 16,
            query_len=256, lp=lp, num_q_heads=28, num_kv_heads=4, head_dim=128,
            generator="frames", seed=1238,
            description=f"long-video stress, H=8/V=16, anchor 2048 + 16x16384 "
            f"+ query 256, lp={lp}")
    w["exact_dense_3b"] = Workload(
        "exact_dense_3b", num_hosts=4, anchor_len=1024, block_lens=[8192] * 8,
        query_len=128, lp=8192, num_q_heads=16, num_kv_heads=2, head_dim=128,
        generator="frames", seed=1239,
        description="3B shape with lp = full block length (dense-exact)")
    w["qwen25vl3b_h2"] = Workload(
        "qwen25vl3b_h2", num_hosts=2, anchor_len=1024, block_lens=[8192] * 4,
        query_len=128, lp=1024, num_q_heads=16, num_kv_heads=2, head_dim=128,
        generator="frames", seed=1240,
        description="half of the 3B-shaped layer (H=2/V=4, anchor 1024 + 4x8192 + "
        "query 128, lp=1024): the profiling case, inputs still larger than L2")
    # long-context text prefill in the shape of the pages' RULER transfer
    # setting: Llama-3.1-8B attention (32 query heads, 8 KV heads, d = 128),
    # 128K input on 8 hosts (16 virtual hosts), la = n/64, lp = n/128 (the
    # ledger's defaults), a 256-token question block
    w["ruler_llama31_8b_128k"] = Workload(
        "ruler_llama31_8b_128k", num_hosts=8, anchor_len=2048, block_lens=[8048] * 16,
        query_len=256, lp=1024, num_q_heads=32, num_kv_heads=8, head_dim=128,
        generator="text", seed=1241,
        description="RULER-shaped text prefill, Llama-3.1-8B attention, n = 131072, H=8/V=16, "
        "anchor 2048 + 16x8048 + query 256, lp = 1024")
    blens = _unequal_blocks(1239, 8, 65536, 4096, 12288)
    w["exact_dense_3b_unequal"] = Workload(
        "exact_dense_3b_unequal", num_hosts=4, anchor_len=1024, block_lens=blens,
        query_len=128, lp=max(blens), num_q_heads=16, num_kv_heads=2,
        head_dim=128, generator="frames", seed=1239,
        description="3B shape, unequal blocks in [4096,12288] summing to 65536, "
        "lp = full block length")
    return w


def _randn(g: torch.Generator, *shape) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def make_inputs(wl: Workload, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw Q, K, V (bf16, CPU) for ``wl``.

    gaussian: every entry N(0,1).
    needles : N(0,1), then in each context block 8 keys at distinct uniform
              positions are replaced (per KV head) by 3 x the mean query-block
              query vector of that head group plus 0.3 N(0,1) noise, so that
              a query-driven top-lp choice has clear winners.
    frames  : context tokens come from 1024-token frames; per frame and KV
              head a basis U_f in R^{16 x d} ~ N(0, 1/16) and per token
              coefficients c ~ N(0, I_16) give K, V = c U_f + 0.3 N(0,1);
              context-row queries use the same frame bases with independent
              coefficients.  Anchor and query tokens are N(0,1).  The query
              block's queries correlate with a random 2% subset T of the
              context keys of their KV head: q = 0.8 k_t + 0.6 N(0,1) with
              t drawn uniformly from T.
    text    : Q, K, V ~ N(0,1) (a needle-in-a-haystack item's shape): per KV
              head, TEXT_NEEDLES context positions hold needle keys; each
              query-block query is 0.8 k_t + 0.6 N(0,1) with t drawn from that
              head's needles, so the question points at a few keys spread over
              the whole context.
    """
    seed = wl.seed if seed is None else seed
    g = torch.Generator().manual_seed(seed)
    n, hq, hkv, d = wl.seq_len, wl.num_q_heads, wl.num_kv_heads, wl.head_dim
    grp = hq // hkv
    la, lq = wl.anchor_len, wl.query_len
    ctx0, ctx1 = la, la + sum(wl.block_lens)
    out = {}
    if wl.generator in ("gaussian", "needles"):
        Q = _randn(g, n, hq, d)
        K = _randn(g, n, hkv, d)
        V = _randn(g, n, hkv, d)
        if wl.generator == "needles":
            qr = Q[ctx1:].to(torch.bfloat16).float()
            start = la
            positions = []
            for L in wl.block_lens:
                cnt = min(8, L)
                pos = torch.randperm(L, generator=g)[:cnt] + start
                positions.append(pos)
                for kv in range(hkv):
                    mean_q = qr[:, kv * grp:(kv + 1) * grp, :].reshape(-1, d).mean(0)
                    K[pos, kv, :] = 3.0 * mean_q + 0.3 * _randn(g, cnt, d)
                start += L
            out["needle_positions"] = torch.cat(positions)
        out.update(Q=Q.to(torch.bfloat16), K=K.to(torch.bfloat16),
                   V=V.to(torch.bfloat16))
        return out

    if wl.generator == "text":
        Q = _randn(g, n, hq, d)
        K = _randn(g, n, hkv, d)
        V = _randn(g, n, hkv, d)
        nctx = ctx1 - ctx0
        needles = []
        for kv in range(hkv):
            pos = torch.randperm(nctx, generator=g)[:TEXT_NEEDLES] + ctx0
            needles.append(pos)
            for gg in range(kv * grp, (kv + 1) * grp):
                pick = pos[torch.randint(0, len(pos), (lq,), generator=g)]
                Q[ctx1:, gg, :] = 0.8 * K[pick, kv, :] + 0.6 * _randn(g, lq, d)
        out.update(Q=Q.to(torch.bfloat16), K=K.to(torch.bfloat16), V=V.to(torch.bfloat16),
                   needle_positions=torch.stack(needles))
        return out
    if wl.generator != "frames":
        raise ValueError(wl.generator)
    Q = torch.empty(n, hq, d, dtype=torch.bfloat16)
    K = torch.empty(n, hkv, d, dtype=torch.bfloat16)
    V = torch.empty(n, hkv, d, dtype=torch.bfloat16)
    # anchor tokens
    Q[:la] = _randn(g, la, hq, d).to(torch.bfloat16)
    K[:la] = _randn(g, la, hkv, d).to(torch.bfloat16)
    V[:la] = _randn(g, la, hkv, d).to(torch.bfloat16)
    # context tokens, frame by frame
    kv_of = torch.arange(hq) // grp
    for f0 in range(ctx0, ctx1, FRAME_TOKENS):
        f1 = min(f0 + FRAME_TOKENS, ctx1)
        t = f1 - f0
        U = _randn(g, hkv, FRAME_RANK, d) / (FRAME_RANK ** 0.5)
        ck = _randn(g, hkv, t, FRAME_RANK)
        cv = _randn(g, hkv, t, FRAME_RANK)
        kf = torch.bmm(ck, U) + NOISE * _randn(g, hkv, t, d)
        vf = torch.bmm(cv, U) + NOISE * _randn(g, hkv, t, d)
        K[f0:f1] = kf.transpose(0, 1).to(torch.bfloat16)
        V[f0:f1] = vf.transpose(0, 1).to(torch.bfloat16)
        cq = _randn(g, hq, t, FRAME_RANK)
        qf = torch.bmm(cq, U[kv_of]) + NOISE * _randn(g, hq, t, d)
        Q[f0:f1] = qf.transpose(0, 1).to(torch.bfloat16)
    # query tokens
    K[ctx1:] = _randn(g, lq, hkv, d).to(torch.bfloat16)
    V[ctx1:] = _randn(g, lq, hkv, d).to(torch.bfloat16)
    nctx = ctx1 - ctx0
    nhit = max(1, int(round(QR_HIT_FRACTION * nctx)))
    qr = torch.empty(lq, hq, d)
    hits = []
    for kv in range(hkv):
        T = torch.randperm(nctx, generator=g)[:nhit] + ctx0
        hits.append(T)
        for gg in range(kv * grp, (kv + 1) * grp):
            pick = T[torch.randint(0, nhit, (lq,), generator=g)]
            qr[:, gg, :] = 0.8 * K[pick, kv, :].float() + 0.6 * _randn(g, lq, d)
    Q[ctx1:] = qr.to(torch.bfloat16)
    out.update(Q=Q, K=K, V=V, hit_positions=torch.stack(hits))
    return out


def random_scores(total: int, num_kv_heads: int, seed: int, ties: bool = True) -> torch.Tensor:
    """fp32 scores [Hkv, total] for exercising the selection step on its own:
    a Gaussian draw, with (optionally) runs of exactly equal values, signed
    zeros and repeated maxima planted so that the tie rule is exercised."""
    g = torch.Generator().manual_seed(seed)
    s = _randn(g, num_kv_heads, total)
    if ties and total >= 8:
        for kv in range(num_kv_heads):
            m = max(2, total // 16)
            pos = torch.randperm(total, generator=g)[:m]
            vals = torch.tensor([0.0, -0.0, 1.5, -2.25], dtype=torch.float32)
            s[kv, pos] = vals[torch.randint(0, 4, (m,), generator=g)]
            s[kv, pos[: max(1, m // 8)]] = s[kv].max()
    return s.contiguous()
