"""CPU oracle for the Spava / APB-V approximate-attention prefill layer.

TEST INFRASTRUCTURE ONLY.  This module is a plain, slow, fp64 restatement of
what the layer computes, written from the pages' description of the method.
Only the tests, the smoke check and the bench's CPU-baseline / reference arm
may import it; the product path (the CUDA library and its binding) never does.
It shares no code with the CUDA path.

Sources (page title, then the part of the page):
  [SC] "Spava: Accelerating Long-Video Understanding via Sequence-Parallelism-
       aware Approximate Attention" (sciencestack.ai): TL;DR; Fig. 2-5 captions.
  [PR] "APB-V: ..." (pith.science machine review): "What carries the
       argument", "Core claim", referee major comment 1 (Eq. 4 and the
       passing-block selection), minor comment 2 (the key list of Eq. 4),
       "Axiom & Free-Parameter Ledger" (lse merge is exact; la, lp).
  [GN] "Technische Samenvatting: APB-V" (gist.science, nl): Methodologie.

Notation: V = 2H virtual hosts = context blocks B^(0..V-1); anchor B_a of la
tokens; query block B_qr of lq tokens; n = la + sum L_h + lq; Hq query heads,
Hkv KV heads, G = Hq / Hkv, query head g reads KV head g // G; scale = 1/sqrt(d)
unless given.  Positions are global sequence indices.

Readings where the pages are silent (each also listed in the design notes):
  R1 importance score of key j in block h for KV head kv is the sum over the
     query block's rows i and the G query heads g of that KV head of the
     scaled logit scale * <q_{i,g}, k_j>  ("ranked by Q_qr K^(h)T" [PR]).
  R2 top-lp keeps min(lp, L_h) keys; larger score first, equal scores ->
     lower index first; indices are reported in ascending order.  The
     decision is taken on the scores rounded to fp32 (the kernel's precision).
  R3 a context row of host h sees B_a, the passing keys of every earlier host
     (for its KV head) and the keys of B^(h) up to itself (Eq. 4 key list
     [K_a, K_p, K^(h)], [PR] minor comment 2; passing blocks of earlier hosts
     only, [PR] "Core claim").
  R4 anchor rows are causal over B_a.
  R5 query rows: host h's partial covers B^(h); host 0's partial also covers
     B_a and B_qr up to the row.  The partials are merged by log-sum-exp
     ([PR] ledger: lse merge is exact; [GN] fused context/query forward).
     So each query row ends up exact dense causal attention.
  R6 lse is the natural log of the sum of exp(scale * q.k) over the row's keys.
  R7 the last block's passing set is never used (no later host), so it is not
     computed.
  R8 selector variants ([PR] major comment 1, "What would settle it"): the
     softmax form normalises each query-block row's logits over the block's
     keys before summing; the context form sums the block's own causal
     attention over its rows ("cumulative attention from all tokens in the
     context block", read as attention within the block).  They change only
     which keys pass; everything after the selection is as above.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np


# --------------------------------------------------------------------------
# context splitting ([SC] Fig. 2 caption; [GN] "Context Splitting")
# --------------------------------------------------------------------------
@dataclass
class Layout:
    anchor_len: int
    block_lens: List[int]
    query_len: int
    lp: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    scale: float

    @property
    def V(self) -> int:
        return len(self.block_lens)

    @property
    def block_starts(self) -> List[int]:
        s, out = self.anchor_len, []
        for L in self.block_lens:
            out.append(s)
            s += L
        return out

    @property
    def query_start(self) -> int:
        return self.anchor_len + sum(self.block_lens)

    @property
    def n(self) -> int:
        return self.query_start + self.query_len

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def lp_eff(self, h: int) -> int:
        return min(self.lp, self.block_lens[h])

    def host_of_row(self, r: int) -> Tuple[str, int]:
        """('anchor', -1) | ('context', h) | ('query', -1)."""
        if r < self.anchor_len:
            return "anchor", -1
        if r >= self.query_start:
            return "query", -1
        for h, s in enumerate(self.block_starts):
            if s <= r < s + self.block_lens[h]:
                return "context", h
        raise IndexError(r)


def make_layout(num_hosts: int, anchor_len: int, block_lens: Sequence[int],
                query_len: int, lp: int, num_q_heads: int, num_kv_heads: int,
                head_dim: int, scale: Optional[float] = None) -> Layout:
    if len(block_lens) != 2 * num_hosts:
        raise ValueError("need 2H context blocks (ZigZag virtual hosts)")
    if num_q_heads % num_kv_heads:
        raise ValueError("Hq must be a multiple of Hkv")
    s = (1.0 / math.sqrt(head_dim)) if (scale is None or scale <= 0) else float(scale)
    return Layout(anchor_len, list(block_lens), query_len, lp, num_q_heads,
                  num_kv_heads, head_dim, s)


def default_hyperparameters(n: int) -> Tuple[int, int]:
    """Default anchor and passing lengths: la = n/64, lp = n/128
    ([PR] "Axiom & Free-Parameter Ledger", free parameters la and lp)."""
    return n // 64, n // 128


def _f64(x) -> np.ndarray:
    """bf16/fp32 torch tensor or numpy array -> float64 numpy (exact widening)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _take(T, rows, head) -> np.ndarray:
    """T[rows, head, :] widened to float64 (index first, so only the rows
    used are ever widened)."""
    try:
        import torch
        if isinstance(T, torch.Tensor):
            r = torch.as_tensor(np.asarray(rows, dtype=np.int64))
            return T[r, head].to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(T[np.asarray(rows, dtype=np.int64), head], dtype=np.float64)


# --------------------------------------------------------------------------
# step 1: KV importance  ([SC] Fig. 5 caption "Q_qr K^T estimates KV
# importance"; [PR] "What carries the argument"; reading R1)
# --------------------------------------------------------------------------
def importance_scores(lay: Layout, Q, K, h: int) -> np.ndarray:
    """fp64 scores [Hkv, L_h] of block h's keys against the query block."""
    qs, s0, L = lay.query_start, lay.block_starts[h], lay.block_lens[h]
    G, d = lay.group, lay.head_dim
    out = np.empty((lay.num_kv_heads, L))
    qrows = np.arange(qs, qs + lay.query_len)
    for kv in range(lay.num_kv_heads):
        q = np.stack([_take(Q, qrows, g) for g in range(kv * G, (kv + 1) * G)], axis=1).reshape(-1, d)
        k = _take(K, np.arange(s0, s0 + L), kv)
        logits = lay.scale * (q @ k.T)          # the Q_qr K^(h)T matrix
        out[kv] = logits.sum(axis=0)            # one importance per key
    return out


# --------------------------------------------------------------------------
# step 1, variants of the importance score.  The pages' selector is the
# summed Q_qr K^(h)T above; the review ([PR] major comment 1, "What would
# settle it") asks how its choice compares with others.  Two alternatives:
#   softmax: each query-block row's attention over block h's keys (softmax of
#            scale <q, k> over the block), summed per key over the rows and
#            the KV head's query heads (the plain normalised form of R1);
#   context: the review's oracle selector -- the cumulative attention each key
#            of block h receives from all tokens of the block: every context
#            row r of block h attends causally to the block's keys up to r
#            (softmax over those keys), summed per key over the rows and the
#            KV head's query heads.  Reading: "all tokens in the context block"
#            attend within the block, i.e. the block's local causal attention.
# --------------------------------------------------------------------------
def _softmax_rows(z: np.ndarray) -> np.ndarray:
    """Row-wise softmax of a logits matrix whose masked entries are -inf."""
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=1, keepdims=True)


def importance_scores_softmax(lay: Layout, Q, K, h: int) -> np.ndarray:
    """fp64 scores [Hkv, L_h]: sum over query-block rows i and query heads g
    of the KV head of softmax_j(scale <q_ig, k_j>) over block h's keys."""
    qs, s0, L = lay.query_start, lay.block_starts[h], lay.block_lens[h]
    G, d = lay.group, lay.head_dim
    out = np.empty((lay.num_kv_heads, L))
    qrows = np.arange(qs, qs + lay.query_len)
    for kv in range(lay.num_kv_heads):
        q = np.stack([_take(Q, qrows, g) for g in range(kv * G, (kv + 1) * G)], axis=1).reshape(-1, d)
        k = _take(K, np.arange(s0, s0 + L), kv)
        out[kv] = _softmax_rows(lay.scale * (q @ k.T)).sum(axis=0)
    return out


def importance_scores_context(lay: Layout, Q, K, h: int) -> np.ndarray:
    """fp64 scores [Hkv, L_h]: sum over block h's own rows r and the query
    heads g of the KV head of the causal softmax, over the block's keys up to
    r, of scale <q_rg, k_j>."""
    s0, L = lay.block_starts[h], lay.block_lens[h]
    G = lay.group
    rows = np.arange(s0, s0 + L)
    causal = np.arange(L)[None, :] <= np.arange(L)[:, None]      # key j visible to row r
    out = np.zeros((lay.num_kv_heads, L))
    for kv in range(lay.num_kv_heads):
        k = _take(K, rows, kv)
        for g in range(kv * G, (kv + 1) * G):
            z = np.where(causal, lay.scale * (_take(Q, rows, g) @ k.T), -np.inf)
            out[kv] += _softmax_rows(z).sum(axis=0)
    return out


SCORES = {"linear": importance_scores, "softmax": importance_scores_softmax,
          "context": importance_scores_context}


def compress_with(lay: Layout, Q, K, kind: str = "linear"):
    """Scores and passing indices of blocks 0..V-2 under one of the selectors
    (reading R7 for the last block, R2 for the selection)."""
    scores = {h: SCORES[kind](lay, Q, K, h) for h in range(lay.V - 1)}
    return scores, select_passing(lay, scores)


def selection_overlap(lay: Layout, idx_a, idx_b) -> float:
    """Fraction of the passing keys two selections share: sum over blocks and
    KV heads of |A & B|, over the number of passing keys."""
    both = total = 0
    for h in range(lay.V - 1):
        for kv in range(lay.num_kv_heads):
            a, b = set(np.asarray(idx_a[h][kv]).tolist()), set(np.asarray(idx_b[h][kv]).tolist())
            both += len(a & b)
            total += len(a)
    return both / total if total else 1.0


# --------------------------------------------------------------------------
# step 2: top-lp selection ([PR] "What carries the argument": compressed to
# the top-lp key-value pairs; reading R2)
# --------------------------------------------------------------------------
def top_lp(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest entries of a 1-D score vector; equal scores
    keep the lower index; result sorted ascending."""
    s = np.asarray(scores)
    k = min(k, s.shape[0])
    if k <= 0:
        return np.zeros(0, dtype=np.int64)
    idx = np.arange(s.shape[0])
    order = sorted(idx.tolist(), key=lambda j: (-float(s[j]), j))
    return np.sort(np.asarray(order[:k], dtype=np.int64))


def select_passing(lay: Layout, scores_by_block: Dict[int, np.ndarray]) -> Dict[int, np.ndarray]:
    """Block-relative passing indices [Hkv, lp_eff(h)] for blocks h < V-1.
    The decision uses the scores rounded to fp32 (reading R2)."""
    out = {}
    for h, s in scores_by_block.items():
        s32 = np.asarray(s, dtype=np.float32)
        out[h] = np.stack([top_lp(s32[kv], lay.lp_eff(h))
                           for kv in range(lay.num_kv_heads)]) \
            if lay.lp_eff(h) > 0 else np.zeros((lay.num_kv_heads, 0), np.int64)
    return out


# --------------------------------------------------------------------------
# step 3: key sets ([PR] "Core claim", minor comment 2; readings R3-R5)
# --------------------------------------------------------------------------
def passing_positions(lay: Layout, idx: Dict[int, np.ndarray], h: int, kv: int) -> np.ndarray:
    """Global positions of the passing keys host h receives: the union of the
    passing blocks of all earlier virtual hosts (the all-gather)."""
    parts = [lay.block_starts[j] + np.asarray(idx[j][kv], dtype=np.int64)
             for j in range(h)]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def key_positions(lay: Layout, idx: Dict[int, np.ndarray], r: int, kv: int) -> np.ndarray:
    """All key positions row r attends to (query rows: the union over hosts)."""
    kind, h = lay.host_of_row(r)
    if kind == "anchor":
        return np.arange(0, r + 1)
    if kind == "context":
        return np.concatenate([np.arange(lay.anchor_len),
                               passing_positions(lay, idx, h, kv),
                               np.arange(lay.block_starts[h], r + 1)])
    return np.arange(0, r + 1)


def query_partial_positions(lay: Layout, h: int, r: int) -> np.ndarray:
    """Keys of host h's partial for query row r (reading R5)."""
    s0, L = lay.block_starts[h], lay.block_lens[h]
    blk = np.arange(s0, s0 + L)
    if h == 0:
        return np.concatenate([np.arange(lay.anchor_len), blk,
                               np.arange(lay.query_start, r + 1)])
    return blk


# --------------------------------------------------------------------------
# step 4: softmax attention over an explicit key set (R6)
# --------------------------------------------------------------------------
def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
           visible: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Rows q [r, d] over keys k [m, d] / values v [m, d]; ``visible`` [r, m]
    marks the keys each row may see.  Returns (o [r, d], lse [r]) with
    o = sum softmax(scale q.k) v and lse = log sum exp(scale q.k)."""
    z = scale * (q @ k.T)
    if visible is not None:
        z = np.where(visible, z, -np.inf)
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    l = e.sum(axis=1, keepdims=True)
    o = (e @ v) / l
    return o, (m + np.log(l))[:, 0]


# --------------------------------------------------------------------------
# step 5: merge of partial query results ([PR] ledger: online-softmax lse
# merging is exact; [GN] fused context and query forward)
# --------------------------------------------------------------------------
def lse_merge(o_parts: np.ndarray, lse_parts: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """o_parts [P, ..., d], lse_parts [P, ...] -> (o [..., d], lse [...]):
    lse = log sum_p exp(lse_p), o = sum_p exp(lse_p - lse) o_p."""
    mx = lse_parts.max(axis=0)
    lse = mx + np.log(np.exp(lse_parts - mx).sum(axis=0))
    w = np.exp(lse_parts - lse)
    return (w[..., None] * o_parts).sum(axis=0), lse


# --------------------------------------------------------------------------
# the layer
# --------------------------------------------------------------------------
def compress(lay: Layout, Q, K) -> Tuple[Dict[int, np.ndarray], Dict[int, np.ndarray]]:
    """Scores and passing indices of blocks 0..V-2 (reading R7)."""
    scores = {h: importance_scores(lay, Q, K, h) for h in range(lay.V - 1)}
    return scores, select_passing(lay, scores)


def context_rows(lay: Layout, Q, K, V, idx, h: int, rows: Sequence[int],
                 heads: Sequence[int]) -> Tuple[np.ndarray, np.ndarray]:
    """Rows (global positions inside B^(h), or inside B_a when h == -1) for
    the given query heads -> (o [len(rows), len(heads), d], lse [len(heads), len(rows)])."""
    rows = np.asarray(rows, dtype=np.int64)
    o = np.empty((len(rows), len(heads), lay.head_dim))
    lse = np.empty((len(heads), len(rows)))
    for hi, g in enumerate(heads):
        kv = g // lay.group
        if h < 0:                       # anchor rows: causal over B_a (R4)
            fixed = np.zeros(0, dtype=np.int64)
            local = np.arange(0, rows.max() + 1)
        else:                           # context rows of host h (R3)
            fixed = np.concatenate([np.arange(lay.anchor_len),
                                    passing_positions(lay, idx, h, kv)])
            local = np.arange(lay.block_starts[h], rows.max() + 1)
        keys = np.concatenate([fixed, local]).astype(np.int64)
        visible = np.zeros((len(rows), len(keys)), dtype=bool)
        visible[:, :len(fixed)] = True
        visible[:, len(fixed):] = local[None, :] <= rows[:, None]
        oo, ll = attend(_take(Q, rows, g), _take(K, keys, kv), _take(V, keys, kv),
                        lay.scale, visible)
        o[:, hi, :], lse[hi] = oo, ll
    return o, lse


def query_partials(lay: Layout, Q, K, V, heads: Optional[Sequence[int]] = None):
    """Per-host partials of the query rows:
    o_part [V, lq, len(heads), d], lse_part [V, len(heads), lq]."""
    heads = list(range(lay.num_q_heads)) if heads is None else list(heads)
    rows = np.arange(lay.query_start, lay.n)
    o = np.empty((lay.V, len(rows), len(heads), lay.head_dim))
    lse = np.empty((lay.V, len(heads), len(rows)))
    for h in range(lay.V):
        for hi, g in enumerate(heads):
            kv = g // lay.group
            keys = query_partial_positions(lay, h, lay.n - 1)
            visible = keys[None, :] <= rows[:, None]
            oo, ll = attend(_take(Q, rows, g), _take(K, keys, kv), _take(V, keys, kv),
                            lay.scale, visible)
            o[h, :, hi, :], lse[h, hi] = oo, ll
    return o, lse


def layer_fwd(lay: Layout, Q, K, V) -> Dict[str, object]:
    """The whole layer at small sizes: every row and head.
    Returns O [n, Hq, d], lse [Hq, n] (fp64) and the intermediates."""
    scores, idx = compress(lay, Q, K)
    n, Hq, d = lay.n, lay.num_q_heads, lay.head_dim
    O = np.empty((n, Hq, d))
    lse = np.empty((Hq, n))
    heads = list(range(Hq))
    if lay.anchor_len:
        rows = np.arange(lay.anchor_len)
        O[rows], lse[:, rows] = context_rows(lay, Q, K, V, idx, -1, rows, heads)
    for h in range(lay.V):
        s0 = lay.block_starts[h]
        rows = np.arange(s0, s0 + lay.block_lens[h])
        O[rows], lse[:, rows] = context_rows(lay, Q, K, V, idx, h, rows, heads)
    o_part, lse_part = query_partials(lay, Q, K, V, heads)
    qo, ql = lse_merge(o_part, lse_part.transpose(0, 2, 1))
    rows = np.arange(lay.query_start, n)
    O[rows], lse[:, rows] = qo, ql.T
    return dict(O=O, lse=lse, scores=scores, idx=idx, o_part=o_part, lse_part=lse_part)


def rows_fwd(lay: Layout, Q, K, V, idx, rows: Sequence[int], heads: Sequence[int]):
    """Selected output rows (any mix of anchor/context/query rows) for the
    given heads, computed one region at a time -> (o [r, h, d], lse [h, r])."""
    rows = np.asarray(sorted(set(int(r) for r in rows)), dtype=np.int64)
    o = np.empty((len(rows), len(heads), lay.head_dim))
    lse = np.empty((len(heads), len(rows)))
    kinds = [lay.host_of_row(int(r)) for r in rows]
    groups: Dict[Tuple[str, int], List[int]] = {}
    for i, kh in enumerate(kinds):
        groups.setdefault(kh, []).append(i)
    for (kind, h), pos in groups.items():
        rr = rows[pos]
        if kind == "anchor":
            oo, ll = context_rows(lay, Q, K, V, idx, -1, rr, heads)
        elif kind == "context":
            oo, ll = context_rows(lay, Q, K, V, idx, h, rr, heads)
        else:
            op, lp_ = query_partials(lay, Q, K, V, heads)
            qo, ql = lse_merge(op, lp_.transpose(0, 2, 1))
            sel = rr - lay.query_start
            oo, ll = qo[sel], ql.T[:, sel]
        o[pos], lse[:, pos] = oo, ll
    return rows, o, lse


def gather_passing(lay: Layout, K, V, idx) -> Tuple[np.ndarray, np.ndarray]:
    """The compacted passing buffers Kp, Vp [sum_h lp_eff(h), Hkv, d] (blocks
    0..V-2 in host order): row (off_h + t, kv) holds key start_h + idx_h[kv][t]
    of KV head kv.  This is the single-GPU stand-in for the all-gather of
    passing blocks ([PR] "What carries the argument")."""
    rows = sum(lay.lp_eff(h) for h in range(lay.V - 1))
    Kp = np.zeros((rows, lay.num_kv_heads, lay.head_dim))
    Vp = np.zeros_like(Kp)
    off = 0
    for h in range(lay.V - 1):
        e = lay.lp_eff(h)
        for kv in range(lay.num_kv_heads):
            pos = lay.block_starts[h] + np.asarray(idx[h][kv], dtype=np.int64)
            Kp[off:off + e, kv] = _take(K, pos, kv)
            Vp[off:off + e, kv] = _take(V, pos, kv)
        off += e
    return Kp, Vp


def flops(lay: Layout) -> int:
    """Algorithmic attention FLOPs: 4 d Hq per visible (row, key) pair."""
    la, lq = lay.anchor_len, lay.query_len
    pairs = la * (la + 1) // 2
    passed = 0
    for h, L in enumerate(lay.block_lens):
        pairs += L * (la + passed) + L * (L + 1) // 2
        if h < lay.V - 1:
            passed += lay.lp_eff(h)
    pairs += lq * (la + sum(lay.block_lens)) + lq * (lq + 1) // 2
    return 4 * lay.head_dim * lay.num_q_heads * pairs
