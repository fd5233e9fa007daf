"""How much the passing-key selectors agree, on the GPU.

The pages select each context block's passing keys by the summed query-block
logits Q_qr K^(h)T; the review ("APB-V ..." pith.science, major comment 1 and
"What would settle it") asks for the overlap of that choice with others, in
particular with the keys the block's own tokens attend to.  For each workload
this computes the three selections (linear = the pages' rule, softmax =
query-block softmax, context = cumulative causal attention from the block's
own rows) with the library's kernels and prints, as one JSON line per
workload:
  overlap      fraction of passing keys (over blocks and KV heads) that a
               selector shares with the linear one;
  needle_recall  for the text workload: fraction of needle keys in
               compressed blocks that each selector keeps;
  score_ms     device time of each selector's scoring step.

    python -m sparse_approximate_attention_b200.overlap [--workload NAME ...]
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import spava
from . import workloads as W

KINDS = ("linear", "softmax", "context")


def selections(wl, inp, dev):
    """{kind: (idx [V-1, Hkv, lp] int array, scoring ms)}."""
    Q, K, V = (inp[k].to(dev) for k in ("Q", "K", "V"))
    out = {}
    for kind in KINDS:
        p = spava.Problem.from_workload(wl, score_kind=kind)
        ws = torch.empty(max(1, p.sizes()["workspace_bytes"]), dtype=torch.uint8, device=dev)
        run = lambda: spava.score_variant(p, Q, K, workspace=ws)
        run()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        scores = run()
        b.record()
        idx = spava.select_topk(p, scores)
        torch.cuda.synchronize(dev)
        out[kind] = (idx.cpu().numpy(), a.elapsed_time(b))
    return out


def overlap(wl, a: np.ndarray, b: np.ndarray) -> float:
    both = total = 0
    for h in range(2 * wl.num_hosts - 1):
        e = min(wl.lp, wl.block_lens[h])
        for kv in range(wl.num_kv_heads):
            both += len(set(a[h, kv, :e].tolist()) & set(b[h, kv, :e].tolist()))
            total += e
    return both / total if total else 1.0


def needle_recall(wl, inp, idx: np.ndarray):
    if "needle_positions" not in inp or inp["needle_positions"].dim() != 2:
        return None
    starts = np.cumsum([wl.anchor_len] + list(wl.block_lens))
    hit = total = 0
    for kv in range(wl.num_kv_heads):
        for pos in inp["needle_positions"][kv].tolist():
            h = int(np.searchsorted(starts, pos, side="right")) - 1
            if 0 <= h < 2 * wl.num_hosts - 1:
                e = min(wl.lp, wl.block_lens[h])
                hit += (pos - starts[h]) in set(idx[h, kv, :e].tolist())
                total += 1
    return hit / total if total else None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", nargs="+", default=["qwen25vl3b_64f", "longvideo_256k_lp4096"])
    args = ap.parse_args()
    dev = torch.device("cuda", 0)
    for name in args.workload:
        wl = W.workloads()[name]
        inp = W.make_inputs(wl)
        sel = selections(wl, inp, dev)
        line = {"workload": name, "lp": wl.lp, "blocks": 2 * wl.num_hosts - 1, "kv_heads": wl.num_kv_heads,
                "overlap": {k: round(overlap(wl, sel[k][0], sel["linear"][0]), 4) for k in KINDS},
                "score_ms": {k: round(sel[k][1], 3) for k in KINDS}}
        recall = {k: needle_recall(wl, inp, sel[k][0]) for k in KINDS}
        if any(v is not None for v in recall.values()):
            line["needle_recall"] = {k: round(v, 4) for k, v in recall.items() if v is not None}
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
