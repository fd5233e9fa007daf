"""Device time of every stage entry of the layer on one workload.

Runs each C entry point of the path on the GPU with CUDA events: the stage
calls of steps 1-3 (spava_score, spava_select_topk, spava_gather_passing,
which spava_layer_fwd falls back to for blocks longer than 24576 keys), the
fused compression (spava_compress), the attention (spava_attn_fwd), the
stand-alone merge (spava_lse_merge) and the whole layer (spava_layer_fwd).
Prints one JSON line per stage.

    python -m sparse_approximate_attention_b200.stages [--workload NAME] [--reps N]
"""
from __future__ import annotations

import argparse
import json

import torch

from . import spava
from . import workloads as W


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="qwen25vl3b_h2")
    ap.add_argument("--reps", type=int, default=5)
    args = ap.parse_args()
    wl = W.workloads()[args.workload]
    inp = W.make_inputs(wl)
    Q, K, V = (inp[k].cuda() for k in ("Q", "K", "V"))
    p = spava.Problem.from_workload(wl)
    qsum, scores = spava.score(p, Q, K)
    idx = spava.select_topk(p, scores)
    Kp, Vp = spava.gather_passing(p, K, V, idx)
    O, lse, O_part, lse_part = spava.attn_fwd(p, Q, K, V, Kp, Vp)
    ws = torch.empty(spava.workspace_size(p), dtype=torch.uint8, device="cuda")
    stages = {
        "spava_score": lambda: spava.score(p, Q, K, qsum, scores),
        "spava_select_topk": lambda: spava.select_topk(p, scores, idx),
        "spava_gather_passing": lambda: spava.gather_passing(p, K, V, idx, Kp, Vp),
        "spava_compress": lambda: spava.compress(p, Q, K, V, qsum, scores, idx, Kp, Vp),
        "spava_attn_fwd": lambda: spava.attn_fwd(p, Q, K, V, Kp, Vp, O, lse, O_part, lse_part),
        "spava_lse_merge": lambda: spava.lse_merge(p, O_part, lse_part, O, lse),
        "spava_layer_fwd": lambda: spava.layer_fwd(p, Q, K, V, O, lse, ws),
    }
    for name, fn in stages.items():
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        print(json.dumps({"workload": wl.name, "stage": name, "ms": round(a.elapsed_time(b) / args.reps, 5)}),
              flush=True)
    assert spava.device_error() == 0


if __name__ == "__main__":
    main()
