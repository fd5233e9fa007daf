"""Device time of every stage entry of the layer on one workload.

Runs each C entry point of the path on the GPU with CUDA events: the stage
calls of steps 1-3 (spava_score, spava_select_topk, spava_gather_passing,
which spava_layer_fwd falls back to for blocks longer than 24576 keys), the
fused compression (spava_compress), the attention (spava_attn_fwd), the
stand-alone merge (spava_lse_merge) and the whole layer (spava_layer_fwd).
Prints one JSON line per stage.  --only runs the named stages alone and
allocates only what they need (a profiler can then capture one kernel of a
large workload without the attention's output buffers).

    python -m sparse_approximate_attention_b200.stages [--workload NAME] [--reps N]
                                                       [--only STAGE ...]
"""
from __future__ import annotations

import argparse
import json

import torch

from . import spava
from . import workloads as W

STAGES = ("spava_score", "spava_select_topk", "spava_gather_passing", "spava_compress", "spava_attn_fwd",
          "spava_lse_merge", "spava_layer_fwd")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="qwen25vl3b_h2")
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--only", nargs="+", choices=STAGES, default=list(STAGES))
    args = ap.parse_args()
    wl = W.workloads()[args.workload]
    inp = W.make_inputs(wl)
    Q, K, V = (inp[k].cuda() for k in ("Q", "K", "V"))
    p = spava.Problem.from_workload(wl)
    want = set(args.only)
    buf = {}

    def passing():
        if "Kp" not in buf:
            buf["qsum"], buf["scores"], buf["idx"], buf["Kp"], buf["Vp"] = spava.compress(p, Q, K, V)
        return buf

    def attn_out():
        if "O" not in buf:
            b = passing()
            buf["O"], buf["lse"], buf["O_part"], buf["lse_part"] = spava.attn_fwd(p, Q, K, V, b["Kp"], b["Vp"])
        return buf

    stages = {}
    if "spava_score" in want or "spava_select_topk" in want:
        qsum, scores = spava.score(p, Q, K)
        stages["spava_score"] = lambda: spava.score(p, Q, K, qsum, scores)
    if "spava_select_topk" in want or "spava_gather_passing" in want:
        idx = spava.select_topk(p, scores if "spava_select_topk" in want else passing()["scores"])
        stages["spava_select_topk"] = lambda: spava.select_topk(p, scores, idx)
    if "spava_gather_passing" in want:
        b = passing()
        stages["spava_gather_passing"] = lambda: spava.gather_passing(p, K, V, b["idx"], b["Kp"], b["Vp"])
    if "spava_compress" in want:
        b = passing()
        stages["spava_compress"] = lambda: spava.compress(p, Q, K, V, b["qsum"], b["scores"], b["idx"], b["Kp"],
                                                          b["Vp"])
    if "spava_attn_fwd" in want:
        b = attn_out()
        stages["spava_attn_fwd"] = lambda: spava.attn_fwd(p, Q, K, V, b["Kp"], b["Vp"], b["O"], b["lse"],
                                                          b["O_part"], b["lse_part"])
    if "spava_lse_merge" in want:
        b = attn_out()
        stages["spava_lse_merge"] = lambda: spava.lse_merge(p, b["O_part"], b["lse_part"], b["O"], b["lse"])
    if "spava_layer_fwd" in want:
        b = attn_out()
        ws = torch.empty(spava.workspace_size(p), dtype=torch.uint8, device="cuda")
        stages["spava_layer_fwd"] = lambda: spava.layer_fwd(p, Q, K, V, b["O"], b["lse"], ws)
    for name in STAGES:
        if name not in want:
            continue
        fn = stages[name]
        fn()
        torch.cuda.synchronize()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.reps):
            fn()
        b_.record()
        torch.cuda.synchronize()
        print(json.dumps({"workload": wl.name, "stage": name, "ms": round(a.elapsed_time(b_) / args.reps, 5)}),
              flush=True)
    assert spava.device_error() == 0


if __name__ == "__main__":
    main()
