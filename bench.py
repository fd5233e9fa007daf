#!/usr/bin/env python
"""Throughput of the approximate-attention prefill layer (Spava / APB-V) on
B200, as prefill tokens/s per layer, with the attention kernel's achieved
TFLOP/s against the measured bf16 tensor-core peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference]

One step = one spava_layer_fwd call over one synthetic input set: the
query-block sum, the compression launch (scores, top-lp, passing gather),
then the attention launch, which also merges the query partials; each starts
while the one before it runs (programmatic dependent launch).  The default workload is the 256K-token long-video
stress case with lp = 4096, the largest that fits one GPU.  Timed on the
device with CUDA events; inputs rotate over three resident sets, each larger
than L2.  The attention, compression and stage-merge kernels are then timed
on their own for their rooflines.  With N > 1 (torchrun) every rank runs an
independent replica of the layer on its own GPU (the layer does not shard:
all virtual hosts live on one GPU) and the job value is the sum of tokens
over the max over ranks of the elapsed time.

--impl reference times the CPU fp64 oracle on the host cores instead (the
reference arm: per step, a bounded sample of the same workload extrapolated
to the whole layer).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "approx-attn prefill tokens/s per layer"
DEFAULT_WORKLOAD = "longvideo_256k_lp4096"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(world, backend):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(x: float, world: int, device=None) -> float:
    """Max of a float over ranks (identity at world size 1)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.index, self.proc, self.lines = self._smi_id(device), None, []

    @staticmethod
    def _smi_id(device) -> str:
        """nvidia-smi id of a torch device (its UUID, so that a remapped
        CUDA_VISIBLE_DEVICES still samples the right GPU)."""
        try:
            import torch
            u = str(torch.cuda.get_device_properties(device).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            return str(getattr(device, "index", 0) or 0)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def source_hash(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def committed_traffic(workload: str):
    """Per-launch DRAM bytes of the attention kernel from the committed ncu
    summary, if it was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "attn_kernel_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    src = os.path.join(ROOT, "sparse_approximate_attention_b200", "csrc", "attention.cuh")
    e = d.get(workload)
    if not e or e.get("source_sha256_16") != source_hash(src):
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ oracle (CPU) arm
_SELECTION = {}


def oracle_sample(wl, inp, seed=0):
    """Time the fp64 oracle on a bounded sample of the workload and
    extrapolate it to the whole layer.

    The sample works on KV head 0 and its query heads: the compression
    (scores and top-lp) of the largest compressed block, and, for query head
    0, one random 128-row tile of every context block, the first anchor tile
    and all query rows.  The whole layer's oracle time is estimated as
        t_compress(block) x (sum of compressed block lengths x Hkv) / L_block
      + t_rows x (attention FLOPs of the layer) / (attention FLOPs of the sampled rows),
    so the estimate does not depend on the sample's size.  Both the GPU arm's
    cpu_baseline and the reference arm call this with the same arguments.
    Returns (tokens/s, estimated seconds per layer, sample seconds, description)."""
    import numpy as np
    import oracle
    lay = oracle.make_layout(wl.num_hosts, wl.anchor_len, wl.block_lens, wl.query_len, wl.lp,
                             wl.num_q_heads, wl.num_kv_heads, wl.head_dim)
    G = wl.num_q_heads // wl.num_kv_heads
    sub = oracle.make_layout(wl.num_hosts, wl.anchor_len, wl.block_lens, wl.query_len, wl.lp, G, 1,
                             wl.head_dim)
    Qs, Ks, Vs = inp["Q"][:, :G], inp["K"][:, :1], inp["V"][:, :1]
    rng = np.random.default_rng(seed)
    hb = int(np.argmax(sub.block_lens[:-1])) if sub.V > 1 else 0
    t_block, compressed = 0.0, 0
    if sub.lp > 0 and sub.V > 1:
        t0 = time.perf_counter()
        sc = oracle.importance_scores(sub, Qs, Ks, hb)
        oracle.top_lp(np.asarray(sc[0], dtype=np.float32), sub.lp_eff(hb))
        t_block = time.perf_counter() - t0
        compressed = sum(sub.block_lens[:-1]) * wl.num_kv_heads
    t_compress = t_block * compressed / sub.block_lens[hb]
    if wl.name not in _SELECTION:   # the selection the sampled rows need (not timed)
        _SELECTION[wl.name] = oracle.compress(sub, Qs, Ks)[1]
    idx = _SELECTION[wl.name]
    rows = []
    for h in range(sub.V):
        s0, L = sub.block_starts[h], sub.block_lens[h]
        r0 = s0 + int(rng.integers(0, max(1, L - 128 + 1)))
        rows += list(range(r0, min(s0 + L, r0 + 128)))
    rows += list(range(min(128, sub.anchor_len)))
    rows += list(range(sub.query_start, sub.n))
    t1 = time.perf_counter()
    oracle.rows_fwd(sub, Qs, Ks, Vs, idx, rows, [0])
    t_rows = time.perf_counter() - t1
    f_sample = 4.0 * sub.head_dim * sum(len(oracle.key_positions(sub, idx, r, 0)) for r in rows)
    f_layer = float(oracle.flops(lay))
    est = t_compress + t_rows * f_layer / f_sample
    desc = (f"fp64 oracle on KV head 0: compression of block {hb} (L={sub.block_lens[hb]}) scaled by length to "
            f"all {sub.V - 1} compressed blocks x {wl.num_kv_heads} KV heads; {len(rows)} rows of query head 0 "
            f"(one random 128-row tile per context block, the first anchor tile, all query rows) = "
            f"{f_sample / f_layer:.4%} of the layer's attention FLOPs, scaled by FLOPs")
    return wl.seq_len / est, est, t_block + t_rows, desc


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        return os.cpu_count()


def run_reference(args, wl):
    import torch  # noqa: F401  (generator)
    from sparse_approximate_attention_b200 import workloads as W
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    inp = W.make_inputs(wl)
    for w in range(args.warmup):
        oracle_sample(wl, inp, seed=1000 + w)
    est_total, sample_s, desc = 0.0, 0.0, ""
    for k in range(args.steps):
        _, est, secs, desc = oracle_sample(wl, inp, seed=k)
        est_total += est
        sample_s += secs
    value = args.steps * wl.seq_len / est_total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * est_total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, wl.seq_len),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": os.cpu_count(),
                         "threads": cpu_threads(), "kind": "oracle", "sample": desc,
                         "sample_seconds_per_step": round(sample_s / args.steps, 2)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(wl, n, parallelism="replicas (one independent layer per GPU)"):
    return {"workload": wl.name, "seq_len": n, "num_hosts": wl.num_hosts,
            "virtual_hosts": 2 * wl.num_hosts, "anchor_len": wl.anchor_len,
            "block_lens": sorted(set(wl.block_lens)) if len(set(wl.block_lens)) == 1 else wl.block_lens,
            "query_len": wl.query_len, "lp": wl.lp, "q_heads": wl.num_q_heads,
            "kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
            "parallelism": parallelism,
            "l2": "3 rotating input sets, each larger than L2"}


# ------------------------------------------------------------------ GPU arm
def timed_loop(fn, steps, stream, dev):
    """Device time (ms per call) of `steps` back-to-back calls of fn(k) on
    `stream`, CUDA events on that stream, synchronized on both sides."""
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    a.record(stream)
    for k in range(steps):
        fn(k)
    b.record(stream)
    torch.cuda.synchronize(dev)
    return a.elapsed_time(b) / steps


def run_gpu(args, wl):
    import torch
    import sparse_approximate_attention_b200 as spava
    from sparse_approximate_attention_b200 import workloads as W

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init(world, "nccl")
    p = spava.Problem.from_workload(wl)
    sz = p.sizes()
    n = sz["seq_len"]
    # three resident input sets (different seeds), each larger than L2
    sets = []
    host_inp = None
    for i in range(3):
        inp = W.make_inputs(wl, seed=wl.seed + 1000 * rank + i)
        if i == 0:
            host_inp = inp
        sets.append({k: inp[k].to(dev) for k in ("Q", "K", "V")})
    hq, hkv, d, V, lq, lp = wl.num_q_heads, wl.num_kv_heads, wl.head_dim, 2 * wl.num_hosts, wl.query_len, wl.lp
    f32, bf = torch.float32, torch.bfloat16
    O = torch.empty(n, hq, d, dtype=bf, device=dev)
    lse = torch.empty(hq, n, dtype=f32, device=dev)
    ws = torch.empty(sz["workspace_bytes"], dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    if args.mode == "hosts":
        # the pages' split: rank r computes the virtual hosts of its mask and
        # the ranks exchange passing rows and query partials (hosts.py)
        from sparse_approximate_attention_b200 import hosts
        sharded = hosts.HostShardedLayer(p, world, rank, dev)
        q = sharded.q

        def layer(k):
            x = sets[k % 3]
            sharded.forward(x["Q"], x["K"], x["V"], O, lse, stream=stream)

        # query sum + compression, attention, merge (collectives are NCCL's)
        launches_per_step = 4 if lp > 0 else 2
    else:
        q = p

        def layer(k):
            x = sets[k % 3]
            spava.layer_fwd(p, x["Q"], x["K"], x["V"], O, lse, ws, stream=stream)

        # query sum + compression, then attention (lp = 0: a memset of the merge counters + attention)
        launches_per_step = 3 if lp > 0 else 1

    for i in range(args.warmup):
        layer(i)
    torch.cuda.synchronize(dev)
    assert spava.device_error() == 0

    # ---------------- timed region: K layer steps
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        barrier(world)
        torch.cuda.synchronize(dev)
        t_begin.record(stream)
        for k in range(args.steps):
            layer(k)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
    elapsed_ms = reduce_max(t_begin.elapsed_time(t_end), world, dev)
    err = spava.device_error()
    assert err == 0, f"device error word {err}"
    ms_per_step = elapsed_ms / args.steps
    # replicas: every rank processes a layer; hosts: the ranks process one together
    value = (1 if args.mode == "hosts" else world) * n / (ms_per_step / 1000.0)

    # ---------------- the kernels on their own (same launch configuration as in the layer)
    qsum = torch.empty(hkv, d, dtype=f32, device=dev)
    scores = torch.empty(hkv, sz["score_cols"], dtype=f32, device=dev)
    idx = torch.empty(V - 1, hkv, lp, dtype=torch.int32, device=dev)
    Kp = torch.empty(max(1, sz["passing_rows"]), hkv, d, dtype=bf, device=dev)[: sz["passing_rows"]]
    Vp = torch.empty_like(Kp)
    O_part = torch.empty(V, lq, hq, d, dtype=f32, device=dev)
    lse_part = torch.empty(V, hq, lq, dtype=f32, device=dev)
    stage_ms = {}
    if lp > 0:
        comp = lambda k: spava.compress(q, sets[k % 3]["Q"], sets[k % 3]["K"], sets[k % 3]["V"], qsum, scores,
                                        idx, Kp, Vp, stream=stream)
        for k in range(3):
            comp(k)
        stage_ms["compress"] = timed_loop(comp, args.steps, stream, dev)
    attn = lambda k: spava.attn_fwd(q, sets[k % 3]["Q"], sets[k % 3]["K"], sets[k % 3]["V"],
                                    Kp if lp else None, Vp if lp else None, O, lse, O_part, lse_part,
                                    stream=stream)
    for k in range(3):
        attn(k)
    with ClockSampler(dev) as clk_attn:
        stage_ms["attn"] = timed_loop(attn, args.steps, stream, dev)
    attn_region_s = stage_ms["attn"] * args.steps / 1000.0
    merge = lambda k: spava.lse_merge(p, O_part, lse_part, O, lse, stream=stream)
    merge(0)
    stage_ms["merge"] = timed_loop(merge, args.steps, stream, dev)
    assert spava.device_error() == 0

    if args.no_e2e or args.mode == "hosts":
        e2e_ms, e2e_value, h2d, d2h = None, None, 0, 0
    else:
        e2e_ms, e2e_value, h2d, d2h = e2e_measure(p, host_inp, sets, O, lse, ws, stream, dev,
                                                   world, n, args.steps)
    if rank != 0:
        return 0
    return report(args, wl, sz, world, n, ms_per_step, elapsed_ms, value, stage_ms, attn_region_s, e2e_ms,
                  e2e_value, h2d, d2h, launches_per_step, clk, clk_attn, host_inp, q.sizes())


def e2e_measure(p, host_inp, sets, O, lse, ws, stream, dev, world, n, steps):
    """The layer through the public call (spava_layer_fwd), end to end: every
    step copies its Q, K, V from pinned host memory to the device and reads O
    and lse back to pinned host memory.  Steps are pipelined over three
    streams (upload, compute, download) with two device buffer sets, so the
    upload of step k+1 and the download of step k-1 overlap the compute of
    step k; the timed region runs from the first upload to the last download."""
    import torch
    import sparse_approximate_attention_b200 as spava
    bf, f32 = torch.bfloat16, torch.float32
    hQ, hK, hV = (host_inp[k].pin_memory() for k in ("Q", "K", "V"))
    dIn = [tuple(torch.empty_like(sets[0][k]) for k in ("Q", "K", "V")) for _ in range(2)]
    dOut = [(torch.empty_like(O), torch.empty_like(lse)) for _ in range(2)]
    hOut = [(torch.empty(O.shape, dtype=bf).pin_memory(), torch.empty(lse.shape, dtype=f32).pin_memory())
            for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in (hQ, hK, hV))
    d2h = hOut[0][0].numel() * 2 + hOut[0][1].numel() * 4
    s_in, s_cp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    in_done, cp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def run(k):
        b = k % 2
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(cp_done[b])          # step k-2 no longer reads buffer b
            for dst, src in zip(dIn[b], (hQ, hK, hV)):
                dst.copy_(src, non_blocking=True)
            in_done[b].record(s_in)
        with torch.cuda.stream(s_cp):
            s_cp.wait_event(in_done[b])
            if k >= 2:
                s_cp.wait_event(out_done[b])         # step k-2's outputs are downloaded
            spava.layer_fwd(p, *dIn[b], dOut[b][0], dOut[b][1], ws, stream=s_cp)
            cp_done[b].record(s_cp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cp_done[b])
            hOut[b][0].copy_(dOut[b][0], non_blocking=True)
            hOut[b][1].copy_(dOut[b][1], non_blocking=True)
            out_done[b].record(s_out)

    for k in range(3):
        run(k)
    torch.cuda.synchronize(dev)
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(6, steps)   # the same steps as the device-timed region; one pipeline fill and drain
    t0.record(s_in)
    for k in range(e2e_steps):
        run(k)
    s_in.wait_stream(s_out)
    t1.record(s_in)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(t0.elapsed_time(t1) / e2e_steps, world, dev)
    return e2e_ms, world * n / (e2e_ms / 1000.0), h2d, d2h


def report(args, wl, sz, world, n, ms_per_step, elapsed_ms, value, stage_ms, attn_region_s, e2e_ms,
           e2e_value, h2d, d2h, launches_per_step, clk, clk_attn, host_inp, rank_sz=None):
    hq, hkv, d, V, lq, lp = (wl.num_q_heads, wl.num_kv_heads, wl.head_dim, 2 * wl.num_hosts,
                             wl.query_len, wl.lp)
    pk, src = peaks()
    burst = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sustained = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    hbm = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    # the attention kernel's timed loop: a region shorter than a second runs
    # at the burst clock, a longer one settles under the power cap
    sustained_region = attn_region_s >= 1.0
    peak_tf = sustained if sustained_region else burst
    hosts_mode = args.mode == "hosts"
    # the attention launch of this rank: all rows, or the rows of its host mask
    flops = (rank_sz or sz)["attn_flops"]
    attn_tf = flops / (stage_ms["attn"] / 1000.0) / 1e12
    S, P = sz["score_cols"], sz["passing_rows"]
    by = {
        # K rows of blocks 0..V-2 read once + scores written + the query block
        # read + indices written + kept K,V rows read and written
        "compress": hkv * S * d * 2 + hkv * S * 4 + lq * hq * d * 2 + (V - 1) * hkv * lp * 4
                    + 2 * 2 * P * hkv * d * 2,
        "merge": V * lq * hq * (d + 1) * 4 + lq * hq * (d * 2 + 4),
    }
    stage_info = {}
    for s_, ms in stage_ms.items():
        e = {"ms": round(ms, 5)}
        if s_ == "attn":
            e.update(tflops=round(attn_tf, 1), frac_of_burst=round(attn_tf / burst, 4),
                     frac_of_sustained=round(attn_tf / sustained, 4), frac_of_datasheet=round(attn_tf / 2250.0, 4),
                     kernel=f"attn_kernel<{d}> via spava_attn_fwd (the layer's launch also merges the query "
                            f"partials of a few CTAs)")
        else:
            gbs = by[s_] / (ms / 1000.0) / 1e9
            e.update(algo_bytes=by[s_], gbs=round(gbs, 1), frac_of_hbm=round(gbs / hbm, 4))
            if s_ == "merge":
                e["note"] = "stage entry spava_lse_merge; inside spava_layer_fwd the merge runs in the attention launch"
        stage_info[s_] = e
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "strong" if hosts_mode else "weak", "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded long-video-shaped Q/K/V: rank-16 per-frame K/V + noise, "
                "query block correlated with 2% of context keys)",
        "config": config_of(wl, n, (f"hosts over {world} GPU(s): rank r holds virtual hosts p and 2H-1-p "
                                    f"for its physical hosts p (p % {world} == r); NCCL all-gather of passing "
                                    f"rows and query partials") if hosts_mode else
                            "replicas (one independent layer per GPU)"),
        "tflops_layer": round(sz["attn_flops"] / (ms_per_step / 1000.0) / 1e12, 1),
        "roofline": {"bound": "tensor", "kernel": f"attn_kernel<{d}>", "achieved": round(attn_tf, 1),
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": round(attn_tf / peak_tf, 4),
                     "traffic": committed_traffic(wl.name),
                     "peak_source": (f"bf16_tflops_{'sustained' if sustained_region else 'burst'} of {src} "
                                     f"MEASURED_PEAKS.json: the kernel's timed loop ran "
                                     f"{attn_region_s:.2f} s"),
                     "frac_of_burst": round(attn_tf / burst, 4), "frac_of_sustained": round(attn_tf / sustained, 4),
                     "algorithmic_flops_per_launch": flops, "clocks": clk_attn.summary()},
        "stages": stage_info,
        "layer": ("per rank: spava_compress and spava_attn_fwd with the rank's host mask, all-gathers of "
                  "passing rows and query partials, spava_lse_merge") if hosts_mode else
                 ("spava_layer_fwd: query-sum launch, compression cluster launch, then attention with the "
                  "query-partial merge (each a programmatic dependent launch of the one before)"),
        "e2e": None if e2e_ms is None else {
            "value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3),
            "api": "spava_layer_fwd; every step uploads Q,K,V from pinned host memory and downloads "
                   "O,lse; upload, compute and download of consecutive steps overlap on three streams"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        tok, est, secs, desc = oracle_sample(wl, host_inp, seed=0)
        line["cpu_baseline"] = {"value": tok, "unit": "tokens/s", "cores": os.cpu_count(),
                                "threads": cpu_threads(), "kind": "oracle", "sample": desc,
                                "sample_seconds": round(secs, 2), "estimated_seconds_per_layer": round(est, 1)}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="spava", choices=["spava", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--mode", default="replicas", choices=["replicas", "hosts"],
                    help="replicas: one independent layer per GPU (default); hosts: the pages' split of "
                         "one layer's virtual hosts over the GPUs")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from sparse_approximate_attention_b200 import workloads as W
    wl = W.workloads()[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    rc = run_gpu(args, wl)
    rank, world, _ = dist_env()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
