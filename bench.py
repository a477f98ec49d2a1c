#!/usr/bin/env python
"""Selective Head Attention decode benchmark (one JSON line on stdout, rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config NAME]

A step is one selective-head decode call over a whole batch (one attention
layer, one decode token per sequence) on the OPT-66B-shaped workload: B=64,
H=72, d=128, N_kv=1920, top_k=22 (30 % head density), fp16, N(0,1) data.
Inputs are resident in HBM when the timed region starts; the active K/V of a
step (1.39 GB) is 11x the 126 MB L2, so no flush is needed between steps.
Device-timed steps are launched by replaying CUDA graphs of 100 steps, as the
pages measure decode throughput under CUDA graphs; e2e calls the API eagerly.

value    = algorithmic bytes of all ranks' steps / max-over-ranks device time
           (active K+V, active Q rows read, active O rows written, the index)
roofline = the same bytes per launch / mean launch time, against the measured
           HBM copy bandwidth of this GPU pool (MEASURED_PEAKS.json, else the
           fallback figure), and beside a copy kernel timed in this run
e2e      = the same metric through the public API with the step's per-token
           inputs (q, index) copied from pinned host memory and the output
           copied back inside the timed region, transfers overlapped with the
           neighbouring steps' decode on separate streams (the serial schedule
           is reported beside it); the KV cache is model state and stays resident
cpu_baseline = the float64 oracle on the host cores, on a sample of units

With --gpus N (torchrun, one process per GPU) every rank decodes its own
batch (weak scaling: the path needs no exchange between GPUs).
--impl reference times the float64 CPU oracle on the same workload instead.
"""
import argparse
import datetime
import glob
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = ("SHA decode: achieved HBM GB/s (% of B200 peak) and decode steps/sec vs density")
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=4000)
    p.add_argument("--warmup", type=int, default=100)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", default="opt66b", choices=sorted(workloads.CONFIGS))
    p.add_argument("--layout", default="head_major",
                   choices=["head_major", "token_major", "varlen", "paged16", "tokens4"],
                   help="K/V cache of the timed step: [B, H_kv, N_kv, d] (sha_decode), "
                        "[B, N_kv, H_kv, d] (sha_decode_strided), per-row lengths uniform in "
                        "[1, N_kv] (sha_decode_varlen), 16-key pages in random pool order "
                        "(sha_decode_paged), or each selected head attending to a seeded "
                        "random quarter of its keys (sha_decode_tokens); all but head_major "
                        "imply --no-extras")
    p.add_argument("--sustained-s", type=float, default=1.5,
                   help="seconds of graph-replayed steps in the sustained leg (0 skips it)")
    p.add_argument("--batch", type=int, default=None,
                   help="override the workload's batch size (small ncu captures)")
    p.add_argument("--no-extras", action="store_true",
                   help="skip the density sweep, e2e and CPU baseline (used for ncu)")
    p.add_argument("--cpu-budget", type=float, default=10.0,
                   help="seconds of oracle work for cpu_baseline")
    p.add_argument("--sweep", action="store_true",
                   help="run the LLaMA-2-7B-shaped scaling sweep instead (one JSON line)")
    p.add_argument("--mlp", action="store_true",
                   help="run the Selective GEMM (OPT-66B MLP) measurement instead")
    p.add_argument("--mlp-density", type=float, nargs="*", default=None,
                   help="union densities for --mlp (default 0.1 0.3 0.5 1.0)")
    return p.parse_args()


# ---------------------------------------------------------------- environment

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback (no MEASURED_PEAKS.json)"


# the sources the selective-head decode kernels are built from (kernels, their
# helpers and the launch path); a change to any of them voids a stored capture
DECODE_SOURCES = ("sha_decode.cu", "sha_device.cuh", "sha_gqa_kernel.cuh", "sha_lookahead.cuh",
                  "sha_merge.cuh", "sha_mha_kernel.cuh", "sha_mma.cuh", "sha_schedule.cuh",
                  "sha_walk.cuh")


def strip_comments(src):
    """C/C++ source without its comments (string and character literals kept),
    so that rewording a comment does not retire the ncu counters taken on the
    code."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "".join(out)


def kernel_source_hash():
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "head_sparse_decode_b200", "csrc", name)) as f:
            code = strip_comments(f.read())
            # blank lines and trailing spaces are where removed comments were
            code = "\n".join(ln.rstrip() for ln in code.splitlines() if ln.strip())
            h.update(name.encode() + b"\0" + code.encode())
    return h.hexdigest()


def profiled_traffic(workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    current = kernel_source_hash()
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        text = open(path).read()
        m_hash = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
        m_val = re.search(r"traffic_bytes_per_launch\[" + re.escape(workload) + r"\]:\s*(\d+)",
                          text)
        if m_hash and m_val and m_hash.group(1) == current:
            return int(m_val.group(1))
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples, stamped with wall time."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.samples = []
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", uuid, "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, RuntimeError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 7:
                self.samples.append((time.time(), parts))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        window = [s for t, s in self.samples if t0 <= t <= t1] or [s for _, s in self.samples]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for s in window for i in range(4)
                          if s[3 + i].lower().startswith("active")})

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(s[0]) for s in window if num(s[0]) is not None]
        mx = [num(s[1]) for s in window if num(s[1]) is not None]
        pw = [num(s[2]) for s in window if num(s[2]) is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "samples": len(window), "reasons": reasons}


# ---------------------------------------------------------------- oracle timing

def gather_units(w, q, k, v, idx, units):
    idx_h = idx.cpu().numpy()
    pairs = [(int(u) // w.top_k, int(idx_h[int(u) // w.top_k, int(u) % w.top_k])) for u in units]
    G = w.G
    qu = torch.stack([q[b, h * G:(h + 1) * G].cpu() for b, h in pairs])
    ku = torch.stack([k[b, h].cpu() for b, h in pairs])
    vu = torch.stack([v[b, h].cpu() for b, h in pairs])
    return qu, ku, vu


def cpu_baseline(w, q, k, v, idx, budget_s, max_units=128):
    import oracle
    rng = np.random.default_rng(0)
    units = rng.choice(w.units, size=min(max_units, w.units), replace=False)
    qu, ku, vu = gather_units(w, q, k, v, idx, units)
    per_unit = w.algorithmic_bytes() / w.units
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.sha_units(qu, ku, vu, w.scale, w.dtype)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            break
    return {"value": per_unit * len(units) * reps / dt / 1e9, "unit": "GB/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(units)} seeded-random (batch row, head) units of {w.name} "
                      f"x {reps} passes, {dt:.1f} s, float64 C oracle with OpenMP"}


# ---------------------------------------------------------------- timing helpers

def timed(fn, steps, stream):
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / 1e3   # seconds


def capture_graph(fn, n, dev):
    """n calls of fn captured into one CUDA graph (fn already warmed up)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(n):
            fn()
    return g


def timed_graphs(fn, steps, dev, stream, chunk=100, per_step=None):
    """Exactly `steps` calls of fn, launched by replaying CUDA graphs of up to
    `chunk` calls (the pages measure decode throughput under CUDA graphs), timed
    with events on `stream`.  Returns seconds.  per_step: a list that receives
    the mean seconds per call of each full graph replay (events between the
    replays, inside the same timed region)."""
    chunk = max(1, min(chunk, steps))
    g_main = capture_graph(fn, chunk, dev)
    rem = steps % chunk
    g_rem = capture_graph(fn, rem, dev) if rem else None
    g_main.replay()                       # first replay uploads the graph
    torch.cuda.synchronize(dev)
    n_main = steps // chunk
    marks = ([torch.cuda.Event(enable_timing=True) for _ in range(n_main + 1)]
             if per_step is not None else None)

    def run():
        for i in range(n_main):
            if marks is not None:
                marks[i].record(stream)
            g_main.replay()
        if marks is not None:
            marks[n_main].record(stream)
        if g_rem is not None:
            g_rem.replay()
    t = timed(run, 1, stream)
    if marks is not None:
        per_step.extend(marks[i].elapsed_time(marks[i + 1]) / 1e3 / chunk for i in range(n_main))
    return t


def step_distribution(per_step, chunk):
    """p10 / median / p90 of the per-call time over the graph replays (us)."""
    if not per_step:
        return None
    xs = sorted(per_step)
    pick = lambda q: xs[min(len(xs) - 1, int(q * (len(xs) - 1) + 0.5))] * 1e6
    return {"p10_us": round(pick(0.1), 3), "median_us": round(pick(0.5), 3),
            "p90_us": round(pick(0.9), 3), "graph_replays": len(xs),
            "calls_per_replay": chunk}


def sync_all(world, local):
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize()


def max_over_ranks(x, world, device="cuda"):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world, device="cuda"):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_workload(config, rank, batch=None):
    """The batch shard rank `rank` decodes: the config's shape, its own seed."""
    base = workloads.CONFIGS[config]
    if batch:
        base = base.with_(B=batch)
    return base.with_(seed=base.seed + 100 * rank)


def aggregate(bytes_per_step, steps, elapsed_s, world, device="cuda"):
    """Whole-job GB/s (all ranks' bytes / slowest rank's time) and that time."""
    t_max = max_over_ranks(elapsed_s, world, device)
    total = sum_over_ranks(bytes_per_step * steps, world, device)
    return total / t_max / 1e9, t_max


# ---------------------------------------------------------------- arms

KV_LAYOUTS = {"head_major": "[B, H_kv, N_kv, d]",
              "token_major": "[B, N_kv, H_kv, d] (strided views)",
              "varlen": "[B, H_kv, N_kv, d], per-row lengths uniform in [1, N_kv]",
              "paged16": "pool [pages, H_kv, 16, d] + block table, random page order",
              "tokens4": "[B, H_kv, N_kv, d], a listed quarter of each selected head's keys"}


def paged_cache(k, v, w, page_size, dev):
    """k, v [B, H_kv, N_kv, d] moved into a page pool in random page order:
    (k_pages, v_pages, block_table, lengths), all on dev."""
    P = -(-w.N_kv // page_size)
    n_pages = w.B * P
    gc = torch.Generator().manual_seed(w.seed + 3)
    table = torch.randperm(n_pages, generator=gc).to(torch.int32).view(w.B, P).to(dev)
    kp = torch.zeros((n_pages, w.H_kv, page_size, w.d), dtype=k.dtype, device=dev)
    vp = torch.zeros_like(kp)
    pad = P * page_size - w.N_kv
    for b in range(w.B):
        kb = torch.nn.functional.pad(k[b], (0, 0, 0, pad)).view(w.H_kv, P, page_size, w.d)
        vb = torch.nn.functional.pad(v[b], (0, 0, 0, pad)).view(w.H_kv, P, page_size, w.d)
        kp[table[b].long()] = kb.permute(1, 0, 2, 3)
        vp[table[b].long()] = vb.permute(1, 0, 2, 3)
    lens = torch.full((w.B,), w.N_kv, dtype=torch.int32, device=dev)
    return kp, vp, table, lens


def sustained_leg(sha, step, bytes_step, launch_s, seconds, dev, stream, world, local, peak):
    """The same step replayed for about `seconds` (graphs of 100 steps), with its
    own clock record: the rate a decode server sees under the power cap, beside
    the short burst of the main timing."""
    steps = max(100, int(math.ceil(seconds / max(launch_s, 1e-7) / 100.0)) * 100)
    sampler = ClockSampler(dev)
    time.sleep(0.3)                       # first samples before the load starts
    sync_all(world, local)
    t0 = time.time()
    elapsed = timed_graphs(step, steps, dev, stream)
    t1 = time.time()
    sync_all(world, local)
    clocks = sampler.stop(t0, t1)
    status = sha.sha_get_device_status()
    if status != sha.SHA_OK:
        raise RuntimeError(f"device status after the sustained leg: {sha.sha_status_string(status)}")
    value, t_max = aggregate(bytes_step, steps, elapsed, world)
    return {"value": round(value, 2), "unit": "GB/s", "steps": steps,
            "seconds": round(t_max, 3), "ms_per_step": round(t_max / steps * 1e3, 5),
            "frac_of_measured": round(bytes_step * steps / t_max / 1e9 / peak, 4),
            "gpu_launches": steps, "clocks": clocks}


def run_ours(args, rank, world, local):
    import head_sparse_decode_b200 as sha

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = rank_workload(args.config, rank, args.batch)   # each rank decodes its own batch
    q, k, v = workloads.make_qkv(w, device=dev)
    idx = workloads.make_index(w).to(dev)
    out = workloads.make_out(w, dev)
    stream = torch.cuda.current_stream(dev)

    bytes_step = w.algorithmic_bytes()
    if args.layout == "token_major":
        # the same values stored [B, N_kv, H_kv, d], read through strided views
        k = k.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
        v = v.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
        torch.cuda.empty_cache()
        args.no_extras = True

        def step():
            sha.sha_decode_strided(q, k, v, idx, w.scale, out)
    elif args.layout == "varlen":
        # row b attends to its first lens[b] keys, lengths uniform in [1, N_kv]
        args.no_extras = True
        g = torch.Generator().manual_seed(w.seed + 11)
        lens = torch.randint(1, w.N_kv + 1, (w.B,), generator=g, dtype=torch.int32)
        lens_d = lens.to(dev)
        bytes_step = (sum(2 * int(L) * w.d * 2 * w.top_k for L in lens.tolist())
                      + 2 * w.units * w.G * w.d * 2 + 4 * w.units + 4 * w.B)

        def step():
            sha.sha_decode_varlen(q, k, v, idx, lens_d, w.scale, out)
    elif args.layout == "tokens4":
        # each selected head attends to a seeded random quarter of its keys
        args.no_extras = True
        n_sel = w.N_kv // 4
        tok = workloads.make_tokens(w, n_sel).to(dev)
        bytes_step = (w.units * 2 * n_sel * w.d * 2 + 2 * w.units * w.G * w.d * 2
                      + 4 * w.units + 4 * w.units * n_sel)

        def step():
            sha.sha_decode_tokens(q, k, v, idx, tok, w.scale, out)
    elif args.layout == "paged16":
        # the cache in 16-key pages scattered over a pool in random order
        args.no_extras = True
        kp, vp, table, lens_d = paged_cache(k, v, w, 16, dev)
        del k, v
        torch.cuda.empty_cache()
        bytes_step = w.algorithmic_bytes() + 4 * w.B + 4 * table.numel()

        def step():
            sha.sha_decode_paged(q, kp, vp, idx, lens_d, table, w.scale, out)
    else:
        def step():
            sha.decode(q, k, v, idx, w.scale, out)

    # same-run HBM copy probe (1 GiB read + 1 GiB written)
    src = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    src.fill_(1)
    for _ in range(3):
        sha.sha_copy_bandwidth_probe(dst, src)
    t = timed(lambda: sha.sha_copy_bandwidth_probe(dst, src), 20, stream)
    copy_gbs = 2 * src.numel() * 20 / t / 1e9
    del src, dst
    torch.cuda.empty_cache()

    sampler = ClockSampler(dev)
    for _ in range(args.warmup):
        step()
    sync_all(world, local)
    t0 = time.time()
    per_step = []
    elapsed = timed_graphs(step, args.steps, dev, stream, per_step=per_step)
    t1 = time.time()
    sync_all(world, local)
    clocks = sampler.stop(t0, t1)
    status = sha.sha_get_device_status()
    if status != sha.SHA_OK:
        raise RuntimeError(f"device status after timing: {sha.sha_status_string(status)}")

    value, t_max = aggregate(bytes_step, args.steps, elapsed, world)
    launch_s = elapsed / args.steps
    achieved = bytes_step / launch_s / 1e9
    peak, peak_src = measured_peak()
    sustained = None
    if args.sustained_s > 0:
        sustained = sustained_leg(sha, step, bytes_step, launch_s, args.sustained_s, dev,
                                  stream, world, local, peak)

    extras = {}
    if not args.no_extras:
        extras["density_sweep"] = density_sweep(sha, w, q, k, v, dev, stream, peak)
        extras["e2e"] = e2e(sha, w, q, k, v, idx, out, dev, stream, args)
        extras["other_configs"] = other_configs(sha, w, dev, stream, peak, rank)
        extras["other_configs"].append(varlen_config(sha, dev, stream, peak, rank))
        extras["other_configs"].append(paged_config(sha, dev, stream, peak, rank))
        extras["other_configs"].append(tokens_config(sha, dev, stream, peak, rank))
        extras["other_configs"].extend(strided_configs(sha, dev, stream, peak, rank))
        mlp = run_mlp(argparse.Namespace(batch=None), dev)
        extras["selective_mlp"] = {"config": mlp["config"], "cublas_dense_us": mlp["cublas_dense_us"],
                                   "points": mlp["points"]}
    plan = sha.sha_decode_plan_ex(
        w.B, w.H_q, w.H_kv, w.N_kv, w.d, w.top_k,
        num_sms=torch.cuda.get_device_properties(dev).multi_processor_count,
        cluster_capacity=sha.sha_decode_cluster_capacity(w.d, dev))
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t_max / args.steps * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic N(0,1), seeded",
        "config": {**w.describe(), "parallelism": f"replicas x{world} (batch sharded by rank)",
                   "accumulation": "fp32", "l2": "no flush: bytes moved per step "
                   f"{bytes_step / 1e9:.2f} GB > 126 MB L2",
                   "blocks": plan["blocks"], "tile_keys": plan["tile_keys"],
                   "cluster": plan["cluster"],
                   "kv_layout": KV_LAYOUTS[args.layout],
                   "launch": "CUDA graph replay, 100 steps per graph"},
        "steps_per_s": round(args.steps / t_max, 2),
        # the per-call time of each 100-call graph replay of the timed region
        "step_time": step_distribution(per_step, min(100, args.steps)),
        "tokens_per_s": round(world * w.B * args.steps / t_max, 1),
        "hbm_frac_of_measured": round(achieved / peak, 4),
        "copy_probe_gbs": round(copy_gbs, 1),
        "clocks": clocks,
        "sustained": sustained,
        "gpu_launches": args.steps,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": profiled_traffic(w.name) if args.layout == "head_major" else None,
                     "peak_source": peak_src,
                     # multi-head calls with d = 128 run on the grouped kernel's tensor cores
                     "kernel": "sha_mha_decode_kernel"
                               if w.G == 1 and (w.d != 128 or args.layout in ("varlen", "paged16"))
                               else "sha_gqa_decode_kernel",
                     "launch_us": round(launch_s * 1e6, 3),
                     "bytes_per_launch": bytes_step},
    }
    if "e2e" in extras:
        line["e2e"] = extras.pop("e2e")
    line.update(extras)
    if rank == 0 and world == 1 and not args.no_extras:
        line["cpu_baseline"] = cpu_baseline(w, q, k, v, idx, args.cpu_budget)
    return line


def density_sweep(sha, w, q, k, v, dev, stream, peak):
    """Same shape at 25/50/75/100 % head density (100 % = the dense reference)."""
    res = []
    for frac in (0.25, 0.5, 0.75, 1.0):
        top_k = max(1, round(frac * w.H_kv))
        wk = w.with_(top_k=top_k)
        idx = workloads.make_index(wk).to(dev)
        out = workloads.make_out(wk, dev)
        for _ in range(20):
            sha.decode(q, k, v, idx, w.scale, out)
        steps = 300
        t = timed_graphs(lambda: sha.decode(q, k, v, idx, w.scale, out), steps, dev, stream)
        gbs = wk.algorithmic_bytes() * steps / t / 1e9
        res.append({"top_k": top_k, "density": round(top_k / w.H_kv, 4),
                    "us_per_step": round(t / steps * 1e6, 2), "gbs": round(gbs, 1),
                    "frac": round(gbs / peak, 4), "steps_per_s": round(steps / t, 1)})
    dense = res[-1]["us_per_step"]
    for r in res:
        r["time_vs_dense"] = round(r["us_per_step"] / dense, 4)
    return res


def other_configs(sha, w_main, dev, stream, peak, rank):
    """The other full-size workloads, timed the same way (fewer steps)."""
    res = []
    for name in ("llama2_7b", "llama31_70b_gqa", "llama2_7b_ctx16k", "llama31_70b_gqa_ctx16k"):
        if name == w_main.name:
            continue
        w = workloads.CONFIGS[name]
        w = w.with_(seed=w.seed + 100 * rank)
        q, k, v = workloads.make_qkv(w, device=dev)
        idx = workloads.make_index(w).to(dev)
        out = workloads.make_out(w, dev)
        for _ in range(20):
            sha.decode(q, k, v, idx, w.scale, out)
        steps = 500
        t = timed_graphs(lambda: sha.decode(q, k, v, idx, w.scale, out), steps, dev, stream)
        gbs = w.algorithmic_bytes() * steps / t / 1e9
        res.append({"workload": name, "us_per_step": round(t / steps * 1e6, 2),
                    "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
                    "steps_per_s": round(steps / t, 1), "G": w.G, "dtype": w.dtype,
                    "bytes_per_step": w.algorithmic_bytes()})
        del q, k, v, idx, out
        torch.cuda.empty_cache()
    return res


def strided_configs(sha, dev, stream, peak, rank):
    """OPT-66B and LLaMA-3.1-70B shapes with the cache stored token-major,
    [B, N_kv, H_kv, d] (sha_decode_strided): each key row of a head is H_kv*d
    elements from the next."""
    res = []
    for name in ("opt66b", "llama31_70b_gqa"):
        w = workloads.CONFIGS[name].with_(seed=workloads.CONFIGS[name].seed + 100 * rank + 7)
        q, k, v = workloads.make_qkv(w, device=dev)
        k = k.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
        v = v.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
        torch.cuda.empty_cache()
        idx = workloads.make_index(w).to(dev)
        out = workloads.make_out(w, dev)

        def call():
            sha.sha_decode_strided(q, k, v, idx, w.scale, out)
        for _ in range(20):
            call()
        steps = 500
        t = timed_graphs(call, steps, dev, stream)
        gbs = w.algorithmic_bytes() * steps / t / 1e9
        res.append({"workload": name + "_token_major", "layout": "[B, N_kv, H_kv, d]",
                    "us_per_step": round(t / steps * 1e6, 2), "gbs": round(gbs, 1),
                    "frac": round(gbs / peak, 4), "steps_per_s": round(steps / t, 1),
                    "bytes_per_step": w.algorithmic_bytes()})
        del q, k, v, idx, out
        torch.cuda.empty_cache()
    return res


def varlen_config(sha, dev, stream, peak, rank):
    """LLaMA-2-7B shape with per-row cache lengths drawn uniformly from [1, 4096]
    (a decode batch of sequences of different lengths)."""
    w = workloads.CONFIGS["llama2_7b"].with_(N_kv=4096, seed=2500 + 100 * rank)
    q, k, v = workloads.make_qkv(w, device=dev)
    idx = workloads.make_index(w).to(dev)
    out = workloads.make_out(w, dev)
    g = torch.Generator().manual_seed(w.seed + 11)
    lens = torch.randint(1, w.N_kv + 1, (w.B,), generator=g, dtype=torch.int32)
    lens_d = lens.to(dev)
    # algorithmic bytes: active K+V of each row's own length, Q/O rows, index, lengths
    kv = sum(2 * int(L) * w.d * 2 * w.top_k for L in lens.tolist())
    nbytes = kv + 2 * w.units * w.G * w.d * 2 + 4 * w.units + 4 * w.B

    def call():
        sha.sha_decode_varlen(q, k, v, idx, lens_d, w.scale, out)
    for _ in range(20):
        call()
    steps = 500
    t = timed_graphs(call, steps, dev, stream)
    gbs = nbytes * steps / t / 1e9
    res = {"workload": "llama2_7b_varlen", "lengths": "uniform [1, 4096], seeded",
           "mean_len": round(float(lens.float().mean()), 1), "us_per_step": round(t / steps * 1e6, 2),
           "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
           "steps_per_s": round(steps / t, 1), "bytes_per_step": nbytes}
    del q, k, v
    torch.cuda.empty_cache()
    return res


def tokens_config(sha, dev, stream, peak, rank, keep=4):
    """OPT-66B shape with head x token sparsity: every selected head attends to a
    seeded random quarter of its keys (sha_decode_tokens)."""
    w = workloads.CONFIGS["opt66b"].with_(seed=1700 + 100 * rank)
    q, k, v = workloads.make_qkv(w, device=dev)
    idx = workloads.make_index(w).to(dev)
    n_sel = w.N_kv // keep
    tok = workloads.make_tokens(w, n_sel).to(dev)
    out = workloads.make_out(w, dev)
    # algorithmic bytes: the listed K+V rows, Q/O rows, the index and the lists
    nbytes = (w.units * 2 * n_sel * w.d * 2 + 2 * w.units * w.G * w.d * 2 + 4 * w.units
              + 4 * w.units * n_sel)

    def call():
        sha.sha_decode_tokens(q, k, v, idx, tok, w.scale, out)
    for _ in range(20):
        call()
    steps = 500
    t = timed_graphs(call, steps, dev, stream)
    gbs = nbytes * steps / t / 1e9
    res = {"workload": "opt66b_tokens_quarter", "keys_per_head": n_sel,
           "us_per_step": round(t / steps * 1e6, 2), "gbs": round(gbs, 1),
           "frac": round(gbs / peak, 4), "steps_per_s": round(steps / t, 1),
           "bytes_per_step": nbytes}
    del q, k, v, tok
    torch.cuda.empty_cache()
    return res


def paged_config(sha, dev, stream, peak, rank, page_size=16):
    """OPT-66B shape with its cache in 16-key pages scattered over a pool in
    random order (the serving layout), every row 1920 long."""
    w = workloads.CONFIGS["opt66b"].with_(seed=1500 + 100 * rank)
    P = -(-w.N_kv // page_size)
    n_pages = w.B * P
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    q = torch.randn((w.B, w.H_q, w.d), generator=g, device=dev).half()
    kp = torch.randn((n_pages, w.H_kv, page_size, w.d), generator=g, device=dev).half()
    vp = torch.randn((n_pages, w.H_kv, page_size, w.d), generator=g, device=dev).half()
    gc = torch.Generator().manual_seed(w.seed + 3)
    table = torch.randperm(n_pages, generator=gc).to(torch.int32).view(w.B, P).to(dev)
    lens = torch.full((w.B,), w.N_kv, dtype=torch.int32, device=dev)
    idx = workloads.make_index(w).to(dev)
    out = workloads.make_out(w, dev)
    nbytes = w.algorithmic_bytes() + 4 * w.B + 4 * w.B * P

    def call():
        sha.sha_decode_paged(q, kp, vp, idx, lens, table, w.scale, out)
    for _ in range(20):
        call()
    steps = 500
    t = timed_graphs(call, steps, dev, stream)
    gbs = nbytes * steps / t / 1e9
    res = {"workload": f"opt66b_paged{page_size}", "page_size": page_size,
           "us_per_step": round(t / steps * 1e6, 2), "gbs": round(gbs, 1),
           "frac": round(gbs / peak, 4), "steps_per_s": round(steps / t, 1),
           "bytes_per_step": nbytes}
    del q, kp, vp
    torch.cuda.empty_cache()
    return res


def e2e(sha, w, q, k, v, idx, out, dev, stream, args):
    """The metric through the public API with each step's per-token inputs (q, the
    head index) copied in from pinned host memory and its output copied back, all
    inside the timed region.  Two schedules of the same calls:

    serial     one stream: copy in, decode, copy out, step after step;
    pipelined  three buffer sets and three streams: step i+1's inputs and step
               i-1's output cross PCIe while step i decodes (what a serving loop
               that overlaps its transfers sees).  This one is the reported value.
    """
    nb = 3
    q_h = [q.cpu().pin_memory() for _ in range(nb)]
    idx_h = [idx.cpu().pin_memory() for _ in range(nb)]
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(nb)]
    q_d = [q] + [torch.empty_like(q) for _ in range(nb - 1)]
    idx_d = [idx] + [torch.empty_like(idx) for _ in range(nb - 1)]
    out_d = [out] + [torch.empty_like(out) for _ in range(nb - 1)]

    def step_serial():
        q.copy_(q_h[0], non_blocking=True)
        idx.copy_(idx_h[0], non_blocking=True)
        sha.decode(q, k, v, idx, w.scale, out)
        out_h[0].copy_(out, non_blocking=True)

    for _ in range(10):
        step_serial()
    steps = max(10, min(args.steps, 2000))
    t_serial = timed(step_serial, steps, stream)

    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(nb)]
    ev_dec = [torch.cuda.Event() for _ in range(nb)]
    ev_out = [torch.cuda.Event() for _ in range(nb)]

    def step_pipelined(i):
        b = i % nb
        with torch.cuda.stream(s_in):
            if i >= nb:
                s_in.wait_event(ev_dec[b])           # step i-nb has read q_d[b], idx_d[b]
            q_d[b].copy_(q_h[b], non_blocking=True)
            idx_d[b].copy_(idx_h[b], non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if i >= nb:
            stream.wait_event(ev_out[b])             # step i-nb's output has left out_d[b]
        with torch.cuda.stream(stream):
            sha.decode(q_d[b], k, v, idx_d[b], w.scale, out_d[b])
        ev_dec[b].record(stream)
        s_out.wait_event(ev_dec[b])
        with torch.cuda.stream(s_out):
            out_h[b].copy_(out_d[b], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(nb + 7):
        step_pipelined(i)
    torch.cuda.synchronize(dev)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    s_in.wait_event(start)
    for i in range(steps):
        step_pipelined(i)
    end.record(s_out)                                # after the last step's output copy
    end.synchronize()
    t = start.elapsed_time(end) / 1e3
    torch.cuda.synchronize(dev)
    h2d = q.numel() * q.element_size() + idx.numel() * idx.element_size()
    d2h = out.numel() * out.element_size()
    nbytes = w.algorithmic_bytes()
    return {"value": round(nbytes * steps / t / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(t / steps * 1e3, 5), "steps": steps,
            "schedule": "pipelined: 3 buffer sets, copy-in / decode / copy-out streams",
            "serial": {"value": round(nbytes * steps / t_serial / 1e9, 2),
                       "ms_per_step": round(t_serial / steps * 1e3, 5)}}


def run_reference(args):
    """The float64 CPU oracle as a bench arm, on bounded samples of the workload."""
    import oracle

    w = workloads.CONFIGS[args.config]
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    q, k, v = workloads.make_qkv(w, device=dev)
    idx = workloads.make_index(w)
    rng = np.random.default_rng(1)
    pool = rng.choice(w.units, size=min(64, w.units), replace=False)
    qu, ku, vu = gather_units(w, q, k, v, idx, pool)
    del q, k, v
    per_unit = w.algorithmic_bytes() / w.units
    oracle.sha_units(qu[:1], ku[:1], vu[:1], w.scale, w.dtype)
    t0 = time.perf_counter()
    oracle.sha_units(qu[:8], ku[:8], vu[:8], w.scale, w.dtype)
    t_unit = (time.perf_counter() - t0) / 8
    budget = 90.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(len(pool), budget // max(t_unit, 1e-9))))

    def step(i):
        s = (i * n) % len(pool)
        sel = [(s + j) % len(pool) for j in range(n)]
        oracle.sha_units(qu[sel], ku[sel], vu[sel], w.scale, w.dtype)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    value = per_unit * n * args.steps / dt / 1e9
    cores = oracle.num_threads()
    sample = (f"each step: {n} of a fixed pool of {len(pool)} seeded-random units of {w.name} "
              f"(float64 C oracle, OpenMP)")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic N(0,1), seeded",
        "config": {**w.describe(), "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


L2_BYTES = 126 * 1024 * 1024


def run_mlp(args, dev=None):
    """Selective GEMM on the OPT-66B MLP (hidden 9216, 36864 neurons) at decode
    batch B: union densities 10-100 %, against the same kernels at 100 % and
    against a dense cuBLAS MLP (torch.matmul) on the same weights."""
    import head_sparse_decode_b200 as sha

    dev = dev if dev is not None else torch.device("cuda", dist_env()[2])
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peak, peak_src = measured_peak()
    base = workloads.MLP_CONFIGS["opt66b_mlp"]
    if args.batch:
        base = base.with_(B=args.batch)
    sampler = ClockSampler(dev)
    t_start = time.time()
    x, W1t, W2t, _ = workloads.make_mlp(base.with_(density=1.0), device=dev)
    ws = torch.empty(sha.sha_selective_mlp_workspace_size(base.B, base.d, base.D, dev),
                     dtype=torch.uint8, device=dev)
    y = torch.empty((base.B, base.d), dtype=x.dtype, device=dev)
    points = []
    densities = getattr(args, "mlp_density", None) or (0.1, 0.3, 0.5, 1.0)
    for dens in densities:
        w = base.with_(density=dens)
        _, _, _, active = workloads.make_mlp(w.with_(d=256), device="cpu")   # mask only
        active = active.to(dev)
        S, n_S = sha.sha_mlp_union(active)
        uws = torch.empty(sha._lib.sha_mlp_union_workspace_size(w.D), dtype=torch.uint8,
                          device=dev)

        def union():
            sha.sha_mlp_union(active, S, n_S, uws)

        def layer():
            union()
            sha.sha_selective_mlp(x, W1t, W2t, S, n_S, y, workspace=ws)
        for _ in range(10):
            layer()
        steps = 200
        t = timed_graphs(layer, steps, dev, stream, chunk=50)
        us = t / steps * 1e6
        # the union's own time, replayed alone the same way
        t_union = timed_graphs(union, steps, dev, stream, chunk=50)
        nbytes = w.algorithmic_bytes()
        points.append({"density": dens, "n_union": w.n_union(), "us_per_layer": round(us, 2),
                       "union_us": round(t_union / steps * 1e6, 2),
                       "gbs": round(nbytes / (us * 1e-6) / 1e9, 1),
                       "frac": round(nbytes / (us * 1e-6) / 1e9 / peak, 4),
                       "bytes_per_layer": nbytes})
    dense_us = points[-1]["us_per_layer"]

    def cublas():
        torch.matmul(torch.relu(torch.matmul(x, W1t.t())), W2t, out=y)
    for _ in range(10):
        cublas()
    t = timed_graphs(cublas, 200, dev, stream, chunk=50)
    cublas_us = t / 200 * 1e6
    clocks = sampler.stop(t_start, time.time())
    for p in points:
        p["speedup_vs_dense_selective"] = round(dense_us / p["us_per_layer"], 3)
        p["speedup_vs_cublas_dense"] = round(cublas_us / p["us_per_layer"], 3)
    del x, W1t, W2t
    torch.cuda.empty_cache()
    return {"metric": "Selective GEMM (OPT-66B MLP): achieved HBM GB/s and speedup vs dense",
            "clocks": clocks,
            "unit": "GB/s", "peak": peak, "peak_source": peak_src,
            "config": {"B": base.B, "d": base.d, "D": base.D, "dtype": base.dtype,
                       "activation": "relu", "launch": "CUDA graph replay (union + MLP)",
                       "l2": "weights 1.36 GB > 126 MB L2"},
            "cublas_dense_us": round(cublas_us, 2), "points": points}


def linear_fit(xs, ys):
    """Least-squares y = a + b x and its R^2."""
    n = len(xs)
    mx, my = sum(xs) / n, sum(ys) / n
    sxx = sum((x - mx) ** 2 for x in xs)
    sxy = sum((x - mx) * (y - my) for x, y in zip(xs, ys))
    b = sxy / sxx
    a = my - b * mx
    ss_res = sum((y - a - b * x) ** 2 for x, y in zip(xs, ys))
    ss_tot = sum((y - my) ** 2 for y in ys)
    return a, b, (1.0 - ss_res / ss_tot) if ss_tot > 0 else 1.0


def run_sweep(args):
    """B x N_kv x density grid of the LLaMA-2-7B shape (H=32, d=128, fp16).

    Where one copy of the inputs would sit in L2, the timed graph cycles
    through enough independent copies (replicas) that every pass touches at
    least 4x L2 of K/V, so the figures are HBM figures."""
    import head_sparse_decode_b200 as sha

    dev = torch.device("cuda", dist_env()[2])
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peak, peak_src = measured_peak()
    points, fits = [], []
    pi = 0
    for B in workloads.SWEEP_B:
        for N in workloads.SWEEP_N:
            w0 = workloads.sweep(B, N, workloads.SWEEP_TOPK[-1], pi)
            kv_bytes = 2 * w0.B * w0.H_kv * w0.N_kv * w0.d * 2
            reps = max(1, math.ceil(4 * L2_BYTES / kv_bytes))
            data = [workloads.make_qkv(w0.with_(seed=w0.seed + 17 * r), device=dev)
                    for r in range(reps)]
            times = []
            for top_k in workloads.SWEEP_TOPK:
                w = w0.with_(top_k=top_k, name=f"sweep_B{B}_N{N}_k{top_k}")
                idx = workloads.make_index(w).to(dev)
                outs = [workloads.make_out(w, dev) for _ in range(reps)]
                calls = [lambda q=q, k=k, v=v, o=o: sha.decode(q, k, v, idx, w.scale, o)
                         for (q, k, v), o in zip(data, outs)]
                for c in calls:
                    c()

                def one_pass():
                    for c in calls:
                        c()
                est = w.algorithmic_bytes() / (0.8 * peak * 1e9)      # s per call
                passes = int(min(200, max(5, math.ceil(0.02 / (est * reps)))))
                t = timed_graphs(one_pass, passes, dev, stream, chunk=max(1, 100 // reps))
                us = t / (passes * reps) * 1e6
                gbs = w.algorithmic_bytes() / (us * 1e-6) / 1e9
                times.append(us)
                points.append({"B": B, "N_kv": N, "top_k": top_k,
                               "density": round(top_k / w.H_kv, 4), "us_per_step": round(us, 3),
                               "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
                               "replicas": reps})
                pi += 1
            a, b, r2 = linear_fit(list(workloads.SWEEP_TOPK), times)
            fits.append({"B": B, "N_kv": N, "intercept_us": round(a, 3),
                         "us_per_head": round(b, 4), "r2": round(r2, 5),
                         "t_over_dense": [round(t / times[-1], 4) for t in times]})
            del data
            torch.cuda.empty_cache()
    return {"metric": METRIC, "sweep": "LLaMA-2-7B shape, H=32, d=128, fp16",
            "unit": "GB/s", "peak": peak, "peak_source": peak_src,
            "densities": [k / 32 for k in workloads.SWEEP_TOPK], "points": points,
            "fits": fits,
            "l2": "inputs rotated over >= 4x L2 of K/V per pass where one copy is smaller",
            "launch": "CUDA graph replay"}


def main():
    args = parse_args()
    rank, world, local = dist_env()
    if args.sweep:
        if rank == 0:
            print(json.dumps(run_sweep(args)), flush=True)
        return
    if args.mlp:
        if rank == 0:
            print(json.dumps(run_mlp(args)), flush=True)
        return
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    try:
        line = run_ours(args, rank, world, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
