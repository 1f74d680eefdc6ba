#!/usr/bin/env python
"""Benchmark of the sparse MoE FFN forward layer (router + dispatch + routed SwiGLU
experts + weighted combine + shared expert) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--workloads perf|none|NAME,...] [--impl ours|reference]

One step = one whole layer call (moe_layer_forward: router, dispatch, experts,
combine, shared expert) on one batch of seeded synthetic inputs shaped like the
workload, inputs already in HBM.  The headline line is the largest single-GPU
configuration (16384-token skewed group-routed prefill); the other performance
configurations (prefill and decode) are measured in the same run, one after
another, and reported under "workloads".  With N > 1 (launched by torchrun, one
rank per GPU) every rank runs its own replica on its own batch (tokens are
independent, no collective on the data path); the step time is the max over
ranks and `value` counts the tokens of all ranks.  Rank 0 prints one JSON line.
`--impl reference` times the plain fp64 CPU oracle on the same workload instead
(the reference arm of this comparison).
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import CONFIGS, DEFAULT_WORKLOAD, PERF_WORKLOADS, make_inputs  # noqa: E402

METRIC = "MoE-layer tokens/s (prefill, decode) and % of bf16 tensor / HBM roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# The layer's stated targets are fractions of nominal B200 figures: prefill grouped
# GEMMs at >= 60 % of the dense bf16 tensor peak, decode at >= 70 % of ~8 TB/s HBM
# over the bytes of the hit experts.
NOMINAL = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
TARGET = {"hbm": 0.70, "tensor": 0.60}
# Near-tie threshold of the routing comparison: an id may differ from the oracle's
# only where the oracle's fp64 margin is below it.
TIE = 1e-6

BF16_KERNELS = ["dispatch_count", "dispatch_scan", "dispatch_scatter", "dispatch_gather",
                "gate_up_swiglu", "down_combine_shared", "combine"]
F32_KERNELS = ["dispatch_count", "dispatch_scan", "dispatch_scatter", "gate_up_routed",
               "gate_up_shared", "down_routed", "down_shared", "combine"]


# What each --pair setting runs for the prefill expert GEMMs (moe_debug_set_pair_mode).
PAIR_MODES = {
    "default": "library default: down on CTA pairs for experts with an even m-tile count, "
               "the rest and all of gate_up on one SM",
    "off": "every tile on one SM",
    "on": "CTA pairs, odd last m-tiles on one SM",
    "pad": "CTA pairs, odd last m-tiles padded",
    "parity": "gate_up and down on CTA pairs for experts with an even m-tile count",
    "down": "down on CTA pairs for experts with an even m-tile count, gate_up on one SM",
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(CONFIGS))
    ap.add_argument("--workloads", default="perf",
                    help="other configurations measured in the same run and reported under "
                         "'workloads': 'perf' (every other performance configuration), "
                         "'none', or a comma-separated list")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target duration of the oracle's CPU-baseline sample")
    ap.add_argument("--set", action="append", default=[], metavar="FIELD=VALUE",
                    help="override a size of the workload (e.g. E=32) for small profiling cases")
    ap.add_argument("--pair", default="default",
                    choices=["default", "off", "on", "pad", "parity", "down"],
                    help="prefill expert GEMMs on CTA pairs: the library's default, never, "
                         "full pairs with one-SM tails, padded pairs only, even-count experts "
                         "on pairs and the rest on one SM, or that split for down only")
    ap.add_argument("--graph", action="store_true",
                    help="capture the K timed steps as one CUDA graph and time one replay "
                         "(default: launch them one by one)")
    return ap.parse_args()


def workload(name, sets):
    cfg = CONFIGS[name]
    over = {}
    for item in sets:
        key, val = item.split("=", 1)
        cur = getattr(cfg, key)
        over[key] = type(cur)(float(val)) if isinstance(cur, (int, float)) else val
    return cfg.with_(**over) if over else cfg, over


def extra_workloads(args):
    if args.workloads == "none":
        return []
    names = PERF_WORKLOADS if args.workloads == "perf" else args.workloads.split(",")
    return [n for n in names if n != args.workload and n in CONFIGS]


def config_dict(cfg, over, gpus):
    """The workload description (identical in both arms of the comparison)."""
    return {"workload": cfg.name, "description": cfg.description, "N": cfg.N, "D": cfg.D,
            "E": cfg.E, "n_group": cfg.n_group, "topk_group": cfg.topk_group, "k": cfg.k,
            "d_moe": cfg.d_moe, "d_sh": cfg.d_sh, "alpha": cfg.alpha,
            "router_dtype": str(cfg.wg_dtype).replace("torch.", ""),
            "overrides": over or None,
            "parallelism": "replicas" if gpus > 1 else "single",
            "l2": "inputs larger than L2 (the hit experts' weights, GBs per step), no flush"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.proc = None
        self.dev = device_index
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
            return
        # Do not start timing before the sampler produces its first line.
        t0 = time.time()
        while time.time() - t0 < 10.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.05)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == len(self.FIELDS):
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def source_sha(rel: str) -> str:
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def stored_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary (profiles/traffic.json),
    or None when there is none or the kernel's source changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel][workload]
        if rec.get("source_sha") != source_sha(rec["source"]):
            return None
        return float(rec["bytes_per_launch"])
    except (OSError, KeyError, ValueError, TypeError):
        return None


# ---- multi-rank host logic (replicas: one independent batch per rank) --------
def replica_token_seed(rank: int) -> int:
    """Seed of rank r's token batch: rank 0 keeps the workload's own batch (seed 0
    draws), every other rank draws a fresh batch so replicas route differently."""
    return 0 if rank == 0 else 1000 + rank


def max_over_ranks(value: float, dist, device) -> float:
    """Max of a per-rank measurement over all ranks (the job ends with the slowest)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(tokens_per_rank: int, world: int, steps: int, max_ms: float) -> float:
    """Tokens of all ranks over the slowest rank's time for `steps` steps."""
    return tokens_per_rank * world * steps / (max_ms / 1e3)


def kernel_work(cfg, name: str, hit: int):
    """Algorithmic FLOPs and bytes of one launch (routed k experts, shared expert,
    router; weights of hit experts read once, x read once, y written once)."""
    es = 2 if cfg.dtype == torch.bfloat16 else 4
    ws = 2 if cfg.wg_dtype == torch.bfloat16 else 4
    N, D, E, k, d, dsh = cfg.N, cfg.D, cfg.E, cfg.k, cfg.d_moe, cfg.d_sh
    if name == "gate_up_swiglu":
        flops = 2.0 * (N * k * 2 * d + N * 2 * dsh) * D
        byts = (hit * 2 * d + 2 * dsh) * D * es + N * D * es
    elif name == "down_combine_shared":
        flops = 2.0 * (N * k * d + N * dsh) * D
        byts = (hit * d + dsh) * D * es + N * D * es
    elif name == "combine":  # prefill: k slot rows and the fp32 shared row in, y out
        flops = 0.0
        byts = N * k * D * es + N * D * 4 + N * D * es
    elif name == "router":
        flops = 2.0 * N * D * E
        byts = E * D * ws + N * D * es
    else:
        flops, byts = 0.0, 0.0
    return flops, byts


def roofline_of(cfg, name: str, hit: int, ms: float, peaks: dict, peak_src: str) -> dict:
    """Achieved algorithmic rate of one kernel launch against the measured peak (the
    roofline's denominator) and against the nominal figure the layer's targets use."""
    flops, byts = kernel_work(cfg, name, hit)
    dur_s = ms / 1e3
    ridge = peaks["bf16_tflops_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if byts > 0 and flops / byts < ridge:
        roof = {"bound": "hbm", "achieved": byts / dur_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
        nominal = NOMINAL["hbm_gbs"]
    else:
        roof = {"bound": "tensor", "achieved": flops / dur_s / 1e12,
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s"}
        nominal = NOMINAL["bf16_tflops"]
    roof["frac"] = roof["achieved"] / roof["peak"] if roof["peak"] else None
    roof["peak_source"] = peak_src + (" sustained bf16" if roof["bound"] == "tensor" else " copy")
    roof["kernel"] = name
    roof["ms_per_launch"] = ms
    roof["algorithmic"] = {"flops": flops, "bytes": byts}
    roof["vs_nominal"] = {
        "peak": nominal, "unit": roof["unit"], "frac": roof["achieved"] / nominal,
        "target": TARGET[roof["bound"]], "target_is_judged_on_this_fraction": True,
        "what": ("the layer's stated target: prefill grouped GEMMs >= 60 % of the nominal "
                 "dense bf16 peak (2.25 PFLOP/s)" if roof["bound"] == "tensor" else
                 "the layer's stated target: decode >= 70 % of ~8 TB/s over the hit "
                 "experts' bytes")}
    return roof


# ---- the oracle on a sample of tokens (CPU baseline and parity summary) ---------
def compact_experts(inp_dev, ids):
    """Host copies of only the experts in `ids` (and the shared expert), with a map
    from global expert id to its row in the copies; the oracle's arithmetic per
    token is unchanged, only the host memory it needs shrinks."""
    E = inp_dev.gate_up.shape[0]
    hit = sorted({int(e) for e in np.asarray(ids).ravel() if 0 <= int(e) < E})
    sel = torch.tensor(hit, dtype=torch.long, device=inp_dev.gate_up.device)
    remap = np.full(E + 1, len(hit), dtype=np.int32)  # the sentinel stays a sentinel
    remap[hit] = np.arange(len(hit), dtype=np.int32)
    weights = (inp_dev.gate_up.index_select(0, sel).cpu(), inp_dev.down.index_select(0, sel).cpu(),
               inp_dev.sh_gate.cpu(), inp_dev.sh_up.cpu(), inp_dev.sh_down.cpu())
    return weights, remap


def oracle_sample(cfg, x_host, W_g_host, b_host, inp_dev, gpu_ids=None):
    """Oracle router on the sampled tokens, then host copies of the experts they hit
    (by the oracle's routing and, if given, the GPU's).  Returns (route, weights, remap)."""
    import oracle

    r = oracle.router(x_host, W_g_host, b_host, cfg.n_group, cfg.topk_group, cfg.k,
                      cfg.norm_topk_prob, cfg.alpha)
    ids = r["idx"] if gpu_ids is None else np.concatenate([r["idx"].ravel(), gpu_ids.ravel()])
    weights, remap = compact_experts(inp_dev, ids)
    return r, weights, remap


def oracle_time(cfg, x_host, W_g_host, b_host, weights, remap, target_s: float, max_reps: int = 50):
    """Run the oracle (router + forward) on the sampled tokens until target_s has
    elapsed; returns (tokens/s, tokens, seconds, reps, last route, last y)."""
    import oracle

    n = x_host.shape[0]
    done, t0, reps = 0, time.perf_counter(), 0
    while True:
        r = oracle.router(x_host, W_g_host, b_host, cfg.n_group, cfg.topk_group, cfg.k,
                          cfg.norm_topk_prob, cfg.alpha)
        y = oracle.forward(x_host, *weights, remap[r["idx"]], r["w"])
        done += n
        reps += 1
        el = time.perf_counter() - t0
        if el >= target_s or reps >= max_reps:
            return done / el, done, el, reps, r, y


def parity_summary(cfg, r, y_ref, gpu_idx, gpu_w, gpu_y, b_host) -> dict:
    """Routing and output agreement of the GPU step with the oracle on the sampled rows:
    id mismatches (allowed only at near-ties of margin < 1e-6), near-tie count,
    weight error over alpha and the output errors (max|y - y_ref| / max|y_ref| and
    the largest row-wise relative L2 error) on the rows whose routing agrees."""
    oi = r["idx"].astype(np.int64)
    gi = gpu_idx.astype(np.int64)
    near = (r["margin_exp"] < TIE) | (r["margin_grp"] < TIE)
    sp = r["s"] + b_host.double().numpy()[None, :]
    chosen = np.take_along_axis(sp, oi, axis=1)
    if oi.shape[1] > 1:
        near |= np.min(chosen[:, :-1] - chosen[:, 1:], axis=1) < TIE
    mism = np.any(gi != oi, axis=1)
    same = ~mism
    werr = float(np.max(np.abs(gpu_w[same] - r["w"][same]))) / cfg.alpha if same.any() else 0.0
    y = gpu_y[same].astype(np.float64)
    ref = y_ref[same]
    scale = np.max(np.abs(ref)) if ref.size else 1.0
    row = (np.linalg.norm(y - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-300)
           if ref.size else np.zeros(1))
    return {"rows": int(len(oi)), "id_mismatch_tokens": int(mism.sum()),
            "unexplained_mismatches": int((mism & ~near).sum()),
            "near_tie_tokens": int(near.sum()), "max_w_err_over_alpha": werr,
            "max_rel": float(np.max(np.abs(y - ref)) / scale) if ref.size else 0.0,
            "max_row_l2_rel": float(np.max(row)),
            "tolerance": 2e-2 if cfg.dtype == torch.bfloat16 else 1e-5}


def run_reference(args):
    """Reference arm: the fp64 CPU oracle on the same workload, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle

    cfg, over = workload(args.workload, args.set)
    gen_dev = "cuda:0" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(cfg, seed=0, device=gen_dev)
    cores = oracle.num_threads()
    W_g_host, b_host = inp.W_g.cpu(), inp.b.cpu()
    # Size each step's sample so that warm-up + timed steps end within ~2 minutes:
    # time a probe of `cores` tokens first.
    probe = min(cfg.N, cores, 16)
    xp = inp.x[:probe].cpu().contiguous()
    _, wts, remap = oracle_sample(cfg, xp, W_g_host, b_host, inp)
    _, _, t1, _, _, _ = oracle_time(cfg, xp, W_g_host, b_host, wts, remap, 0.0, max_reps=1)
    per_tok = t1 / probe
    budget = 120.0 / max(args.steps + args.warmup, 1)
    # at most 64 tokens: the host copies hold only the experts the sample hits
    sample = int(max(1, min(cfg.N, 64, budget / max(per_tok, 1e-9))))
    x = inp.x[:sample].cpu().contiguous()
    _, wts, remap = oracle_sample(cfg, x, W_g_host, b_host, inp)
    del inp
    if torch.cuda.is_available():
        torch.cuda.empty_cache()

    def step():
        r = oracle.router(x, W_g_host, b_host, cfg.n_group, cfg.topk_group, cfg.k,
                          cfg.norm_topk_prob, cfg.alpha)
        oracle.forward(x, *wts, remap[r["idx"]], r["w"])

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = sample * args.steps / el
    desc = ("fp64 oracle (router + forward) on the first %d of the %d tokens of %s per step "
            "(host copies of the experts those tokens hit)" % (sample, cfg.N, cfg.name))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(cfg, over, args.gpus),
            "sample_tokens_per_step": sample,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def link_bandwidth(nbytes: int, dev) -> dict:
    """Pinned host <-> device copy rates for one step's x / y size (the e2e bound):
    host-to-device alone, device-to-host alone, and both at once on two streams."""
    n = max(nbytes // 2, 1)
    h_in = torch.empty(n, dtype=torch.bfloat16).pin_memory()
    h_out = torch.empty(n, dtype=torch.bfloat16).pin_memory()
    d_in = torch.empty(n, dtype=torch.bfloat16, device=dev)
    d_out = torch.empty(n, dtype=torch.bfloat16, device=dev)
    s1, s2 = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    res = {}

    def timed(fn, reps=5):
        fn()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(reps):
            fn()
        torch.cuda.synchronize()
        return (time.perf_counter() - t0) / reps

    def h2d():
        with torch.cuda.stream(s1):
            d_in.copy_(h_in, non_blocking=True)

    def d2h():
        with torch.cuda.stream(s2):
            h_out.copy_(d_out, non_blocking=True)

    def both():
        h2d()
        d2h()

    b = 2 * n
    res["h2d_gbs"] = b / timed(h2d) / 1e9
    res["d2h_gbs"] = b / timed(d2h) / 1e9
    t = timed(both)
    res["concurrent_h2d_plus_d2h_gbs"] = 2 * b / t / 1e9
    res["bytes"] = b
    res["ms_per_step_copies_alone"] = t * 1e3
    return res


def measure(cfg, over, args, dev, dist, rank, world, local, moe, full: bool):
    """Time K layer steps of one configuration; returns the result dict (every rank
    takes the same collective steps).  full: also the e2e link diagnostics."""
    inp = make_inputs(cfg, seed=0, device=dev)
    if rank > 0:  # each replica gets its own batch of tokens
        from workloads import make_tokens
        inp.x = make_tokens(cfg, cfg.N, seed=replica_token_seed(rank), device=dev)
    N, D = cfg.N, cfg.D
    ws = torch.empty(max(moe.moe_layer_forward_workspace(N, D, cfg.E, cfg.d_moe, cfg.d_sh, cfg.k,
                                                         cfg.dtype, cfg.wg_dtype), 256),
                     dtype=torch.uint8, device=dev)
    y = torch.empty((N, D), dtype=cfg.dtype, device=dev)
    idx = torch.empty((N, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((N, cfg.k), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    kernels = BF16_KERNELS if cfg.dtype == torch.bfloat16 else F32_KERNELS
    if cfg.N * cfg.k <= 2048:  # one fused dispatch kernel; its marks fill the first slot
        kernels = ["dispatch", "_", "_"] + kernels[3:]

    def step(x, st=None, out=None):
        # one library call: router, dispatch, experts, combine, shared expert
        moe.moe_layer(x, inp.W_g, inp.b, inp.gate_up, inp.down, inp.sh_gate, inp.sh_up,
                      inp.sh_down, cfg.n_group, cfg.topk_group, cfg.k, cfg.norm_topk_prob,
                      cfg.alpha, ws, y if out is None else out, idx, w,
                      stream if st is None else st)

    for _ in range(max(args.warmup, 3)):
        step(inp.x)
    status = moe.moe_device_status(stream)
    if status != 0:
        raise SystemExit("device status after warm-up: %s" % moe.moe_status_string(status))
    loads = torch.bincount(idx.flatten().long(), minlength=cfg.E)
    hit = int((loads > 0).sum().item())
    # Routing collisions: (token, expert) pairs served per distinct expert whose
    # weights the step streams, and the routed weight bytes fetched per token.
    routing = {"hit_experts": hit,
               "max_over_mean_load": float(loads.max().item() / loads.float().mean().item()),
               "reuse_factor": float(loads.sum().item()) / max(hit, 1),
               "routed_weight_bytes_per_token":
                   hit * 3.0 * cfg.D * cfg.d_moe * inp.gate_up.element_size() / cfg.N}

    # Events at the layer call's kernel boundaries: start, after the router (which
    # includes the dispatch and gather when they are fused into it), then after each
    # later kernel.  Recording all of them costs the decode step about 2 % (event
    # records between kernels), so an untimed profiling pass with every boundary
    # gives the per-kernel times and names the dominant kernel, and the timed
    # region records only the two events around that kernel.
    K = args.steps
    nk = len(kernels)
    names = ["router"] + kernels               # kernel i spans events i .. i + 1

    def make_rows(n):
        # external=True: recorded as graph nodes when the steps are captured into a graph
        rows = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(nk + 2)]
                for _ in range(n)]
        for row in rows:  # create the underlying CUDA events
            for e in row:
                e.record(stream)
        return rows

    P = min(K, 50)
    prof_rows = make_rows(P)
    torch.cuda.synchronize()
    for s_ in range(P):
        moe.moe_profile_set_events(prof_rows[s_])
        step(inp.x)
    moe.moe_profile_set_events([])
    torch.cuda.synchronize()
    per = {}
    for i, name in enumerate(names):
        if name != "_":
            per[name] = sum(prof_rows[s][i].elapsed_time(prof_rows[s][i + 1])
                            for s in range(P)) / P
    dom = max(per, key=per.get)
    di = names.index(dom)
    evs = make_rows(K)
    torch.cuda.synchronize()

    def timed_steps():
        st = torch.cuda.current_stream()  # the capture stream while a graph is captured
        for s_ in range(K):
            row = [e if j in (di, di + 1) else None for j, e in enumerate(evs[s_])]
            moe.moe_profile_set_events(row)
            step(inp.x, st)
        moe.moe_profile_set_events([])

    # With --graph the K steps are captured once as a CUDA graph (kernel launches,
    # their profiling events and all) and replayed once inside the timed region.
    graph = None
    launches_per_replay = None
    if args.graph:
        try:
            g = torch.cuda.CUDAGraph()
            c0 = moe.moe_launch_count()
            with torch.cuda.graph(g):
                timed_steps()
            launches_per_replay = moe.moe_launch_count() - c0
            g.replay()  # untimed first replay (graph upload), also a warm-up pass
            torch.cuda.synchronize()
            graph = g
        except RuntimeError as exc:  # capture refused: fall back to launching the steps
            print("graph capture failed, timing launches instead: %s" % exc, file=sys.stderr)
            moe.moe_profile_set_events([])
            graph = None
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    launches0 = moe.moe_launch_count()
    start.record(stream)
    if graph is not None:
        graph.replay()
    else:
        timed_steps()
    end.record(stream)
    end.synchronize()
    launches = launches_per_replay if graph is not None else moe.moe_launch_count() - launches0
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    status = moe.moe_device_status(stream)
    if status != 0:
        raise SystemExit("device status after timing: %s" % moe.moe_status_string(status))
    total_ms = max_over_ranks(start.elapsed_time(end), dist, dev)
    ms_per_step = total_ms / K
    value = whole_job_tokens_per_s(N, world, K, total_ms)

    # The dominant kernel's duration over the timed region (its two events per step).
    dom_ms = sum(evs[s][di].elapsed_time(evs[s][di + 1]) for s in range(K)) / K
    peaks, peak_src = load_peaks()
    roof = roofline_of(cfg, dom, hit, dom_ms, peaks, peak_src)
    roof["traffic"] = stored_traffic(dom, cfg.name) if not over else None
    # Every expert kernel's rate from the untimed profiling pass (same denominators).
    per_kernel = {name: {k2: v for k2, v in roofline_of(cfg, name, hit, per[name], peaks,
                                                         peak_src).items()
                         if k2 in ("bound", "achieved", "unit", "frac", "ms_per_launch")}
                  for name in ("router", "gate_up_swiglu", "down_combine_shared", "combine")
                  if name in per and kernel_work(cfg, name, hit) != (0.0, 0.0)}
    for name, rec in per_kernel.items():
        rec["frac_of_nominal"] = rec["achieved"] / (NOMINAL["hbm_gbs"] if rec["bound"] == "hbm"
                                                    else NOMINAL["bf16_tflops"])

    # End to end: every step copies its x in from pinned host memory, runs the layer
    # and copies its y out to pinned host memory, all inside the timed region.  As in a
    # serving loop the copies run on two copy streams with two buffer sets, so step
    # i+1's x comes in and step i-1's y goes out while step i computes.
    NB = 2
    x_host = [inp.x.cpu().pin_memory() for _ in range(NB)]
    y_host = [torch.empty((N, D), dtype=cfg.dtype).pin_memory() for _ in range(NB)]
    x_dev = [torch.empty_like(inp.x) for _ in range(NB)]
    y_dev = [torch.empty_like(y) for _ in range(NB)]
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_steps(n, start):
        arrived = [torch.cuda.Event() for _ in range(NB)]
        computed = [torch.cuda.Event() for _ in range(NB)]
        left = [torch.cuda.Event() for _ in range(NB)]
        h2d.wait_event(start)
        d2h.wait_event(start)
        for i in range(n):
            bi = i % NB
            with torch.cuda.stream(h2d):
                if i >= NB:
                    h2d.wait_event(computed[bi])  # step i-2 has read x_dev[bi]
                x_dev[bi].copy_(x_host[bi], non_blocking=True)
                arrived[bi].record(h2d)
            stream.wait_event(arrived[bi])
            if i >= NB:
                stream.wait_event(left[bi])       # step i-2's y_dev[bi] is on the host
            step(x_dev[bi], out=y_dev[bi])
            computed[bi].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(computed[bi])
                y_host[bi].copy_(y_dev[bi], non_blocking=True)
                left[bi].record(d2h)
        for bi in range(min(n, NB)):
            stream.wait_event(left[bi])

    s0 = torch.cuda.Event()
    s0.record(stream)
    e2e_steps(3, s0)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_steps(K, e0)
    e1.record(stream)
    e1.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    e2e_value = whole_job_tokens_per_s(N, world, K, e2e_ms)
    # the layer is bitwise deterministic: the last step's y on the host must equal the
    # device-timed steps' y (same tokens)
    e2e_matches = bool(torch.equal(y_host[(K - 1) % NB].to(dev), y))
    es = inp.x.element_size()
    clocks = sampler.stop()
    e2e = {"value": e2e_value, "unit": UNIT, "ms_per_step": e2e_ms / K,
           "h2d_bytes_per_step": N * D * es, "d2h_bytes_per_step": N * D * es,
           "copies": "pinned host buffers, two copy streams, double-buffered: overlapped "
                     "with the neighbouring steps' compute",
           "copies_declared": True, "output_matches_device_step": e2e_matches}
    if full:
        e2e["link"] = link_bandwidth(N * D * es, dev)

    res = {"value": value, "ms_per_step": ms_per_step, "routing": routing, "roofline": roof,
           "kernels": per_kernel, "kernel_ms": per, "e2e": e2e, "gpu_launches": int(launches),
           "timing": "one replay of a CUDA graph of the K steps" if graph is not None
                     else "K steps launched one by one",
           "clocks": clocks}
    # What the CPU leg needs, kept on the host (rank 0 of a one-GPU run only): the
    # sampled tokens, the GPU's routing and output rows for them, and host copies
    # of the experts they hit.
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n = min(cfg.N, 16 if full else 8)
        res["_sample"] = {"x": inp.x[:n].cpu().contiguous(), "W_g": inp.W_g.cpu(),
                          "b": inp.b.cpu(), "idx": idx[:n].cpu().numpy(),
                          "w": w[:n].cpu().double().numpy(), "y": y[:n].float().cpu().numpy()}
        _, wts, remap = oracle_sample(cfg, res["_sample"]["x"], res["_sample"]["W_g"],
                                      res["_sample"]["b"], inp, res["_sample"]["idx"])
        res["_sample"]["weights"], res["_sample"]["remap"] = wts, remap
    del graph
    del inp, ws, y, idx, w, x_host, y_host, x_dev, y_dev
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def cpu_leg(cfg, smp, seconds):
    """The oracle on the sampled tokens for ~`seconds` (the CPU baseline), and the parity
    summary of the GPU step's rows against that oracle run."""
    import oracle

    v, done, el, reps, r, y_ref = oracle_time(cfg, smp["x"], smp["W_g"], smp["b"],
                                              smp["weights"], smp["remap"], seconds)
    n = smp["x"].shape[0]
    cpu = {"value": v, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
           "sample": "fp64 oracle router + forward on the first %d tokens of the %d-token "
                     "batch, %d repetitions, %.1f s" % (n, cfg.N, reps, el)}
    par = parity_summary(cfg, r, y_ref, smp["idx"], smp["w"], smp["y"], smp["b"])
    return cpu, par


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    import sparse_moe_layer_02_b200 as moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=60), device_id=dev)

    moe.moe_debug_set_pair_mode(
        {"default": -1, "off": 0, "on": 1, "pad": 2, "parity": 3, "down": 4}[args.pair])
    cfg, over = workload(args.workload, args.set)
    head = measure(cfg, over, args, dev, dist, rank, world, local, moe, full=True)
    cpu, par = None, None
    if "_sample" in head:  # rank 0 of a one-GPU run: the oracle on the host cores
        cpu, par = cpu_leg(cfg, head.pop("_sample"), args.cpu_seconds)
    others, others_par = {}, {}
    for name in extra_workloads(args):
        c2, o2 = workload(name, [])
        others[name] = measure(c2, o2, args, dev, dist, rank, world, local, moe, full=False)
        if "_sample" in others[name]:
            _, others_par[name] = cpu_leg(c2, others[name].pop("_sample"), 0.0)

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if cfg.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": config_dict(cfg, over, world),
        "routing": head["routing"],
        "roofline": head["roofline"],
        "kernels": head["kernels"],
        "kernel_ms": head["kernel_ms"],
        "kernel_ms_source": "untimed profiling pass of %d steps with an event at every kernel "
                            "boundary; the timed region records only the two events around "
                            "the dominant kernel (roofline.ms_per_launch)" % min(args.steps, 50),
        "cpu_baseline": cpu,
        "parity": par,
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "timing": head["timing"],
        "gemm_pairs": PAIR_MODES[args.pair],
        "clocks": head["clocks"],
        "workloads": {
            name: {"value": res["value"], "unit": UNIT, "ms_per_step": res["ms_per_step"],
                   "config": config_dict(CONFIGS[name], None, world),
                   "routing": res["routing"], "roofline": res["roofline"],
                   "kernels": res["kernels"], "kernel_ms": res["kernel_ms"], "e2e": res["e2e"],
                   "gpu_launches": res["gpu_launches"], "clocks": res["clocks"],
                   "parity": others_par.get(name)}
            for name, res in others.items()},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
