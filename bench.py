#!/usr/bin/env python
"""Benchmark of the sparse MoE FFN forward layer (router + dispatch + routed SwiGLU
experts + weighted combine + shared expert) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one whole layer call (moe_router then moe_forward) on one batch of
seeded synthetic inputs shaped like the workload, inputs already in HBM.  With
N > 1 (launched by torchrun, one rank per GPU) every rank runs its own replica
on its own batch (tokens are independent, no collective on the data path); the
step time is the max over ranks and `value` counts the tokens of all ranks.
Rank 0 prints one JSON line.  `--impl reference` times the plain fp64 CPU oracle
on the same workload instead (the reference arm of this comparison).
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

import torch  # noqa: E402

from workloads import CONFIGS, DEFAULT_WORKLOAD, make_inputs  # noqa: E402

METRIC = "MoE-layer tokens/s (prefill, decode) and % of bf16 tensor / HBM roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

BF16_KERNELS = ["dispatch_count", "dispatch_scan", "dispatch_scatter", "dispatch_gather",
                "gate_up_swiglu", "down_combine_shared", "combine"]
F32_KERNELS = ["dispatch_count", "dispatch_scan", "dispatch_scatter", "gate_up_routed",
               "gate_up_shared", "down_routed", "down_shared", "combine"]


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target duration of the oracle's CPU-baseline sample")
    ap.add_argument("--set", action="append", default=[], metavar="FIELD=VALUE",
                    help="override a size of the workload (e.g. E=32) for small profiling cases")
    ap.add_argument("--graph", action="store_true",
                    help="capture the K timed steps as one CUDA graph and time one replay "
                         "(default: launch them one by one)")
    return ap.parse_args()


def workload(args):
    cfg = CONFIGS[args.workload]
    over = {}
    for item in args.set:
        key, val = item.split("=", 1)
        cur = getattr(cfg, key)
        over[key] = type(cur)(float(val)) if isinstance(cur, (int, float)) else val
    return cfg.with_(**over) if over else cfg, over


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


def oracle_time(cfg, inp_host, n_tokens: int, target_s: float, max_reps: int = 50):
    """Run the oracle (router + forward) on the first n_tokens of the batch until
    target_s has elapsed; returns (tokens/s, tokens, seconds, reps)."""
    import oracle

    x = inp_host.x[:n_tokens].contiguous()
    done, t0, reps = 0, time.perf_counter(), 0
    while True:
        r = oracle.router(x, inp_host.W_g, inp_host.b, cfg.n_group, cfg.topk_group, cfg.k,
                          cfg.norm_topk_prob, cfg.alpha)
        oracle.forward(x, inp_host.gate_up, inp_host.down, inp_host.sh_gate, inp_host.sh_up,
                       inp_host.sh_down, r["idx"], r["w"])
        done += n_tokens
        reps += 1
        el = time.perf_counter() - t0
        if el >= target_s or reps >= max_reps:
            return done / el, done, el, reps


def run_reference(args):
    """Reference arm: the fp64 CPU oracle on the same workload, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle

    cfg, over = workload(args)
    gen_dev = "cuda:0" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(cfg, seed=0, device=gen_dev).to("cpu")
    cores = oracle.num_threads()
    # Size each step's sample so that warm-up + timed steps end within ~2 minutes.
    _, _, t1, _ = oracle_time(cfg, inp, min(cfg.N, cores), 0.0, max_reps=1)
    per_tok = t1 / min(cfg.N, cores)
    budget = 120.0 / max(args.steps + args.warmup, 1)
    sample = int(max(1, min(cfg.N, budget / max(per_tok, 1e-9))))
    x = inp.x[:sample].contiguous()

    def step():
        r = oracle.router(x, inp.W_g, inp.b, cfg.n_group, cfg.topk_group, cfg.k,
                          cfg.norm_topk_prob, cfg.alpha)
        oracle.forward(x, inp.gate_up, inp.down, inp.sh_gate, inp.sh_up, inp.sh_down, r["idx"],
                       r["w"])

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = sample * args.steps / el
    desc = "fp64 oracle (router + forward) on the first %d of %d tokens of %s per step" % (
        sample, cfg.N, cfg.name)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "description": cfg.description, "N": cfg.N,
                       "D": cfg.D, "E": cfg.E, "k": cfg.k, "d_moe": cfg.d_moe,
                       "sample_tokens_per_step": sample, "overrides": over or None},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


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

    cfg, over = workload(args)
    inp = make_inputs(cfg, seed=0, device=dev)
    if rank > 0:  # each replica gets its own batch of tokens
        from workloads import make_tokens
        inp.x = make_tokens(cfg, cfg.N, seed=replica_token_seed(rank), device=dev)
    N, D = cfg.N, cfg.D
    ws = torch.empty(max(moe.moe_forward_workspace(N, D, cfg.E, cfg.d_moe, cfg.d_sh, cfg.k,
                                                   cfg.dtype), 256), dtype=torch.uint8, device=dev)
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
    max_over_mean = float(loads.max().item() / loads.float().mean().item())
    # Routing collisions: (token, expert) pairs served per distinct expert whose
    # weights the step streams, and the routed weight bytes fetched per token.
    reuse = float(loads.sum().item()) / max(hit, 1)
    routed_bytes_per_token = hit * 3.0 * cfg.D * cfg.d_moe * inp.gate_up.element_size() / cfg.N

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
    flops, byts = kernel_work(cfg, dom, hit)
    dur_s = dom_ms / 1e3
    ridge = peaks["bf16_tflops_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if byts > 0 and flops / byts < ridge:
        roof = {"bound": "hbm", "achieved": byts / dur_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": flops / dur_s / 1e12,
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"] if roof["peak"] else None
    roof["traffic"] = stored_traffic(dom, cfg.name) if not over else None
    roof["kernel"] = dom
    roof["peak_source"] = peak_src + (" sustained bf16" if roof["bound"] == "tensor" else " copy")
    roof["ms_per_launch"] = dom_ms
    roof["algorithmic"] = {"flops": flops, "bytes": byts}

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
    e2e_value = whole_job_tokens_per_s(N, world, K, max_over_ranks(e0.elapsed_time(e1), dist, dev))
    # the layer is bitwise deterministic: the last step's y on the host must equal the
    # device-timed steps' y (same tokens)
    e2e_matches = bool(torch.equal(y_host[(K - 1) % NB].to(dev), y))
    es = inp.x.element_size()
    clocks = sampler.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        host = inp.to("cpu")
        n = min(cfg.N, 32)
        v, done, el, reps = oracle_time(cfg, host, n, args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
               "sample": "fp64 oracle router + forward on the first %d tokens of the %d-token "
                         "batch, %d repetitions, %.1f s" % (n, cfg.N, reps, el)}

    used_graph = graph is not None
    del graph
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if cfg.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": {"workload": cfg.name, "description": cfg.description, "N": N, "D": D,
                   "E": cfg.E, "n_group": cfg.n_group, "topk_group": cfg.topk_group, "k": cfg.k,
                   "d_moe": cfg.d_moe, "d_sh": cfg.d_sh, "alpha": cfg.alpha,
                   "router_dtype": str(cfg.wg_dtype).replace("torch.", ""),
                   "hit_experts": hit, "max_over_mean_load": max_over_mean,
                   "reuse_factor": reuse, "routed_weight_bytes_per_token": routed_bytes_per_token,
                   "overrides": over or None,
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "inputs larger than L2 (hit-expert weights %.2f GB per step)"
                         % (kernel_work(cfg, "gate_up_swiglu", hit)[1] / 1e9
                            + kernel_work(cfg, "down_combine_shared", hit)[1] / 1e9)},
        "roofline": roof,
        "kernel_ms": per,
        "kernel_ms_source": "untimed profiling pass of %d steps with an event at every kernel "
                            "boundary; the timed region records only the two events around "
                            "the dominant kernel (roofline.ms_per_launch)" % P,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": N * D * es,
                "d2h_bytes_per_step": N * D * es,
                "copies": "pinned host buffers, two copy streams, double-buffered: overlapped "
                          "with the neighbouring steps' compute",
                "output_matches_device_step": e2e_matches},
        "gpu_launches": int(launches),
        "timing": "one replay of a CUDA graph of the K steps" if used_graph
                  else "K steps launched one by one",
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
