"""Benchmark: GLM-5.2-shaped routed-MoE decode layer on B200.

Workload (one "step"): 1000 independent seeded tokens, each run at batch 1
through one MoE layer (hidden 6144, expert inter 2048, 256 int4 experts + 1
shared, top-8, n_group 8, topk_group 4, rsf 2.5), every token a full
moe_layer_forward call (router, noaux_tc selection, 8 routed + shared expert
FFNs, combine).  Tokens rotate over C independently generated layer copies
(default 8, 43.7 GB) so the weights are never L2-resident: each token reads
197.4 MB > 126 MB of L2, and a copy's shared expert and router are re-read
only after 7 other copies' traffic.

Metric: token-layers per second at batch-1 decode (whole job, all ranks),
plus achieved HBM GB/s of the decode kernel against the measured peak.
With --gpus N (torchrun) each rank runs its own replica of the workload
(independent tokens, no data-path collective): weak scaling.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload on the host cores (the reference arm of this build).
"""
import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed-MoE decode tok/s (GLM-5.2 shape) and HBM GB/s as % of B200 peak"
UNIT = "tok/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--tokens", type=int, default=1000, help="tokens per step")
    p.add_argument("--copies", type=int, default=8, help="rotating layer copies")
    p.add_argument("--no-graph", action="store_true", help="launch eagerly instead of a CUDA graph")
    p.add_argument("--cpu-sample", type=int, default=6, help="tokens in the CPU-baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--small", action="store_true", help="tiny layer (smoke/profiling only)")
    p.add_argument("--experts", type=int, default=0,
                   help="routed experts per layer (profiling only; default: the shape's 256)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes_per_token(shape):
    """9 experts (8 routed + shared) + fp32 router + bias + bf16 x + fp32 y."""
    E, H = shape.n_experts, shape.hidden
    return ((shape.top_k + shape.n_shared) * shape.expert_bytes + E * H * 4 + E * 4 + H * 2 + H * 4)


def kernel_source_hash():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "int4_routed_expert_noaux_b200", "csrc")
    for fn in sorted(os.listdir(d)):
        h.update(open(os.path.join(d, fn), "rb").read())
    return h.hexdigest()[:16]


def traffic_from_profile(kernel):
    """dram bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    ent = d.get(kernel)
    if not ent or ent.get("source_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        self.p.wait()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle leg

def cpu_oracle_rate(shape, n_tokens, seed=0):
    """Time the fp64 oracle (all host threads) on n_tokens tokens of layer
    copy 0: router + selection + 9 expert FFNs + combine per token.  Inputs
    are generated before the clock starts."""
    import oracle
    import synth
    threads = oracle.set_threads(0)
    W, b = synth.router(shape, seed, 0)
    x_bits = synth.tokens(shape, seed, 0, n_tokens)
    lg = oracle.router_logits(shape, W, x_bits[:1])
    idx_all = []
    for t in range(n_tokens):
        lg = oracle.router_logits(shape, W, x_bits[t:t + 1])
        idx, _, _, _ = oracle.route(shape, lg, b)
        idx_all.append(idx[0])
    needed = sorted(set(int(e) for r in idx_all for e in r))
    experts = {e: synth.expert(shape, seed, 0, e) for e in needed}
    shared = synth.expert(shape, seed, 0, shape.n_experts)
    t0 = time.perf_counter()
    for t in range(n_tokens):
        lg = oracle.router_logits(shape, W, x_bits[t:t + 1])
        idx, w, _, _ = oracle.route(shape, lg, b)
        xd = synth.bf16_to_f32(x_bits[t:t + 1]).astype(np.float64)
        oracle.experts_combine(shape, experts, shared, xd, idx, w)
    dt = time.perf_counter() - t0
    return n_tokens / dt, threads, dt


def run_reference(args, shape):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = max(1, args.cpu_sample // 3)
    for _ in range(args.warmup):
        cpu_oracle_rate(shape, 1)
    times, threads = [], 1
    for _ in range(args.steps):
        rate, threads, dt = cpu_oracle_rate(shape, per_step)
        times.append(dt)
    total = sum(times)
    value = per_step * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(args, shape, per_step),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{per_step} tokens per step of layer copy 0, full layer"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(args, shape, tokens):
    return {"workload": ("GLM-5.2-shaped MoE layer, batch-1 decode, all experts resident in HBM"
                         if not args.small else "tiny MoE layer, batch-1 decode"),
            "hidden": shape.hidden, "inter": shape.inter, "n_experts": shape.n_experts,
            "n_shared": shape.n_shared, "top_k": shape.top_k, "n_group": shape.n_group,
            "topk_group": shape.topk_group, "rsf": shape.rsf, "tokens_per_step": tokens,
            "batch": 1, "layer_copies": args.copies,
            "l2": "inputs larger than L2 (197 MB per token; copies rotate)",
            "parallelism": f"replicas x{args.gpus}"}


# ---------------------------------------------------------------------------
# GPU leg

def main():
    args = parse()
    import synth
    shape = synth.TINY if args.small else synth.GLM
    if args.experts:
        import dataclasses
        shape = dataclasses.replace(shape, n_experts=args.experts)
    if args.impl == "reference":
        run_reference(args, shape)
        return

    import torch
    import int4_routed_expert_noaux_b200 as moe
    from synth.layers import DeviceLayer

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    cfg = moe.Config.from_shape(shape)
    copies = max(1, args.copies)
    layers, views = [], []
    for c in range(copies):
        dl = DeviceLayer(shape, 0, c)
        layers.append(dl)
        views.append(moe.Layer(cfg, dl.w_router, dl.bias, dl.routed, dl.shared))
    torch.cuda.synchronize()

    n = args.tokens
    x_bits = synth.tokens(shape, 1000 * rank, 0, n)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    y = torch.empty((n, shape.hidden), dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(cfg, 1)
    stream = torch.cuda.Stream()

    def step(s):
        for t in range(n):
            views[t % copies].forward(x[t:t + 1], y[t:t + 1], ws, stream=s)

    with torch.cuda.stream(stream):
        step(stream)
    stream.synchronize()
    moe.ws_check(ws, stream)

    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step(stream)
        stream.synchronize()

    def run_once():
        if graph is not None:
            graph.replay()
        else:
            step(stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            run_once()
    stream.synchronize()

    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = Clocks(local)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps):
            run_once()
        ev1.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1)
    moe.ws_check(ws, stream)
    if dist:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
        dist.barrier()
    ms_step = ms / args.steps
    tokens_total = n * args.steps * world
    value = tokens_total / (ms / 1000.0)

    # e2e: host buffers, per-token pinned H2D of x and D2H of y in the timed region
    x_host = torch.from_numpy(x_bits.view(np.int16)).pin_memory()
    y_host = torch.empty((n, shape.hidden), dtype=torch.float32).pin_memory()
    xd = torch.empty((1, shape.hidden), dtype=torch.int16, device="cuda")
    yd = torch.empty((1, shape.hidden), dtype=torch.float32, device="cuda")

    def e2e_step():
        for t in range(n):
            xd.copy_(x_host[t:t + 1], non_blocking=True)
            views[t % copies].forward(xd, yd, ws, stream=stream)
            y_host[t:t + 1].copy_(yd, non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_step()
    stream.synchronize()
    e2e_steps = max(1, min(args.steps, 3))
    if dist:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
    stream.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if dist:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_value = n * e2e_steps * world / (e2e_ms / 1000.0)
    if not np.all(np.isfinite(y_host.numpy())):
        raise RuntimeError("non-finite outputs")

    peak, peak_kind = peaks()
    bytes_tok = algorithmic_bytes_per_token(shape)
    launch_us = ms_step * 1000.0 / n
    achieved = bytes_tok / (launch_us * 1e-6) / 1e9
    kernel = "moe_layer_forward (per token)"
    roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": traffic_from_profile(kernel),
            "peak_source": peak_kind, "kernel": kernel,
            "algorithmic_bytes_per_launch": bytes_tok, "launch_us": launch_us}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, threads, dt = cpu_oracle_rate(shape, args.cpu_sample)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{args.cpu_sample} tokens of layer copy 0, full layer, {dt:.1f} s"}

    if dist:
        dist.barrier()
        graph = None
        dist.destroy_process_group()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4xf32",
            "data": "synthetic", "config": config_dict(args, shape, n),
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT,
                    "h2d_bytes_per_step": n * shape.hidden * 2,
                    "d2h_bytes_per_step": n * shape.hidden * 4},
            "gpu_launches": n * args.steps * launches_per_forward(),
            "clocks": clk, "graph": graph is not None or not args.no_graph,
            "hbm_gbs": achieved,
        }
        print(json.dumps(line), flush=True)


def launches_per_forward():
    return 1


if __name__ == "__main__":
    main()
