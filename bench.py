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
workload on the host cores: there is no other implementation to run.
"""
import argparse
import ctypes
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
    p.add_argument("--cpu-sample", type=int, default=64, help="tokens in the CPU-baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--small", action="store_true", help="tiny layer (smoke/profiling only)")
    p.add_argument("--experts", type=int, default=0,
                   help="routed experts per layer (profiling only; default: the shape's 256)")
    p.add_argument("--mode", default="layer",
                   choices=["layer", "verify", "stack", "stream", "timeline"],
                   help="layer: batch-1 decode of one layer (the headline); verify: T-token "
                        "calls; stack: one token through 24 layers; stream: host-streamed "
                        "experts through the LRU cache; timeline: per-phase times of the "
                        "one-token kernel from its probe build")
    p.add_argument("--verify-T", default="2,3,4,8,32", help="tokens per verify call")
    p.add_argument("--timeline-sm-mhz", type=float, default=1965.0,
                   help="timeline: SM clock that converts clock64 probes to time")
    p.add_argument("--correlated", action="store_true",
                   help="verify: draft tokens x0 + 0.05 eps (heavily shared experts)")
    p.add_argument("--stack-layers", type=int, default=24)
    p.add_argument("--stream-layers", type=int, default=75,
                   help="stream: at most this many layers in pinned host memory (75, the "
                        "model's MoE layers; fewer when host memory is smaller)")
    p.add_argument("--stream-caps", default="8,16,32,64,128", help="stream: cache slots per layer")
    p.add_argument("--stream-router-caps", default="32,128",
                   help="stream: cache sizes also run with the device router's ids")
    p.add_argument("--stream-tokens", type=int, default=512)
    p.add_argument("--top-p", type=float, default=1.0,
                   help="adaptive expert top-p of every layer (>= 1: off, the headline)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes_per_token(shape, routed=None):
    """routed experts (top_k, or the mean kept by top-p) + the shared one +
    fp32 router + bias + bf16 x + fp32 y (9 experts: 197,432,320 B for the
    GLM layer)."""
    E, H = shape.n_experts, shape.hidden
    r = shape.top_k if routed is None else routed
    return int(round((r + shape.n_shared) * shape.expert_bytes + E * H * 4 + E * 4 + H * 2 + H * 4))


DECODE_SOURCES = ("decode.cu", "decode.h", "common.cuh", "async.cuh", "forward.cu")


def kernel_source_hash():
    """Hash of the sources of the one-token decode kernel (the kernel the
    roofline's traffic figure belongs to)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "int4_routed_expert_noaux_b200", "csrc")
    for fn in DECODE_SOURCES:
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
            "top_p": getattr(args, "top_p", 1.0) if getattr(args, "top_p", 1.0) < 1.0 else None,
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
    if args.mode == "timeline":
        run_timeline(args, shape)
        return
    if args.mode != "layer":
        run_mode(args, shape)
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
        if args.top_p < 1.0:
            views[-1].set_top_p(args.top_p)
    torch.cuda.synchronize()

    n = args.tokens
    x_bits = synth.tokens(shape, 1000 * rank, 0, n)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    y = torch.empty((n, shape.hidden), dtype=torch.float32, device="cuda")
    idx = torch.empty((n, shape.top_k), dtype=torch.int32, device="cuda")
    ws = moe.alloc_workspace(cfg, 1)
    stream = torch.cuda.Stream()

    def step(s):
        for t in range(n):
            views[t % copies].forward(x[t:t + 1], y[t:t + 1], ws, idx=idx[t:t + 1], stream=s)

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
        ms = max_over_ranks(ms, dist)
        dist.barrier()
    ms_step = ms / args.steps
    value = job_rate(n * args.steps, world, ms)

    # e2e: host buffers, per-token pinned H2D of x and D2H of y in the timed
    # region.  The copies run on their own streams, double-buffered: token
    # t + 1's input goes up while token t computes, and token t's output
    # comes down while token t + 1 computes.
    x_host = torch.from_numpy(x_bits.view(np.int16)).pin_memory()
    y_host = torch.empty((n, shape.hidden), dtype=torch.float32).pin_memory()
    xd = [torch.empty((1, shape.hidden), dtype=torch.int16, device="cuda") for _ in range(2)]
    yd = [torch.empty((1, shape.hidden), dtype=torch.float32, device="cuda") for _ in range(2)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_k = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step():
        for t in range(n):
            b = t & 1
            up.wait_event(ev_k[b])            # x buffer b: token t - 2 has computed
            with torch.cuda.stream(up):
                xd[b].copy_(x_host[t:t + 1], non_blocking=True)
                ev_in[b].record(up)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])      # y buffer b: token t - 2 is down
            views[t % copies].forward(xd[b], yd[b], ws, stream=stream)
            ev_k[b].record(stream)
            down.wait_event(ev_k[b])
            with torch.cuda.stream(down):
                y_host[t:t + 1].copy_(yd[b], non_blocking=True)
                ev_out[b].record(down)
        stream.wait_event(ev_out[(n - 1) & 1])  # the step ends with its last output on the host

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
        e2e_ms = max_over_ranks(e2e_ms, dist)
    e2e_value = job_rate(n * e2e_steps, world, e2e_ms)
    if not np.all(np.isfinite(y_host.numpy())):
        raise RuntimeError("non-finite outputs")

    peak, peak_kind = peaks()
    # experts read per token: top_k, or those adaptive top-p keeps
    kept = float((idx >= 0).sum(dim=1).float().mean().item())
    bytes_tok = algorithmic_bytes_per_token(shape, kept)
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
            "routed_experts_per_token": kept,
            "clocks": clk, "graph": graph is not None or not args.no_graph,
            "hbm_gbs": achieved,
        }
        print(json.dumps(line), flush=True)


def launches_per_forward():
    return 1


def launches_per_verify_call(T, shape):
    """Kernels of one T-token moe_layer_forward: router, selection, x groups,
    expert lists, gate/up, h groups, down, combine; plus row scales, packing
    and the tensor-core kernel for both projections when 16 or more tokens
    can share an expert (the tensor-core path's shapes: H, I multiples of 512)."""
    tc = T >= 16 and shape.hidden % 512 == 0 and shape.inter % 512 == 0
    return 8 + (6 if tc else 0)


def max_over_ranks(value, dist=None, device="cuda"):
    """The largest value over all ranks (every rank gets it): a multi-GPU
    time is the slowest rank's."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank, world, ms):
    """Whole-job throughput: units of all ranks over the slowest rank's time."""
    return units_per_rank * world / (ms / 1000.0)


# ---------------------------------------------------------------------------
# other modes: one JSON line per configuration, same keys where they apply

def _timed(stream, fn, steps, warmup):
    import torch
    with torch.cuda.stream(stream):
        for _ in range(max(3, warmup)):
            fn()
    stream.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(steps):
            fn()
        ev1.record(stream)
    stream.synchronize()
    return ev0.elapsed_time(ev1)


def _graph(stream, fn):
    import torch
    with torch.cuda.stream(stream):
        fn()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    stream.synchronize()
    return g


def _line(args, shape, extra):
    base = {"metric": METRIC, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": max(3, args.warmup), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int4xf32", "data": "synthetic", "mode": args.mode}
    base.update(extra)
    print(json.dumps(base), flush=True)


# Share of the host's free memory the streamed store may pin; the rest stays
# with the operating system, the CUDA driver and this process.
STREAM_HOST_FRACTION = 0.75


def host_free_bytes():
    """Free host memory: psutil's available figure, bounded by the cgroup's
    remaining limit where there is one."""
    import psutil
    free = psutil.virtual_memory().available
    for lim_path, use_path in (("/sys/fs/cgroup/memory.max", "/sys/fs/cgroup/memory.current"),
                               ("/sys/fs/cgroup/memory/memory.limit_in_bytes",
                                "/sys/fs/cgroup/memory/memory.usage_in_bytes")):
        try:
            lim = int(open(lim_path).read().strip())
            use = int(open(use_path).read().strip())
        except (OSError, ValueError):
            continue
        free = min(free, max(0, lim - use))
    return free


class HostStore:
    """Routed experts of L layers in page-locked host memory (numpy buffers
    registered with cudaHostRegister, so that no allocator rounds them up),
    filled by the device generator and copied back, laid out as
    synth.layers.expert_offsets per expert."""

    def __init__(self, shape, n_layers):
        import torch
        from synth.layers import DeviceLayer, expert_offsets
        E, B = shape.n_experts, shape.expert_bytes
        offs = expert_offsets(shape)
        self.layer_bytes = E * B
        self.bufs, self.experts = [], []
        cudart = torch.cuda.cudart()
        for l in range(n_layers):
            raw = np.empty(self.layer_bytes + 4096, dtype=np.uint8)
            base = (raw.ctypes.data + 4095) // 4096 * 4096
            view = raw[base - raw.ctypes.data: base - raw.ctypes.data + self.layer_bytes]
            rc = int(cudart.cudaHostRegister(base, self.layer_bytes, 0))
            if rc != 0:
                self.close()
                raise RuntimeError(f"cudaHostRegister failed ({rc}) at layer {l}")
            self.bufs.append((raw, base, view))
            dl = DeviceLayer(shape, 0, l)
            torch.from_numpy(view).copy_(dl.slab[: self.layer_bytes])
            del dl
            self.experts.append([{k: base + e * B + o for k, o in offs.items()}
                                 for e in range(E)])
        torch.cuda.synchronize()

    def close(self):
        import torch
        cudart = torch.cuda.cudart()
        for raw, base, view in self.bufs:
            cudart.cudaHostUnregister(base)
        self.bufs = []


def hot_set(counts, n):
    """The n most used experts of a usage log (ties to the lower id), ascending."""
    order = np.lexsort((np.arange(len(counts)), -np.asarray(counts, dtype=np.int64)))
    return np.sort(order[:n])


def run_stream(args, shape, cfg, stream):
    """Host-streamed experts: an LRU cache per layer in HBM over a pinned host
    store of as many layers as STREAM_HOST_FRACTION of the free host memory
    holds.  Per cache size: the Zipf trace with plain LRU, the same trace with
    the hot-store (experts pinned at start-up from the usage log of an earlier
    session of the same popularity), and, with --stream-router, ids from the
    device router of each layer read back to the host before the acquire."""
    import torch
    import int4_routed_expert_noaux_b200 as moe
    import synth
    from synth.layers import DeviceLayer
    E, H, k = shape.n_experts, shape.hidden, shape.top_k
    layer_bytes = E * shape.expert_bytes
    free = host_free_bytes()
    L = max(1, min(args.stream_layers, int(free * STREAM_HOST_FRACTION) // layer_bytes))
    t0 = time.time()
    store = HostStore(shape, L)
    fill_s = time.time() - t0
    dls = [DeviceLayer(shape, 0, l, routed=False) for l in range(L)]
    # measured host->device bandwidth of the store (2 GiB copies)
    probe = torch.empty(min(layer_bytes, 2 << 30), dtype=torch.uint8, device="cuda")
    src = torch.from_numpy(store.bufs[0][2][: probe.numel()])
    hb_ms = _timed(stream, lambda: probe.copy_(src, non_blocking=True), 3, 1)
    h2d_gbs = 3 * probe.numel() / (hb_ms / 1000.0) / 1e9
    del probe, src
    Tn = args.stream_tokens
    # tokens [0, Tn) are the earlier session whose usage log the hot-store
    # pins from; tokens [Tn, 2 Tn) are the measured trace
    full = synth.zipf_trace(5, L, E, k, 2 * Tn)
    learn, trace = full[:Tn], np.ascontiguousarray(full[Tn:])
    usage = [np.bincount(learn[:, l].ravel(), minlength=E) for l in range(L)]
    xb = synth.tokens(shape, 0, 0, Tn)
    x = torch.from_numpy(xb.view(np.int16)).cuda()
    ids_dev = torch.from_numpy(trace).cuda()
    w = torch.full((1, k), shape.rsf / k, dtype=torch.float32, device="cuda")
    y = torch.empty((1, H), dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(cfg, 1)
    ridx = torch.empty((1, k), dtype=torch.int32, device="cuda")
    rw = torch.empty((1, k), dtype=torch.float32, device="cuda")
    ids_host = torch.empty((1, k), dtype=torch.int32, pin_memory=True)
    ev_ids = torch.cuda.Event()
    caps = [int(v) for v in args.stream_caps.split(",")]
    router_caps = [int(v) for v in args.stream_router_caps.split(",") if v]

    def pins_for(cap):
        """Experts to pin per layer: the hottest n of the usage log, n chosen
        among five candidates by replaying the earlier session."""
        best_n, best_h = 0, -1
        for n in sorted({0, (cap - k) // 4, (cap - k) // 2, 3 * (cap - k) // 4, cap - k}):
            pinned = np.stack([hot_set(usage[l], n) for l in range(L)])
            h, _ = moe.lru_replay(learn, E, cap, pinned=pinned if n else None)
            if int(h.sum()) > best_h:
                best_n, best_h = n, int(h.sum())
        return best_n, [hot_set(usage[l], best_n) for l in range(L)]

    def one(cap, arm):
        try:
            cache = moe.Cache(cfg, store.experts, cap)
        except moe.MoeError as e:
            print(json.dumps({"mode": "stream", "cache_slots_per_layer": cap,
                              "skipped": str(e)}), flush=True)
            return
        views = [cache.layer(l, dls[l].w_router, dls[l].bias, dls[l].shared) for l in range(L)]
        n_pin = 0
        if arm == "hot-store":
            n_pin, pins = pins_for(cap)
            for l in range(L):
                if n_pin:
                    cache.pin(l, pins[l], stream=stream)
        cache.sync()
        torch.cuda.synchronize()
        before = [cache.stats(l) for l in range(L)]
        launches = 0
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for t in range(Tn):
                for l in range(L):
                    # the resident experts first, each copied one once its copy
                    # is done (moe_cache_expert_ffn)
                    if arm == "router":
                        views[l].route(x[t:t + 1], ridx, rw, ws, stream=stream)
                        ids_host.copy_(ridx, non_blocking=True)
                        ev_ids.record(stream)
                        ev_ids.synchronize()
                        nm = cache.expert_ffn(l, x[t:t + 1], ridx, rw, ids_host.numpy()[0], y, ws,
                                              stream=stream)
                        launches += 2
                    else:
                        nm = cache.expert_ffn(l, x[t:t + 1], ids_dev[t, l:l + 1], w, trace[t, l],
                                              y, ws, stream=stream)
                    cache.release(l, stream=stream)
                    # per part call: x groups, lists, gate/up, h groups, down;
                    # one combine; one pointer-table update when something missed
                    launches += 5 * (1 + nm) + 1 + (1 if nm else 0)
            ev1.record(stream)
        stream.synchronize()
        cache.sync()
        ms = ev0.elapsed_time(ev1)
        moe.ws_check(ws, stream)
        hits = misses = moved = 0
        for l in range(L):
            h, m, b = cache.stats(l)
            hits += h - before[l][0]
            misses += m - before[l][1]
            moved += b - before[l][2]
        link = moved / (ms / 1000.0) / 1e9
        routing = {"lru": "Zipf trace, plain LRU",
                   "hot-store": f"Zipf trace, {n_pin} experts per layer pinned from the usage "
                                "log of an earlier session, LRU on the other slots",
                   "router": "device router of each layer (ids read back to the host), "
                             "plain LRU"}[arm]
        _line(args, shape, {
            "value": Tn / (ms / 1000.0), "ms_per_step": ms,
            "config": {"workload": f"{L} GLM-5.2-shaped MoE layers in pinned host memory "
                                   f"({L * layer_bytes / 1e9:.1f} GB), per-layer cache in HBM",
                       "layers": L, "host_free_bytes": free,
                       "host_fraction_pinned": STREAM_HOST_FRACTION,
                       "host_fill_s": round(fill_s, 1), "cache_slots_per_layer": cap,
                       "policy": arm, "pinned_per_layer": n_pin, "tokens": Tn,
                       "routing": routing, "hit_rate": hits / max(1, hits + misses),
                       "compute": "resident experts first, each copied expert after its own "
                                  "copy event (moe_cache_expert_ffn)",
                       "expert_bytes": shape.expert_bytes},
            "roofline": {"bound": "h2d", "achieved": link, "peak": h2d_gbs, "unit": "GB/s",
                         "frac": link / h2d_gbs, "traffic": moved, "peak_source":
                         "measured pinned host->device copy, same run",
                         "kernel": "expert loads (cudaMemcpyAsync, side stream)"},
            "gpu_launches": launches})
        cache.close()

    try:
        for cap in caps:
            one(cap, "lru")
            if cap - k >= 1:
                one(cap, "hot-store")
        for cap in router_caps:
            one(cap, "router")
    finally:
        store.close()


# Probe points of the one-token kernel's -DMOE_TRACE build (TRACE_AT indices).
TIMELINE_PHASES = {0: "entry", 1: "router fill issued", 2: "router rows landed",
                   15: "router dot products done", 3: "records published",
                   4: "all records seen", 17: "group scores", 18: "groups ranked",
                   19: "candidate lists sorted", 12: "producer has pick 0",
                   6: "first routed gate/up fill issued", 20: "all picks found",
                   5: "selection published", 22: "last shared gate/up item finalised",
                   21: "shared h group published", 7: "first down fill issued",
                   11: "last fill issued", 10: "exit"}


def run_timeline(args, shape):
    """Per-phase times of the one-token kernel: the probe build of the same
    sources records clock64 at fixed points of every CTA (and globaltimer at
    entry); CUDA-graph replay of 64 tokens over 8 layer copies; medians over
    CTAs, then over replays."""
    import torch
    import int4_routed_expert_noaux_b200 as moe
    from int4_routed_expert_noaux_b200 import build as B
    import synth
    from synth.layers import DeviceLayer
    moe.LIB_PATH = B.build(trace=True)
    L = moe.lib()
    L.moe_debug_set_trace.argtypes = [ctypes.c_void_p]
    L.moe_debug_set_trace.restype = None
    torch.cuda.set_device(0)
    cfg = moe.Config.from_shape(shape)
    copies = max(1, args.copies)
    dls = [DeviceLayer(shape, 0, c) for c in range(copies)]
    views = [moe.Layer(cfg, d.w_router, d.bias, d.routed, d.shared) for d in dls]
    n = 64
    x = torch.from_numpy(synth.tokens(shape, 0, 0, n).view(np.int16)).cuda()
    y = torch.empty((n, shape.hidden), dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(cfg, 1)
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    tr = torch.zeros(nsm * 128 + 128, dtype=torch.int64, device="cuda")
    L.moe_debug_set_trace(ctypes.c_void_p(tr.data_ptr()))
    stream = torch.cuda.Stream()

    def step():
        for t in range(n):
            views[t % copies].forward(x[t:t + 1], y[t:t + 1], ws, stream=stream)
    g = _graph(stream, step)
    clocks = Clocks(0)
    f_ghz = []
    acc = {i: [] for i in TIMELINE_PHASES}
    per_call = []
    for rep in range(8):
        tr.zero_()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        stream.synchronize()
        per_call.append(e0.elapsed_time(e1) * 1000.0 / n)
        if rep < 2:
            continue
        raw = tr.cpu().numpy()[: nsm * 128].reshape(nsm, 128).astype(np.float64)
        gt0, c0 = raw[:, 127], raw[:, 96]  # each CTA's entry: globaltimer ns, clock64
        f_ghz.append(args.timeline_sm_mhz / 1000.0)
        t0 = gt0.min()
        for i in TIMELINE_PHASES:
            v = raw[:, 96 + i]
            m = v != 0
            if m.any():
                acc[i].append(np.median((gt0[m] + (v[m] - c0[m]) / f_ghz[-1] - t0) / 1000.0))
    clk = clocks.stop()
    moe.ws_check(ws, stream)
    L.moe_debug_set_trace(None)
    phases = {TIMELINE_PHASES[i]: round(float(np.median(v)), 2)
              for i, v in sorted(acc.items(), key=lambda kv: np.median(kv[1]) if kv[1] else 1e9)
              if v}
    print(json.dumps({"mode": "timeline", "workload": "one GLM-5.2-shaped layer per token, "
                      f"{copies} rotating layer copies, CUDA-graph replay of {n} tokens",
                      "library": "probe build (-DMOE_TRACE) of the same sources",
                      "us_per_token_probe_build": round(float(np.median(per_call[2:])), 2),
                      "phases_us_median_over_ctas": phases,
                      "clock_mhz_assumed": args.timeline_sm_mhz, "clocks": clk}), flush=True)


def run_mode(args, shape):
    import torch
    import int4_routed_expert_noaux_b200 as moe
    import synth
    from synth.layers import DeviceLayer
    torch.cuda.set_device(0)
    cfg = moe.Config.from_shape(shape)
    peak, peak_kind = peaks()
    stream = torch.cuda.Stream()
    E, H = shape.n_experts, shape.hidden
    fixed = E * H * 4 + E * 4

    if args.mode == "verify":
        copies = max(1, args.copies)
        dls = [DeviceLayer(shape, 0, c) for c in range(copies)]
        views = [moe.Layer(cfg, d.w_router, d.bias, d.routed, d.shared) for d in dls]
        for T in [int(v) for v in args.verify_T.split(",")]:
            calls = max(copies, args.tokens // T)
            if args.correlated:
                xb = np.concatenate([synth.correlated_tokens(shape, 7 + c, T) for c in range(calls)])
            else:
                xb = synth.tokens(shape, 0, 0, calls * T)
            x = torch.from_numpy(xb.view(np.int16)).cuda()
            y = torch.empty((calls * T, H), dtype=torch.float32, device="cuda")
            idx = torch.empty((calls * T, shape.top_k), dtype=torch.int32, device="cuda")
            ws = moe.alloc_workspace(cfg, T)

            def step():
                for c in range(calls):
                    sl = slice(c * T, (c + 1) * T)
                    views[c % copies].forward(x[sl], y[sl], ws, idx=idx[sl], stream=stream)
            g = _graph(stream, step)
            ms = _timed(stream, g.replay, args.steps, args.warmup)
            moe.ws_check(ws, stream)
            ids = idx.cpu().numpy().reshape(calls, T, shape.top_k)
            uniq = [len(np.unique(ids[c])) for c in range(calls)]
            byts = sum(fixed + (u + shape.n_shared) * shape.expert_bytes + T * (H * 2 + H * 4)
                       for u in uniq)
            call_us = ms * 1000.0 / (args.steps * calls)
            achieved = byts / calls / (call_us * 1e-6) / 1e9
            _line(args, shape, {
                "value": calls * T * args.steps / (ms / 1000.0), "ms_per_step": ms / args.steps,
                "config": {"workload": "GLM-5.2-shaped MoE layer, batched verify calls",
                           "T": T, "calls_per_step": calls, "correlated": args.correlated,
                           "layer_copies": copies, "mean_distinct_routed_experts": float(np.mean(uniq))},
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                             "frac": achieved / peak, "traffic": None, "peak_source": peak_kind,
                             "kernel": "moe_layer_forward (T tokens)",
                             "algorithmic_bytes_per_launch": byts / calls, "launch_us": call_us},
                "gpu_launches": calls * args.steps * launches_per_verify_call(T, shape)})
        return

    if args.mode == "stack":
        L = args.stack_layers
        dls = [DeviceLayer(shape, 0, l) for l in range(L)]
        views = [moe.Layer(cfg, d.w_router, d.bias, d.routed, d.shared) for d in dls]
        n = max(1, min(args.tokens, 200))
        xb = synth.tokens(shape, 0, 0, n)
        x0 = torch.from_numpy(synth.bf16_to_f32(xb)).cuda()
        xo = torch.empty_like(x0)
        tmp = torch.empty((H,), dtype=torch.float32, device="cuda")
        ws = moe.alloc_workspace(cfg, 1)

        def step():
            for t in range(n):
                moe.stack_forward(views, x0[t], xo[t], tmp, ws, stream=stream)
        g = _graph(stream, step)
        ms = _timed(stream, g.replay, args.steps, args.warmup)
        moe.ws_check(ws, stream)
        if not torch.isfinite(xo).all():
            raise RuntimeError("non-finite stack outputs")
        byts = L * algorithmic_bytes_per_token(shape)
        tok_us = ms * 1000.0 / (args.steps * n)
        achieved = byts / (tok_us * 1e-6) / 1e9
        _line(args, shape, {
            "value": n * args.steps / (ms / 1000.0), "ms_per_step": ms / args.steps,
            "config": {"workload": f"{L} GLM-5.2-shaped MoE layers, one token through all "
                                   "(pre-norm residual stream), all experts resident",
                       "layers": L, "tokens_per_step": n,
                       "hbm_weight_bytes": L * ((E + shape.n_shared) * shape.expert_bytes + fixed)},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None, "peak_source": peak_kind,
                         "kernel": "moe_stack_forward (per token)",
                         "algorithmic_bytes_per_launch": byts, "launch_us": tok_us},
            "gpu_launches": n * args.steps * L})
        return

    if args.mode == "stream":
        run_stream(args, shape, cfg, stream)
        return
        return


if __name__ == "__main__":
    main()
