"""Benchmark of the routed MoE half on B200.

Workload (default): the 24-layer gpt-oss-20b-shaped stack (hidden 2880,
moe_inter 2880, 32 MXFP4 experts, top-4 with an FP32 router bias, clamped
SwiGLU; ~10 GB of expert weights, far beyond L2) at M = 16 tokens per layer,
independent seeded x per layer.  One step = one routed-half forward through
all 24 layers (24 x ts_moe_forward = 24 layer-kernel launches), replayed as
a CUDA graph.

Prints one JSON line: tokens/s through the stack (whole job over all ranks),
achieved HBM GB/s on the weight bytes the routing touched, the dominant
kernel's roofline fraction, an end-to-end number through host buffers, and the
FP64 oracle timed on the host cores as a CPU baseline.

--impl reference runs the oracle as the reference arm (CPU, bounded sample).
Multi-GPU: one process per GPU (torchrun); each rank runs an independent
replica on its own micro-batches (weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_moe_routed_router_b200 import synth  # noqa: E402

METRIC = "routed-MoE tokens/s and HBM GB/s vs ~8 TB/s roofline at M=1 and M=16"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--M", type=int, default=16)
    ap.add_argument("--cfg", type=int, default=5)
    ap.add_argument("--layers", type=int, default=0, help="override the number of layers (0 = the workload's)")
    ap.add_argument("--no-sweep", action="store_true", help="skip timing M in {1,2,4,8,16} (key m_sweep) and the one-launch M = 64 prefill (key prefill)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    return ap.parse_args()


def dist_setup(n):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.f = None

    def start(self):
        try:
            self.f = tempfile.TemporaryFile(mode="w+")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.idx)], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.seek(0)
        rows = [l.strip().split(",") for l in self.f.read().splitlines() if l.strip()]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except Exception:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


KERNEL_SOURCES = os.path.join(ROOT, "quantized_moe_routed_router_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "layer_kernel_traffic.json")
PREFILL_M = 64  # the prefill point of the sweep: one 64-token launch per layer


def kernel_sources_sha256() -> str:
    """Hash of the CUDA sources the layer kernel is built from (csrc/*.cu, *.cuh)."""
    import hashlib
    h = hashlib.sha256()
    for name in sorted(os.listdir(KERNEL_SOURCES)):
        if name.endswith((".cu", ".cuh")):
            h.update(name.encode())
            h.update(open(os.path.join(KERNEL_SOURCES, name), "rb").read())
    return h.hexdigest()


def measured_traffic(algo_bytes_per_launch: float):
    """DRAM bytes (read + write) per layer-kernel launch from the committed ncu
    capture, scaled from the captured launch to this run's launches by their
    algorithmic bytes; None when the kernel sources changed since the capture."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    d = json.load(open(TRAFFIC_FILE))
    if d.get("sources_sha256") != kernel_sources_sha256():
        return None
    return round(d["dram_bytes_per_launch"] * algo_bytes_per_launch / d["algorithmic_bytes_per_launch"])


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ----------------------------------------------------------------------------- oracle CPU baseline
def cpu_baseline(shape, layers_host, xs_host, M, budget_s):
    """The FP64 oracle as it stands, on the host cores, over whole layers of the
    same workload until `budget_s` of work is done; scaled to the stack."""
    from oracle import oracle as O
    O.build()
    th = O.nthreads()
    orcs = [O.Oracle(shape, Lh) for Lh in layers_host]
    t0 = time.perf_counter()
    done = 0
    while True:  # cycle over the host layers until the budget is spent
        l = done % len(orcs)
        orcs[l].forward(xs_host[l][:M], nthreads=th)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    per_layer = dt / done
    tps = M / (per_layer * shape.num_layers)
    return {"value": tps, "unit": "tokens/s", "cores": th, "kind": "oracle",
            "sample": f"{done} layer passes at M={M} over {len(orcs)} of the {shape.num_layers} layers "
                      f"(FP64 C++ oracle, {th} threads), {dt:.1f} s, scaled to the {shape.num_layers}-layer stack"}


L2_BYTES = 126e6


def workload_config(shape, NL, M, world):
    """The `config` keys both arms report for the same workload, including how
    the timed steps stand to the 126 MB L2 (no flush: the weights a step
    streams are many times larger than L2 when the stack is)."""
    stack = NL * (shape.num_experts * shape.expert_bytes() + shape.router_bytes() + shape.shared_bytes())
    if stack >= 4 * L2_BYTES:
        l2 = (f"inputs larger than L2: the {NL}-layer stack holds {stack / 1e9:.2f} GB of weights, "
              f"{stack / L2_BYTES:.0f}x the 126 MB L2; no flush between steps")
    else:
        l2 = (f"weights ({stack / 1e6:.0f} MB) within 4x the 126 MB L2 and not flushed: "
              "steps may hit L2, an upper bound")
    return {"workload": f"{shape.name}, {NL} layers x M={M} tokens (independent x per layer)",
            "hidden": shape.hidden, "moe_inter": shape.moe_inter, "experts": shape.num_experts,
            "top_k": shape.top_k, "M": M, "layers": NL, "parallelism": f"replicas x{world}", "l2": l2}


def host_layers_for_oracle(shape, layers, n):
    return [layers[l].host_numpy() for l in range(n)]


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local):
    from quantized_moe_routed_router_b200 import binding, build
    build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    shape = synth.CONFIGS[args.cfg]
    if args.layers:
        shape = shape.replace(num_layers=args.layers)
    M = args.M
    shape = shape.replace(max_tokens=max(M, PREFILL_M if (not args.no_sweep) else M))
    NL, H = shape.num_layers, shape.hidden
    layers = [synth.make_layer(shape, l, device=dev) for l in range(NL)]
    moe = binding.MoE(shape, layers)
    info = moe.info()
    # keep two layers' blobs on the host for the CPU baseline, free the rest
    need_cpu = rank == 0 and not args.no_cpu_baseline
    lay_host = host_layers_for_oracle(shape, layers, min(NL, 3)) if need_cpu else None
    del layers
    torch.cuda.empty_cache()

    master = 1000 + rank  # each replica draws its own micro-batches
    Mr = max(16, M)
    xs = torch.stack([synth.make_x(shape, l, Mr, device=dev, master=master) for l in range(NL)])  # [NL,Mr,H]
    rs = torch.stack([synth.make_x(shape, l, Mr, device=dev, master=master, tensor=synth.T_RESID) for l in range(NL)])
    stream = torch.cuda.Stream(device=dev)

    LT = info.launch_tokens  # tokens per layer-kernel launch

    def touched_bytes(Mx, src=xs):
        """Weight bytes one step streams: per layer, per launch of up to LT
        tokens, each touched expert once per 16 routes it receives (its
        entries) + the router (+ the shared expert once per 16 tokens)."""
        idx = torch.empty(Mx, shape.top_k, dtype=torch.int32, device=dev)
        w = torch.empty(Mx, shape.top_k, device=dev)
        n_entries, n_touched = [], []
        with torch.cuda.stream(stream):
            for l in range(NL):
                moe.route(l, src[l, :Mx], idx, w, stream=stream)
                stream.synchronize()
                ih = idx.cpu().numpy()
                ent, tch = [], []
                for c in range(0, Mx, LT):
                    cnt = np.bincount(ih[c:c + LT].ravel(), minlength=shape.num_experts)
                    ent.append(int(((cnt + 15) // 16).sum()))
                    tch.append(int((cnt > 0).sum()))
                n_entries.append(ent)
                n_touched.append(tch)
        per_layer = [sum(n * info.expert_bytes + info.router_bytes +
                         -(-min(LT, Mx - i * LT) // 16) * info.shared_bytes for i, n in enumerate(nl))
                     for nl in n_entries]
        return sum(per_layer), [n for nl in n_touched for n in nl], per_layer

    def make_graph(Mx, out, src=xs):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for l in range(NL):  # eager warm-up of every layer once
                moe.forward(l, src[l, :Mx], out[l, :Mx], None, stream=stream)
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for l in range(NL):
                    moe.forward(l, src[l, :Mx], out[l, :Mx], None, stream=stream)
        return g

    def time_graph(g, steps, warmup, sampler=None):
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if sampler:
            sampler.start()
            time.sleep(0.3)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(steps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        clocks = sampler.stop() if sampler else None
        barrier(world)
        ms = e0.elapsed_time(e1)
        return max_over_ranks(ms, world) / steps, clocks

    out = rs.clone()
    g = make_graph(M, out)
    algo_bytes, n_touched, layer_bytes = touched_bytes(M)
    sampler = ClockSampler(local)
    ms_step, clocks = time_graph(g, args.steps, args.warmup, sampler)
    moe.device_status(stream)
    tok_s = world * M / (ms_step * 1e-3)
    gbs = algo_bytes / (ms_step * 1e-3) / 1e9

    # the layer kernel (the only kernel of a forward): CUDA events on the launching stream around each launch
    prof_steps = max(3, min(20, args.steps // 10))
    ev_all = []
    with torch.cuda.stream(stream):
        for _ in range(2):  # warm
            for l in range(NL):
                moe.forward(l, xs[l, :M], out[l, :M], None, stream=stream)
        stream.synchronize()
        for s in range(prof_steps):
            for l in range(NL):
                evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
                moe.set_timing_events(evs)
                moe.forward(l, xs[l, :M], out[l, :M], None, stream=stream)
                ev_all.append((l, evs))
        moe.set_timing_events(None)
        stream.synchronize()
    t_layer = [e[0].elapsed_time(e[1]) for _, e in ev_all]
    iso_ms = statistics.mean(t_layer)
    iso_bytes = statistics.mean(layer_bytes[l] for l, _ in ev_all)
    peak, peak_kind = measured_peaks()
    # The headline kernel time: the graph's timed region holds nothing but the
    # layer-kernel launches (PDL-chained), so the events around it divided by
    # the launches give the kernel's average duration inside the step.
    launches_per_step = NL * ((M + LT - 1) // LT)
    avg_ms = ms_step / launches_per_step
    bytes_per_launch = algo_bytes / launches_per_step
    achieved = bytes_per_launch / (avg_ms * 1e-3) / 1e9
    fmt_name = {synth.FMT_Q8_0: "Q8_0", synth.FMT_MXFP4: "MXFP4", synth.FMT_INT4_AFFINE: "INT4-affine"}[shape.expert_fmt]
    instance = "prefill" if M > 16 else "decode"
    roofline = {"bound": "hbm", "kernel": f"layer_kernel<{fmt_name}, {instance}> (route + gate/up + down + combine)",
                "achieved": round(achieved, 1), "peak": peak, "peak_kind": f"{peak_kind} HBM copy bandwidth",
                "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": measured_traffic(bytes_per_launch),
                "avg_launch_us": round(avg_ms * 1e3, 2), "algorithmic_bytes_per_launch": int(bytes_per_launch),
                "timing": f"CUDA events around the {args.steps} timed graph replays on the launching stream, "
                          f"/ {launches_per_step} launches per step",
                "avg_launch_us_isolated": round(iso_ms * 1e3, 2),
                "frac_isolated": round(iso_bytes / (iso_ms * 1e-3) / 1e9 / peak, 4)}

    # end to end through host buffers: pinned H2D of x and resid, D2H of the updated resid
    x_h = xs[:, :M].cpu().pin_memory()
    r_h = rs[:, :M].cpu().pin_memory()
    o_h = torch.empty_like(r_h).pin_memory()
    xd = torch.empty_like(xs[:, :M])
    rd = torch.empty_like(rs[:, :M])
    e2e_steps = max(3, args.steps // 4)

    def e2e_step():
        xd.copy_(x_h, non_blocking=True)
        rd.copy_(r_h, non_blocking=True)
        for l in range(NL):
            moe.forward(l, xd[l], rd[l], None, stream=stream)
        o_h.copy_(rd, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(2):
            e2e_step()
        stream.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        stream.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    h2d = x_h.numel() * 2 + r_h.numel() * 2
    d2h = o_h.numel() * 2

    sweep = prefill = None
    if (not args.no_sweep):
        sweep = {}
        for Ms in (1, 2, 4, 8, 16):
            o2 = rs.clone()
            g2 = make_graph(Ms, o2)
            b2, nt2, _ = touched_bytes(Ms)
            ms2, _ = time_graph(g2, max(20, args.steps // 2), args.warmup)
            sweep[str(Ms)] = {"tokens_per_s": round(world * Ms / (ms2 * 1e-3), 1), "ms_per_step": round(ms2, 4),
                              "GB_per_s": round(b2 / (ms2 * 1e-3) / 1e9, 1),
                              "frac_of_8TBs": round(b2 / (ms2 * 1e-3) / 8e12, 4),
                              "touched_experts_per_layer": round(sum(nt2) / len(nt2), 2)}
            del g2
        # prefill: M = 64 tokens per layer in one launch (each touched expert read once per 16 routes)
        xp = torch.stack([synth.make_x(shape, l, PREFILL_M, device=dev, master=master) for l in range(NL)])
        op = torch.stack([synth.make_x(shape, l, PREFILL_M, device=dev, master=master, tensor=synth.T_RESID)
                          for l in range(NL)])
        gp = make_graph(PREFILL_M, op, xp)
        bp, ntp, _ = touched_bytes(PREFILL_M, xp)
        msp, _ = time_graph(gp, max(20, args.steps // 2), args.warmup)
        prefill = {"M": PREFILL_M, "launches_per_layer": (PREFILL_M + LT - 1) // LT,
                   "tokens_per_s": round(world * PREFILL_M / (msp * 1e-3), 1), "ms_per_step": round(msp, 4),
                   "streamed_GB_per_step": round(bp / 1e9, 3),
                   "streamed_GB_per_s": round(bp / (msp * 1e-3) / 1e9, 1),
                   "touched_experts_per_launch": round(sum(ntp) / len(ntp), 2)}
        del gp, xp, op

    cpu = None
    if need_cpu:
        xs_host = [synth.bf16_bits_np(xs[l]) for l in range(min(NL, 3))]
        cpu = cpu_baseline(shape, lay_host, xs_host, M, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(tok_s, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16",
            "dtype_detail": ("mxfp4" if shape.expert_fmt else "q8_0") + " weights dequantised exactly to f16, "
                            "f16 MMA with f32 accumulation, f32 routing and epilogue",
            "data": "synthetic (seeded N(0,0.02) weights encoded to the block formats; N(0,1) bf16 x)",
            "config": workload_config(shape, NL, M, world),
            "launch": f"CUDA graph of {NL} ts_moe_forward calls per step ({NL * ((M + 15) // 16)} layer-kernel launches)",
            "GB_per_s": round(gbs, 1), "frac_of_8TBs": round(gbs / 8000.0, 4),
            "frac_of_measured_hbm": round(gbs / peak, 4),
            "algorithmic_bytes_per_step": int(algo_bytes),
            "touched_experts_per_layer": round(sum(n_touched) / len(n_touched), 2),
            "roofline": roofline,
            "e2e": {"value": round(world * M / (e2e_ms * 1e-3), 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
            "gpu_launches": args.steps * NL * ((M + LT - 1) // LT),
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        if sweep:
            line["m_sweep"] = sweep
            line["prefill"] = prefill
        print(json.dumps(line), flush=True)
    moe.close()


# ----------------------------------------------------------------------------- reference arm (the oracle)
def run_reference(args, rank, world, local):
    if rank != 0:
        return
    from oracle import oracle as O
    O.build()
    shape = synth.CONFIGS[args.cfg]
    if args.layers:
        shape = shape.replace(num_layers=args.layers)
    M = args.M
    th = O.nthreads()
    layer = synth.make_layer(shape, 0, device="cpu").host_numpy()
    x = synth.bf16_bits_np(synth.make_x(shape, 0, M, master=1000))
    orc = O.Oracle(shape, layer)
    # Each step is a bounded sample of the workload: one layer of the stack at
    # M tokens (every layer has the same shape); the rate is scaled to the stack.
    for _ in range(args.warmup):
        orc.forward(x, nthreads=th)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.forward(x, nthreads=th)
    ms_step = (time.perf_counter() - t0) / args.steps * 1e3
    tps = M / (ms_step * 1e-3 * shape.num_layers)
    line = {"impl": "reference", "metric": METRIC, "value": round(tps, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "step": f"one layer of the {shape.num_layers}-layer stack (a bounded sample); value scaled to the stack",
            "config": workload_config(shape, shape.num_layers, M, world),
            "cpu_baseline": {"value": round(tps, 3), "unit": "tokens/s", "cores": th, "kind": "oracle",
                             "sample": f"{args.steps} timed steps, each one layer of the {shape.num_layers}-layer "
                                       f"stack at M={M} on {th} threads, tokens/s scaled to the stack"},
            "e2e": {"value": round(tps, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world, local)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
