#!/usr/bin/env python
"""Benchmark of the large-chunk TTT layer on B200: update + apply tokens/s per
layer on the 700-frame scene (961,800 image tokens in one bidirectional chunk,
4 heads x d=256, SwiGLU hidden 512, 16 ray-map target views = 21,984 ray
queries, a 24-layer stack with independent seeded weights per layer).

One step = for each of the 24 layers: ttt_update over all 961,800 tokens,
ttt_apply to the 961,800 image queries and ttt_apply to the 21,984 ray
queries.  value = 961,800 * 24 / step time (tokens/s per layer), summed over
ranks for N > 1 (each rank reconstructs its own scene: weak scaling, no
collective on the data path).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the fp64 CPU oracle (the reference arm of this build)
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from recon_chunk_ttt_b200 import workloads as wl  # noqa: E402

METRIC = "TTT update+apply tokens/s per layer @700 frames"
UNIT = "tokens/s"
GEMM_UNIT = lambda d, h: 2 * d * h  # noqa: E731  flops of one d x h matrix-vector product


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="scene700")
    ap.add_argument("--layers", type=int, default=None)
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-stream", action="store_true")
    ap.add_argument("--ns-steps", type=int, default=0,
                    help="Newton-Schulz steps on the gradient in the timed step (0: off)")
    ap.add_argument("--no-gate-probe", action="store_true",
                    help="skip the gated-output-unit measurement")
    ap.add_argument("--no-shard-probe", action="store_true",
                    help="skip the token-sharded update measurement")
    ap.add_argument("--no-ns-probe", action="store_true",
                    help="skip the separate 5-step Newton-Schulz update measurement")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--only-stream", action="store_true",
                    help="run only the streaming measurement (stream256, one frame per "
                         "ttt_stream_step) and print its JSON object")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def workload_config(w: wl.Workload, layers: int) -> dict:
    return {
        "workload": (f"{w.name}: {w.frames} frames x {w.p} tokens = {w.n_tokens} tokens "
                     f"{'fed one frame per update' if w.name.startswith('stream') else 'in one chunk'}"
                     f", {w.heads} heads x d={w.d}, SwiGLU hidden {w.hidden}, {layers} "
                     f"layers, {w.n_ray} ray queries"),
        "tokens": w.n_tokens, "ray_queries": w.n_ray, "layers": layers, "heads": w.heads,
        "d": w.d, "hidden": w.hidden, "renorm": "row",
        "l2": "inputs larger than L2 (K, V, Q bf16 = %.1f GB)" % (3 * w.n_tokens * w.heads * w.d
                                                                  * 2 / 1e9),
    }


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"ttt_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except OSError:  # no nvidia-smi on this machine
            self.proc = None
            self.f.close()
            os.unlink(self.path)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        under = [s for s in sm if s > 500] or sm
        return {"sm_mhz": statistics.median(under) if under else None,
                "sm_max_mhz": max(mx) if mx else None, "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------- distributed
def dist_setup(args=None):
    """(world size, rank, local rank) from the torchrun environment."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(v: float, world: int, device) -> float:
    """Max of a per-rank value over all ranks (identity for one rank)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(world: int, tokens: int, layers: int, ms: float) -> float:
    """Whole-job tokens/s per layer: every rank processes its own scene of
    `tokens` tokens through `layers` layers in `ms` (the slowest rank's
    time)."""
    return world * tokens * layers / (ms / 1e3)


def kernel_work(d: int, hid: int) -> dict:
    """Algorithmic work per unit (a token-head for the update, a query-head for
    the apply) and the resource that bounds it.  Flops count the GEMMs (a GEMM
    unit is 2 d hid): the update is 6 units (forward 2, backward 1, token
    reduction 3), the apply 3.  Bytes are what the algorithm must move: the
    update reads k, v (bf16) and eta (fp32) once, the apply reads q and writes o
    (bf16); the intermediates (u, dh) are not algorithmic bytes.  Both are dense
    contractions at hundreds of flop per byte, so the tensor pipe bounds them."""
    unit = GEMM_UNIT(d, hid)
    return {"tc_update_fused": {"bound": "tensor", "flops": 6 * unit, "bytes": 2 * d * 2 + 4},
            "tc_apply": {"bound": "tensor", "flops": 3 * unit, "bytes": 2 * d * 2}}


def renorm_bytes(H: int, d: int, hid: int, splits: int) -> float:
    """Bytes one reduce + renorm launch must move: the split partials and W
    read (fp32), W-hat written (fp32) and its bf16 shadow."""
    mat = 3 * H * hid * d
    return (splits + 1) * mat * 4 + mat * 4 + mat * 2


def roofline_entry(flops: float, bytes_: float, ms: float, pk: dict, bound: str) -> dict:
    """Achieved rate of one kernel (all its launches: `flops`, `bytes_` in `ms`)
    against the resource its algorithm is bound by: the bf16 tensor pipe
    (fraction of the sustained GEMM peak, the burst fraction beside it) or HBM
    bandwidth.  A fraction above 1 means the timing or the work count is wrong:
    it is reported as an error with frac = None, never as a rate."""
    if bound == "tensor":
        ach = flops / (ms / 1e3) / 1e12
        peak = pk["bf16_tflops_sustained"]
        ent = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
               "frac": ach / peak, "peak_kind": "bf16_tflops_sustained",
               "burst_frac": ach / pk["bf16_tflops"]}
    else:
        ach = bytes_ / (ms / 1e3) / 1e9
        peak = pk["hbm_gbs"]
        ent = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
               "frac": ach / peak, "peak_kind": "hbm_gbs"}
    if ent["frac"] > 1.0:
        ent["error"] = (f"achieved {ach:.1f} {ent['unit']} is above the measured peak "
                        f"({ent['frac']:.3f}): timing or work count wrong")
        ent["frac"] = None
        ent.pop("burst_frac", None)
    return ent


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(w: wl.Workload, frames: int, seed_layer: int = 0):
    """Time the fp64 oracle's update + apply on `frames` frames of the
    workload (one layer).  Returns (tokens, seconds)."""
    import oracle as O
    x = wl.make_inputs(w, n_tokens=frames * w.p, layer=seed_layer)
    t0 = time.perf_counter()
    if w.name.startswith("stream"):
        # streaming: one update + apply per frame, the state carried over
        O.ttt_stream(x.W1, x.W2, x.W3, x.K, x.V, x.eta, x.Q, w.p, O.RENORM_ROW)
    else:
        Wh = O.ttt_update(x.W1, x.W2, x.W3, x.K, x.V, x.eta, O.RENORM_ROW)
        O.ttt_apply(*Wh, x.Q)
    return frames * w.p, time.perf_counter() - t0


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(w: wl.Workload, seconds: float) -> dict:
    tok, dt = oracle_sample(w, 1)
    frames = max(1, min(w.frames, int(seconds / max(dt, 1e-3))))
    tok, dt = oracle_sample(w, frames)
    return {"value": tok / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": (f"fp64 numpy oracle, one layer of {w.name}: update + image apply on "
                       f"{frames} frames ({tok} tokens, {w.heads} heads) in {dt:.1f} s")}


def run_reference(args, w: wl.Workload, world: int, rank: int):
    if rank != 0:
        return
    layers = args.layers or w.layers
    # size one step at about 5 s of CPU work
    tok, dt = oracle_sample(w, 1)
    frames = max(1, min(w.frames, int(5.0 / max(dt, 1e-3))))
    for _ in range(args.warmup):
        oracle_sample(w, frames)
    times = []
    for _ in range(args.steps):
        tok, dt = oracle_sample(w, frames)
        times.append(dt)
    t = sum(times) / len(times)
    value = tok / t
    what = ("per-frame update + apply (streaming)" if w.name.startswith("stream")
            else "update + image apply")
    sample = (f"fp64 numpy oracle, one layer of {w.name}: {what} on {frames} "
              f"frames ({tok} tokens, {w.heads} heads) per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, layers),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm
def run_ours(args, w: wl.Workload, world: int, rank: int, local: int):
    import torch
    import recon_chunk_ttt_b200 as R
    from recon_chunk_ttt_b200 import build as B

    B.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                device_id=dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    def rank_max(v: float) -> float:
        return max_over_ranks(v, world, dev)

    layers = args.layers or w.layers
    H, d, hid = w.heads, w.d, w.hidden
    T, M = w.n_tokens, w.n_ray
    cfg = R.make_config(H, d, hid, renorm=R.RENORM_ROW, precision=R.PREC_BF16_TC,
                        ns_steps=args.ns_steps)
    cfg_ns = R.make_config(H, d, hid, renorm=R.RENORM_ROW, precision=R.PREC_BF16_TC,
                           ns_steps=max(args.ns_steps, 5))

    x = wl.make_inputs(w, bits=True)
    to_bf = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)  # noqa: E731
    hK, hV, hQ = to_bf(x.K), to_bf(x.V), to_bf(x.Q)
    hQr = to_bf(x.Qray) if x.Qray is not None else torch.zeros((0, H * d), dtype=torch.bfloat16)
    heta = torch.from_numpy(x.eta)
    hW = []
    for layer in range(layers):
        xl = x if layer == 0 else None
        if xl is None:
            rngw = np.random.default_rng([w.seed, layer])
            W1, W2, W3 = wl.draw_weights(rngw, H, d, hid, 1.0 / d, 1.0 / hid)
        else:
            W1, W2, W3 = xl.W1, xl.W2, xl.W3
        hW.append(tuple(torch.from_numpy(a) for a in (W1, W2, W3)))
    del x

    K, V, Q, Qr = (t.to(dev) for t in (hK, hV, hQ, hQr))
    eta = heta.to(dev)
    Win = [tuple(t.to(dev) for t in ws) for ws in hW]
    Wout = [tuple(torch.empty_like(t) for t in ws) for ws in Win]
    shadow = R.alloc_shadow(cfg, dev)
    ws_buf = R.alloc_workspace(cfg_ns, T, dev)  # also large enough for cfg
    O = torch.empty((T, H * d), dtype=torch.bfloat16, device=dev)
    Or = torch.empty((M, H * d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(o_hook=None):
        for layer in range(layers):
            W1, W2, W3 = Win[layer]
            a, b, c = Wout[layer]
            R.ttt_update(cfg, W1, W2, W3, K, V, eta, a, b, c, shadow=shadow, workspace=ws_buf,
                         stream=stream)
            R.ttt_apply(cfg, Q, O, shadow=shadow, stream=stream)
            if M:
                R.ttt_apply(cfg, Qr, Or, shadow=shadow, stream=stream)
            if o_hook is not None:
                o_hook(layer)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    R.ttt_check_device_error()

    # -------------------------------------------------- timed region
    R.ttt_trace_enable(True)
    R.ttt_trace_read(reset=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    R.ttt_trace_enable(False)
    trace = R.ttt_trace_read(reset=True)
    R.ttt_check_device_error()
    ms = rank_max(e0.elapsed_time(e1) / args.steps)
    value = aggregate_value(world, T, layers, ms)

    # -------------------------------------------------- roofline
    pk, pk_kind = peaks()
    reps = layers * args.steps
    kw = kernel_work(d, hid)
    units = {"tc_update_fused": T * H * reps, "tc_apply": (T + M) * H * reps}
    splits = R.ttt_update_splits(cfg, T)
    per_kernel = {k: {"launches": v[0], "ms_total": v[1], "ms_avg": v[1] / max(v[0], 1)}
                  for k, v in trace.items()}
    for k, ent in kw.items():
        if k in trace:
            per_kernel[k]["roofline"] = roofline_entry(ent["flops"] * units[k],
                                                       ent["bytes"] * units[k], trace[k][1], pk,
                                                       ent["bound"])
    if "reduce_renorm" in trace:
        by = renorm_bytes(H, d, hid, splits) * trace["reduce_renorm"][0]
        per_kernel["reduce_renorm"]["roofline"] = roofline_entry(0.0, by,
                                                                 trace["reduce_renorm"][1], pk,
                                                                 "hbm")
        per_kernel["reduce_renorm"]["splits"] = splits
    dom = max((k for k in kw if k in trace), key=lambda k: trace[k][1])
    launches = trace[dom][0]
    roof = dict(per_kernel[dom]["roofline"])
    roof["peak_kind"] += f" ({pk_kind})"
    roof["kernel"] = dom
    roof["algorithmic_per_launch"] = kw[dom]["flops"] * units[dom] / max(launches, 1)
    roof["algorithmic_bytes_per_launch"] = kw[dom]["bytes"] * units[dom] / max(launches, 1)
    # DRAM bytes per launch from the committed ncu capture (None if its
    # kernel sources changed since); apply launches alternate image and ray
    # queries, so one averages (T + M) / 2 queries
    roof["traffic"] = traffic_per_launch(dom, (T + M) * H / 2 if dom == "tc_apply" else T * H)
    roof["traffic_over_algorithmic_bytes"] = (roof["traffic"] / roof["algorithmic_bytes_per_launch"]
                                              if roof["traffic"] else None)
    upd_ms = trace.get("tc_update_fused", (0, 0.0))[1]
    upd_all_ms = upd_ms + trace.get("reduce_renorm", (0, 0.0))[1]
    upd_flops = kw["tc_update_fused"]["flops"] * T * H * reps
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded normal q/k/v, L2-normalised per head; no dataset)",
            "config": workload_config(w, layers), "roofline": roof,
            "update_gemm_tensor_frac": {
                "value": upd_flops / (upd_ms / 1e3) / 1e12 / pk["bf16_tflops_sustained"]
                if upd_ms else None,
                "of": "bf16_tflops_sustained",
                "burst_frac": (upd_flops / (upd_ms / 1e3) / 1e12 / pk["bf16_tflops"]
                               if upd_ms else None),
                "update_gemm_ms_per_layer": upd_ms / reps,
                "update_ms_per_layer": upd_all_ms / reps},
            "kernels": per_kernel, "clocks": clk,
            "gpu_launches": int(sum(v[0] for v in trace.values()))}
    if args.ns_steps:
        line["config"]["ns_steps"] = args.ns_steps

    # -------------------------------------------------- ray queries on their own
    if M:
        er0, er1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        er0.record(stream)
        for _ in range(5):
            R.ttt_apply(cfg, Qr, Or, shadow=shadow, stream=stream)
        er1.record(stream)
        torch.cuda.synchronize(dev)
        ray_ms = rank_max(er0.elapsed_time(er1) / 5)
        img_ms = ms / layers - ray_ms
        line["ray_apply"] = {"queries": M, "ms_per_layer": ray_ms,
                             "update_plus_image_apply_ms_per_layer": img_ms,
                             "tokens_per_s_update_plus_image_apply":
                                 aggregate_value(world, T, 1, img_ms)}
    # -------------------------------------------------- e2e through host buffers
    if not args.no_e2e:
        line["e2e"] = e2e(args, R, torch, dev, cfg, hK, hV, hQ, hQr, heta, hW, K, V, Q, Qr, eta,
                          Win, Wout, shadow, ws_buf, O, Or, layers, T, M, world, barrier,
                          rank_max)
    # -------------------------------------------------- Newton-Schulz update
    if not args.no_ns_probe:
        line["ns_update"] = ns_probe(R, torch, dev, cfg_ns, K, V, eta, Win[0], Wout[0], shadow,
                                     ws_buf, stream, d, hid, H, pk, rank_max)
    # -------------------------------------------------- token-sharded update
    if not args.no_shard_probe:
        line["sharded_update"] = shard_probe(R, torch, dev, cfg, K, V, eta, Win[0], Wout[0],
                                             shadow, ws_buf, stream, T, world, rank, rank_max)
    # -------------------------------------------------- gated output unit
    if not args.no_gate_probe:
        line["gate"] = gate_probe(R, torch, dev, cfg, O, H, d, T, stream, pk, rank_max)
    # -------------------------------------------------- streaming (stream256)
    if not args.no_stream:
        line["stream"] = stream_bench(R, torch, dev, rank_max)
    # -------------------------------------------------- CPU baseline
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def ns_probe(R, torch, dev, cfg, K, V, eta, Win, Wout, shadow, ws, stream, d, hid, H, pk,
             rank_max, reps: int = 5) -> dict:
    """One layer's update with Newton-Schulz on (cfg.ns_steps steps of Muon's
    quintic on each of the 3*H gradient matrices), after 2 untimed runs.
    Reports the whole update per layer and the NS stages from the library's
    trace (events on the stream).  Algorithmic NS flops per matrix and step:
    2 Rp^2 hidden (X X^T) + 2 Rp^3 (A A) + 2 Rp^2 hidden (B X), Rp = d."""
    steps = cfg.ns_steps
    for _ in range(2):
        R.ttt_update(cfg, *Win, K, V, eta, *Wout, shadow=shadow, workspace=ws, stream=stream)
    torch.cuda.synchronize(dev)
    R.ttt_trace_enable(True)
    R.ttt_trace_read(reset=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        R.ttt_update(cfg, *Win, K, V, eta, *Wout, shadow=shadow, workspace=ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    R.ttt_trace_enable(False)
    tr = R.ttt_trace_read(reset=True)
    R.ttt_check_device_error()
    upd = rank_max(e0.elapsed_time(e1) / reps)
    ns_names = ("ns_prepare", "ns_tc_iterate", "ns_finish")
    ns_ms = sum(tr.get(k, (0, 0.0))[1] for k in ns_names) / reps
    it_ms = tr.get("ns_tc_iterate", (0, 0.0))[1] / reps
    flops = 3 * H * steps * (4 * d * d * hid + 2 * d ** 3)
    ach = flops / (it_ms / 1e3) / 1e12 if it_ms else None
    return {"ns_steps": steps, "update_ms_per_layer": upd,
            "ns_stage_ms": ns_ms, "ns_iterate_ms": it_ms,
            "ns_stage_share_of_update": ns_ms / upd if upd else None,
            "ns_iterate_tflops": ach,
            "ns_iterate_frac_of_burst": ach / pk["bf16_tflops"] if ach else None,
            "stages_ms": {k: tr[k][1] / reps for k in ns_names if k in tr},
            "note": "NS GEMMs issue 3 bf16 MMAs per product (hi/lo operand split); "
                    "achieved counts the algorithmic flops once"}


def shard_probe(R, torch, dev, cfg, K, V, eta, Win, Wout, shadow, ws, stream, T, world, rank,
                rank_max, reps: int = 5) -> dict:
    """One layer's update of the whole scene split over the ranks: each rank
    reduces its token shard (ttt_update_partial), the partials are exchanged
    by one NCCL all-gather, and every rank finishes the same Ŵ
    (ttt_update_finish).  Timed with events on the stream, max over ranks."""
    from recon_chunk_ttt_b200.sharded import exchange_partials, shard_range
    a, b = shard_range(T, rank, world)
    Kr, Vr, er = K[a:b], V[a:b], eta[a:b]
    partial = torch.empty(R.ttt_partial_floats(cfg), dtype=torch.float32, device=dev)
    fin_ws = torch.empty(max(R.ttt_finish_workspace_bytes(cfg), 1), dtype=torch.uint8,
                         device=dev)

    def one():
        R.ttt_update_partial(cfg, *Win, Kr, Vr, er, partial=partial, workspace=ws, stream=stream)
        gathered = exchange_partials(partial) if world > 1 else partial.view(1, -1)
        R.ttt_update_finish(cfg, *Win, gathered, *Wout, shadow=shadow, workspace=fin_ws,
                            stream=stream)

    for _ in range(2):
        one()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    R.ttt_check_device_error()
    return shard_fields(world, b - a, T, rank_max(e0.elapsed_time(e1) / reps))


def shard_fields(world: int, tokens_per_rank: int, T: int, ms: float) -> dict:
    """The token-sharded update's line: ms is already the max over ranks; the
    throughput is the one scene's T tokens over that time (strong scaling:
    the scene is fixed, the ranks share it)."""
    return {"ranks": world, "tokens_per_rank": tokens_per_rank, "tokens": T,
            "ms_per_layer_update": ms, "update_tokens_per_s_one_scene": T / (ms / 1e3),
            "scaling": "strong",
            "exchange": "NCCL all-gather of one fp32 partial per rank" if world > 1 else "none"}


def gate_probe(R, torch, dev, cfg, O, H, d, T, stream, pk, rank_max, reps: int = 5) -> dict:
    """The gated output unit on the layer's image output (T x H*d bf16, larger
    than L2), in place, after 2 untimed runs; W_g ~ N(0, 1/d), bf16.
    Algorithmic bytes per launch: o' read + o written, 4 * T * H * d; flops
    2 d^2 per row and head (128 flop/B: HBM-bound)."""
    rng = np.random.default_rng(8)
    Wg = torch.from_numpy((rng.standard_normal((H, d, d)) / np.sqrt(d)).astype(np.float32))
    Wg = Wg.to(torch.bfloat16).to(dev)
    for _ in range(2):
        R.ttt_gate(cfg, Wg, O, O=O, stream=stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        R.ttt_gate(cfg, Wg, O, O=O, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    R.ttt_check_device_error()
    ms = rank_max(e0.elapsed_time(e1) / reps)
    by = 4.0 * T * H * d
    gbs = by / (ms / 1e3) / 1e9
    traffic = traffic_per_launch("tc_gate", T * H)
    return {"ms_per_launch": ms, "rows": T, "achieved_gbs": gbs,
            "frac_of_hbm": gbs / pk["hbm_gbs"], "tflops": 2.0 * d * d * T * H / (ms / 1e3) / 1e12,
            "bytes_per_launch": by, "traffic": traffic}


def stream_bench(R, torch, dev, rank_max, warm_frames: int = 8) -> dict:
    """The streaming row: stream256 (256 frames of 1374 tokens, 4 heads x 256,
    hidden 512) fed one frame per ttt_stream_step call (update in place, then
    apply to the frame's queries).  Per-frame latency from CUDA events on the
    stream around each call (it includes host launch time when the host is
    slower than the GPU); tokens/s over all frames."""
    w = wl.WORKLOADS["stream256"]
    x = wl.make_inputs(w, bits=True)
    to_bf = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa
    K, V, Q = to_bf(x.K), to_bf(x.V), to_bf(x.Q)
    eta = torch.from_numpy(x.eta).to(dev)
    cfg = R.make_config(w.heads, w.d, w.hidden, renorm=R.RENORM_ROW)
    W1, W2, W3 = (torch.from_numpy(a).to(dev) for a in (x.W1, x.W2, x.W3))
    shadow = R.alloc_shadow(cfg, dev)
    p = w.p
    ws = R.alloc_workspace(cfg, p, dev)
    O = torch.empty((p, w.heads * w.d), dtype=torch.bfloat16, device=dev)
    st = torch.cuda.current_stream(dev)

    def frame(f):
        s, e = f * p, (f + 1) * p
        R.ttt_stream_step(cfg, W1, W2, W3, shadow, K[s:e], V[s:e], eta[s:e], Q[s:e], O,
                          workspace=ws, stream=st)

    for f in range(warm_frames):
        frame(f)
    W1.copy_(torch.from_numpy(x.W1))
    W2.copy_(torch.from_numpy(x.W2))
    W3.copy_(torch.from_numpy(x.W3))
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(w.frames + 1)]
    ev[0].record(st)
    h0 = time.perf_counter()
    for f in range(w.frames):
        frame(f)
        ev[f + 1].record(st)
    host_ms = (time.perf_counter() - h0) * 1e3 / w.frames
    torch.cuda.synchronize(dev)
    R.ttt_check_device_error()
    lat = sorted(ev[f].elapsed_time(ev[f + 1]) for f in range(w.frames))
    total_ms = rank_max(ev[0].elapsed_time(ev[-1]))
    flops = (12 + 6) * w.d * w.hidden * w.heads * p * w.frames
    # Where a frame's time goes: a separate, untimed pass with every launch
    # bracketed by events (the events add their own small cost).
    nf = min(64, w.frames)
    R.ttt_trace_enable(True)
    R.ttt_trace_read(reset=True)
    for f in range(nf):
        frame(f)
    torch.cuda.synchronize(dev)
    R.ttt_trace_enable(False)
    tr = R.ttt_trace_read(reset=True)
    per_kernel_us = {k: v[1] * 1e3 / nf for k, v in tr.items()}
    busy_us = sum(per_kernel_us.values())
    p50 = lat[len(lat) // 2]
    return {"workload": f"stream256: {w.frames} frames x {p} tokens, {w.heads} heads x d={w.d}, "
                        f"hidden {w.hidden}, one ttt_stream_step per frame",
            "frame_ms_p50": p50, "frame_ms_p99": lat[min(len(lat) - 1, int(0.99 * len(lat)))],
            "host_enqueue_ms_per_frame": host_ms,
            "tokens_per_s": w.frames * p / (total_ms / 1e3),
            "achieved_tflops": flops / (total_ms / 1e3) / 1e12,
            "kernel_us_per_frame": per_kernel_us,
            "kernel_busy_us_per_frame": busy_us,
            "launches_per_frame": sum(v[0] for v in tr.values()) / nf,
            "between_kernels_us_per_frame": p50 * 1e3 - busy_us}


def e2e(args, R, torch, dev, cfg, hK, hV, hQ, hQr, heta, hW, K, V, Q, Qr, eta, Win, Wout,
        shadow, ws_buf, O, Or, layers, T, M, world, barrier, max_over_ranks):
    """The same step through the public API with the inputs in pinned host
    memory: every step copies K, V, Q, ray Q, eta and the 24 layers' weights
    host -> device, runs the stack, and copies every layer's outputs (image
    and ray O) and updated weights device -> host (on a second stream,
    overlapped with the next layer)."""
    pin = lambda t: t.pin_memory()  # noqa: E731
    pK, pV, pQ, pQr, peta = (pin(t) for t in (hK, hV, hQ, hQr, heta))
    pW = [tuple(pin(t) for t in ws) for ws in hW]
    oO = [torch.empty(O.shape, dtype=O.dtype, pin_memory=True) for _ in range(2)]
    oOr = [torch.empty(Or.shape, dtype=Or.dtype, pin_memory=True) for _ in range(2)]
    oW = [tuple(torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in ws) for ws in Win]
    st = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(dev)
    h2d = sum(t.numel() * t.element_size() for t in (pK, pV, pQ, pQr, peta)) + \
        sum(t.numel() * t.element_size() for ws in pW for t in ws)
    d2h = layers * (O.numel() * O.element_size() + Or.numel() * Or.element_size()) + \
        sum(t.numel() * t.element_size() for ws in Win for t in ws)
    # Outputs of layer l go to host buffer l % 2 on the side stream; the
    # device O/Or buffers are double-buffered too so compute never overwrites
    # an output still being copied.
    Ob = [O, torch.empty_like(O)]
    Orb = [Or, torch.empty_like(Or)]
    done = [torch.cuda.Event(), torch.cuda.Event()]

    def one():
        for src, dst in ((pK, K), (pV, V), (pQ, Q), (pQr, Qr), (peta, eta)):
            dst.copy_(src, non_blocking=True)
        for ws_h, ws_d in zip(pW, Win):
            for a, b in zip(ws_h, ws_d):
                b.copy_(a, non_blocking=True)
        for layer in range(layers):
            b = layer % 2
            st.wait_event(done[b]) if layer >= 2 else None
            W1, W2, W3 = Win[layer]
            a1, a2, a3 = Wout[layer]
            R.ttt_update(cfg, W1, W2, W3, K, V, eta, a1, a2, a3, shadow=shadow,
                         workspace=ws_buf, stream=st)
            R.ttt_apply(cfg, Q, Ob[b], shadow=shadow, stream=st)
            if M:
                R.ttt_apply(cfg, Qr, Orb[b], shadow=shadow, stream=st)
            ev = torch.cuda.Event()
            ev.record(st)
            side.wait_event(ev)
            with torch.cuda.stream(side):
                oO[b].copy_(Ob[b], non_blocking=True)
                oOr[b].copy_(Orb[b], non_blocking=True)
                for t_h, t_d in zip(oW[layer], Wout[layer]):
                    t_h.copy_(t_d, non_blocking=True)
            done[b].record(side)
        st.wait_stream(side)

    one()
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.e2e_steps):
        one()
    e1.record(st)
    torch.cuda.synchronize(dev)
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps)
    return {"value": aggregate_value(world, T, layers, ms), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": args.e2e_steps}


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")


def traffic_per_launch(kernel: str, units: float, path: str = TRAFFIC_JSON):
    """DRAM bytes of one launch of `kernel` processing `units` token- or
    query-heads, from the per-unit figure an ncu capture left in
    profiles/traffic.json; None when there is no entry or the kernel sources
    changed since the capture (their hash no longer matches)."""
    if not os.path.exists(path):
        return None
    with open(path) as f:
        ent = json.load(f).get(kernel)
    if not ent or ent.get("source_sha") != kernel_source_sha(ent.get("sources")):
        return None
    return ent["bytes_per_unit"] * units


def kernel_source_sha(files=None) -> str:
    """Hash of the kernel sources (all of csrc/, or the listed files of it)."""
    import hashlib
    csrc = os.path.join(ROOT, "recon_chunk_ttt_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(files if files else os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def run_stream_only():
    """The streaming row alone on one GPU (used to profile a frame's kernels)."""
    import torch
    import recon_chunk_ttt_b200 as R
    from recon_chunk_ttt_b200 import build as B
    B.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    print(json.dumps({"stream": stream_bench(R, torch, dev, lambda v: v)}), flush=True)


def main():
    args = parse()
    if args.only_stream:
        run_stream_only()
        return
    world, rank, local = dist_setup(args)
    w = wl.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w, world, rank)
    else:
        run_ours(args, w, world, rank, local)


if __name__ == "__main__":
    main()
