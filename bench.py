#!/usr/bin/env python
"""Benchmark of the B200 MoE layer (libmok) -- one JSON line on rank 0.

A step is one forward + backward pass of the DeepSeek-V3-shaped BF16 layer
(T=4096, H=7168, E=256, top-8, I=2048, one shared expert, sigmoid + bias
group-limited routing) over one batch of seeded synthetic tokens, through the
C ABI (moe_fwd, moe_bwd).  Inputs are resident in HBM when the timed region
starts; the 22.6 GB of expert weights exceed the 126 MB L2, so no flush is
needed between steps.  With N GPUs (torchrun) every rank runs its own replica
on its own tokens (the layer has no exchange step on one GPU's experts):
value = tokens of all ranks / max-over-ranks time, scaling "weak".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl mok|reference]

--impl reference times the fp64 CPU oracle on the host cores (rank 0 only) on
a bounded token sample of the same workload.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s fwd MXFP8 & BF16, bwd BF16; % of tensor-core peak"
FWD_PHASES = ["router", "dispatch", "gate_up_gemm", "down_gemm", "combine"]
BWD_PHASES = ["down_dgrad_gemm", "slot_grad", "drouter_partial", "drouter_reduce", "down_wgrad_gemm",
              "gate_up_dgrad_gemm", "gate_up_wgrad_gemm", "dx_sum"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="dsv3")
    ap.add_argument("--impl", default="mok", choices=["mok", "reference"])
    ap.add_argument("--schedule", default="persistent", choices=["persistent", "split"],
                    help="forward schedule of the timed steps (the A/B leg runs both)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-ab", action="store_true", help="skip the schedule A/B legs (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--extra-workloads", default="small,dsv3_zipf",
                    help="BF16 workloads also measured, comma-separated ('none' to skip)")
    ap.add_argument("--mx-workload", default="dsv3_mxfp8",
                    help="MXFP8 forward workload measured after the main one ('none' to skip)")
    ap.add_argument("--ep-world", type=int, default=8,
                    help="ranks of the expert-parallel layer emulated on one GPU (0 to skip)")
    ap.add_argument("--ep-only", action="store_true",
                    help="run only the emulated expert-parallel measurement (profiling runs)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def fp8_peak(dev, seconds=2.0):
    """Dense FP8 (e4m3, fp32 accumulate, bf16 out) matmul throughput of this GPU through
    the library routine torch._scaled_mm at 8192^3: the best of 20 calls (burst) and
    the mean over a loop of about `seconds` (sustained), in TFLOP/s, CUDA events on the
    current stream."""
    import torch
    n = 8192
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
    one = torch.ones((), device=dev)
    mm = lambda: torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    for _ in range(5):
        mm()
    torch.cuda.synchronize()
    flop = 2.0 * n ** 3
    best = 0.0
    for _ in range(20):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        mm()
        e.record()
        e.synchronize()
        best = max(best, flop / (s.elapsed_time(e) / 1e3) / 1e12)
    iters = max(10, int(seconds / (flop / (best * 1e12))))
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(iters):
        mm()
    e.record()
    e.synchronize()
    sustained = flop * iters / (s.elapsed_time(e) / 1e3) / 1e12
    del a, b
    return {"burst_tflops": best, "sustained_tflops": sustained, "source": "torch._scaled_mm e4m3 8192^3, "
            "per-tensor scales, bf16 out, measured in this run"}


# ------------------------------------------------------------------ clocks
class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.path = tempfile.mktemp(prefix="clocks", suffix=".csv")
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ replicas
def replica_throughput(ms_local: float, tokens_local: int, dist=None, device=None):
    """Whole-job throughput of independent replicas: every rank's tokens over the
    slowest rank's time (max over ranks).  Returns (tokens/s, max ms, total tokens)."""
    import torch
    t = torch.tensor([ms_local, float(tokens_local)], dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        mx = t[:1].clone()
        dist.all_reduce(mx, op=dist.ReduceOp.MAX)
        tok = t[1:].clone()
        dist.all_reduce(tok, op=dist.ReduceOp.SUM)
        t = torch.cat([mx, tok])
    ms, tokens = float(t[0]), int(t[1])
    return tokens / (ms / 1e3), ms, tokens


# ------------------------------------------------------------------ algorithmic counts
def algorithmic(wl, counts):
    """FLOPs and bytes of each GEMM phase (per launch) from the routing counts."""
    T, H, I, E, S, k = wl.T, wl.H, wl.I, wl.E, wl.S, wl.k
    R = T * (k + S)
    groups = int((counts > 0).sum()) + S          # experts whose weights are streamed
    wgu = groups * 2 * I * H * 2
    wdn = groups * H * I * 2
    G = E + S
    out = {
        "gate_up_gemm": (4 * H * I * R, wgu + T * H * 2 + R * I * 2 * 2 + R * 2 * I * 2),
        "down_gemm": (2 * H * I * R, wdn + R * I * 2 + T * (k + S) * H * 4),
        "down_dgrad_gemm": (2 * H * I * R, wdn + T * H * 2 + R * 2 * I * 2 * 2),
        "down_wgrad_gemm": (2 * H * I * R, T * H * 2 + R * I * 2 + G * H * I * 2),
        "gate_up_dgrad_gemm": (4 * H * I * R, wgu + R * 2 * I * 2 + T * (k + S) * H * 4),
        "gate_up_wgrad_gemm": (4 * H * I * R, R * 2 * I * 2 + T * H * 2 + G * 2 * I * H * 2),
    }
    return out


def forward_algorithmic(wl, counts):
    """FLOPs and bytes of one whole forward (the persistent kernel's work): the two
    expert GEMMs plus the router (x read, three bf16 router terms written and read,
    partial logits) and the combine (slot rows read, y written)."""
    alg = algorithmic(wl, counts)
    T, H, E, k, S = wl.T, wl.H, wl.E, wl.k, wl.S
    slot_bytes = 2 if wl.mxfp8 else 4
    fl = alg["gate_up_gemm"][0] + alg["down_gemm"][0] + 2 * 3 * H * E * T
    nb = (alg["gate_up_gemm"][1] + alg["down_gemm"][1] + T * H * 2 + 2 * E * 3 * H * 2
          + T * (k + S) * H * slot_bytes + T * H * 2)
    return fl, nb


def backward_algorithmic(wl, counts):
    """FLOPs and bytes of one whole backward (the persistent kernel's work): the four
    expert GEMMs plus the slot and router gradients (x read) and the dx sum (slot rows
    read, dx written)."""
    alg = algorithmic(wl, counts)
    T, H, E, k, S = wl.T, wl.H, wl.E, wl.k, wl.S
    names = ["down_dgrad_gemm", "down_wgrad_gemm", "gate_up_dgrad_gemm", "gate_up_wgrad_gemm"]
    fl = sum(alg[n][0] for n in names) + 2 * T * k * H
    nb = sum(alg[n][1] for n in names) + T * H * 2 + T * (k + S) * H * 4 + T * H * 2 + E * H * 4
    return fl, nb


BWD_STAMP_PHASES = ["q0_zero", "dgrads", "down_wgrad_after_dgrads", "gate_up_wgrad_after_down_wgrad", "slot_grad",
                    "router_partial", "dx_sum", "router_reduce"]


STAMP_PHASES = ["p0_zero_split_quant", "router_gemm", "select", "dispatch", "gate_up_gemm", "down_after_gate_up",
                "combine"]


def stamp_phases(bufs, sms, names=None):
    """Phase spans (ms) of the persistent forward from its device stamps, averaged over
    steps: a phase runs from the last CTA's end of the previous phase (the barrier
    release) to the last CTA's end of its own; the down GEMM overlaps the gate/up
    tail, so its span counts only the part after the last gate/up tile."""
    import numpy as np
    names = names or STAMP_PHASES
    acc = np.zeros(len(names))
    for b in bufs:
        t = b.view(-1, sms).cpu().numpy().astype(np.float64)[: len(names) + 1]
        ends = t.max(axis=1)
        acc[0] += ends[1] - t[0].min()
        acc[1:] += np.diff(ends[1:])
    return {n: round(float(v) / len(bufs) / 1e6, 4) for n, v in zip(names, acc)}


def _ab(layer, run, K, legs, trace_split, stamp_names):
    """Interleaved A/B of the schedules: in each of K rounds every leg runs once, timed
    with CUDA events around the pass (power and clock drift then hits every leg
    alike).  The split leg also records an event per step, the persistent leg its
    device stamps."""
    import torch
    from mixture_experts_layer_persistent_b200 import abi
    dev = layer.device
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mk = lambda: torch.cuda.Event(enable_timing=True)
    restore = abi.moe_get_schedule()
    for name, sched in legs:                       # warm-up of every leg
        abi.moe_set_schedule(sched)
        run(None, None)
        run(None, None)
    n_ev = (abi.MOK_FWD_PHASES if trace_split == "fwd" else abi.MOK_BWD_PHASES) + 1
    rec = {name: {"t": [], "ev": [], "st": []} for name, _ in legs}
    # events and stamp buffers made before the rounds; torch creates a CUDA event at its
    # first record, so every event is recorded once before the library records it
    evs = [[mk() for _ in range(n_ev)] for _ in range(K)]
    for e in [e for ev in evs for e in ev]:
        e.record()
    sts = [torch.zeros(abi.MOK_TRACE_POINTS * sms, dtype=torch.int64, device=dev) for _ in range(K)]
    torch.cuda.synchronize()
    for i in range(K):
        for name, sched in legs:
            abi.moe_set_schedule(sched)
            s, e = mk(), mk()
            ev = evs[i] if name == "split" else None
            st = sts[i] if name == "persistent" else None
            s.record()
            run(ev, st)
            e.record()
            rec[name]["t"].append((s, e))
            rec[name]["ev"].append(ev)
            rec[name]["st"].append(st)
            rec[name]["launches"] = abi.moe_launch_count()
    torch.cuda.synchronize()
    abi.moe_set_schedule(restore)
    out = {}
    for name, _ in legs:
        r = rec[name]
        o = {"ms": statistics.mean(a.elapsed_time(b) for a, b in r["t"]), "launches": r["launches"]}
        if name == "split":
            names = FWD_PHASES if trace_split == "fwd" else BWD_PHASES
            o["phases_ms"] = {n: round(statistics.mean(ev[j].elapsed_time(ev[j + 1]) for ev in r["ev"]), 4)
                              for j, n in enumerate(names)}
        if name == "persistent":
            o["device_phases_ms"] = stamp_phases(r["st"], sms, stamp_names)
        out[name] = o
    out["persistent_over_split_speedup"] = out["split"]["ms"] / out["persistent"]["ms"]
    out["split_pdl_over_split_speedup"] = out["split"]["ms"] / out["split_pdl"]["ms"]
    out["order"] = "interleaved: each round runs split, split_pdl, persistent once"
    return out


def _legs():
    from mixture_experts_layer_persistent_b200 import abi
    return (("split", abi.MOK_SCHEDULE_SPLIT), ("split_pdl", abi.MOK_SCHEDULE_SPLIT_PDL),
            ("persistent", abi.MOK_SCHEDULE_PERSISTENT))


def forward_ab(layer, x, y, K):
    """Forward only: split, PDL-split and persistent schedules, interleaved."""
    from mixture_experts_layer_persistent_b200 import abi, moe_trace_events

    def run(ev, st):
        if ev is not None:
            moe_trace_events([e.cuda_event for e in ev], None)
        if st is not None:
            abi.moe_trace_device(st.data_ptr(), st.numel() * 8)
        layer.forward(x, y)
        moe_trace_events(None, None)
        abi.moe_trace_device(None, 0)

    out = _ab(layer, run, K, _legs(), "fwd", STAMP_PHASES)
    for leg in ("split", "split_pdl", "persistent"):     # names kept for readers of earlier lines
        out[leg]["ms_per_fwd"] = out[leg]["ms"]
    return out


def backward_ab(layer, x, dy, grads, K):
    """Backward only: split, PDL-split and persistent schedules, interleaved."""
    from mixture_experts_layer_persistent_b200 import abi, moe_trace_events

    def run(ev, st):
        if ev is not None:
            moe_trace_events(None, [e.cuda_event for e in ev])
        if st is not None:
            abi.moe_trace_device(None, 0, st.data_ptr(), st.numel() * 8)
        layer.backward(x, dy, grads)
        moe_trace_events(None, None)
        abi.moe_trace_device(None, 0)

    out = _ab(layer, run, K, _legs(), "bwd", BWD_STAMP_PHASES)
    for leg in ("split", "split_pdl", "persistent"):
        out[leg]["ms_per_bwd"] = out[leg]["ms"]
    return out


def source_hash():
    """sha256 over the CUDA sources: DRAM counters are reported only for the sources they
    were taken from."""
    import glob
    import hashlib
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "mixture_experts_layer_persistent_b200", "csrc", "*"))):
        h.update(open(f, "rb").read())
    return h.hexdigest()


def measured_traffic(wl, kernel):
    """DRAM bytes per launch of `kernel` on this workload, from the committed ncu capture of
    the 16-expert workload of the same expert shape and rows per expert (dsv3_e16_r128,
    profiles/dram_traffic_dsv3_e16.json) scaled by the ratio of tokens (every expert-,
    row- and token-proportional stream scales with it), or None when the workload differs
    or the kernel sources changed since the capture."""
    path = os.path.join(ROOT, "profiles", "dram_traffic_dsv3_e16.json")
    if wl.name != "dsv3" or not os.path.exists(path):
        return None
    rec = json.load(open(path))
    if rec.get("source_sha256") != source_hash() or kernel not in rec["per_launch_bytes"]:
        return None
    return int(rec["per_launch_bytes"][kernel] * wl.T / rec["tokens"])


# ------------------------------------------------------------------ CPU oracle sample
def oracle_sample(wl, params, x, dy, seconds, log=None):
    """Time the fp64 oracle's forward + dx backward on a token sample of the workload."""
    import numpy as np
    import oracle
    from mixture_experts_layer_persistent_b200 import synth
    from tests._support import oracle_layer

    L = oracle_layer(wl, params, synth.bf16_bits(x), synth.bf16_bits(dy))
    idx, w, _ = L.route(tokens=np.arange(1))
    t0 = time.perf_counter()
    L.route(tokens=np.arange(1), into=(idx, w, np.zeros(wl.T)))
    L.fwd(idx, w, tokens=[0])
    L.bwd(idx, w, tokens=[0])
    one = time.perf_counter() - t0
    cores = oracle.num_threads()          # the oracle parallelises over tokens
    n = int(max(cores, min(wl.T, cores * int(seconds / max(one, 1e-6)))))
    toks = np.arange(n, dtype=np.int32)
    t0 = time.perf_counter()
    gap = np.zeros(wl.T)
    L.route(tokens=toks, into=(idx, w, gap))
    L.fwd(idx, w, tokens=toks)
    L.bwd(idx, w, tokens=toks)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "tokens/s (routing + forward + dx backward; weight gradients excluded)",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"routing + forward + dx backward of {n} of the {wl.T} tokens of the {wl.name} "
                      f"workload (fp64 C oracle, OpenMP over tokens; weight gradients not in the sample)",
            "seconds": dt}


# ------------------------------------------------------------------ main
def main():
    args = parse()
    from mixture_experts_layer_persistent_b200 import build as _build
    _build.build()          # no-op unless a source is newer than libmok.so
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.impl == "reference":
        if rank == 0:
            reference_arm(args, world)
        if world > 1:
            dist.destroy_process_group()
        return

    from mixture_experts_layer_persistent_b200 import MoELayer, abi, cfg_for, synth, moe_trace_events

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    sched = abi.MOK_SCHEDULE_SPLIT if args.schedule == "split" else abi.MOK_SCHEDULE_PERSISTENT
    abi.moe_set_schedule(sched)
    wl = synth.WORKLOADS[args.workload]
    wl = synth.scaled(wl, seed=wl.seed + 1000 * rank)
    if args.ep_only:
        W = max(1, args.ep_world)
        ep = ep_emulated_run(synth.scaled(wl, name=wl.name + "_ep", T=wl.T // W, seed=wl.seed + 7), W, dev,
                             args.steps, args.warmup)
        if args.mx_workload and args.mx_workload != "none":
            torch.cuda.empty_cache()
            mwl = synth.WORKLOADS[args.mx_workload]
            ep["mxfp8"] = ep_emulated_mx_run(synth.scaled(mwl, name=mwl.name + "_ep", T=mwl.T // W,
                                                          seed=mwl.seed + 7), W, dev, args.steps, args.warmup)
        if rank == 0:
            print(json.dumps({"ep_emulated": ep}))
        if world > 1:
            dist.destroy_process_group()
        return
    params = synth.draw_params(wl, dev)
    x = synth.draw_x(wl, dev)
    dy = synth.draw_dy(wl, dev)
    layer = MoELayer(cfg_for(wl), params, training=True, device=dev)
    y = torch.empty_like(x)
    grads = layer.new_grads()
    routing = layer.new_routing()
    layer.forward(x, y, routing=routing)
    torch.cuda.synchronize()
    counts = routing["counts"].cpu().numpy()

    launches = [0, 0]               # kernels per forward, per backward (counted by the library)

    def step():
        layer.forward(x, y)
        launches[0] = abi.moe_launch_count()
        layer.backward(x, dy, grads)
        launches[1] = abi.moe_launch_count()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert layer.status() == 0

    K = args.steps
    mk = lambda: torch.cuda.Event(enable_timing=True)
    fev = [[mk() for _ in range(abi.MOK_FWD_PHASES + 1)] for _ in range(K)]
    bev = [[mk() for _ in range(abi.MOK_BWD_PHASES + 1)] for _ in range(K)]
    start, end = mk(), mk()
    for e in [e for ev in fev + bev for e in ev]:
        e.record()              # torch creates the CUDA event on its first record
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    stamps = [torch.zeros(abi.MOK_TRACE_POINTS * sms, dtype=torch.int64, device=dev) for _ in range(K)]
    bstamps = [torch.zeros(abi.MOK_TRACE_POINTS * sms, dtype=torch.int64, device=dev) for _ in range(K)]
    torch.cuda.synchronize()
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    if not uuid.startswith("GPU-"):
        uuid = "GPU-" + uuid
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = Clocks(uuid)
    time.sleep(0.4)
    start.record()
    for i in range(K):
        moe_trace_events([e.cuda_event for e in fev[i]], [e.cuda_event for e in bev[i]])
        abi.moe_trace_device(stamps[i].data_ptr(), stamps[i].numel() * 8, bstamps[i].data_ptr(),
                             bstamps[i].numel() * 8)
        step()
    end.record()
    torch.cuda.synchronize()
    moe_trace_events(None, None)
    abi.moe_trace_device(None, 0)
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    value, ms_max, _ = replica_throughput(start.elapsed_time(end), wl.T * K, dist, dev)
    status = layer.status()

    # the forward is one persistent launch (events around it); the backward's steps are
    # separate launches with an event each
    # each pass is one persistent launch (events around it), or split launches with an
    # event each (--schedule split)
    persistent = sched == abi.MOK_SCHEDULE_PERSISTENT
    fwd_name = "fwd_persistent" if persistent else "fwd_split"
    bwd_name = "bwd_persistent" if persistent else "bwd_split"
    phase = {fwd_name: statistics.mean(fev[i][0].elapsed_time(fev[i][-1]) for i in range(K)),
             bwd_name: statistics.mean(bev[i][0].elapsed_time(bev[i][-1]) for i in range(K))}
    if not persistent:
        for n_i, name in enumerate(BWD_PHASES):
            phase[name] = statistics.mean(bev[i][n_i].elapsed_time(bev[i][n_i + 1]) for i in range(K))
    fwd_ms = phase[fwd_name]
    bwd_ms = phase[bwd_name]
    fwd_device_phases = stamp_phases(stamps, sms) if persistent else None
    bwd_device_phases = stamp_phases(bstamps, sms, BWD_STAMP_PHASES) if persistent else None

    # forward A/B: split schedule (events per step, the per-GEMM attribution below) against
    # the persistent one, forward only
    ab = bab = None
    if not args.no_ab:
        ab = forward_ab(layer, x, y, K)
        for n_i, name in enumerate(FWD_PHASES):
            phase["split_" + name] = ab["split"]["phases_ms"][name]
        layer.forward(x, y)
        bab = backward_ab(layer, x, dy, grads, K)
        for name in BWD_PHASES:
            phase["split_" + name] = bab["split"]["phases_ms"][name]

    pk = peaks()
    alg = algorithmic(wl, counts)
    kern = {fwd_name: forward_algorithmic(wl, counts), bwd_name: backward_algorithmic(wl, counts)}
    kern.update({n: alg[n] for n in alg if n in phase})
    dom = max(kern, key=lambda n: phase[n])
    flops, nbytes = kern[dom]
    t_dom = phase[dom] / 1e3
    t_tc = flops / (pk["bf16_sustained"] * 1e12)
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": nbytes / t_dom / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": flops / t_dom / 1e12, "peak": pk["bf16_sustained"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = measured_traffic(wl, dom)
    roof["kernel"] = dom
    roof["peak_source"] = pk["source"] + (" sustained bf16" if roof["bound"] == "tensor" else " hbm copy")
    roof["algorithmic_flops"] = flops
    roof["algorithmic_bytes"] = nbytes
    # every GEMM phase against both measured peaks (algorithmic bytes and FLOPs / its event time)
    phase_roofline = {}
    for name, (fl, nb) in list(alg.items()) + [(fwd_name, kern[fwd_name]), (bwd_name, kern[bwd_name])]:
        if name not in phase and "split_" + name not in phase:
            continue
        t = (phase[name] if name in phase else phase["split_" + name]) / 1e3
        phase_roofline[name] = {"ms": round(t * 1e3, 4), "hbm_frac": round(nb / t / 1e9 / pk["hbm_gbs"], 4),
                                "tc_frac_sustained": round(fl / t / 1e12 / pk["bf16_sustained"], 4)}

    total_flops = 6 * wl.H * wl.I * wl.T * (wl.k + wl.S)
    fwd_tps = wl.T / (fwd_ms / 1e3)
    bwd_tps = wl.T / (bwd_ms / 1e3)

    # ---------------- end to end through the host-buffer entry points
    e2e = None
    if not args.no_e2e:
        e2e = e2e_run(layer, wl, x, dy, grads, K, world, dist)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(wl, params, x, dy, args.cpu_seconds)

    del layer, grads, params
    torch.cuda.empty_cache()

    # ---------------- the other BF16 workloads (the small forward, the skewed fwd+bwd)
    extra = {}
    for name in ([] if args.extra_workloads in ("", "none") else args.extra_workloads.split(",")):
        ewl = synth.WORKLOADS[name]
        extra[name] = bf16_workload_run(synth.scaled(ewl, seed=ewl.seed + 1000 * rank), dev, K, args.warmup, world,
                                        dist, pk, not args.no_ab)
        torch.cuda.empty_cache()

    # ---------------- MXFP8 forward (block-scaled e4m3) on its own workload
    mx = None
    if args.mx_workload and args.mx_workload != "none":
        mwl = synth.WORKLOADS[args.mx_workload]
        mx = mxfp8_run(synth.scaled(mwl, seed=mwl.seed + 1000 * rank), dev, K, args.warmup, world, dist, pk,
                       not args.no_ab)

    # ---------------- expert-parallel forward, its ranks emulated on this GPU
    ep = None
    if args.ep_world > 0:
        ep = ep_emulated_run(synth.scaled(wl, name=wl.name + "_ep", T=wl.T // args.ep_world,
                                          seed=wl.seed + 1000 * rank + 7), args.ep_world, dev, K, args.warmup)
        torch.cuda.empty_cache()
        if args.mx_workload and args.mx_workload != "none":
            mwl = synth.WORKLOADS[args.mx_workload]
            ep["mxfp8"] = ep_emulated_mx_run(
                synth.scaled(mwl, name=mwl.name + "_ep", T=mwl.T // args.ep_world, seed=mwl.seed + 1000 * rank + 7),
                args.ep_world, dev, K, args.warmup)
            torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_max / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{wl.name}: MoE layer fwd+bwd BF16, T={wl.T}, H={wl.H}, E={wl.E}, "
                                   f"top-{wl.k}, I={wl.I}, {wl.S} shared expert(s), "
                                   + (f"sigmoid+bias routing, {wl.n_group} groups / top-{wl.topk_group}"
                                      if wl.score_fn else "softmax routing")
                                   + (f", Zipf({wl.zipf}) logit term" if wl.zipf else ""),
                       "tokens_per_gpu": wl.T, "parallelism": f"replicas x{world}",
                       "forward_schedule": args.schedule,
                       "l2": "inputs larger than L2 (22.6 GB expert weights streamed per pass)"},
            # persistent schedule: one kernel per pass (split: 9 + 10)
            "gpu_launches": K * (launches[0] + launches[1]),
            "clocks": clk, "device_status": status,
            "phases_ms": {k2: round(v, 4) for k2, v in phase.items()},
            "fwd_device_phases_ms": fwd_device_phases,
            "bwd_device_phases_ms": bwd_device_phases,
            "forward_schedule_ab": ab,
            "backward_schedule_ab": bab,
            "breakdown": {
                "fwd_bf16_tokens_per_s": fwd_tps, "bwd_bf16_tokens_per_s": bwd_tps,
                "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
                "fwd_tc_peak_frac_of_measured_burst": (6 * wl.H * wl.I * wl.T * (wl.k + wl.S) / (fwd_ms / 1e3))
                / (pk["bf16"] * 1e12),
                "bwd_tc_peak_frac_of_measured_burst": (12 * wl.H * wl.I * wl.T * (wl.k + wl.S) / (bwd_ms / 1e3))
                / (pk["bf16"] * 1e12),
                "step_tflops": 3 * total_flops / (ms_max / K / 1e3) / 1e12,
                "expert_load_max_over_mean": float(counts.max() / counts.mean()),
                "empty_experts": int((counts == 0).sum()),
            },
            "roofline": roof,
            "phase_roofline": phase_roofline,
            "mxfp8": mx,
            "bf16_workloads": extra,
            "ep_emulated": ep,
            "e2e": e2e, "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


def bf16_workload_run(wl, dev, K, warmup, world, dist, pk, do_ab=True):
    """Tokens/s and tensor-core fractions of the BF16 layer on another workload (forward, and
    backward when the workload has one), per-phase CUDA events on the layer's stream."""
    import torch
    from mixture_experts_layer_persistent_b200 import MoELayer, abi, cfg_for, moe_trace_events, synth
    params = synth.draw_params(wl, dev)
    x = synth.draw_x(wl, dev)
    dy = synth.draw_dy(wl, dev) if wl.backward else None
    layer = MoELayer(cfg_for(wl), params, training=wl.backward, device=dev)
    y = torch.empty_like(x)
    grads = layer.new_grads() if wl.backward else None
    routing = layer.new_routing()
    layer.forward(x, y, routing=routing)
    counts = routing["counts"].cpu().numpy()
    for _ in range(warmup):
        layer.forward(x, y)
        if wl.backward:
            layer.backward(x, dy, grads)
    torch.cuda.synchronize()
    mk = lambda: torch.cuda.Event(enable_timing=True)
    fev = [[mk() for _ in range(abi.MOK_FWD_PHASES + 1)] for _ in range(K)]
    bev = [[mk() for _ in range(abi.MOK_BWD_PHASES + 1)] for _ in range(K)]
    for e in [e for ev in fev + bev for e in ev]:
        e.record()
    start, end = mk(), mk()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    start.record()
    for i in range(K):
        moe_trace_events([e.cuda_event for e in fev[i]], [e.cuda_event for e in bev[i]] if wl.backward else None)
        layer.forward(x, y)
        if wl.backward:
            layer.backward(x, dy, grads)
    end.record()
    torch.cuda.synchronize()
    moe_trace_events(None, None)
    status = layer.status()
    t = torch.tensor([start.elapsed_time(end)], device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item()) / K
    fwd_ms = statistics.mean(fev[i][0].elapsed_time(fev[i][-1]) for i in range(K))
    bwd_ms = statistics.mean(bev[i][0].elapsed_time(bev[i][-1]) for i in range(K)) if wl.backward else 0.0
    ab = forward_ab(layer, x, y, K) if do_ab else None
    bab = None
    if wl.backward and do_ab:
        layer.forward(x, y)
        bab = backward_ab(layer, x, dy, grads, K)
    fwd_flops = 6 * wl.H * wl.I * wl.T * (wl.k + wl.S)
    out = {"forward_schedule_ab": ab, "backward_schedule_ab": bab,
           "workload": f"{wl.name}: MoE layer {'fwd+bwd' if wl.backward else 'fwd'} BF16, T={wl.T}, H={wl.H}, "
                       f"E={wl.E}, top-{wl.k}, I={wl.I}, {wl.S} shared"
                       + (f", Zipf({wl.zipf}) logit term" if wl.zipf else ""),
           "tokens_per_s": wl.T * world / (ms / 1e3), "ms_per_step": ms,
           "fwd_ms": fwd_ms, "fwd_tokens_per_s": wl.T / (fwd_ms / 1e3),
           "fwd_tc_peak_frac_of_measured_burst": fwd_flops / (fwd_ms / 1e3) / 1e12 / pk["bf16"],
           "fwd_tc_peak_frac_of_measured_sustained": fwd_flops / (fwd_ms / 1e3) / 1e12 / pk["bf16_sustained"],
           "expert_load_max_over_mean": float(counts.max() / max(1e-9, counts.mean())),
           "empty_experts": int((counts == 0).sum()), "device_status": status}
    if wl.backward:
        out.update({"bwd_ms": bwd_ms, "bwd_tokens_per_s": wl.T / (bwd_ms / 1e3),
                    "bwd_tc_peak_frac_of_measured_burst": 2 * fwd_flops / (bwd_ms / 1e3) / 1e12 / pk["bf16"],
                    "bwd_tc_peak_frac_of_measured_sustained":
                        2 * fwd_flops / (bwd_ms / 1e3) / 1e12 / pk["bf16_sustained"]})
    del layer, params, grads
    return out


def ep_emulated_run(wl, W, dev, K, warmup):
    """The expert-parallel layer with its W ranks (wl.T tokens each) run on this GPU in
    stream order, against the one-GPU layer on the same W * wl.T tokens: forward, and
    forward + backward.  Both do the same expert arithmetic; the difference is what the
    rank split adds on one device (the owners' row layouts, the pull copies of the
    received x and dy rows, per-rank launches and tails).  No NVLink is crossed: this is
    the data path, not a multi-GPU measurement."""
    import torch
    from mixture_experts_layer_persistent_b200 import EPWorld, MoELayer, cfg_for, new_rank_grads, split_params, synth
    params = synth.draw_params(wl, dev)
    xs = [synth.draw_x(synth.scaled(wl, seed=wl.seed * 100 + r), dev) for r in range(W)]
    dys = [synth.draw_dy(synth.scaled(wl, seed=wl.seed * 100 + 50 + r), dev) for r in range(W)]
    cfg = cfg_for(wl)
    ep = EPWorld(cfg, W, [split_params(params, W, r, wl.E) for r in range(W)], training=True, device=dev)
    ys = [torch.empty_like(x) for x in xs]
    eg = [new_rank_grads(cfg, W, dev) for _ in range(W)]
    whole = synth.scaled(wl, T=wl.T * W)
    one = MoELayer(cfg_for(whole), params, training=True, device=dev)
    og = one.new_grads()
    xw, dyw = torch.cat(xs), torch.cat(dys)
    yw = torch.empty_like(xw)
    routing = one.new_routing()
    one.forward(xw, yw, routing=routing)
    counts = routing["counts"].cpu().numpy()
    recv = counts.reshape(W, wl.E // W).sum(axis=1)        # expert rows each rank's experts receive
    owner = routing["topk_idx"].long() // (wl.E // W)      # owning rank of every (token, slot)
    pairs = int(torch.zeros(W * wl.T, W, device=owner.device).scatter_(1, owner, 1.0).sum().item())
    for _ in range(warmup):
        ep.forward(xs, ys)
        ep.backward(dys, eg)
        one.forward(xw, yw)
        one.backward(xw, dyw, og)
    torch.cuda.synchronize()
    mk = lambda: torch.cuda.Event(enable_timing=True)
    legs = {"ep": [], "one": []}
    for _ in range(K):                                  # interleaved legs
        ev = [mk() for _ in range(3)]
        ev[0].record(); ep.forward(xs, ys); ev[1].record(); ep.backward(dys, eg); ev[2].record()
        legs["ep"].append(ev)
        ev = [mk() for _ in range(3)]
        ev[0].record(); one.forward(xw, yw); ev[1].record(); one.backward(xw, dyw, og); ev[2].record()
        legs["one"].append(ev)
    torch.cuda.synchronize()
    fwd = {k: statistics.mean(e[0].elapsed_time(e[1]) for e in v) for k, v in legs.items()}
    step = {k: statistics.mean(e[0].elapsed_time(e[2]) for e in v) for k, v in legs.items()}
    status = one.status()
    n = W * wl.T
    out = {"workload": f"{wl.name}: {W} ranks x {wl.T} tokens, E={wl.E} experts ({wl.E // W} per rank), "
                       f"top-{wl.k}, H={wl.H}, I={wl.I}, {wl.S} shared, BF16, all ranks on one GPU",
           "world": W, "tokens_per_rank": wl.T,
           "fwd_ms": fwd["ep"], "fwd_tokens_per_s": n / (fwd["ep"] / 1e3),
           "step_ms": step["ep"], "step_tokens_per_s": n / (step["ep"] / 1e3),
           "one_gpu_fwd_ms": fwd["one"], "one_gpu_step_ms": step["one"],
           "ep_over_one_gpu_fwd_time": fwd["ep"] / fwd["one"],
           "ep_over_one_gpu_step_time": step["ep"] / step["one"],
           "received_rows_per_rank": [int(v) for v in recv],
           "received_rows_max_over_mean": float(recv.max() / max(1e-9, recv.mean())),
           "pulled_rows_per_token": pairs / (W * wl.T),
           "pull_bytes_per_step": int(2 * (pairs + W * wl.T) * wl.H * 2),
           "device_status": status,
           "note": "ranks emulated in stream order on one device; no link crossed"}
    del ep, one, params, xs, ys, dys, eg, og, xw, yw, dyw
    return out


def ep_emulated_mx_run(wl, W, dev, K, warmup):
    """The MXFP8 expert-parallel layer with its W ranks (wl.T tokens each) on this GPU in
    stream order, against the one-GPU MXFP8 layer on the same tokens: the forward
    (inference), and the training step (forward with saved state + MXFP8 backward).
    Each rank quantises its own experts' weights (both copies) and its own x; owners
    pull e4m3 rows and scales of x and the bf16 dy rows.  No link is crossed: the data
    path, not a multi-GPU measurement."""
    import torch
    from mixture_experts_layer_persistent_b200 import (EPWorld, MoELayer, cfg_for, new_rank_grads,
                                                       quantize_mxfp8_weights, quantize_mxfp8_weights_t, synth)
    params = synth.draw_params(wl, dev)
    full = {k: params[k] for k in ("router_w", "e_bias", "logit_bias")}
    for name, sname in (("w_gate_up", "s_gate_up"), ("w_down", "s_down"), ("ws_gate_up", "ss_gate_up"),
                        ("ws_down", "ss_down")):
        full[name], full[sname] = quantize_mxfp8_weights(params[name]) if params.get(name) is not None else (None, None)
    for name in ("w_gate_up", "w_down", "ws_gate_up", "ws_down"):
        t = "wt" + name[1:] if name.startswith("w_") else "wst" + name[2:]
        ts = "st" + name[1:] if name.startswith("w_") else "sst" + name[2:]
        if params.get(name) is not None:
            full[t], full[ts] = quantize_mxfp8_weights_t(params[name])
    el = wl.E // W
    ranks = []
    for r in range(W):
        p = dict(full)
        for name, sname, t, ts in (("w_gate_up", "s_gate_up", "wt_gate_up", "st_gate_up"),
                                   ("w_down", "s_down", "wt_down", "st_down")):
            sl = params[name][r * el:(r + 1) * el].contiguous()
            p[name], p[sname] = quantize_mxfp8_weights(sl)
            p[t], p[ts] = quantize_mxfp8_weights_t(sl)
        ranks.append(p)
    del params
    xs = [synth.draw_x(synth.scaled(wl, seed=wl.seed * 100 + r), dev) for r in range(W)]
    dys = [synth.draw_dy(synth.scaled(wl, seed=wl.seed * 100 + 50 + r), dev) for r in range(W)]
    cfg = cfg_for(wl)
    ep = EPWorld(cfg, W, ranks, device=dev)
    ept = EPWorld(cfg, W, ranks, training=True, device=dev)
    ys = [torch.empty_like(x) for x in xs]
    eg = [new_rank_grads(cfg, W, dev) for _ in range(W)]
    whole = synth.scaled(wl, T=wl.T * W)
    one = MoELayer(cfg_for(whole), full, training=False, device=dev)
    onet = MoELayer(cfg_for(whole), full, training=True, device=dev)
    og = onet.new_grads()
    xw, dyw = torch.cat(xs), torch.cat(dys)
    yw = torch.empty_like(xw)
    for _ in range(warmup):
        ep.forward(xs, ys)
        one.forward(xw, yw)
        ept.forward(xs, ys)
        ept.backward(dys, eg)
        onet.forward(xw, yw)
        onet.backward(xw, dyw, og)
    torch.cuda.synchronize()
    mk = lambda: torch.cuda.Event(enable_timing=True)
    legs = {"ep": [], "one": [], "ep_train": [], "one_train": []}
    for _ in range(K):
        for key, run in (("ep", lambda: ep.forward(xs, ys)), ("one", lambda: one.forward(xw, yw)),
                         ("ep_train", lambda: (ept.forward(xs, ys), ept.backward(dys, eg))),
                         ("one_train", lambda: (onet.forward(xw, yw), onet.backward(xw, dyw, og)))):
            a, b = mk(), mk()
            a.record(); run(); b.record()
            legs[key].append((a, b))
    torch.cuda.synchronize()
    ms = {k: statistics.mean(a.elapsed_time(b) for a, b in v) for k, v in legs.items()}
    n = W * wl.T
    out = {"workload": f"{wl.name}: MXFP8 layer of {W} ranks x {wl.T} tokens, E={wl.E} experts "
                       f"({el} per rank), top-{wl.k}, H={wl.H}, I={wl.I}, {wl.S} shared, all ranks on one GPU",
           "world": W, "tokens_per_rank": wl.T, "fwd_ms": ms["ep"], "fwd_tokens_per_s": n / (ms["ep"] / 1e3),
           "one_gpu_fwd_ms": ms["one"], "ep_over_one_gpu_fwd_time": ms["ep"] / ms["one"],
           "training_step_ms": ms["ep_train"], "training_step_tokens_per_s": n / (ms["ep_train"] / 1e3),
           "one_gpu_training_step_ms": ms["one_train"],
           "ep_over_one_gpu_training_step_time": ms["ep_train"] / ms["one_train"],
           "device_status": onet.status(),
           "note": "ranks emulated in stream order on one device; no link crossed"}
    del ep, ept, one, onet, full, ranks, xs, ys, xw, yw, dys, dyw, eg, og
    return out


def mxfp8_run(wl, dev, K, warmup, world, dist, pk, do_ab=True):
    """Forward tokens/s of the MXFP8 layer (weights quantised once, outside the timed region)."""
    import torch
    from mixture_experts_layer_persistent_b200 import (MoELayer, abi, cfg_for, moe_trace_events,
                                                       quantize_mxfp8_weights_both, synth)
    p = synth.draw_params(wl, dev)
    params = {k: p[k] for k in ("router_w", "e_bias", "logit_bias")}
    master = {}                 # the bf16 weights the training step requantises
    for name, sname, tname, tsname in (("w_gate_up", "s_gate_up", "wt_gate_up", "st_gate_up"),
                                       ("w_down", "s_down", "wt_down", "st_down"),
                                       ("ws_gate_up", "ss_gate_up", "wst_gate_up", "sst_gate_up"),
                                       ("ws_down", "ss_down", "wst_down", "sst_down")):
        if p.get(name) is None:
            params[name] = params[sname] = params[tname] = params[tsname] = None
        else:
            # the forward's copy, and the backward's (transposed, quantised along the other axis)
            params[name], params[sname], params[tname], params[tsname] = quantize_mxfp8_weights_both(p[name])
            master[name] = (p[name], (params[name], params[sname], params[tname], params[tsname]))
    del p
    torch.cuda.empty_cache()
    x = synth.draw_x(wl, dev)
    layer = MoELayer(cfg_for(wl), params, training=False, device=dev)
    y = torch.empty_like(x)
    for _ in range(warmup):
        layer.forward(x, y)
    torch.cuda.synchronize()
    mk = lambda: torch.cuda.Event(enable_timing=True)
    fev = [[mk() for _ in range(abi.MOK_FWD_PHASES + 1)] for _ in range(K)]
    for e in [e for ev in fev for e in ev]:
        e.record()
    start, end = mk(), mk()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    start.record()
    for i in range(K):
        moe_trace_events([e.cuda_event for e in fev[i]], None)
        layer.forward(x, y)
    end.record()
    torch.cuda.synchronize()
    moe_trace_events(None, None)
    status = layer.status()
    t = torch.tensor([start.elapsed_time(end)], device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item()) / K
    if do_ab:
        ab = forward_ab(layer, x, y, K)
        phases = ab["split"]["phases_ms"]          # per-step times: the split schedule's events
    else:
        ab = None
        phases = {n: statistics.mean(fev[i][j].elapsed_time(fev[i][j + 1]) for i in range(K))
                  for j, n in enumerate(FWD_PHASES)}
    flops = 6 * wl.H * wl.I * wl.T * (wl.k + wl.S)
    gemm_ms = max(1e-9, phases["gate_up_gemm"] + phases["down_gemm"])
    del layer
    torch.cuda.empty_cache()
    train = mxfp8_train(wl, params, x, y, dev, K, warmup, world, dist, do_ab, master)
    del params, x, y, master
    torch.cuda.empty_cache()
    # the FP8 denominator: a library FP8 GEMM measured on this GPU in this run; the MXFP8
    # forward loop is short (K forwards of a few ms), so the burst figure is its peak
    fp8 = fp8_peak(dev)
    peak = fp8["burst_tflops"]
    return {"workload": f"{wl.name}: MoE layer fwd MXFP8 (e4m3, 1x32 ue8m0), T={wl.T}, H={wl.H}, E={wl.E}, "
                        f"top-{wl.k}, I={wl.I}, {wl.S} shared",
            "tokens_per_s": wl.T * world / (ms / 1e3), "ms_per_fwd": ms, "split_phases_ms": phases,
            "forward_schedule_ab": ab,
            "layer_tflops": flops / (ms / 1e3) / 1e12,
            "fp8_peak": fp8, "fp8_peak_tflops": peak,
            "fp8_peak_source": "measured burst (torch._scaled_mm e4m3 8192^3 on this GPU)",
            "tc_peak_frac": flops / (ms / 1e3) / 1e12 / peak,
            "tc_peak_frac_of_sustained": flops / (ms / 1e3) / 1e12 / fp8["sustained_tflops"],
            "expert_gemm_tc_peak_frac": flops / (gemm_ms / 1e3) / 1e12 / peak,
            "gate_up_tc_peak_frac": 4 * wl.H * wl.I * wl.T * (wl.k + wl.S) / (max(1e-9, phases["gate_up_gemm"]) / 1e3)
            / 1e12 / peak,
            "device_status": status,
            "training_step": mxfp8_train_roofline(train, wl, peak, pk["bf16"])}


def mxfp8_train(wl, params, x, y, dev, K, warmup, world, dist, do_ab=True, master=None):
    """One MXFP8 training step per iteration: the forward with saved state, then the
    backward (MXFP8 data gradients, BF16 weight gradients), timed together with CUDA
    events under the default schedule; then the backward alone in the interleaved
    schedule A/B (per-step times from the split schedule's events)."""
    import torch
    from mixture_experts_layer_persistent_b200 import MoELayer, abi, cfg_for, moe_trace_events, synth
    layer = MoELayer(cfg_for(wl), params, training=True, device=dev)
    dy = synth.draw_dy(wl, dev)
    grads = layer.new_grads()
    for _ in range(warmup):
        layer.forward(x, y)
        layer.backward(x, dy, grads)
    torch.cuda.synchronize()
    mk = lambda: torch.cuda.Event(enable_timing=True)
    start, end = mk(), mk()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    start.record()
    for i in range(K):
        layer.forward(x, y)
        layer.backward(x, dy, grads)
    end.record()
    torch.cuda.synchronize()
    status = layer.status()
    t = torch.tensor([start.elapsed_time(end)], device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item()) / K
    launches = abi.moe_launch_count()
    # the requantisation after an optimizer step: both MXFP8 copies of every expert
    # weight tensor from its bf16 master, in place (one read of each master)
    from mixture_experts_layer_persistent_b200 import quantize_mxfp8_weights_both
    requant_ms = None
    if master:
        def requant():
            for w, out in master.values():
                quantize_mxfp8_weights_both(w, out)
        requant()
        torch.cuda.synchronize()
        s0, s1 = mk(), mk()
        s0.record()
        for _ in range(K):
            requant()
        s1.record()
        torch.cuda.synchronize()
        requant_ms = s0.elapsed_time(s1) / K
    # the backward alone, per schedule (down_dgrad_gemm includes the quantisation of dy)
    ab = backward_ab(layer, x, dy, grads, K) if do_ab else None
    del layer, grads, dy
    torch.cuda.empty_cache()
    wbytes = sum(w.numel() * 2 for w, _ in master.values()) if master else 0
    out = {"ms_per_step": ms, "tokens_per_s": wl.T * world / (ms / 1e3), "bwd_launches": launches,
           "backward_schedule_ab": ab, "device_status": status}
    if requant_ms is not None:
        # bytes: the bf16 masters read once, both e4m3 copies and their scales written
        nb = wbytes + wbytes + wbytes // 32
        out.update({"requant_ms": requant_ms, "requant_gbs": nb / (requant_ms / 1e3) / 1e9,
                    "tokens_per_s_with_requant": wl.T * world / ((ms + requant_ms) / 1e3)})
    return out


def mxfp8_train_roofline(train, wl, fp8_peak_tf, bf16_peak_tf):
    """The training step against its compute floor: the forward and the two data
    gradients are MXFP8 products (12 H I FLOP per (token, slot) row), the two weight
    gradients BF16 (6 H I); floor = each at its own measured peak."""
    R = wl.T * (wl.k + wl.S)
    mx_flop, bf_flop = 12.0 * wl.H * wl.I * R, 6.0 * wl.H * wl.I * R
    floor_ms = (mx_flop / (fp8_peak_tf * 1e12) + bf_flop / (bf16_peak_tf * 1e12)) * 1e3
    out = dict(train)
    out.update({"workload": f"{wl.name}: MXFP8 training step (fwd + bwd)",
                "tflops": (mx_flop + bf_flop) / (train["ms_per_step"] / 1e3) / 1e12,
                "compute_floor_ms": floor_ms, "frac_of_compute_floor": floor_ms / train["ms_per_step"],
                "floor_peaks": {"fp8_tflops": fp8_peak_tf, "bf16_tflops": bf16_peak_tf}})
    return out


def e2e_run(layer, wl, x, dy, grads, K, world, dist):
    import torch
    from mixture_experts_layer_persistent_b200 import abi
    c = layer.cfg
    hx = x.cpu().pin_memory()
    hdy = dy.cpu().pin_memory()
    hy = torch.empty_like(hx).pin_memory()
    hdx = torch.empty_like(hx).pin_memory()
    n = max(abi.moe_host_scratch_size(c, False), abi.moe_host_scratch_size(c, True),
            abi.moe_host_scratch_size(c, 2))
    scratch = torch.empty(n, dtype=torch.uint8, device=x.device)
    g = abi.moe_grads(None, grads["dw_gate_up"].data_ptr(), grads["dw_down"].data_ptr(),
                      grads["drouter_w"].data_ptr(),
                      grads["dws_gate_up"].data_ptr() if grads["dws_gate_up"] is not None else None,
                      grads["dws_down"].data_ptr() if grads["dws_down"] is not None else None)
    st = layer.stream()

    def step():
        # one call: dy's upload and y's download overlap the passes on a second stream
        abi.moe_step_host(c, hx.data_ptr(), hdy.data_ptr(), layer.cparams, hy.data_ptr(), hdx.data_ptr(),
                          layer.ctx.data_ptr(), layer.ctx_bytes, g, scratch.data_ptr(), n, st)

    def two_calls():
        abi.moe_fwd_host(c, hx.data_ptr(), layer.cparams, hy.data_ptr(), layer.ctx.data_ptr(),
                         layer.ctx_bytes, 1, scratch.data_ptr(), n, st)
        # x stays in the scratch between the two calls (x_host = NULL): uploaded once per step
        abi.moe_bwd_host(c, None, hdy.data_ptr(), layer.cparams, layer.ctx.data_ptr(),
                         layer.ctx_bytes, hdx.data_ptr(), g, scratch.data_ptr(), n, st)

    # pipelined steps: two pinned copies of the inputs alternate, so every step uploads
    # its own x (prefetched by the call before) and dy; each step's y and dx come back
    hxs, hdys = [hx, hx.clone().pin_memory()], [hdy, hdy.clone().pin_memory()]
    na = abi.moe_host_scratch_size(c, 3)
    scratch_a = torch.empty(na, dtype=torch.uint8, device=x.device)
    calls = [0]

    def pipe_step():
        i = calls[0]
        calls[0] += 1
        abi.moe_step_host_async(c, hxs[i & 1].data_ptr(), hxs[(i + 1) & 1].data_ptr(), hdys[i & 1].data_ptr(),
                                layer.cparams, hy.data_ptr(), hdx.data_ptr(), layer.ctx.data_ptr(), layer.ctx_bytes,
                                g, scratch_a.data_ptr(), na, st)

    def timed(fn, drain=None):
        fn()
        if drain:
            drain()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(K):
            fn()
        if drain:
            drain()            # every transfer of the K steps has landed
        e.record()
        torch.cuda.synchronize()
        t = torch.tensor([s.elapsed_time(e)], device=x.device)
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    msp = timed(pipe_step, lambda: abi.moe_step_host_sync(st))
    ms = timed(step)
    ms2 = timed(two_calls)
    nb = wl.T * wl.H * 2
    return {"value": wl.T * world * K / (msp / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": 2 * nb,
            "d2h_bytes_per_step": 2 * nb, "ms_per_step": msp / K,
            "api": "moe_step_host_async (pinned host x, dy -> y, dx per step; the next step's x is uploaded during "
                   "this step's backward, dy during the forward, y during the backward, dx during the next step)",
            "one_call": {"value": wl.T * world * K / (ms / 1e3), "ms_per_step": ms / K,
                         "api": "moe_step_host (dy's upload and y's download overlap the passes; x and dx do not)"},
            "two_calls": {"value": wl.T * world * K / (ms2 / 1e3), "ms_per_step": ms2 / K,
                          "api": "moe_fwd_host + moe_bwd_host (x uploaded once per step)"}}


def reference_arm(args, world):
    """The fp64 oracle on the host cores, bounded token sample per step."""
    import torch
    from mixture_experts_layer_persistent_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    gdev = "cuda" if torch.cuda.is_available() else "cpu"
    params = synth.draw_params(wl, gdev)
    x = synth.draw_x(wl, gdev)
    dy = synth.draw_dy(wl, gdev)
    per_step = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    res = []
    for i in range(args.warmup + args.steps):
        r = oracle_sample(wl, params, x, dy, per_step)
        if i >= args.warmup:
            res.append(r)
    value = statistics.mean(r["value"] for r in res)
    ms = statistics.mean(r["seconds"] for r in res) * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{wl.name} (oracle on a token sample)", "tokens_per_gpu": wl.T},
        "cpu_baseline": {"value": value, "unit": res[0]["unit"], "cores": res[0]["cores"], "kind": "oracle",
                         "sample": res[0]["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
