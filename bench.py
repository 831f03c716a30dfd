#!/usr/bin/env python
"""Benchmark of the MoE FFN layer on B200.

Default workload (decode_t1): one V4-Flash MoE layer (hidden 4096, 256
routed IQ2_XXS/Q2_K experts of intermediate 2048, top-6, one Q8_0 shared
expert) on one token per call, 1000 timed calls rotating over 8 layer
weight sets (8 x 1.84 GB, far beyond the 126 MB L2) after warm-up calls.
A step is one layer call.  Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_t1|decode_t32|prefill_t4096|stack43_t8|stack43_t8_q2q4|
                                decode_t1_q4k|quantize_q2k|quantize_q80|quantize_q4k]

decode_t1_q4k is decode_t1 with Q4_K routed experts (the q2-q4 build's
upgraded layers; 8 rotating weight sets of 3.6 GB); stack43_t8_q2q4 is the
43-layer stack with layers 37-42 in Q4_K.

quantize_q2k / quantize_q80 time the offline encoder (moe_quantize) on
8 x 2048 x 4096 fp32 values per step, in values/s against the HBM roofline.

Multi-GPU (torchrun, one rank per GPU): every rank runs the same workload on
its own GPU with no exchange (replicas; the layer has no data-path
collective), timed between barriers, max over ranks.

--impl reference times the fp64 CPU oracle on the host (rank 0 only; there
is no other implementation of this layer to run): W warm-up and K timed
steps, each an exact fraction of one layer call on the same shapes.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time
from dataclasses import replace

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s and % HBM roofline (decode) / % bf16 TC roofline (prefill)"


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="decode_t1",
                   choices=["decode_t1", "tiny", "decode_t32", "prefill_t4096", "stack43_t8", "stack43_t8_q2q4",
                            "decode_t1_q4k", "quantize_q2k", "quantize_q80", "quantize_q4k"])
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--deterministic", action="store_true",
                   help="layers made with MOE_FLAG_DETERMINISTIC (fixed-order combine above 32 tokens)")
    p.add_argument("--weight-sets", type=int, default=0, help="override the number of rotating weight sets")
    p.add_argument("--sweep", action="store_true",
                   help="time one layer call at T = 1, 2, 4, ..., 256 (skewed bias; one JSON line per T)")
    p.add_argument("--no-extras", action="store_true",
                   help="decode_t1 only: skip the other workloads and the sweep that the default run adds")
    return p.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


NOMINAL_HBM_GBS = 8000.0     # B200 HBM3e, nominal
NOMINAL_BF16_TFLOPS = 2250.0  # B200 dense bf16, nominal


def box_peaks() -> dict:
    """This box's own achievable peaks, measured after the workloads: a
    device-to-device copy of 2 GiB (bytes read + written per second, best of
    10 timed copies after 3 warm-up copies) and a cuBLAS bf16 GEMM of
    8192 x 8192 x 8192 (best of 10 after 3).  Reported beside the roofline,
    whose peak stays the pool's figure."""
    import torch

    out = {"copy": "torch copy_ of 2 GiB on the device, best of 10",
           "gemm": "torch.matmul bf16 8192^3 (cuBLAS), best of 10"}
    try:
        torch.cuda.empty_cache()
        a = torch.empty(1 << 31, dtype=torch.uint8, device="cuda")
        b = torch.empty_like(a)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        best = float("inf")
        for i in range(13):
            ev[0].record()
            b.copy_(a)
            ev[1].record()
            torch.cuda.synchronize()
            if i >= 3:
                best = min(best, ev[0].elapsed_time(ev[1]))
        out["copy_gbs"] = 2 * a.numel() / (best / 1e3) / 1e9
        del a, b
        n = 8192
        x = torch.randn(n, n, device="cuda", dtype=torch.bfloat16)
        y = torch.randn(n, n, device="cuda", dtype=torch.bfloat16)
        best = float("inf")
        for i in range(13):
            ev[0].record()
            torch.matmul(x, y)
            ev[1].record()
            torch.cuda.synchronize()
            if i >= 3:
                best = min(best, ev[0].elapsed_time(ev[1]))
        out["bf16_tflops"] = 2 * n ** 3 / (best / 1e3) / 1e12
        del x, y
        torch.cuda.empty_cache()
    except Exception as ex:  # a failed measurement leaves the line as it is
        out["error"] = str(ex)[:200]
    return out


def add_box_fracs(line: dict, bp: dict) -> None:
    """The roofline's achieved figure also as fractions of this box's
    measured peak and of the nominal one."""
    r = line.get("roofline")
    if not r or "achieved" not in r:
        return
    if r.get("unit") == "GB/s":
        box, nominal = bp.get("copy_gbs"), NOMINAL_HBM_GBS
    elif r.get("unit") == "TFLOP/s":
        box, nominal = bp.get("bf16_tflops"), NOMINAL_BF16_TFLOPS
    else:
        return
    if box:
        r["frac_of_box_peak"] = r["achieved"] / box
    r["frac_of_nominal"] = r["achieved"] / nominal


def load_traffic(workload: str):
    """DRAM bytes per launch of the workload's dominant kernel from the ncu
    capture recorded in profiles/traffic.txt, or None when the kernel's
    sources changed since that capture."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    csrc = os.path.join(ROOT, "bit_moe_expert_sqrtsoftplus_b200", "csrc")
    with open(path) as f:
        for line in f:
            parts = line.split()
            if not parts or parts[0].startswith("#") or parts[0] != workload or len(parts) < 5:
                continue
            h = hashlib.sha256()
            for name in parts[4].split(","):
                with open(os.path.join(csrc, name), "rb") as g:
                    h.update(g.read())
            return int(parts[2]) if h.hexdigest() == parts[3] else None
    return None


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples every 50 ms while the workload runs (warm-up, the
    timed region and the passes after it)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- distributed

def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    """All ranks meet, then this rank's device work drains (on CPU-only
    process groups, as in the gloo tests, only the meeting)."""
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(world, value: float) -> float:
    """The largest of every rank's value (device timings: the slowest rank)."""
    import torch
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, tokens_per_step: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank runs `steps` steps of `tokens_per_step`
    tokens (weak scaling), timed as the slowest rank's `ms_max`."""
    return world * steps * tokens_per_step / (ms_max / 1e3)


# ----------------------------------------------------------------- workloads

def layer_flops(s: synth.LayerShape) -> dict:
    """Multiply-add FLOPs (2 per MAC) of one call at s.tokens tokens."""
    T = s.tokens
    gateup = 2 * T * s.top_k * 2 * s.hidden * s.inter
    down = 2 * T * s.top_k * s.inter * s.hidden
    shared = 2 * T * 3 * s.hidden * s.shared_inter
    router = 2 * T * s.n_experts * s.hidden
    return {"layer": gateup + down + shared + router, "gateup_routed": gateup}


def decode_bytes(s: synth.LayerShape, n_distinct: float) -> dict:
    """Algorithmic bytes: packed weights each selected expert / the shared
    expert contributes once per call, plus the router."""
    gate_up_routed = 2 * s.gate_bytes_per_expert
    shared_gate_up = 2 * s.shared_inter * s.row_bytes(synth.KIND_Q80, s.hidden)
    router = s.n_experts * s.hidden * 2
    experts = n_distinct * s.expert_bytes + s.shared_bytes
    return {"layer": experts + router, "experts": experts, "k2_experts": experts,
            "gate_up": n_distinct * gate_up_routed + shared_gate_up}


def run_ours(args, world, rank):
    import torch

    import bit_moe_expert_sqrtsoftplus_b200 as moe

    s = synth.workload(args.workload)
    T = s.tokens
    nsets = args.weight_sets if args.weight_sets > 0 else s.weight_sets
    layers, weights = [], []
    scratch = None
    for i in range(nsets):
        W = synth.device_layer(0, i, s, q4k=s.q4k)
        cfg = moe.make_config(s.hidden, s.inter, s.n_experts, s.top_k, s.shared_inter, vocab=s.vocab,
                              routed_scaling=s.routed_scaling,
                              flags=moe.MOE_FLAG_DETERMINISTIC if args.deterministic else 0,
                              routed_format=moe.MOE_ROUTED_Q4K if s.q4k else moe.MOE_ROUTED_Q2)
        L = moe.Layer(cfg, W, max_tokens=T, scratch=scratch)
        scratch = L.scratch
        layers.append(L)
        weights.append(W)
    npool = 16 if T <= 64 else 2
    xs = [torch.from_numpy(synth.activations(7 + rank, T, s.hidden, stream=j)).cuda() for j in range(npool)]
    ys = [torch.empty_like(xs[0]) for _ in range(npool)]
    torch.cuda.synchronize()

    def step(i):
        layers[i % nsets].forward(xs[i % npool], None, ys[i % npool])

    # distinct experts per call (for the byte count): from the routing of the pool
    nd = []
    for j in range(min(npool, 8)):
        idx, _ = layers[j % nsets].route(xs[j])
        nd.append(len(np.unique(idx.cpu().numpy())))
    n_distinct = float(np.mean(nd))

    stream = torch.cuda.current_stream()
    clock = ClockSampler(torch.cuda.current_device())
    with clock:
        # warm-up: W steps, continued (untimed) to at least 0.4 s so that the
        # clock samples cover the load right before the timed region
        t_w = time.perf_counter()
        wu = 0
        while wu < args.warmup or time.perf_counter() - t_w < 0.4:
            step(wu)
            wu += 1
            if wu % 64 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        layers[0].poll()
        # pass 1: the timed region
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            step(args.warmup + i)
        e1.record(stream)
        barrier(world)
        ms = e0.elapsed_time(e1)
        # pass 2: the dominant kernel, timed live around each launch
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for i in range(args.steps):
            L = layers[(args.warmup + i) % nsets]
            # torch only reports elapsed time for events it recorded itself; the
            # library re-records the same events around the kernel afterwards
            evs[i][0].record(stream)
            evs[i][1].record(stream)
            moe.moe_set_timing_events(L.handle, *evs[i])
            step(args.warmup + i)
        torch.cuda.synchronize()
        for L in layers:
            moe.moe_set_timing_events(L.handle)
        k2_times = [a.elapsed_time(b) for a, b in evs]
        k2_ms = float(np.mean(k2_times))
        k2_median = float(np.median(k2_times))
        # pass 3: end to end with host buffers (pinned), copies inside the timed
        # region: (a) one stream, copy in / forward / copy out one after the
        # other; (b) as a server runs it: double-buffered device rows, the
        # copies on their own streams, so step i+1's input and step i-1's
        # output cross the host link while step i computes
        hx = [xs[j].cpu().pin_memory() for j in range(npool)]
        hy = [torch.empty_like(hx[0]).pin_memory() for _ in range(npool)]
        dx = torch.empty_like(xs[0])
        dy = torch.empty_like(xs[0])
        barrier(world)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(args.steps):
            j = i % npool
            dx.copy_(hx[j], non_blocking=True)
            layers[i % nsets].forward(dx, None, dy)
            hy[j].copy_(dy, non_blocking=True)
        f1.record(stream)
        barrier(world)
        e2e_serial_ms = f0.elapsed_time(f1)
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        dxs = [torch.empty_like(xs[0]) for _ in range(2)]
        dys = [torch.empty_like(xs[0]) for _ in range(2)]
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def pipelined(n):
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            for i in range(n):
                j, b2 = i % npool, i % 2
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_done[b2])  # step i-2 has read dxs[b2]
                    dxs[b2].copy_(hx[j], non_blocking=True)
                    ev_in[b2].record(s_in)
                stream.wait_event(ev_in[b2])
                if i >= 2:
                    stream.wait_event(ev_out[b2])  # step i-2's output has left dys[b2]
                layers[i % nsets].forward(dxs[b2], None, dys[b2])
                ev_done[b2].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[b2])
                    hy[j].copy_(dys[b2], non_blocking=True)
                    ev_out[b2].record(s_out)
            stream.wait_stream(s_out)

        pipelined(max(3, args.warmup))  # untimed: the copy streams' first use
        torch.cuda.synchronize()
        barrier(world)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        pipelined(args.steps)
        g1.record(stream)
        barrier(world)
        e2e_ms = g0.elapsed_time(g1)
    for L in layers:
        L.poll()

    ms = max_over_ranks(world, ms)
    e2e_ms = max_over_ranks(world, e2e_ms)
    e2e_serial_ms = max_over_ranks(world, e2e_serial_ms)
    k2_ms = max_over_ranks(world, k2_ms)
    k2_median = max_over_ranks(world, k2_median)
    ms_step = ms / args.steps
    value = job_throughput(world, args.steps, T, ms)
    e2e_value = job_throughput(world, args.steps, T, e2e_ms)
    e2e_serial = job_throughput(world, args.steps, T, e2e_serial_ms)
    peaks = load_peaks()
    b = decode_bytes(s, n_distinct)
    achieved = b["k2_experts"] / (k2_ms / 1e3) / 1e9
    layer_gbs = b["experts"] / (ms_step / 1e3) / 1e9
    clocks = clock.summary()
    large = T > moe.MOE_SMALL_T_MAX
    if large:
        fl = layer_flops(s)
        tc_achieved = fl["gateup_routed"] / (k2_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": "routed gate/up grouped GEMM (tcgen05 kind::f16, IQ2_XXS dequantised "
                                             "to f16 in producer warps)",
                "achieved": tc_achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": tc_achieved / peaks["bf16_tflops"], "traffic": load_traffic(args.workload),
                "traffic_unit": "bytes per launch (ncu)", "peak_source": peaks["source"],
                "algorithmic_flops_per_launch": fl["gateup_routed"], "ms_per_launch": k2_ms,
                "median_ms_per_launch": k2_median}
        layer = {"flops_per_call": fl["layer"], "achieved_tflops": fl["layer"] / (ms_step / 1e3) / 1e12,
                 "frac": fl["layer"] / (ms_step / 1e3) / 1e12 / peaks["bf16_tflops"],
                 "frac_of_nominal_2250": fl["layer"] / (ms_step / 1e3) / 1e12 / 2250.0}
    out = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "us_per_layer": ms_step * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        # small-token path: int8 weights x int8 activation limbs, exact int32
        # products, fp32 scaling; batched path: tcgen05 f16 (gate/up) and
        # bf16 (down) operands with fp32 accumulation
        "dtype": "f16/bf16" if large else "s8",
        "data": "synthetic (seeded generator; V4-Flash shapes, random weights)",
        "config": {"workload": f"{args.workload}: V4-Flash MoE layer, T={T} tokens/call, hidden {s.hidden}, "
                               f"{s.n_experts} experts top-{s.top_k}, inter {s.inter}, shared {s.shared_inter}",
                   "tokens_per_call": T, "weight_sets_rotated": nsets,
                   **({"combine": "deterministic (slot rows summed in expert order)"} if args.deterministic else {}),
                   "l2": (f"{nsets} rotating weight set(s) of {s.n_experts * s.expert_bytes / 1e9:.2f} GB "
                          "(inputs far larger than the 126 MB L2)" if s.n_experts * s.expert_bytes > 126e6 else
                          f"one weight set of {(s.n_experts * s.expert_bytes + s.shared_bytes) / 1e6:.2f} MB, "
                          "resident in the 126 MB L2 (a latency figure)"),
                   "parallelism": f"replicas x{world}"},
        "roofline": roof if large else
        {"bound": "hbm", "kernel": ("Q4_K expert kernels (input, gate/up with SwiGLU, down with the combine)" if s.q4k
                                    else "k2_experts (routed IQ2_XXS gate/up and Q2_K down, shared Q8_0 expert)"),
         "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
         "traffic": load_traffic(args.workload), "traffic_unit": "bytes per launch (ncu)",
         "peak_source": peaks["source"],
         "algorithmic_bytes_per_launch": b["k2_experts"], "ms_per_launch": k2_ms, "median_ms_per_launch": k2_median},
        ("layer_tensor" if large else "layer_hbm"): layer if large else
        {"bytes_per_call": b["experts"], "router_bytes": s.n_experts * s.hidden * 2,
         "achieved_gbs": layer_gbs, "frac": layer_gbs / peaks["hbm_gbs"], "distinct_experts_per_call": n_distinct},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * s.hidden * 4,
                "d2h_bytes_per_step": T * s.hidden * 4,
                "copies": "pinned host rows; copy-in and copy-out streams double-buffered against the layer",
                "serial_value": e2e_serial},
        # batched: router (4), permutation (3), input, 4 GEMMs, from 257 tokens
        # the 3 expansions of the shared expert's rows, and with the
        # deterministic flag the slot sum; small-token: k1 and k2, or for Q4_K
        # layers k1, the routing kernel and the 4 expert kernels
        "gpu_launches": ((15 if T >= 257 else 12) + (1 if args.deterministic else 0) if large else
                         6 if s.q4k else 2) * args.steps,
        "clocks": clocks,
    }
    return out


def run_stack(args, world, rank):
    """43 chained layers at T=8 (layers 0-2 hash-routed), x <- x + MoE(RMSNorm(x));
    a step is one pass through the whole stack.  stack43_t8_q2q4 keeps the
    routed experts of its last six layers in Q4_K."""
    import torch

    import bit_moe_expert_sqrtsoftplus_b200 as moe

    s = synth.workload(args.workload)
    T = s.tokens
    cfgs = []
    for l in range(s.layers):
        router = l >= s.hash_layers
        sl = s.layer_shape(l)
        cfgs.append(moe.make_config(s.hidden, s.inter, s.n_experts, s.top_k, s.shared_inter, vocab=s.vocab,
                                    routed_scaling=s.routed_scaling, rms_eps=1e-6,
                                    mode=moe.MOE_ROUTE_ROUTER if router else moe.MOE_ROUTE_HASH,
                                    flags=moe.MOE_FLAG_PRENORM_RESIDUAL,
                                    routed_format=moe.MOE_ROUTED_Q4K if sl.q4k else moe.MOE_ROUTED_Q2))
    # one scratch buffer serves every layer (they run one after another on
    # one stream): the largest any layer asks for (Q4_K layers ask for more)
    sbytes = max(moe.moe_workspace_size(c, T)[1] for c in cfgs)
    scratch = torch.empty(max(sbytes, 16), dtype=torch.uint8, device="cuda")
    layers = []
    for l, cfg in enumerate(cfgs):
        sl = s.layer_shape(l)
        W = synth.device_layer(0, l, sl, router=l >= s.hash_layers, q4k=sl.q4k)
        layers.append(moe.Layer(cfg, W, max_tokens=T, scratch=scratch))
    x0 = torch.from_numpy(synth.activations(7 + rank, T, s.hidden, stream=4242)).cuda()
    tok = torch.from_numpy(synth.token_ids(7 + rank, T, s.vocab, stream=4242)).cuda()
    x = x0.clone()
    # the stacked forward: every layer prefetches the next one's router and
    # shared-expert weights into L2; one CUDA graph replays the whole pass
    stack = moe.Stack(layers, graph=True)

    def step():
        stack.forward(x, tok)

    for _ in range(args.warmup):
        x.copy_(x0)
        step()
    torch.cuda.synchronize()
    # distinct experts per layer for the byte count (routing of the warm-up pass)
    x.copy_(x0)
    nd_bytes = 0.0
    for l, L in enumerate(layers):
        idx, _ = L.route(x, tok)
        nd = len(np.unique(idx.cpu().numpy()))
        nd_bytes += (nd * s.layer_shape(l).expert_bytes + s.shared_bytes +
                     (s.n_experts * s.hidden * 2 if l >= s.hash_layers else 0))
        L.forward(x, tok, y=x)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    clock = ClockSampler(torch.cuda.current_device())
    with clock:
        x.copy_(x0)
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        barrier(world)
        ms = e0.elapsed_time(e1)
        # end to end: x from pinned host memory, the final state back to the host, every step
        hx = x0.cpu().pin_memory()
        hy = torch.empty_like(hx).pin_memory()
        barrier(world)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            x.copy_(hx, non_blocking=True)
            step()
            hy.copy_(x, non_blocking=True)
        f1.record(stream)
        barrier(world)
        e2e_ms = f0.elapsed_time(f1)
    for L in layers:
        L.poll()
    stack.close()
    ms = max_over_ranks(world, ms)
    e2e_ms = max_over_ranks(world, e2e_ms)
    peaks = load_peaks()
    ms_step = ms / args.steps
    gbs = nd_bytes / (ms_step / 1e3) / 1e9
    return {
        "metric": METRIC, "value": job_throughput(world, args.steps, T, ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "us_per_layer": ms_step * 1e3 / s.layers, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s8",
        "data": "synthetic (seeded generator; V4-Flash shapes, random weights)",
        "config": {"workload": f"{args.workload}: {s.layers} chained V4-Flash MoE layers (0-{s.hash_layers - 1} hash-"
                               f"routed), T={T}, x <- x + MoE(RMSNorm(x)); one CUDA graph per pass, each layer "
                               "prefetching the next one's router and shared-expert weights into L2",
                   "l2": f"{s.layers} distinct layer weight sets ({s.layers * s.n_experts * s.expert_bytes / 1e9:.1f} "
                         "GB, far larger than the 126 MB L2)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": (f"whole stack step ({s.layers - s.q4k_layers} x k1/k2"
                                              + (f", {s.q4k_layers} Q4_K layers x 5 launches)" if s.q4k_layers
                                                 else ")")), "achieved": gbs,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": peaks["source"], "algorithmic_bytes_per_step": nd_bytes},
        "e2e": {"value": job_throughput(world, args.steps, T, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": T * s.hidden * 4, "d2h_bytes_per_step": T * s.hidden * 4},
        "gpu_launches": (2 * (s.layers - s.q4k_layers) + 6 * s.q4k_layers) * args.steps,
        "clocks": clock.summary(),
    }


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_rate(s: synth.LayerShape, budget_s: float, max_steps: int, seed: int = 0, threads: int = 1):
    """Tokens/s of the fp64 oracle on layer calls of the workload's shapes
    (weight set 0, inputs resident), as many calls as fit in the budget.
    A call takes a slice of min(T, max(4, threads)) tokens, split over
    `threads` threads (the oracle splits a call's tokens)."""
    import oracle
    W = synth.host_layer(seed, 0, s, q4k=s.q4k)
    Wr, b = W["router_w"], W["bias"]
    T = min(s.tokens, max(4, threads))
    n = 0
    elapsed = 0.0
    while n < max_steps and (n == 0 or elapsed < budget_s):
        x = synth.activations(7, T, s.hidden, stream=100 + n).astype(np.float64)
        a = time.perf_counter()
        idx, w, _ = oracle.route(x, Wr, b, s.top_k, s.routed_scaling)
        oracle.layer(W, s, x, idx, w, threads=threads)
        elapsed += time.perf_counter() - a
        n += 1
    return n * T / elapsed, n, elapsed, T


class OracleSampler:
    """Steps of the fp64 oracle, each an exact 1/F share of one layer call on a
    slice of at most 4 tokens: for every token, E/F router rows, I/F gate and
    up rows and H/F down rows of each selected expert, Is/F gate/up rows and
    H/F down rows of the shared expert; step c takes row block c mod F.  The
    down rows read the SwiGLU outputs of the whole call, computed once at set-up
    (the work of a down row does not depend on their values).  F is sized so a
    step takes about 0.1 s, which keeps a run of K timed and W warm-up steps
    within a few minutes."""

    def __init__(self, s: synth.LayerShape, seed: int = 0):
        import oracle
        self.o, self.s = oracle, s
        self.T = min(s.tokens, 4)
        self.F = 32 * self.T
        assert s.n_experts % self.F == 0 and s.inter % self.F == 0 and s.hidden % self.F == 0
        assert s.shared_inter % self.F == 0
        t0 = time.perf_counter()
        self.x = synth.activations(7, self.T, s.hidden, stream=100).astype(np.float64)
        self.Wr = synth.router_weight(seed, 0, s.n_experts, s.hidden)
        b = synth.bias(seed, 0, s.n_experts, s.skew)
        self.idx, self.w, _ = oracle.route(self.x, self.Wr, b, s.top_k, s.routed_scaling)
        self.W = synth.host_layer(seed, 0, s, experts=np.unique(self.idx), q4k=s.q4k)
        g = self.W["grid"]
        K2, K8 = self.W["gate_kind"], synth.KIND_Q80
        self.h, self.hs = {}, []
        for t in range(self.T):
            xt = self.x[t]
            for e in self.idx[t]:
                a = oracle.matvec(K2, self.W["gate"][e], s.inter, s.hidden, xt, g)
                u = oracle.matvec(K2, self.W["up"][e], s.inter, s.hidden, xt, g)
                self.h[(t, int(e))] = a / (1.0 + np.exp(-a)) * u
            a = oracle.matvec(K8, self.W["sh_gate"], s.shared_inter, s.hidden, xt)
            u = oracle.matvec(K8, self.W["sh_up"], s.shared_inter, s.hidden, xt)
            self.hs.append(a / (1.0 + np.exp(-a)) * u)
        self.y = np.zeros((self.T, s.hidden))
        self.c = 0
        self.setup_s = time.perf_counter() - t0

    def step(self):
        o, s, g = self.o, self.s, self.W["grid"]
        K2, KQ, K8 = self.W["gate_kind"], self.W["down_kind"], synth.KIND_Q80
        c, F = self.c % self.F, self.F
        nE, nI, nH, nS = s.n_experts // F, s.inter // F, s.hidden // F, s.shared_inter // F
        rE, rI, rH, rS = (slice(c * n, (c + 1) * n) for n in (nE, nI, nH, nS))
        for t in range(self.T):
            xt = self.x[t]
            o.router_logits(self.x[t:t + 1], self.Wr[rE])
            for e, wt in zip(self.idx[t], self.w[t]):
                e = int(e)
                a = o.matvec(K2, self.W["gate"][e][rI], nI, s.hidden, xt, g)
                u = o.matvec(K2, self.W["up"][e][rI], nI, s.hidden, xt, g)
                _ = a / (1.0 + np.exp(-a)) * u
                self.y[t, rH] += wt * o.matvec(KQ, self.W["down"][e][rH], nH, s.inter, self.h[(t, e)])
            a = o.matvec(K8, self.W["sh_gate"][rS], nS, s.hidden, xt)
            u = o.matvec(K8, self.W["sh_up"][rS], nS, s.hidden, xt)
            _ = a / (1.0 + np.exp(-a)) * u
            self.y[t, rH] += o.matvec(K8, self.W["sh_down"][rH], nH, s.shared_inter, self.hs[t])
        self.c += 1

    @property
    def tokens_per_step(self) -> float:
        return self.T / self.F


# ------------------------------------------------------- offline encoders

QUANT_ROWS, QUANT_COLS, QUANT_MATS = 2048, 4096, 8  # eight gate-projection-sized matrices per step
QUANT_METRIC = "encoded values/s (offline Q2_K / Q8_0 encoder) and % HBM roofline"


def quant_format(workload: str):
    """(binary format id, values per block, bytes per block) of an encoder workload."""
    return {"quantize_q2k": (1, 256, 84), "quantize_q4k": (2, 256, 144)}.get(workload, (0, 32, 34))


def run_quant(args, world, rank):
    """moe_quantize over 8 x 2048 x 4096 fp32 values (268 MB, beyond the
    126 MB L2) per step; HBM roofline on 4 bytes read plus the block bytes
    written per value."""
    import torch

    import bit_moe_expert_sqrtsoftplus_b200 as moe

    fmt, per, nbytes = quant_format(args.workload)
    n = QUANT_ROWS * QUANT_COLS * QUANT_MATS
    gen = torch.Generator(device="cuda").manual_seed(7 + rank)
    x = torch.randn(n, device="cuda", generator=gen) * 0.02
    out = torch.empty(n // per * nbytes, dtype=torch.uint8, device="cuda")
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(args.warmup):
        moe.moe_quantize(fmt, x, out, bad)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    clock = ClockSampler(torch.cuda.current_device())
    with clock:
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            moe.moe_quantize(fmt, x, out, bad)
        e1.record(stream)
        barrier(world)
        ms = e0.elapsed_time(e1)
        # end to end: pinned host values -> device -> encoder -> pinned host blocks
        hx = x.cpu().pin_memory()
        hy = torch.empty_like(out, device="cpu").pin_memory()
        barrier(world)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            x.copy_(hx, non_blocking=True)
            moe.moe_quantize(fmt, x, out, bad)
            hy.copy_(out, non_blocking=True)
        f1.record(stream)
        barrier(world)
        e2e_ms = f0.elapsed_time(f1)
    if int(bad.item()) != 0:
        raise RuntimeError("the encoder counted non-finite blocks in finite input")
    ms = max_over_ranks(world, ms)
    e2e_ms = max_over_ranks(world, e2e_ms)
    peaks = load_peaks()
    ms_launch = ms / args.steps
    bytes_launch = n * 4 + n // per * nbytes
    gbs = bytes_launch / (ms_launch / 1e3) / 1e9
    return {
        "metric": QUANT_METRIC, "value": job_throughput(world, args.steps, n, ms), "unit": "values/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_launch,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (N(0, 0.02^2) fp32 values from torch's generator)",
        "config": {"workload": f"{args.workload}: {QUANT_MATS} x {QUANT_ROWS} x {QUANT_COLS} fp32 values per step "
                               f"-> {args.workload[len('quantize_'):].upper().replace('Q80', 'Q8_0')} blocks",
                   "l2": f"{n * 4 / 1e6:.0f} MB of input per step, beyond the 126 MB L2",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": f"k_{args.workload}", "achieved": gbs,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                     "traffic": load_traffic(args.workload), "traffic_unit": "bytes per launch (ncu)",
                     "peak_source": peaks["source"], "algorithmic_bytes_per_launch": bytes_launch,
                     "ms_per_launch": ms_launch},
        "e2e": {"value": job_throughput(world, args.steps, n, e2e_ms), "unit": "values/s",
                "h2d_bytes_per_step": n * 4, "d2h_bytes_per_step": n // per * nbytes},
        "gpu_launches": args.steps,
        "clocks": clock.summary(),
    }


def oracle_quant_rate(workload: str, steps: int, warmup: int, values_per_step: int = 1 << 20):
    """Values/s of the oracle's encoder on steps of 2^20 values."""
    import oracle
    fmt = quant_format(workload)[0]
    kind = {0: oracle.KIND_Q80, 1: oracle.KIND_Q2K, 2: oracle.KIND_Q4K}[fmt]
    x = (np.random.default_rng(7).standard_normal(values_per_step) * 0.02).astype(np.float32)
    for _ in range(warmup):
        oracle.quantize(kind, x)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.quantize(kind, x)
    elapsed = time.perf_counter() - t0
    return steps * values_per_step / elapsed, elapsed


def run_reference(args, world, rank):
    if rank != 0:
        return None
    if args.workload.startswith("quantize_"):
        value, elapsed = oracle_quant_rate(args.workload, args.steps, args.warmup)
        sample = (f"{args.steps} steps of 2^20 values through the C oracle's encoder, single thread, "
                  f"{elapsed:.2f} s after {args.warmup} warm-up steps")
        return {"metric": QUANT_METRIC, "value": value, "unit": "values/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": 1e3 * elapsed / max(args.steps, 1), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "impl": "reference", "config": {"workload": f"{args.workload} (2^20 values per step)"},
                "cpu_baseline": {"value": value, "unit": "values/s", "cores": 1, "kind": "oracle", "sample": sample},
                "e2e": {"value": value, "unit": "values/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    s = synth.workload(args.workload)
    smp = OracleSampler(s)
    for _ in range(args.warmup):
        smp.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        smp.step()
    elapsed = time.perf_counter() - t0
    # the stack workload's metric counts tokens through all its layers, which
    # each cost one layer call (the hash layers skip only the small router)
    layers = s.layers
    value = args.steps * smp.tokens_per_step / elapsed / layers
    sample = (f"{args.steps} steps of the fp64 C oracle, single thread, each 1/{smp.F} of a {smp.T}-token layer call "
              f"(router, routed and shared expert row blocks; {args.steps * smp.tokens_per_step:g} tokens' work "
              f"in {elapsed:.1f} s after {args.warmup} warm-up steps and {smp.setup_s:.1f} s of set-up)"
              + (f"; tokens/s through the {layers}-layer stack = one layer's rate / {layers}" if layers > 1 else ""))
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * elapsed / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": f"{args.workload} (same shapes), weights resident on the host",
                       "tokens_per_call": s.tokens, "tokens_per_step": smp.tokens_per_step},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


SWEEP_T = (1, 2, 4, 8, 16, 32, 64, 128, 256)


def run_sweep(args, world, rank):
    """Latency and bandwidth of one layer call against the union of the
    experts its tokens select: V4-Flash shapes with the skewed bias, one
    weight set, T = 1 ... 256 (the small-token path up to 32, twice up to 64,
    the batched path above).  Bytes per call = distinct experts x 7,077,888 + the shared expert
    + the router, the least a call must read."""
    import torch

    import bit_moe_expert_sqrtsoftplus_b200 as moe

    base = synth.workload("decode_t32")
    W = synth.device_layer(0, 0, base)
    cfg = moe.make_config(base.hidden, base.inter, base.n_experts, base.top_k, base.shared_inter,
                          vocab=base.vocab, routed_scaling=base.routed_scaling)
    peaks = load_peaks()
    lines = []
    for T in SWEEP_T:
        L = moe.Layer(cfg, W, max_tokens=T)
        xs = [torch.from_numpy(synth.activations(7 + rank, T, base.hidden, stream=600 + j)).cuda() for j in range(8)]
        ys = [torch.empty_like(x) for x in xs]
        nd = float(np.mean([len(np.unique(L.route(x)[0].cpu().numpy())) for x in xs]))
        for i in range(max(args.warmup, 3)):
            L.forward(xs[i % 8], None, ys[i % 8])
        steps = max(5, min(args.steps, 200))
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(steps):
            L.forward(xs[i % 8], None, ys[i % 8])
        e1.record()
        barrier(world)
        L.poll()
        ms = max_over_ranks(world, e0.elapsed_time(e1)) / steps
        nbytes = nd * base.expert_bytes + base.shared_bytes + base.n_experts * base.hidden * 2
        gbs = nbytes / (ms / 1e3) / 1e9
        lines.append({"sweep_T": T, "path": "small-token" if T <= moe.MOE_SMALL_T_MAX else
                      "small-token, two chunks" if T <= moe.MOE_CHUNKED_T_MAX else "batched",
                      "ms_per_call": ms, "tokens_per_s": job_throughput(world, 1, T, ms),
                      "distinct_experts": nd, "bytes_per_call": nbytes, "achieved_gbs": gbs,
                      "hbm_frac": gbs / peaks["hbm_gbs"], "floor_ms": nbytes / (peaks["hbm_gbs"] * 1e9) * 1e3,
                      "n_gpus": world, "steps": steps})
        del L
    return lines


def cpu_baseline(args, budget: float = 0.0) -> dict:
    """The oracle on a bounded sample of the workload, on the host's cores."""
    budget = budget or args.cpu_seconds
    if args.workload.startswith("quantize_"):
        steps = max(1, int(budget / 0.005))  # about 5 ms per 2^20 values
        value, elapsed = oracle_quant_rate(args.workload, steps, 3)
        return {"value": value, "unit": "values/s", "cores": 1, "kind": "oracle",
                "sample": f"{steps} x 2^20 values through the C oracle's encoder, single thread, {elapsed:.1f} s"}
    s = synth.workload(args.workload)
    stack = s.layers > 1
    if stack:  # one router layer of the stack, with its pre-norm and skew settings
        s = replace(s, layers=1, hash_layers=0, q4k_layers=0)
    threads = min(host_cores(), s.tokens)
    value, n, elapsed, T = oracle_rate(s, budget, 1000, threads=threads)
    why = ("; one thread because the oracle splits a call's tokens over threads and this call has one token"
           if s.tokens == 1 else "")
    out = {"value": value / (synth.workload(args.workload).layers if stack else 1), "unit": "tokens/s",
           "cores": threads, "kind": "oracle",
           "sample": f"{n} layer calls of {T} tokens (the workload's shapes) of the fp64 C oracle on weight set 0, "
                     f"{threads} thread(s), {elapsed:.1f} s{why}"
                     + (f"; tokens/s through the {synth.workload(args.workload).layers}-layer stack = one layer's "
                        f"rate / {synth.workload(args.workload).layers}" if stack else "")}
    return out


EXTRA_WORKLOADS = ("tiny", "decode_t32", "prefill_t4096", "stack43_t8")


def run_extras(args, world, rank):
    """The other configurations of the layer, each measured like the headline
    (its own timed region, dominant-kernel roofline, end-to-end pass, clocks
    and oracle baseline), then the batch sweep."""
    import torch
    out = {}
    for name in EXTRA_WORKLOADS:
        sub = argparse.Namespace(**vars(args))
        sub.workload = name
        sub.weight_sets = 0
        r = run_stack(sub, world, rank) if name.startswith("stack") else run_ours(sub, world, rank)
        torch.cuda.empty_cache()
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            r["cpu_baseline"] = cpu_baseline(sub, budget=args.cpu_seconds / 2)
        for k in ("metric", "n_gpus", "higher_is_better", "scaling", "vs_baseline", "data"):
            r.pop(k, None)
        out[name] = r
    sweep = run_sweep(args, world, rank)
    torch.cuda.empty_cache()
    return out, sweep


def main():
    args = parse()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    world, rank, _ = dist_setup(args)
    if args.sweep:
        for line in run_sweep(args, world, rank):
            if rank == 0:
                print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if args.workload.startswith("quantize_"):
        out = run_quant(args, world, rank)
    elif args.workload.startswith("stack"):
        out = run_stack(args, world, rank)
    else:
        out = run_ours(args, world, rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args)
    if args.workload == "decode_t1" and not args.no_extras:
        extras, sweep = run_extras(args, world, rank)
        out["workloads"] = extras
        out["sweep"] = sweep
        out["gpu_launches_all_workloads"] = out["gpu_launches"] + sum(r["gpu_launches"] for r in extras.values())
    bp = box_peaks()
    out["box_peaks"] = bp
    add_box_fracs(out, bp)
    for r in out.get("workloads", {}).values():
        add_box_fracs(r, bp)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
