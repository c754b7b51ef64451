"""Throughput of the routed MoE FFN forward pass on B200.

One step = one whole layer call (router + top-k, dispatch with X quantisation,
grouped gate/up GEMM with SwiGLU + requantisation, grouped down GEMM with the
routing weight, combine) over one batch of T tokens of the workload.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--tokens T]
                  [--impl ours|reference]

With N > 1 (launched by torchrun) every rank runs its own replica on its own
batch: the tokens of a batch are independent, so the path shards by tokens
with no data-path collective (weak scaling).  Timing: CUDA events on the
launching stream, barrier + synchronize on both sides, max over ranks.
The reference arm times the CPU oracle on a bounded sample of the same batch.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_topk_b200 import synth  # noqa: E402
from mixture_experts_topk_b200.workloads import FMT_NVFP4, WORKLOADS  # noqa: E402

METRIC = "fused MoE layer tokens/s & TFLOP/s on 1 B200; % of FP8/FP4 peak or HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms for the whole
    measurement; each sample keeps the host time it was read at, so that every
    timed region gets the samples that fell inside it."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [c.strip() for c in line.split(",")]))

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0=None, t1=None):
        rows = [r for t, r in self.rows if (t0 is None or t >= t0) and (t1 is None or t <= t1) and len(r) >= 9]
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        for r in rows:
            for n, v in zip(self.REASONS, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


class Regions:
    """Host-time windows of the timed regions, for the clock samples."""

    def __init__(self):
        self.spans = {}

    def __call__(self, name):
        reg = self

        class _Span:
            def __enter__(self):
                torch.cuda.synchronize()
                self.t0 = time.time()

            def __exit__(self, *a):
                torch.cuda.synchronize()
                reg.spans[name] = (self.t0, time.time())
        return _Span()


def kernel_sources_hash():
    """First 16 hex digits of a sha256 over the GEMM sources with comments and
    whitespace removed, so that an edit of comments or layout keeps a capture
    valid and any change of the code itself invalidates it."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in ("gemm.cuh", "gemm_mx.cuh", "common.cuh"):
        src = open(os.path.join(ROOT, "mixture_experts_topk_b200", "csrc", f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update(re.sub(r"\s+", "", src).encode())
    return h.hexdigest()[:16]


def gemm_traffic(workload, T):
    """DRAM bytes per launch of the gate/up GEMM from the committed ncu capture,
    or None when the capture is of another workload or the kernel sources
    changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "grouped_gemm_mixtral8x7b_t4096_traffic.json")
    if workload != "mixtral-8x7b" or T != 4096 or not os.path.exists(p):
        return None
    d = json.load(open(p))
    if kernel_sources_hash() != d["kernel_sources_sha256_16"]:
        return None
    return d["gate_up"]["dram_read_bytes"] + d["gate_up"]["dram_write_bytes"]


def n_proj(wl):
    """Weight matrices per expert: gate, up, down; ReLU^2 experts have no gate."""
    return 2 if wl.act == ACTS["relu2"][0] else 3


def algorithmic_work(wl, T, counts):
    """FLOPs and bytes of one layer call (intermediates excluded)."""
    A = T * wl.k
    npj = n_proj(wl)
    flops_tensor = 2.0 * A * npj * wl.H * wl.I
    flops_router = 2.0 * T * wl.E * wl.H
    touched = int((counts > 0).sum())
    if wl.fmt == FMT_NVFP4:
        per_expert = npj * wl.H * wl.I * (0.5 + 1.0 / 16)
    elif wl.fmt == 0:
        per_expert = npj * wl.H * wl.I + 4 * ((npj - 1) * wl.I + wl.H)
    else:
        per_expert = npj * wl.H * wl.I + 4 * npj * (wl.H // 128) * (wl.I // 128)
    byts = touched * per_expert + wl.E * wl.H * 4 + 2 * T * wl.H * 2
    return flops_tensor, flops_router, byts, touched


def workload_config(wl, act, T, world, counts):
    """The workload a bench line measures; both arms print the same dict (the
    expert histogram is the routing's, identical on both arms)."""
    byts = algorithmic_work(wl, T, counts)[2]
    return {"workload": f"{wl.name} T={T}", "H": wl.H, "I": wl.I, "E": wl.E, "k": wl.k, "activation": act,
            "T_per_gpu": T, "parallelism": f"replicas x{world} (token batches)",
            "l2": "inputs larger than L2 (expert weights %.2f GB per step)" % (byts / 1e9)}


def max_over_ranks(ms, world, device):
    """The largest of the ranks' times (every rank calls it, in the same order)."""
    if world == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, steps, world, ms_max):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms_max * 1e-3)


# gated activations: (act id, alpha, limit); the clamp of 10 is the bounded-SwiGLU
# setting the LightMoE README gives, alpha 1.702 / limit 7 the common SwiGLU-OAI one
ACTS = {"swiglu": (0, 0.0, 0.0), "bounded": (1, 0.0, 10.0), "oai": (2, 1.702, 7.0), "geglu": (3, 0.0, 0.0),
        "reglu": (4, 0.0, 0.0), "relu2": (5, 0.0, 0.0)}
ACT_LABEL = {"swiglu": "SwiGLU", "bounded": "bounded SwiGLU", "oai": "SwiGLU-OAI", "geglu": "GeGLU",
             "reglu": "ReGLU", "relu2": "ReLU2, up only"}


def workload_of(args):
    import dataclasses
    wl = WORKLOADS[args.workload]
    act, alpha, limit = ACTS[args.act]
    return dataclasses.replace(wl, act=act, act_alpha=alpha, act_limit=limit)


def tensor_peaks(wl, pk):
    """Dense tensor peaks of the layer's format in TFLOP/s: (burst, sustained).
    fp8 = 2 x and fp4 = 4 x the measured bf16 figures (nominal ratios)."""
    r = 4.0 if wl.fmt == FMT_NVFP4 else 2.0
    return r * pk["bf16_tflops"], r * pk["bf16_tflops_sustained"]


def launches_per_step(wl, T):
    """Kernels of one moe_forward call: router (logits + top-k; one fused kernel
    for T <= 128 and E <= 32; above 128 tokens with more than 8 experts the
    fixed-point rows, the integer tensor-core pass and the candidate select),
    dispatch (hist, scan, rank, quantise; for T*k <= 1024 one kernel for all
    four with FP8, one for the first three with NVFP4; + amax for NVFP4),
    gate/up, down, combine."""
    if T <= 128:
        route = 1 if wl.E <= 32 else 2
    else:
        route = 3 if wl.E > 8 else 2
    if T * wl.k <= 1024:
        dispatch = 3 if wl.fmt == FMT_NVFP4 else 1     # fused dispatch + quantisation for FP8
    else:
        dispatch = 5 if wl.fmt == FMT_NVFP4 else 4
    return route + dispatch + 3


def measure(native, layer, wl, T, x, wr, bias, args, world, dev, clk, e2e=True, min_region_s=0.5):
    """One workload point: graph-replayed steps, per-kernel events and (when
    e2e) the end-to-end steps fed from pinned host memory.  Every region runs
    at least min_region_s of the same work (untimed pre-roll for the step and
    e2e regions, more iterations for the per-kernel region), so that the
    clock sampler sees it under load; each region reports its own clocks."""
    y = torch.empty(T, wl.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    regions = Regions()

    def call():
        native.moe_forward(layer.h, x, T, wr, bias, layer.packed, y, layer.ws)

    step = call
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    graph = None
    if args.launch == "graph":
        # the layer call, captured once and replayed: the same kernels with the
        # same arguments, minus the host's per-launch cost
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            call()
        torch.cuda.synchronize()
        step = graph.replay
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
    st, msg = layer.status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {msg}")
    counts = layer.region("counts", torch.int32, wl.E).cpu().numpy()
    m_tiles = int(layer.region("num_tiles", torch.int32, 1).item())
    pick = layer.region("pick", torch.int32, 2).cpu().tolist()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(3):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    est_ms = max(ev0.elapsed_time(ev1) / 3, 1e-3)
    fill = max(1, int(math.ceil(min_region_s * 1e3 / est_ms)))

    # ---- device-timed steps (inputs already resident), after an untimed pre-roll
    with regions("steps"):
        for _ in range(fill):
            step()
        barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms_max = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    st, msg = layer.status()
    if st != 0:
        raise RuntimeError(f"device status after the timed steps: {msg}")

    # ---- per-kernel durations (events between the C-ABI calls), averaged over
    # enough calls to fill the region
    ids_t = layer.region("ids", torch.int32, T * wl.k)
    w_t = layer.region("w", torch.float32, T * wl.k)
    names = ["route", "dispatch", "gate_up", "down", "combine"]
    n_k = max(args.steps, fill)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(n_k)]
    with regions("kernels"):
        for s_ in range(n_k):
            e = evs[s_]
            e[0].record(stream)
            native.moe_route(layer.h, x, T, wr, bias, ids_t, w_t, layer.ws)
            e[1].record(stream)
            native.moe_dispatch(layer.h, x, ids_t, T, layer.ws)
            e[2].record(stream)
            native.moe_gate_up(layer.h, layer.packed, T, layer.ws)
            e[3].record(stream)
            native.moe_down(layer.h, layer.packed, w_t, T, layer.ws)
            e[4].record(stream)
            native.moe_combine(layer.h, T, y, layer.ws)
            e[5].record(stream)
    per = {n: sum(evs[s_][i].elapsed_time(evs[s_][i + 1]) for s_ in range(n_k)) / n_k
           for i, n in enumerate(names)}

    out = {"ms_max": ms_max, "counts": counts, "m_tiles": m_tiles, "pick": pick, "kernel_ms": per,
           "graph": graph is not None, "regions": regions}
    if e2e:
        # end to end through the public call with host buffers: every step
        # copies its X from pinned host memory and its Y back to pinned host
        # memory.  Copies run on their own streams, double-buffered, so step i's
        # copies overlap the layer of steps i-1 / i+1 (a serving loop's pipeline).
        x_host = x.cpu().pin_memory()
        y_host = [torch.empty(T, wl.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        x_dev = [torch.empty_like(x) for _ in range(2)]
        y_dev = [torch.empty_like(y) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

        def e2e_steps(n, ev_first=None, ev_last=None):
            done_in = [torch.cuda.Event() for _ in range(n)]
            done_fw = [torch.cuda.Event() for _ in range(n)]
            done_out = [torch.cuda.Event() for _ in range(n)]
            if ev_first is not None:
                ev_first.record(s_in)
            for i in range(n):
                b = i & 1
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(done_fw[i - 2])          # x_dev[b] free again
                    x_dev[b].copy_(x_host, non_blocking=True)
                    done_in[i].record(s_in)
                stream.wait_event(done_in[i])
                if i >= 2:
                    stream.wait_event(done_out[i - 2])           # y_dev[b] read back already
                native.moe_forward(layer.h, x_dev[b], T, wr, bias, layer.packed, y_dev[b], layer.ws)
                done_fw[i].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(done_fw[i])
                    y_host[b].copy_(y_dev[b], non_blocking=True)
                    done_out[i].record(s_out)
            if ev_last is not None:
                s_out.wait_stream(s_in)
                ev_last.record(s_out)

        e2e_steps(2)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with regions("e2e"):
            e2e_steps(fill)
            torch.cuda.synchronize()
            barrier()
            e2e_steps(args.steps, e0, e1)
            torch.cuda.synchronize()
            barrier()
        out["e2e_ms"] = max_over_ranks(e0.elapsed_time(e1), world, dev)
        out["h2d"] = int(x.numel() * 2)
        out["d2h"] = int(y.numel() * 2)
    del graph
    return out


def region_clocks(clk, regions, ms_of):
    """Per timed region: its median SM clock and its time per step scaled to the
    largest SM clock (ms x median MHz / max MHz), so regions that ran at
    different power-capped clocks can be compared."""
    res = {}
    for name, (t0, t1) in regions.spans.items():
        c = clk.summary(t0, t1)
        ms = ms_of.get(name)
        if ms is not None and c["sm_mhz"] and c["sm_max_mhz"]:
            c["ms_per_step"] = ms
            c["ms_at_max_clock"] = ms * c["sm_mhz"] / c["sm_max_mhz"]
        res[name] = c
    return res


def roofline_numbers(wl, T, counts, step_ms, gu_ms, pk):
    """Layer roofline and the gate/up GEMM's fraction of the tensor peak, both
    against the burst and the sustained measured peaks."""
    fl_t, fl_r, byts, touched = algorithmic_work(wl, T, counts)
    burst, sustained = tensor_peaks(wl, pk)
    simt_peak = 148 * 128 * 2 * pk.get("sm_max_mhz", 1965.0) * 1e6   # fp32 FMA lanes x 2 x max clock

    def t_roof(tp):
        return max(fl_t / (tp * 1e12) + fl_r / simt_peak, byts / (pk["hbm_gbs"] * 1e9)) * 1e3

    gu_flops = 2.0 * T * wl.k * (n_proj(wl) - 1) * wl.H * wl.I
    achieved = gu_flops / (gu_ms * 1e-3) / 1e12
    return {"flops_tensor": fl_t, "flops_router": fl_r, "bytes": byts, "touched": touched,
            "t_roof_ms": t_roof(burst), "frac": t_roof(burst) / step_ms,
            "frac_sustained": t_roof(sustained) / step_ms,
            "bound": "tensor" if fl_t / (burst * 1e12) > byts / (pk["hbm_gbs"] * 1e9) else "hbm",
            "gu_achieved": achieved, "gu_frac": achieved / burst, "gu_frac_sustained": achieved / sustained,
            "burst": burst, "sustained": sustained}


# every (workload, T) point the layer is benchmarked on
SWEEP = [(name, T) for name, wl in WORKLOADS.items() for T in wl.tokens]


def per_workload_sweep(native, args, dev, clk, pk):
    """All (workload, T) points in this invocation: ms/step, layer roofline
    fraction, gate/up fraction and clocks for each."""
    res = []
    for name, wl in WORKLOADS.items():
        d = synth.layer(wl, seed=0, device=dev)
        for T in wl.tokens:
            layer = native.Layer(wl, d, max_T=T, device=dev)
            x = synth.tokens(wl, T, seed=0, device=dev)
            m = measure(native, layer, wl, T, x, d["wr"], d["bias"], args, 1, dev, clk, e2e=False,
                        min_region_s=0.25)
            step_ms = m["ms_max"] / args.steps
            rf = roofline_numbers(wl, T, m["counts"], step_ms, m["kernel_ms"]["gate_up"], pk)
            rc = region_clocks(clk, m["regions"], {"steps": step_ms,
                                                   "kernels": sum(m["kernel_ms"].values())})
            res.append({"workload": f"{name} T={T}", "ms_per_step": step_ms, "tokens_per_s": T / (step_ms * 1e-3),
                        "bound": rf["bound"], "layer_roofline_frac": rf["frac"],
                        "layer_roofline_frac_sustained": rf["frac_sustained"],
                        "gate_up_frac": rf["gu_frac"], "gate_up_frac_sustained": rf["gu_frac_sustained"],
                        "kernel_ms": m["kernel_ms"], "touched_experts": rf["touched"],
                        "clocks": rc.get("steps"), "kernel_clocks": rc.get("kernels")})
            layer.close()
            del x
        del d
        torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, local_rank):
    from mixture_experts_topk_b200 import native
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = workload_of(args)
    T = args.tokens
    d = synth.layer(wl, seed=0, device=dev)
    layer = native.Layer(wl, d, max_T=T, device=dev)
    if args.down_bn:
        native.moe_set_tile_config(layer.h, args.down_bn)
    if args.cta_pairs is not None:
        native.moe_set_gemm_options(layer.h, args.cta_pairs)
    if args.gate_up_bn:
        native.moe_set_gate_up_tile(layer.h, args.gate_up_bn)
    wr = d["wr"]
    bias = d["bias"]
    del d                      # the packed copy is all the layer reads
    torch.cuda.empty_cache()
    x = synth.tokens(wl, T, seed=rank, device=dev)
    if args.profile:
        # plain layer calls for a profiler's launch list: --warmup calls, then
        # --steps more, nothing else launched and nothing timed
        y = torch.empty(T, wl.H, dtype=torch.bfloat16, device=dev)
        for _ in range(args.warmup + args.steps):
            native.moe_forward(layer.h, x, T, wr, bias, layer.packed, y, layer.ws)
        torch.cuda.synchronize()
        st, msg = layer.status()
        layer.close()
        if st != 0:
            raise RuntimeError(f"device status: {msg}")
        return {"profile": f"{wl.name} T={T}", "calls": args.warmup + args.steps,
                "launches_per_call": launches_per_step(wl, T)}
    pk, pk_kind = peaks()
    with ClockSampler(local_rank) as clk:
        time.sleep(0.2)
        m = measure(native, layer, wl, T, x, wr, bias, args, world, dev, clk)
        layer.close()
        sweep = None
        if world == 1 and not args.no_per_workload:
            sweep = per_workload_sweep(native, args, dev, clk, pk)
    ms_max = m["ms_max"]
    step_ms = ms_max / args.steps
    per = m["kernel_ms"]
    rf = roofline_numbers(wl, T, m["counts"], step_ms, per["gate_up"], pk)
    e2e_step_ms = m["e2e_ms"] / args.steps
    clocks = region_clocks(clk, m["regions"], {"steps": step_ms, "kernels": sum(per.values()), "e2e": e2e_step_ms})
    out = {
        "metric": METRIC,
        "value": job_throughput(T, args.steps, world, ms_max),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8-e4m3 (fp32 accumulate)" if wl.fmt != FMT_NVFP4 else "nvfp4-e2m1 (fp32 accumulate)",
        "data": "synthetic (seeded; X ~ N(0,1) bf16, weights ~ N(0,1/fan_in) quantised offline)",
        "config": workload_config(wl, args.act, T, world, m["counts"]),
        "run": {"touched_experts": rf["touched"], "m_tiles": m["m_tiles"],
                "launch": "CUDA graph of one moe_forward call, replayed per step" if m["graph"]
                          else "moe_forward per step",
                "down_tile": args.down_bn or {0: 256, 1: 128, 2: 64}[m["pick"][0]],
                "down_tile_source": "fixed" if args.down_bn else "picked from the histogram",
                "down_k_split": m["pick"][1]},
        "tflops": (rf["flops_tensor"] + rf["flops_router"]) * world * args.steps / (ms_max * 1e-3) / 1e12,
        "layer_roofline": {"t_roof_ms": rf["t_roof_ms"], "frac": rf["frac"], "frac_sustained": rf["frac_sustained"],
                           "bound": rf["bound"],
                           "model": "max(tensor FLOPs / P_tensor + router FLOPs / P_fp32, algorithmic bytes / HBM)",
                           "peaks": f"{pk_kind}: P_tensor = (2 fp8 | 4 fp4) x bf16_tflops (burst; frac_sustained: "
                                    "x bf16_tflops_sustained), hbm_gbs; P_fp32 = 148 SMs x 128 lanes x 2 x sm_max_mhz"},
        "roofline": {"kernel": f"grouped_gemm gate/up ({ACT_LABEL[args.act]} + requant epilogue)", "bound": "tensor",
                     "achieved": rf["gu_achieved"], "peak": rf["burst"], "unit": "TFLOP/s",
                     "frac": rf["gu_frac"], "frac_sustained": rf["gu_frac_sustained"],
                     "traffic": gemm_traffic(args.workload, T),
                     "algorithmic_bytes": int(T * wl.k * wl.H + (n_proj(wl) - 1) * wl.I * wl.H * rf["touched"]
                                              + T * wl.k * wl.I),
                     "peak_source": f"{pk_kind} bf16_tflops (burst: the kernel is timed call by call) x "
                                    f"{4 if wl.fmt == FMT_NVFP4 else 2} (nominal fp8:bf16 = 2, fp4:bf16 = 4); "
                                    "frac_sustained uses bf16_tflops_sustained"},
        "kernel_ms": per,
        "e2e": {"value": job_throughput(T, args.steps, world, m["e2e_ms"]), "unit": "tokens/s",
                "h2d_bytes_per_step": m["h2d"], "d2h_bytes_per_step": m["d2h"], "ms_per_step": e2e_step_ms},
        "gpu_launches": launches_per_step(wl, T) * args.steps,
        "clocks": clocks.get("steps"),
        "region_clocks": clocks,
    }
    if sweep is not None:
        out["per_workload"] = sweep
    return out


def cpu_baseline(wl, T, n_sel, seed=0):
    """The oracle as it stands on the host cores: full routing of the T-token
    batch plus the expert MLP and combine of n_sel sampled tokens."""
    import numpy as np
    import oracle
    x = synth.tokens(wl, T, seed=seed)
    d_router = synth.router(wl, seed=0)
    sel = np.linspace(0, T - 1, n_sel).astype(np.int32)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    lg = oracle.router_logits(xb, d_router[0].numpy(), None if d_router[1] is None else d_router[1].numpy())
    ids, _ = oracle.topk(lg, wl.k, wl.score)
    used = sorted(set(ids[sel].reshape(-1).tolist()))
    d = synth.experts(wl, seed=0, experts_subset=used)
    slot = np.full(wl.E, -1, np.int32)
    slot[used] = np.arange(len(used))
    sub = {k_: v[used] for k_, v in d.items()}
    L = oracle.Layer(wl, sub, expert_slot=slot)
    t0 = time.perf_counter()
    L.forward(xb, d_router[0].numpy(), None if d_router[1] is None else d_router[1].numpy(), sel=sel)
    dt = time.perf_counter() - t0
    return {"value": n_sel / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n_sel} of {T} tokens through the expert MLP and combine; router and top-k over all {T}",
            "seconds": dt, "counts": np.bincount(ids.reshape(-1), minlength=wl.E)}


def run_reference(args, world):
    wl = workload_of(args)
    T = args.tokens
    for _ in range(args.warmup):
        cpu_baseline(wl, T, 1)
    vals, secs = [], 0.0
    for _ in range(args.steps):
        r = cpu_baseline(wl, T, args.ref_sample)
        vals.append(r["value"])
        secs += r["seconds"]
    v = args.steps * args.ref_sample / secs
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (fp32 router)",
            "data": "synthetic (seeded)", "config": workload_config(wl, args.act, T, world, r["counts"]),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                             "sample": r["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mixtral-8x7b")
    ap.add_argument("--tokens", type=int, default=4096)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-sample", type=int, default=2,
                    help="tokens per step through the oracle's expert MLP in --impl reference")
    ap.add_argument("--cpu-sample", type=int, default=40,
                    help="tokens through the oracle's expert MLP for cpu_baseline (about 10 s of host work)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the sweep over every (workload, T) point (done at N = 1 only)")
    ap.add_argument("--down-bn", type=int, default=0, help="down GEMM tile width (0 = chosen per call)")
    ap.add_argument("--gate-up-bn", type=int, default=0, choices=[0, 128, 256],
                    help="gated FP8_ROW gate/up tile width (0 = by batch size)")
    ap.add_argument("--cta-pairs", type=int, default=None, choices=[0, 1, 2],
                    help="FP8_ROW GEMMs on CTA pairs: 0 never, 1 by the library's rule (default), 2 always")
    ap.add_argument("--act", default="swiglu", choices=sorted(ACTS),
                    help="gated activation of the expert MLP (bounded: clamp 10; oai: alpha 1.702, limit 7)")
    ap.add_argument("--profile", action="store_true",
                    help="only run --warmup + --steps plain layer calls (for a profiler's launch list)")
    ap.add_argument("--launch", default="graph", choices=["graph", "stream"],
                    help="timed steps replay a CUDA graph of the layer call, or call it directly")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)))
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    out = run_ours(args, rank, world, local_rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline and not args.profile:
            cb = cpu_baseline(workload_of(args), args.tokens, args.cpu_sample)
            cb.pop("seconds")
            cb.pop("counts")
            out["cpu_baseline"] = cb
        print(json.dumps(out))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
