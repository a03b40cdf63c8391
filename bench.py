"""Throughput of the DoRA hot path on B200, as a fraction of roofline.

One step = one pass of the whole path over one batch of synthetic input on the
headline module (d_out = d_in = 8192, r = 384, alpha = 768, bf16) with
[4096, 8192] activations:
    factored norm (Gram, fused norm GEMM, finalize with g = m / max(n, eps))
    -> compose forward -> compose backward (d_base, d_lora, dm).

Metric: "norm TFLOP/s + compose GB/s (% of B200 roofline)".  `value` is the
roofline time of the step's work (norm: the slower of its 2 d_out d_in r
FLOPs at the measured bf16 tensor peak and its W0 + A + B bytes at the
measured HBM bandwidth; compose forward / backward: 3 / 5 activation passes at
HBM bandwidth) divided by the measured step time, in percent, summed over
ranks (each rank runs its own module and batch: weak scaling, no collective on
the data path).  The per-part TFLOP/s and GB/s are reported under
"components".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "headline_8192_r384"
METRIC = "norm TFLOP/s + compose GB/s (% of B200 roofline), d=8192 r=384 bf16"
UNIT = "% of B200 roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# --------------------------------------------------------------------------- peaks

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def work_model(d_out, d_in, r, T):
    """Algorithmic work of one step."""
    norm_flops = 2.0 * d_out * d_in * r
    norm_bytes = 2.0 * (d_out * d_in + r * d_in + d_out * r)
    act = 2.0 * T * d_out
    return {"norm_flops": norm_flops, "norm_bytes": norm_bytes,
            "fwd_bytes": 3 * act, "bwd_bytes": 5 * act}


def roofline_times(wm, peaks):
    t_norm = max(wm["norm_flops"] / (peaks["bf16_tflops"] * 1e12),
                 wm["norm_bytes"] / (peaks["hbm_gbs"] * 1e9))
    t_fwd = wm["fwd_bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_bwd = wm["bwd_bytes"] / (peaks["hbm_gbs"] * 1e9)
    return t_norm, t_fwd, t_bwd


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"dora_bench_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(1.0)
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
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        if not sm:
            return None
        loaded = [x for x in sm if mx is None or x > 0.3 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- distributed

def dist_setup(n_gpus: int):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        import torch
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    return rank, world, local, pg


def barrier(pg, local):
    if pg is not None:
        if pg.get_backend() == "nccl":
            pg.barrier(device_ids=[local])
        else:
            pg.barrier()


def max_over_ranks(pg, x: float) -> float:
    if pg is None:
        return x
    import torch
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------- oracle arm

def oracle_step_seconds(H, frac=1.0):
    """Times one step of the fp64 oracle on the host: the dense norm of W0 + sBA
    (with g = m / max(n, eps)), then the compose forward and backward, over
    the leading `frac` of the rows and of the tokens (the whole step when
    frac = 1).  Returns the seconds taken."""
    import oracle
    d_out, T = H["W0"].shape[0], H["base"].shape[0]
    rows = max(1, int(round(frac * d_out)))
    toks = max(1, int(round(frac * T)))
    t0 = time.perf_counter()
    n = oracle.rows_dense_row_norm(H["W0"][:rows], H["A"], H["B"][:rows], H["s"])
    oracle.magnitude_scale(H["m"][:rows], n, H["eps"])
    if rows < d_out:  # the compose reads a norm for every column
        import numpy as np
        n = np.concatenate([n, np.full(d_out - rows, float(np.mean(n)))])
    oracle.compose_fwd(H["base"][:toks], H["lora"][:toks], H["m"], n, H["s"], H["eps"])
    oracle.compose_bwd(H["dy"][:toks], H["base"][:toks], H["lora"][:toks], H["m"], n, H["s"],
                       H["eps"])
    return time.perf_counter() - t0


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([int(i.get("num_threads", 1)) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def host_step_inputs():
    """The headline workload's full inputs on the host in fp64 (bf16-rounded
    values, drawn with the same recipe as the GPU run)."""
    import numpy as np
    from dora_adapter_factored_b200 import synth
    w = synth.WORKLOADS[WORKLOAD]
    W0, A, B = synth.module_weights(w)
    m = synth.magnitude_from_base_rows(w, W0).double().numpy()
    base, lora, dy = synth.activations(w, w.tokens, W0.shape[0])
    f = lambda t: t.double().numpy()
    return {"W0": f(W0), "A": f(A), "B": f(B), "m": m, "base": f(base), "lora": f(lora),
            "dy": f(dy), "s": w.modules[0].s, "eps": synth.eps_for("bf16")}


# Host seconds the oracle arm may spend on its timed and warm-up steps.
ORACLE_BUDGET_S = 150.0


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from dora_adapter_factored_b200 import synth
    w = synth.WORKLOADS[WORKLOAD]
    ms = w.modules[0]
    peaks = load_peaks()
    wm = work_model(ms.d_out, ms.d_in, ms.r, w.tokens)
    t_roof = sum(roofline_times(wm, peaks))
    H = host_step_inputs()
    # Whole steps when the run fits the budget; otherwise every step is the
    # same leading fraction of the rows and tokens (the value then compares
    # that fraction of the roofline work with the time measured for it).
    t_first = oracle_step_seconds(H)
    frac = min(1.0, ORACLE_BUDGET_S / max(1e-9, (args.steps + args.warmup) * t_first))
    for _ in range(max(0, args.warmup - 1)):
        oracle_step_seconds(H, frac)
    ts = [oracle_step_seconds(H, frac) for _ in range(args.steps)]
    t = statistics.mean(ts)
    value = 100.0 * frac * t_roof / t
    if frac >= 1.0:
        sample = (f"whole steps: fp64 dense norm of all {ms.d_out} rows, compose fwd+bwd on all "
                  f"{w.tokens} tokens")
    else:
        sample = (f"each step the leading {frac:.4f} of the {ms.d_out} norm rows and "
                  f"{w.tokens} tokens (a whole step takes {t_first:.2f} s); value against that "
                  "fraction of the roofline work")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w):
    ms = w.modules[0]
    return {"workload": w.key, "d_out": ms.d_out, "d_in": ms.d_in, "r": ms.r, "alpha": ms.alpha,
            "tokens": w.tokens, "storage": "bf16",
            "step": "gram + fused norm GEMM + finalize(g) + compose fwd + compose bwd(dm)",
            "l2": "inputs larger than L2 (W0 134 MB, activations 3 x 64 MB) and 2 rotating input sets"}


# --------------------------------------------------------------------------- GPU arm

def run_gpu(args):
    import torch
    import dora_adapter_factored_b200 as dora
    from dora_adapter_factored_b200 import synth

    rank, world, local, pg = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.WORKLOADS[WORKLOAD]
    ms = w.modules[0]
    d_out, d_in, r, T, s = ms.d_out, ms.d_in, ms.r, w.tokens, ms.s
    eps = synth.eps_for("bf16")
    peaks = load_peaks()
    wm = work_model(d_out, d_in, r, T)
    t_roof_norm, t_roof_fwd, t_roof_bwd = roofline_times(wm, peaks)
    t_roof = t_roof_norm + t_roof_fwd + t_roof_bwd
    stream = torch.cuda.current_stream()

    # Two independent input sets (weights + activations), rotated every step.
    sets = []
    for k in range(2):
        W0, A, B = synth.module_weights(w, device=dev)
        base, lora, dy = synth.activations(w, T, d_out, device=dev, index=k)
        n_tmp, _ = dora.dora_factored_norm(W0, A, B, s)
        m = synth.magnitude_near_unity(w, n_tmp, index=k)  # |g - 1| < 1e-2, as the workload asks
        if k == 1:  # a distinct module for the second set
            W0 = W0.flip(0).contiguous()
            B = B.flip(0).contiguous()
            m = m.flip(0).contiguous()
        sets.append(dict(W0=W0, A=A, B=B, m=m, base=base, lora=lora, dy=dy))
    outs = dict(n=torch.empty(d_out, device=dev), g=torch.empty(d_out, device=dev),
                y=torch.empty(T, d_out, dtype=torch.bfloat16, device=dev),
                d_base=torch.empty(T, d_out, dtype=torch.bfloat16, device=dev),
                d_lora=torch.empty(T, d_out, dtype=torch.bfloat16, device=dev),
                dm=torch.empty(d_out, device=dev))
    ws_norm = torch.empty(dora.dora_factored_norm_workspace_size(d_out, d_in, r, torch.bfloat16),
                          dtype=torch.uint8, device=dev)
    ws_bwd = torch.empty(max(256, dora.dora_compose_bwd_workspace_size(T, d_out, torch.bfloat16)),
                         dtype=torch.uint8, device=dev)

    from cuda.bindings import runtime as cudart

    def mark(ev, graph_events):
        if graph_events:  # an event-record node of the graph being captured
            err, = cudart.cudaEventRecordWithFlags(ev.cuda_event,
                                                   torch.cuda.current_stream().cuda_stream,
                                                   cudart.cudaEventRecordExternal)
            if err != cudart.cudaError_t.cudaSuccess:
                raise RuntimeError(f"cudaEventRecordWithFlags: {err}")
        else:
            ev.record(torch.cuda.current_stream())

    def step(i, ev=None, graph_events=False):
        S_ = sets[i % 2]
        if ev is not None:
            mark(ev["s0"], graph_events)
            dora.dora_set_timing_events(ev["nk0"], ev["nk1"])
        dora.dora_factored_norm(S_["W0"], S_["A"], S_["B"], s, S_["m"], eps, n_out=outs["n"],
                                g_out=outs["g"], ws=ws_norm)
        if ev is not None:
            mark(ev["s1"], graph_events)
            dora.dora_set_timing_events(ev["fk0"], ev["fk1"])
        dora.dora_compose_fwd(S_["base"], S_["lora"], S_["m"], outs["n"], s, eps, y=outs["y"])
        if ev is not None:
            mark(ev["s2"], graph_events)
            dora.dora_set_timing_events(ev["bk0"], ev["bk1"])
        dora.dora_compose_bwd(S_["dy"], S_["base"], S_["lora"], S_["m"], outs["n"], s, eps,
                              d_base=outs["d_base"], d_lora=outs["d_lora"], dm=outs["dm"],
                              ws=ws_bwd)
        if ev is not None:
            mark(ev["s3"], graph_events)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if dora.dora_get_device_status() != 0:
        raise RuntimeError("a kernel reported an error during warm-up")

    def timed(run, steps):
        barrier(pg, local)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(steps):
            run(i)
        b.record(stream)
        torch.cuda.synchronize()
        barrier(pg, local)
        return max_over_ranks(pg, a.elapsed_time(b)) / steps

    # Eager submission through the API, for reference.
    eager_ms = timed(step, min(args.steps, 200))

    # The timed step: one CUDA graph per input set, captured from the same API
    # calls (programmatic launches keep their overlap inside the graph).
    graphs = []
    cap = torch.cuda.Stream()
    kernels_per_step = 0
    for k in range(2):
        g = torch.cuda.CUDAGraph()
        c0 = dora.dora_launch_count()
        with torch.cuda.graph(g, stream=cap):
            step(k)
        kernels_per_step = dora.dora_launch_count() - c0  # our kernels in one step's graph
        graphs.append(g)
    for i in range(args.warmup):
        graphs[i % 2].replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    clocks = ClockSampler(local)
    clocks.start()
    ms_step = timed(lambda i: graphs[i % 2].replay(), args.steps)
    launches = args.steps * kernels_per_step
    clk = clocks.stop()
    if dora.dora_get_device_status() != 0:
        raise RuntimeError("a kernel reported an error in the timed region")

    # Per-call durations: each API call captured K times back to back into a
    # graph (input sets alternating, as in the step), the graph replayed R
    # times between a pair of CUDA events on this stream: the call's time as
    # it runs in a stream of such calls, with the same launch overlap as in
    # the step (so the three add up to about the step time).
    def amortized_s(call, K=10, R=None):
        R = R if R is not None else max(3, min(args.steps, 20))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for i in range(K):
                call(i)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        a_ = torch.cuda.Event(enable_timing=True)
        b_ = torch.cuda.Event(enable_timing=True)
        st_ = torch.cuda.current_stream()
        a_.record(st_)
        for _ in range(R):
            g.replay()
        b_.record(st_)
        torch.cuda.synchronize()
        del g
        return a_.elapsed_time(b_) * 1e-3 / (R * K)

    def norm_call(i):
        S_ = sets[i % 2]
        dora.dora_factored_norm(S_["W0"], S_["A"], S_["B"], s, S_["m"], eps, n_out=outs["n"],
                                g_out=outs["g"], ws=ws_norm)

    def fwd_call(i):
        S_ = sets[i % 2]
        dora.dora_compose_fwd(S_["base"], S_["lora"], S_["m"], outs["n"], s, eps, y=outs["y"])

    def bwd_call(i):
        S_ = sets[i % 2]
        dora.dora_compose_bwd(S_["dy"], S_["base"], S_["lora"], S_["m"], outs["n"], s, eps,
                              d_base=outs["d_base"], d_lora=outs["d_lora"], dm=outs["dm"],
                              ws=ws_bwd)

    t_norm_call = amortized_s(norm_call)
    t_fwd_call = amortized_s(fwd_call)
    t_bwd_call = amortized_s(bwd_call)

    # The fused norm GEMM alone: its CTAs stamp %globaltimer at entry and
    # exit (the library's trace hook); the kernel's span is the last exit
    # less the first entry, from one-call graphs replayed one at a time.
    trace = torch.zeros(16 * 2 * 148, dtype=torch.int64, device=dev)
    dora.dora_set_trace_buffer(trace)
    tgraphs = []
    for k in range(2):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            norm_call(k)
        tgraphs.append(g)
    dora.dora_set_trace_buffer(None)
    spans = []
    for i in range(max(6, min(args.steps, 40)) + 2):
        trace.zero_()
        tgraphs[i % 2].replay()
        torch.cuda.synchronize()
        if i < 2:
            continue
        tr = trace.view(-1, 16).cpu()
        ran = tr[:, 1] > 0
        spans.append(float((tr[ran, 1].max() - tr[ran, 0].min()).item()) * 1e-9)
    del tgraphs
    t_norm_k = statistics.median(spans)
    value = world * 100.0 * t_roof / (ms_step * 1e-3)

    tc_peak, hbm_peak = peaks["bf16_tflops"], peaks["hbm_gbs"]
    kernels = {
        "norm_main_kernel": {"us": t_norm_k * 1e6, "bound": "tensor",
                             "achieved": wm["norm_flops"] / t_norm_k / 1e12, "peak": tc_peak,
                             "unit": "TFLOP/s",
                             "timing": "in-kernel %globaltimer span (first CTA entry to last "
                                       "exit), median of one-call graph replays"},
        "compose_fwd_kernel": {"us": t_fwd_call * 1e6, "bound": "hbm",
                               "achieved": wm["fwd_bytes"] / t_fwd_call / 1e9, "peak": hbm_peak,
                               "unit": "GB/s",
                               "timing": "the call (this one kernel), graph of 10 calls"},
        "compose_bwd_kernel": {"us": t_bwd_call * 1e6, "bound": "hbm",
                               "achieved": wm["bwd_bytes"] / t_bwd_call / 1e9, "peak": hbm_peak,
                               "unit": "GB/s",
                               "timing": "the call (all its kernels), graph of 10 calls"},
    }
    for k in kernels.values():
        k["frac"] = k["achieved"] / k["peak"]
    # The roofline entry is the fused norm GEMM: the kernel with the largest
    # share of the step in the ncu launch list (profiles/), and the one whose
    # TFLOP/s the metric names.
    dominant = "norm_main_kernel"
    dk = kernels[dominant]
    traffic = load_traffic(dominant)
    components = {
        "norm_tflops": wm["norm_flops"] / t_norm_call / 1e12,
        "norm_frac_of_roofline": t_roof_norm / t_norm_call,
        "norm_us": t_norm_call * 1e6,
        "compose_fwd_gbs": wm["fwd_bytes"] / t_fwd_call / 1e9,
        "compose_fwd_frac_of_hbm": wm["fwd_bytes"] / t_fwd_call / 1e9 / hbm_peak,
        "compose_fwd_us": t_fwd_call * 1e6,
        "compose_bwd_gbs": wm["bwd_bytes"] / t_bwd_call / 1e9,
        "compose_bwd_frac_of_hbm": wm["bwd_bytes"] / t_bwd_call / 1e9 / hbm_peak,
        "compose_bwd_us": t_bwd_call * 1e6,
        "calls_sum_us": (t_norm_call + t_fwd_call + t_bwd_call) * 1e6,
        "roofline_us": {"norm": t_roof_norm * 1e6, "compose_fwd": t_roof_fwd * 1e6,
                        "compose_bwd": t_roof_bwd * 1e6},
        "timing": "each call captured 10 times back to back into a graph (input sets "
                  "alternating), replayed; time per call",
        "peaks": f"{peaks['source']}: HBM {hbm_peak} GB/s, bf16 {tc_peak} TFLOP/s (burst)",
    }
    # The norm call (its small counter kernel and the fused kernel) against
    # the >= 60 % of roofline the norm is held to; the compose calls against
    # their >= 75 % of HBM.
    components["targets"] = {
        "norm_call": {"frac": t_roof_norm / t_norm_call, "target": 0.60,
                      "met": t_roof_norm / t_norm_call >= 0.60},
        "compose_fwd_call": {"frac": components["compose_fwd_frac_of_hbm"], "target": 0.75,
                             "met": components["compose_fwd_frac_of_hbm"] >= 0.75},
        "compose_bwd_call": {"frac": components["compose_bwd_frac_of_hbm"], "target": 0.75,
                             "met": components["compose_bwd_frac_of_hbm"] >= 0.75},
    }

    e2e = measure_e2e(args, dora, w, sets[0], s, eps, t_roof, dev, stream, pg, local, world)

    cpu = None
    if rank == 0 and world == 1:
        cpu = measure_cpu_baseline(t_roof)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; bf16 weights and activations, no checkpoint)",
            "config": config_dict(w),
            "roofline": {"kernel": dominant, "bound": dk["bound"], "achieved": dk["achieved"],
                         "peak": dk["peak"], "unit": dk["unit"], "frac": dk["frac"],
                         "traffic": traffic, "peak_source": peaks["source"]},
            "kernels": kernels,
            "components": components,
            "clocks": clk,
            "gpu_launches": int(launches),
            "launch": f"CUDA graph replay of the step's API calls ({kernels_per_step} kernels, "
                      "programmatic dependent launches)",
            "eager_ms_per_step": eager_ms,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()
    return 0


def kernel_source_hash() -> str:
    """sha256 of the CUDA sources, to tell whether stored ncu counters still
    describe the kernels being run."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dora_adapter_factored_b200", "csrc")
    for path in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))):
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode() + b"\0" + f.read())
    return h.hexdigest()


def load_traffic(kernel: str):
    """DRAM bytes (read + write) per launch of `kernel` on this workload, from
    the committed ncu summary profiles/traffic.json -- or None when those
    counters were taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        if t.get("source_sha256") != kernel_source_hash():
            return None
        return t.get(WORKLOAD, {}).get(kernel)
    except Exception:
        return None


def measure_e2e(args, dora, w, S_, s, eps, t_roof, dev, stream, pg, local, world):
    """The same step through the public API with host (pinned) buffers: every
    step copies its inputs host->device and reads its results back.  Copies
    and kernels are pipelined on three streams (PCIe is full duplex): the
    norm starts once W0, A and B have landed while the activations are still
    crossing, y goes back while the backward runs, and the next step's inputs
    cross while this step computes and returns (device buffers alternate
    between two sets)."""
    import torch
    keys_w = ("W0", "A", "B", "m")
    keys_a = ("base", "lora", "dy")
    host = {k: S_[k].cpu().pin_memory() for k in keys_w + keys_a}
    T, d_out = S_["base"].shape
    dev_in = [{k: torch.empty_like(S_[k]) for k in host} for _ in range(2)]

    def outs():
        return dict(n=torch.empty(d_out, device=dev), g=torch.empty(d_out, device=dev),
                    y=torch.empty(T, d_out, dtype=torch.bfloat16, device=dev),
                    d_base=torch.empty(T, d_out, dtype=torch.bfloat16, device=dev),
                    d_lora=torch.empty(T, d_out, dtype=torch.bfloat16, device=dev),
                    dm=torch.empty(d_out, device=dev))
    dev_out = [outs() for _ in range(2)]
    host_out = [{k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in o.items()}
                for o in dev_out]
    ws_norm = [torch.empty(dora.dora_factored_norm_workspace_size(
        S_["W0"].shape[0], S_["W0"].shape[1], S_["A"].shape[0], torch.bfloat16),
        dtype=torch.uint8, device=dev) for _ in range(2)]
    ws_bwd = [torch.empty(max(256, dora.dora_compose_bwd_workspace_size(T, d_out, torch.bfloat16)),
                          dtype=torch.uint8, device=dev) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    done_cmp = [ev(), ev()]   # set k's inputs are free again
    done_out = [ev(), ev()]   # set k's outputs have been read back
    for k in range(2):
        done_cmp[k].record(s_cmp)
        done_out[k].record(s_out)

    def e2e_step(i):
        k = i % 2
        D, O, HO = dev_in[k], dev_out[k], host_out[k]
        ev_w, ev_a, ev_y, ev_b = ev(), ev(), ev(), ev()
        with torch.cuda.stream(s_in):
            s_in.wait_event(done_cmp[k])
            for x in keys_w:
                D[x].copy_(host[x], non_blocking=True)
            ev_w.record(s_in)
            for x in keys_a:
                D[x].copy_(host[x], non_blocking=True)
            ev_a.record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(done_out[k])
            s_cmp.wait_event(ev_w)
            dora.dora_factored_norm(D["W0"], D["A"], D["B"], s, D["m"], eps, n_out=O["n"],
                                    g_out=O["g"], ws=ws_norm[k])
            s_cmp.wait_event(ev_a)
            dora.dora_compose_fwd(D["base"], D["lora"], D["m"], O["n"], s, eps, y=O["y"])
            ev_y.record(s_cmp)
            dora.dora_compose_bwd(D["dy"], D["base"], D["lora"], D["m"], O["n"], s, eps,
                                  d_base=O["d_base"], d_lora=O["d_lora"], dm=O["dm"],
                                  ws=ws_bwd[k])
            ev_b.record(s_cmp)
            done_cmp[k].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_y)
            for x in ("n", "g", "y"):
                HO[x].copy_(O[x], non_blocking=True)
            s_out.wait_event(ev_b)
            for x in ("d_base", "d_lora", "dm"):
                HO[x].copy_(O[x], non_blocking=True)
            done_out[k].record(s_out)

    steps = max(3, min(20, args.steps))
    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(pg, local)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(steps):
        e2e_step(i)
    s_in.wait_stream(s_out)
    b.record(s_in)
    torch.cuda.synchronize()
    barrier(pg, local)
    ms = max_over_ranks(pg, a.elapsed_time(b)) / steps
    return {"value": world * 100.0 * t_roof / (ms * 1e-3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": ms, "steps": steps,
            "pipeline": "H2D / kernels / D2H on three streams, two device buffer sets"}


def measure_cpu_baseline(t_roof):
    """The oracle as it stands on the host cores: whole steps of the same
    workload (the function the reference arm times), about 10-20 s of them."""
    H = host_step_inputs()
    ts = [oracle_step_seconds(H)]
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < 10.0 and len(ts) < 50:
        ts.append(oracle_step_seconds(H))
    ts = ts[1:] if len(ts) > 1 else ts
    t = statistics.mean(ts)
    return {"value": 100.0 * t_roof / t, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": (f"{len(ts)} whole steps (fp64 dense norm of all 8192 rows, compose "
                       f"fwd+bwd on all 4096 tokens), {t:.2f} s per step")}


# --------------------------------------------------------------------------- suite

def _device_time(fn, iters, flush):
    """Median device time (s) of fn(i), each call bracketed by CUDA events on
    the current stream; a write of a buffer larger than L2 runs between calls
    (outside the events), so every call starts with a cold L2."""
    import torch
    st = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(iters)]
    for i in range(iters):
        flush.zero_()
        evs[i][0].record(st)
        fn(i)
        evs[i][1].record(st)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in evs) * 1e-3


def _back_to_back_time(fn, K=10, R=5):
    """Device time (s) per call of fn(i) in a stream of such calls: K calls
    (input sets alternating, the two sets together larger than L2, so each
    call reads its inputs from HBM) captured in a CUDA graph and replayed R
    times between a pair of CUDA events; no L2 flush between calls, so no
    write-back of a flush buffer runs under the call either."""
    import torch
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for i in range(K):
            fn(i)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(R):
        g.replay()
    b.record(st)
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) * 1e-3 / (R * K)


def _oracle_seconds(fn, scale, budget_s=2.0):
    """Mean wall time of the oracle sample fn(), times `scale` (the sample's
    share of the full call), over about budget_s seconds."""
    fn()
    ts = []
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s and len(ts) < 50:
        t1 = time.perf_counter()
        fn()
        ts.append(time.perf_counter() - t1)
    return statistics.mean(ts) * scale, len(ts)


def run_suite(args):
    """One JSON line per workload beyond the headline step, each timed on the
    device against the roofline of its algorithmic work (measured peaks), with
    the oracle timed on a host sample beside it."""
    import numpy as np
    import torch
    import oracle
    import dora_adapter_factored_b200 as dora
    from dora_adapter_factored_b200 import synth
    if int(os.environ.get("WORLD_SIZE", "1")) != 1:
        raise SystemExit("--suite runs on one GPU")
    peaks = load_peaks()
    HBM, TC = peaks["hbm_gbs"] * 1e9, peaks["bf16_tflops"] * 1e12
    dev = torch.device("cuda")
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)  # 256 MB > L2
    eps = synth.eps_for("bf16")
    iters = max(5, min(args.steps, 30))
    cores = blas_threads()

    def emit(name, workload, t_gpu, flops, nbytes, oracle_s=None, sample=None, extra=None,
             t_b2b=None):
        t_roof = max(flops / TC, nbytes / HBM)
        bound = "tensor" if flops / TC >= nbytes / HBM else "hbm"
        line = {"suite": name, "workload": workload, "us": t_gpu * 1e6,
                "roofline_us": t_roof * 1e6, "frac_of_roofline": t_roof / t_gpu, "bound": bound,
                "achieved": (flops / t_gpu / 1e12) if bound == "tensor" else (nbytes / t_gpu / 1e9),
                "peak": peaks["bf16_tflops"] if bound == "tensor" else peaks["hbm_gbs"],
                "unit": "TFLOP/s" if bound == "tensor" else "GB/s",
                "algorithmic": {"flops": flops, "bytes": nbytes}, "l2": "flushed between calls",
                "peak_source": peaks["source"]}
        if oracle_s is not None:
            line["cpu_baseline"] = {"kind": "oracle", "seconds_per_call": oracle_s,
                                    "cores": cores, "sample": sample,
                                    "gpu_speedup": oracle_s / t_gpu}
        if t_b2b is not None:
            line["us_back_to_back"] = t_b2b * 1e6
            line["frac_back_to_back"] = t_roof / t_b2b
        if extra:
            line.update(extra)
        print(json.dumps(line), flush=True)

    def two_sets(w, index=0):
        W0, A, B = synth.module_weights(w, index=index, device=dev)
        return [(W0, A, B), (W0.flip(0).contiguous(), A, B.flip(0).contiguous())]

    # ---- factored norm on each single-module configuration
    for key in ("norm_4096_r64", "headline_8192_r384", "mlp_up_25600x5120_r384"):
        w = synth.WORKLOADS[key]
        ms = w.modules[0]
        sets = two_sets(w)
        n = torch.empty(ms.d_out, device=dev)
        ws = torch.empty(dora.dora_factored_norm_workspace_size(ms.d_out, ms.d_in, ms.r,
                                                               torch.bfloat16),
                         dtype=torch.uint8, device=dev)
        fn = lambda i: dora.dora_factored_norm(*sets[i % 2], ms.s, n_out=n, ws=ws)
        for i in range(3):
            fn(i)
        t = _device_time(fn, iters, flush)
        tb = _back_to_back_time(fn)
        W0h, Ah, Bh = (x.float().cpu().numpy() for x in sets[0])
        rows = 16
        o_s, reps = _oracle_seconds(lambda: oracle.rows_dense_row_norm(
            W0h[:rows].astype(np.float64), Ah.astype(np.float64), Bh[:rows].astype(np.float64),
            ms.s), ms.d_out / rows)
        emit("factored_norm", key, t, 2.0 * ms.d_out * ms.d_in * ms.r,
             2.0 * (ms.d_out * ms.d_in + ms.r * ms.d_in + ms.d_out * ms.r), o_s,
             f"fp64 dense norm of {rows} of {ms.d_out} rows ({reps} repeats), scaled",
             t_b2b=tb if ms.d_out * ms.d_in * 2 * 2 > (126 << 20) else None)
        del sets, ws

    # ---- grouped norm over the 56-module layer stack
    w = synth.WORKLOADS["layer_stack_56"]
    mods = []
    for i, ms in enumerate(w.modules):
        W0, A, B = synth.module_weights(w, index=i, device=dev)
        mods.append(dict(W0=W0, A=A, B=B, s=ms.s, n_out=torch.empty(ms.d_out, device=dev)))
    ws = torch.empty(dora.dora_factored_norm_grouped_workspace_size(mods), dtype=torch.uint8,
                     device=dev)
    fn = lambda i: dora.dora_factored_norm_grouped(mods, ws=ws)
    for i in range(3):
        fn(i)
    t = _device_time(fn, max(5, iters // 3), flush)
    fl = sum(2.0 * m_.d_out * m_.d_in * m_.r for m_ in w.modules)
    by = sum(2.0 * (m_.d_out * m_.d_in + m_.r * m_.d_in + m_.d_out * m_.r) for m_ in w.modules)
    kinds = {}
    for i, m_ in enumerate(w.modules[:7]):
        kinds[i] = m_
    def stack_sample():
        for i, m_ in kinds.items():
            p = mods[i]
            oracle.rows_dense_row_norm(p["W0"][:4].float().cpu().numpy().astype(np.float64),
                                       p["A"].float().cpu().numpy().astype(np.float64),
                                       p["B"][:4].float().cpu().numpy().astype(np.float64), m_.s)
    layer_rows = sum(m_.d_out for m_ in w.modules[:7])
    o_s, reps = _oracle_seconds(stack_sample, (layer_rows / 28.0) * (len(w.modules) / 7), 3.0)
    emit("grouped_norm", "layer_stack_56", t, fl, by, o_s,
         f"fp64 dense norm of 4 rows of each of one layer's 7 modules ({reps} repeats), scaled "
         "to all rows of the 56 modules", {"modules": len(w.modules)})
    del mods, ws

    # ---- compose forward / backward on the MLP up-projection activations
    def acts(T, d_out, seed):
        g = torch.Generator(device=dev).manual_seed(seed)
        a = {k: torch.randn(T, d_out, device=dev, generator=g).bfloat16()
             for k in ("base", "lora", "dy")}
        a["n"] = torch.rand(d_out, device=dev, generator=g) + 1.0
        a["m"] = a["n"] * (1.0 + 0.005 * torch.randn(d_out, device=dev, generator=g))
        return a

    def eager_fwd(a, s):
        nc = a["n"].clamp_min(eps)
        g = a["m"] / nc
        gm1 = (a["m"] - nc) / nc
        b, l = a["base"], a["lora"]
        return b + (gm1.to(b.dtype) * b + (g * s).to(b.dtype) * l)  # 4 elementwise ops

    def eager_bwd(a, s):
        nc = a["n"].clamp_min(eps)
        g = a["m"] / nc
        d = a["dy"]
        db = d * g.to(d.dtype)
        dl = d * (g * s).to(d.dtype)
        dm = (d.float() * (a["base"].float() + s * a["lora"].float())).sum(0) / nc
        return db, dl, dm

    def compose_pair(key, T, d_out, s, label):
        sets = [acts(T, d_out, 11), acts(T, d_out, 12)]
        ws = torch.empty(max(256, dora.dora_compose_bwd_workspace_size(T, d_out, torch.bfloat16)),
                         dtype=torch.uint8, device=dev)
        y = torch.empty(T, d_out, dtype=torch.bfloat16, device=dev)
        db, dl = torch.empty_like(y), torch.empty_like(y)
        dm = torch.empty(d_out, device=dev)
        act = 2.0 * T * d_out
        res = {}
        for direction, fused, eager, passes in (
                ("fwd", lambda i: dora.dora_compose_fwd(sets[i % 2]["base"], sets[i % 2]["lora"],
                                                        sets[i % 2]["m"], sets[i % 2]["n"], s,
                                                        eps, y=y),
                 lambda i: eager_fwd(sets[i % 2], s), 3),
                ("bwd", lambda i: dora.dora_compose_bwd(sets[i % 2]["dy"], sets[i % 2]["base"],
                                                        sets[i % 2]["lora"], sets[i % 2]["m"],
                                                        sets[i % 2]["n"], s, eps, d_base=db,
                                                        d_lora=dl, dm=dm, ws=ws),
                 lambda i: eager_bwd(sets[i % 2], s), 5)):
            for i in range(3):
                fused(i)
                eager(i)
            tf = _device_time(fused, iters, flush)
            te = _device_time(eager, max(5, iters // 3), flush)
            res[direction] = (tf, te, passes)
        return res, act, sets

    res, act, sets = compose_pair("mlp_up", 8192, 25600, 2.0, "C4")
    h = {k: v[:64].float().cpu().numpy().astype(np.float64) for k, v in sets[0].items()
         if k in ("base", "lora", "dy")}
    mh, nh = sets[0]["m"].double().cpu().numpy(), sets[0]["n"].double().cpu().numpy()
    for direction, (tf, te, passes) in res.items():
        if direction == "fwd":
            smp = lambda: oracle.compose_fwd(h["base"], h["lora"], mh, nh, 2.0, eps)
        else:
            smp = lambda: oracle.compose_bwd(h["dy"], h["base"], h["lora"], mh, nh, 2.0, eps)
        o_s, reps = _oracle_seconds(smp, 8192 / 64)
        emit(f"compose_{direction}", "mlp_up [8192, 25600] bf16", tf, 0.0, passes * act, o_s,
             f"fp64 compose {direction} on 64 of 8192 tokens ({reps} repeats), scaled",
             {"eager_torch_us": te * 1e6, "speedup_vs_eager": te / tf})
    del sets

    # ---- training-step variants at the headline activations
    T, d_out, s = 4096, 8192, 2.0
    sets = [acts(T, d_out, 21), acts(T, d_out, 22)]
    for a in sets:
        a["inner"] = torch.empty_like(a["base"])
    y = torch.empty(T, d_out, dtype=torch.bfloat16, device=dev)
    db, dl = torch.empty_like(y), torch.empty_like(y)
    dm = torch.empty(d_out, device=dev)
    ws = torch.empty(dora.dora_compose_bwd_workspace_size(T, d_out, torch.bfloat16),
                     dtype=torch.uint8, device=dev)
    act = 2.0 * T * d_out
    variants = (
        ("compose_fwd_train", 4, lambda i: dora.dora_compose_fwd_train(
            sets[i % 2]["base"], sets[i % 2]["lora"], sets[i % 2]["m"], sets[i % 2]["n"], s, eps,
            y=y, inner=sets[i % 2]["inner"])),
        ("compose_bwd_inner", 4, lambda i: dora.dora_compose_bwd_inner(
            sets[i % 2]["dy"], sets[i % 2]["inner"], sets[i % 2]["m"], sets[i % 2]["n"], s, eps,
            d_base=db, d_lora=dl, dm=dm, ws=ws)),
        ("compose_bwd_frozen", 3, lambda i: dora.dora_compose_bwd_frozen(
            sets[i % 2]["dy"], sets[i % 2]["m"], sets[i % 2]["n"], s, eps, d_base=db, d_lora=dl)),
    )
    hb = {k: v[:64].float().cpu().numpy().astype(np.float64) for k, v in sets[0].items()
          if k in ("base", "lora", "dy")}
    mh, nh = sets[0]["m"].double().cpu().numpy(), sets[0]["n"].double().cpu().numpy()
    samples = {
        "compose_fwd_train": lambda: (oracle.compose_fwd(hb["base"], hb["lora"], mh, nh, s, eps),
                                      oracle.compose_inner(hb["base"], hb["lora"], s)),
        "compose_bwd_inner": lambda: oracle.compose_bwd_from_inner(
            hb["dy"], hb["base"] + s * hb["lora"], mh, nh, s, eps),
        "compose_bwd_frozen": lambda: oracle.compose_bwd_frozen(hb["dy"], mh, nh, s, eps),
    }
    for name, passes, fn in variants:
        for i in range(3):
            fn(i)
        t = _device_time(fn, iters, flush)
        tb = _back_to_back_time(fn)
        o_s, reps = _oracle_seconds(samples[name], T / 64)
        emit(name, "headline [4096, 8192] bf16", t, 0.0, passes * act, o_s,
             f"fp64 on 64 of {T} tokens ({reps} repeats), scaled", t_b2b=tb)
    del sets

    # ---- compose sweep: fused vs eager over the layer-stack shapes
    for d in (1024, 4096, 14336):
        for T in (512, 2048, 8192, 32768):
            res, act, sets = compose_pair("sweep", T, d, 2.0, "C5")
            for direction, (tf, te, passes) in res.items():
                emit(f"compose_sweep_{direction}", f"[{T}, {d}] bf16", tf, 0.0, passes * act,
                     extra={"eager_torch_us": te * 1e6, "speedup_vs_eager": te / tf})
            del sets

    # ---- grouped compose: one decoder layer's 7 modules
    layer = (4096, 1024, 1024, 4096, 14336, 14336, 4096)
    for T in (512, 2048, 8192):
        mods = [acts(T, d, 31 + i) for i, d in enumerate(layer)]
        for a in mods:
            a["y"] = torch.empty_like(a["base"])
            a["d_base"], a["d_lora"] = torch.empty_like(a["base"]), torch.empty_like(a["base"])
            a["dm_out"] = torch.empty(a["base"].shape[1], device=dev)
            a["ws"] = torch.empty(max(256, dora.dora_compose_bwd_workspace_size(
                T, a["base"].shape[1], torch.bfloat16)), dtype=torch.uint8, device=dev)
        fitems = [dict(base=a["base"], lora=a["lora"], m=a["m"], n=a["n"], s=2.0, y=a["y"])
                  for a in mods]
        bitems = [dict(dy=a["dy"], base=a["base"], lora=a["lora"], m=a["m"], n=a["n"], s=2.0,
                       d_base=a["d_base"], d_lora=a["d_lora"], dm=a["dm_out"]) for a in mods]
        gws = torch.empty(max(256, dora.dora_compose_bwd_grouped_workspace_size(bitems)),
                          dtype=torch.uint8, device=dev)
        act = sum(2.0 * T * d for d in layer)
        cases = (
            ("fwd", 3, lambda i: dora.dora_compose_fwd_grouped(fitems, eps),
             lambda i: [dora.dora_compose_fwd(a["base"], a["lora"], a["m"], a["n"], 2.0, eps,
                                              y=a["y"]) for a in mods]),
            ("bwd", 5, lambda i: dora.dora_compose_bwd_grouped(bitems, eps, ws=gws),
             lambda i: [dora.dora_compose_bwd(a["dy"], a["base"], a["lora"], a["m"], a["n"], 2.0,
                                              eps, d_base=a["d_base"], d_lora=a["d_lora"],
                                              dm=a["dm_out"], ws=a["ws"]) for a in mods]),
        )
        for direction, passes, grouped, single in cases:
            for i in range(3):
                grouped(i)
                single(i)
            tg = _device_time(grouped, iters, flush)
            ts_ = _device_time(single, iters, flush)
            emit(f"compose_grouped_{direction}", f"one layer (7 modules) at T={T} bf16", tg, 0.0,
                 passes * act, extra={"seven_calls_us": ts_ * 1e6, "speedup_vs_calls": ts_ / tg})
        del mods

    # ---- merged inference weight
    for key in ("headline_8192_r384", "mlp_up_25600x5120_r384"):
        w = synth.WORKLOADS[key]
        ms = w.modules[0]
        sets = two_sets(w)
        ns = []
        for W0, A, B in sets:
            n_, _ = dora.dora_factored_norm(W0, A, B, ms.s)
            ns.append((n_, n_ * 1.001))
        out = torch.empty_like(sets[0][0])
        ws = torch.empty(dora.dora_merge_weight_workspace_size(ms.d_out, ms.d_in, ms.r),
                         dtype=torch.uint8, device=dev)
        fn = lambda i: dora.dora_merge_weight(*sets[i % 2], ns[i % 2][1], ns[i % 2][0], ms.s, eps,
                                              W_out=out, ws=ws)
        for i in range(3):
            fn(i)
        t = _device_time(fn, iters, flush)
        tb = _back_to_back_time(fn)
        W0h, Ah, Bh = (x.float().cpu().numpy().astype(np.float64) for x in sets[0])
        mh, nh = ns[0][1].double().cpu().numpy(), ns[0][0].double().cpu().numpy()
        rows = 16
        o_s, reps = _oracle_seconds(lambda: oracle.merge_weight_given_norm(
            W0h[:rows], Ah, Bh[:rows], mh[:rows], nh[:rows], ms.s, eps), ms.d_out / rows)
        emit("merge_weight", key, t, 2.0 * ms.d_out * ms.d_in * ms.r,
             2.0 * (2 * ms.d_out * ms.d_in + ms.r * ms.d_in + ms.d_out * ms.r), o_s,
             f"fp64 merge of {rows} of {ms.d_out} rows ({reps} repeats), scaled", t_b2b=tb)
        del sets, ws, out

    # ---- one column shard of the headline module (d_in-sharded norm, 2 ranks)
    w = synth.WORKLOADS["headline_8192_r384"]
    ms = w.modules[0]
    W0, A, B = synth.module_weights(w, device=dev)
    a0, b0 = dora.column_shard(ms.d_in, 0, 2)
    shards = [(W0[:, a0:b0].contiguous(), A[:, a0:b0].contiguous(), B),
              (W0.flip(0)[:, a0:b0].contiguous(), A[:, a0:b0].contiguous(), B.flip(0).contiguous())]
    del W0
    sq = torch.empty(ms.d_out, device=dev)
    ws = torch.empty(dora.dora_factored_norm_workspace_size(ms.d_out, b0 - a0, ms.r,
                                                           torch.bfloat16),
                     dtype=torch.uint8, device=dev)
    fn = lambda i: dora.dora_factored_norm_sq(*shards[i % 2], ms.s, sq_out=sq, ws=ws)
    for i in range(3):
        fn(i)
    t = _device_time(fn, iters, flush)
    tb = _back_to_back_time(fn)
    wd = b0 - a0
    emit("factored_norm_sq_shard", f"headline module, columns [{a0}, {b0}) of 2 shards", t,
         2.0 * ms.d_out * wd * ms.r, 2.0 * (ms.d_out * wd + ms.r * wd + ms.d_out * ms.r),
         t_b2b=tb)
    # ---- stable compose against a naive bf16 evaluation near g = 1 ("Scaling
    # DoRA", section 3: about 3.0x lower peak error at d_out = 8192, d_in =
    # 2048, against fp64); read as [2048, 8192] activations, g = 1 + N(0, 0.0015)
    T, d_out, s = 2048, 8192, 2.0
    g_ = torch.Generator().manual_seed(2048)
    base = torch.randn(T, d_out, generator=g_).bfloat16()
    lora = torch.randn(T, d_out, generator=g_).bfloat16()
    n = torch.empty(d_out).uniform_(0.5, 2.0, generator=g_)
    m = (n.double() * (1.0 + 0.0015 * torch.randn(d_out, generator=g_).double())).float()
    y = dora.dora_compose_fwd(base.to(dev), lora.to(dev), m.to(dev), n.to(dev), s, eps)
    gb = (m.to(dev) / n.to(dev).clamp_min(eps)).bfloat16()
    bd, ld = base.to(dev), lora.to(dev)
    y_naive = bd + ((gb - 1) * bd + (gb * s) * ld)
    torch.cuda.synchronize()
    ref = oracle.compose_fwd(base.double().numpy(), lora.double().numpy(), m.double().numpy(),
                             n.double().numpy(), s, eps)
    e_st = float(np.max(np.abs(y.double().cpu().numpy() - ref)))
    e_nv = float(np.max(np.abs(y_naive.double().cpu().numpy() - ref)))
    print(json.dumps({"suite": "compose_stability", "workload": "[2048, 8192] bf16, g = 1 + N(0, 0.0015)",
                      "peak_abs_err_stable": e_st, "peak_abs_err_naive_bf16": e_nv,
                      "ratio": e_nv / e_st, "pages_ratio": 3.0,
                      "naive": "g rounded to bf16, base + ((g - 1) base + g s lora) in bf16 ops"}),
          flush=True)

    if dora.dora_get_device_status() != 0:
        raise RuntimeError("a kernel reported an error during the suite")
    return 0


# --------------------------------------------------------------------------- single cases

CASES = ("merge", "fwd_train", "bwd_inner", "bwd_frozen", "fwd_grouped", "bwd_grouped",
         "norm_grouped", "norm_sq_shard", "norm")


def run_case(args):
    """One API call, repeated on two rotating input sets (each larger than L2
    except where noted): the headline module / activations for the merge, the
    training and frozen compose variants and the d_in shard; one decoder
    layer (7 modules, [2048, d_out] activations) for the grouped compose;
    one layer's 7 modules for the grouped norm; the headline module's norm
    (with g) for `norm`."""
    import torch
    import dora_adapter_factored_b200 as dora
    from dora_adapter_factored_b200 import synth
    dev = torch.device("cuda")
    eps = synth.eps_for("bf16")
    w = synth.WORKLOADS[WORKLOAD]
    ms = w.modules[0]
    name = args.case
    if name in ("merge", "norm_sq_shard", "norm"):
        W0, A, B = synth.module_weights(w, device=dev)
        sets = [(W0, A, B), (W0.flip(0).contiguous(), A, B.flip(0).contiguous())]
        if name == "norm":
            m = synth.magnitude_from_base_rows(w, W0)
            n_out, g_out = torch.empty_like(m), torch.empty_like(m)
            ws = torch.empty(dora.dora_factored_norm_workspace_size(ms.d_out, ms.d_in, ms.r,
                                                                   torch.bfloat16),
                             dtype=torch.uint8, device=dev)
            fn = lambda i: dora.dora_factored_norm(*sets[i % 2], ms.s, m=m, eps=eps, n_out=n_out,
                                                   g_out=g_out, ws=ws)
        elif name == "merge":
            ns = [dora.dora_factored_norm(*x, ms.s)[0] for x in sets]
            out = torch.empty_like(W0)
            ws = torch.empty(dora.dora_merge_weight_workspace_size(ms.d_out, ms.d_in, ms.r),
                             dtype=torch.uint8, device=dev)
            fn = lambda i: dora.dora_merge_weight(*sets[i % 2], ns[i % 2] * 1.001, ns[i % 2], ms.s,
                                                  eps, W_out=out, ws=ws)
        else:
            a, b = dora.column_shard(ms.d_in, 0, 2)
            sh = [(x[0][:, a:b].contiguous(), x[1][:, a:b].contiguous(), x[2]) for x in sets]
            sq = torch.empty(ms.d_out, device=dev)
            ws = torch.empty(dora.dora_factored_norm_workspace_size(ms.d_out, b - a, ms.r,
                                                                   torch.bfloat16),
                             dtype=torch.uint8, device=dev)
            fn = lambda i: dora.dora_factored_norm_sq(*sh[i % 2], ms.s, sq_out=sq, ws=ws)
    elif name in ("fwd_train", "bwd_inner", "bwd_frozen"):
        T, d = w.tokens, ms.d_out
        sets = []
        for k in range(2):
            base, lora, dy = synth.activations(w, T, d, device=dev, index=k)
            n = torch.full((d,), 1.3, device=dev)
            sets.append(dict(base=base, lora=lora, dy=dy, inner=torch.empty_like(base), n=n,
                             m=n * 1.001))
        y, db, dl = (torch.empty(T, d, dtype=torch.bfloat16, device=dev) for _ in range(3))
        dm = torch.empty(d, device=dev)
        ws = torch.empty(dora.dora_compose_bwd_workspace_size(T, d, torch.bfloat16),
                         dtype=torch.uint8, device=dev)
        if name == "fwd_train":
            fn = lambda i: dora.dora_compose_fwd_train(
                sets[i % 2]["base"], sets[i % 2]["lora"], sets[i % 2]["m"], sets[i % 2]["n"], ms.s,
                eps, y=y, inner=sets[i % 2]["inner"])
        elif name == "bwd_inner":
            fn = lambda i: dora.dora_compose_bwd_inner(
                sets[i % 2]["dy"], sets[i % 2]["base"], sets[i % 2]["m"], sets[i % 2]["n"], ms.s,
                eps, d_base=db, d_lora=dl, dm=dm, ws=ws)
        else:
            fn = lambda i: dora.dora_compose_bwd_frozen(
                sets[i % 2]["dy"], sets[i % 2]["m"], sets[i % 2]["n"], ms.s, eps, d_base=db,
                d_lora=dl)
    elif name in ("fwd_grouped", "bwd_grouped"):
        T = 2048
        groups = []
        for k in range(2):
            items = []
            for i, d in enumerate((4096, 1024, 1024, 4096, 14336, 14336, 4096)):
                g = torch.Generator(device=dev).manual_seed(100 * k + i)
                t = {x: torch.randn(T, d, device=dev, generator=g).bfloat16()
                     for x in ("base", "lora", "dy")}
                n = torch.full((d,), 1.3, device=dev)
                if name == "fwd_grouped":
                    items.append(dict(base=t["base"], lora=t["lora"], m=n * 1.001, n=n, s=2.0,
                                      y=torch.empty_like(t["base"])))
                else:
                    items.append(dict(dy=t["dy"], base=t["base"], lora=t["lora"], m=n * 1.001,
                                      n=n, s=2.0, d_base=torch.empty_like(t["base"]),
                                      d_lora=torch.empty_like(t["base"]),
                                      dm=torch.empty(d, device=dev)))
            groups.append(items)
        if name == "fwd_grouped":
            fn = lambda i: dora.dora_compose_fwd_grouped(groups[i % 2], eps)
        else:
            gws = torch.empty(max(256, dora.dora_compose_bwd_grouped_workspace_size(groups[0])),
                              dtype=torch.uint8, device=dev)
            fn = lambda i: dora.dora_compose_bwd_grouped(groups[i % 2], eps, ws=gws)
    else:  # norm_grouped: one layer (7 modules) of the layer stack
        ws_ = synth.WORKLOADS["layer_stack_56"]
        mods = []
        for i, m_ in enumerate(ws_.modules[:7]):
            W0, A, B = synth.module_weights(ws_, index=i, device=dev)
            mods.append(dict(W0=W0, A=A, B=B, s=m_.s, n_out=torch.empty(m_.d_out, device=dev)))
        ws = torch.empty(dora.dora_factored_norm_grouped_workspace_size(mods), dtype=torch.uint8,
                         device=dev)
        fn = lambda i: dora.dora_factored_norm_grouped(mods, ws=ws)
    for i in range(args.warmup):
        fn(i)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        evs[i][0].record(st)
        fn(i)
        evs[i][1].record(st)
    torch.cuda.synchronize()
    if dora.dora_get_device_status() != 0:
        raise RuntimeError("a kernel reported an error")
    us = statistics.median(a.elapsed_time(b) for a, b in evs) * 1e3
    print(json.dumps({"case": name, "us": us, "steps": args.steps, "warmup": args.warmup}),
          flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--case", default=None, choices=sorted(CASES),
                    help="run one API call on its workload (steps + warmup times) and print "
                         "its median device time: a small, fixed command for kernel profiles")
    ap.add_argument("--suite", action="store_true",
                    help="instead of the headline line: one JSON line per further workload "
                         "(the other configurations and the training / grouped / merge / "
                         "sharded calls), each against its roofline with the oracle beside it")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.steps < 1:
        raise SystemExit("--steps must be at least 1")
    if args.impl == "reference":
        return run_reference(args)
    import torch
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    with torch.cuda.stream(torch.cuda.Stream()):  # a non-default stream for the whole run
        if args.case:
            return run_case(args)
        if args.suite:
            return run_suite(args)
        return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
