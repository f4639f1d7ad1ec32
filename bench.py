"""Benchmark of the FAVOR+ hot path on B200 (one JSON line on rank 0).

A step is one full pass of the path over one batch of synthetic input:
key pass -> state reduction -> query pass, with Q, K, V resident in HBM.
The headline workload is B=4, H=12, L=16384, d=64, m=256 bf16 with
heavy-tailed key norms.  `value` is whole-job Mtoken*heads/s (units = B*H*L
query tokens x heads, summed over ranks); `e2e` is the same metric through
the host-buffer C-ABI call (host->device copies and the copy back included).
`per_workload` repeats the device measurement on every synthetic workload
(both W variants of the L=131072 one), each with its roofline terms, the
fraction of its own roof that each kernel reaches and the clocks seen.

Multi-GPU: every rank runs its own replica of the workload (the path has no
exchange step), so scaling is weak; time is the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
"""
import argparse
import importlib.util
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)


def _load_workloads():
    """The seeded input generator, loaded by file path: importing the package would map the
    CUDA library, which the oracle arm must not do."""
    spec = importlib.util.spec_from_file_location(
        "favor_bench_workloads", os.path.join(ROOT, "linear_approximate_softmax_b200", "workloads.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


wl = _load_workloads()

METRIC = "FAVOR+ Mtoken*heads/s at L=16K,d=64,m=256 bf16"
UNIT = "Mtoken*heads/s"
DEFAULT_WORKLOAD = "bf16_L16384_heavykeys"
L2_BYTES = 126 * 2**20
STAGES = ["key_pass", "state_reduce", "query_pass"]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=wl.WORKLOAD_ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--batch", type=int, default=None, help="override the workload's B (profiling runs)")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, "fallback"


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of a kernel on a workload,
# from one ncu capture of the kernel as it stands; an entry is removed whenever its kernel changes
# (the bench then reports traffic null until the kernel is captured again).
PROFILED_TRAFFIC = {
    # query_pass_d64_sm100<false> as of "Linformer on the tensor cores end to end ..." (W row stride, per-head W)
    ("bf16_L16384_heavykeys", "query_pass"): 157.76e6,
    # key_pass_pp_sm100<true, false> as of "Key pass: the key norms folded into the projection ..."
    ("bf16_L16384_heavykeys", "key_pass"): 205.39e6,
}

# Per-SM issue rates of one B200 SM per clock, times 148 SMs and the maximum SM clock: the MUFU
# ex2 rate (16 results per clock) bounds the exponentials; the fp32 FMA rate (128 per clock, 2
# flop each) bounds the fp32 path, which runs on CUDA cores.
MUFU_PER_SM_CLK = 16
FFMA_PER_SM_CLK = 128
NUM_SMS = 148


def max_over_ranks(x, dist):
    """The largest of a per-rank float64 tensor over all ranks (in place), as a float."""
    if dist:
        import torch.distributed as td
        td.all_reduce(x, op=td.ReduceOp.MAX)
    return float(x.item())


def whole_job_rate(units_per_rank, world, ms_per_step):
    """Mtoken*heads/s of the whole job: every rank runs its own replica of the workload."""
    return units_per_rank * world / (ms_per_step * 1e-3) / 1e6


def _peaks_per_s(w, peaks):
    clk = peaks["sm_max_mhz"] * 1e6
    mufu = MUFU_PER_SM_CLK * NUM_SMS * clk
    if w.dtype == torch.bfloat16:
        flops, fname = peaks["bf16_tflops"] * 1e12, "bf16 tensor"
    else:
        flops, fname = 2 * FFMA_PER_SM_CLK * NUM_SMS * clk, "fp32 FMA"
    return mufu, flops, fname, peaks["hbm_gbs"] * 1e9


def roofline_terms(w, peaks):
    """Algorithmic work per step and the time each resource needs for it at peak."""
    G = w.H // w.Hkv
    units = w.units
    elt = 2 if w.dtype == torch.bfloat16 else 4
    flops = units * (1 + 1 / G) * (2 * w.d * w.m + 2 * w.m * (w.d + 1))
    exps = units * (1 + 1 / G) * w.m
    hbm = units * elt * (2 * w.d + 2 * w.d / G)
    mufu, fpk, _, hbm_pk = _peaks_per_s(w, peaks)
    return {
        "flops": flops, "exps": exps, "hbm_bytes": hbm,
        "t_tensor_us": flops / fpk * 1e6,
        "t_mufu_us": exps / mufu * 1e6,
        "t_hbm_us": hbm / hbm_pk * 1e6,
        "mufu_peak_gexps": mufu / 1e9,
    }


def stage_work(w, part_bytes=0, state_bytes=0):
    """Algorithmic work of one launch of each kernel: exponentials, flops and DRAM bytes.

    Key pass: m exponentials, 2dm + 2m(d+1) flop and 2d elements (K and V) per key token of each
    kv head; query pass: the same per query token of each query head, reading Q and writing out;
    reduction: it reads the partial states (part_bytes) and writes the state (state_bytes).
    """
    elt = 2 if w.dtype == torch.bfloat16 else 4
    kv_tok = w.B * w.Hkv * w.L
    q_tok = w.B * w.H * w.L
    per_tok = 2 * w.d * w.m + 2 * w.m * (w.d + 1)
    return {
        "key_pass": {"exps": kv_tok * w.m, "flops": kv_tok * per_tok, "bytes": kv_tok * 2 * w.d * elt},
        "state_reduce": {"exps": 0, "flops": 0, "bytes": part_bytes + state_bytes},
        "query_pass": {"exps": q_tok * w.m, "flops": q_tok * per_tok, "bytes": q_tok * 2 * w.d * elt},
    }


def kernel_roofline(w, peaks, stage, ms, scratch=(0, 0)):
    """The fraction of its own binding roof (MUFU, tensor/FMA or HBM) one kernel reaches."""
    mufu, fpk, fname, hbm_pk = _peaks_per_s(w, peaks)
    wk = stage_work(w, *scratch)[stage]
    t = {"alu": wk["exps"] / mufu, "tensor": wk["flops"] / fpk, "hbm": wk["bytes"] / hbm_pk}
    bound = max(t, key=t.get)
    sec = ms * 1e-3
    if bound == "alu":
        ach, pk, unit = wk["exps"] / sec / 1e9, mufu / 1e9, "Gexp/s"
    elif bound == "tensor":
        ach, pk, unit = wk["flops"] / sec / 1e12, fpk / 1e12, "TFLOP/s"
    else:
        ach, pk, unit = wk["bytes"] / sec / 1e9, hbm_pk / 1e9, "GB/s"
    return {"kernel": stage, "bound": bound, "achieved": ach, "peak": pk, "unit": unit, "frac": ach / pk,
            "us": ms * 1e3, "work": wk}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        busy = [x for x in mhz if x > 0.5 * (mx or max(mhz))] or mhz
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(mhz)}


def config_of(w, world):
    """The `config` object of both arms' lines (the same keys and values for the same workload)."""
    return {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "L": w.L, "d": w.d, "m": w.m,
            "orthogonal_W": bool(w.orthogonal[0]), "parallelism": f"replicas x{world}",
            "l2": "input sets rotated so that every step reads inputs that are not in L2"}


def host_cores():
    return os.cpu_count() or 1


def oracle_rate(w, budget_s, max_heads=None, inputs=None, start=0, orthogonal=None):
    """The fp64 oracle, as it stands, on whole (batch, head) pairs of the workload until the budget is spent.

    Input generation and W construction happen before the clock starts; pairs are taken from
    index `start` on (wrapping), so successive samples cover different heads.
    """
    from oracle import favor as ofv
    from threadpoolctl import threadpool_info
    Q, K, V = inputs if inputs is not None else wl.make_inputs(w)
    Wo = ofv.make_features_f32(w.w_seed, w.m, w.d, w.orthogonal[0] if orthogonal is None else orthogonal)
    G = w.H // w.Hkv
    t0 = time.perf_counter()
    heads = 0
    state = {}
    for i in range(w.B * w.H):
        bh = (start + i) % (w.B * w.H)
        b, h = divmod(bh, w.H)
        key = (b, h // G)
        if key not in state:
            state[key], _ = ofv.key_state(K[b, h // G].double().numpy(), V[b, h // G].double().numpy(), Wo)
        ofv.query_output(Q[b, h].double().numpy(), Wo, state[key])
        heads += 1
        if time.perf_counter() - t0 >= budget_s or (max_heads and heads >= max_heads):
            break
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return heads * w.L / dt / 1e6, heads, dt, threads


def run_reference(args, rank, world):
    """--impl reference: the fp64 CPU oracle timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    w = wl.WORKLOADS[args.workload]
    steps = args.steps or 3
    inputs = wl.make_inputs(w)
    for _ in range(min(args.warmup, 1)):
        oracle_rate(w, 0.0, max_heads=1, inputs=inputs)
    total_heads, busy, threads = 0, 0.0, 1
    for k in range(steps):  # each step: one bounded sample of 2 (batch, head) pairs
        r, heads, dt, threads = oracle_rate(w, 1.0, max_heads=2, inputs=inputs, start=2 * k)
        total_heads += heads
        busy += dt
    value = total_heads * w.L / busy / 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": steps,
        "warmup": args.warmup, "ms_per_step": busy / steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(), "blas_threads": threads,
                         "kind": "oracle",
                         "sample": f"{total_heads} (batch, head) pairs x L={w.L}, up to 2 per step, numpy fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


class Bench:
    """One workload resident on the device, with enough input sets that no step reads inputs
    left in L2 by the step before it, and the library's scratch."""

    def __init__(self, fv, w, dev, orthogonal=True):
        self.fv, self.w, self.dev = fv, w, dev
        self.host = wl.make_inputs(w)
        self.Wh = fv.favor_make_features(w.w_seed, w.m, w.d, orthogonal)
        Q, K, V = (t.to(dev) for t in self.host)
        self.W = self.Wh.to(dev)
        set_bytes = (2 * Q.numel() + K.numel() + V.numel()) * Q.element_size()
        self.nsets = max(1, math.ceil(2 * L2_BYTES / set_bytes))
        self.sets = [(Q, K, V, torch.empty_like(Q))]
        for _ in range(self.nsets - 1):
            self.sets.append((Q.clone(), K.clone(), V.clone(), torch.empty_like(Q)))
        self.set_bytes = set_bytes
        self.part = torch.empty(fv.favor_partials_bytes(w.B, w.Hkv, w.L, w.d, w.m), dtype=torch.uint8, device=dev)
        self.state = torch.empty(fv.favor_state_bytes(w.B, w.Hkv, w.d, w.m), dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        self.i = 0

    def step(self, evs=None):
        fv, w, st = self.fv, self.w, self.stream
        Q, K, V, out = self.sets[self.i % self.nsets]
        self.i += 1
        if evs:
            evs[0].record(st)
        fv.favor_key_pass(K, V, self.W, self.part, st)
        if evs:
            evs[1].record(st)
        fv.favor_state_reduce(self.part, self.state, w.B, w.Hkv, w.L, w.d, w.m, st)
        if evs:
            evs[2].record(st)
        fv.favor_query_pass(Q, self.W, self.state, w.Hkv, out, st)
        if evs:
            evs[3].record(st)

    def timed(self, steps, gpu_index, dist=False):
        """ms per step over `steps` plain steps (events only at both ends, so each kernel's set-up
        overlaps the end of the one before it), with the clocks sampled meanwhile."""
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist:
            import torch.distributed as td
            td.barrier()
        torch.cuda.synchronize(self.dev)
        with ClockSampler(gpu_index) as clocks:
            start.record(self.stream)
            for _ in range(steps):
                self.step()
            stop.record(self.stream)
            torch.cuda.synchronize(self.dev)
        if dist:
            td.barrier()
        return start.elapsed_time(stop), clocks.summary()

    def stage_ms(self, n):
        """Each kernel's own duration: events on the launching stream between the stages, in
        steps of their own (the events serialise the kernels)."""
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
        for i in range(n):
            self.step(evs[i])
        torch.cuda.synchronize(self.dev)
        return [sum(e[j].elapsed_time(e[j + 1]) for e in evs) / n for j in range(3)]

    def estimate_ms(self):
        for _ in range(3):
            self.step()
        torch.cuda.synchronize(self.dev)
        t = time.perf_counter()
        for _ in range(5):
            self.step()
        torch.cuda.synchronize(self.dev)
        return (time.perf_counter() - t) / 5 * 1e3


def workload_entry(fv, w, dev, gpu_index, peaks, min_steps, orthogonal=True, min_seconds=0.4):
    """Device measurement of one workload for the `per_workload` list."""
    b = Bench(fv, w, dev, orthogonal)
    est = b.estimate_ms()
    fv.favor_device_check()  # stop at once if a kernel gave up waiting
    steps = max(min_steps, math.ceil(min_seconds * 1e3 / max(est, 1e-3)))
    ms_total, clocks = b.timed(steps, gpu_index)
    ms = ms_total / steps
    stage = b.stage_ms(min(steps, 50))
    rt = roofline_terms(w, peaks)
    bound_us = max(rt["t_tensor_us"], rt["t_mufu_us"], rt["t_hbm_us"])
    scratch = (b.part.numel(), b.state.numel())
    kern = {s: kernel_roofline(w, peaks, s, stage[j], scratch) for j, s in enumerate(STAGES)}
    dom = max(STAGES, key=lambda s: kern[s]["us"])
    entry = {
        "workload": w.name, "orthogonal_W": orthogonal, "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "steps": steps, "ms_per_step": ms, "value": whole_job_rate(w.units, 1, ms), "unit": UNIT,
        "roofline_path": {"t_tensor_us": rt["t_tensor_us"], "t_mufu_us": rt["t_mufu_us"], "t_hbm_us": rt["t_hbm_us"],
                          "bound_us": bound_us, "frac": bound_us / (ms * 1e3)},
        "stage_us": {s: stage[j] * 1e3 for j, s in enumerate(STAGES)},
        "kernels": {s: {k: kern[s][k] for k in ("bound", "achieved", "peak", "unit", "frac")} for s in STAGES},
        "dominant": {"kernel": dom, "bound": kern[dom]["bound"], "frac": kern[dom]["frac"]},
        "input_sets": b.nsets, "clocks": clocks,
    }
    del b
    torch.cuda.empty_cache()
    return entry


DECODE = dict(B=16, H=16, Hkv=1, d=128, m=256)  # the multi-query shape, one token per step


def decode_entry(fv, dev, peaks, steps=400, graph_steps=100, T=256):
    """Incremental decoding: microseconds per step (one new token for each of the B sequences, H query
    heads each) from a resident state, launched one by one and replayed from a CUDA graph, with the
    state's HBM traffic (read and written once per step) as the roofline."""
    c = DECODE
    B, H, Hkv, d, m = c["B"], c["H"], c["Hkv"], c["d"], c["m"]
    g = torch.Generator("cpu").manual_seed(0)
    q = torch.randn(T, B, H, d, generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn(T, B, Hkv, d, generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn(T, B, Hkv, d, generator=g).to(torch.bfloat16).to(dev)
    W = fv.favor_make_features(1, m, d).to(dev)
    state = torch.empty(fv.favor_decode_state_bytes(B, Hkv, d, m), dtype=torch.uint8, device=dev)
    out = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)
    st = torch.cuda.current_stream(dev)
    fv.favor_decode_init(state, B, Hkv, d, m, st)

    def step(t):
        fv.favor_decode_step(q[t % T], k[t % T], v[t % T], W, state, out, st)

    for t in range(20):
        step(t)
    fv.favor_device_check()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for t in range(steps):
        step(t)
    e1.record(st)
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) / steps * 1e3
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=torch.cuda.Stream(dev)):
        for t in range(graph_steps):
            fv.favor_decode_step(q[t % T], k[t % T], v[t % T], W, state, out, torch.cuda.current_stream(dev))
    graph.replay()
    torch.cuda.synchronize(dev)
    e0.record(st)
    for _ in range(4):
        graph.replay()
    e1.record(st)
    torch.cuda.synchronize(dev)
    us_graph = e0.elapsed_time(e1) / (4 * graph_steps) * 1e3
    fv.favor_device_check()
    del graph
    state_bytes = state.numel()
    io = (B * H * d * 2 + 2 * B * Hkv * d) * 2 + m * d * 4
    traffic = 2 * state_bytes + io  # the state read and written once, q, k, v, out and W
    best = min(us, us_graph)
    ach = traffic / (best * 1e-6) / 1e9
    return {"workload": "bf16_decode_mqa_d128_m256", **c, "dtype": "bf16", "us_per_step": us, "us_per_step_graph": us_graph,
            "tokens_per_step": B, "unit": "us per decoded token (all B sequences, H query heads)",
            "roofline": {"bound": "hbm", "bytes_per_step": traffic, "achieved": ach, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": ach / peaks["hbm_gbs"]}}


def relu_entry(fv, dev, peaks, min_seconds=0.4):
    """Kernelizable attention with f = ReLU (favor_attention_relu) on the headline shape: ms per call,
    with the path's roofline (the bf16 tensor-core flops of both passes, or HBM bytes)."""
    w = wl.WORKLOADS["bf16_L16384_heavykeys"]
    Q, K, V = (t.to(dev) for t in wl.make_inputs(w))
    W = fv.favor_make_features(w.w_seed, w.m, w.d).to(dev)
    set_bytes = (2 * Q.numel() + K.numel() + V.numel()) * Q.element_size()
    sets = [(Q, K, V, torch.empty_like(Q))]
    for _ in range(max(1, math.ceil(2 * L2_BYTES / set_bytes)) - 1):
        sets.append((Q.clone(), K.clone(), V.clone(), torch.empty_like(Q)))
    st = torch.cuda.current_stream(dev)

    def call(i):
        q, k, v, o = sets[i % len(sets)]
        fv.favor_attention_relu(q, k, v, W, o, st)

    for i in range(3):
        call(i)
    fv.favor_device_check()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    call(0)
    e1.record(st)
    torch.cuda.synchronize(dev)
    steps = max(5, math.ceil(min_seconds * 1e3 / max(e0.elapsed_time(e1), 1e-3)))
    e0.record(st)
    for i in range(steps):
        call(i)
    e1.record(st)
    torch.cuda.synchronize(dev)
    fv.favor_device_check()
    ms = e0.elapsed_time(e1) / steps
    # bf16 with d = 64 runs on the tensor-core kernels with the map swapped: the same contractions
    # and bytes as the exponential map, no exponentials (so no MUFU term)
    rt = roofline_terms(w, peaks)
    t = {"tensor": rt["t_tensor_us"], "hbm": rt["t_hbm_us"]}
    bound = max(t, key=t.get)
    return {"workload": w.name + "_relu", "feature_map": "relu", "dtype": "bf16", "steps": steps, "ms_per_step": ms,
            "value": whole_job_rate(w.units, 1, ms), "unit": UNIT,
            "roofline_path": {"t_tensor_us": t["tensor"], "t_hbm_us": t["hbm"], "bound": bound,
                              "frac": t[bound] / (ms * 1e3)},
            "input_sets": len(sets)}


def linformer_entry(fv, dev, peaks, kp=256, min_seconds=0.4):
    """Linformer projected attention (favor_linformer) on the headline shape with k = 256 projected
    rows: ms per call, with the path's roofline (the projections' bf16 tensor flops, then the attention
    over k on the tensor cores and the MUFU; or HBM bytes of Q, K, V, out, E and F)."""
    w = wl.WORKLOADS["bf16_L16384_heavykeys"]
    Q, K, V = (t.to(dev) for t in wl.make_inputs(w))
    g = torch.Generator("cpu").manual_seed(5)
    E = (torch.randn(kp, w.L, generator=g) / math.sqrt(w.L)).to(dev)
    F = (torch.randn(kp, w.L, generator=g) / math.sqrt(w.L)).to(dev)
    set_bytes = (2 * Q.numel() + K.numel() + V.numel()) * Q.element_size()
    sets = [(Q, K, V, torch.empty_like(Q))]
    for _ in range(max(1, math.ceil(2 * L2_BYTES / set_bytes)) - 1):
        sets.append((Q.clone(), K.clone(), V.clone(), torch.empty_like(Q)))
    st = torch.cuda.current_stream(dev)

    def call(i):
        q, k, v, o = sets[i % len(sets)]
        fv.favor_linformer(q, k, v, E, F, o, st)

    for i in range(3):
        call(i)
    fv.favor_device_check()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    call(0)
    e1.record(st)
    torch.cuda.synchronize(dev)
    steps = max(5, math.ceil(min_seconds * 1e3 / max(e0.elapsed_time(e1), 1e-3)))
    e0.record(st)
    for i in range(steps):
        call(i)
    e1.record(st)
    torch.cuda.synchronize(dev)
    fv.favor_device_check()
    ms = e0.elapsed_time(e1) / steps
    # the projections E K and F V (bf16 tensor flops) and the attention over the k projected rows
    # (tensor flops and MUFU exponentials) are separate kernels, one after the other, so the path's
    # bound is the projections' time plus the attention's.
    kv_heads, q_heads = w.B * w.Hkv, w.B * w.H
    clk = peaks["sm_max_mhz"] * 1e6
    proj_flops = kv_heads * 2 * (2 * kp * w.L * w.d)
    att_flops = q_heads * w.L * (2 * kp * w.d + 2 * kp * (w.d + 1))
    exps = q_heads * w.L * kp
    hbm = w.units * 2 * (2 * w.d + 2 * w.d * w.Hkv / w.H) + 2 * kp * w.L * 4
    t = {"proj_tensor": proj_flops / (peaks["bf16_tflops"] * 1e12) * 1e6,
         "att_tensor": att_flops / (peaks["bf16_tflops"] * 1e12) * 1e6,
         "att_mufu": exps / (MUFU_PER_SM_CLK * NUM_SMS * clk) * 1e6,
         "hbm": hbm / (peaks["hbm_gbs"] * 1e9) * 1e6}
    bound_us = max(t["proj_tensor"] + max(t["att_tensor"], t["att_mufu"]), t["hbm"])
    return {"workload": w.name + "_linformer_k256", "dtype": "bf16", "kp": kp, "steps": steps, "ms_per_step": ms,
            "value": whole_job_rate(w.units, 1, ms), "unit": UNIT,
            "roofline_path": {"t_proj_tensor_us": t["proj_tensor"], "t_att_tensor_us": t["att_tensor"],
                              "t_att_mufu_us": t["att_mufu"], "t_hbm_us": t["hbm"],
                              "bound": "projections (tensor) + attention (slower of tensor and MUFU)",
                              "bound_us": bound_us, "frac": bound_us / (ms * 1e3)},
            "input_sets": len(sets)}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = world > 1
    if dist:
        import datetime
        import torch.distributed as td
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        td.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    if args.impl == "reference":
        run_reference(args, rank, world)
        if dist:
            import torch.distributed as td
            td.barrier()
            td.destroy_process_group()
        return

    import linear_approximate_softmax_b200 as fv
    # every kernel on this stream is the library's own and no call reads what an earlier call
    # wrote (each step's inputs are written once, before the first step): the first kernel of
    # each call may overlap the end of the previous call (favor.h)
    fv.favor_set_launch_overlap(True)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = wl.WORKLOADS[args.workload]
    if args.batch:
        import dataclasses
        w = dataclasses.replace(w, B=args.batch, name=f"{w.name}_B{args.batch}")
    peaks, peak_src = load_peaks()
    b = Bench(fv, w, dev)
    for _ in range(max(args.warmup, 3)):
        b.step()
    fv.favor_device_check()  # synchronises; stops at once if a kernel gave up waiting
    steps = args.steps
    if steps is None:  # default: about 3 s of timed work
        steps = int(min(5000, max(20, 3.0 / max(b.estimate_ms() * 1e-3, 1e-6))))
    ms_total, clocks = b.timed(steps, local, dist)
    stage_ms = b.stage_ms(min(steps, 50))
    ms_per_step = max_over_ranks(torch.tensor([ms_total], device=dev, dtype=torch.float64), dist) / steps
    value = whole_job_rate(w.units, world, ms_per_step)

    # end to end through the host-buffer C-ABI call (pinned host memory)
    Qh, Kh, Vh = b.host
    Wh = b.Wh
    nsets, set_bytes = b.nsets, b.set_bytes
    scratch = (b.part.numel(), b.state.numel())
    del b
    torch.cuda.empty_cache()
    Qp, Kp, Vp, Op = Qh.pin_memory(), Kh.pin_memory(), Vh.pin_memory(), torch.empty_like(Qh).pin_memory()
    stream = torch.cuda.current_stream(dev)
    fv.favor_attention_host(Qp, Kp, Vp, Wh, Op, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        import torch.distributed as td
        td.barrier()
    e0.record(stream)
    for _ in range(args.e2e_steps):
        fv.favor_attention_host(Qp, Kp, Vp, Wh, Op, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(torch.tensor([e0.elapsed_time(e1) / args.e2e_steps], device=dev, dtype=torch.float64), dist)
    e2e_value = whole_job_rate(w.units, world, e2e_ms)
    elt = Qh.element_size()
    h2d = (Qh.numel() + Kh.numel() + Vh.numel()) * elt + Wh.numel() * 4
    d2h = Qh.numel() * elt
    del Qp, Kp, Vp, Op

    rt = roofline_terms(w, peaks)
    kern = {s: kernel_roofline(w, peaks, s, stage_ms[j], scratch) for j, s in enumerate(STAGES)}
    dom = max(STAGES, key=lambda s: kern[s]["us"])
    dk = kern[dom]
    bound_us = max(rt["t_tensor_us"], rt["t_mufu_us"], rt["t_hbm_us"])
    cfg = config_of(w, world)
    cfg["l2"] = (f"{nsets} input set(s) of {set_bytes / 1e6:.0f} MB (Q, K, V, out) rotated, at least twice the "
                 f"126 MB L2, so that no step reads inputs left in L2 by the step before it")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": cfg, "launch_overlap": True,
        "roofline": {"kernel": dom, "bound": dk["bound"], "achieved": dk["achieved"], "peak": dk["peak"],
                     "unit": dk["unit"], "frac": dk["frac"],
                     "traffic": PROFILED_TRAFFIC.get((w.name, dom)),
                     "peak_source": (f"MUFU 16/clk/SM x 148 SMs x {peaks['sm_max_mhz']:.0f} MHz" if dk["bound"] == "alu"
                                     else f"{peak_src} peaks")},
        "roofline_path": {"t_tensor_us": rt["t_tensor_us"], "t_mufu_us": rt["t_mufu_us"], "t_hbm_us": rt["t_hbm_us"],
                          "bound_us": bound_us, "frac": bound_us / (ms_per_step * 1e3),
                          "peaks": f"{peak_src}: HBM {peaks['hbm_gbs']} GB/s, bf16 {peaks['bf16_tflops']} TFLOP/s"},
        "stage_ms": dict(zip(STAGES, stage_ms)),
        "kernels": {s: {k: kern[s][k] for k in ("bound", "achieved", "peak", "unit", "frac")} for s in STAGES},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms},
        "gpu_launches": 3 * steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_per_workload and not args.batch:
        entries = []
        for name in wl.WORKLOAD_ORDER:
            wk = wl.WORKLOADS[name]
            for orth in wk.orthogonal:
                entries.append(workload_entry(fv, wk, dev, local, peaks, args.steps or 20, orth))
        line["per_workload"] = entries
        line["decode"] = decode_entry(fv, dev, peaks)
        line["relu"] = relu_entry(fv, dev, peaks)
        line["linformer"] = linformer_entry(fv, dev, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r, heads, dt, threads = oracle_rate(w, 10.0)
        line["cpu_baseline"] = {"value": r, "unit": UNIT, "cores": host_cores(), "blas_threads": threads,
                                "kind": "oracle",
                                "sample": f"{heads} of {w.B * w.H} (batch, head) pairs x L={w.L} in {dt:.1f} s, numpy fp64"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        td.barrier()
        td.destroy_process_group()


if __name__ == "__main__":
    main()
