"""Benchmark of the FAVOR+ hot path on B200 (one JSON line on rank 0).

A step is one full pass of the path over one batch of synthetic input:
key pass -> state reduction -> query pass, with Q, K, V resident in HBM.
The headline workload is B=4, H=12, L=16384, d=64, m=256 bf16 with
heavy-tailed key norms.  `value` is whole-job Mtoken*heads/s (units = B*H*L
query tokens x heads, summed over ranks); `e2e` is the same metric through
the host-buffer C-ABI call (host->device copies and the copy back included).

Multi-GPU: every rank runs its own replica of the workload (the path has no
exchange step), so scaling is weak; time is the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
"""
import argparse
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

from linear_approximate_softmax_b200 import workloads as wl  # noqa: E402

METRIC = "FAVOR+ Mtoken*heads/s at L=16K,d=64,m=256 bf16"
UNIT = "Mtoken*heads/s"
DEFAULT_WORKLOAD = "bf16_L16384_heavykeys"
L2_BYTES = 126 * 2**20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=wl.WORKLOAD_ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--batch", type=int, default=None, help="override the workload's B (profiling runs)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, "fallback"


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of each kernel on the
# headline workload, from the ncu captures summarised in the named profiles/ files; a kernel
# whose code changed after its capture gets no entry (traffic null).
PROFILED_TRAFFIC = {
    ("bf16_L16384_heavykeys", "query_pass"): (103.354112e6 + 57.198080e6,
                                              "profiles/query_pass_sm100_bf16_L16384_heavykeys.md"),
    ("bf16_L16384_heavykeys", "key_pass"): (201.485824e6 + 9.511424e6,
                                            "profiles/key_pass_pp_sm100_bf16_L16384_heavykeys.md"),
}

# MUFU ex2 issue rate of one B200 SM (16 results per clock) x 148 SMs x the
# maximum SM clock: the exp roof of the path (derived from unit counts and clocks).
MUFU_PER_SM_CLK = 16
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


def roofline_terms(w, peaks):
    """Algorithmic work per step and the time each resource needs for it at peak."""
    G = w.H // w.Hkv
    units = w.units
    elt = 2 if w.dtype == torch.bfloat16 else 4
    flops = units * (1 + 1 / G) * (2 * w.d * w.m + 2 * w.m * (w.d + 1))
    exps = units * (1 + 1 / G) * w.m
    hbm = units * elt * (2 * w.d + 2 * w.d / G)
    mufu_peak = MUFU_PER_SM_CLK * NUM_SMS * peaks["sm_max_mhz"] * 1e6
    return {
        "flops": flops, "exps": exps, "hbm_bytes": hbm,
        "t_tensor_us": flops / (peaks["bf16_tflops"] * 1e12) * 1e6,
        "t_mufu_us": exps / mufu_peak * 1e6,
        "t_hbm_us": hbm / (peaks["hbm_gbs"] * 1e9) * 1e6,
        "mufu_peak_gexps": mufu_peak / 1e9,
    }


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


def oracle_rate(w, budget_s, max_heads=None, inputs=None, start=0):
    """The fp64 oracle, as it stands, on whole (batch, head) pairs of the workload until the budget is spent.

    Input generation and W construction happen before the clock starts; pairs are taken from
    index `start` on (wrapping), so successive samples cover different heads.
    """
    from oracle import favor as ofv
    from threadpoolctl import threadpool_info
    Q, K, V = inputs if inputs is not None else wl.make_inputs(w)
    Wo = ofv.make_features_f32(w.w_seed, w.m, w.d, w.orthogonal[0])
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
    total_heads, busy = 0, 0.0
    for k in range(steps):  # each step: one bounded sample of 2 (batch, head) pairs
        r, heads, dt, threads = oracle_rate(w, 1.0, max_heads=2, inputs=inputs, start=2 * k)
        total_heads += heads
        busy += dt
    value = total_heads * w.L / busy / 1e6
    wall = busy
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": steps,
        "warmup": args.warmup, "ms_per_step": wall / steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "L": w.L, "d": w.d, "m": w.m},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{total_heads} (batch, head) pairs x L={w.L}, up to 2 per step, numpy fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


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
    # every kernel on this stream is the library's own, none lets its dependents start early:
    # the first kernel of each call may overlap the end of the previous call (favor.h)
    fv.favor_set_launch_overlap(True)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = wl.WORKLOADS[args.workload]
    if args.batch:
        import dataclasses
        w = dataclasses.replace(w, B=args.batch, name=f"{w.name}_B{args.batch}")
    Qh, Kh, Vh = wl.make_inputs(w)
    Wh = fv.favor_make_features(w.w_seed, w.m, w.d, w.orthogonal[0])
    Q, K, V, W = Qh.to(dev), Kh.to(dev), Vh.to(dev), Wh.to(dev)
    out = torch.empty_like(Q)
    part = torch.empty(fv.favor_partials_bytes(w.B, w.Hkv, w.L, w.d, w.m), dtype=torch.uint8, device=dev)
    state = torch.empty(fv.favor_state_bytes(w.B, w.Hkv, w.d, w.m), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        fv.favor_key_pass(K, V, W, part, stream)
        if evs:
            evs[1].record(stream)
        fv.favor_state_reduce(part, state, w.B, w.Hkv, w.L, w.d, w.m, stream)
        if evs:
            evs[2].record(stream)
        fv.favor_query_pass(Q, W, state, w.Hkv, out, stream)
        if evs:
            evs[3].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    steps = args.steps
    if steps is None:  # default: about 3 s of timed work
        t = time.perf_counter()
        for _ in range(5):
            step()
        torch.cuda.synchronize(dev)
        per = (time.perf_counter() - t) / 5
        steps = int(min(5000, max(20, 3.0 / max(per, 1e-6))))

    # the timed region: plain steps, so that each kernel's set-up overlaps the end of the one
    # before it (events between the kernels would serialise them)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        import torch.distributed as td
        td.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        start.record(stream)
        for i in range(steps):
            step()
        stop.record(stream)
        torch.cuda.synchronize(dev)
    if dist:
        td.barrier()
    ms_total = start.elapsed_time(stop)
    # each kernel's own duration: events on the launching stream between the stages, in
    # separate steps after the timed region
    nst = min(steps, 50)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nst)]
    for i in range(nst):
        step(evs[i])
    torch.cuda.synchronize(dev)
    stage_ms = [sum(e[j].elapsed_time(e[j + 1]) for e in evs) / nst for j in range(3)]
    ms_per_step = max_over_ranks(torch.tensor([ms_total], device=dev, dtype=torch.float64), dist) / steps
    value = whole_job_rate(w.units, world, ms_per_step)

    # end to end through the host-buffer C-ABI call (pinned host memory)
    Qp, Kp, Vp, Op = Qh.pin_memory(), Kh.pin_memory(), Vh.pin_memory(), torch.empty_like(Qh).pin_memory()
    fv.favor_attention_host(Qp, Kp, Vp, Wh, Op, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
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

    peaks, peak_src = load_peaks()
    rt = roofline_terms(w, peaks)
    names = ["key_pass", "state_reduce", "query_pass"]
    dom = max(range(3), key=lambda j: stage_ms[j])
    G = w.H // w.Hkv
    dom_exps = w.units * w.m / (G if dom == 0 else 1) if dom != 1 else w.B * w.Hkv * w.m
    achieved = dom_exps / (stage_ms[dom] * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "L": w.L, "d": w.d, "m": w.m,
                   "parallelism": f"replicas x{world}", "launch_overlap": True,
                   "l2": f"inputs larger than L2 ({(Qh.numel() + Kh.numel() + Vh.numel()) * elt / 1e6:.0f} MB of Q,K,V per step)"},
        "roofline": {"kernel": names[dom], "bound": "alu", "achieved": achieved,
                     "peak": rt["mufu_peak_gexps"], "unit": "Gexp/s", "frac": achieved / rt["mufu_peak_gexps"],
                     "traffic": PROFILED_TRAFFIC.get((w.name, names[dom]), (None, None))[0],
                     "traffic_source": PROFILED_TRAFFIC.get((w.name, names[dom]), (None, None))[1],
                     "peak_source": f"MUFU 16/clk/SM x 148 SMs x {peaks['sm_max_mhz']:.0f} MHz"},
        "roofline_path": {"t_tensor_us": rt["t_tensor_us"], "t_mufu_us": rt["t_mufu_us"], "t_hbm_us": rt["t_hbm_us"],
                          "bound_us": max(rt["t_tensor_us"], rt["t_mufu_us"], rt["t_hbm_us"]),
                          "frac": max(rt["t_tensor_us"], rt["t_mufu_us"], rt["t_hbm_us"]) / (ms_per_step * 1e3),
                          "peaks": f"{peak_src}: HBM {peaks['hbm_gbs']} GB/s, bf16 {peaks['bf16_tflops']} TFLOP/s"},
        "stage_ms": dict(zip(names, stage_ms)),
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms},
        "gpu_launches": 3 * steps,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r, heads, dt, threads = oracle_rate(w, 10.0)
        line["cpu_baseline"] = {"value": r, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": f"{heads} of {w.B * w.H} (batch, head) pairs x L={w.L} in {dt:.1f} s, numpy fp64"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        td.barrier()
        td.destroy_process_group()


if __name__ == "__main__":
    main()
