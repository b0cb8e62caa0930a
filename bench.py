"""Benchmark of the BitLinear W1.58A8 decode hot path on B200.

One step = one pass of the decode hot path over one synthetic token batch of
the FFN up/down decode workload (M = 1, bf16 activations with 1% x20 outlier
channels):
    quantise x_up  [1, 4096]  + ternary GEMV with W_up   [11008, 4096]
    quantise x_dn  [1, 11008] + ternary GEMV with W_down [4096, 11008]
both through one call of the batched C-ABI entry bitlinear_forward_fp_batch
(one kernel launch per step; the projections are independent).  Weights are prepared once (absmean ternarisation + 2-bit
packing, outside the timed region) and rotate over enough copies that every
step reads its weights from HBM (working set > L2).  The timed steps are CUDA
graphs uploaded to the device before the start event, behind a ~1 ms
device-side spin, so the timed region holds exactly the replayed steps.

Printed metric: algorithmic GB/s (packed weights + activations + outputs per
step / step time), whole job over all ranks, plus the roofline of the GEMV
against the measured HBM copy bandwidth, the CPU oracle timed on the host,
an end-to-end figure through the public API with host buffers (per step one
H2D copy, one call, one D2H copy, recorded in CUDA graphs; the same sequence
issued eagerly is reported beside it), and SM clocks.  Extra sections
(--sections): the prefill GEMM (M = 2048) in int8 TOPS against the int8
tensor peak, small-batch decode, a decoder block, the 1-bit weight variant
(decode GEMV and prefill GEMM), the MatMul-free GLU channel mixer and group
quantisation (G = 4) at decode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "BitLinear W1.58A8 GEMV GB/s (frac of HBM peak); prefill GEMM int8 TOPS vs peak"
WORKLOAD = workloads.W2
PEAK_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 4.5 / 2.25  # nominal dense int8 : bf16 tensor ratio

# Compute-side bounds of the small-batch paths, from rates measured on B200
# with single-SM probes: a tcgen05.mma kind::i8 of 128 x N x 32 takes ~186
# cycles for every N <= 256; dp4a alone issues 64 lanes per cycle per SM, and
# an even mix of dp4a and LOP3 85.  At the nominal maximum SM clock.
MMA_CYCLES = 186
DP4A_LANES_PER_CLK = 64
MIXED_LANES_PER_CLK = 85
NOMINAL_SM_HZ = 1.965e9


def small_batch_bound(M, K, N, nbytes, hbm_gbs, sms, path):
    """Lower bounds (us) of one small-batch call on the path it takes
    ("cuda_cores", "swap_ab" or "gemm", as the library reports it): HBM time
    of its algorithmic bytes, and the compute time of the path's own
    instruction stream spread evenly over the SMs -- dp4a + mask per 4 trits
    on CUDA cores, 128 weight rows x 32 k per MMA for the swap-AB kernel,
    128 tokens x 256 weight rows x 32 k per MMA for the GEMM.  The bound is
    the larger."""
    hbm_us = nbytes / (hbm_gbs * 1e3)
    if path == "cuda_cores":
        dp4a, lop3 = N * K / 16 * 4 * M, N * K / 16 * 4
        clk = max(dp4a / DP4A_LANES_PER_CLK, (dp4a + lop3) / MIXED_LANES_PER_CLK) / sms
        comp_us, kind = clk / NOMINAL_SM_HZ * 1e6, "alu (dp4a + mask)"
    elif path == "swap_ab":
        mmas = N * K / (128 * 32)
        comp_us, kind = mmas / sms * MMA_CYCLES / NOMINAL_SM_HZ * 1e6, "tensor (swap-AB, 128 rows x 32 k per MMA)"
    else:
        mmas = -(-M // 128) * -(-N // 256) * K / 32
        comp_us, kind = mmas / sms * MMA_CYCLES / NOMINAL_SM_HZ * 1e6, "tensor (GEMM, 128 x 256 x 32 per MMA)"
    return {"hbm_us": hbm_us, "compute_us": comp_us, "compute": kind, "bound_us": max(hbm_us, comp_us),
            "bound": "hbm" if hbm_us >= comp_us else kind.split()[0]}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemv_decode_m1_traffic.json")


def step_bytes() -> int:
    return sum(s.algorithmic_bytes for s in WORKLOAD.shapes)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAK_FALLBACK), "fallback"


def kernel_source_hash() -> str:
    """Hash of what defines the decode GEMV's device code: its source, the
    device headers it includes, and the output-mode enum it reads (the rest of
    kernels.cuh declares host launchers)."""
    import re
    csrc = os.path.join(ROOT, "ternary_weight_linear_forward_b200", "csrc")
    h = hashlib.sha256()
    for name in ("k_gemv.cu", "gemv_inl.cuh", "act_inl.cuh", "common.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    with open(os.path.join(csrc, "kernels.cuh")) as f:
        h.update(re.search(r"enum YMode[^}]*\}", f.read()).group(0).encode())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current GEMV source; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    return d.get("dram_bytes_per_launch")


_CUDA_DRV = None


def upload_graphs(gs, stream) -> bool:
    """Upload each graph's executable to the device on `stream` (driver
    cuGraphUpload), so that its first replay does not pay for it.  Returns
    False where the driver entry point is not available."""
    global _CUDA_DRV
    import ctypes
    if _CUDA_DRV is None:
        try:
            _CUDA_DRV = ctypes.CDLL("libcuda.so.1")
            _CUDA_DRV.cuGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
            _CUDA_DRV.cuGraphUpload.restype = ctypes.c_int
        except (OSError, AttributeError):
            _CUDA_DRV = False
    if not _CUDA_DRV:
        return False
    ok = True
    for g in gs:
        rc = _CUDA_DRV.cuGraphUpload(ctypes.c_void_p(g.raw_cuda_graph_exec()), ctypes.c_void_p(stream.cuda_stream))
        ok = ok and rc == 0
    return ok


def lead_cycles(n_graphs: int) -> int:
    """Device-side spin queued ahead of a timed region: long enough (about
    1 ms plus 100 us per graph at ~2 GHz) for the host to submit the graphs
    before the start event is reached, even on a busy host.  (A 75 us spin
    was once outrun by the host's submission of a single graph: the 20
    timed steps then read 13.6 instead of 9.0 us each.)"""
    return int((1000 + 100 * n_graphs) * 2000)


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason sampler (reads only)."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip()
                if out:
                    self.samples.append([v.strip() for v in out.split(",")])
            except (OSError, subprocess.SubprocessError):
                return
            self._stop.wait(0.05)

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join(timeout=10)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for s in self.samples for n, v in zip(names, s[5:9]) if v.strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------

def cpu_oracle_step_fn(row_frac: float = 1.0):
    """One oracle step over the workload; with row_frac < 1 only the first
    row_frac of each weight matrix's output rows (a bounded sample).
    Returns (step function, algorithmic bytes per step)."""
    import oracle
    prepared, nbytes = [], 0
    for s in WORKLOAD.shapes:
        rows = max(1, int(round(s.N * row_frac)))
        W_t, beta = oracle.quantize_weights(s.weights())
        prepared.append((s.inputs(), np.ascontiguousarray(W_t[:rows]), beta))
        xb = 2 if s.x_dtype == "bf16" else 4
        nbytes += rows * (s.K // 16) * 4 + s.M * s.K * xb + s.M * rows * 4

    def step():
        for x, W_t, beta in prepared:
            r = oracle.forward(x, W_t, beta)
            _ = r["y"]
    return step, nbytes


def run_cpu_oracle(budget_s: float, max_steps: int | None = None, step=None):
    """Time the oracle, as it stands, on one host core: steps until max_steps
    or until budget_s has elapsed."""
    if step is None:
        step, _ = cpu_oracle_step_fn()
    step()  # warm caches, page in
    n, t0 = 0, time.perf_counter()
    while True:
        step()
        n += 1
        el = time.perf_counter() - t0
        if (max_steps and n >= max_steps) or el >= budget_s:
            break
    return n, el


REF_ROW_FRAC = 1.0 / 8.0


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline_child(setting: str, budget_s: float):
    """Run inside a child process: time the oracle on the full decode step
    (both projections) and print one JSON line.  `single`: the plain build,
    the process pinned to one core; `all`: the OpenMP build of the same
    source on every core the process may use."""
    cores = sorted(os.sched_getaffinity(0))
    if setting == "single":
        os.sched_setaffinity(0, {cores[0]})
        threads = 1
    else:
        threads = len(cores)
    step, _ = cpu_oracle_step_fn()
    n, el = run_cpu_oracle(budget_s, step=step)
    print(json.dumps({"steps": n, "seconds": el, "threads": threads,
                      "cpus": sorted(os.sched_getaffinity(0))[:4]}), flush=True)


def cpu_baseline(budget_s: float):
    """The oracle, as it stands, timed on the host in two settings (one
    pinned core; all cores with the OpenMP build), each in a child process
    that touches no GPU.  Returns the cpu_baseline object of the JSON line."""
    out = {}
    ncores = len(os.sched_getaffinity(0))
    for setting in ("single", "all"):
        env = dict(os.environ)
        if setting == "all":
            env.update(ORACLE_OPENMP="1", OMP_NUM_THREADS=str(ncores), OMP_PROC_BIND="spread")
        else:
            env.update(OMP_NUM_THREADS="1")
        env["CUDA_VISIBLE_DEVICES"] = ""
        r = subprocess.run([sys.executable, os.path.abspath(__file__), "--cpu-baseline-child", setting,
                            "--cpu-budget", str(budget_s)], env=env, capture_output=True, text=True,
                           timeout=budget_s * 20 + 600)
        if r.returncode != 0:
            out[setting] = {"error": (r.stderr or r.stdout)[-300:]}
            continue
        d = json.loads(r.stdout.strip().splitlines()[-1])
        out[setting] = {"value": step_bytes() * d["steps"] / d["seconds"] / 1e9, "cores": d["threads"],
                        "ms_per_step": d["seconds"] / d["steps"] * 1e3,
                        "sample": f"{d['steps']} full steps of the workload (both projections) in "
                                  f"{d['seconds']:.1f} s"}
    main = out.get("all", {})
    one = out.get("single", {})
    return {"value": main.get("value"), "unit": "GB/s", "cores": main.get("cores"), "kind": "oracle",
            "sample": ("the plain C oracle, compiled a second time with -fopenmp (the (m, n) pairs of the integer "
                       "contraction shared among threads, arithmetic unchanged), on every host core; "
                       + main.get("sample", main.get("error", ""))),
            "single_core": dict(one, kind="oracle", pinned="one core (sched_setaffinity)",
                                build="plain gcc -O2"),
            "cpu_model": cpu_model(), "host_cores": ncores}


def max_over_ranks(t: float, world: int, device) -> float:
    """The slowest rank's time.  Every rank must call it at the same point
    (one all-reduce); with one rank the time is returned as it is."""
    if world <= 1:
        return t
    import torch
    import torch.distributed as dist
    x = torch.tensor([t], dtype=torch.float64, device=device)
    dist.all_reduce(x, op=dist.ReduceOp.MAX)
    return float(x.item())


def job_gbs(bytes_per_rank_step: int, steps: int, world: int, t_max: float) -> float:
    """Whole-job throughput: every rank moves its bytes per step; the job
    takes as long as its slowest rank."""
    return world * bytes_per_rank_step * steps / t_max / 1e9


def reference_arm(args):
    """The reference arm is the CPU oracle (there is no other implementation):
    W untimed warm-up steps, then exactly K timed steps, each over the first
    1/8 of every weight matrix's output rows."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    fn, nbytes = cpu_oracle_step_fn(REF_ROW_FRAC)
    for _ in range(args.warmup):
        fn()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fn()
    el = time.perf_counter() - t0
    v = nbytes * args.steps / el / 1e9
    sample = (f"each step: quantiser on the full activations + ternary GEMV over the first 1/8 of the output "
              f"rows of both projections ({nbytes} algorithmic bytes per step)")
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8xt2->i32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD.name, "shapes": [s.name for s in WORKLOAD.shapes], "row_fraction": REF_ROW_FRAC},
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

class PartRanges:
    """NVTX push/pop ranges around the parts of the run (decode, e2e, prefill,
    small, ...), so that a profiler can select the launches of one part, e.g.
    ``ncu --nvtx --nvtx-include "small/" ...``.  Calling it with a name closes
    the open range and opens the named one; with None it only closes."""

    def __init__(self):
        self.open = False

    def __call__(self, name):
        import torch
        if self.open:
            torch.cuda.nvtx.range_pop()
        self.open = name is not None
        if name is not None:
            torch.cuda.nvtx.range_push(name)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="run the decode step only (no extra sections)")
    ap.add_argument("--sections", default="prefill,small,block,binary,glu,grouped",
                    help="extra measured sections after the decode step, comma separated")
    ap.add_argument("--cpu-baseline-child", choices=["single", "all"], help=argparse.SUPPRESS)
    ap.add_argument("--cpu-budget", type=float, default=float(os.environ.get("BENCH_CPU_BUDGET_S", "12")))
    args = ap.parse_args()
    if args.cpu_baseline_child:
        cpu_baseline_child(args.cpu_baseline_child, args.cpu_budget)
        return 0
    sections = set() if args.no_prefill else {x for x in args.sections.split(",") if x}
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return reference_arm(args)

    import torch
    import torch.distributed as dist

    import ternary_weight_linear_forward_b200 as bl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    props = torch.cuda.get_device_properties(dev)
    L2 = props.L2_cache_size

    # ---- offline weight preparation (not timed) ----
    shapes = WORKLOAD.shapes
    packed_bytes = sum(s.packed_bytes for s in shapes)
    copies = max(2, int(4 * L2 // packed_bytes) + 1)       # working set >= 4x L2
    layers = []
    for s in shapes:
        W = torch.from_numpy(s.weights()).to(dev)
        W_t, beta = bl.quantize_weights(W)
        W_p = bl.pack(W_t)
        del W, W_t
        xb = torch.from_numpy(s.inputs_bf16_bits().view(np.int16)).to(dev).view(torch.bfloat16)
        y = torch.empty((s.M, s.N), dtype=torch.float32, device=dev)
        layers.append({"shape": s, "W_p": [W_p] + [W_p.clone() for _ in range(copies - 1)], "beta": beta,
                       "x": xb, "y": y})
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)

    def step(i, which=None):
        # both projections are independent: one batched launch per step
        probs = [{"x": L["x"], "W_p": L["W_p"][i % copies], "beta": L["beta"], "out": L["y"]}
                 for j, L in enumerate(layers) if which is None or which == j]
        bl.forward_fp_batch(probs, stream=stream)

    def capture(n, start, which=None):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    step(start + i, which)
        return g

    # graphs of at most CHUNK steps; the timed region replays exactly K steps
    CHUNK = 256
    with torch.cuda.stream(stream):
        for i in range(3):
            step(i)
    torch.cuda.synchronize()

    def graphs_for(n, which=None):
        gs, done = [], 0
        while done < n:
            k = min(CHUNK, n - done)
            gs.append(capture(k, done, which))
            done += k
        return gs

    warm = graphs_for(args.warmup)
    timed = graphs_for(args.steps)

    def run(gs):
        for g in gs:
            g.replay()

    def timed_run(gs):
        # The graphs are uploaded to the device before the start event, and a
        # short device-side spin is queued ahead of it, so the timed region
        # holds exactly the replayed steps: neither the first replay's upload
        # nor the host's submission of the first graph falls inside it.
        if world > 1:
            dist.barrier()
        upload_graphs(gs, stream)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            torch.cuda._sleep(lead_cycles(len(gs)))
        e0.record(stream)
        with torch.cuda.stream(stream):
            run(gs)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3

    part = PartRanges()
    part("decode")
    # SM clocks are sampled over the whole measured part of the run (the timed
    # decode region alone is far shorter than one sampling period)
    clk = ClockSampler(local).__enter__()
    with torch.cuda.stream(stream):
        run(warm)
    torch.cuda.synchronize()
    t_step = timed_run(timed)
    t_max = max_over_ranks(t_step, world, dev)
    ms_per_step = t_max / args.steps * 1e3
    value = job_gbs(step_bytes(), args.steps, world, t_max)

    # ---- roofline of the dominant kernel: one batched GEMV launch per step, so
    # the per-launch time is the timed region's per-step time; each projection
    # launched alone is reported beside it ----
    peaks, peak_kind = load_peaks()
    per_shape = {}
    for j, L in enumerate(layers):
        n = max(64, min(args.steps, 1024))
        gw = graphs_for(32, which=j)
        with torch.cuda.stream(stream):
            run(gw)
        gs = graphs_for(n, which=j)
        t = timed_run(gs)
        s = L["shape"]
        per_shape[s.name] = {"us_per_launch": t / n * 1e6, "GB/s": s.algorithmic_bytes * n / t / 1e9,
                             "bytes_per_launch": s.algorithmic_bytes}
        del gs, gw
    achieved = step_bytes() * args.steps / t_step / 1e9
    traffic = recorded_traffic()
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback",
                "kernel": "gemv_group_kernel (fused absmax int8 quantiser + ternary GEMV; both projections, "
                          "one launch per step)",
                "bytes_per_launch": step_bytes(), "us_per_launch": t_step / args.steps * 1e6,
                "alone_per_shape": per_shape}

    part("e2e")
    # ---- end to end through the public API with pinned host buffers ----
    # The step's inputs (both projections' x) sit in one pinned host buffer and
    # its outputs in one device / one pinned host buffer, so a step is one H2D
    # copy, one library call (marshalled once per weight copy) and one D2H copy.
    xs = [L["x"].reshape(-1) for L in layers]
    ys = [L["y"].reshape(-1) for L in layers]
    host_x = torch.cat([x.cpu() for x in xs]).pin_memory()
    dev_xcat = torch.empty_like(host_x, device=dev)
    ycat = torch.empty(sum(y.numel() for y in ys), dtype=torch.float32, device=dev)
    host_y = torch.empty_like(ycat, device="cpu").pin_memory()
    dev_x, dev_y, ox, oy = [], [], 0, 0
    for L, x, y in zip(layers, xs, ys):
        dev_x.append(dev_xcat[ox:ox + x.numel()].view(L["x"].shape))
        dev_y.append(ycat[oy:oy + y.numel()].view(L["y"].shape))
        ox += x.numel()
        oy += y.numel()
    plans = [bl.BatchPlan([{"x": dev_x[j], "W_p": L["W_p"][c], "beta": L["beta"], "out": dev_y[j]}
                           for j, L in enumerate(layers)]) for c in range(copies)]
    h2d = host_x.numel() * host_x.element_size()
    d2h = host_y.numel() * host_y.element_size()
    n_e2e = max(16, min(args.steps, 2000))

    def e2e_step(i):
        with torch.cuda.stream(stream):
            dev_xcat.copy_(host_x, non_blocking=True)
            plans[i % copies].run(stream=stream)
            host_y.copy_(ycat, non_blocking=True)

    def e2e_timed(fn):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)

    def e2e_eager():
        for i in range(n_e2e):
            e2e_step(i)

    # Pipelined steps: NB sets of device input / output buffers and pinned
    # output buffers; step i copies its input on s_in, runs the call on the
    # compute stream and copies its output back on s_out, so the copies of
    # steps i +- 1 overlap the kernel of step i.  Buffer set i % NB is reused
    # only after the kernel (input side) and the D2H copy (output side) of
    # step i - NB are done.  Recorded in CUDA graphs of <= CHUNK steps; every
    # graph forks and joins the copy streams, so chunks do not overlap.
    NB = 3
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    px = [dev_xcat] + [torch.empty_like(dev_xcat) for _ in range(NB - 1)]
    py = [ycat] + [torch.empty_like(ycat) for _ in range(NB - 1)]
    phy = [host_y] + [torch.empty_like(host_y).pin_memory() for _ in range(NB - 1)]
    pplans = []
    for bi in range(NB):
        dx, dy, ox, oy = [], [], 0, 0
        for L, x, y in zip(layers, xs, ys):
            dx.append(px[bi][ox:ox + x.numel()].view(L["x"].shape))
            dy.append(py[bi][oy:oy + y.numel()].view(L["y"].shape))
            ox += x.numel()
            oy += y.numel()
        pplans.append([bl.BatchPlan([{"x": dx[j], "W_p": L["W_p"][c], "beta": L["beta"], "out": dy[j]}
                                     for j, L in enumerate(layers)]) for c in range(copies)])

    def pipe_graphs(n):
        gs, done = [], 0
        while done < n:
            k = min(CHUNK, n - done)
            g = torch.cuda.CUDAGraph()
            ev_in = [torch.cuda.Event() for _ in range(NB)]
            ev_comp = [torch.cuda.Event() for _ in range(NB)]
            ev_out = [torch.cuda.Event() for _ in range(NB)]
            used = set()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    s_in.wait_stream(stream)
                    s_out.wait_stream(stream)
                    for j in range(k):
                        i, bi = done + j, j % NB
                        if bi in used:
                            s_in.wait_event(ev_comp[bi])     # kernel of step i - NB has read px[bi]
                        with torch.cuda.stream(s_in):
                            px[bi].copy_(host_x, non_blocking=True)
                            ev_in[bi].record(s_in)
                        stream.wait_event(ev_in[bi])
                        if bi in used:
                            stream.wait_event(ev_out[bi])    # D2H of step i - NB has read py[bi]
                        pplans[bi][i % copies].run(stream=stream)
                        ev_comp[bi].record(stream)
                        s_out.wait_event(ev_comp[bi])
                        with torch.cuda.stream(s_out):
                            phy[bi].copy_(py[bi], non_blocking=True)
                            ev_out[bi].record(s_out)
                        used.add(bi)
                    stream.wait_stream(s_in)
                    stream.wait_stream(s_out)
            gs.append(g)
            done += k
        return gs

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    t_eager = e2e_timed(e2e_eager)
    eg = pipe_graphs(n_e2e)
    with torch.cuda.stream(stream):
        run(pipe_graphs(8))
    torch.cuda.synchronize()

    def e2e_replay():
        with torch.cuda.stream(stream):
            run(eg)
    t_e2e = e2e_timed(e2e_replay)
    del eg
    e2e = {"value": job_gbs(step_bytes(), n_e2e, world, t_e2e), "unit": "GB/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": n_e2e, "us_per_step": t_e2e / n_e2e * 1e6,
           "path": "per step: one pinned H2D copy of both inputs (copy stream) + bitlinear_forward_fp_batch "
                   "(both projections, descriptors marshalled once per buffer set and weight copy) + one D2H copy "
                   f"of both outputs into pinned memory (second copy stream); {NB} buffer sets, so copies of "
                   f"neighbouring steps overlap the kernel; recorded in CUDA graphs of <= {CHUNK} steps and "
                   f"replayed; weights rotate over {copies} copies",
           "eager": {"value": job_gbs(step_bytes(), n_e2e, world, t_eager), "us_per_step": t_eager / n_e2e * 1e6,
                     "path": "the same three operations issued from the host every step on one stream, "
                             "no graph, no overlap"}}

    part("prefill")
    # ---- prefill GEMM (M = 2048): int8 tensor-core TOPS ----
    prefill = None
    if "prefill" in sections:
        prefill = {}
        int8_peak_burst = peaks["bf16_tflops"] * INT8_OVER_BF16
        for s in workloads.W4.shapes:
            W = torch.from_numpy(s.weights()).to(dev)
            W_t, beta = bl.quantize_weights(W)
            W_p = bl.pack(W_t)
            del W, W_t
            x = torch.from_numpy(s.inputs()).to(dev)
            x_q, gamma = bl.quant_act(x)
            y = torch.empty((s.M, s.N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(bl.forward_workspace(s.M, s.N, s.K), dtype=torch.uint8, device=dev)
            reps = 20
            with torch.cuda.stream(stream):
                for _ in range(5):
                    bl.forward(x_q, gamma, W_p, beta, out=y, ws=ws, stream=stream)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    for _ in range(reps):
                        bl.forward(x_q, gamma, W_p, beta, out=y, ws=ws, stream=stream)
            g.replay()
            t = timed_run([g])
            tops = s.ops * reps / t / 1e12
            prefill[s.name] = {"us_per_call": t / reps * 1e6, "TOPS": tops,
                               "frac_of_int8_peak": tops / int8_peak_burst,
                               "frac_of_nominal_4500": tops / 4500.0}
            del g, W_p, x, x_q, y, ws
        prefill["int8_peak_TOPS"] = int8_peak_burst
        prefill["int8_peak_source"] = (f"{peak_kind} bf16_tflops {peaks['bf16_tflops']} x nominal int8/bf16 ratio "
                                       f"{INT8_OVER_BF16}")

    part("small")
    # ---- small-batch decode (M = 4, 16, 64; K = 4096; N = 4096, 11008) ----
    small = None
    if "small" in sections:
        small = {}
        for s in workloads.W3.shapes:
            W = torch.from_numpy(s.weights()).to(dev)
            W_t, beta = bl.quantize_weights(W)
            W_p0 = bl.pack(W_t)
            del W, W_t
            nc = max(2, int(4 * L2 // (W_p0.numel() * 4)) + 1)
            W_ps = [W_p0] + [W_p0.clone() for _ in range(nc - 1)]
            x = torch.from_numpy(s.inputs()).to(dev)
            y = torch.empty((s.M, s.N), dtype=torch.float32, device=dev)
            ws = torch.empty(max(1, bl.forward_fp_workspace(s.M, s.N, s.K)), dtype=torch.uint8, device=dev)
            reps = 4 * nc
            with torch.cuda.stream(stream):
                for i in range(4):
                    bl.forward_fp(x, W_ps[i % nc], beta, out=y, ws=ws, stream=stream)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    for i in range(reps):
                        bl.forward_fp(x, W_ps[i % nc], beta, out=y, ws=ws, stream=stream)
            g.replay()
            t = timed_run([g])
            gbs = s.algorithmic_bytes * reps / t / 1e9
            us = t / reps * 1e6
            path = bl.forward_path(s.M, s.N, s.K)
            rl = small_batch_bound(s.M, s.K, s.N, s.algorithmic_bytes, peaks["hbm_gbs"], props.multi_processor_count,
                                   path)
            rl["frac_of_bound"] = rl["bound_us"] / us
            small[s.name] = {"us_per_call": us, "GB/s": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"],
                             "roofline": rl,
                             "path": {"cuda_cores": "CUDA-core GEMV, quantiser fused",
                                      "swap_ab": "quantiser + tcgen05 swap-AB decode",
                                      "gemm": "quantiser writing the row sums + tcgen05 GEMM, K split + finishing pass"}[path]}
            del g, W_ps, W_p0, x, y, ws

    part("block")
    # ---- decoder block at batch-1 decode (hidden 2560, intermediate 6912) ----
    block = None
    if "block" in sections:
        bw = {p: torch.from_numpy(w).to(dev) for p, w in workloads.block_weights().items()}
        nblk = max(2, int(1.2 * L2 // sum(w.numel() // 4 for w in bw.values())) + 1)   # >= 1.2x L2 of weights
        blocks = [bl.DecoderBlock.from_float(bw) for _ in range(nblk)]
        del bw
        bx = torch.from_numpy(workloads.block_input()).to(dev)
        wbytes = sum(L.W_p.numel() * 4 for L in blocks[0].layers.values())
        with torch.cuda.stream(stream):
            for b_ in blocks:
                b_(bx)
        torch.cuda.synchronize()
        reps = 8 * nblk
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for i in range(reps):
                    blocks[i % nblk](bx)
        g.replay()
        t = timed_run([g])
        us = t / reps * 1e6
        block = {"us_per_block": us, "weight_bytes": wbytes, "GB/s": wbytes / (t / reps) / 1e9,
                 "frac_of_hbm": wbytes / (t / reps) / 1e9 / peaks["hbm_gbs"], "kernels_per_block": 9,
                 "copies": nblk}
        del g, blocks

    part("binary")
    # ---- 1-bit weights (Sign(W - mean W)): decode GEMV and prefill GEMM ----
    binary = None
    if "binary" in sections:
        binary = {}
        for s in workloads.W2.shapes:
            W_b, _, beta = bl.binarize_weights(torch.from_numpy(s.weights()).to(dev))
            W_p0 = bl.pack_bits(W_b)
            del W_b
            nc = max(2, int(4 * L2 // (W_p0.numel() * 4)) + 1)
            W_ps = [W_p0] + [W_p0.clone() for _ in range(nc - 1)]
            xb = torch.from_numpy(s.inputs_bf16_bits().view(np.int16)).to(dev).view(torch.bfloat16)
            y = torch.empty((s.M, s.N), dtype=torch.float32, device=dev)
            # algorithmic bytes: 1-bit weights, bf16 x, f32 y, beta
            nbytes = s.N * s.K // 8 + s.M * s.K * 2 + s.M * s.N * 4 + 4
            reps = 8 * nc
            with torch.cuda.stream(stream):
                for i in range(4):
                    bl.forward_binary_fp(xb, W_ps[i % nc], beta, out=y, stream=stream)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    for i in range(reps):
                        bl.forward_binary_fp(xb, W_ps[i % nc], beta, out=y, stream=stream)
            g.replay()
            t = timed_run([g])
            gbs = nbytes * reps / t / 1e9
            binary["decode_" + s.name] = {"us_per_call": t / reps * 1e6, "GB/s": gbs,
                                          "frac_of_hbm": gbs / peaks["hbm_gbs"], "bytes_per_call": nbytes,
                                          "path": "CUDA-core GEMV on 1-bit words, quantiser fused"}
            del g, W_ps, W_p0, xb, y
        for s in workloads.W4.shapes:
            W_b, _, beta = bl.binarize_weights(torch.from_numpy(s.weights()).to(dev))
            W_p = bl.pack_bits(W_b)
            del W_b
            x_q, gamma = bl.quant_act(torch.from_numpy(s.inputs()).to(dev))
            y = torch.empty((s.M, s.N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(bl.lib().bitlinear_forward_binary_workspace(s.M, s.N, s.K), dtype=torch.uint8,
                             device=dev)
            reps = 20
            with torch.cuda.stream(stream):
                for _ in range(5):
                    bl.forward_binary(x_q, gamma, W_p, beta, out=y, ws=ws, stream=stream)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    for _ in range(reps):
                        bl.forward_binary(x_q, gamma, W_p, beta, out=y, ws=ws, stream=stream)
            g.replay()
            t = timed_run([g])
            tops = s.ops * reps / t / 1e12
            binary["prefill_" + s.name] = {"us_per_call": t / reps * 1e6, "TOPS": tops,
                                           "frac_of_int8_peak": tops / (peaks["bf16_tflops"] * INT8_OVER_BF16),
                                           "path": "tcgen05 GEMM, 1-bit unpack"}
            del g, W_p, x_q, y, ws

    part("grouped")
    # ---- group quantisation along K (G = 4): decode M = 1 on the FFN shapes ----
    grouped = None
    if "grouped" in sections:
        grouped = {}
        G = 4
        for s in workloads.W2.shapes:
            W_t, beta = bl.quantize_weights_grouped(torch.from_numpy(s.weights()).to(dev), G)
            W_p0 = bl.pack_grouped(W_t)
            del W_t
            nc = max(2, int(4 * L2 // (W_p0.numel() * 4)) + 1)
            W_ps = [W_p0] + [W_p0.clone() for _ in range(nc - 1)]
            xb = torch.from_numpy(s.inputs_bf16_bits().view(np.int16)).to(dev).view(torch.bfloat16)
            y = torch.empty((s.M, s.N), dtype=torch.float32, device=dev)
            ws = torch.empty(bl.lib().bitlinear_forward_grouped_fp_workspace(s.M, s.N, s.K, G), dtype=torch.uint8,
                             device=dev)
            reps = 8 * nc
            with torch.cuda.stream(stream):
                for i in range(4):
                    bl.forward_grouped_fp(xb, W_ps[i % nc], beta, out=y, ws=ws, stream=stream)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    for i in range(reps):
                        bl.forward_grouped_fp(xb, W_ps[i % nc], beta, out=y, ws=ws, stream=stream)
            g.replay()
            t = timed_run([g])
            gbs = s.algorithmic_bytes * reps / t / 1e9
            grouped["decode_g4_" + s.name] = {"us_per_call": t / reps * 1e6, "GB/s": gbs,
                                              "frac_of_hbm": gbs / peaks["hbm_gbs"], "launches": 2,
                                              "path": "one GEMV launch over the 4 groups, each group's quantiser "
                                                      "fused into its prologue and its rescaled binary32 term "
                                                      "written, + the ordered sum of the terms"}
            del g, W_ps, W_p0, xb, y, ws

    part("glu")
    # ---- MatMul-free GLU channel mixer (hidden 2560, intermediate 6912) ----
    glu = None
    if "glu" in sections:
        glu = {}
        D, F = 2560, 6912
        gw = {p: workloads.latent_weights(1060 + i, *shape)
              for i, (p, shape) in enumerate((("gate", (F, D)), ("up", (F, D)), ("down", (D, F))))}
        base = {p: bl.BitLinear.from_float(torch.from_numpy(w).to(dev)) for p, w in gw.items()}
        del gw
        wbytes = sum(L.W_p.numel() * 4 for L in base.values())
        for M in (1, 2048):
            nc = max(2, int(4 * L2 // wbytes) + 1) if M == 1 else 1
            sets = [base] + [{p: bl.BitLinear(L.W_p.clone(), L.beta) for p, L in base.items()}
                             for _ in range(nc - 1)]
            x = torch.from_numpy(workloads.activations(2060, M, D, outliers=True)).to(dev)
            y = torch.empty((M, D), dtype=torch.float32, device=dev)
            ws = torch.empty(bl.lib().bitlinear_glu_workspace(M, D, F), dtype=torch.uint8, device=dev)
            reps = 8 * nc if M == 1 else 10
            with torch.cuda.stream(stream):
                for i in range(3):
                    S = sets[i % nc]
                    bl.glu_forward(x, S["gate"], S["up"], S["down"], out=y, ws=ws, stream=stream)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    for i in range(reps):
                        S = sets[i % nc]
                        bl.glu_forward(x, S["gate"], S["up"], S["down"], out=y, ws=ws, stream=stream)
            g.replay()
            t = timed_run([g]) / reps
            if M == 1:
                glu["decode_m1"] = {"us_per_call": t * 1e6, "weight_bytes": wbytes, "GB/s": wbytes / t / 1e9,
                                    "frac_of_hbm": wbytes / t / 1e9 / peaks["hbm_gbs"], "launches": 4,
                                    "copies": nc}
            else:
                ops = 2 * M * 3 * D * F
                glu["prefill_m2048"] = {"us_per_call": t * 1e6, "TOPS": ops / t / 1e12,
                                        "frac_of_int8_peak": ops / t / 1e12 / (peaks["bf16_tflops"] * INT8_OVER_BF16),
                                        "launches": 8}
            del g, sets, x, y, ws
        del base

    clk.__exit__()
    part(None)
    clocks = clk.summary()
    clocks["window"] = "whole GPU part of the run (decode warm-up and timed steps, roofline, e2e and sections)"

    # ---- CPU oracle baseline (rank 0, N = 1 only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_budget)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "i8xt2->i32", "data": "synthetic",
            "config": {"workload": WORKLOAD.name, "shapes": [s.name for s in shapes],
                       "x_dtype": "bf16", "y_dtype": "f32", "outlier_channels": "1% x20",
                       "l2": f"inputs larger than L2: weights rotate over {copies} copies "
                             f"({copies * packed_bytes / 1e6:.0f} MB vs L2 {L2 / 1e6:.0f} MB)",
                       "parallelism": f"replicas x{world}", "graph_chunk_steps": CHUNK},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps, "clocks": clocks, "prefill": prefill, "small_batch": small, "block": block,
            "binary": binary, "glu": glu, "grouped": grouped,
            "device": props.name,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
