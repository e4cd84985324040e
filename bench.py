#!/usr/bin/env python3
"""Benchmark of the In-Place TTT fast-weight MLP layer forward (prefill) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one whole forward of the layer (gate/up GEMM, look-ahead conv,
target GEMM, fused delta+prefix-scan, apply GEMM) over one batch of the
workload's seeded synthetic inputs.  `value` is whole-job tokens/s with the
inputs resident in HBM; L2 is flushed (256 MiB write) before every timed
step and each step is bracketed by CUDA events on the launching stream.
`e2e` times the same call with the inputs H, X0 copied from pinned host
memory and O, W_down_final read back inside the timed region.

With N > 1 (torchrun, one process per GPU) every rank runs its own batch:
sequences are independent (the fast weight is reset per document), so the
work shards with no collective on the data path ("scaling": "weak").

--impl reference times the CPU fp64 oracle on this host's cores over a
bounded sample of the same workload (one chunk per step).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "fast-weight MLP prefill tokens/s per layer; TFLOP/s vs B200 bf16 peak"
DEFAULT_WORKLOAD = "qwen3-4b"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# What defines each probed kernel and its launch: the headers it is built
# from and, from api.cu, its launch functions and the build switches they read.
KERNEL_SOURCES = {
    "gated_gemm": (("common.cuh", "simt.cuh", "tc_gemm.cuh"),
                   ("ittt_status gated_bf16(", "ittt_status launch_tc(", "bool make_map("),
                   r"#define ITTT_(?:PAIR|PDL|STAGES_GATED|CONV_IN_GATED|TARGET_CONV) .*"),
    # the forward's steps 3-5: the fused scan, the apply and (prefix form) the
    # dual-form kernels of chunks 0-1, or the one-launch kernel when built so
    "recurrence": (("common.cuh", "simt.cuh", "tc_gemm.cuh", "tc_recur.cuh"),
                   ("ittt_status recurrence_bf16(", "ittt_status scan_bf16(",
                    "ittt_status apply_bf16(", "ittt_status gram_bf16(", "ittt_status dualo_bf16(",
                    "ittt_status recur_fused_bf16(", "ittt_status launch_tc(", "bool make_map(",
                    "bool make_map_3d(", "bool make_store_map(", "Layout plan("),
                   r"#define ITTT_(?:PAIR|PDL|FUSED_RECUR|TAIL_DUAL|STAGES_\w+|MCAST_COMMIT|"
                   r"RECUR_\w+|SCAN_\w+|APPLY_\w+|ETA_IN_VHAT) .*"),
}


def kernel_source_hash(kernel: str = "gated_gemm") -> str:
    """Hash of the sources that define `kernel` (see KERNEL_SOURCES).  DRAM
    traffic recorded from an ncu capture of another build is not reported."""
    import hashlib
    import re

    headers, funcs, macros = KERNEL_SOURCES[kernel]
    csrc = os.path.join(ROOT, "weight_gated_mlp_b200", "csrc")
    h = hashlib.sha256()
    for name in headers:
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(name.encode() + b"\0" + fh.read())
    api = open(os.path.join(csrc, "api.cu")).read()
    for head in funcs:
        i = api.find(head)
        j = api.find("\n}\n", i)
        h.update(api[i:j].encode() if i >= 0 else head.encode())
    for m in re.findall(macros, api):
        h.update(m.encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload_name: str):
    """DRAM bytes per launch from profiles/dram_traffic.txt if recorded for this build."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    want = kernel_source_hash(kernel)
    for ln in lines:
        parts = ln.split()
        if len(parts) >= 4 and not ln.startswith("#") and parts[0] == kernel and \
                parts[1] == workload_name and parts[3] == want:
            return float(parts[2])
    return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def choose_peak_kind(region_s: float, clock_summary: dict) -> str:
    """Which measured GEMM peak a kernel timed in this run is held against.

    The burst figure (a short cuBLAS run at full clocks) for a timed region
    shorter than a second whose median SM clock stayed within 5% of the
    maximum; the sustained figure (seconds of back-to-back GEMMs under the
    power cap) for a longer region or one where the clocks had dropped."""
    sm, smax = clock_summary.get("sm_mhz"), clock_summary.get("sm_max_mhz")
    full_clock = sm is None or smax is None or sm >= 0.95 * smax
    return "burst" if region_s < 1.0 and full_clock else "sustained"


class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU while the timed
    region runs: NVML read-only queries every 10 ms (the device matched by PCI
    bus id), else nvidia-smi every 100 ms."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (all but "gpu_idle")
    REASON_BITS = {"applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
                   "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
                   "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.samples = []          # (sm_mhz, reason bits) from NVML
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.source = None

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        try:
            import torch

            pr = torch.cuda.get_device_properties(self.gpu)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll(self, nv, h):
        reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), reasons(h)))
            except Exception:
                pass
            self._stop.wait(0.01)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self._t.start()
            self.source = "nvml"
            return self
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
            self.source = "nvidia-smi"
            t0 = time.time()
            while not self.lines and time.time() - t0 < 2.0:   # first sample before timing
                time.sleep(0.01)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        elif self._t is not None:
            self._t.join(timeout=1)
        return False

    def summary(self):
        sm, mx, reasons = [], self.max_mhz, set()
        for mhz, bits in self.samples:
            sm.append(float(mhz))
            for name, bit in self.REASON_BITS.items():
                if bits & bit:
                    reasons.add(name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_min_mhz": min(sm) if sm else None,
                "sm_max_mhz": float(mx) if mx is not None else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


def cpu_oracle_rate(w, budget_s: float, seed: int = 0):
    """Tokens/s of the CPU fp64 oracle (sequential chunk loop) on a bounded sample."""
    import numpy as np
    from oracle import ittt_oracle as orc
    from synthetic import make_inputs

    inp = make_inputs(w, seed=seed)
    H, X0 = inp["H"][0], inp["X0"][0]
    W = inp["W_down0"].astype(np.float64)
    Wt = inp["W_target"].astype(np.float64)
    done = 0
    t0 = time.perf_counter()
    for i, (s, e) in enumerate(orc.chunk_bounds(w.T, w.C)):
        Z_i = orc.gated_activations(H[s:e], inp["W_gate"], inp["W_up"])
        V_i = orc.lookahead_conv(X0[s:min(e + w.k - 1, w.T)], inp["conv_kernel"])[: e - s] @ Wt
        _, W = orc.apply_then_update(Z_i, V_i, W, w.eta)
        done += e - s
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return done / dt, done, dt


def blas_threads():
    """Threads numpy's BLAS runs the oracle's matrix products with (what the
    CPU baseline actually used); the CPU affinity count if it cannot be read."""
    import numpy  # noqa: F401  (loads the BLAS whose pool is read)
    try:
        from threadpoolctl import threadpool_info
        pools = [p for p in threadpool_info() if p.get("user_api") == "blas"]
        if pools:
            return max(int(p["num_threads"]) for p in pools)
    except Exception:
        pass
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def blas_name():
    """numpy's BLAS library and version, e.g. "openblas 0.3.30", or "unknown"."""
    import numpy  # noqa: F401
    try:
        from threadpoolctl import threadpool_info
        pools = [p for p in threadpool_info() if p.get("user_api") == "blas"]
        if pools:
            return f"{pools[0].get('internal_api', '?')} {pools[0].get('version', '?')}"
    except Exception:
        pass
    return "unknown"


def run_reference(args, w):
    """--impl reference: the CPU oracle, one chunk of the workload per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    from oracle import ittt_oracle as orc
    from synthetic import make_inputs

    inp = make_inputs(w, seed=0)
    H, X0 = inp["H"][0], inp["X0"][0]
    W = inp["W_down0"].astype(np.float64)
    Wt = inp["W_target"].astype(np.float64)
    bounds = orc.chunk_bounds(w.T, w.C)
    times = []
    for it in range(args.warmup + args.steps):
        s, e = bounds[it % len(bounds)]
        if it % len(bounds) == 0:
            W = inp["W_down0"].astype(np.float64)
        t0 = time.perf_counter()
        Z_i = orc.gated_activations(H[s:e], inp["W_gate"], inp["W_up"])
        V_i = orc.lookahead_conv(X0[s:min(e + w.k - 1, w.T)], inp["conv_kernel"])[: e - s] @ Wt
        _, W = orc.apply_then_update(Z_i, V_i, W, w.eta)
        dt = time.perf_counter() - t0
        if it >= args.warmup:
            times.append(dt)
    ms = 1e3 * statistics.mean(times)
    tok_s = w.C / (ms / 1e3)
    cores = blas_threads()
    sample = f"one chunk ({w.C} tokens of {w.T}) of the sequential fp64 chunk loop per step"
    line = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded, shapes of the workload)",
            "config": config_of(w, "sequential"),
            "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample, "blas": blas_name()},
            "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's step time (every rank must call this, in the same order)."""
    import torch

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(tokens_per_rank: int, world: int, max_ms: float) -> float:
    """Tokens/s of the whole job: every rank's batch divided by the slowest rank's time."""
    return world * tokens_per_rank / (max_ms / 1e3)


def input_mb(w) -> float:
    """MB of one forward's inputs: H, X0 and the weights."""
    es = 2 if w.dtype == "bf16" else 4
    return es * (2 * w.B * w.T * w.d + 3 * w.d * w.f + w.d * w.d + w.d * w.k) / 1e6


def config_of(w, form):
    return {"workload": w.name, "B": w.B, "T": w.T, "d_model": w.d, "d_ff": w.f, "C": w.C,
            "k": w.k, "eta": w.eta, "form": form,
            "l2": "flushed before every timed step (256 MiB write)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--form", default="auto", choices=["auto", "prefix", "dual", "hybrid"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of CPU oracle time for cpu_baseline (0 disables)")
    ap.add_argument("--only", default=None,
                    choices=["gated", "conv", "target", "scan", "apply", "recur", "clip",
                             "forward"],
                    help="profiling aid: run one step entry point --warmup + --steps times "
                         "and exit (no JSON line)")
    ap.add_argument("--T", type=int, default=None, help="override the workload's T (profiling)")
    ap.add_argument("--C", type=int, default=None, help="override the workload's C (--compare-forms)")
    ap.add_argument("--B", type=int, default=None, help="override the workload's B (--compare-forms)")
    ap.add_argument("--paired", action="store_true",
                    help="--compare-forms: run the forms in turn within every step (launch by launch) "
                         "and report each form's median ratio to the first form's time in the same step")
    ap.add_argument("--decode", type=int, default=0, metavar="B",
                    help="time the decode step for B lockstep sequences (1..8) instead of prefill")
    ap.add_argument("--clip", type=float, default=0.0,
                    help="update-norm clipping bound tau (0 = off; qwen3-4b chunk deltas are ~0.61)")
    ap.add_argument("--cp-segments", type=int, default=0, metavar="G",
                    help="time the context-parallel steps for one sequence cut into G segments, "
                         "run in turn on this GPU (per-rank compute of a G-rank run)")
    ap.add_argument("--l2", default="flush", choices=["flush", "none"],
                    help="between timed steps: flush L2 with a 256 MiB write (default), or none "
                         "(every step's inputs, 247 MB at qwen3-4b, exceed the 126 MB L2 anyway)")
    ap.add_argument("--cp", action="store_true",
                    help="context parallelism: one sequence of the workload split over the ranks "
                         "(launch one rank per GPU with torchrun; strong scaling)")
    ap.add_argument("--sweep-forms", action="store_true",
                    help="time the prefix and dual forms over a (T, C) grid at the workload's "
                         "widths and print one JSON line per point (the data behind AUTO)")
    ap.add_argument("--sweep-T", default="1024,2048,4096,8192,16384",
                    help="--sweep-forms: comma-separated sequence lengths")
    ap.add_argument("--sweep-B", default="1", help="--sweep-forms: comma-separated batch sizes")
    ap.add_argument("--compare-forms", default=None, metavar="FORMS",
                    help="comma-separated forms (prefix,dual,hybrid) timed at the workload's own "
                         "T and C, one JSON line with time, workspace and the outputs' distance "
                         "from the first form's")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from synthetic import workload

    w = workload(args.workload)
    if args.T is not None:
        w = w.with_(T=args.T)
    if args.C is not None:
        w = w.with_(C=args.C)
    if args.B is not None:
        w = w.with_(B=args.B)
    if (args.T, args.C, args.B) != (None, None, None):  # another shape: another name
        w = w.with_(name=f"{w.name}[B={w.B},T={w.T},C={w.C}]")
    if args.only is not None:
        return run_only(args, w)
    if args.sweep_forms:
        return sweep_forms(args, w)
    if args.compare_forms:
        return compare_forms(args, w)
    if args.decode:
        return decode_bench(args, w)
    if args.cp_segments:
        return cp_bench(args, w)
    if args.cp:
        return cp_run(args, w)
    if args.impl == "reference":
        return run_reference(args, w)

    # the CPU baseline runs before any CUDA work (numpy BLAS threads, no fork after CUDA)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    cpu = None
    if rank == 0 and world == 1 and args.cpu_budget > 0:
        rate, tokens, secs = cpu_oracle_rate(w, args.cpu_budget)
        cpu = {"value": rate, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"first {tokens} tokens ({tokens // w.C} chunks) of the workload, "
                         f"sequential fp64 chunk loop, {secs:.1f} s", "blas": blas_name()}

    import numpy as np
    import torch

    import weight_gated_mlp_b200 as ittt
    from synthetic import make_inputs

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    inp = make_inputs(w, seed=rank)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dev = {k: torch.from_numpy(v).to("cuda", tdt).contiguous() for k, v in inp.items()}
    del inp
    p = ittt.problem_from(dev["H"], dev["W_gate"], dev["conv_kernel"], w.eta, w.C, args.form,
                          args.clip)
    ws = torch.empty(ittt.workspace_size(p), dtype=torch.uint8, device="cuda")
    O = torch.empty((w.B, w.T, w.d), dtype=tdt, device="cuda")
    Wf = torch.empty((w.B, w.d, w.f), dtype=torch.float32, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        ittt.fast_mlp_forward(dev["H"], dev["X0"], dev["W_gate"], dev["W_up"], dev["W_down0"],
                              dev["conv_kernel"], dev["W_target"], w.eta, w.C, form=args.form,
                              workspace=ws, out=O, w_final=Wf, stream=stream, clip=args.clip)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = ittt.get_last_error()
    if st != ittt.OK:
        raise SystemExit(f"device error: {ittt.status_string(st)}")

    # ---- timed region: K steps, L2 flushed before each, events on the stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    # the dominant kernel (gate/up GEMM) timed inside every timed forward by the
    # library's probe: CUDA events on the stream around its launch
    ittt.probe_start(args.steps)
    with ClockSampler(local_rank) as clocks:
        for i in range(args.steps):
            if args.l2 == "flush":
                flush.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    gated_live_ms, recur_live_ms = ittt.probe_read2(args.steps)
    if dist is not None:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    ms = statistics.mean(step_ms)
    qs = statistics.quantiles(step_ms, n=10) if len(step_ms) >= 10 else [min(step_ms), max(step_ms)]
    step_dist = {"min": min(step_ms), "p10": qs[0], "median": statistics.median(step_ms),
                 "p90": qs[-1], "max": max(step_ms),
                 "first10_mean": statistics.mean(step_ms[:10]),
                 "last10_mean": statistics.mean(step_ms[-10:])}
    if dist is not None:
        ms = max_over_ranks(ms, dist, "cuda")
    tokens = w.B * w.T
    value = whole_job_rate(tokens, world, ms)
    flops = w.flops()

    # ---- per-kernel breakdown through the step entry points (same kernels)
    breakdown = kernel_breakdown(ittt, dev, w, ws, flush, stream, args)
    launches_per_step = breakdown.pop("_launches")
    resolved_form = breakdown.pop("_form")

    # ---- end to end: pinned host inputs in, results out, inside the timed region
    e2e = end_to_end(ittt, dev, w, args, stream)
    e2e["with_state_to_host"] = {k: v for k, v in end_to_end(ittt, dev, w, args, stream, True).items()
                                 if k != "note"}

    # ---- context: the same shapes through torch / cuBLAS (not this library)
    context = library_context(dev, w, flush, ms)

    peaks, peak_src = load_peaks()
    bf16_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    bf16_sustained = float(peaks.get("bf16_tflops_sustained",
                                     FALLBACK_PEAKS["bf16_tflops_sustained"]))
    clock_summary = clocks.summary()
    region_s = sum(step_ms) / 1e3
    peak_kind = choose_peak_kind(region_s, clock_summary)
    peak = bf16_peak if peak_kind == "burst" else bf16_sustained
    # the library's default build runs the look-ahead conv as its own kernel after the
    # gate/up GEMM, outside the probed events (a build with the conv warps in the
    # gate/up kernel would time both together)
    conv_beside = False
    stack_bytes = 2.0 * w.B * (w.n_chunks - 1) * w.d * w.f
    live = {
        # kernel: (name in the line, live times, algorithmic FLOP, algorithmic bytes)
        "gated_gemm": ("gated_gemm (tc_gemm_kernel<TC_GATED>" +
                       (", with the look-ahead conv beside it)" if conv_beside else ")"),
                       gated_live_ms, 4.0 * w.B * w.T * w.d * w.f,
                       2.0 * w.B * w.T * (w.d + w.f) + 4.0 * w.d * w.f +
                       (4.0 * w.B * w.T * w.d if conv_beside else 0.0)),
        "recurrence": ("recurrence (the forward's steps 3-5, " + resolved_form + " form: " +
                       ("the fused scan, then the apply; chunks 0-1 by the dual-form kernels "
                        "beside the scan" if resolved_form == "prefix" else "its kernels") + ")",
                       recur_live_ms, 4.0 * w.B * w.T * w.d * w.f,
                       # Vhat, Z in and O out; Z again and W_down0 twice; the stack
                       # written and read; W_down_final written (fp32)
                       4.0 * w.B * w.T * (w.d + w.f) + 4.0 * w.d * w.f + 2 * stack_bytes +
                       4.0 * w.B * w.d * w.f),
    }

    def roofline(kernel):
        name, times, fl, nbytes = live[kernel]
        kms = statistics.mean(times) if times else breakdown[kernel]["ms"]
        ach = fl / (kms / 1e3) / 1e12
        return {"kernel": name, "bound": "tensor", "achieved": ach, "peak": peak,
                "unit": "TFLOP/s", "frac": ach / peak,
                "traffic": recorded_traffic(kernel, w.name), "traffic_algorithmic_bytes": nbytes,
                "kernel_ms": kms,
                "timing": "CUDA events on the launching stream around the kernel in every timed "
                          f"forward ({len(times)} launches)",
                "peak_kind": peak_kind,
                "peak_source": f"{peak_src} bf16_tflops" + ("" if peak_kind == "burst" else "_sustained"),
                "timed_region_s": region_s,
                "frac_of_burst_peak": ach / bf16_peak,
                "frac_of_sustained_peak": ach / bf16_sustained}

    # the forward's recurrence as probed in the timed forwards (scan + apply timed alone otherwise)
    breakdown["recurrence"] = {"ms": statistics.mean(recur_live_ms) if recur_live_ms else
                               breakdown["scan_fused"]["ms"] + breakdown["apply_gemm"]["ms"],
                               "tflops": 4.0 * w.B * w.T * w.d * w.f / 1e12 / (
                                   (statistics.mean(recur_live_ms) if recur_live_ms else
                                    breakdown["scan_fused"]["ms"] + breakdown["apply_gemm"]["ms"]) / 1e3)}
    roofs = {k: roofline(k) for k in live}
    dominant = max(roofs, key=lambda k: roofs[k]["kernel_ms"])
    roof = roofs[dominant]
    roof_other = roofs["recurrence" if dominant == "gated_gemm" else "gated_gemm"]

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic (seeded normal inputs and random weights of the workload's shapes)",
            "config": dict(config_of(w, args.form), resolved_form=resolved_form, clip=args.clip,
                           **({} if args.l2 == "flush" else {
                               "l2": "not flushed: every step reads its inputs H, X0 and the "
                                     "weights (%.0f MB) and streams a %.0f MB workspace, against "
                                     "a 126 MB L2" % (input_mb(w), ws.numel() / 1e6)})),
            "tflops": world * flops / (ms / 1e3) / 1e12,
            "frac_of_bf16_peak": world * flops / (ms / 1e3) / 1e12 / bf16_peak,
            "roofline": roof, "roofline_other": roof_other, "kernels": breakdown,
            "gpu_launches": launches_per_step * args.steps,
            "e2e": e2e, "clocks": clock_summary, "step_ms": step_dist, "cpu_baseline": cpu,
            "context": context,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def library_context(dev, w, flush, forward_ms):
    """Context rows timed with torch (cuBLAS), median of 10 after 3 warm-ups, L2
    flushed: the plain gated MLP of the same shape (silu(H W_gate^T) * (H W_up^T)
    then the W_down0 projection, 6 B T d f FLOP), the per-layer analogue of the
    pages' overhead figure; and one bf16 GEMM of the gate/up shape."""
    import torch

    if w.dtype != "bf16":
        return None
    H = dev["H"].reshape(-1, w.d)
    Wgu = torch.cat([dev["W_gate"], dev["W_up"]], dim=0)          # [2f, d]

    def plain():
        gu = H @ Wgu.t()
        z = torch.nn.functional.silu(gu[:, : w.f]) * gu[:, w.f:]
        return z @ dev["W_down0"].t()

    def gemm():
        return H @ Wgu.t()

    def timed(fn):
        ts = []
        for it in range(13):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if it >= 3:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    plain_ms, gemm_ms = timed(plain), timed(gemm)
    BT = w.B * w.T
    return {"torch_plain_gated_mlp_ms": plain_ms,
            "forward_over_plain_mlp": forward_ms / plain_ms,
            "torch_gate_up_gemm_ms": gemm_ms,
            "torch_gate_up_gemm_tflops": 4.0 * BT * w.d * w.f / (gemm_ms / 1e3) / 1e12}


def _time_forms(args, w, dev, forms, flush, keep=False):
    """Median whole-forward time (ms) and workspace bytes of each form on the
    same device inputs; with keep, also the outputs (O, W_down_final)."""
    import statistics as st

    import torch

    import weight_gated_mlp_b200 as ittt

    res, outs = {}, {}
    O = torch.empty((w.B, w.T, w.d), dtype=torch.bfloat16, device="cuda")
    Wf = torch.empty((w.B, w.d, w.f), dtype=torch.float32, device="cuda")
    for form in forms:
        p = ittt.problem_from(dev["H"], dev["W_gate"], dev["conv_kernel"], w.eta, w.C, form)
        ws = torch.empty(ittt.workspace_size(p), dtype=torch.uint8, device="cuda")
        ts = []
        for it in range(args.warmup + args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            ittt.fast_mlp_forward(dev["H"], dev["X0"], dev["W_gate"], dev["W_up"],
                                  dev["W_down0"], dev["conv_kernel"], dev["W_target"], w.eta, w.C,
                                  form=form, workspace=ws, out=O, w_final=Wf)
            b.record()
            torch.cuda.synchronize()
            if it >= args.warmup:
                ts.append(a.elapsed_time(b))
        if ittt.get_last_error() != ittt.OK:
            raise RuntimeError(f"form {form}: {ittt.status_string(ittt.get_last_error())}")
        res[form] = (st.median(ts), ws.numel(), ittt.resolve_form(p))
        if keep:
            outs[form] = (O.float(), Wf.clone())
        del ws
    return res, outs


def _time_forms_paired(args, w, dev, forms, flush):
    """Like _time_forms, but every step runs each form once in turn (L2 flushed
    before each forward), so the forms share the box's thermal state; also the
    median and quartiles over steps of each form's time divided by the first
    form's in the same step."""
    import statistics as st

    import torch

    import weight_gated_mlp_b200 as ittt

    O = {f: torch.empty((w.B, w.T, w.d), dtype=torch.bfloat16, device="cuda") for f in forms}
    Wf = {f: torch.empty((w.B, w.d, w.f), dtype=torch.float32, device="cuda") for f in forms}
    ps = {f: ittt.problem_from(dev["H"], dev["W_gate"], dev["conv_kernel"], w.eta, w.C, f) for f in forms}
    ws = {f: torch.empty(ittt.workspace_size(ps[f]), dtype=torch.uint8, device="cuda") for f in forms}
    ts = {f: [] for f in forms}
    for it in range(args.warmup + args.steps):
        for form in forms:
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            ittt.fast_mlp_forward(dev["H"], dev["X0"], dev["W_gate"], dev["W_up"],
                                  dev["W_down0"], dev["conv_kernel"], dev["W_target"], w.eta, w.C,
                                  form=form, workspace=ws[form], out=O[form], w_final=Wf[form])
            b.record()
            torch.cuda.synchronize()
            if it >= args.warmup:
                ts[form].append(a.elapsed_time(b))
        if ittt.get_last_error() != ittt.OK:
            raise RuntimeError(f"forms {forms}: {ittt.status_string(ittt.get_last_error())}")
    res = {f: (st.median(ts[f]), ws[f].numel(), ittt.resolve_form(ps[f])) for f in forms}
    outs = {f: (O[f].float(), Wf[f]) for f in forms}
    ratios = {}
    for f in forms:
        r = sorted(x / y for x, y in zip(ts[f], ts[forms[0]]))
        ratios[f] = {"median": round(st.median(r), 4), "p25": round(r[len(r) // 4], 4),
                     "p75": round(r[(3 * len(r)) // 4], 4), "n": len(r)}
    return res, outs, ratios


def sweep_forms(args, base):
    """Whole-forward time of the prefix and the dual form over (T, C)."""
    import torch

    from synthetic import make_inputs

    torch.cuda.set_device(0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    Ts = [int(x) for x in args.sweep_T.split(",")]
    Bs = [int(x) for x in args.sweep_B.split(",")]
    grid = [(B, T, C) for B in Bs for T in Ts for C in (256, 512, 1024, 2048)
            if C < T and T % C == 0]
    for B, T, C in grid:
        w = base.with_(T=T, C=C, B=B)
        inp = make_inputs(w, seed=0)
        dev = {k: torch.from_numpy(v).to("cuda", torch.bfloat16).contiguous() for k, v in inp.items()}
        res, _ = _time_forms(args, w, dev, ("prefix", "dual"), flush)
        ms = {k: v[0] for k, v in res.items()}
        if res["dual"][2] != "dual":   # fp32 runs the prefix form for every request
            raise RuntimeError("the dual form does not run at this shape")
        print(json.dumps({"sweep": "forms", "B": B, "d": w.d, "f": w.f, "T": T, "C": C,
                          "prefix_ms": ms["prefix"], "dual_ms": ms["dual"],
                          "faster": min(ms, key=ms.get)}), flush=True)
    return 0


def compare_forms(args, w):
    """The listed forms at the workload's own T and C: time, workspace, and
    the normwise distance of O and W_down_final from the first form's."""
    import torch

    from synthetic import make_inputs

    torch.cuda.set_device(0)
    forms = [f.strip() for f in args.compare_forms.split(",") if f.strip()]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    inp = make_inputs(w, seed=0)
    dev = {k: torch.from_numpy(v).to("cuda", torch.bfloat16).contiguous() for k, v in inp.items()}
    del inp
    if args.paired:
        res, outs, ratios = _time_forms_paired(args, w, dev, forms, flush)
    else:
        res, outs = _time_forms(args, w, dev, forms, flush, keep=True)
        ratios = {}
    O0, W0 = outs[forms[0]]

    def rel(a, b):
        return float((a - b).norm() / b.norm())

    line = {"compare": "forms", "workload": w.name, "B": w.B, "T": w.T, "C": w.C, "d": w.d,
            "f": w.f, "steps": args.steps, "warmup": args.warmup,
            "l2": "flushed before every forward (256 MiB write)",
            "timing": "forms in turn within each step" if args.paired else "each form's steps in a block"}
    for form in forms:
        ms, nbytes, ran = res[form]
        line[form] = {"ran": ran, "ms": round(ms, 4),
                      "tflops": round(w.flops() / (ms / 1e3) / 1e12, 1),
                      "workspace_gib": round(nbytes / 2**30, 3),
                      "rel_O": rel(outs[form][0], O0), "rel_W_final": rel(outs[form][1], W0)}
        if form in ratios:
            line[form]["paired_ratio"] = ratios[form]
    print(json.dumps(line), flush=True)
    return 0


def decode_bench(args, w):
    """Per-token time of the decode step (chunk-end padding) at the workload's widths."""
    import torch

    import weight_gated_mlp_b200 as ittt
    from synthetic import make_inputs

    torch.cuda.set_device(0)
    B = args.decode
    inp = make_inputs(w.with_(T=2 * w.C, B=B), seed=0)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dev = {k: torch.from_numpy(v).to("cuda", tdt).contiguous() for k, v in inp.items()}
    dec = ittt.Decoder(dev["W_gate"], dev["W_up"], dev["W_down0"], dev["conv_kernel"],
                       dev["W_target"], B, w.eta, w.C, clip=args.clip)
    H = dev["H"].transpose(0, 1).contiguous()   # [T, B, d]
    X = dev["X0"].transpose(0, 1).contiguous()
    out = torch.empty((B, w.d), dtype=tdt, device="cuda")
    tok_ms, upd_ms = [], []
    # one token at a time, synchronised: the latency of a step as called
    for t in range(2 * w.C):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dec.step(H[t], X[t], out=out)
        b.record()
        torch.cuda.synchronize()
        if t >= w.C:  # second chunk: warm
            (upd_ms if (t + 1) % w.C == 0 else tok_ms).append(a.elapsed_time(b))
    # the C - 1 tokens before a chunk's end back to back: the device time per
    # token once the host runs ahead of the GPU
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = 2 * w.C
    dec.step(H[t0 % (2 * w.C)], X[t0 % (2 * w.C)], out=out)   # position 0 of a chunk
    a.record()
    for t in range(1, w.C - 1):
        dec.step(H[t], X[t], out=out)
    b.record()
    torch.cuda.synchronize()
    pipe_ms = a.elapsed_time(b) / (w.C - 2)
    # the same through CUDA graphs (one per chunk position, the token's rows
    # copied into the graphs' input buffers): synchronised and back to back
    dec.capture()
    while dec.pos % w.C:
        dec.replay(H[dec.pos % (2 * w.C)], X[dec.pos % (2 * w.C)])
    torch.cuda.synchronize()
    g_tok = []
    for t in range(w.C - 1):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dec.replay(H[t], X[t])
        b.record()
        torch.cuda.synchronize()
        if t > 0:
            g_tok.append(a.elapsed_time(b))
    dec.replay(H[w.C - 1], X[w.C - 1])          # chunk end
    dec.replay(H[0], X[0])
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for t in range(1, w.C - 1):
        dec.replay(H[t], X[t])
    b.record()
    torch.cuda.synchronize()
    g_pipe_ms = a.elapsed_time(b) / (w.C - 2)
    st = ittt.get_last_error()
    es = 2 if w.dtype == "bf16" else 4
    # per token: W_gate + W_up, and the state the apply GEMV reads (its bf16
    # rounding on the bf16 path, the fp32 state on the fp32 path)
    weight_bytes = 2 * w.f * w.d * es + B * w.d * w.f * es
    ms = statistics.median(tok_ms)
    print(json.dumps({"decode": {"workload": w.name, "B": B, "C": w.C, "dtype": w.dtype,
                                 "token_ms_median": ms, "tokens_per_s": B / (ms / 1e3),
                                 "weight_GBps": weight_bytes / (ms / 1e3) / 1e9,
                                 "pipelined_token_ms": pipe_ms,
                                 "pipelined_weight_GBps": weight_bytes / (pipe_ms / 1e3) / 1e9,
                                 "graph_token_ms_median": statistics.median(g_tok),
                                 "graph_pipelined_token_ms": g_pipe_ms,
                                 "graph_pipelined_weight_GBps":
                                     weight_bytes / (g_pipe_ms / 1e3) / 1e9,
                                 "chunk_end_step_ms": upd_ms[-1] if upd_ms else None,
                                 "status": ittt.status_string(st)}}), flush=True)
    return 0 if st == ittt.OK else 1


def cp_bench(args, w):
    """Context-parallel steps of one sequence cut into G segments, each timed
    on its own (CUDA events, L2 flushed before each): what one rank of a
    G-rank run computes, next to the one-GPU forward of the whole sequence.
    The NCCL exchange is not run here (one GPU); its bytes are reported."""
    import torch

    import weight_gated_mlp_b200 as ittt
    from synthetic import make_inputs
    from weight_gated_mlp_b200 import parallel

    torch.cuda.set_device(0)
    G = args.cp_segments
    if w.T % (G * w.C):
        raise SystemExit(f"T = {w.T} does not split into {G} segments of whole chunks")
    inp = make_inputs(w, seed=0)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dev = {k: torch.from_numpy(v).to("cuda", tdt).contiguous() for k, v in inp.items()}
    del inp
    ops = parallel.CudaSegmentOps(dev["W_gate"], dev["W_up"], dev["W_down0"], dev["conv_kernel"],
                                  dev["W_target"], w.eta, w.C, clip=args.clip)
    Tr, k = w.T // G, w.k
    segs = []
    for r in range(G):
        s, e = r * Tr, (r + 1) * Tr
        stop = e + (k - 1 if r < G - 1 else 0)
        segs.append((dev["H"][:, s:e].contiguous(), dev["X0"][:, s:stop].contiguous()))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    S_all = torch.empty((G, w.B, w.d, w.f), dtype=torch.float32, device="cuda")

    def timed(fn):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        out = fn()
        b.record()
        return out, (a, b)

    rec = {"delta": [], "prefix": [], "apply": [], "forward": []}
    for it in range(args.warmup + args.steps):
        ev = {"delta": [], "prefix": [], "apply": [], "forward": []}
        states = []
        for r, (H, X) in enumerate(segs):
            (_, st), e = timed(lambda: ops.delta(H, X, S_out=S_all[r]))
            states.append(st)
            ev["delta"].append(e)
        P_all, e = timed(lambda: ops.prefix(S_all))
        ev["prefix"].append(e)
        for r in range(G):
            _, e = timed(lambda: ops.apply(states[r], P_all[r]))
            ev["apply"].append(e)
        _, e = timed(lambda: ittt.fast_mlp_forward(dev["H"], dev["X0"], dev["W_gate"], dev["W_up"],
                                                   dev["W_down0"], dev["conv_kernel"],
                                                   dev["W_target"], w.eta, w.C, clip=args.clip))
        ev["forward"].append(e)
        torch.cuda.synchronize()
        if it >= args.warmup:
            for key, evs in ev.items():
                rec[key].append(sum(a.elapsed_time(b) for a, b in evs))
    st = ittt.get_last_error()
    med = {key: statistics.median(v) for key, v in rec.items()}
    dfb = 4 * w.B * w.d * w.f
    xbytes = 2 * (G - 1) / G * dfb + (k - 1) * w.B * w.d * (2 if w.dtype == "bf16" else 4)
    rank_ms = (med["delta"] + med["apply"]) / G + med["prefix"] / G
    peer_gbs = 770.0
    xms = xbytes / (peer_gbs * 1e9) * 1e3
    print(json.dumps({"context_parallel": {
        "workload": w.name, "segments": G, "segment_tokens": Tr, "clip": args.clip,
        "delta_ms_per_segment": med["delta"] / G, "apply_ms_per_segment": med["apply"] / G,
        "prefix_ms_all_rows": med["prefix"], "rank_compute_ms": rank_ms,
        "forward_ms_one_gpu": med["forward"],
        "compute_overhead": (med["delta"] + med["apply"]) / med["forward"] - 1.0,
        "exchange_bytes_per_rank": xbytes,
        "exchange_ms_at_770GBps": xms,
        "projected_tokens_per_s": w.B * w.T / ((rank_ms + xms) / 1e3),
        "one_gpu_tokens_per_s": w.B * w.T / (med["forward"] / 1e3),
        "status": ittt.status_string(st)}}), flush=True)
    return 0 if st == ittt.OK else 1


def cp_run(args, w):
    """The workload's sequences split over the ranks (context parallelism over
    NCCL): rank r runs segment r of every sequence through
    parallel.context_parallel_forward.  Timed like the main mode: warm-up, K
    steps between barriers with CUDA events, L2 flushed, max over ranks; value
    = the whole sequences' tokens / the slowest rank's time (strong scaling)."""
    import datetime
    import socket

    import torch
    import torch.distributed as dist

    import weight_gated_mlp_b200 as ittt
    from synthetic import make_inputs
    from weight_gated_mlp_b200 import parallel

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if w.T % (world * w.C):
        raise SystemExit(f"T = {w.T} does not split into {world} segments of whole chunks")
    torch.cuda.set_device(local_rank)
    if "MASTER_ADDR" not in os.environ:      # one process without torchrun
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(sk.getsockname()[1]))
    dist.init_process_group("nccl", rank=rank, world_size=world,
                            device_id=torch.device("cuda", local_rank),
                            timeout=datetime.timedelta(seconds=120))
    try:
        inp = make_inputs(w, seed=0)          # every rank draws the same sequences
        tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        Tr = w.T // world
        s0, s1 = rank * Tr, (rank + 1) * Tr
        H = torch.from_numpy(inp["H"][:, s0:s1].copy()).to("cuda", tdt).contiguous()
        # room for the halo (the next rank's first k-1 rows) on every rank but the last
        X = inp["X0"][:, s0:s1 + (w.k - 1 if rank < world - 1 else 0)]
        X0 = torch.from_numpy(X.copy()).to("cuda", tdt).contiguous()
        wts = {k: torch.from_numpy(inp[k]).to("cuda", tdt).contiguous()
               for k in ("W_gate", "W_up", "W_down0", "conv_kernel", "W_target")}
        del inp
        ops = parallel.CudaSegmentOps(wts["W_gate"], wts["W_up"], wts["W_down0"],
                                      wts["conv_kernel"], wts["W_target"], w.eta, w.C,
                                      clip=args.clip)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

        def step():
            return parallel.context_parallel_forward(H, X0, ops)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(local_rank) as clocks:
            for i in range(args.steps):
                flush.zero_()
                ev[i][0].record()
                step()
                ev[i][1].record()
            torch.cuda.synchronize()
        dist.barrier()
        st = ittt.get_last_error()
        ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
        ms = max_over_ranks(ms, dist, "cuda")
        if rank == 0:
            tokens = w.B * w.T
            print(json.dumps({
                "metric": METRIC, "value": tokens / (ms / 1e3), "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
                "dtype": w.dtype, "data": "synthetic (seeded normal inputs and random weights)",
                "config": dict(config_of(w, "prefix"), clip=args.clip, parallelism=f"cp{world}",
                               segment_tokens=Tr),
                "tflops": w.flops() / (ms / 1e3) / 1e12, "clocks": clocks.summary(),
                "status": ittt.status_string(st)}), flush=True)
    finally:
        dist.destroy_process_group()
    return 0 if st == ittt.OK else 1


def run_only(args, w):
    """Run one step entry point (or the whole forward) repeatedly, for ncu captures."""
    import ctypes

    import torch

    import weight_gated_mlp_b200 as ittt
    from synthetic import make_inputs

    torch.cuda.set_device(0)
    inp = make_inputs(w, seed=0)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dev = {k: torch.from_numpy(v).to("cuda", tdt).contiguous() for k, v in inp.items()}
    lib = ittt.load_library()
    p = ittt.problem_from(dev["H"], dev["W_gate"], dev["conv_kernel"], w.eta, w.C, args.form)
    B, T, d, f, n = w.B, w.T, w.d, w.f, w.n_chunks
    ws = torch.empty(ittt.workspace_size(p), dtype=torch.uint8, device="cuda")
    Z = ittt.gated_activations(dev["H"], dev["W_gate"], dev["W_up"])
    V = ittt.lm_target(dev["X0"], dev["conv_kernel"], dev["W_target"], C=w.C)
    Y = torch.empty((B, T, d), dtype=tdt, device="cuda")
    stack = torch.empty((B, max(n - 1, 1), d, f), dtype=tdt, device="cuda")
    Wf = torch.empty((B, d, f), dtype=torch.float32, device="cuda")
    O = torch.empty((B, T, d), dtype=tdt, device="cuda")
    assert lib.ittt_fast_weight_scan(ctypes.byref(p), V.data_ptr(), Z.data_ptr(),
                                     dev["W_down0"].data_ptr(), stack.data_ptr(), Wf.data_ptr(),
                                     None) == 0
    P = ctypes.byref(p)
    pc = ittt.problem_from(dev["H"], dev["W_gate"], dev["conv_kernel"], w.eta, w.C, args.form,
                           args.clip if args.clip > 0 else 0.3)
    norms = torch.empty((B, n), dtype=torch.float32, device="cuda")
    fn = {
        "gated": lambda: lib.ittt_gated_activations(P, dev["H"].data_ptr(), dev["W_gate"].data_ptr(),
                                                    dev["W_up"].data_ptr(), Z.data_ptr(), None),
        "conv": lambda: lib.ittt_lookahead_conv(P, dev["X0"].data_ptr(), dev["conv_kernel"].data_ptr(),
                                                Y.data_ptr(), None),
        "target": lambda: lib.ittt_lm_target(P, dev["X0"].data_ptr(), dev["conv_kernel"].data_ptr(),
                                             dev["W_target"].data_ptr(), V.data_ptr(), ws.data_ptr(),
                                             ws.numel(), None),
        "scan": lambda: lib.ittt_fast_weight_scan(P, V.data_ptr(), Z.data_ptr(),
                                                  dev["W_down0"].data_ptr(), stack.data_ptr(),
                                                  Wf.data_ptr(), None),
        "apply": lambda: lib.ittt_apply(P, Z.data_ptr(), dev["W_down0"].data_ptr(), stack.data_ptr(),
                                        O.data_ptr(), None),
        "recur": lambda: lib.ittt_chunk_recurrence(P, Z.data_ptr(), V.data_ptr(),
                                                   dev["W_down0"].data_ptr(), O.data_ptr(),
                                                   Wf.data_ptr(), ws.data_ptr(), ws.numel(), None),
        "clip": lambda: lib.ittt_clip_update_targets(ctypes.byref(pc), Z.data_ptr(), V.data_ptr(),
                                                     norms.data_ptr(), None),
        "forward": lambda: lib.ittt_fast_mlp_forward(P, dev["H"].data_ptr(), dev["X0"].data_ptr(),
                                                     dev["W_gate"].data_ptr(), dev["W_up"].data_ptr(),
                                                     dev["W_down0"].data_ptr(),
                                                     dev["conv_kernel"].data_ptr(),
                                                     dev["W_target"].data_ptr(), O.data_ptr(),
                                                     Wf.data_ptr(), ws.data_ptr(), ws.numel(), None),
    }[args.only]
    torch.cuda.synchronize()
    for _ in range(args.warmup + args.steps):
        assert fn() == 0
    torch.cuda.synchronize()
    st = ittt.get_last_error()
    print(f"only={args.only} workload={w.name} T={w.T} status={ittt.status_string(st)}")
    return 0 if st == ittt.OK else 1


def kernel_breakdown(ittt, dev, w, ws, flush, stream, args):
    """Average time of every kernel of the prefix form, timed between events."""
    import ctypes

    import torch

    lib = ittt.load_library()
    p = ittt.problem_from(dev["H"], dev["W_gate"], dev["conv_kernel"], w.eta, w.C, "prefix")
    B, T, d, f, n = w.B, w.T, w.d, w.f, w.n_chunks
    tdt = dev["H"].dtype
    Z = torch.empty((B * T, f), dtype=tdt, device="cuda")
    Y = torch.empty((B, T, d), dtype=tdt, device="cuda")
    V = torch.empty((B * T, d), dtype=tdt, device="cuda")
    stack = torch.empty((B, max(n - 1, 1), d, f), dtype=tdt, device="cuda")
    Wf = torch.empty((B, d, f), dtype=torch.float32, device="cuda")
    O = torch.empty((B, T, d), dtype=tdt, device="cuda")
    if ws.numel() < ittt.workspace_size(p):  # the forward ran another form
        ws = torch.empty(ittt.workspace_size(p), dtype=torch.uint8, device="cuda")
    s = int(stream.cuda_stream) or None
    P = ctypes.byref(p)
    steps = [
        ("gated_gemm", 4.0 * B * T * d * f, 0,
         lambda: lib.ittt_gated_activations(P, dev["H"].data_ptr(), dev["W_gate"].data_ptr(),
                                            dev["W_up"].data_ptr(), Z.data_ptr(), s)),
        ("lookahead_conv", 2.0 * B * T * d * w.k, 2 * 2 * B * T * d,
         lambda: lib.ittt_lookahead_conv(P, dev["X0"].data_ptr(), dev["conv_kernel"].data_ptr(),
                                         Y.data_ptr(), s)),
        ("target_gemm", 2.0 * B * T * d * d, 0, None),
        ("scan_fused", 2.0 * B * T * d * f, B * (n - 1) * d * f * 2 + B * d * f * 4,
         lambda: lib.ittt_fast_weight_scan(P, V.data_ptr(), Z.data_ptr(), dev["W_down0"].data_ptr(),
                                           stack.data_ptr(), Wf.data_ptr(), s)),
        ("apply_gemm", 2.0 * B * T * d * f, B * (n - 1) * d * f * 2,
         lambda: lib.ittt_apply(P, Z.data_ptr(), dev["W_down0"].data_ptr(), stack.data_ptr(),
                                O.data_ptr(), s)),
        # the recurrence step entry point: on the prefix form one persistent launch
        # of the fused scan and the apply (plus the clearing of its work counter)
        ("recurrence_one_launch", 4.0 * B * T * d * f, B * (n - 1) * d * f * 2 * 2 + B * d * f * 4,
         lambda: lib.ittt_chunk_recurrence(P, Z.data_ptr(), V.data_ptr(), dev["W_down0"].data_ptr(),
                                           O.data_ptr(), Wf.data_ptr(), ws.data_ptr(), ws.numel(), s)),
    ]
    # the target GEMM alone = lm_target minus the conv it starts with
    lm = lambda: lib.ittt_lm_target(P, dev["X0"].data_ptr(), dev["conv_kernel"].data_ptr(),
                                    dev["W_target"].data_ptr(), V.data_ptr(), ws.data_ptr(),
                                    ws.numel(), s)
    times = {name: [] for name, *_ in steps}
    lm_times = []
    reps = max(3, min(args.steps, 10))
    for it in range(reps + 2):
        for name, _, _, fn in steps:
            if fn is None:
                continue
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            assert fn() == 0, name
            b.record(stream)
            torch.cuda.synchronize()
            if it >= 2:
                times[name].append(a.elapsed_time(b))
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        assert lm() == 0
        b.record(stream)
        torch.cuda.synchronize()
        if it >= 2:
            lm_times.append(a.elapsed_time(b))
    times["target_gemm"] = [max(x - statistics.mean(times["lookahead_conv"]), 1e-6) for x in lm_times]
    if args.clip > 0:  # the clipping step (gram norms + rescale of Vhat)
        pc = ittt.make_problem(B, T, d, f, w.C, w.k, w.eta, w.dtype, clip=args.clip)
        norms = torch.empty((B, n), dtype=torch.float32, device="cuda")
        ct = []
        for it in range(reps + 2):
            assert lm() == 0  # fresh, unclipped targets
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            assert lib.ittt_clip_update_targets(ctypes.byref(pc), Z.data_ptr(), V.data_ptr(),
                                                norms.data_ptr(), s) == 0
            b.record(stream)
            torch.cuda.synchronize()
            if it >= 2:
                ct.append(a.elapsed_time(b))
        times["clip_norms"] = ct
        steps.append(("clip_norms", 2.0 * B * T * w.C * (d + f) / 2, 0, None))
    out = {}
    for name, fl, algo_bytes, _ in steps:
        ms = statistics.mean(times[name])
        out[name] = {"ms": ms, "tflops": fl / (ms / 1e3) / 1e12}
        if algo_bytes:
            out[name]["algo_GBps"] = algo_bytes / (ms / 1e3) / 1e9
    out["_launches"] = forward_launches(ittt, w, args)
    out["_form"] = ittt.resolve_form(ittt.make_problem(B, T, d, f, w.C, w.k, w.eta, w.dtype, args.form))
    return out


def forward_launches(ittt, w, args) -> int:
    """Kernels one forward launches with the library's default build: gate/up,
    conv and target GEMM, then by form (bf16): prefix — scan and apply, plus the
    gram and dual-output kernels of chunks 0-1 when there are at least three
    chunks of a multiple of 256 tokens; dual — gram, dual output and a one-chunk
    scan for W_down_final; hybrid — scan of the group starts, gram, dual output;
    eta = 0 — a W_down0 broadcast and the apply.  Clipping adds its norms and
    row-scaling kernels.  fp32: the SIMT GEMMs (gate/up, target, deltas and the
    last chunk's delta, apply of chunk 0 and of the rest), conv and scan."""
    n = w.n_chunks
    form = ittt.resolve_form(ittt.make_problem(w.B, w.T, w.d, w.f, w.C, w.k, w.eta, w.dtype, args.form))
    clip = 2 if (getattr(args, "clip", 0) > 0 and w.eta != 0) else 0
    if w.dtype != "bf16":
        return 3 + (2 if n > 1 else 1) + 1 + (2 if n > 1 else 1) + (1 if clip else 0)
    if w.eta == 0:
        return 3 + 2
    if form == "prefix":
        tail_dual = n >= 3 and w.C % 256 == 0
        return 3 + 2 + (2 if tail_dual else 0) + clip
    return 3 + 3 + clip


def end_to_end(ittt, dev, w, args, stream, state_to_host: bool = False):
    """Every step through the public call with its inputs H, X0 copied in from
    pinned host memory and its result O copied back, inside the timed region;
    with state_to_host also the fast-weight state W_down_final (fp32), which a
    caller prefilling a document in segments keeps on the device as the next
    segment's W_down0.  Steps are pipelined the way a serving loop runs them: the
    inputs of step i+1 go up on one copy stream and the results of step i-1
    come down on another while step i computes (two buffers of each, ordered by
    events), so the host-device copies overlap one another and the compute."""
    import torch

    nbuf = 2
    H_h = dev["H"].cpu().pin_memory()
    X_h = dev["X0"].cpu().pin_memory()
    H_d = [torch.empty_like(dev["H"]) for _ in range(nbuf)]
    X_d = [torch.empty_like(dev["X0"]) for _ in range(nbuf)]
    O_h = [torch.empty((w.B, w.T, w.d), dtype=dev["H"].dtype).pin_memory() for _ in range(nbuf)]
    W_h = [torch.empty((w.B, w.d, w.f), dtype=torch.float32).pin_memory() for _ in range(nbuf)]
    O = [torch.empty((w.B, w.T, w.d), dtype=dev["H"].dtype, device="cuda") for _ in range(nbuf)]
    Wf = [torch.empty((w.B, w.d, w.f), dtype=torch.float32, device="cuda") for _ in range(nbuf)]
    p = ittt.problem_from(dev["H"], dev["W_gate"], dev["conv_kernel"], w.eta, w.C, args.form)
    ws = torch.empty(ittt.workspace_size(p), dtype=torch.uint8, device="cuda")
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    uploaded = [ev() for _ in range(nbuf)]   # inputs of the buffer are on the device
    computed = [ev() for _ in range(nbuf)]   # the forward has read the inputs and written O, Wf
    fetched = [ev() for _ in range(nbuf)]    # O, Wf of the buffer are on the host
    for e in computed + fetched:
        e.record(stream)

    def upload(i):
        k = i % nbuf
        up.wait_event(computed[k])           # the forward of step i-2 is done with this buffer
        with torch.cuda.stream(up):
            H_d[k].copy_(H_h, non_blocking=True)
            X_d[k].copy_(X_h, non_blocking=True)
        uploaded[k].record(up)

    def compute(i):
        k = i % nbuf
        stream.wait_event(uploaded[k])
        stream.wait_event(fetched[k])        # the results of step i-2 have left this buffer
        ittt.fast_mlp_forward(H_d[k], X_d[k], dev["W_gate"], dev["W_up"], dev["W_down0"],
                              dev["conv_kernel"], dev["W_target"], w.eta, w.C, form=args.form,
                              workspace=ws, out=O[k], w_final=Wf[k], stream=stream)
        computed[k].record(stream)

    def download(i):
        k = i % nbuf
        down.wait_event(computed[k])
        with torch.cuda.stream(down):
            O_h[k].copy_(O[k], non_blocking=True)
            if state_to_host:
                W_h[k].copy_(Wf[k], non_blocking=True)
        fetched[k].record(down)

    def run(n, t0=None, t1=None):
        if t0 is not None:
            t0.record(up)
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            compute(i)
            download(i)
        if t1 is not None:
            t1.record(down)

    run(3)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(3, min(args.steps, 20))
    run(n, a, b)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    h2d = H_h.numel() * H_h.element_size() + X_h.numel() * X_h.element_size()
    d2h = O_h[0].numel() * O_h[0].element_size() + \
        (W_h[0].numel() * W_h[0].element_size() if state_to_host else 0)
    # the uploads alone, back to back: the floor the pipelined loop cannot go below
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(up)
    with torch.cuda.stream(up):
        for _ in range(n):
            H_d[0].copy_(H_h, non_blocking=True)
            X_d[0].copy_(X_h, non_blocking=True)
    c1.record(up)
    torch.cuda.synchronize()
    up_ms = c0.elapsed_time(c1) / n
    return {"value": w.B * w.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "h2d_alone_ms": up_ms, "h2d_alone_gbs": h2d / 1e9 / (up_ms / 1e3),
            "note": "inputs H, X0 from pinned host memory and O read back every step" +
                    (", and the fp32 state W_down_final" if state_to_host else
                     "; the fp32 state W_down_final stays on the device (the next segment's "
                     "W_down0)") +
                    "; copies of neighbouring steps overlap the compute (two buffers)"}

if __name__ == "__main__":
    sys.exit(main())
