"""Benchmark of the chunked-SGMV LoRA shrink/expand pair on B200.

Workload: the Qwen3-8B-like q/k/v decode case -- K=4096, three output slices
of 4096/1024/1024 columns, 8 adapters of rank 16 in bf16, one segment per
adapter, shuffled permutation -- swept over tok = 50 ... 8192.  One step is
one pass of the hot path over the sweep: for every tok, lora_shrink and then
lora_expand of the shrink's own output (18 calls).  The L2 cache is flushed
(256 MB write) before every call and each call is bracketed by CUDA events on
the launching stream, as on the sgl-kernel-xpu page ("Performance":
do_bench with the L2 flushed between runs).

value = algorithmic bytes of all calls / their summed device time (GB/s),
with bytes = gathered x + A of the adapters used + rank activations written
(shrink) and rank activations + B + base read and written (expand).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs the same sweep on its own GPU (independent
batches, no collective on the data path: weak scaling); rank 0 prints one JSON
line with the whole-job value (sum over ranks / max-over-ranks time).
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from scatter_gemm_b200 import workloads as W  # noqa: E402

METRIC = "LoRA shrink/expand effective GB/s (bf16, tok 50–8192) and % of HBM peak"
WORKLOAD = ("qkv decode sweep: K=4096, slices q/k/v 4096/1024/1024, 8 adapters rank 16 bf16, "
            "one segment per adapter, shuffled permutation, tok 50..8192; step = shrink then "
            "expand at every tok")
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# sources of the expand kernel (the dominant one) and of its launch: the ncu
# traffic in profiles/traffic.json is reported only while these are unchanged
EXPAND_SOURCES = ("expand_tc.cuh", "sched.cuh", "sm100.cuh", "common.cuh", "general.cuh",
                  "lora_sgmv.cu")


def csrc_hash():
    h = hashlib.sha256()
    for name in EXPAND_SOURCES:
        with open(os.path.join(ROOT, "scatter_gemm_b200", "csrc", name), "rb") as fh:
            h.update(name.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_traffic():
    """ncu DRAM traffic of the dominant kernel, if taken on the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("csrc_hash") != csrc_hash():
        return None
    return d


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        p = torch.cuda.get_device_properties(device)
        self.bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.bus],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.25)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------
# device problem
# ----------------------------------------------------------------------------

class DevProblem:
    def __init__(self, p, device):
        self.p = p
        tdt = torch.bfloat16 if p.dtype == "bf16" else torch.float16
        mis = int(p.misalign)  # elements past a 16-byte boundary (the tail workload: 2)

        def up(bits):
            # every data tensor starts `mis` elements into its allocation
            flat = torch.from_numpy(np.ascontiguousarray(bits).reshape(-1).view(np.int16))
            buf = torch.zeros(flat.numel() + mis + 8, dtype=torch.int16, device=device)
            buf[mis: mis + flat.numel()].copy_(flat)
            return buf[mis: mis + flat.numel()].view(tdt).view(*bits.shape)

        self.x = up(p.x)[:, : p.K]
        self.A = up(p.A)
        self.B = up(p.B)
        self.base = up(p.base)
        self.si = torch.from_numpy(p.seg_indptr).to(device)
        self.wi = torch.from_numpy(p.weight_indices).to(device)
        self.pm = torch.from_numpy(p.permutation).to(device)
        self.sc = torch.from_numpy(p.scalings).to(device)
        self.out = up(np.zeros((p.tok, p.S * p.rs), dtype=np.uint16))
        self.off = [int(v) for v in p.slice_offsets]
        from scatter_gemm_b200 import lora
        self.ws = lora.make_workspace(p.tok, p.nseg, p.L, device)
        self.bytes_shrink = W.bytes_shrink(p)
        self.bytes_expand = W.bytes_expand(p)
        self.rows = int(p.seg_indptr[-1] - p.seg_indptr[0])

    def shrink(self, lora):
        lora.lora_shrink(self.x, self.A, self.si, self.wi, self.pm, self.out,
                         num_slices=self.p.S, rank=self.p.r, workspace=self.ws)

    def expand(self, lora):
        lora.lora_expand(self.out, self.B, self.si, self.wi, self.pm, self.off, self.sc,
                         self.base, rank=self.p.r, workspace=self.ws)

    def pair(self, lora):
        lora.lora_shrink_expand(self.x, self.A, self.B, self.si, self.wi, self.pm, self.off,
                                self.sc, self.out, self.base, rank=self.p.r, workspace=self.ws)


def time_fused(probs, lora, flush, stream, steps, warmup, nap):
    """lora_shrink_expand on the decode-sized cases of the sweep (tok <= 512),
    timed like the sweep: L2 flushed and a GPU sleep before each call, CUDA
    events around it.  Reported beside the separately timed pair, not part of
    `value` (the pages measure the two ops one by one)."""
    out = []
    for dp in probs:
        if dp.p.tok > 512:
            continue
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for k in range(warmup + steps):
            flush.zero_()
            torch.cuda._sleep(nap)
            if k >= warmup:
                ev[k - warmup][0].record(stream)
            dp.pair(lora)
            if k >= warmup:
                ev[k - warmup][1].record(stream)
        torch.cuda.synchronize()
        ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
        # algorithmic bytes of the fused call: both ops' bytes less the rank
        # activations the expand would read back
        nbytes = dp.bytes_shrink + dp.bytes_expand - dp.rows * dp.p.S * dp.p.r * 2
        out.append({"tok": dp.p.tok, "fused_us": round(ms * 1e3, 2),
                    "fused_path": bool(lora.last_path() & lora.PATH_FUSED),
                    "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1)})
    return out


def time_base_expand(lora, flush, stream, device, toks, steps, warmup, nap):
    """lora_base_expand (the projection with the expand folded in) on the qkv
    workload, beside the unfused route: cuBLAS x W^T (torch.matmul) then
    lora_expand.  Timed like the sweep (L2 flushed, GPU sleep, CUDA events);
    reported beside `value`, which the pages' two ops define."""
    out = []
    for tok in toks:
        p = W.make_problem("qkv", seed=7, tok=tok)
        dp = DevProblem(p, device)
        tdt = dp.x.dtype
        wt = torch.from_numpy(W.make_base_weight(p, 7).view(np.int16)).to(device).view(tdt)
        inr = torch.from_numpy(p.in_r.view(np.int16)).to(device).view(tdt)
        res = dp.base.clone()
        xk = dp.x[:, : p.K]

        def fused():
            lora.lora_base_expand(xk, wt, inr, dp.B, dp.si, dp.wi, dp.pm, dp.off, dp.sc, res,
                                  rank=p.r)

        def separate():
            torch.matmul(xk, wt.t(), out=res[:, dp.off[0]: dp.off[-1]])
            lora.lora_expand(inr, dp.B, dp.si, dp.wi, dp.pm, dp.off, dp.sc, res, rank=p.r,
                             workspace=dp.ws)

        ms = {}
        for name, fn in (("fused", fused), ("separate", separate)):
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(steps)]
            for k in range(warmup + steps):
                flush.zero_()
                torch.cuda._sleep(nap)
                if k >= warmup:
                    ev[k - warmup][0].record(stream)
                fn()
                if k >= warmup:
                    ev[k - warmup][1].record(stream)
            torch.cuda.synchronize()
            ms[name] = float(np.mean([a.elapsed_time(b) for a, b in ev]))
        flops = 2.0 * tok * (dp.off[-1] - dp.off[0]) * p.K + 2.0 * tok * (dp.off[-1] - dp.off[0]) * p.r
        tf = flops / (ms["fused"] * 1e-3) / 1e12
        out.append({"tok": tok, "fused_us": round(ms["fused"] * 1e3, 1),
                    "cublas_plus_expand_us": round(ms["separate"] * 1e3, 1),
                    "tflops": round(tf, 1)})
    return out


# the other workloads of the pages' "Performance"/"Testing" sections, one line
# each (the headline `value` stays the qkv sweep)
CONFIG_LINES = (("tiny", "bf16"), ("gate_up", "bf16"), ("gate_up", "fp16"), ("tail", "fp16"),
                ("many_small", "bf16"))


def path_names(bits, lora):
    names = [("tensor", lora.PATH_TENSOR), ("general", lora.PATH_GENERAL),
             ("grouped", lora.PATH_GROUPED), ("splitk", lora.PATH_SPLITK),
             ("fused", lora.PATH_FUSED)]
    return "+".join(n for n, b in names if bits & b)


def time_configs(lora, flush, stream, device, steps, warmup, nap, peak, which=CONFIG_LINES):
    """Shrink and expand of each workload in `which`, timed like the sweep (L2
    flushed and a GPU sleep before each call, CUDA events around it)."""
    out = []
    for name, dt in which:
        p = W.make_problem(name, seed=0, dtype=dt)
        dp = DevProblem(p, device)
        row = {"config": name, "dtype": dt, "tok": p.tok, "K": p.K,
               "slices": [int(v) for v in np.diff(p.slice_offsets)], "rank": p.r,
               "adapters": p.L, "segments": p.nseg, "misalign_elems": p.misalign}
        for op, fn, nbytes in (("shrink", dp.shrink, dp.bytes_shrink),
                               ("expand", dp.expand, dp.bytes_expand)):
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(steps)]
            for k in range(warmup + steps):
                flush.zero_()
                torch.cuda._sleep(nap)
                if k >= warmup:
                    ev[k - warmup][0].record(stream)
                fn(lora)
                if k >= warmup:
                    ev[k - warmup][1].record(stream)
            torch.cuda.synchronize()
            t = [a.elapsed_time(b) for a, b in ev]
            ms = float(np.mean(t))
            gbs = nbytes / (ms * 1e-3) / 1e9
            row[f"{op}_us"] = round(ms * 1e3, 2)
            row[f"{op}_us_median"] = round(float(np.median(t)) * 1e3, 2)
            row[f"{op}_mb"] = round(nbytes / 1e6, 2)
            row[f"{op}_gbs"] = round(gbs, 1)
            row[f"{op}_frac_of_measured"] = round(gbs / peak, 4)
            row[f"{op}_frac_of_nominal_8tbs"] = round(gbs / NOMINAL_HBM_GBS, 4)
            row[f"{op}_path"] = path_names(lora.last_path(), lora)
        out.append(row)
        del dp
    return out


# ----------------------------------------------------------------------------
# CPU oracle timing (baseline; never the product path)
# ----------------------------------------------------------------------------

# bounded samples of each workload for the per-config CPU baseline: the
# workload's own recipe at a smaller token count where the full one would take
# the oracle more than a few seconds on one thread
CPU_SAMPLES = (("tiny", "bf16", {}), ("qkv", "bf16", {"tok": 512}),
               ("gate_up", "bf16", {"tok": 128}), ("gate_up", "fp16", {"tok": 128}),
               ("tail", "fp16", {}), ("many_small", "bf16", {"tok": 256, "nseg": 32}))


def time_oracle_configs(reps=3):
    """The oracle on one thread and on all host threads, median of `reps`
    runs of shrink + expand, per workload sample (GB/s of algorithmic bytes)."""
    import oracle
    all_threads = oracle.max_threads()
    rows = []
    for name, dt, over in CPU_SAMPLES:
        p = W.make_problem(name, seed=0, dtype=dt, **over)
        nbytes = W.bytes_shrink(p) + W.bytes_expand(p)
        row = {"config": name, "dtype": dt, "tok": p.tok, "segments": p.nseg,
               "mb": round(nbytes / 1e6, 2)}
        for label, n in (("single", 1), ("all", all_threads)):
            oracle.set_threads(n)
            ts = []
            for _ in range(reps):
                t0 = time.perf_counter()
                h = oracle.shrink_problem(p)
                oracle.expand_problem(p, in_r=h)
                ts.append(time.perf_counter() - t0)
            row[f"{label}_s"] = round(statistics.median(ts), 4)
            row[f"{label}_gbs"] = round(nbytes / statistics.median(ts) / 1e9, 4)
        rows.append(row)
    oracle.set_threads(all_threads)
    return rows, all_threads


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def time_oracle(toks, min_seconds):
    import oracle
    probs = [W.make_problem("qkv", seed=0, tok=t) for t in toks]
    nbytes = sum(W.bytes_shrink(p) + W.bytes_expand(p) for p in probs)
    t0 = time.perf_counter()
    passes = 0
    while True:
        for p in probs:
            h = oracle.shrink_problem(p)
            oracle.expand_problem(p, in_r=h)
        passes += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return nbytes * passes / el / 1e9, el, passes, oracle.max_threads()


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle timed on the host cores, rank 0 only,
    on the same nine-token sweep as our arm: a step is shrink + expand at every
    tok of the sweep (about 1.5 s of oracle work on the host's threads).  With
    more than 60 timed steps a step covers one tok of the sweep, in rotation,
    so that the run stays within minutes; the bytes and times still add up over
    the sweep."""
    if rank != 0:
        return
    import oracle
    toks = [int(t) for t in args.toks.split(",")]
    probs = [W.make_problem("qkv", seed=0, tok=t) for t in toks]
    full = args.steps <= 60

    def step_problems(k):
        return probs if full else [probs[k % len(probs)]]

    for k in range(min(args.warmup, 1)):
        for p in step_problems(k):
            h = oracle.shrink_problem(p)
            oracle.expand_problem(p, in_r=h)
    nbytes = 0
    el = 0.0
    for k in range(args.steps):
        for p in step_problems(k):
            nbytes += W.bytes_shrink(p) + W.bytes_expand(p)
            t0 = time.perf_counter()
            h = oracle.shrink_problem(p)
            oracle.expand_problem(p, in_r=h)
            el += time.perf_counter() - t0
    value = nbytes / el / 1e9
    cores = oracle.max_threads()
    sample = ("shrink + expand at every tok of the sweep per step (CPU oracle, fp32 sequential "
              "sums, OpenMP over the rows of a segment)" if full else
              "shrink + expand at one tok of the sweep per step, in rotation over the sweep "
              "(CPU oracle, fp32 sequential sums)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "toks": toks, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def run_ours(args, rank, world, device):
    from scatter_gemm_b200 import lora
    import torch.distributed as dist

    toks = [int(t) for t in args.toks.split(",")]
    probs = [DevProblem(W.make_problem("qkv", seed=rank, tok=t), device) for t in toks]
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream()
    n_calls = 2 * len(probs)

    # ~50 us of GPU sleep after each flush keeps the GPU behind the host, so no
    # host-side enqueue latency can fall between a call's two events
    nap = 100000  # cycles (about 50-75 us)

    def step(ev):
        for j, dp in enumerate(probs):
            flush.zero_()
            torch.cuda._sleep(nap)
            if ev is not None:
                ev[2 * j][0].record(stream)
            dp.shrink(lora)
            if ev is not None:
                ev[2 * j][1].record(stream)
            flush.zero_()
            torch.cuda._sleep(nap)
            if ev is not None:
                ev[2 * j + 1][0].record(stream)
            dp.expand(lora)
            if ev is not None:
                ev[2 * j + 1][1].record(stream)

    for _ in range(args.warmup):
        step(None)
    torch.cuda.synchronize()

    events = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_calls)] for _ in range(args.steps)]
    wall0, wall1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(device) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    lora.reset_launch_count()
    wall0.record(stream)
    for k in range(args.steps):
        step(events[k])
    wall1.record(stream)
    torch.cuda.synchronize()
    launches = lora.launch_count()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None

    # per-call device times (ms), [steps, calls]
    t = np.array([[s.elapsed_time(e) for (s, e) in row] for row in events], dtype=np.float64)
    kernel_ms = float(t.sum())
    wall_ms = wall0.elapsed_time(wall1)
    bytes_step = sum(dp.bytes_shrink + dp.bytes_expand for dp in probs)
    if world > 1:
        red = torch.tensor([kernel_ms, wall_ms], dtype=torch.float64, device=device)
        dist.all_reduce(red, op=dist.ReduceOp.MAX)
        kernel_ms, wall_ms = float(red[0]), float(red[1])

    # e2e: host buffers in pinned memory, H2D + both calls + D2H inside the timed region
    fused = None
    if not args.no_fused:
        fused = time_fused(probs, lora, flush, stream, min(args.steps, 200), 3, nap)
    base_fused = None
    if not args.no_base_expand:
        base_fused = time_base_expand(lora, flush, stream, device, (512, 2048, 8192),
                                      min(args.steps, 20), 3, nap)
    configs = None
    if not args.no_configs:
        which = CONFIG_LINES
        if args.configs:
            which = tuple(tuple(c.split(":")) for c in args.configs.split(","))
        configs = time_configs(lora, flush, stream, device, min(args.steps, 100), 3, nap,
                               measured_peaks()[0], which)
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, probs, lora, device, stream, world)

    if rank != 0:
        return
    peak, peak_kind = measured_peaks()
    # per call, ms: means (CUDA event timestamps tick in ~2 us steps, so medians
    # of single calls are quantized; the mean over steps is not)
    med = np.median(t, axis=0)
    avg = t.mean(axis=0)
    detail = []
    fr = []
    for j, dp in enumerate(probs):
        s_ms, e_ms = avg[2 * j], avg[2 * j + 1]
        gbs = (dp.bytes_shrink + dp.bytes_expand) / ((s_ms + e_ms) * 1e-3) / 1e9
        detail.append({"tok": dp.p.tok,
                       "shrink_us": round(s_ms * 1e3, 2), "expand_us": round(e_ms * 1e3, 2),
                       "shrink_us_median": round(med[2 * j] * 1e3, 2),
                       "expand_us_median": round(med[2 * j + 1] * 1e3, 2),
                       "shrink_gbs": round(dp.bytes_shrink / (s_ms * 1e-3) / 1e9, 1),
                       "expand_gbs": round(dp.bytes_expand / (e_ms * 1e-3) / 1e9, 1),
                       "gbs": round(gbs, 1)})
        if dp.p.tok >= 1024:
            fr.append(gbs)
    geo = math.exp(sum(math.log(v) for v in fr) / len(fr)) if fr else None
    if fused:
        pair = {d["tok"]: d["shrink_us"] + d["expand_us"] for d in detail}
        for f in fused:
            if f["tok"] in pair:
                f["pair_us"] = round(pair[f["tok"]], 2)
                f["speedup_vs_pair"] = round(pair[f["tok"]] / f["fused_us"], 2)
    mean_case = statistics.mean(d["gbs"] for d in detail)

    # roofline of the dominant kernel (larger summed time of the two ops)
    s_tot, e_tot = t[:, 0::2].sum(), t[:, 1::2].sum()
    dom = "expand" if e_tot >= s_tot else "shrink"
    cols = t[:, 1::2] if dom == "expand" else t[:, 0::2]
    alg = [dp.bytes_expand if dom == "expand" else dp.bytes_shrink for dp in probs]
    achieved = sum(alg) * args.steps / (cols.sum() * 1e-3) / 1e9
    tr = load_traffic()
    traffic = None
    if tr is not None and tr.get("op") == dom:
        traffic = tr.get("dram_bytes_per_launch")
    roof = {"bound": "hbm", "kernel": f"lora_{dom} kernels over the sweep",
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} copy bandwidth",
            "traffic": traffic,
            "algorithmic_bytes_per_launch": round(sum(alg) / len(alg)),
            "share_of_step": round(float(max(s_tot, e_tot) / (s_tot + e_tot)), 3)}

    cpu = None
    if world == 1 and not args.no_cpu:
        v, el, passes, cores = time_oracle([50, 128, 256, 512, 1024], args.cpu_seconds)
        cpu = {"value": round(v, 3), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"tok 50,128,256,512,1024 of the sweep, shrink + expand, "
                         f"{passes} pass(es) in {el:.1f} s, all host threads",
               "nproc": os.cpu_count(), "cpu_model": cpu_model()}
        if not args.no_configs:
            rows, _ = time_oracle_configs()
            cpu["per_config"] = rows
            cpu["per_config_note"] = ("median of 3 runs of shrink + expand on one thread and "
                                      "on all host threads, per workload sample")

    value = bytes_step * args.steps * world / (kernel_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(kernel_ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "toks": toks, "l2": "flushed before every call "
                   "(256 MB write, outside the events), then ~50 us GPU sleep",
                   "parallelism": f"dp{world}",
                   "step_ms_incl_flush": round(wall_ms / args.steps, 4)},
        "frac_of_peak": round(value / world / peak, 4),
        "frac_of_nominal_8tbs": round(value / world / NOMINAL_HBM_GBS, 4),
        "geomean_gbs_tok_ge_1024": round(geo, 1) if geo else None,
        "geomean_frac_tok_ge_1024": round(geo / peak, 4) if geo else None,
        "geomean_frac_nominal_tok_ge_1024": round(geo / NOMINAL_HBM_GBS, 4) if geo else None,
        "mean_case_gbs": round(mean_case, 1),
        "per_tok": detail,
        "per_config": configs,
        "fused_decode": fused,
        "base_expand": base_fused,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches) * world,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def run_e2e(args, probs, lora, device, stream, world):
    """Same sweep through the public API with host buffers: H2D of the step's
    inputs (x, tables, base) from pinned memory, both calls, D2H of base."""
    import torch.distributed as dist
    host = []
    for dp in probs:
        h = {k: getattr(dp, k).cpu().pin_memory() for k in ("x", "base", "si", "wi", "pm")}
        h["base_back"] = torch.empty_like(h["base"]).pin_memory()
        host.append(h)
    h2d = sum(sum(v.numel() * v.element_size() for k, v in h.items() if k != "base_back")
              for h in host)
    d2h = sum(h["base_back"].numel() * h["base_back"].element_size() for h in host)
    steps = max(3, min(args.steps, args.e2e_steps))

    def step():
        for dp, h in zip(probs, host):
            dp.x.copy_(h["x"], non_blocking=True)
            dp.base.copy_(h["base"], non_blocking=True)
            dp.si.copy_(h["si"], non_blocking=True)
            dp.wi.copy_(h["wi"], non_blocking=True)
            dp.pm.copy_(h["pm"], non_blocking=True)
            dp.shrink(lora)
            dp.expand(lora)
            h["base_back"].copy_(dp.base, non_blocking=True)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if world > 1:
        red = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(red, op=dist.ReduceOp.MAX)
        ms = float(red[0])
    nbytes = sum(dp.bytes_shrink + dp.bytes_expand for dp in probs) * steps * world
    return {"value": round(nbytes / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps}


# ----------------------------------------------------------------------------
# Launch floor: an empty kernel with each of the library's launch shapes
# ----------------------------------------------------------------------------

# (name, grid, threads, dynamic shared memory bytes, cluster size): the shapes
# the qkv sweep's kernels launch with (from its ncu launch list)
LAUNCH_SHAPES = (
    ("one warp", 1, 32, 0, 1),
    ("shrink, qkv tok 50", 144, 160, 94408, 16),
    ("shrink, qkv tok 8192", 288, 160, 94408, 4),
    ("expand, qkv tok 50", 216, 416, 91784, 1),
    ("expand, qkv tok 8192", 288, 416, 91784, 1),
    ("fused, qkv tok 256", 80, 416, 216936, 8),
)


def run_launch_floor(args, device):
    """Times an empty kernel (compiled here with NVRTC, launched through the
    driver API) with each launch shape of LAUNCH_SHAPES, with the sweep's
    method: 256 MB L2-flush write and a GPU sleep before each launch, CUDA
    events around it.  What remains of a call beyond this is the kernel's own
    work."""
    from cuda.bindings import driver as cu, nvrtc

    def check(res):
        err = res[0]
        assert int(err) == 0, err
        return res[1] if len(res) > 1 else None

    prog = check(nvrtc.nvrtcCreateProgram(b'extern "C" __global__ void lora_empty() {}',
                                          b"empty.cu", 0, [], []))
    opts = [b"--gpu-architecture=sm_100a"]
    check(nvrtc.nvrtcCompileProgram(prog, len(opts), opts))
    cubin = b" " * check(nvrtc.nvrtcGetCUBINSize(prog))
    check(nvrtc.nvrtcGetCUBIN(prog, cubin))
    torch.cuda.synchronize()  # the runtime's primary context is current
    mod = check(cu.cuModuleLoadData(cubin))
    fn = check(cu.cuModuleGetFunction(mod, b"lora_empty"))
    fa = cu.CUfunction_attribute
    check(cu.cuFuncSetAttribute(fn, fa.CU_FUNC_ATTRIBUTE_MAX_DYNAMIC_SHARED_SIZE_BYTES,
                                227 * 1024))
    check(cu.cuFuncSetAttribute(fn, fa.CU_FUNC_ATTRIBUTE_NON_PORTABLE_CLUSTER_SIZE_ALLOWED, 1))
    stream = torch.cuda.current_stream(device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    nap = 100000
    rows = []
    for name, grid, threads, smem, cluster in LAUNCH_SHAPES:
        cfg = cu.CUlaunchConfig()
        cfg.gridDimX, cfg.gridDimY, cfg.gridDimZ = grid, 1, 1
        cfg.blockDimX, cfg.blockDimY, cfg.blockDimZ = threads, 1, 1
        cfg.sharedMemBytes = smem
        cfg.hStream = cu.CUstream(stream.cuda_stream)
        attr = cu.CUlaunchAttribute()
        attr.id = cu.CUlaunchAttributeID.CU_LAUNCH_ATTRIBUTE_CLUSTER_DIMENSION
        attr.value.clusterDim.x, attr.value.clusterDim.y, attr.value.clusterDim.z = cluster, 1, 1
        cfg.attrs = [attr]
        cfg.numAttrs = 1
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for k in range(args.warmup + args.steps):
            flush.zero_()
            torch.cuda._sleep(nap)
            if k >= args.warmup:
                ev[k - args.warmup][0].record(stream)
            check(cu.cuLaunchKernelEx(cfg, fn, None, 0))
            if k >= args.warmup:
                ev[k - args.warmup][1].record(stream)
        torch.cuda.synchronize()
        t = [a.elapsed_time(b) * 1e3 for a, b in ev]
        rows.append({"shape": name, "grid": grid, "threads": threads, "smem_bytes": smem,
                     "cluster": cluster, "us_mean": round(float(np.mean(t)), 2),
                     "us_median": round(float(np.median(t)), 2)})
    check(cu.cuModuleUnload(mod))
    print(json.dumps({"mode": "launch_floor", "unit": "us", "steps": args.steps,
                      "warmup": args.warmup, "l2": "flushed before every launch (256 MB write), "
                      "then ~50 us GPU sleep", "launches": rows}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--toks", default=",".join(str(t) for t in W.QKV_TOK_SWEEP))
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-fused", action="store_true")
    ap.add_argument("--no-base-expand", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--configs", default="",
                    help="per-config lines to time, e.g. gate_up:fp16,tail:fp16 (default: all)")
    ap.add_argument("--launch-floor", action="store_true",
                    help="time an empty kernel with each of the library's launch shapes, then exit")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if args.launch_floor:
        run_launch_floor(args, device)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    try:
        run_ours(args, rank, world, device)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
