#!/usr/bin/env python
"""Benchmark of the MatMamba block at Matryoshka widths on B200.

Metric: block prefill tokens/s per width m_i (headline: the 130M-class block,
batch 8 x 2048 tokens, at full width m = 768) and the SSD scan's fraction of
its roofline (standalone scan, batch 4 x 8192 tokens, 24 heads and the 12-head
prefix).  Inputs are seeded synthetic tensors already resident in HBM; L2 is
flushed (256 MiB write) before every timed step and each step is timed with
CUDA events on the launching stream.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica on its own GPU (sequences shard with no exchange), and value is the
tokens of all ranks divided by the slowest rank's time.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MatMamba block prefill tokens/sec per width m_i; SSD scan % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--skip-stack-decode", action="store_true",
                    help="leave out the 48-layer stack and the decode step (profiling aid)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["block", "scan", "decode"], default=None,
                    help="profiling aid: run just the headline block or just the standalone scan, print per-stage "
                         "times and no benchmark line")
    ap.add_argument("--ncu-summary", metavar="CSV", default=None,
                    help="print a per-kernel table (launches, device time, share, DRAM bytes per launch) of an "
                         "ncu --csv log and exit")
    ap.add_argument("--stub", action="store_true",
                    help="launcher check on CPU: every rank times a small host matmul over gloo and rank 0 prints "
                         "the rank count and the whole-job rate (no GPU, no library)")
    a = ap.parse_args()
    if a.gpus < 1:
        ap.error("--gpus must be at least 1")
    if a.only is None:
        a.warmup = max(a.warmup, 3)
    return a


def ncu_summary(path):
    """Group an `ncu --csv` metrics log by kernel: launches, summed gpu__time_duration, share of the total,
    and the mean per launch of every other metric (DRAM bytes, for instance)."""
    import csv
    scale = {"nsecond": 1e-3, "usecond": 1.0, "msecond": 1e3, "second": 1e6, "ns": 1e-3, "us": 1.0, "ms": 1e3,
             "s": 1e6}
    byte_scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}
    launches, per = {}, {}
    with open(path) as f:
        rows = [r for r in csv.reader(line for line in f if line.startswith('"'))]
    hdr, rows = rows[0], rows[1:]
    col = {k: hdr.index(k) for k in ("ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value")}
    for r in rows:
        name = r[col["Kernel Name"]]
        name = name.replace("(anonymous namespace)::", "").replace("void ", "").split("(")[0]
        key = (name, r[col["ID"]])
        unit, val = r[col["Metric Unit"]], float(r[col["Metric Value"]].replace(",", ""))
        metric = r[col["Metric Name"]]
        if metric == "gpu__time_duration.sum":
            val *= scale.get(unit, 1.0)
        elif unit in byte_scale:
            val *= byte_scale[unit]
        launches.setdefault(name, set()).add(key[1])
        per.setdefault(name, {}).setdefault(metric, []).append(val)
    total = sum(sum(m.get("gpu__time_duration.sum", [])) for m in per.values())
    others = sorted({k for m in per.values() for k in m} - {"gpu__time_duration.sum"})
    print("| kernel | launches | total us | share |" + "".join(" %s per launch |" % o for o in others))
    print("|---|---|---|---|" + "---|" * len(others))
    for name, m in sorted(per.items(), key=lambda kv: -sum(kv[1].get("gpu__time_duration.sum", [0]))):
        t = sum(m.get("gpu__time_duration.sum", [0]))
        extra = "".join(" %.4g |" % (sum(m[o]) / len(m[o])) if o in m else " |" for o in others)
        print("| %s | %d | %.1f | %.3f |%s" % (name, len(launches[name]), t, t / total if total else 0, extra))


def traffic_for(stage):
    """DRAM bytes per launch (read + write) of a stage's kernel from profiles/traffic.txt, or None when the
    kernel's source has changed since the capture (its sha256 prefix no longer matches)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == stage:
                src = os.path.join(ROOT, parts[1])
                if not os.path.exists(src):
                    return None
                with open(src, "rb") as g:
                    if hashlib.sha256(g.read()).hexdigest()[:16] != parts[2]:
                        return None
                return float(parts[3])
    return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------------ workload sizes

# device spin before each timed step (about 200 us at B200 clocks), longer than the host needs to enqueue one
LEAD_CYCLES = 400_000

BLOCK = dict(workload="block_130m_b8_L2048", batch=8, seq_len=2048, d_model=768, d_inner=1536, d_head=64,
             d_state=128, ngroups=1, d_conv=4, chunk=256, widths=[768, 384, 192, 96])
SCAN = dict(workload="ssd_b4_L8192_h24", batch=4, seq_len=8192, heads=24, d_head=64, d_state=128, chunk=256,
            head_slices=[24, 12])


def block_work(m, T, Dm=768, E=1536, P=64, N=128):
    """Algorithmic work of each launch stage of one block forward on T tokens at width m."""
    d = E * m // Dm
    h = d // P
    nconv = d + 2 * N
    return {
        "in_proj_conv": ("tensor", 2.0 * T * Dm * (2 * d + 2 * N + h)),
        "ssd_scan_gate": ("hbm", T * ((d + 2 * N) * 2 + h * 4 + d * 2 + d * 2 + 2 * h * 4)),
        "out_proj_norm": ("tensor", 2.0 * T * d * Dm),
        "in_proj": ("tensor", 2.0 * T * Dm * (2 * d + 2 * N + h)),
        "conv_silu_dt": ("hbm", T * (nconv * 2 * 2 + h * 4 * 2)),
        "ssd_scan": ("hbm", T * (2 * d * 2 + 2 * N * 2 + h * 4)),
        "gate_rmsnorm": ("hbm", T * d * 2 * 3),
        "out_proj": ("tensor", 2.0 * T * d * Dm),
    }


STACK = dict(workload="stack48_1p4b_b4_L4096", batch=4, seq_len=4096, d_model=2048, d_inner=4096, d_head=64,
             d_state=128, nlayers=48, chunk=256, widths=[2048, 1024, 512, 256])
DECODE = dict(workload="decode_b256_1p4b", batch=256, d_model=2048, d_inner=4096, d_head=64, d_state=128,
              steps=1000, graph_steps=100, widths=[2048, 1024, 512])


def stack_work(m, T, Dm=2048, E=4096, P=64, N=128):
    """Algorithmic work of each launch stage of one stack layer on T tokens at width m: the block's stages
    (out_proj adds into the fp32 residual) and the pre-norm (fp32 residual read, bf16 row written)."""
    w = block_work(m, T, Dm, E, P, N)
    w["prenorm"] = ("hbm", T * Dm * (4 + 2))
    return w


def decode_work(m, Bt, Dm=2048, E=4096, P=64, N=128, K=4):
    """HBM bytes of each launch stage of one recurrent step for Bt sequences at width m."""
    d = E * m // Dm
    h = d // P
    nconv = d + 2 * N
    return {
        "step_in_proj": ("hbm", (2 * d + 2 * N + h) * Dm * 2 + Bt * Dm * 2 + Bt * ((d + nconv) * 2 + h * 4)),
        "step_conv_dt": ("hbm", Bt * (nconv * (K - 1) * 2 * 2 + nconv * 2 * 2 + h * 4 * 2)),
        "step_scan": ("hbm", Bt * (h * P * N * 4 * 2 + nconv * 2 + h * 4 + d * 2)),
        "step_gate_rmsnorm": ("hbm", Bt * d * 2 * 3),
        "step_out_proj": ("hbm", Dm * d * 2 + Bt * d * 2 + Bt * Dm * 2),
        # fused forms: the state update with the gate (state read and written, xBC, dt and z read, the
        # gated row and its per-half sums of squares written), and out_proj with the 1/RMS row scale
        "step_scan_gate": ("hbm", Bt * (h * P * N * 4 * 2 + nconv * 2 + h * 4 + d * 2 + d * 2 + 2 * h * 4)),
        "step_out_proj_norm": ("hbm", Dm * d * 2 + Bt * d * 2 + Bt * 2 * h * 4 + Bt * Dm * 2),
    }


def stage_table(stages, work, pk, per_launch_divisor=1):
    """Per traced stage: mean launch time, share of the traced time, and achieved work against the peak
    (bf16 tensor FLOP/s or HBM GB/s).  per_launch_divisor splits a stage's launches into the unit the work
    is quoted for (e.g. 48 layers)."""
    tot_ms = sum(v[2] for v in stages.values()) or 1.0
    out = {}
    for k, (n, kern, ms) in stages.items():
        kd, amt = work.get(k, (None, 0.0))
        per = ms / n
        row = {"ms_per_launch": per, "launches": n, "share": ms / tot_ms}
        if kd is not None:
            ach = amt / (per / 1e3) / (1e12 if kd == "tensor" else 1e9)
            peak = pk["bf16_tflops"] if kd == "tensor" else pk["hbm_gbs"]
            row.update({"bound": kd, "achieved": ach, "unit": "TFLOP/s" if kd == "tensor" else "GB/s",
                        "frac": ach / peak})
        out[k] = row
    return out


def scan_bytes(T, h, P=64, N=128):
    """x read + y write (bf16), B and C read (bf16), dt read (fp32) per token."""
    return T * (2 * h * P * 2 + 2 * N * 2 + h * 4)


# ------------------------------------------------------------------------------------ multi-rank aggregation

def max_over_ranks(value, world, dist=None, device=None):
    """Largest value over all ranks (the slowest rank's time); plain value for one rank."""
    if world == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step, steps, world, slowest_seconds):
    """Throughput of the whole job: every rank's units over the slowest rank's time."""
    return world * units_per_rank_step * steps / slowest_seconds


# ------------------------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and clock-event reasons of this rank's GPU, polled through NVML
    every few milliseconds while a timed region is open (`active`).  Falls back
    to one nvidia-smi query per timed region when NVML cannot be loaded."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, device):
        self.device = device
        self.samples = []  # (sm_mhz, max_mhz, reasons bitmask)
        self.active = threading.Event()
        self.stop = threading.Event()
        self.thread = None
        self.handle = None
        self.nvml = None

    def _open(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        prop = torch.cuda.get_device_properties(self.device)
        bus = "%08x:%02x:%02x.0" % (prop.pci_domain_id, prop.pci_bus_id, prop.pci_device_id)
        self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        self.nvml = pynvml

    def _sample(self):
        n = self.nvml
        sm = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
        mx = n.nvmlDeviceGetMaxClockInfo(self.handle, n.NVML_CLOCK_SM)
        rs = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
        self.samples.append((float(sm), float(mx), int(rs)))

    def _loop(self):
        while not self.stop.is_set():
            if self.active.wait(0.05):
                try:
                    self._sample()
                except Exception:  # noqa: BLE001 - a failed poll only loses one sample
                    pass
                time.sleep(0.002)

    def __enter__(self):
        try:
            self._open()
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
        except Exception:  # noqa: BLE001 - NVML missing: nvidia-smi fallback in region_end
            self.nvml = None
        return self

    def __exit__(self, *exc):
        self.stop.set()
        self.active.set()
        if self.thread is not None:
            self.thread.join(timeout=2)
        if self.nvml is not None:
            try:
                self.nvml.nvmlShutdown()
            except Exception:  # noqa: BLE001
                pass

    def region_begin(self):
        self.active.set()

    def region_end(self):
        """Call with work still queued on the GPU (before the closing synchronize)."""
        if self.nvml is None:
            self._smi_sample()
            self.active.clear()
            return
        try:
            self._sample()  # at least one sample per region, taken under load
        except Exception:  # noqa: BLE001
            pass
        self.active.clear()

    def _smi_sample(self):
        try:
            import torch
            idx = torch.cuda.current_device()
            out = subprocess.run(["nvidia-smi", "-i", str(idx), "--query-gpu=clocks.sm,clocks.max.sm,"
                                  "clocks_event_reasons.active", "--format=csv,noheader,nounits"],
                                 capture_output=True, text=True, timeout=10).stdout.strip().split(",")
            self.samples.append((float(out[0]), float(out[1]), int(out[2].strip(), 16)))
        except Exception:  # noqa: BLE001
            pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        reasons = sorted({name for _, _, rs in self.samples for name, bit in self.REASONS if rs & bit})
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": max(s[1] for s in self.samples), "reasons": reasons,
                "samples": len(self.samples), "source": "nvml" if self.nvml is not None else "nvidia-smi"}


# ------------------------------------------------------------------------------------ our arm

def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import nested_mamba2_selective_b200 as mm
    from nested_mamba2_selective_b200 import build, synth

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    mm.load()
    pk, pk_src = peaks()

    def barrier():
        if world > 1:
            dist.barrier()

    def slowest(v):
        return max_over_ranks(v, world, dist, dev)

    stream = torch.cuda.current_stream()
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clk = ClockSampler(dev).__enter__()  # samples only inside timed regions

    def timed(fn, steps, warmup, trace=False):
        """Device time of each of `steps` calls of fn between CUDA events, L2 flushed before each.  Before
        every step the device spins for LEAD_CYCLES so that the host has enqueued the whole step when the
        first event is reached: the events then bracket device work only, not Python and launch latency.
        With trace, a second pass of the same steps (untimed) collects the library's per-stage device times
        and its kernel count, so the stage events never sit inside the timed steps."""
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        barrier()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        barrier()
        clk.region_begin()
        for e0, e1 in ev:
            flush_buf.zero_()
            torch.cuda._sleep(LEAD_CYCLES)
            e0.record(stream)
            fn()
            e1.record(stream)
        clk.region_end()
        torch.cuda.synchronize()
        barrier()
        ms = [e0.elapsed_time(e1) for e0, e1 in ev]
        tr = None
        if trace:
            mm.mm_trace_enable(steps * 32)
            for _ in range(steps):
                flush_buf.zero_()
                torch.cuda._sleep(LEAD_CYCLES)
                fn()
            torch.cuda.synchronize()
            tr = mm.mm_trace_collect()
            mm.mm_trace_enable(0)
        return ms, tr

    if args.only:
        rc = run_only(args, mm, synth, torch, dev, timed)
        clk.__exit__(None, None, None)
        return rc

    # ---------------- block workload (headline)
    B = BLOCK
    arrays = synth.block_params(B["d_model"], B["d_inner"], B["d_head"], B["d_state"], dtype="bf16", seed=1002)
    wt = mm.BlockWeights.from_arrays(arrays, B["d_model"], B["d_inner"], B["d_head"], B["d_state"],
                                     dtype=torch.bfloat16, device=dev)
    u_np = synth.activations((B["batch"], B["seq_len"], B["d_model"]), "bf16", seed=1002 + 30 + rank)
    u = torch.from_numpy(u_np).to(dev).bfloat16()
    out = torch.empty_like(u)
    T = B["batch"] * B["seq_len"]
    ws = torch.empty(max(mm.matmamba_block_workspace(wt, B["batch"], B["seq_len"], m, B["chunk"])
                         for m in B["widths"]), dtype=torch.uint8, device=dev)

    per_width = {}
    head = None
    for m in B["widths"]:
        fn = lambda m=m: mm.matmamba_block_fwd(wt, u, m, B["chunk"], out=out, workspace=ws)  # noqa: E731
        ms, tr = timed(fn, args.steps, args.warmup, trace=True)
        total = slowest(sum(ms))
        per_width[str(m)] = {"tokens_per_s": whole_job_rate(T, args.steps, world, total / 1e3),
                             "ms_per_step": total / args.steps,
                             "stages": stage_table(tr[0], block_work(m, T), pk)}
        if m == B["widths"][0]:
            head = (ms, total, tr)
    ms, total, (stages, kernels) = head
    m0 = B["widths"][0]
    value = whole_job_rate(T, args.steps, world, total / 1e3)

    # dominant stage of the headline step -> roofline object
    work = block_work(m0, T)
    stage_rows = stage_table(stages, work, pk)
    dom = max(stages, key=lambda k: stages[k][2])
    avg_ms = stages[dom][2] / stages[dom][0]
    sr = stage_rows[dom]
    roof = {"bound": sr["bound"], "achieved": sr["achieved"],
            "peak": pk["bf16_tflops"] if sr["bound"] == "tensor" else pk["hbm_gbs"], "unit": sr["unit"],
            "frac": sr["frac"], "traffic": traffic_for(dom), "kernel": dom, "peak_source": pk_src,
            "avg_launch_ms": avg_ms}

    # ---------------- standalone SSD scan (the graded scan roofline)
    S = SCAN
    inp = synth.ssd_inputs(S["batch"], S["seq_len"], S["heads"], S["d_head"], S["d_state"], 1, "bf16", seed=1001)
    g = {k: torch.from_numpy(v).to(dev) for k, v in inp.items()}
    for k in ("x", "B", "C"):
        g[k] = g[k].bfloat16()
    Ts = S["batch"] * S["seq_len"]
    scan = {}
    for h in S["head_slices"]:
        y = torch.empty((S["batch"], S["seq_len"], h, S["d_head"]), dtype=torch.bfloat16, device=dev)
        sws = torch.empty(max(mm.ssd_scan_workspace(torch.bfloat16, S["batch"], S["seq_len"], h, 64, 128, 1,
                                                    S["chunk"]), 1), dtype=torch.uint8, device=dev)
        fn = lambda h=h, y=y, sws=sws: mm.ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], h=h,  # noqa
                                                   chunk=S["chunk"], y=y, workspace=sws)
        sms, str_ = timed(fn, args.steps, args.warmup, trace=True)
        avg = slowest(sum(sms)) / args.steps
        nbytes = scan_bytes(Ts, h)
        scan[str(h)] = {"tokens_per_s": world * Ts / (avg / 1e3), "us_per_call": avg * 1e3,
                        "kernels_per_call": str_[1] // args.steps,
                        "roofline": {"bound": "hbm", "achieved": nbytes / (avg / 1e3) / 1e9, "peak": pk["hbm_gbs"],
                                     "unit": "GB/s", "frac": nbytes / (avg / 1e3) / 1e9 / pk["hbm_gbs"],
                                     "algorithmic_bytes": nbytes, "traffic": traffic_for("ssd_scan_h%d" % h),
                                     "peak_source": pk_src}}
    del g, inp

    # ---------------- end to end through the host-buffer entry point
    u_host = torch.from_numpy(u_np).bfloat16().pin_memory()
    out_host = torch.empty_like(u_host).pin_memory()
    u_dev, out_dev = torch.empty_like(u), torch.empty_like(u)
    e2e_fn = lambda: mm.matmamba_block_fwd_host(wt, u_host, m0, B["chunk"], out_host, u_dev, out_dev, ws)  # noqa
    for _ in range(args.warmup):
        e2e_fn()
    barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        e2e_fn()
    e2e_s = slowest(time.perf_counter() - t0)
    io_bytes = T * B["d_model"] * 2
    link = copy_rates(torch, u_host, out_host, u_dev, out_dev)
    del ws, u_dev, out_dev

    stack = decode = None
    if not args.skip_stack_decode:
        stack = run_stack(args, mm, torch, dev, timed, slowest, world, pk)
        decode = run_decode(args, mm, torch, dev, timed, slowest, world, pk)
    clk.__exit__(None, None, None)
    clocks = clk.summary()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": B["workload"], "batch": B["batch"], "seq_len": B["seq_len"],
                       "d_model": B["d_model"], "d_inner": B["d_inner"], "d_head": B["d_head"],
                       "d_state": B["d_state"], "ngroups": 1, "d_conv": 4, "chunk": B["chunk"],
                       "scan_block_tokens": 128,
                       "chunk_note": "the chunked scan's result does not depend on chunk; the bf16 kernels "
                                     "evaluate every chunk of 256 as two 128-token blocks",
                       "width": m0, "parallelism": "replicas%d" % world,
                       "l2": "flushed (256 MiB write) before every timed step",
                       "timing": "CUDA events around each step after a device spin that lets the host enqueue "
                                 "the whole step; per-stage times from a separate traced pass"},
            "per_width": per_width,
            "roofline": roof,
            "stages": stage_rows,
            "ssd_scan": {"workload": S["workload"], "by_heads": scan},
            "e2e": {"value": whole_job_rate(T, args.steps, world, e2e_s), "unit": "tokens/s",
                    "h2d_bytes_per_step": io_bytes, "d2h_bytes_per_step": io_bytes,
                    "h2d_gbs": link["h2d_gbs"], "d2h_gbs": link["d2h_gbs"],
                    "both_directions_ms": link["both_ms"],
                    "copy_bound": whole_job_rate(T, 1, world, link["both_ms"] / 1e3),
                    "note": "copy_bound = tokens per step / the time of one step's upload and download "
                            "running at once (pinned buffers, no compute)"},
            "gpu_launches": kernels,
            "clocks": clocks,
        }
        if stack:
            line["stack48"] = stack
        if decode:
            line["decode"] = decode
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(arrays, u_np, m0)
            line["cpu_baseline_scan"] = cpu_baseline_scan()
            if stack:
                line["cpu_baseline_stack"] = cpu_baseline_stack()
            if decode:
                line["cpu_baseline_decode"] = cpu_baseline_decode()
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def copy_rates(torch, u_host, out_host, u_dev, out_dev, reps=5):
    """PCIe rates of one step's copies between pinned host buffers and the device: the upload alone,
    the download alone (GB/s, CUDA events on the copy's stream) and both at once on two streams (ms
    between events on a third stream that waits for both)."""
    s_in, s_out, s_main = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.current_stream()
    nbytes = u_host.numel() * u_host.element_size()

    def one(dst, src, stream):
        with torch.cuda.stream(stream):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            dst.copy_(src, non_blocking=True)
            e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    h2d = min(one(u_dev, u_host, s_in) for _ in range(reps))
    d2h = min(one(out_host, out_dev, s_out) for _ in range(reps))
    both = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_main)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        with torch.cuda.stream(s_in):
            u_dev.copy_(u_host, non_blocking=True)
        with torch.cuda.stream(s_out):
            out_host.copy_(out_dev, non_blocking=True)
        s_main.wait_stream(s_in)
        s_main.wait_stream(s_out)
        e1.record(s_main)
        torch.cuda.synchronize()
        both.append(e0.elapsed_time(e1))
    return {"h2d_gbs": nbytes / (h2d / 1e3) / 1e9, "d2h_gbs": nbytes / (d2h / 1e3) / 1e9, "both_ms": min(both)}


def device_block_weights(mm, torch, gen, Dm, E, P, N, dev, K=4):
    """Full-width block weights drawn on the device from a seeded generator with the synthetic recipe
    (weights ~ N(0, 0.02) in bf16, norm_w = 1 + N(0, 0.02), A = -exp(U(log 1, log 16)), dt_bias =
    softplus^-1 of a log-uniform dt in [1e-3, 1e-1], D ~ N(0, 1))."""
    H = E // P

    def nrm(*shape, std=0.02, mean=0.0):
        return (torch.randn(*shape, generator=gen, device=dev) * std + mean).bfloat16().contiguous()

    def uni(n, lo, hi):
        return torch.rand(n, generator=gen, device=dev) * (hi - lo) + lo

    import math
    dt0 = torch.exp(uni(H, math.log(1e-3), math.log(1e-1))).double()
    return mm.BlockWeights(Dm, E, P, N, 1, K, 1e-5, nrm(2 * E + 2 * N + H, Dm), nrm(E + 2 * N, K), nrm(E + 2 * N),
                           (dt0 + torch.log(-torch.expm1(-dt0))).float().contiguous(),
                           (-torch.exp(uni(H, 0.0, math.log(16.0)))).contiguous(),
                           torch.randn(H, generator=gen, device=dev).contiguous(), nrm(E, mean=1.0), nrm(Dm, E))


def graph_of(torch, fn, reps=1):
    """Capture `reps` consecutive calls in one CUDA graph (after an eager call that does the per-device
    set-up)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    torch.cuda.synchronize()
    return g


def run_stack(args, mm, torch, dev, timed, slowest, world, pk):
    """48-layer pre-norm stack (b4 L4096, d_model 2048, 64 heads) per width: the forward timed as CUDA-graph
    replays (L2 flushed before each), and each stage's roofline fraction from one traced eager forward."""
    S = STACK
    Dm, E, nl = S["d_model"], S["d_inner"], S["nlayers"]
    gen = torch.Generator(device=dev)
    gen.manual_seed(1003)
    layers = [device_block_weights(mm, torch, gen, Dm, E, S["d_head"], S["d_state"], dev) for _ in range(nl)]
    pws = [(1.0 + 0.02 * torch.randn(Dm, generator=gen, device=dev)).bfloat16() for _ in range(nl)]
    u = torch.randn(S["batch"], S["seq_len"], Dm, generator=gen, device=dev).bfloat16()
    out = torch.empty_like(u)
    T = S["batch"] * S["seq_len"]
    ws = torch.empty(max(mm.matmamba_stack_workspace(layers, [m] * nl, S["batch"], S["seq_len"])
                         for m in S["widths"]), dtype=torch.uint8, device=dev)
    res = {"workload": S["workload"], "timing": "CUDA-graph replay of the 48-layer forward, L2 flushed before each",
           "by_width": {}}
    for m in S["widths"]:
        ms_list = [m] * nl
        fn = lambda ms_list=ms_list: mm.matmamba_stack_fwd(layers, pws, u, ms_list, out=out, workspace=ws)  # noqa
        steps = max(2, min(args.steps, 5))
        g = graph_of(torch, fn)
        ms, _ = timed(g.replay, steps, 1)
        avg = slowest(sum(ms)) / steps
        del g
        mm.mm_trace_enable(nl * 8 + 16)
        fn()
        torch.cuda.synchronize()
        stg, kern = mm.mm_trace_collect()
        mm.mm_trace_enable(0)
        res["by_width"][str(m)] = {"ms_per_forward": avg, "tokens_per_s": world * T / (avg / 1e3),
                                   "kernels_per_forward": kern,
                                   "stages_per_layer": stage_table(stg, stack_work(m, T, Dm, E), pk)}
    del layers, ws
    return res


def run_decode(args, mm, torch, dev, timed, slowest, world, pk):
    """1000 consecutive recurrent steps of the 1.4B-class block for 256 sequences per width, from a
    prefilled N(0, 1) state: ten replays of a CUDA graph of 100 steps form the timed region (the state,
    537 MB, exceeds L2); each stage's roofline fraction from traced eager steps."""
    D = DECODE
    Dm, E, Bt = D["d_model"], D["d_inner"], D["batch"]
    H = E // D["d_head"]
    gen = torch.Generator(device=dev)
    gen.manual_seed(1004)
    w = device_block_weights(mm, torch, gen, Dm, E, D["d_head"], D["d_state"], dev)
    res = {"workload": D["workload"], "steps": D["steps"],
           "timing": "%d CUDA-graph replays of %d consecutive steps (state larger than L2, no flush)"
                     % (D["steps"] // D["graph_steps"], D["graph_steps"]), "by_width": {}}
    for m in D["widths"]:
        s = torch.randn(Bt, H, D["d_head"], D["d_state"], generator=gen, device=dev)
        c = torch.randn(Bt, E + 2 * D["d_state"], 3, generator=gen, device=dev).bfloat16()
        ut = torch.randn(Bt, Dm, generator=gen, device=dev).bfloat16()
        ot = torch.empty_like(ut)
        ws = torch.empty(mm.ssd_step_workspace(w, Bt, m), dtype=torch.uint8, device=dev)
        fn = lambda m=m, s=s, c=c, ut=ut, ot=ot, ws=ws: mm.ssd_step(w, s, c, ut, m, out_t=ot, workspace=ws)  # noqa
        g = graph_of(torch, fn, D["graph_steps"])
        reps = D["steps"] // D["graph_steps"]

        def run_all():
            for _ in range(reps):
                g.replay()
        ms, _ = timed(run_all, 1, 1)
        total_ms = slowest(ms[0])
        del g
        _, (stg, _) = timed(fn, 5, 2, trace=True)
        per = total_ms / D["steps"]
        res["by_width"][str(m)] = {"us_per_step": per * 1e3, "tokens_per_s": world * Bt / (per / 1e3),
                                   "stages": stage_table(stg, decode_work(m, Bt, Dm, E), pk)}
    return res


def run_only(args, mm, synth, torch, dev, timed):
    """One workload piece with few launches, for ncu captures; prints per-stage device times."""
    if args.only == "decode":
        pk, _ = peaks()
        res = run_decode(args, mm, torch, dev, timed, lambda v: v, 1, pk)
        print(json.dumps({"only": "decode", "by_width": {m: {"us_per_step": v["us_per_step"],
                                                            "stages_us": {k: s["ms_per_launch"] * 1e3
                                                                          for k, s in v["stages"].items()}}
                                                        for m, v in res["by_width"].items()}}))
        return
    if args.only == "block":
        B = BLOCK
        arrays = synth.block_params(B["d_model"], B["d_inner"], B["d_head"], B["d_state"], dtype="bf16", seed=1002)
        wt = mm.BlockWeights.from_arrays(arrays, B["d_model"], B["d_inner"], B["d_head"], B["d_state"],
                                         dtype=torch.bfloat16, device=dev)
        u = torch.from_numpy(synth.activations((B["batch"], B["seq_len"], B["d_model"]), "bf16", seed=1032)).to(dev)
        u = u.bfloat16()
        fn = lambda: mm.matmamba_block_fwd(wt, u, B["widths"][0], B["chunk"])  # noqa: E731
    else:
        S = SCAN
        inp = synth.ssd_inputs(S["batch"], S["seq_len"], S["heads"], S["d_head"], S["d_state"], 1, "bf16", seed=1001)
        g = {k: torch.from_numpy(v).to(dev) for k, v in inp.items()}
        for k in ("x", "B", "C"):
            g[k] = g[k].bfloat16()
        fn = lambda: mm.ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk=S["chunk"])  # noqa: E731
    ms, (stages, kernels) = timed(fn, args.steps, args.warmup, trace=True)
    print(json.dumps({"only": args.only, "ms_per_step": sum(ms) / len(ms), "stages": stages, "kernels": kernels}))


def cpu_baseline_scan(budget_s=6.0):
    """The fp64 oracle's sequential scan on rows of the standalone-scan workload (24 heads): whole 8192-token
    batch rows with every OpenMP thread for about budget_s, and one 2048-token prefix of a row on a single
    thread (a separate process started with OMP_NUM_THREADS=1)."""
    import numpy as np

    import oracle
    from nested_mamba2_selective_b200 import synth
    S = SCAN
    inp = synth.ssd_inputs(S["batch"], S["seq_len"], S["heads"], S["d_head"], S["d_state"], 1, "bf16", seed=1001)
    rows, t0 = 0, time.perf_counter()
    while rows < S["batch"] and time.perf_counter() - t0 < budget_s:
        sl = slice(rows, rows + 1)
        oracle.ssd_scan(inp["x"][sl], inp["dt"][sl], inp["A"], inp["B"][sl], inp["C"][sl], inp["D"])
        rows += 1
    el = time.perf_counter() - t0
    res = {"value": rows * S["seq_len"] / el, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
           "sample": "%d of %d batch rows x %d tokens, 24 heads (fp64 sequential scan, OpenMP)"
                     % (rows, S["batch"], S["seq_len"])}
    code = ("import sys, time; sys.path.insert(0, %r)\n"
            "import oracle\nfrom nested_mamba2_selective_b200 import synth\n"
            "i = synth.ssd_inputs(1, 2048, 24, 64, 128, 1, 'bf16', seed=1001)\n"
            "t = time.perf_counter(); oracle.ssd_scan(i['x'], i['dt'], i['A'], i['B'], i['C'], i['D'])\n"
            "print(2048 / (time.perf_counter() - t), oracle.num_threads())\n" % ROOT)
    try:
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120,
                           env=dict(os.environ, OMP_NUM_THREADS="1"))
        v, c = r.stdout.split()
        res["one_core"] = {"value": float(v), "unit": "tokens/s", "cores": int(c),
                           "sample": "one batch row x 2048 tokens, 24 heads"}
    except Exception as e:  # noqa: BLE001 - the 1-core figure is informative only
        res["one_core"] = {"error": str(e)[:200]}
    return res


def cpu_baseline_stack(layers=4, tokens=256):
    """The fp64 oracle's stack forward at full width on a bounded slice of the 48-layer workload: one batch
    row, a causal prefix of `tokens` tokens (exact for those outputs, by causality and batch independence)
    through `layers` layers of random weights; the rate for all 48 layers is the measured per-layer rate
    divided by 48 (layers cost the same)."""
    import numpy as np

    import oracle
    from nested_mamba2_selective_b200 import synth
    S = STACK
    dims = oracle.Dims(S["d_model"], S["d_inner"], S["d_head"], S["d_state"])
    params = [{k: v.astype(np.float64) for k, v in synth.block_params(S["d_model"], S["d_inner"], S["d_head"],
                                                                       S["d_state"], dtype="bf16",
                                                                       seed=1003 + l).items()} for l in range(layers)]
    prenorm = np.ones(S["d_model"])
    u = synth.activations((1, tokens, S["d_model"]), "bf16", seed=1003)
    t0 = time.perf_counter()
    oracle.stack_fwd(dims, layers, lambda l: params[l], lambda l: prenorm, u, [S["d_model"]] * layers)
    el = time.perf_counter() - t0
    return {"value": tokens / (el * S["nlayers"] / layers), "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "one batch row x %d-token prefix through %d of the 48 layers at width %d, scaled to 48 layers "
                      "(fp64 oracle, OpenMP)" % (tokens, layers, S["d_model"])}


def cpu_baseline_decode(seqs=4, steps=50):
    """The fp64 oracle's recurrent step at full width on `seqs` of the 256 sequences for `steps` consecutive
    tokens from an N(0, 1) state (sequences are independent)."""
    import numpy as np

    import oracle
    from nested_mamba2_selective_b200 import synth
    D = DECODE
    dims = oracle.Dims(D["d_model"], D["d_inner"], D["d_head"], D["d_state"])
    p = {k: v.astype(np.float64) for k, v in synth.block_params(D["d_model"], D["d_inner"], D["d_head"],
                                                                  D["d_state"], dtype="bf16", seed=1004).items()}
    H = D["d_inner"] // D["d_head"]
    ssm, conv = synth.states(seqs, H, D["d_head"], D["d_state"], D["d_inner"] + 2 * D["d_state"], 4, "bf16", seed=1004)
    ssm, conv = ssm.astype(np.float64), conv.astype(np.float64)
    u = synth.activations((steps, seqs, D["d_model"]), "bf16", seed=1004)
    t0 = time.perf_counter()
    for i in range(steps):
        oracle.block_step(dims, p, u[i], D["d_model"], ssm, conv)
    el = time.perf_counter() - t0
    return {"value": seqs * steps / el, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d of %d sequences x %d consecutive steps at width %d (fp64 oracle, OpenMP)"
                      % (seqs, D["batch"], steps, D["d_model"])}


def cpu_baseline(arrays, u_np, m, budget_s=10.0):
    """The fp64 oracle on whole batch rows of the headline workload until ~budget_s of CPU time."""
    import numpy as np

    import oracle
    dims = oracle.Dims(BLOCK["d_model"], BLOCK["d_inner"], BLOCK["d_head"], BLOCK["d_state"])
    p64 = {k: v.astype(np.float64) for k, v in arrays.items()}
    L = BLOCK["seq_len"]
    rows, t0 = 0, time.perf_counter()
    while rows < u_np.shape[0] and time.perf_counter() - t0 < budget_s:
        oracle.block_fwd(dims, p64, u_np[rows:rows + 1], m)
        rows += 1
    el = time.perf_counter() - t0
    return {"value": rows * L / el, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d of %d batch rows x %d tokens at width %d (fp64 sequential oracle, OpenMP)"
                      % (rows, u_np.shape[0], L, m)}


# ------------------------------------------------------------------------------------ reference arm

def run_reference(args):
    """The fp64 CPU oracle on the headline workload's config, a bounded sample per step."""
    import numpy as np

    import oracle
    from nested_mamba2_selective_b200 import synth
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if rank != 0:
        return
    oracle.build()
    B = BLOCK
    arrays = synth.block_params(B["d_model"], B["d_inner"], B["d_head"], B["d_state"], dtype="bf16", seed=1002)
    p64 = {k: v.astype(np.float64) for k, v in arrays.items()}
    u = synth.activations((B["batch"], B["seq_len"], B["d_model"]), "bf16", seed=1002 + 30)
    dims = oracle.Dims(B["d_model"], B["d_inner"], B["d_head"], B["d_state"])
    Ls = 256
    m0 = B["widths"][0]
    for i in range(args.warmup):
        oracle.block_fwd(dims, p64, u[i % B["batch"]:i % B["batch"] + 1, :Ls], m0)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.block_fwd(dims, p64, u[i % B["batch"]:i % B["batch"] + 1, :Ls], m0)
    el = time.perf_counter() - t0
    value = args.steps * Ls / el
    sample = "one batch row x %d tokens per step at width %d (fp64 sequential oracle, OpenMP)" % (Ls, m0)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": B["workload"], "batch": B["batch"], "seq_len": B["seq_len"],
                       "d_model": B["d_model"], "width": m0, "chunk": B["chunk"]},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def launch_ranks(args):
    """Start one rank per GPU when --gpus N > 1 and this process is not already a rank.

    Returns None when this process should run the benchmark itself (N = 1, or a rank started by
    torch.distributed.run whose WORLD_SIZE agrees with N), else an exit status: that of the
    launched job, or 2 when WORLD_SIZE and --gpus disagree."""
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is not None:
        if int(env_world) != args.gpus:
            sys.stderr.write("bench.py: --gpus %d but WORLD_SIZE=%s; launch one rank per GPU with matching counts\n"
                             % (args.gpus, env_world))
            return 2
        return None
    if args.gpus == 1:
        return None
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(args.gpus),
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    try:
        return subprocess.run(cmd, timeout=3600).returncode
    except subprocess.TimeoutExpired:
        sys.stderr.write("bench.py: the %d-rank job did not finish within an hour\n" % args.gpus)
        return 3


def run_stub(args):
    """Launcher check without a GPU: ranks over gloo, a host matmul as the step."""
    import numpy as np
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    a = np.random.default_rng(rank).standard_normal((128, 128))
    for _ in range(args.warmup):
        a = np.tanh(a @ a)
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        a = np.tanh(a @ a)
    slowest = max_over_ranks(time.perf_counter() - t0, world, dist, "cpu")
    if rank == 0:
        print(json.dumps({"impl": "stub", "metric": "host matmul steps/s (launcher check)", "n_gpus": world,
                          "value": whole_job_rate(1, args.steps, world, slowest), "unit": "steps/s",
                          "steps": args.steps, "warmup": args.warmup, "data": "stub"}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    a = parse()
    rc = None if a.ncu_summary else launch_ranks(a)
    if rc is not None:
        sys.exit(rc)
    if a.stub:
        run_stub(a)
    elif a.ncu_summary:
        ncu_summary(a.ncu_summary)
    elif a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
