"""Benchmark of the Hyena gated FFT long convolution on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload d768_l8k] [--no-cpu-baseline]

A step is one hyena_gated_fftconv call over the whole workload (short conv,
all order steps, output gate) with inputs resident in HBM.  Default workload:
B=4, C=768, L=8192, order 2, bf16 storage / fp32 math (the 1-D operator at
width 768 and 8K context).  The spectrum cache is built once, before timing.
Every step reads ~252 MB (> the 126 MB L2), so no explicit L2 flush is needed.
The K timed steps run back to back between two CUDA events on the launching
stream; the roofline's launch duration is that region's time per step (one
step is one call: at L = 8192 one kernel launch).

N > 1 (torchrun): every rank runs the same per-GPU workload on its own GPU
(rows are independent: no exchange), so scaling is weak; the time is the max
over ranks and value = all ranks' tokens / that time.

`--impl reference` times the float64 CPU oracle on the host cores on a
bounded sample of rows per step (the pages ship no runnable reference code).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Hyena op fwd tokens/s (B·L/s) at D=768, L=8K on 1×B200; % of HBM roofline"
UNIT = "tokens/s"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def load_bf16_peak():
    """Dense bf16 tensor-core peak (TFLOP/s) for a kernel timed alone (burst)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        if "bf16_tflops" in pk:
            return float(pk["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def time_events(fn, stream, steps: int, warmup: int = 3) -> float:
    """Median milliseconds per call of fn, CUDA events on `stream`."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return float(np.median([a.elapsed_time(b) for a, b in ev]))


def layer_extras(p, dev, stream, steps: int):
    """The layer around the operator on the same workload: in_proj and out_proj
    (tcgen05 GEMMs, bf16 in/out, fp32 accumulation) against the bf16 peak, and
    the spectrum build from the implicit filter (once per filter change)."""
    import torch
    from fft_long_convolution_02_b200 import binding as hb
    from fft_long_convolution_02_b200 import inputs as I
    out = {}
    if p.dtype == "bf16" and p.ndim == 1 and not p.per_sample and p.C % 8 == 0 and p.L % 8 == 0:
        lay = I.make_layer(p)
        bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        x, Wi, Wo = bf(lay["x"]), bf(lay["W_in"]), bf(lay["W_out"])
        bi, bo = torch.from_numpy(lay["b_in"]).to(dev), torch.from_numpy(lay["b_out"]).to(dev)
        u = torch.empty((p.B, p.Ctot, p.L), dtype=torch.bfloat16, device=dev)
        yv = torch.empty((p.B, p.C, p.L), dtype=torch.bfloat16, device=dev).normal_()
        o = torch.empty((p.B, p.L, p.C), dtype=torch.bfloat16, device=dev)
        t_in = time_events(lambda: hb.hyena_in_proj(x, Wi, bi, u, p.order, stream), stream, steps)
        t_out = time_events(lambda: hb.hyena_out_proj(yv, Wo, bo, o, stream), stream, steps)
        peak, kind = load_bf16_peak()
        f_in = 2.0 * p.B * p.L * p.C * p.Ctot
        f_out = 2.0 * p.B * p.L * p.C * p.C
        out["projections"] = {
            "kernel": "k_gemm_bf16 (tcgen05, TMA, bf16 operands, fp32 accumulation in tensor memory)",
            "in_proj_us": t_in * 1e3, "in_proj_tflops": f_in / (t_in / 1e3) / 1e12,
            "out_proj_us": t_out * 1e3, "out_proj_tflops": f_out / (t_out / 1e3) / 1e12,
            "peak_tflops": peak, "peak_kind": kind,
            "in_proj_frac": f_in / (t_in / 1e3) / 1e12 / peak, "out_proj_frac": f_out / (t_out / 1e3) / 1e12 / peak}
    if p.ndim == 1 and p.L <= 16384 and not p.per_sample:
        prm = I.implicit_filter_params(p)
        dprm = {k: (torch.from_numpy(v).to(dev) if isinstance(v, np.ndarray) else v) for k, v in prm.items()}
        D = torch.from_numpy(I.D_all(p)).to(dev)
        spec = torch.empty(hb.hyena_spectrum_bytes(p.C, p.shape, p.order), dtype=torch.uint8, device=dev)
        ws = torch.empty(hb.hyena_implicit_filter_workspace_bytes(p.L, prm["width"]), dtype=torch.uint8, device=dev)
        t_imp = time_events(lambda: hb.hyena_filter_spectrum_implicit(dprm, D, p.C, p.L, p.order, spec, ws,
                                                                      stream=stream), stream, max(3, steps // 5))
        k = torch.empty((p.order - 1, p.C, p.L), dtype=torch.float32, device=dev).normal_()
        t_st = time_events(lambda: hb.hyena_filter_spectrum(k, D, p.C, p.shape, p.order, spec, stream), stream,
                           max(3, steps // 5))
        out["implicit_filter_spectrum"] = {
            "what": "filter generation (embedding, Sin MLP width 64 with 2 inner layers, modulation) fused into the "
                    "spectrum build, once per filter change; not in the timed step",
            "ms": t_imp, "stored_filter_spectrum_ms": t_st}
    hb.hyena_kernel_status(stream)
    return out


def algorithmic_bytes(p, spectrum_row_bytes: int) -> int:
    """One read of u (all order+1 chunks), one read of the stored spectra
    (C rows per order step, B*C with per-sample filters), one write of y."""
    es = 2 if p.dtype == "bf16" else 4
    u = p.B * p.Ctot * p.n * es
    y = p.B * p.C * p.n * es
    spec = (p.order - 1) * p.FC * spectrum_row_bytes
    return u + spec + y


def paired_2d(p) -> bool:
    """256 x 256 images with bf16 storage and an even batch: the two images of a
    channel travel as one complex image through tensor-core passes (both forms)."""
    return (p.ndim == 2 and p.dtype == "bf16" and p.H == 256 and p.W == 256 and p.B % 2 == 0
            and not p.per_sample and p.order <= 3)


def spectrum_row_bytes(p) -> int:
    """Spectrum bytes per (step, channel) row the convolution kernel reads."""
    if p.ndim == 3:
        return (p.W + 1) * 2 * p.H * 2 * p.N1 * 8
    if p.ndim == 2:
        if paired_2d(p):
            # paired images: the whole bf16 plane (H x W circular, 2H x 2W padded)
            return (1 if p.circular else 4) * p.W * p.H * 4
        if p.circular:
            return (p.W // 2 + 1) * p.H * 8
        if p.dtype == "bf16" and p.H == 256 and p.W % 32 == 0 and p.order <= 3:
            # tensor-core column pass: bf16 plane of bins 0..W-1, complex64 last column
            return p.W * 2 * p.H * 4 + 2 * p.H * 8
        return (p.W + 1) * 2 * p.H * 8
    if p.L == 8192:
        return 8 * p.L                      # one plane: bf16 2L bins, or fp32 position layout
    if p.L <= 16384:
        return (p.L // 2 + 1) * 16
    return 8 * p.L


def source_hash(files) -> str:
    """Hash of the kernel sources a profile was taken on."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fft_long_convolution_02_b200", "csrc")
    for f in sorted(files):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary (profiles/traffic.json),
    only if it was taken on the kernel's current sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        entries = json.load(f)
    for e in entries:
        if e.get("kernel") == kernel and e.get("workload") == workload and \
                e.get("source_hash") == source_hash(e.get("sources", [])):
            return e.get("dram_bytes_per_launch")
    return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"hyena_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": float(max(smax)) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def _oracle_rows(orc, p, data, rows, cores):
    """The float64 oracle (FFT form) on rows b*C + c of the stacked inputs."""
    return orc.hyena_stacked(data["u"], data["k"], data["D"], data["sc_w"], data["sc_b"], B=p.B, C=p.C,
                             order=p.order, shape=p.shape, rows=rows, per_sample=p.per_sample,
                             circular=p.circular, method=2, nthreads=cores)


def cpu_baseline(p, data, budget_s: float = 15.0):
    """Time the float64 oracle (as it stands) on a bounded sample of rows."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    orc = oracle.default()
    rng = np.random.default_rng(0)
    rows = rng.choice(p.B * p.C, size=min(p.B * p.C, 8 * cores), replace=False)
    t0 = time.perf_counter()
    _oracle_rows(orc, p, data, rows, cores)
    dt = time.perf_counter() - t0
    # grow the sample to use about budget_s of CPU time
    n_more = int(len(rows) * max(0.0, budget_s / max(dt, 1e-3) - 1.0))
    n_more = min(n_more, p.B * p.C - len(rows))
    total_rows, total_t = len(rows), dt
    if n_more > 0:
        rows2 = rng.choice(p.B * p.C, size=n_more, replace=False)
        t0 = time.perf_counter()
        _oracle_rows(orc, p, data, rows2, cores)
        total_t += time.perf_counter() - t0
        total_rows += n_more
    # a row is one (b, c) pair; the operator's tokens are B*n over all C channels
    tok_s = total_rows * p.n / (p.C * total_t)
    return {"value": tok_s, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{total_rows} of {p.B * p.C} (b,c) rows, radix-2 FFT oracle in float64, "
                      f"{total_t:.1f} s; tokens/s = rows*n/(C*t)"}


def run_reference(args, p):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from fft_long_convolution_02_b200 import inputs as I
    cores = len(os.sched_getaffinity(0))
    orc = oracle.default()
    rng = np.random.default_rng(1)
    per_step = max(cores, 16)
    data = I.make_all(p)
    samples = [rng.choice(p.B * p.C, size=per_step, replace=False) for _ in range(args.warmup + args.steps)]
    for rows in samples[:args.warmup]:
        _oracle_rows(orc, p, data, rows, cores)
    t0 = time.perf_counter()
    for rows in samples[args.warmup:]:
        _oracle_rows(orc, p, data, rows, cores)
    dt = time.perf_counter() - t0
    tok_s = args.steps * per_step * p.n / (p.C * dt)
    line = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": config_of(p, "float64 (the oracle)"),
            "cpu_baseline": {"value": tok_s, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{per_step} (b,c) rows per step of {p.B * p.C}; float64 radix-2 "
                                       f"FFT oracle; tokens/s = rows*n/(C*t)"},
            "e2e": {"value": tok_s, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def kernel_of(p) -> str:
    """The dominant kernel hyena_gated_fftconv launches for problem p."""
    if p.ndim == 1 and p.L == 8192:
        return "k_conv_8192_tc" if (p.dtype == "bf16" and not p.per_sample and p.order <= 3) else "k_conv_4096"
    if p.ndim == 1 and p.L <= 16384:
        return "k_conv_onchip"
    if p.ndim == 1 and p.L == 65536 and p.dtype == "bf16" and not p.per_sample and p.order <= 3:
        return "k_conv_cluster"
    return "multipass" if p.ndim == 1 else ("grid2d" if p.ndim == 2 else "grid3d")


def launches_per_step(p) -> int:
    """Kernels one hyena_gated_fftconv call launches for problem p with the
    default workspace (the whole batch in one row group), as dispatched."""
    steps = p.order - 1
    if p.ndim == 1:
        if p.L <= 16384 or kernel_of(p) == "k_conv_cluster":
            return 1                          # every order step inside one kernel
        return 1 + 2 * steps                  # columns forward, then per step rows and inverse columns
    if p.ndim == 2:
        if paired_2d(p):
            return 3 * steps                  # paired images, per step: rows, columns, rows inverse
        if p.circular:
            return 1 + 2 * steps              # rows forward, per step columns and rows inverse
        if p.dtype == "bf16" and p.H == 256 and p.W % 32 == 0 and p.order <= 3:
            return 1 + 3 * steps              # per step: tensor-core columns, last column, rows inverse
        return 1 + 2 * steps
    return 1 + 4 * steps                      # 3-D: per step columns, depth, columns inverse, rows inverse


def math_of(p, kernel: str) -> str:
    """What the measured kernel computes in, as built."""
    if kernel == "k_conv_8192_tc":
        return ("DFT stages on tcgen05 tensor cores: bf16 operands and DFT matrices, fp32 accumulation; "
                "short conv, gates, twiddles and spectrum products fp32; spectrum read as bf16 (re, im)")
    if kernel == "k_conv_cluster":
        return ("2L-point transform split over 8-CTA clusters: 8-point DFTs, short conv, gates and twiddles fp32 "
                "on the CUDA cores; 16384-point DFT stages per CTA on tcgen05 tensor cores with bf16 operands and "
                "fp32 accumulation; exchanges as bf16 pairs; spectrum read as bf16 (re, im)")
    if paired_2d(p) and p.circular:
        return ("the two images of a channel as one complex image: row, column and row passes as 256-point DFTs "
                "(two 16-point stages) on tcgen05 tensor cores (bf16 operands, fp32 accumulation), gates and "
                "twiddles fp32, spectrum read as a bf16 (re, im) plane, intermediate kept as bf16 pairs in the "
                "workspace")
    if paired_2d(p):
        return ("the two images of a channel as one complex image: row, column and row passes as 512-point DFT "
                "stages on tcgen05 tensor cores (bf16 operands, fp32 accumulation), gates and twiddles fp32, "
                "spectrum read as a bf16 (re, im) plane, intermediate kept as bf16 pairs in the workspace")
    if p.ndim == 2 and not p.circular and p.dtype == "bf16" and p.H == 256 and p.W % 32 == 0 and p.order <= 3:
        return ("row passes fp32 on the CUDA cores; column pass of bins 0..W-1 as 512-point DFT stages on tcgen05 "
                "tensor cores (bf16 operands, fp32 accumulation, spectrum read as bf16 (re, im)), last bin column "
                "fp32; intermediate kept as bf16 pairs in the workspace between passes")
    if p.dtype == "bf16" and (p.ndim > 1 or p.L > 16384):
        return "fp32 (intermediate kept as bf16 pairs in the workspace between passes)"
    return "fp32"


def config_of(p, math: str):
    cfg = {"workload": p.name, "B": p.B, "C": p.C, "order": p.order,
           "shortconv": p.shortconv, "storage": p.dtype, "math": math}
    if p.per_sample:
        cfg["filters"] = "per-sample (one filter per (b, c) row)"
    if p.circular:
        cfg["boundary"] = "circular"
    if p.ndim == 1:
        cfg["L"] = p.L
    elif p.ndim == 2:
        cfg["H"], cfg["W"] = p.H, p.W
    else:
        cfg["N1"], cfg["H"], cfg["W"] = p.N1, p.H, p.W
    return cfg


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="d768_l8k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--channels", type=int, default=0,
                    help="override the workload's channel count C (smaller captures for ncu; "
                         "lines printed with it are not the workload's bench line)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from fft_long_convolution_02_b200 import inputs as I
    p = I.WORKLOADS[args.workload]
    if args.channels:
        import dataclasses
        p = dataclasses.replace(p, C=args.channels)
    if args.impl == "reference":
        run_reference(args, p)
        return

    import torch
    from fft_long_convolution_02_b200 import binding as hb
    from fft_long_convolution_02_b200 import dist as hd

    world, rank, local = hd.env_ranks()
    torch.cuda.set_device(local)
    hd.init("nccl", 120.0, torch.device("cuda", local))
    barrier = hd.barrier

    hb.load()
    dev = torch.device("cuda", local)
    data = I.make_all(p)
    if p.dtype == "bf16":
        u_host = torch.from_numpy(data["u"].view(np.int16)).view(torch.bfloat16)
        k_dev = torch.from_numpy(data["k"].view(np.int16)).view(torch.bfloat16).to(dev)
        tdt = torch.bfloat16
    else:
        u_host = torch.from_numpy(data["u"])
        k_dev = torch.from_numpy(data["k"]).to(dev)
        tdt = torch.float32
    u = u_host.to(dev)
    D = torch.from_numpy(data["D"]).to(dev)
    sc_w = torch.from_numpy(data["sc_w"]).to(dev) if data["sc_w"] is not None else None
    shape = hb.Circular(p.shape) if p.circular else p.shape      # the ABI's shape argument
    spec = torch.empty(hb.hyena_spectrum_bytes(p.FC, shape, p.order), dtype=torch.uint8, device=dev)
    y = torch.empty((p.B, p.C) + p.shape, dtype=tdt, device=dev)
    wsb = hb.hyena_gated_fftconv_workspace_bytes(p.B, p.C, shape, p.order)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev) if wsb else None
    stream = torch.cuda.current_stream()
    hb.hyena_filter_spectrum(k_dev, D, p.FC, shape, p.order, spec, stream)
    conv = hb.hyena_gated_fftconv_per_sample if p.per_sample else hb.hyena_gated_fftconv
    torch.cuda.synchronize()

    def step(uu=None):
        conv(u if uu is None else uu, y, spec, sc_w, None, p.B, p.C, shape, p.order, ws,
                               stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()

    clocks = ClockSampler(local)
    clocks.start()
    # keep the GPU under the same load (untimed steps) for the sampler's first
    # samples, so that the clocks it reports are the clocks under this load
    t_load = time.perf_counter() + 0.4
    while time.perf_counter() < t_load:
        for _ in range(8):
            step()
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("hyena timed steps")
    # the K steps back to back between two events on the launching stream (events
    # between the steps would add their own gaps); a step is one call, so the
    # average step of this region is the average duration of the call's kernels
    t_start.record(stream)
    for i in range(args.steps):
        step()
    t_stop.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    elapsed_ms = t_start.elapsed_time(t_stop)
    launch_ms = [elapsed_ms / args.steps]
    elapsed_ms = hd.max_over_ranks(elapsed_ms, dev)

    # the same workload with every transform multiply in fp32 (bf16 storage,
    # fp32 arithmetic: HYENA_FLAG_FP32_TRANSFORM), where that changes the kernel
    fp32_ms = None
    if kernel_of(p) == "k_conv_8192_tc":
        def step32():
            hb.hyena_gated_fftconv_ex(u, y, spec, sc_w, None, p.B, p.C, shape, p.order, ws,
                                      flags=hb.HYENA_FLAG_FP32_TRANSFORM, stream=stream)
        for _ in range(args.warmup):
            step32()
        torch.cuda.synchronize()
        barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            step32()
        f1.record(stream)
        torch.cuda.synchronize()
        fp32_ms = hd.max_over_ranks(f0.elapsed_time(f1), dev)

    extras = layer_extras(p, dev, stream, args.steps)

    # end to end through the C ABI with host buffers (pinned), copies timed:
    # hyena_gated_fftconv_host pipelines each step's chunk copies against the
    # kernels (per-sample filters: copy, convolve, copy back on one stream)
    u_pin = u_host.pin_memory()
    y_pin = torch.empty(y.shape, dtype=tdt).pin_memory()
    u_e2e = torch.empty_like(u)

    def e2e_step():
        if p.per_sample:
            u_e2e.copy_(u_pin, non_blocking=True)
            step(u_e2e)
            y_pin.copy_(y, non_blocking=True)
        else:
            hb.hyena_gated_fftconv_host(u_pin, y_pin, u_e2e, y, spec, sc_w, None, p.B, p.C, shape, p.order, ws,
                                        chunk_rows=0, stream=stream)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("hyena end-to-end steps")
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = hd.max_over_ranks(e2e_ms, dev)

    tokens_per_step = p.B * p.n
    value = world * tokens_per_step * args.steps / (elapsed_ms / 1e3)
    e2e_value = world * tokens_per_step * args.e2e_steps / (e2e_ms / 1e3)
    peak, peak_kind = load_peaks()
    spec_row = spectrum_row_bytes(p)
    alg = algorithmic_bytes(p, spec_row)
    avg_launch_s = float(np.mean(launch_ms)) / 1e3
    achieved = alg / avg_launch_s / 1e9
    kernel = kernel_of(p)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if p.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": dict(config_of(p, math_of(p, kernel)), parallelism=f"replicas{world}" if world > 1 else "single",
                       l2="inputs larger than L2 (%.0f MB per step)" % (alg / 1e6)),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "frac_of_8TBps": achieved / 8000.0,
                     "traffic": committed_traffic(kernel, p.name),
                     "algorithmic_bytes_per_launch": alg, "kernel": kernel,
                     "avg_launch_us": avg_launch_s * 1e6},
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": u.numel() * u.element_size(),
                "d2h_bytes_per_step": y.numel() * y.element_size()},
        "gpu_launches": args.steps * launches_per_step(p),
        "fp32_transform": None if fp32_ms is None else {
            "kernel": "k_conv_4096", "flag": "HYENA_FLAG_FP32_TRANSFORM",
            "math": "fp32 throughout (register FFT on the CUDA cores; complex64 spectrum plane)",
            "value": world * tokens_per_step * args.steps / (fp32_ms / 1e3), "unit": UNIT,
            "ms_per_step": fp32_ms / args.steps,
            "roofline_frac": alg / (fp32_ms / args.steps / 1e3) / 1e9 / peak},
        "clocks": clk,
    }
    line.update(extras)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(p, data)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
