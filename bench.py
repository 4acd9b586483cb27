#!/usr/bin/env python
"""Benchmark of the SVDQuant W4A4 linear layer (svdq_linear) on B200.

Workload: FLUX.1-like FFN up projection, M=4608 tokens (4096 image + 512
text), K=3072, N=12288, rank 32, NVFP4 (E2M1 + E4M3 per 16 + fp32 tensor
scale), bf16 activations with 1% outlier channels x50 -- synthetic data of
that shape (no trained weights or activations exist here).

One step = one svdq_linear call (activation quantisation + down projection
kernel, then the tcgen05 GEMM with the fused low-rank epilogue) over one batch
of 4608 tokens resident in HBM.  L2 is flushed (256 MiB write) before every
timed step; each step is timed with CUDA events on the launching stream.  The
K timed steps are one pass; the pass is repeated (each pass bracketed by a
barrier and a device synchronisation) until the clock sampler has seen the
load, and the median pass gives ms_per_step.

Few tokens (M <= 256, `--workload ... --tokens M`): one step is a CUDA-graph
replay of 200 calls, rotating over enough copies of the prepared weights that
together they exceed twice the L2, so every call streams its weights from HBM.

Metric: TFLOP/s = (2 M K N + 2 M r (K + N)) / t.  Multi-GPU (torchrun): one
independent layer replica per GPU, each with its own token batch (weak
scaling, no data-path collective); value = all ranks' FLOPs / max-over-ranks
time.  `--impl reference` times the CPU oracle on the host cores instead, and
`--impl reference --error-report` prints the oracle's error against the
unquantised X W + b at rank 0 and at rank r for every workload preset.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "flux_ffn_up_nvfp4"
METRIC = "fused SVDQuant W4A4 linear TFLOP/s and % of B200 FP4/INT8 tensor peak"
NOMINAL_FP4_TFLOPS = 9000.0
NOMINAL_FP8_TFLOPS = 4500.0
NOMINAL_BF16_TFLOPS = 2250.0
FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20
GRAPH_CALLS = 200
SMALL_M = 256
MIN_TIMED_SECONDS = 0.6


def flops(M, K, N, r):
    return 2.0 * M * K * N + 2.0 * M * r * (K + N)


def gemm_alg_bytes(M, K, N, r, fmt):
    """Algorithmic bytes of one GEMM launch (kernel 2): quantised X codes and
    scales + the down projection in, weight codes/scales + L2 + bias in,
    bf16 Y out."""
    xq = M * K // 2 + M * K // 16 if fmt == "nvfp4" else M * K + M * (K // 64) * 4
    wq = N * K // 2 + N * K // 16 if fmt == "nvfp4" else N * K + N * (K // 64) * 4
    return xq + M * 2 * r * 2 + wq + N * 2 * r * 2 + N * 4 + M * N * 2


def layer_alg_bytes(M, K, N, r, fmt):
    """Algorithmic bytes of the whole layer: X once, Y once, the weight codes
    and scales, L1, L2, b and inv_lambda (the quantised-X hand-off between the
    two kernels is implementation traffic, not counted)."""
    wq = N * K // 2 + N * K // 16 if fmt == "nvfp4" else N * K // 2 + N * (K // 64) * 4
    return M * K * 2 + M * N * 2 + wq + K * r * 2 + r * N * 2 + N * 4 + K * 4


# The files that define the kernels and the data layouts they read: an ncu
# summary's counters stand for these exact sources (host-only API additions
# to the public header do not invalidate them).
DEVICE_SOURCES = ("rank_gemm_svdq_b200/csrc/svdq_device.cu", "rank_gemm_svdq_b200/csrc/ptx.cuh",
                  "rank_gemm_svdq_b200/csrc/layout.h")
GEMM_PROFILE = "profiles/gemm_nvfp4_pair_kernel_flux_ffn_up.md"


def profiled_traffic():
    """DRAM bytes per GEMM launch from the committed ncu summary, or None when
    the device sources changed since that capture (its source_sha256)."""
    import hashlib
    try:
        h = hashlib.sha256()
        for f in DEVICE_SOURCES:
            with open(os.path.join(ROOT, f), "rb") as fh:
                h.update(fh.read())
        fields = {}
        with open(os.path.join(ROOT, GEMM_PROFILE)) as fh:
            for line in fh:
                if ":" in line and line.split(":")[0] in ("traffic_bytes_per_launch", "source_sha256"):
                    k, v = line.split(":", 1)
                    fields[k] = v.strip()
        if fields.get("source_sha256") == h.hexdigest():
            return int(fields["traffic_bytes_per_launch"])
    except Exception:
        pass
    return None


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 50 ms in a thread."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_id: str):
        self.dev_id = dev_id
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", self.dev_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        rows = [s for (t, s) in self.samples if t0 <= t <= t1]
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0])); mx = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def device_smi_id(torch, dev):
    try:
        pr = torch.cuda.get_device_properties(dev)
        return f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        return vis.split(",")[dev] if vis else str(dev)


def oracle_layer_from_library(wl, X_cal):
    """The CPU oracle's layer, built from the library's host-prepared factors
    (so that the CPU baseline of the product arm runs the same layer as the
    GPU; the offline SVD is not part of the timed linear)."""
    import rank_gemm_svdq_b200 as sv
    import synth
    from oracle import svdquant as sq
    p = sv.params(wl.K, wl.N, wl.rank, wl.fmt, wl.dtype, wl.alpha, wl.smooth)
    blob, _ = sv.prepare(p, wl.Wt, wl.bias, X_cal)
    c = sv.blob_export(p, blob)
    if wl.dtype == "fp16":
        L1, L2 = c.L1.view(np.float16).astype(np.float64), c.L2.view(np.float16).astype(np.float64)
    else:
        L1, L2 = synth.bf16_bits_to_f64(c.L1), synth.bf16_bits_to_f64(c.L2)
    return sq.prepare(synth.dtype_to_f64(X_cal, wl.dtype), wl.Wt, wl.bias, wl.rank, wl.fmt, wl.dtype, wl.alpha,
                      wl.smooth, factors=(c.inv_lambda, L1, L2))


def oracle_layer_own(wl, X_cal, rank=None, smooth=None):
    """The CPU oracle's layer prepared by the oracle alone (LAPACK route to the
    truncated SVD for full-size layers): the reference arm's layer."""
    import synth
    from oracle import svdquant as sq
    rank = wl.rank if rank is None else rank
    smooth = wl.smooth if smooth is None else smooth
    return sq.prepare(synth.dtype_to_f64(X_cal, wl.dtype), wl.Wt, wl.bias, rank, wl.fmt, wl.dtype, wl.alpha,
                      smooth, svd="lapack")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(i["num_threads"] for i in threadpool_info())
    except Exception:
        return os.cpu_count()


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return None


def oracle_rate(x, ref, M, K, N, r, min_seconds):
    from oracle import svdquant as sq
    reps, t0 = 0, time.perf_counter()
    while True:
        sq.forward(x, ref)
        reps += 1
        if time.perf_counter() - t0 >= min_seconds:
            break
    dt = (time.perf_counter() - t0) / reps
    return flops(M, K, N, r) / dt / 1e12, reps, dt


def cpu_baseline(wl, ref, min_seconds=10.0):
    """The oracle's linear part over the whole layer (all M tokens), repeated
    until at least `min_seconds` of CPU work, on all host cores; plus the tiny
    INT4 layer on one core."""
    value, reps, dt = oracle_rate(wl.x_f64(), ref, wl.M, wl.K, wl.N, wl.rank, min_seconds)
    out = {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
           "sample": f"whole layer ({wl.M} tokens) x {reps} repetitions, {dt:.2f} s each, float64 numpy/BLAS",
           "cpu": cpu_model()}
    try:
        import synth
        from threadpoolctl import threadpool_limits
        tiny = synth.make_workload("tiny_int4")
        tref = oracle_layer_own(tiny, tiny.X)
        with threadpool_limits(limits=1):
            v1, reps1, dt1 = oracle_rate(tiny.x_f64(), tref, tiny.M, tiny.K, tiny.N, tiny.rank, 2.0)
        out["tiny_int4_single_thread"] = {"value": v1, "unit": "TFLOP/s", "cores": 1,
                                          "sample": f"tiny INT4 layer (256 x 512 x 512, rank 16) x {reps1}, "
                                                    f"{1e3 * dt1:.1f} ms each"}
    except Exception as e:  # the main baseline stands without it
        out["tiny_int4_single_thread"] = {"error": str(e)}
    return out


def replica_batch(wl, rank):
    """Token batch of replica `rank`: rank 0 keeps the workload's own X, every
    other rank draws its own seeded batch of the same preset (same shape and
    outlier model; weak scaling: one independent batch per GPU, same layer
    weights)."""
    import synth
    if rank == 0:
        return wl.X
    if wl.name in synth.PRESETS:
        return synth.make_workload(wl.name, seed=rank, M=wl.M, with_w=False).X
    return synth.make_x(rank, wl.M, wl.K, wl.dtype, int(wl.info.get("outlier_channels", 0)),
                        float(wl.info.get("outlier_factor", 1.0)))


def max_over_ranks(value, dist, device):
    """Largest `value` over all ranks (the job's time is its slowest rank)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def config_dict(wl, world, small):
    if wl.name == WORKLOAD and wl.M == 4608:
        desc = (f"{WORKLOAD}: FLUX.1-like FFN up projection M={wl.M} K={wl.K} N={wl.N} rank={wl.rank} "
                f"NVFP4 (E2M1, E4M3/16, fp32 tensor scale), bf16 X, 1% outlier channels x50")
    else:
        desc = f"{wl.name}: M={wl.M} K={wl.K} N={wl.N} rank={wl.rank} {wl.fmt} {wl.dtype} X"
    d = {"workload": desc, "M": wl.M, "K": wl.K, "N": wl.N, "rank": wl.rank, "format": wl.fmt,
         "act_dtype": wl.dtype, "parallelism": f"replicas x{world} (token batches, no collective)"}
    if small:
        d["l2"] = (f"step = CUDA-graph replay of {GRAPH_CALLS} calls rotating over weight copies "
                   f"larger than 2x L2 together")
    else:
        d["l2"] = "flushed by a 256 MiB write before every timed step"
    return d


def gemm_roofline(wl, ms_gemm, ms_act, ms_step, peaks, probed):
    """Roofline of the dominant kernel (the GEMM) and of the whole layer.

    Below the ridge (~1380 flop/B for FP4, ~690 for E4M3-coded INT4: M <= 256
    here) the GEMM is bound by HBM: algorithmic bytes against the measured copy
    bandwidth.  Above it, by the tensor cores: `peak` is the measured burst
    cuBLAS bf16 rate times the nominal dense ratio of the MMA kind (FP4 x4,
    FP8 x2); the same achieved rate is also given against the tcgen05 MMA rate
    probed live in this run and against the nominal dense peak.  `layer` holds
    the same fractions for the whole svdq_linear step (both kernels)."""
    M, K, N, r = wl.M, wl.K, wl.N, wl.rank
    nvfp4 = wl.fmt == "nvfp4"
    kernel = "gemm_nvfp4_pair_kernel" if nvfp4 else "gemm_int4_kernel"
    f = flops(M, K, N, r)
    alg_bytes = gemm_alg_bytes(M, K, N, r, wl.fmt)
    nominal = NOMINAL_FP4_TFLOPS if nvfp4 else NOMINAL_FP8_TFLOPS
    probe = (probed or {}).get("mxf4nvf4_pair" if nvfp4 else "e4m3")
    common = {"kernel": kernel, "alg_flops_per_launch": f, "alg_bytes_per_launch": alg_bytes,
              "traffic": profiled_traffic() if wl.name == WORKLOAD and wl.M == 4608 else None,
              "kernel_ms": {"gemm": ms_gemm, "act_quant": ms_act}}
    layer_tflops = f / (ms_step * 1e-3) / 1e12
    layer_bytes = layer_alg_bytes(M, K, N, r, wl.fmt)
    if M <= SMALL_M:
        achieved = alg_bytes / (ms_gemm * 1e-3) / 1e9
        if peaks and "hbm_gbs" in peaks:
            peak, note = float(peaks["hbm_gbs"]), f"of measured: copy bandwidth {peaks['hbm_gbs']} GB/s"
        else:
            peak, note = 6650.0, "of fallback: 6.65 TB/s"
        layer_gbs = layer_bytes / (ms_step * 1e-3) / 1e9
        return dict(bound="hbm", achieved=achieved, peak=peak, unit="GB/s", frac=achieved / peak,
                    peak_source=note, layer={"achieved_gbs": layer_gbs, "alg_bytes": layer_bytes,
                                             "frac_of_measured_hbm": layer_gbs / peak,
                                             "achieved_tflops": layer_tflops}, **common)
    ratio = nominal / NOMINAL_BF16_TFLOPS
    # The timed loop lasts tens of milliseconds at full clocks, so the GEMM is
    # compared with the burst (not the power-capped sustained) cuBLAS figure.
    if peaks and "bf16_tflops" in peaks:
        peak = float(peaks["bf16_tflops"]) * ratio
        note = (f"of measured: burst cuBLAS bf16 {peaks['bf16_tflops']} TFLOP/s x {ratio:g} "
                f"(nominal dense {'FP4' if nvfp4 else 'FP8'}/BF16 ratio)")
    else:
        peak, note = 1590.0 * ratio, f"of fallback: 1.59 PFLOP/s burst bf16 x {ratio:g}"
    achieved = f / (ms_gemm * 1e-3) / 1e12
    out = dict(bound="tensor", achieved=achieved, peak=peak, unit="TFLOP/s", frac=achieved / peak,
               peak_source=note, frac_of_nominal=achieved / nominal, **common)
    lay = {"achieved_tflops": layer_tflops, "frac_of_measured": layer_tflops / peak,
           "frac_of_nominal": layer_tflops / nominal}
    if probe:
        out["probed_mma_tflops"] = probe
        out["frac_of_probed_mma"] = achieved / probe
        lay["frac_of_probed_mma"] = layer_tflops / probe
    out["layer"] = lay
    return out


def probe_tensor_peaks(sv, torch):
    """tcgen05 MMA rates of this GPU, TFLOP/s, measured now by the library's
    probe kernel: every SM issues back-to-back MMAs (timed with events)."""
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    shapes = {"mxf4nvf4_pair": (1, 256 * 256 * 64), "mxf4nvf4": (0, 128 * 256 * 64),
              "bf16": (2, 128 * 256 * 16), "e4m3": (3, 128 * 256 * 32), "s8": (4, 128 * 256 * 32)}
    iters = 4096
    cycles = torch.zeros(sms + 2, dtype=torch.int64, device="cuda")
    out = {}
    for name, (op, mnk) in shapes.items():
        units = sms // 2 if op == 1 else sms
        best = 0.0
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            sv.probe_tc(op, iters, sms, cycles)
            b.record()
            torch.cuda.synchronize()
            best = max(best, 2.0 * mnk * iters * units / (a.elapsed_time(b) * 1e-3) / 1e12)
        out[name] = best
    assert sv.get_status() == sv.OK
    return out


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on the host cores, for
    the same workload (prepared by the oracle itself), a bounded sample of
    tokens per step."""
    if rank != 0:
        return
    import synth
    from oracle import svdquant as sq
    if args.error_report:
        error_report(args)
        return
    wl = synth.make_workload(args.workload)
    X_cal = wl.X
    if args.tokens:
        wl.X = np.ascontiguousarray(wl.X[:args.tokens])
        wl.M = args.tokens
    ref = oracle_layer_own(wl, X_cal)
    x = wl.x_f64()
    S = min(256, wl.M)
    times = []
    for it in range(args.warmup + args.steps):
        r0 = (it * S) % wl.M
        rows = slice(r0, min(r0 + S, wl.M))
        t0 = time.perf_counter()
        sq.forward(x[rows], ref)
        dt = time.perf_counter() - t0
        if it >= args.warmup:
            times.append((dt, rows.stop - rows.start))
    tot = sum(t for t, _ in times)
    toks = sum(n for _, n in times)
    value = flops(toks, wl.K, wl.N, wl.rank) / tot / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(wl, world, small=wl.M <= SMALL_M),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                             "cpu": cpu_model(),
                             "sample": f"each step: {S} consecutive of the {wl.M} tokens (rotating), "
                                       f"oracle float64 numpy/BLAS, layer prepared by the oracle "
                                       f"(LAPACK truncated SVD)"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def error_report(args):
    """The oracle's relative Frobenius error against the unquantised layer
    X W + b, at rank 0 without smoothing (plain W4A4) and at the preset's rank
    with smoothing (SVDQuant), for every preset at its full token count."""
    import synth
    from oracle import svdquant as sq
    names = args.error_report.split(",") if args.error_report != "all" else list(synth.PRESETS)
    for name in names:
        wl = synth.make_workload(name)
        t0 = time.perf_counter()
        x = wl.x_f64()
        exact = sq.exact_output(x, wl.Wt, wl.bias)
        e0 = sq.rel_fro(sq.forward(x, oracle_layer_own(wl, wl.X, rank=0, smooth=False)), exact)
        p = oracle_layer_own(wl, wl.X)
        er = sq.rel_fro(sq.forward(x, p), exact)
        # rank r without smoothing and rank 0 with smoothing, for the split of the gain
        e0s = sq.rel_fro(sq.forward(x, oracle_layer_own(wl, wl.X, rank=0, smooth=True)), exact)
        print(json.dumps({"workload": name, "M": wl.M, "K": wl.K, "N": wl.N, "rank": wl.rank, "format": wl.fmt,
                          "E_0": e0, "E_0_smoothed": e0s, "E_r": er,
                          "max_over_median_amax": wl.info.get("max_over_median_amax"),
                          "seconds": time.perf_counter() - t0}), flush=True)


def run_chain(args):
    """Two chained layers, FLUX FFN up (M 4608, K 3072 -> N 12288) into an FFN
    down projection (12288 -> 3072, rank 32), both NVFP4: the up projection's
    GEMM emits the down projection's quantised input (svdq_gemm_chain) against
    the same two layers run one after the other (svdq_linear twice, the
    12288-wide bf16 output written and read back).  One step = both layers
    after a 256 MiB flush; prints one JSON line (TFLOP/s over both layers)."""
    import torch
    import rank_gemm_svdq_b200 as sv
    import synth

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    wl = synth.make_workload(WORKLOAD, seed=0)
    M, K, N, r = wl.M, wl.K, wl.N, wl.rank
    N2, r2 = 3072, 32
    p1 = sv.params(K, N, r, "nvfp4", "bf16", wl.alpha, wl.smooth)
    blob1 = torch.from_numpy(sv.prepare(p1, wl.Wt, wl.bias, wl.X)[0]).to(dev)
    X = torch.from_numpy(wl.X.view(np.int16)).to(dev).view(torch.bfloat16)
    ws1 = torch.empty(sv.workspace_bytes(p1, M), dtype=torch.uint8, device=dev)
    Y1 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    sv.linear(p1, blob1, X, M, Y1, ws1)
    torch.cuda.synchronize()
    # the down projection is calibrated on what it sees: the up projection's output
    p2 = sv.params(N, N2, r2, "nvfp4", "bf16")
    Wt2, b2 = synth.make_weight(1, N2, N), synth.make_bias(1, N2)
    blob2 = torch.from_numpy(sv.prepare(p2, Wt2, b2, Y1.view(torch.int16).cpu().numpy())[0]).to(dev)
    ws = torch.empty(sv.chain_workspace_bytes(p1, p2, M), dtype=torch.uint8, device=dev)
    ws2 = torch.empty(sv.workspace_bytes(p2, M), dtype=torch.uint8, device=dev)
    Y2 = torch.empty((M, N2), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def chained(i):
        sv.quantize_act(p1, blob1, X, M, ws, stream)
        sv.gemm_chain(p1, blob1, M, p2, blob2, ws, ws2, stream)
        sv.gemm(p2, blob2, M, Y2, ws2, stream)

    def unfused(i):
        sv.linear(p1, blob1, X, M, Y1, ws1, stream)
        sv.linear(p2, blob2, Y1, M, Y2, ws2, stream)

    def timed(fn, steps):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        with torch.cuda.stream(stream):
            for i in range(steps):
                flush.fill_(i & 0xFF)
                evs[i][0].record(stream)
                fn(i)
                evs[i][1].record(stream)
        torch.cuda.synchronize()
        return float(np.median([a.elapsed_time(b) for a, b in evs]))

    for fn in (chained, unfused):
        timed(fn, args.warmup)
    assert sv.get_status() == sv.OK
    sampler = ClockSampler(device_smi_id(torch, dev.index or 0))
    sampler.start()
    time.sleep(0.3)
    t0 = time.time()
    ms_cs, ms_us = [], []
    while time.time() - t0 < MIN_TIMED_SECONDS or len(ms_cs) < 3:   # long enough for the clock samples
        ms_cs.append(timed(chained, args.steps))
        ms_us.append(timed(unfused, args.steps))
    ms_c, ms_u = float(np.median(ms_cs)), float(np.median(ms_us))
    t1 = time.time()
    sampler.stop()
    st = sv.get_status()
    assert st == sv.OK, sv.status_string(st)
    fl = flops(M, K, N, r) + flops(M, N, N2, r2)
    print(json.dumps({
        "metric": METRIC, "value": fl / (ms_c * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_c, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD} -> ffn down {N}x{N2} r{r2}, chained", "M": M,
                   "layers": [[K, N, r], [N, N2, r2]], "l2": "256 MiB flush per step"},
        "unfused": {"ms_per_step": ms_u, "value": fl / (ms_u * 1e-3) / 1e12},
        "timing": {"passes": len(ms_cs), "per_step": "median over steps, then over passes"},
        "clocks": sampler.summary(t0, t1), "gpu_launches": 8 * args.steps * len(ms_cs)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="another synthetic layer preset (synth.PRESETS); the default is the headline layer")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run on the first M tokens of the workload (calibration still uses all of them)")
    ap.add_argument("--error-report", default="",
                    help="with --impl reference: 'all' or comma-separated presets; prints E_0 / E_r")
    ap.add_argument("--chain", action="store_true",
                    help="two chained NVFP4 layers (FFN up -> down), fused next-layer input vs unfused")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.chain:
        run_chain(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import rank_gemm_svdq_b200 as sv
    import synth

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()

    wl = synth.make_workload(args.workload, seed=0)
    X_cal = wl.X
    if args.tokens:
        wl.X = np.ascontiguousarray(wl.X[:args.tokens])
        wl.M = args.tokens
    wl.X = replica_batch(wl, rank)
    if not args.tokens:
        X_cal = wl.X
    small = wl.M <= SMALL_M
    p = sv.params(wl.K, wl.N, wl.rank, wl.fmt, wl.dtype, wl.alpha, wl.smooth)
    blob_host, _ = sv.prepare(p, wl.Wt, wl.bias, X_cal)
    dev = torch.device("cuda", local)
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float16
    X = torch.from_numpy(wl.X.view(np.int16)).to(dev).view(tdt)
    Y = torch.empty((wl.M, wl.N), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(sv.workspace_bytes(p, wl.M), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    M, K, N, r = wl.M, wl.K, wl.N, wl.rank
    # weight copies: one, or (few tokens) enough to exceed twice the L2 together
    n_copies = max(4, math.ceil(2 * L2_BYTES / blob_host.nbytes)) if small else 1
    n_copies = min(n_copies, 64)
    blobs = [torch.from_numpy(blob_host).to(dev) for _ in range(n_copies)]
    blob = blobs[0]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    probed = probe_tensor_peaks(sv, torch)

    if small:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            sv.linear(p, blob, X, M, Y, ws, stream)     # set-up outside the capture
            stream.synchronize()
            with torch.cuda.graph(graph, stream=stream):
                for i in range(GRAPH_CALLS):
                    sv.linear(p, blobs[i % n_copies], X, M, Y, ws, stream)
        calls_per_step = GRAPH_CALLS

        def step(i):
            graph.replay()
    else:
        calls_per_step = 1

        def step(i):
            flush.fill_(i & 0xFF)
            sv.linear(p, blob, X, M, Y, ws, stream)

    def timed_pass(fn, steps):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        with torch.cuda.stream(stream):
            for i in range(steps):
                if not small:
                    flush.fill_(i & 0xFF)
                evs[i][0].record(stream)
                fn(i)
                evs[i][1].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    def step_body(i):
        if small:
            graph.replay()
        else:
            sv.linear(p, blob, X, M, Y, ws, stream)

    # warm-up
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize()
    assert sv.get_status() == sv.OK
    w0 = time.time()
    timed_pass(step_body, args.steps)
    pass_s = max(time.time() - w0, 1e-4)
    passes = int(min(500, max(5, math.ceil(MIN_TIMED_SECONDS / pass_s))))

    sampler = ClockSampler(device_smi_id(torch, local))
    sampler.start()
    time.sleep(0.3)
    pass_ms = []
    t0 = time.time()
    for _ in range(passes):
        barrier()
        torch.cuda.synchronize()
        ms = timed_pass(step_body, args.steps)
        torch.cuda.synchronize()
        barrier()
        pass_ms.append(max_over_ranks(float(sum(ms)), dist, dev))
    t1 = time.time()
    time.sleep(0.1)
    sampler.stop()
    clocks = sampler.summary(t0, t1)
    st = sv.get_status()
    assert st == sv.OK, sv.status_string(st)

    ms_per_step = float(np.median(pass_ms)) / args.steps
    ms_per_call = ms_per_step / calls_per_step
    value = flops(M, K, N, r) * world / (ms_per_call * 1e-3) / 1e12

    # per-kernel timing (same flush protocol), for the roofline of the dominant kernel
    def quant_only(i):
        sv.quantize_act(p, blobs[i % n_copies], X, M, ws, stream)

    def gemm_only(i):
        sv.gemm(p, blobs[i % n_copies], M, Y, ws, stream)

    ksteps = 100
    if small:
        # few tokens: the kernels one at a time after a flush each (their
        # launch and set-up costs included), median
        def flushed(fn):
            evs = []
            with torch.cuda.stream(stream):
                for i in range(ksteps):
                    flush.fill_(i & 0xFF)
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream); fn(i); b.record(stream)
                    evs.append((a, b))
            torch.cuda.synchronize()
            return float(np.median([a.elapsed_time(b) for a, b in evs]))
        ms_act = flushed(quant_only)
        with torch.cuda.stream(stream):
            quant_only(0)
        ms_gemm = flushed(gemm_only)
    else:
        ms_act = float(np.mean(timed_pass(quant_only, ksteps)))
        with torch.cuda.stream(stream):
            quant_only(0)
        ms_gemm = float(np.mean(timed_pass(gemm_only, ksteps)))

    # End to end through the C ABI with host buffers: every step copies its X in
    # from pinned host memory and its Y back out.  Steps are pipelined over
    # three streams (copy in / compute / copy out) with two device buffer sets,
    # so one step's transfers overlap its neighbours' work, as a serving loop
    # would run; the time is first copy-in to last copy-out, over all steps.
    Xh = torch.from_numpy(wl.X.view(np.int16)).view(tdt).pin_memory()
    Yh = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    Xd = [torch.empty_like(X) for _ in range(2)]
    Yd = [Y, torch.empty_like(Y)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_pipeline(n):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(n):
            b = i & 1
            if i >= 2:
                s_in.wait_event(ev_c[b])          # X slot b: step i-2 has consumed it
            with torch.cuda.stream(s_in):
                Xd[b].copy_(Xh, non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])      # Y slot b: step i-2's copy-out is done
            sv.linear(p, blobs[i % n_copies], Xd[b], M, Yd[b], ws, stream)
            ev_c[b].record(stream)
            s_out.wait_event(ev_c[b])
            with torch.cuda.stream(s_out):
                Yh[b].copy_(Yd[b], non_blocking=True)
            ev_out[b].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    esteps = 50 if not small else 200
    e2e_pipeline(3)
    barrier()
    e_total = max_over_ranks(e2e_pipeline(esteps), dist, dev)
    e2e_value = flops(M, K, N, r) * world / (e_total / esteps * 1e-3) / 1e12
    assert sv.get_status() == sv.OK

    roofline = gemm_roofline(wl, ms_gemm, ms_act, ms_per_call, measured_peaks(), probed)

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": wl.fmt, "data": "synthetic",
            "config": config_dict(wl, world, small),
            "roofline": roofline, "clocks": clocks,
            "timing": {"passes": passes, "pass_ms_min": min(pass_ms), "pass_ms_median": float(np.median(pass_ms)),
                       "pass_ms_max": max(pass_ms), "calls_per_step": calls_per_step,
                       "ms_per_call": ms_per_call, "weight_copies": n_copies},
            "gpu_launches": 2 * calls_per_step * args.steps * passes,
            "tc_peaks_probed_tflops": probed,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": int(X.numel() * 2),
                    "d2h_bytes_per_step": int(Y.numel() * 2)},
            "frac_of_nominal_fp4": value / NOMINAL_FP4_TFLOPS if wl.fmt == "nvfp4" else None}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, oracle_layer_from_library(wl, X_cal))
    if dist is not None:
        barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
