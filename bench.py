#!/usr/bin/env python
"""Throughput of the RVQ visual-tokenization hot path on B200.

One step = one pass of the whole path over one batch of synthetic native-resolution
patch features, through the C ABI:
    rvq_build_norms (codeword norms + bf16 operand copy)
    rvq_encode      (greedy RVQ: ids and the fp32 final residual)
    rvq_decode      (gather-sum of the produced ids: the reconstruction)
Metric: tokens (feature vectors) per second, in millions.  `value` is measured with the
inputs resident in HBM; `e2e` repeats it through the same calls with the features copied
from pinned host memory every step and the ids + decoded recon copied back.

    python bench.py [--gpus N --steps K --warmup W] [--workload detok] [--impl reference]
The default workload is the largest single-GPU configuration, `detok`: 2^20 tokens x 8 levels of
16384 codewords at D = 1024 (bf16 codebooks), decoded to fp32 features that the step re-encodes
and decodes again.  The encode-only figures of `offline` and `packed` are added to the same line
(--also).
Multi-GPU: launched by torchrun, one rank per GPU; every rank quantizes its own batch
(weak scaling, no data-path collective); times are the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402
from multimodal_visual_tokenization_b200 import sharding  # noqa: E402

METRIC = "RVQ encode Mtokens/s (L levels, K codes, dim D) and % tensor-core peak; decode GB/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 512 << 20          # > 126 MB L2
GEMM_KERNEL_SRC = os.path.join(ROOT, "multimodal_visual_tokenization_b200", "csrc", "rvq_encode.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "encode_traffic.txt")


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default="detok", choices=sorted(workloads.WORKLOADS))
    p.add_argument("--also", default="offline,packed",
                   help="comma-separated workloads whose encode alone is timed in the same run ('none': skip)")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--rows", type=int, default=None, help="smaller N with the same recipe (profiling)")
    p.add_argument("--gemm-events", choices=("timed", "separate"), default="timed",
                   help="bracket distance-GEMM launches with events inside the timed steps, or in a "
                        "separate pass of the same steps")
    return p.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def workload_label(spec):
    return (f"{spec.name}: N={spec.N} D={spec.D} L={spec.L} K={spec.K}, "
            f"{spec.f_dtype} features, {spec.cb_dtype} codebooks; {spec.description}")


def run_config(spec, world):
    """The `config` of both arms' lines: the workload and what one step does to it."""
    return {"workload": workload_label(spec), "N": spec.N, "D": spec.D, "L": spec.L, "K": spec.K,
            "step": "build codeword norms, encode every row through all L levels (ids + residual), "
                    "decode the ids",
            "l2": "flushed between timed steps (GPU arm; the oracle's sample is not L2-resident either)",
            "parallelism": f"replicas x{world}, rows independent, no data-path collective"}


# ------------------------------------------------------------------ clocks during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            time.sleep(0.15)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
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
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        busy = [v for v in sm if v > 0.5 * (mx or 0)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ replica timing

class EventTimer:
    """Per-step CUDA events recorded on the launching stream."""

    def __init__(self, steps, stream):
        import torch
        self.stream = stream
        self.starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        self.ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]

    def start(self, k):
        self.starts[k].record(self.stream)

    def stop(self, k):
        self.ends[k].record(self.stream)

    def total_ms(self):
        self.ends[-1].synchronize()
        return sum(s.elapsed_time(e) for s, e in zip(self.starts, self.ends))


def replica_measure(step, steps, timer, units, between=None, sync=None, device=None):
    """Time `steps` steps of this rank's replica: a barrier and a sync on both sides, `between`
    (the L2 flush) outside each step's timer.  Returns (ms_per_step, value, total_ms): the total
    is the max over ranks, value = the units all ranks processed per step / ms_per_step (units/s)."""
    import torch.distributed as dist
    grouped = dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1
    if sync:
        sync()
    if grouped:
        dist.barrier()
    if sync:
        sync()
    for k in range(steps):
        if between:
            between()
        timer.start(k)
        step()
        timer.stop(k)
    if sync:
        sync()
    if grouped:
        dist.barrier()
    total_ms = sharding.max_over_ranks(timer.total_ms(), device)
    all_units = sharding.sum_over_ranks(float(units), device)
    ms_per_step = total_ms / steps
    return ms_per_step, all_units / (ms_per_step / 1e3), total_ms


# ------------------------------------------------------------------ helpers

def gpu_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [v.strip() for v in vis.split(",") if v.strip()]
    return ids[local_rank] if local_rank < len(ids) else str(local_rank)

def file_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def read_traffic(workload, kernel):
    """ncu DRAM bytes per launch of the dominant encode kernel for this workload, if captured from
    the current kernel source (profiles/encode_traffic.txt lines: workload kernel bytes_per_launch
    source_sha)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    sha = file_sha(GEMM_KERNEL_SRC)
    with open(TRAFFIC_FILE) as f:
        for ln in f:
            parts = ln.split()
            if (len(parts) >= 4 and not ln.startswith("#") and parts[0] == workload and parts[1] == kernel
                    and parts[3] == sha):
                return float(parts[2])
    return None


def cpu_model():
    """The host CPU's model string (logged beside the oracle's figures)."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_rows(g, rows):
    """Feature rows of the workload as the oracle gets them (detok: decoded from the planted ids)."""
    import oracle
    if g["x"] is not None:
        return np.ascontiguousarray(g["x"][rows])
    return oracle.decode(g["planted"][rows], g["codebooks"]).astype(np.float32)


def cpu_baseline(g, seconds, threads=0):
    """The fp64 oracle, as it stands, on a bounded seeded row sample on this host's cores: per row the
    step's work, the greedy encode of all L levels and the decode of the ids it chose.  Rows are
    independent, so the sample's tokens/s is the whole batch's.  threads=0: all cores (OpenMP
    default); the thread setting is restored afterwards."""
    import oracle
    C = g["codebooks"]
    spec = g["spec"]
    default = oracle.threads(0)
    cores = oracle.threads(threads) if threads > 0 else default
    try:
        def run(rows):
            xs = oracle_rows(g, rows)          # input preparation, not timed
            t0 = time.perf_counter()
            ids, _, _, _ = oracle.encode(xs, C)
            oracle.decode(ids, C)
            return time.perf_counter() - t0
        probe = workloads.sample_rows(spec.N, cores, seed=8)
        dt = max(run(probe), 1e-6)
        rows = int(max(cores, min(spec.N, len(probe) * seconds / dt)))
        sample = workloads.sample_rows(spec.N, rows, seed=10)
        dt = run(sample)
    finally:
        oracle.threads(default)
    return {"value": len(sample) / dt / 1e6, "unit": "Mtokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(sample)} of {spec.N} rows (seeded), encode of all levels + decode per row, "
                      f"fp64 plain C + OpenMP over rows, {dt:.2f} s"}


# ------------------------------------------------------------------ reference arm (the oracle)

def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle timed on this host's cores, rank 0 only."""
    if rank != 0:
        return
    g = workloads.generate(args.workload, n_override=args.rows)
    spec = g["spec"]
    per_step = max(0.5, min(args.cpu_seconds, 90.0 / max(1, args.steps + args.warmup)))
    vals = []
    cb = None
    for k in range(args.warmup + args.steps):
        cb = cpu_baseline(g, per_step)
        if k >= args.warmup:
            vals.append(cb["value"])
    cb["cpu_model"] = cpu_model()
    cb["host_cpus"] = os.cpu_count()
    value = statistics.median(vals)
    line = {"metric": METRIC, "value": value, "unit": "Mtokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": spec.N / (value * 1e6) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": run_config(spec, world),
            "note": "fp64 oracle on host cores; each step a bounded seeded row sample; "
                    "ms_per_step extrapolated to the full batch (rows are independent)",
            "cpu_baseline": dict(cb, value=value),
            "e2e": {"value": value, "unit": "Mtokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

def encode_figures(name, dev, peaks, flush_l2, reps=3):
    """rvq_encode alone on another workload (inputs resident, L2 flushed before each timed call):
    time, tokens/s and the distance GEMM's share of the bf16 peaks."""
    import torch

    import multimodal_visual_tokenization_b200 as mvt
    g = workloads.generate(name)
    spec = g["spec"]
    N, D, L, K = spec.N, spec.D, spec.L, spec.K
    cb = torch.from_numpy(g["codebooks"]).to(dev)
    if spec.cb_dtype == "bf16":
        cb = cb.to(torch.bfloat16)
    x = torch.from_numpy(g["x"]).to(dev)
    if spec.f_dtype == "bf16":
        x = x.to(torch.bfloat16)
    tok = mvt.Tokenizer(cb)
    off = torch.from_numpy(g["offsets"]).to(dev)
    fb = torch.zeros(L, dtype=torch.int32, device=dev)
    out = {"ids": torch.empty((N, L), dtype=torch.int32, device=dev)}
    stream = torch.cuda.current_stream(dev)
    for _ in range(2):
        tok.encode(x, offsets=off, out=out, fallbacks=fb)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    for _ in range(reps):
        fb.zero_()
        flush_l2()
        e0.record(stream)
        tok.encode(x, offsets=off, out=out, fallbacks=fb, status=status, check=False)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ts.append(e0.elapsed_time(e1))
    if int(status.item()) != 0:
        raise mvt.RVQError(int(status.item()), f"rvq_encode ({name}, device)")
    ms = statistics.median(ts)
    # the decode of the ids just produced (gather-sum back to fp32 features)
    rec = torch.empty((N, D), dtype=torch.float32, device=dev)
    td = []
    for _ in range(reps):
        flush_l2()
        e0.record(stream)
        tok.decode(out["ids"], out=rec, status=status, check=False)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        td.append(e0.elapsed_time(e1))
    if int(status.item()) != 0:
        raise mvt.RVQError(int(status.item()), f"rvq_decode ({name}, device)")
    dms = statistics.median(td)
    ids_h = out["ids"].cpu().numpy()
    s_cb = 2 if spec.cb_dtype == "bf16" else 4
    rows_used = sum(int(np.unique(ids_h[:, l]).size) for l in range(L))
    dbytes = N * L * 4 + rows_used * D * s_cb + N * D * 4
    hbm = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
    del rec
    tflops = 2.0 * N * K * D * L / (ms / 1e3) / 1e12
    sus = float(peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"]))
    burst = float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
    code, lpl = mvt.rvq_encode_levels_per_launch(N, D, L, K)
    return {"workload": workload_label(spec), "N": N, "D": D, "L": L, "K": K, "encode_ms": ms,
            "Mtok_per_s": N / (ms / 1e3) / 1e6, "tflops": tflops, "frac_sustained": tflops / sus,
            "frac_burst": tflops / burst, "fallbacks_per_level": fb.cpu().tolist(),
            "decode_ms": dms, "decode_algorithmic_bytes": dbytes,
            "decode_frac_hbm": dbytes / (dms / 1e3) / 1e9 / hbm,
            "kernel": "encode_flow_kernel" if lpl > 1 else "dist_topk_kernel per level",
            "timing": f"median of {reps} calls, L2 flushed before each"}


def run_ours(args, rank, world, local_rank):
    import torch

    import multimodal_visual_tokenization_b200 as mvt

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()

    g = workloads.generate(args.workload, batch=rank, n_override=args.rows)
    spec = g["spec"]
    N, D, L, K = spec.N, spec.D, spec.L, spec.K

    def to_dev(a, dt):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.to(torch.bfloat16) if dt == "bf16" else t).to(dev)

    cb = to_dev(g["codebooks"], spec.cb_dtype)
    tok = mvt.Tokenizer(cb)
    detok_only = g["x"] is None
    if detok_only:
        ids_in = torch.from_numpy(g["planted"]).to(dev)
        x = tok.decode(ids_in)                       # fp32 features to re-encode
        x_host_np = None
    else:
        x = to_dev(g["x"], spec.f_dtype)
    f_code = mvt._dtype_code(x)
    ids = torch.empty((N, L), dtype=torch.int32, device=dev)
    res = torch.empty((N, D), dtype=torch.float32, device=dev)
    rec = torch.empty((N, D), dtype=torch.float32, device=dev)
    rec2 = torch.empty((N, D), dtype=torch.float32, device=dev)
    fb = torch.zeros(L, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws, ws_bytes = tok.workspace(N)
    off = torch.from_numpy(g["offsets"]).to(dev)
    B = off.numel() - 1
    stream = torch.cuda.current_stream(dev)

    def check(code, what):
        if code != 0:
            raise mvt.RVQError(code, what)

    def step(xin, dec_ids=None):
        check(mvt.rvq_build_norms(cb, tok.cb_dtype, L, K, D, tok.norms, tok.level_stats, tok.operand, stream),
              "rvq_build_norms")
        check(mvt.rvq_encode(xin, f_code, N, D, cb, tok.cb_dtype, tok.operand, tok.norms, tok.level_stats, L, K,
                             off, B, ids, res, None, fb, ws, ws_bytes, status, stream), "rvq_encode")
        check(mvt.rvq_decode(ids if dec_ids is None else dec_ids, N, L, cb, tok.cb_dtype, K, D, rec2, status,
                             stream), "rvq_decode")

    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush_l2():
        """Write a buffer larger than L2, then read it back: no line of the step's data stays in L2,
        and the flush's own dirty lines are written back here, not during the next timed step."""
        flush.zero_()
        flush.max()

    for _ in range(args.warmup):
        step(x)
    torch.cuda.synchronize(dev)

    # -------------------------------------------------- timed region, device-resident inputs
    timer = EventTimer(args.steps, stream)
    with ClockSampler(gpu_index(local_rank)) as clk:
        in_timed = args.gemm_events == "timed"
        mvt.rvq_profile_enable(in_timed)
        launches0 = mvt.rvq_launch_count()
        ms_per_step, value, total_ms = replica_measure(lambda: step(x), args.steps, timer, N, between=flush_l2,
                                                       sync=lambda: torch.cuda.synchronize(dev), device=dev)
        launches = mvt.rvq_launch_count() - launches0
        if not in_timed:  # the same steps again, GEMM launches bracketed by events
            mvt.rvq_profile_enable(True)
            for k in range(args.steps):
                flush_l2()
                step(x)
            torch.cuda.synchronize(dev)
        code, gemm_n, gemm_ms = mvt.rvq_profile_read()
        mvt.rvq_profile_enable(False)
    st = int(status.item())
    if st != 0:
        raise mvt.RVQError(st, "device status during the timed region")
    value /= 1e6  # tokens/s -> Mtokens/s

    # -------------------------------------------------- per-call breakdown (separate pass)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    br = {"norms": [], "encode": [], "decode": []}
    for _ in range(min(args.steps, 20)):
        flush_l2()
        ev[0].record(stream)
        check(mvt.rvq_build_norms(cb, tok.cb_dtype, L, K, D, tok.norms, tok.level_stats, tok.operand, stream), "")
        ev[1].record(stream)
        check(mvt.rvq_encode(x, f_code, N, D, cb, tok.cb_dtype, tok.operand, tok.norms, tok.level_stats, L, K,
                             off, B, ids, res, None, fb, ws, ws_bytes, status, stream), "")
        ev[2].record(stream)
        check(mvt.rvq_decode(ids, N, L, cb, tok.cb_dtype, K, D, rec2, status, stream), "")
        ev[3].record(stream)
        torch.cuda.synchronize(dev)
        br["norms"].append(ev[0].elapsed_time(ev[1]))
        br["encode"].append(ev[1].elapsed_time(ev[2]))
        br["decode"].append(ev[2].elapsed_time(ev[3]))
    breakdown = {k: statistics.median(v) for k, v in br.items()}
    s_cb = 2 if spec.cb_dtype == "bf16" else 4
    # algorithmic minimum of a decode: ids read once, every referenced codeword row read once, recon
    # written once.  When every codeword is referenced (detok) this is N*L*4 + L*K*D*s + N*D*4; a
    # small batch (image) references only part of the codebooks.
    ids_h = ids.cpu().numpy()
    rows_used = sum(int(np.unique(ids_h[:, l]).size) for l in range(L))
    decode_bytes = N * L * 4 + rows_used * D * s_cb + N * D * 4
    decode_gbs = decode_bytes / (breakdown["decode"] / 1e3) / 1e9

    # -------------------------------------------------- k-means update of level 0 (offline)
    # One Lloyd update of the level-0 codebook from the features and their level-0 ids: the step
    # that fits the fixed tokenizer.  Points are the features widened to fp32 (outside the events).
    kmeans = None
    if args.workload == "offline":
        pts = x.float()
        ids0 = ids[:, 0].contiguous()
        old0 = torch.from_numpy(np.ascontiguousarray(g["codebooks"][0], np.float32)).to(dev)
        new0 = torch.empty_like(old0)
        sums = torch.empty_like(old0)
        cnt = torch.empty(K, dtype=torch.int32, device=dev)
        ev3 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        km = []
        for _ in range(min(args.steps + 2, 6)):
            flush_l2()
            ev3[0].record(stream)
            check(mvt.rvq_codebook_update(pts, ids0, N, D, K, old0, new0, sums, cnt, status, stream),
                  "rvq_codebook_update")
            ev3[1].record(stream)
            torch.cuda.synchronize(dev)
            km.append(ev3[0].elapsed_time(ev3[1]))
        km_ms = statistics.median(km[1:])
        # algorithmic minimum: points and ids read once, old codebook read, new codebook written
        km_bytes = N * D * 4 + N * 4 + 2 * K * D * 4 + K * 4
        kmeans = {"ms": km_ms, "GB_per_s": km_bytes / (km_ms / 1e3) / 1e9, "algorithmic_bytes": km_bytes,
                  "frac_hbm": km_bytes / (km_ms / 1e3) / 1e9 / float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])),
                  "level": 0, "kernels": "embed_backward_kernel (sums, counts) + kmeans_finalize_kernel"}
        del pts, old0, new0, sums, cnt

    # -------------------------------------------------- codebook-sharded encode (image)
    # The codebook axis split in two shards that this one GPU both holds (one process standing in
    # for two ranks, so the exchange of (distance, id) pairs is empty): per level a distance GEMM
    # over each half, the shards' certificates and the apply kernel.  The ids must equal the
    # one-GPU encode's; the GEMM launches are timed with the profiling events.
    sharded = None
    if args.workload == "image" and world == 1:
        from multimodal_visual_tokenization_b200.sharded import ShardedTokenizer
        stok = ShardedTokenizer.local(cb, 2)
        for _ in range(2):
            stok.encode(x, status=status)
        ev5 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        sh = []
        mvt.rvq_profile_enable(True)
        for _ in range(6):
            flush_l2()
            ev5[0].record(stream)
            sids, _, sfb = stok.encode(x, status=status)
            ev5[1].record(stream)
            torch.cuda.synchronize(dev)
            sh.append(ev5[0].elapsed_time(ev5[1]))
        code, sg_n, sg_ms = mvt.rvq_profile_read()
        mvt.rvq_profile_enable(False)
        sh_ms = statistics.median(sh)
        sg_tflops = 6 * 2.0 * N * K * D * L / (sg_ms / 1e3) / 1e12 if sg_ms > 0 else None
        sharded = {"shards": 2, "ms": sh_ms, "Mtok_per_s": N / (sh_ms / 1e3) / 1e6,
                   "ids_equal_one_gpu": bool(torch.equal(sids, ids)),
                   "gemm_tflops": sg_tflops,
                   "gemm_frac": (sg_tflops / float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
                                 if sg_tflops else None),
                   "fallback_rows": int(sfb.sum().item()),
                   "kernels": "dist_topk_kernel per shard + shard_select/fallback + shard_apply",
                   "note": "both shards on one GPU; exchange empty"}
        del stok

    # -------------------------------------------------- packing for data-parallel ranks (packed)
    # The batch's images balanced over 8 ranks by token count (host), then every rank's share
    # gathered from the id cache (the ids just computed) into rank-major packed order (GPU).
    pack = None
    if args.workload == "packed":
        lengths = np.diff(g["offsets"])
        code, owner, pload = mvt.rvq_balance_sequences(lengths, 8)
        check(code, "rvq_balance_sequences")
        select = np.concatenate([np.nonzero(owner == r)[0] for r in range(8)]).astype(np.int64)
        out_off = np.concatenate([[0], np.cumsum(lengths[select])]).astype(np.int64)
        sel_d = torch.from_numpy(select).to(dev)
        oo_d = torch.from_numpy(out_off).to(dev)
        packed_ids = torch.empty_like(ids)
        ev4 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        pk = []
        for _ in range(6):
            flush_l2()
            ev4[0].record(stream)
            check(mvt.rvq_gather_sequences(ids, L, off, B, sel_d, B, oo_d, packed_ids, status, stream),
                  "rvq_gather_sequences")
            ev4[1].record(stream)
            torch.cuda.synchronize(dev)
            pk.append(ev4[0].elapsed_time(ev4[1]))
        pk_ms = statistics.median(pk[1:])
        pk_bytes = 2 * N * L * 4 + B * 8 * 3
        pack = {"ms": pk_ms, "GB_per_s": pk_bytes / (pk_ms / 1e3) / 1e9, "algorithmic_bytes": pk_bytes,
                "frac_hbm": pk_bytes / (pk_ms / 1e3) / 1e9 / float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])),
                "world": 8, "images": int(B), "max_over_mean_rank_tokens": float(pload.max() / pload.mean()),
                "kernel": "gather_sequences_kernel"}
        del packed_ids

    # -------------------------------------------------- embedding backward (detok ids)
    # The backbone's visual-token embedding e[n] = sum_l E_l[ids[n,l]] is the decode gather-sum
    # with learned tables; its table gradient is the scatter-add grad[l, ids[n,l]] += g[n].  On
    # the detok ids (level 0 Zipf-skewed) the decoded fp32 recon serves as a synthetic g [N,D],
    # accumulated into fp32 tables [L,K,D] zeroed before each launch (outside the events).
    embed = None
    if detok_only:
        gtab = torch.zeros((L, K, D), dtype=torch.float32, device=dev)
        code, eb_ws_bytes = mvt.rvq_embed_backward_workspace_size(N, L, K, D)
        check(code, "rvq_embed_backward_workspace_size")
        eb_ws = torch.empty(eb_ws_bytes, dtype=torch.uint8, device=dev)
        ev2 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

        def time_backward(call):
            t = []
            for _ in range(min(args.steps + 2, 6)):
                gtab.zero_()
                flush_l2()
                ev2[0].record(stream)
                call()
                ev2[1].record(stream)
                torch.cuda.synchronize(dev)
                t.append(ev2[0].elapsed_time(ev2[1]))
            return statistics.median(t[1:]) if len(t) > 1 else t[0]

        det_ms = time_backward(lambda: check(mvt.rvq_embed_backward_sorted(
            ids_in, N, L, K, D, rec2, gtab, eb_ws, eb_ws_bytes, status, stream), "rvq_embed_backward_sorted"))
        at_ms = time_backward(lambda: check(mvt.rvq_embed_backward(ids_in, N, L, K, D, rec2, gtab, status, stream),
                                            "rvq_embed_backward"))
        # algorithmic minimum: ids and g read once, every referenced gradient row read and written once
        used = sum(int(np.unique(g["planted"][:, l]).size) for l in range(L))
        eb_bytes = N * L * 4 + N * D * 4 + 2 * used * D * 4
        # what the sorted kernel has to move: every g row once per level (the rows a level visits are in
        # id order, so L2 cannot keep them between levels), the gradient rows read and written once
        moved = N * L * D * 4 + 2 * used * D * 4 + 3 * N * L * 4
        hbm = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
        embed = {"ms": det_ms, "GB_per_s": eb_bytes / (det_ms / 1e3) / 1e9, "algorithmic_bytes": eb_bytes,
                 "frac_hbm": eb_bytes / (det_ms / 1e3) / 1e9 / hbm,
                 "bytes_moved": moved, "frac_hbm_of_moved": moved / (det_ms / 1e3) / 1e9 / hbm,
                 "kernels": "ss_hist/ss_prefix/ss_scan/ss_scatter (stable sort by id) + ss_rowsum + ss_fix "
                            "(deterministic)",
                 "atomic_ms": at_ms, "atomic_kernel": "embed_backward_kernel (fp32x4 atomics)",
                 "atomic_frac_hbm": eb_bytes / (at_ms / 1e3) / 1e9 / hbm,
                 "g": "decoded fp32 recon [N,D]"}
        del gtab, eb_ws

    # -------------------------------------------------- end to end through host buffers
    # Every step copies its features from pinned host memory and its ids + decoded recon back.
    # Two buffer sets and separate copy/compute streams let step k's copies overlap the compute of
    # its neighbours, as a pipeline tokenizing a stream of images would run.
    e2e = None
    if not args.no_e2e:
        copy_in = torch.cuda.Stream(dev)
        copy_out = torch.cuda.Stream(dev)
        if detok_only:
            h_in = [torch.from_numpy(g["planted"]).pin_memory() for _ in range(2)]
            d_in = [torch.empty_like(ids) for _ in range(2)]
        else:
            src = torch.from_numpy(g["x"]).to(torch.bfloat16) if spec.f_dtype == "bf16" else torch.from_numpy(g["x"])
            h_in = [src.pin_memory() for _ in range(2)]
            d_in = [torch.empty_like(x) for _ in range(2)]
        d_ids = [torch.empty_like(ids) for _ in range(2)]
        d_rec = [torch.empty_like(rec2) for _ in range(2)]
        d_x = [torch.empty_like(x) for _ in range(2)] if detok_only else None
        h_ids = [torch.empty((N, L), dtype=torch.int32).pin_memory() for _ in range(2)]
        h_rec = [torch.empty((N, D), dtype=torch.float32).pin_memory() for _ in range(2)]
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def pipe_step(k):
            b = k % 2
            with torch.cuda.stream(copy_in):
                if k >= 2:
                    copy_in.wait_event(ev_done[b])       # the compute of step k-2 is done with d_in[b]
                d_in[b].copy_(h_in[b], non_blocking=True)
                ev_in[b].record(copy_in)
            stream.wait_event(ev_in[b])
            if k >= 2:
                stream.wait_event(ev_out[b])             # step k-2's results have left d_ids/d_rec[b]
            if detok_only:
                xin = tok.decode(d_in[b], out=d_x[b], check=False)
            else:
                xin = d_in[b]
            check(mvt.rvq_build_norms(cb, tok.cb_dtype, L, K, D, tok.norms, tok.level_stats, tok.operand, stream),
                  "rvq_build_norms")
            check(mvt.rvq_encode(xin, f_code, N, D, cb, tok.cb_dtype, tok.operand, tok.norms, tok.level_stats, L,
                                 K, off, B, d_ids[b], res, None, fb, ws, ws_bytes, status, stream), "rvq_encode")
            check(mvt.rvq_decode(d_ids[b], N, L, cb, tok.cb_dtype, K, D, d_rec[b], status, stream), "rvq_decode")
            ev_done[b].record(stream)
            with torch.cuda.stream(copy_out):
                copy_out.wait_event(ev_done[b])
                h_ids[b].copy_(d_ids[b], non_blocking=True)
                h_rec[b].copy_(d_rec[b], non_blocking=True)
                ev_out[b].record(copy_out)

        for k in range(2):
            pipe_step(k)
        torch.cuda.synchronize(dev)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(copy_in)
        for k in range(args.steps):
            pipe_step(k)
        copy_out.wait_event(ev_out[(args.steps - 1) % 2])
        t1.record(copy_out)
        torch.cuda.synchronize(dev)
        e_ms = sharding.max_over_ranks(t0.elapsed_time(t1), dev)
        h2d = h_in[0].numel() * h_in[0].element_size()
        d2h = h_ids[0].numel() * 4 + h_rec[0].numel() * 4
        e2e = {"value": N * world / (e_ms / args.steps / 1e3) / 1e6, "unit": "Mtokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e_ms / args.steps,
               "pipeline": "2 buffer sets; copy-in, compute and copy-out streams overlap across steps"}

    # -------------------------------------------------- roofline of the distance GEMM
    # a step longer than 20 ms runs under the power cap: the sustained bf16 figure is its peak; the
    # fraction of the burst figure is reported beside it
    long_step = ms_per_step > 20.0
    peak_key = "bf16_tflops_sustained" if long_step else "bf16_tflops"
    peak = float(peaks.get(peak_key, PEAKS_FALLBACK[peak_key]))
    peak_burst = float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
    # the dominant encode kernel: one launch per level (distance GEMM + top-8), or one launch for
    # all levels (dataflow kernel: GEMM, top-8, certificate and residual update)
    code, lpl = mvt.rvq_encode_levels_per_launch(N, D, L, K)
    check(code, "levels per launch")
    kernel = "encode_flow_kernel" if lpl > 1 else "dist_topk_kernel"
    flops_per_launch = 2.0 * N * K * D * lpl  # every (row, codeword) dot product of the levels covered
    enc_launches = max(1, gemm_n // lpl)
    launch_ms = gemm_ms / enc_launches
    achieved = flops_per_launch / (launch_ms / 1e3) / 1e12
    traffic = read_traffic(args.workload, kernel)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic,
                "frac_burst": achieved / peak_burst, "peak_burst": peak_burst,
                "kernel": kernel, "levels_per_launch": lpl, "launch_ms": launch_ms,
                "launches_timed": enc_launches, "flops_per_launch": flops_per_launch,
                "peak_source": f"{peak_src} {peak_key}"}

    # -------------------------------------------------- quick parity sample + CPU baseline
    parity = None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        rows = workloads.sample_rows(N, 6, seed=11)
        xs = x[torch.from_numpy(rows).to(dev)].float().cpu().numpy()   # the rows the GPU encoded
        want, _, _, _ = oracle.encode(xs, g["codebooks"])
        got = ids.cpu().numpy()[rows]
        parity = {"rows": int(len(rows)), "ids_equal_oracle": bool(np.array_equal(want, got))}
        cpu = cpu_baseline(g, args.cpu_seconds)
        one = cpu_baseline(g, min(args.cpu_seconds, 8.0), threads=1)
        cpu.update({"value_1thread": one["value"], "sample_1thread": one["sample"], "cpu_model": cpu_model(),
                    "host_cpus": os.cpu_count()})

    also = {}
    if world == 1 and args.also != "none" and args.rows is None:
        for name in [w for w in args.also.split(",") if w and w != args.workload]:
            also[name] = encode_figures(name, dev, peaks, flush_l2)

    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "Mtokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": run_config(spec, world),
        "calls": "rvq_build_norms + rvq_encode(ids, residual) + rvq_decode(ids -> recon); L2 flush = 512 MiB "
                 "memset + read-back outside the step events",
        "gemm_events": args.gemm_events,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
        "breakdown_ms": breakdown,
        "decode": {"GB_per_s": decode_gbs, "algorithmic_bytes": decode_bytes,
                   "frac_hbm": decode_gbs / float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))},
        **({"embed_backward": embed} if embed is not None else {}),
        **({"pack": pack} if pack is not None else {}),
        **({"sharded": sharded} if sharded is not None else {}),
        **({"codebook_update": kmeans} if kmeans is not None else {}),
        **({"encode_other_workloads": also} if also else {}),
        "fallbacks_per_level": fb.cpu().tolist(),
        "parity_sample": parity,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if world != args.gpus and "RANK" in os.environ:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if world > 1 and args.impl == "ours":
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
