#!/usr/bin/env python
"""Benchmark of the NVFP4 W4A4 linear layer on B200.

Primary line (the decode-shaped workload): one step = the fused gate+up layer
(K=5120, N=34816 as two modules with their own weight global scales) called
once each for M = 1, 8 and 32 tokens, the whole path per call (dynamic
activation amax, quantize, block-scaled FP4 GEMM, per-segment epilogue, bf16
out).  value = algorithmic HBM bytes of the step / device time (GB/s).  Every
call reads a different copy of the packed weights (copies rotate over >= 4x
the 126 MB L2), so each call streams its weights from HBM.

The same JSON line carries the dominant kernel's roofline (the GEMM, timed
alone with CUDA events on its stream), the end-to-end number through host
buffers, the clocks seen during the timed region, the CPU oracle as a
baseline, and the other workloads (prefill TFLOP/s, standalone quantize GB/s)
under "workloads".

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl nvfp4|reference]
Under torchrun each rank runs its own replica of the step on its own GPU
(independent batches, no data-path collective: weak scaling).
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

METRIC = "NVFP4 linear TFLOP/s (prefill) & GB/s (decode, quantize) as % of B200 roofline"
L2_BYTES = 126 * 2 ** 20
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP4_OVER_BF16 = 4.0          # nominal dense ratio 9 PFLOP/s fp4 : 2.25 PFLOP/s bf16


# ----------------------------------------------------------------------------- peaks / clocks

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=FALLBACK_HBM_GBS, bf16_tflops=FALLBACK_BF16_TFLOPS,
                    bf16_tflops_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi sampled every 50 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def _target(self):
        import torch
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            return vis.split(",")[self.dev] if vis else str(self.dev)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self._target(), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.reader.join(timeout=2)
        sm, mx, reasons = [], None, set()
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
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- helpers

def gen_device(shape, dist, seed, outlier_frac=0.0, outlier_mult=1.0, sigma=1.0):
    """Seeded synthetic bf16 tensor generated on the GPU (Philox), with the
    workloads' distributions: N(0, sigma) or Student-t nu=3, plus scaled
    outlier channels."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    if dist == "normal":
        x = torch.randn(shape, generator=g, device="cuda", dtype=torch.float32) * sigma
    else:  # Student-t, nu = 3: z / sqrt(chi2_3 / 3)
        z = torch.randn(shape, generator=g, device="cuda", dtype=torch.float32)
        c = torch.zeros(shape, device="cuda", dtype=torch.float32)
        for _ in range(3):
            c.add_(torch.randn(shape, generator=g, device="cuda", dtype=torch.float32).square_())
        x = z / torch.sqrt(c / 3.0)
        del z, c
    if outlier_frac > 0:
        k = shape[1]
        n_out = max(1, int(round(outlier_frac * k)))
        cols = torch.randperm(k, generator=g, device="cuda")[:n_out]
        x[:, cols] *= outlier_mult
    return x.to(torch.bfloat16)


def flush_l2(buf, clean=None, sink=None):
    """Evicts the timed call's inputs from L2: writes `buf` (larger than L2), then,
    when `clean` is given, reads that second buffer (also larger than L2) so that
    the lines left in L2 are clean ones and the timed call does not pay for
    writing the first buffer back to HBM."""
    buf.add_(1)
    if clean is not None:
        import torch
        torch.sum(clean, dim=0, out=sink)


def time_reps(fn, reps, warmup, flush=None):
    """Per-rep CUDA-event times (ms) on the current stream, L2 flushed before each rep."""
    import torch
    for _ in range(warmup):
        if flush is not None:
            flush()
        fn()
    torch.cuda.synchronize()
    out = []
    s = torch.cuda.current_stream()
    for _ in range(reps):
        if flush is not None:
            flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        fn()
        e1.record(s)
        out.append((e0, e1))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in out]


def capture_graph(fn):
    """Capture fn() (a sequence of library calls on the current stream) into a
    CUDA graph so that replays carry no host launch overhead."""
    import torch
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()                                 # warm: first-call set-up happens outside capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_graph(g, reps, per_replay):
    """Average device time (ms) of one unit when a graph holding per_replay units
    is replayed back to back `reps` times."""
    import torch
    g.replay()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(reps):
        g.replay()
    e1.record(s)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / (reps * per_replay)


def code_only(text: str) -> str:
    """C++ source with its comments and blank space removed: what the compiler
    sees, so that editing a comment does not change a kernel's hash."""
    import re
    out, i, n = [], 0, len(text)
    while i < n:
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif text[i] == '"':                     # string literal (PTX text): kept as written
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(text[i])
            i += 1
    return re.sub(r"\s+", " ", "".join(out)).strip()


def kernel_source_hash(files):
    """Hash of a kernel's own source files (under the package's csrc/), comments
    and blank space excluded."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nvfp4_w4a4_block_b200", "csrc")
    for name in files:
        h.update(code_only(open(os.path.join(csrc, name)).read()).encode())
    return h.hexdigest()[:16]


DECODE_KERNEL_FILES = ("gemm_decode.cuh", "sm100_ptx.cuh")


def committed_traffic(summary: str, files):
    """DRAM bytes per launch recorded in a committed ncu summary under profiles/
    (its 'dram bytes per launch' and 'kernel source hash' lines), if that capture
    was taken on the kernel's current sources; else None."""
    import re
    try:
        text = open(os.path.join(ROOT, "profiles", summary)).read()
        b = re.search(r"dram bytes per launch:\s*([0-9]+)", text)
        hsh = re.search(r"kernel source hash:\s*([0-9a-f]+)", text)
        if not b or not hsh or hsh.group(1) != kernel_source_hash(files):
            return None
        return int(b.group(1))
    except Exception:
        return None


# ----------------------------------------------------------------------------- ranks

def max_over_ranks(x: float, device="cpu") -> float:
    """The largest value of x over all ranks of the default process group (x
    itself without one).  Every rank must call it, in the same order."""
    import torch
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, step_bytes: int, steps: int, ms_max: float) -> float:
    """Aggregate throughput of `world` replicas that each moved step_bytes per
    step for `steps` steps, over the slowest rank's time."""
    return world * step_bytes * steps / (ms_max * 1e-3) / 1e9


# ----------------------------------------------------------------------------- workload bytes

def decode_call_bytes(m, n, k, dynamic=True, gemm_only=False):
    """Algorithmic HBM bytes of one decode-shaped call: packed weights (codes
    N*K/2 + scales N*K/16), activations in (bf16, read twice in dynamic mode:
    amax and encode), activation codes+scales written and read back
    (0.5625 B/elem each way), bf16 output."""
    w = n * k // 2 + n * k // 16
    act_q = m * k // 2 + m * k // 16
    y = 2 * m * n
    if gemm_only:
        return w + act_q + y
    x = 2 * m * k * (2 if dynamic else 1)
    return w + x + 2 * act_q + y


# ----------------------------------------------------------------------------- nvfp4 arm

def run_nvfp4(args, rank, world, local_rank):
    import numpy as np
    import torch

    import nvfp4_w4a4_block_b200 as nv
    from nvfp4_w4a4_block_b200 import workloads as W

    torch.cuda.set_device(local_rank)
    nv.lib()
    peaks = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    wl = W.DECODE
    n, k, off = wl.n, wl.k, wl.seg_offsets
    ms = list(W.DECODE_M)
    mmax = max(ms)

    # Packed weights: one pack, replicated into enough copies to defeat the L2.
    w = gen_device((n, k), "normal", 1000 + rank, sigma=0.02)
    w[off[1]:] *= 2.75                                       # second module: distinct global scale
    pw0 = nv.pack_weight(w, off)
    del w
    wbytes = pw0.q.numel() + pw0.sf.numel()
    copies = max(4, int(np.ceil(4 * L2_BYTES / wbytes)))
    pws = [pw0] + [nv.PackedWeight(pw0.q.clone(), pw0.sf.clone(), pw0.gscale.clone(), pw0.n, pw0.k, pw0.seg_offsets)
                   for _ in range(copies - 1)]
    x_full = gen_device((mmax, k), "normal", 2000 + rank, wl.outlier_frac, wl.outlier_mult)
    xs = {m: x_full[:m].contiguous() for m in ms}
    ys = {m: torch.empty((m, n), dtype=torch.bfloat16, device="cuda") for m in ms}
    wss = {m: torch.empty(nv.workspace_bytes(m, n, k), dtype=torch.uint8, device="cuda") for m in ms}
    torch.cuda.synchronize()

    # One step = the three calls; call j of the run reads weight copy j % copies.
    # Steps are replayed from CUDA graphs (one per rotation offset), so the timed
    # region measures device work, not Python launch overhead.
    def make_step(first_copy):
        def step():
            for j, m in enumerate(ms):
                nv.linear_fused(xs[m], pws[(first_copy + j) % copies], out=ys[m], ws=wss[m])
        return step

    n_rot = copies // np.gcd(copies, len(ms))
    graphs = []
    for r in range(n_rot):
        before = nv.launch_count()
        graphs.append(capture_graph(make_step((r * len(ms)) % copies)))
        # capture_graph runs the step once eagerly (warm-up) and once under capture
        launches_per_step = (nv.launch_count() - before) // 2

    def step_i(i):
        graphs[i % n_rot].replay()

    step_bytes = sum(decode_call_bytes(m, n, k) for m in ms)

    for i in range(args.warmup):
        step_i(i)
    torch.cuda.synchronize()
    if nv.get_device_error() != nv.OK:
        raise RuntimeError("device error during warm-up")

    # ---- timed region: exactly K steps
    sampler = ClockSampler(local_rank)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.15)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for i in range(args.steps):
        step_i(i)
    e1.record(s)
    # The same step keeps running (untimed) for >= 0.6 s so that the clock
    # sampler sees the load even when the timed region is short.
    t_soak = time.perf_counter()
    i = 0
    while time.perf_counter() - t_soak < 0.6:
        for _ in range(50):
            step_i(i)
            i += 1
        torch.cuda.synchronize()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if clocks is not None:
        clocks["window"] = "timed region + 0.6 s continuation of the same step"
    if world > 1:
        torch.distributed.barrier()
    ms_total = e0.elapsed_time(e1)
    if nv.get_device_error() != nv.OK:
        raise RuntimeError("device error in the timed region")
    ms_max = max_over_ranks(ms_total, "cuda")
    ms_per_step = ms_max / args.steps
    value = whole_job_gbs(world, step_bytes, args.steps, ms_max)
    del graphs

    # ---- dominant kernel: the GEMM alone, per M.  A graph holds `copies` launches
    # (one per weight copy, so every launch streams from HBM); events on the
    # replaying stream bracket many replays.
    per_m = {}
    for m in ms:
        qx, sfx, sx = nv.quantize_act(xs[m])
        ym = ys[m]

        def gemms():
            # The packed weights are static here (packed once before the run), so
            # each GEMM may request its first weight stages while the previous
            # one finishes (NVFP4_FLAG_STATIC_WEIGHTS).
            for c in range(copies):
                nv.gemm(qx, sfx, sx, m, pws[c], out=ym, flags=nv.FLAG_STATIC_WEIGHTS)

        def gemms_plain():
            for c in range(copies):
                nv.gemm(qx, sfx, sx, m, pws[c], out=ym)

        def calls():
            for c in range(copies):
                nv.linear_fused(xs[m], pws[c], out=ym, ws=wss[m])

        static = sx.clone()                 # a calibrated (static) activation scale

        def calls_static():
            for c in range(copies):
                nv.linear_fused(xs[m], pws[c], act_gscale=static, out=ym, ws=wss[m])

        before = nv.launch_count()
        gc = capture_graph(calls)
        call_launches = (nv.launch_count() - before) // (2 * copies)
        gg, gp, gs = capture_graph(gemms), capture_graph(gemms_plain), capture_graph(calls_static)
        tg = time_graph(gg, 20, copies)
        tp = time_graph(gp, 20, copies)
        tf = time_graph(gc, 20, copies)
        ts = time_graph(gs, 20, copies)
        del gg, gp, gc, gs
        gb = decode_call_bytes(m, n, k, gemm_only=True)
        fb = decode_call_bytes(m, n, k)
        per_m[str(m)] = dict(gemm_us=round(tg * 1e3, 3), gemm_gbs=round(gb / (tg * 1e-3) / 1e9, 1),
                             gemm_no_static_flag_us=round(tp * 1e3, 3),
                             gemm_no_static_flag_gbs=round(gb / (tp * 1e-3) / 1e9, 1),
                             call_us=round(tf * 1e3, 3), call_gbs=round(fb / (tf * 1e-3) / 1e9, 1),
                             call_static_scale_us=round(ts * 1e3, 3),
                             call_launches=call_launches,
                             gemm_bytes=gb, call_bytes=fb)
    gm = per_m[str(mmax)]
    roofline = dict(bound="hbm", kernel="nvfp4_gemm_decode_kernel", workload=f"decode M={mmax}",
                    launches="nvfp4_gemm back to back over rotating weight copies, NVFP4_FLAG_STATIC_WEIGHTS "
                             "(weights packed once; see workloads.decode_per_m for the launches without it)",
                    achieved=round(gm["gemm_gbs"], 1), peak=peaks["hbm_gbs"], unit="GB/s",
                    frac=round(gm["gemm_gbs"] / peaks["hbm_gbs"], 4),
                    traffic=committed_traffic(f"nvfp4_gemm_decode_kernel_m{mmax}.md", DECODE_KERNEL_FILES),
                    algorithmic_bytes_per_launch=gm["gemm_bytes"], peak_source=peaks["source"])

    # ---- end to end through host buffers (pinned), H2D of X and D2H of Y inside the region
    # Steps are pipelined as a serving loop over independent batches runs them: the
    # inputs of step s go up on s_in (one copy for its three calls) and its results
    # come back on s_out (one copy) while later steps compute.  Device and pinned
    # host buffers alternate between two sets, and a set is refilled only after the
    # copies that read it have completed, so every step's inputs and results really
    # cross PCIe inside the timed region.
    E2E_STEPS = 8                         # steps per captured graph (one pipeline fill and drain each)
    order = sorted(ms, reverse=True)
    rows_at, r0 = {}, 0
    for m in order:                       # the step's inputs (and results) as one block of rows
        rows_at[m] = r0
        r0 += m
    hx = torch.cat([xs[m] for m in order]).cpu().pin_memory()
    hy = [torch.empty((r0, n), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    dx = [torch.empty((r0, k), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    dy = [torch.empty((r0, n), dtype=torch.bfloat16, device="cuda") for _ in range(2)]

    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_steps(first_copy):
        cur = torch.cuda.current_stream()
        start = torch.cuda.Event()
        start.record(cur)
        s_in.wait_event(start)
        s_out.wait_event(start)
        computed, read_back = [], []      # per step: its calls done / its results read back
        for st in range(E2E_STEPS):
            b = st % 2
            if st >= 2:
                s_in.wait_event(computed[st - 2])   # set b's inputs were consumed two steps ago
                cur.wait_event(read_back[st - 2])   # and its results were read back
            with torch.cuda.stream(s_in):
                dx[b].copy_(hx, non_blocking=True)  # the step's three inputs, one copy
            landed = torch.cuda.Event()
            landed.record(s_in)
            cur.wait_event(landed)
            for j, m in enumerate(order):
                pw = pws[(first_copy + st * len(ms) + j) % copies]
                a = rows_at[m]
                nv.linear_fused(dx[b][a:a + m], pw, out=dy[b][a:a + m], ws=wss[m])
            ev_c = torch.cuda.Event()
            ev_c.record(cur)
            s_out.wait_event(ev_c)
            with torch.cuda.stream(s_out):
                hy[b].copy_(dy[b], non_blocking=True)   # the step's three results, one copy
            ev_r = torch.cuda.Event()
            ev_r.record(s_out)
            computed.append(ev_c)
            read_back.append(ev_r)
        cur.wait_event(read_back[-1])

    # Replayed from CUDA graphs; two graphs alternate over different weight copies
    # so that consecutive calls do not share weights.
    e2e_graphs = [capture_graph(lambda c=c: e2e_steps(c)) for c in (0, len(ms) * E2E_STEPS)]
    flip = [0]

    def e2e_replay():
        e2e_graphs[flip[0] % 2].replay()
        flip[0] += 1

    reps = max(3, min(args.steps, 200) // E2E_STEPS)
    te = time_reps(e2e_replay, reps, 3)
    del e2e_graphs
    e2e_ms = statistics.median(te) / E2E_STEPS
    h2d = sum(xs[m].numel() * 2 for m in ms)
    d2h = sum(m * n * 2 for m in ms)
    e2e = dict(value=round(step_bytes / (e2e_ms * 1e-3) / 1e9, 1), unit="GB/s", h2d_bytes_per_step=h2d,
               d2h_bytes_per_step=d2h, ms_per_step=round(e2e_ms, 4),
               pipelining=f"{E2E_STEPS} steps per graph, one H2D and one D2H copy per step, double-buffered; "
                          "each step's copies overlap other steps' calls")

    del pws, pw0
    torch.cuda.empty_cache()
    workloads = {}
    if rank == 0 and not args.skip_secondary:
        workloads = secondary_workloads(nv, W, peaks, fp4_peak, local_rank)
    workloads["decode_per_m"] = per_m

    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3 block16, fp32 accumulate, bf16 out)",
        "data": "synthetic (seeded Philox on device: X ~ N(0,1) with 0.5% outlier channels x50, "
                "W ~ N(0,0.02) / N(0,0.055) per module)",
        "config": {"workload": "decode-shaped fused gate+up: M in {1,8,32} tokens (one call each per step), "
                               "K=5120, N=34816 = 2 x 17408 modules with distinct weight global scales, "
                               "dynamic activation scale",
                   "l2": f"inputs larger than L2: packed weights rotate over {copies} copies "
                         f"({copies * wbytes / 2**20:.0f} MiB), a different copy per call",
                   "parallelism": f"replicas x{world} (one independent step per GPU)"},
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "timing": "timed steps replayed from CUDA graphs (device time, CUDA events on the replay stream)",
        "clocks": clocks,
        "peaks": {"hbm_gbs": peaks["hbm_gbs"],
                  "fp4_tflops_measured": workloads.get("fp4_peak", {}).get("measured_tflops"),
                  "fp4_measured_source": "workloads.fp4_peak (own MMA-only probe, library GEMM at 16384^3)",
                  "fp4_tflops_proxy": round(fp4_peak, 1),
                  "fp4_proxy_source": f"{peaks['source']} bf16 {peaks['bf16_tflops']} TFLOP/s x {FP4_OVER_BF16} "
                                      f"(nominal dense fp4:bf16 ratio)"},
        "workloads": workloads,
    }
    return line


def secondary_workloads(nv, W, peaks, fp4_peak, device_index=0):
    """The standalone quantize and the conversions (GB/s vs HBM), then the
    prefill-shaped GEMMs and calls (TFLOP/s vs the dense FP4 peak), each rep
    timed alone with the L2 flushed before it.  The HBM-bound, partly
    issue-bound kernels are timed first, before the GEMMs have brought the part
    to its power cap; the SM clocks seen in each phase are reported."""
    import torch
    out = {}
    flush_buf = torch.empty(256 * 2 ** 20 // 4, dtype=torch.float32, device="cuda")
    clean_buf = torch.ones(256 * 2 ** 20 // 4, dtype=torch.float32, device="cuda")
    sink = torch.empty((), dtype=torch.float32, device="cuda")

    def flush():
        flush_l2(flush_buf, clean_buf, sink)

    sampler = ClockSampler(device_index)
    sampler.start()
    out.update(conversion_workloads(nv, W, peaks, flush))

    # standalone activation quantize on the long-prefill tensor (HBM-bound)
    wl = W.LONG_DOWN
    m, k = wl.m, wl.k
    x = gen_device((m, k), "normal", 77, wl.outlier_frac, wl.outlier_mult)
    q = torch.empty((m, k // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty(nv.sf_bytes(m, k), dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    td = statistics.median(time_reps(lambda: nv.quantize_act(x, q=q, sf=sf, gscale_out=s), 10, 3, flush))
    static = s.clone()
    ts = statistics.median(time_reps(lambda: nv.quantize_act(x, gscale=static, q=q, sf=sf, gscale_out=s), 10, 3,
                                     flush))
    elems = m * k
    b_static = elems * (2 + 0.5 + 1 / 16)
    b_dyn = elems * (4 + 0.5 + 1 / 16)
    out["quantize_32768x17408"] = dict(
        dynamic_ms=round(td, 4), dynamic_gbs=round(b_dyn / (td * 1e-3) / 1e9, 1),
        dynamic_frac_hbm=round(b_dyn / (td * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
        static_ms=round(ts, 4), static_gbs=round(b_static / (ts * 1e-3) / 1e9, 1),
        static_frac_hbm=round(b_static / (ts * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
        bytes_dynamic=int(b_dyn), bytes_static=int(b_static))
    del x, q, sf
    torch.cuda.empty_cache()
    out["clocks_hbm_phase"] = sampler.stop()

    sampler = ClockSampler(device_index)
    sampler.start()
    for wl in (W.PREFILL, W.FUSED_QKVG, W.LONG_DOWN):
        m, n, k, off = wl.m, wl.n, wl.k, wl.seg_offsets
        sig = torch.tensor(wl.seg_sigma, dtype=torch.float32)
        w = gen_device((n, k), "normal", 31 + wl.cfg_id)
        for i in range(len(off) - 1):
            w[off[i]:off[i + 1]] *= float(sig[i])
        pw = nv.pack_weight(w, off)
        x = gen_device((m, k), wl.x_dist, 41 + wl.cfg_id, wl.outlier_frac, wl.outlier_mult)
        y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(nv.workspace_bytes(m, n, k), dtype=torch.uint8, device="cuda")
        qx, sfx, sx = nv.quantize_act(x)
        static = sx.clone()                     # a calibrated (static) activation scale
        reps = 10 if wl is not W.LONG_DOWN else 6
        tf = statistics.median(time_reps(lambda: nv.linear_fused(x, pw, out=y, ws=ws), reps, 3, flush))
        ts = statistics.median(time_reps(lambda: nv.linear_fused(x, pw, act_gscale=static, out=y, ws=ws), reps, 3,
                                         flush))
        tg = statistics.median(time_reps(lambda: nv.gemm(qx, sfx, sx, m, pw, out=y), reps, 3, flush))
        fl = 2.0 * m * n * k
        tl = library_nvfp4_ms(m, n, k, reps, flush)
        wb = w.to(torch.bfloat16)
        tb = statistics.median(time_reps(lambda: torch.matmul(x, wb.t()), reps, 2, flush))
        out[wl.name] = dict(
            call_ms=round(tf, 4), call_tflops=round(fl / (tf * 1e-3) / 1e12, 1),
            call_static_scale_ms=round(ts, 4), call_static_scale_tflops=round(fl / (ts * 1e-3) / 1e12, 1),
            gemm_ms=round(tg, 4), gemm_tflops=round(fl / (tg * 1e-3) / 1e12, 1),
            library_nvfp4_gemm_ms=None if tl is None else round(tl, 4),
            library_nvfp4_gemm_tflops=None if tl is None else round(fl / (tl * 1e-3) / 1e12, 1),
            bf16_matmul_ms=round(tb, 4), speedup_over_bf16_call=round(tb / tf, 3), segments=len(off) - 1)
        del w, wb, pw, x, y, ws, qx, sfx
        torch.cuda.empty_cache()
    out["clocks_prefill_phase"] = sampler.stop()

    # The dense FP4 peak, measured after the GEMMs (which ran first, alone, as a
    # user's call would): the library's NVFP4 GEMM at 16384^3 for context, then
    # this repository's tensor-core probe, short (burst) and for >= 1 s (sustained).
    tl = library_nvfp4_ms(16384, 16384, 16384, 5, flush)
    lib_tflops = None if tl is None else 2.0 * 16384 ** 3 / (tl * 1e-3) / 1e12
    probe = fp4_peak_probe(nv, device_index)
    measured = max(v for v in (probe["burst_tflops"], lib_tflops) if v is not None)
    out["fp4_peak"] = dict(probe, library_nvfp4_16384_cubed_tflops=None if lib_tflops is None else round(lib_tflops, 1),
                           measured_tflops=round(measured, 1),
                           measured_source="max of the repository's MMA-only burst probe and the library NVFP4 "
                                           "GEMM at 16384^3",
                           proxy_tflops=round(fp4_peak, 1),
                           proxy_source="measured bf16 burst x 4 (nominal dense fp4:bf16 ratio)")
    for wl in (W.PREFILL, W.FUSED_QKVG, W.LONG_DOWN):
        e = out[wl.name]
        for key in ("gemm", "call", "call_static_scale"):
            e[f"{key}_frac_fp4_peak"] = round(e[f"{key}_tflops"] / measured, 4)
            e[f"{key}_frac_fp4_proxy"] = round(e[f"{key}_tflops"] / fp4_peak, 4)
    out["l2"] = ("each rep timed alone after an L2 flush: 256 MiB written, then another 256 MiB read, "
                 "so every input is cold in HBM and L2 holds only clean lines")
    del flush_buf, clean_buf
    torch.cuda.empty_cache()
    return out


def library_nvfp4_ms(m, n, k, reps, flush):
    """Context only: the median time (ms) of the library's NVFP4 GEMM (torch's
    scaled_mm on cuBLASLt: E2M1 operands, 16-element E4M3 block scales, bf16
    out) on random operands of the same shape, each rep after an L2 flush; None
    where this torch build cannot run it."""
    import torch
    try:
        import torch.nn.functional as F
        a = torch.randint(0, 256, (m, k // 2), dtype=torch.uint8, device="cuda").view(torch.float4_e2m1fn_x2)
        b = torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device="cuda").view(torch.float4_e2m1fn_x2).t()
        sa = torch.randint(0x30, 0x40, (m * k // 16,), dtype=torch.uint8, device="cuda").view(torch.float8_e4m3fn)
        sb = torch.randint(0x30, 0x40, (n * k // 16,), dtype=torch.uint8, device="cuda").view(torch.float8_e4m3fn)
        g = torch.ones((), dtype=torch.float32, device="cuda")
        blk = [F.ScalingType.BlockWise1x16, F.ScalingType.TensorWise]
        swz = [F.SwizzleType.SWIZZLE_32_4_4, F.SwizzleType.NO_SWIZZLE]

        def call():
            return F.scaled_mm(a, b, [sa, g], blk, [sb, g], blk, swizzle_a=swz, swizzle_b=swz,
                               output_dtype=torch.bfloat16)

        t = statistics.median(time_reps(call, reps, 2, flush))
        del a, b, sa, sb
        torch.cuda.empty_cache()
        return t
    except Exception:
        torch.cuda.empty_cache()
        return None


def fp4_peak_probe(nv, device_index=0):
    """The dense block-scaled FP4 rate of this device from the library's own
    tensor-core probe (nvfp4_mma_peak_probe: the GEMM's pair MMA issued back to
    back from shared-memory-resident operands, no global-memory traffic, one CTA
    per SM).  Burst: launches of ~2 ms after an idle pause, median.  Sustained:
    launches of ~0.25 s back to back for >= 1 s, with the SM clock sampled.  The
    burst is also taken with the GEMM's per-stage scale-factor copies included."""
    import torch
    s = torch.cuda.current_stream()

    def timed(iters, copies):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        fl = nv.mma_peak_probe(iters, with_scale_copies=copies)
        e1.record(s)
        torch.cuda.synchronize()
        return fl / (e0.elapsed_time(e1) * 1e-3) / 1e12

    out = {}
    for copies in (False, True):
        timed(2000, copies)                                  # warm
        rate = timed(20000, copies)                          # calibration
        burst_iters = max(1000, int(2e-3 * rate * 1e12 / (2 * 256 * 256 * 64 * 4 * 74)))
        burst = []
        for _ in range(7):
            time.sleep(0.05)
            burst.append(timed(burst_iters, copies))
        tag = "with_scale_copies_" if copies else ""
        out[f"{tag}burst_tflops"] = round(statistics.median(burst), 1)
        if copies:
            continue                                         # the sustained run is MMA-only
        sustained_iters = burst_iters * 125                  # ~0.25 s per launch
        sampler = ClockSampler(device_index)
        sampler.start()
        time.sleep(0.1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        fl = 0.0
        for _ in range(4):
            fl += nv.mma_peak_probe(sustained_iters, with_scale_copies=copies)
        e1.record(s)
        torch.cuda.synchronize()
        clocks = sampler.stop()
        sec = e0.elapsed_time(e1) * 1e-3
        out[f"{tag}sustained_tflops"] = round(fl / sec / 1e12, 1)
        out[f"{tag}sustained_seconds"] = round(sec, 3)
        out[f"{tag}sustained_clocks"] = clocks
    if nv.get_device_error() != nv.OK:
        raise RuntimeError("device error in the FP4 peak probe")
    out["probe"] = ("tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16, M=256 N=256 K=64, "
                    "operands and scales resident in shared memory, one CTA per SM, 74 pairs")
    return out


def conversion_workloads(nv, W, peaks, flush):
    """Expansion of the decode weights to bf16, checkpoint import of their block
    scales, and harmonization of the fused q/k/v/gate scales (GB/s vs HBM, each
    rep timed alone after an L2 flush)."""
    import torch
    out = {}

    def entry(ms, nbytes):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return dict(ms=round(ms, 4), gbs=round(gbs, 1), frac_hbm=round(gbs / peaks["hbm_gbs"], 4), bytes=int(nbytes))

    wl = W.DECODE
    n, k, off = wl.n, wl.k, wl.seg_offsets
    w = gen_device((n, k), "normal", 51, sigma=0.02)
    w[off[1]:] *= 2.75
    pw = nv.pack_weight(w, off)
    del w
    y = torch.empty((n, k), dtype=torch.bfloat16, device="cuda")
    t = statistics.median(time_reps(lambda: nv.dequantize(pw.q, pw.sf, k, pw.gscale, off, out=y), 10, 3, flush))
    out[f"dequantize_{n}x{k}"] = entry(t, n * k * (0.5 + 1 / 16 + 2))
    del y
    lin = torch.randint(0, 0x7F, (n, k // 16), dtype=torch.uint8, device="cuda")
    sfo = torch.empty_like(pw.sf)
    t = statistics.median(time_reps(lambda: nv.import_weight_scales(lin, n, k, out=sfo), 10, 3, flush))
    out[f"import_scales_{n}x{k}"] = entry(t, n * k // 16 + sfo.numel())
    del lin, sfo, pw
    wl = W.FUSED_QKVG
    n, k, off = wl.n, wl.k, wl.seg_offsets
    w = gen_device((n, k), "normal", 52)
    for i in range(len(off) - 1):
        w[off[i]:off[i + 1]] *= float(wl.seg_sigma[i])
    pw = nv.pack_weight(w, off)
    del w
    t = statistics.median(time_reps(lambda: nv.harmonize_scales(pw), 10, 3, flush))
    out[f"harmonize_{n}x{k}"] = entry(t, 2 * pw.sf.numel())
    del pw
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- CPU oracle

def oracle_step(sample_cols: int):
    """One decode-shaped step on the CPU oracle over a column sample; returns
    (seconds, algorithmic bytes of the sampled work, threads)."""
    import numpy as np

    import oracle
    from nvfp4_w4a4_block_b200 import workloads as W
    wl = W.DECODE
    k = wl.k
    rng = np.random.default_rng(5)
    wb = W.f32_to_bf16_bits(rng.standard_normal((sample_cols, k), dtype=np.float32) * np.float32(0.02))
    s_w = oracle.segment_scales(wb, [0, sample_cols])
    qw, sfw = oracle.quantize(wb, s_w[0])                  # offline packing, not timed
    x32 = wl.x(max(W.DECODE_M))
    t0 = time.perf_counter()
    for m in W.DECODE_M:
        xb = np.ascontiguousarray(x32[:m])
        s_x = oracle.global_scale(oracle.amax(xb))
        qx, sfx = oracle.quantize(xb, s_x)
        oracle.linear_rows(qx, sfx, s_x, np.arange(m), qw, sfw, np.full(sample_cols, s_w[0], np.float32))
    dt = time.perf_counter() - t0
    nbytes = sum(decode_call_bytes(m, sample_cols, k) for m in W.DECODE_M)
    return dt, nbytes, oracle.num_threads()


def cpu_baseline(target_s=10.0):
    """The oracle on the full decode step (all 34816 columns), repeated until
    about target_s seconds of CPU work."""
    total_t, total_b, reps, threads = 0.0, 0, 0, 1
    while total_t < target_s and reps < 50:
        dt, nbytes, threads = oracle_step(34816)
        total_t += dt
        total_b += nbytes
        reps += 1
    return dict(value=round(total_b / total_t / 1e9, 4), unit="GB/s", cores=threads, kind="oracle",
                sample=f"{reps} x one full decode step (M=1,8,32; K=5120; N=34816; weights pre-packed), "
                       f"fp64 GEMM, {total_t:.1f} s")


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on this machine's host cores.
    Each step is the decode step over a column sample sized so that the whole
    --warmup + --steps run takes about 90 s."""
    if rank != 0:
        return None
    t_cal, _, _ = oracle_step(512)
    per_col = t_cal / 512
    budget = min(0.5, 90.0 / (args.steps + args.warmup))
    cols = int(max(64, min(34816, round(budget / per_col / 8) * 8)))
    for _ in range(args.warmup):
        oracle_step(cols)
    times, nbytes, threads = [], 0, 1
    for _ in range(args.steps):
        dt, nbytes, threads = oracle_step(cols)
        times.append(dt)
    total = sum(times)
    value = nbytes * args.steps / total / 1e9
    sample = f"one decode step (M=1,8,32; K=5120) over {cols} of 34816 weight columns per step"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle GEMM)",
        "data": "synthetic (seeded NumPy PCG64)",
        "config": {"workload": "decode-shaped fused gate+up, M in {1,8,32}, K=5120, N=34816 (column sample)",
                   "parallelism": "host cores of rank 0"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }



# ----------------------------------------------------------------------------- profiling cases

def _prof_gemm(m, n, k, seg_offsets, launches, dist="normal"):
    import torch

    import nvfp4_w4a4_block_b200 as nv
    w = gen_device((n, k), "normal", 5, sigma=0.02)
    pw = nv.pack_weight(w, seg_offsets)
    del w
    x = gen_device((m, k), dist, 6, 0.005, 50.0)
    qx, sfx, sx = nv.quantize_act(x)
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    for _ in range(launches):
        nv.gemm(qx, sfx, sx, m, pw, out=y)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK


def _prof_quantize(m, k, launches, static):
    import torch

    import nvfp4_w4a4_block_b200 as nv
    x = gen_device((m, k), "normal", 7, 0.005, 50.0)
    q = torch.empty((m, k // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty(nv.sf_bytes(m, k), dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    nv.quantize_act(x, q=q, sf=sf, gscale_out=s)
    g = s.clone() if static else None
    torch.cuda.synchronize()
    for _ in range(launches):
        nv.quantize_act(x, gscale=g, q=q, sf=sf, gscale_out=s)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK


def _prof_decode_call(m, launches):
    import torch

    import nvfp4_w4a4_block_b200 as nv
    n, k, off = 34816, 5120, [0, 17408, 34816]
    w = gen_device((n, k), "normal", 5, sigma=0.02)
    pw = nv.pack_weight(w, off)
    del w
    x = gen_device((m, k), "normal", 6, 0.005, 50.0)
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    for _ in range(launches):
        nv.linear_fused(x, pw, out=y)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK


def _prof_convert(kind, launches):
    import torch

    import nvfp4_w4a4_block_b200 as nv
    n, k, off = 34816, 5120, [0, 17408, 34816]
    w = gen_device((n, k), "normal", 5, sigma=0.02)
    pw = nv.pack_weight(w, off)
    del w
    y = torch.empty((n, k), dtype=torch.bfloat16, device="cuda") if kind == "dequantize" else None
    lin = torch.randint(0, 0x7F, (n, k // 16), dtype=torch.uint8, device="cuda") if kind == "import" else None
    sfo = torch.empty_like(pw.sf)
    torch.cuda.synchronize()
    for _ in range(launches):
        if kind == "dequantize":
            nv.dequantize(pw.q, pw.sf, k, pw.gscale, off, out=y)
        elif kind == "import":
            nv.import_weight_scales(lin, n, k, out=sfo)
        else:
            nv.harmonize_scales(pw)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK


def _prof_mma_peak(launches):
    import torch

    import nvfp4_w4a4_block_b200 as nv
    for _ in range(launches):
        nv.mma_peak_probe(20000)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK


PROFILE_CASES = {
    "mma_peak": _prof_mma_peak,
    "gemm_decode_m32": lambda L: _prof_gemm(32, 34816, 5120, [0, 17408, 34816], L),
    "gemm_decode_m128": lambda L: _prof_gemm(128, 34816, 5120, [0, 17408, 34816], L),
    "gemm_prefill_8192x17408x5120": lambda L: _prof_gemm(8192, 17408, 5120, [0, 17408], L, "student_t3"),
    "gemm_long_32768x5120x17408": lambda L: _prof_gemm(32768, 5120, 17408, [0, 5120], L),
    "quantize_32768x17408_static": lambda L: _prof_quantize(32768, 17408, L, True),
    "quantize_32768x17408_dynamic": lambda L: _prof_quantize(32768, 17408, L, False),
    "decode_call_m32": lambda L: _prof_decode_call(32, L),
    "decode_call_m8": lambda L: _prof_decode_call(8, L),
    "dequantize_34816x5120": lambda L: _prof_convert("dequantize", L),
    "import_scales_34816x5120": lambda L: _prof_convert("import", L),
    "harmonize_34816x5120": lambda L: _prof_convert("harmonize", L),
}


def run_profile_case(name, launches):
    import torch

    import nvfp4_w4a4_block_b200 as nv
    torch.cuda.set_device(0)
    nv.lib()
    PROFILE_CASES[name](launches)
    print(json.dumps({"profile_case": name, "launches": launches, "ok": True}))

# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="nvfp4", choices=["nvfp4", "reference"])
    ap.add_argument("--skip-secondary", action="store_true", help="primary line only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", default=None, choices=sorted(PROFILE_CASES),
                    help="run one kernel case a few times and exit (for ncu captures)")
    ap.add_argument("--launches", type=int, default=3, help="launches of --profile-case")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.profile_case is not None:
        run_profile_case(args.profile_case, args.launches)
        return

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import datetime

    import torch
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_nvfp4(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline()
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
