"""Benchmark of the MXCode W4A4 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--m 16]

Workload: the decode GEMV shaped like a fused QKV projection -- PostScale,
E4M3-B16-FP4, K_in = 4096, N_out = 9216, M = 16 tokens, one FP4 codebook per
256 x 256 QBlock (synthetic, seeded; see vector_quantized_mx_b200/synth.py).
One step = one pass of the whole path over one batch: activation tensor amax,
BF16 -> FP4 activation quantization, and the split-K W4A4 linear layer that
decodes the VQ weights on the fly.  Steps are captured in a CUDA graph and
rotate over 12 copies of the packed weights (145 MB > 126 MB L2), so every
step streams its weights from HBM.

Metric: effective weight bandwidth -- compressed weight bytes consumed per
second (GB/s), whole job over all ranks.  Extra keys report TFLOPS, the
roofline of the dominant kernel, the same step with native FP4 weights
(4.50 bits/weight) on the same decoded values, the oracle on the host cores,
and the end-to-end number through the Python API with host buffers.

--impl reference times the CPU oracle (oracle/) on a bounded sample of the
same workload (a slice of the output channels per step).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "decode GEMV (fused-QKV shape): PostScale E4M3-B16-FP4, M=16, K=4096, N=9216, 256x256 QBlocks"
N_COPIES = 12


def peaks():
    """(HBM GB/s, its kind) from MEASURED_PEAKS.json, else the machine's fallback figure."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def fp4_peak(sustained: bool = False):
    """Dense block-scaled FP4 tensor peak in TFLOP/s and how it was obtained: the
    measured cuBLAS bf16 peak (burst, or sustained for a kernel timed inside a long
    step) times 4, the nominal FP4 / BF16 dense ratio (9 / 2.25 PFLOP/s)."""
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return 4.0 * float(p[key]), f"measured {key} x 4 (nominal FP4/BF16 ratio)"
    except Exception:
        return 4.0 * (1400.0 if sustained else 1590.0), "fallback bf16 x 4 (nominal FP4/BF16 ratio)"


# ---------------------------------------------------------------------------
# clocks sampled while the timed region runs
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU legs (oracle)
# ---------------------------------------------------------------------------

def oracle_sample(w, x, rows: slice):
    """The oracle on a slice of output channels: (seconds, weight bytes consumed, Y, sum |a w|)."""
    from oracle import mxcode_oracle as O
    from vector_quantized_mx_b200 import synth
    t0 = time.perf_counter()
    sub = synth.weight_rows(w, rows.start, rows.stop)
    ref, sabs = O.w4a4_linear(x, sub)
    dt = time.perf_counter() - t0
    return dt, O.storage_bytes(sub), ref, sabs


def oracle_tile(w, x_rows, cols: slice, tscale=None):
    """The oracle on a tile: the given activation rows (quantized with the tensor
    scale of the whole activation, `tscale`) times the weight rows `cols`.
    Returns (seconds, Y tile, sum |a w| tile)."""
    from oracle import mxcode_oracle as O
    from vector_quantized_mx_b200 import synth
    t0 = time.perf_counter()
    codes, sf, s = O.quantize_act(x_rows, w.fmt, tscale)
    a_hat = O.dequant_act(codes, sf, w.fmt, s)
    w_hat = O.dequant_weight(synth.weight_rows(w, cols.start, cols.stop))
    ref, sabs = O.linear(a_hat, w_hat), O.abs_linear(a_hat, w_hat)
    return time.perf_counter() - t0, ref, sabs


def tile_baseline(w, x, tiles, y_gpu, budget_s, tscale=None):
    """Times the oracle on (row-slice, column-slice) tiles of a layer until budget_s
    seconds of CPU work; each tile is also compared with the GPU output (a NumPy
    array, FP32 or BF16 as float): |gpu - oracle| <= 1e-4 * sum |a w| (+ BF16
    rounding when y_gpu came from a BF16 output).  Returns (TFLOP/s, tiles, seconds)."""
    t_tot, flops, n = 0.0, 0.0, 0
    for r, c, bf16 in tiles:
        dt, ref, sabs = oracle_tile(w, x[r], c, tscale)
        got = np.asarray(y_gpu[r, c], dtype=np.float64)
        bound = 1e-4 * sabs + (np.abs(ref) * 2.0 ** -8 if bf16 else 0.0)
        if not np.all(np.abs(got - ref) <= bound):
            raise SystemExit(f"bench: GPU tile rows {r} cols {c} does not match the oracle")
        t_tot += dt
        flops += 2.0 * (r.stop - r.start) * (c.stop - c.start) * w.K
        n += 1
        if t_tot >= budget_s:
            break
    return flops / t_tot / 1e12, n, t_tot


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w, x, y_gpu=None, budget_s=12.0):
    """The oracle timed on the host cores.  With y_gpu (the GPU step's FP32 output as
    a NumPy array) each distinct slice it computes is also compared with the GPU
    result (|gpu - oracle| <= 1e-4 * sum |a w|); a mismatch stops the bench."""
    rows_per = 1024           # 1/9 of N_out per sample (whole 256-row QBlocks)
    t_tot, b_tot, n = 0.0, 0, 0
    while t_tot < budget_s and n < 200:
        r0 = (n * rows_per) % w.N
        dt, b, ref, sabs = oracle_sample(w, x, slice(r0, r0 + rows_per))
        if y_gpu is not None and n * rows_per < w.N:
            got = y_gpu[:, r0:r0 + rows_per]
            if not np.all(np.abs(got - ref) <= 1e-4 * sabs):
                raise SystemExit(f"bench: GPU output channels {r0}..{r0 + rows_per} do not match the oracle")
        t_tot += dt
        b_tot += b
        n += 1
    return {"value": b_tot / t_tot / 1e9, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} oracle calls, each M=16 x K=4096 over {rows_per} of the 9216 output channels "
                      f"(FP64 dequant + activation quant + FP64 GEMM), {t_tot:.1f} s"}


def run_reference(args, rank, world):
    from vector_quantized_mx_b200 import synth
    if rank != 0:
        return
    w, x = synth.config2(args.m)
    rows_per = 1024
    for i in range(args.warmup):
        oracle_sample(w, x, slice((i * rows_per) % w.N, (i * rows_per) % w.N + rows_per))
    t0 = time.perf_counter()
    b = 0
    for i in range(args.steps):
        r0 = (i * rows_per) % w.N
        _, bb, _, _ = oracle_sample(w, x, slice(r0, r0 + rows_per))
        b += bb
    dt = time.perf_counter() - t0
    v = b / dt / 1e9
    out = {"impl": "reference", "metric": "MXCode W4A4 effective weight bandwidth (compressed bytes/s)",
           "value": v, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": WORKLOAD, "M": args.m, "K": 4096, "N": 9216,
                      "sample": f"{rows_per} of 9216 output channels per step"},
           "cpu_baseline": {"value": v, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                            "sample": f"{rows_per} of 9216 output channels per step, M={args.m}"},
           "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ---------------------------------------------------------------------------
# Multi-rank arithmetic (host side; covered by CPU tests over gloo)
# ---------------------------------------------------------------------------

def measured_traffic(key: str):
    """dram__bytes_read.sum + dram__bytes_write.sum of one launch of a kernel, from the
    ncu capture recorded in profiles/traffic.txt under `key`, or None."""
    prof = os.path.join(ROOT, "profiles", "traffic.txt")
    if os.path.exists(prof):
        for line in open(prof):
            parts = line.split()
            if len(parts) == 2 and parts[0] == key:
                return int(parts[1])
    return None


def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """The largest value over all ranks of the process group (the slowest rank's
    time); x itself without one.  Every rank must call it at the same point."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbps(world: int, bytes_per_step: float, ms_per_step: float) -> float:
    """Whole-job GB/s: each of `world` replicas consumes bytes_per_step every step."""
    return world * bytes_per_step / (ms_per_step * 1e-3) / 1e9


# ---------------------------------------------------------------------------
# GPU leg
# ---------------------------------------------------------------------------

def run_gpu(args, rank, world, dist):
    import torch
    from vector_quantized_mx_b200 import build, mxc, synth

    build.build()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    M = args.m
    w, x = synth.config2(M)
    # weights: N_COPIES packed copies (identical values, distinct buffers)
    pw0 = mxc.pack_weight(w, device=dev)
    copies = [pw0] + [mxc.PackedWeight(pw0.fmt, pw0.strategy, pw0.N, pw0.K, pw0.qn, pw0.qk, pw0.idx.clone(),
                                       pw0.cb.clone(), pw0.scales.clone(), None, None, pw0.w_tscale)
                      for _ in range(N_COPIES - 1)]
    wbytes = pw0.storage_bytes()
    x_host = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    x_dev = x_host.to(dev)
    act = mxc.empty_act(M, w.K, w.fmt, dev)
    qws = torch.zeros(256, dtype=torch.uint8, device=dev)
    lws = mxc.linear_workspace(M, w.N, w.K, w.fmt, dev)
    y = torch.empty((M, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(i):
        mxc.quantize_act(x_dev, w.fmt, out=act, ws=qws, stream=stream)
        mxc.linear(act, copies[i % N_COPIES], y=y, ws=lws, stream=stream)

    # gate before timing: one step runs clean (the oracle comparison is part of the
    # CPU-baseline leg below, and MXCode is checked bit for bit against native FP4)
    with torch.cuda.stream(stream):
        step(0)
    stream.synchronize()
    if mxc.get_device_error(stream) != 0 or not bool(torch.isfinite(y).all()):
        raise SystemExit("bench: the GPU step failed")

    def capture(n_steps, fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            fn(0)                                   # warm the launch path outside capture
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n_steps):
                    fn(i)
        return g

    def time_graph(g):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):          # replay() launches on the current stream
            start.record(stream)
            g.replay()
            end.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        return max_over_ranks(start.elapsed_time(end), dist, dev)

    steps, warmup = args.steps, args.warmup
    g_warm = capture(max(warmup, 1), step)
    g_main = capture(steps, step)
    with torch.cuda.stream(stream):
        g_warm.replay()
        g_main.replay()                          # first replay uploads the graph
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    ms = time_graph(g_main)
    clocks = sampler.stop()
    ms_step = ms / steps
    value = job_gbps(world, wbytes, ms_step)
    flops = 2.0 * M * w.K * w.N
    tflops = world * flops / (ms_step * 1e-3) / 1e12

    # dominant kernel alone: the linear layer, back to back over the rotating copies
    def lin_only(i):
        mxc.linear(act, copies[i % N_COPIES], y=y, ws=lws, stream=stream)
    g_lin = capture(steps, lin_only)
    with torch.cuda.stream(stream):
        g_lin.replay()
    ms_lin = time_graph(g_lin) / steps
    a_bytes = M * w.K // 2 + M * w.K // 16
    alg_bytes = wbytes + a_bytes + M * w.N * 4
    hbm_peak, peak_kind = peaks()
    achieved = alg_bytes / (ms_lin * 1e-3) / 1e9

    # native FP4 on the same decoded values (4.50 bits/weight), same rotation
    nat0 = mxc.decode_weight(pw0)
    nats = [nat0] + [mxc.MXTensor(nat0.q.clone(), nat0.sf.clone(), nat0.tscale.clone(), nat0.rows, nat0.K, nat0.fmt)
                     for _ in range(N_COPIES - 1)]
    with torch.cuda.stream(stream):
        yn = mxc.native_linear(act, nats[0], stream=stream)
    stream.synchronize()
    y_ref = torch.empty_like(y)
    with torch.cuda.stream(stream):
        mxc.linear(act, pw0, y=y_ref, ws=lws, stream=stream)
    stream.synchronize()
    same = bool(torch.equal(yn, y_ref))

    def nat_step(i):
        mxc.quantize_act(x_dev, w.fmt, out=act, ws=qws, stream=stream)
        mxc.native_linear(act, nats[i % N_COPIES], y=y, ws=lws, stream=stream)
    g_nat = capture(steps, nat_step)
    with torch.cuda.stream(stream):
        g_nat.replay()
    ms_nat = time_graph(g_nat) / steps
    nat_bytes = w.N * w.K // 2 + w.N * w.K // 16

    # end to end through the Python API with host buffers (pinned): the same calls
    # captured in a CUDA graph (how a serving loop issues them), and issued eagerly
    y_host = torch.empty((M, w.N), dtype=torch.float32).pin_memory()

    def e2e_step(i):
        x_dev.copy_(x_host, non_blocking=True)
        mxc.quantize_act(x_dev, w.fmt, out=act, ws=qws, stream=stream)
        mxc.linear(act, copies[i % N_COPIES], y=y, ws=lws, stream=stream)
        y_host.copy_(y, non_blocking=True)
    g_e2e = capture(steps, e2e_step)
    with torch.cuda.stream(stream):
        g_e2e.replay()
    ms_e2e_serial = time_graph(g_e2e) / steps
    del g_e2e

    # the same step as a serving loop runs it: double-buffered input and output, the
    # host->device copy and the result read-back on copy streams, overlapped with the
    # neighbouring steps' compute (each step still copies its input in and its result out)
    h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    xb = [torch.empty_like(x_dev) for _ in range(2)]
    yb = [torch.empty_like(y) for _ in range(2)]
    yh = [torch.empty((M, w.N), dtype=torch.float32).pin_memory() for _ in range(2)]
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "quant", "lin", "out")}

    def e2e_pipelined(i):
        b = i % 2
        if i >= 2:
            h2d.wait_event(ev["quant"][b])            # step i-2 has read this input buffer
        with torch.cuda.stream(h2d):
            xb[b].copy_(x_host, non_blocking=True)
        ev["in"][b].record(h2d)
        stream.wait_event(ev["in"][b])
        if i >= 2:
            stream.wait_event(ev["out"][b])           # step i-2's result has left this buffer
        mxc.quantize_act(xb[b], w.fmt, out=act, ws=qws, stream=stream)
        ev["quant"][b].record(stream)
        mxc.linear(act, copies[i % N_COPIES], y=yb[b], ws=lws, stream=stream)
        ev["lin"][b].record(stream)
        d2h.wait_event(ev["lin"][b])
        with torch.cuda.stream(d2h):
            yh[b].copy_(yb[b], non_blocking=True)
        ev["out"][b].record(d2h)

    def e2e_pipelined_run(n):
        fork = torch.cuda.Event()                     # the copy streams join the capture
        fork.record(stream)
        h2d.wait_event(fork)
        d2h.wait_event(fork)
        for i in range(n):
            e2e_pipelined(i)
        for st in (h2d, d2h):                         # join the copy streams
            j = torch.cuda.Event()
            j.record(st)
            stream.wait_event(j)

    g_pipe = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        e2e_pipelined_run(2)
        stream.synchronize()
        with torch.cuda.graph(g_pipe, stream=stream):
            e2e_pipelined_run(steps)
        g_pipe.replay()
    ms_e2e_graph = time_graph(g_pipe) / steps
    torch.cuda.synchronize()
    e2e_same = bool(torch.equal(yh[0], yh[1]) and torch.equal(yh[(steps - 1) % 2].cuda(dev), y))
    del g_pipe
    with torch.cuda.stream(stream):
        for i in range(warmup):
            e2e_step(i)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for i in range(steps):
            e2e_step(i)
        s1.record(stream)
        torch.cuda.synchronize()
    ms_e2e = max_over_ranks(s0.elapsed_time(s1) / steps, dist, dev)

    extra = {}
    with_cpu = not args.no_cpu_baseline and world == 1 and rank == 0
    if "prefill" in args.legs:
        extra["prefill"] = prefill_leg(dev, stream, capture, time_graph, steps, world, with_cpu)
    if "moe" in args.legs:
        extra["moe"] = moe_leg(dev, stream, capture, time_graph, steps, world, with_cpu)
    if "sweep" in args.legs:
        extra["sweep"] = sweep_leg(dev, stream, capture, time_graph, steps, world)
    if rank != 0:
        return
    # our kernels per step: the activation quantizer (one launch up to 16 x 8192
    # elements, else tensor amax + quantize) and the linear layer
    launches_per_step = (1 if M * w.K <= 16 * 8192 else 2) + 1
    traffic = measured_traffic("decode_gemv_m16_bytes_per_launch")
    out = {
        "metric": "MXCode W4A4 effective weight bandwidth (compressed bytes/s)",
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e2m1 x e2m1 -> f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "K": w.K, "N": w.N, "bits_per_weight": wbytes * 8 / (w.N * w.K),
                   "l2": f"rotating {N_COPIES} weight copies ({N_COPIES * wbytes / 1e6:.0f} MB > 126 MB L2)",
                   "parallelism": f"replicas x{world}"},
        "tflops": tflops,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": traffic, "peak_kind": peak_kind,
                     "kernel": "gemv_kernel<E4M3, VQ direct> (cluster split-K decode GEMV)",
                     "ms_per_launch": ms_lin, "alg_bytes_per_launch": alg_bytes},
        "native_fp4": {"ms_per_step": ms_nat, "weight_bytes": nat_bytes,
                       "weight_GBps": job_gbps(world, nat_bytes, ms_nat),
                       "mxcode_speedup": ms_nat / ms_step, "bitwise_equal_outputs": same},
        "e2e": {"value": job_gbps(world, wbytes, ms_e2e_graph), "unit": "GB/s",
                "h2d_bytes_per_step": int(x_host.numel() * 2), "d2h_bytes_per_step": int(y_host.numel() * 4),
                "ms_per_step": ms_e2e_graph,
                "launch": "CUDA graph of the API calls; double-buffered input/output, both copies on copy "
                          "streams overlapped with the neighbouring steps' compute",
                "results_match_device_step": e2e_same,
                "serial_graph": {"value": job_gbps(world, wbytes, ms_e2e_serial), "ms_per_step": ms_e2e_serial},
                "eager": {"value": job_gbps(world, wbytes, ms_e2e), "ms_per_step": ms_e2e}},
        "gpu_launches": launches_per_step * steps,
        "clocks": clocks,
    }
    if not args.no_cpu_baseline and world == 1:       # the oracle on the host: rank 0 at N=1 only
        out["cpu_baseline"] = cpu_baseline(w, x, y_ref.cpu().numpy())
    if extra is not None:
        out.update(extra)
    print(json.dumps(out), flush=True)


def rotated(pw0, n):
    """n packed copies of one weight (the same values in distinct buffers)."""
    from vector_quantized_mx_b200 import mxc
    cl = lambda t: None if t is None else t.clone()
    return [pw0] + [mxc.PackedWeight(pw0.fmt, pw0.strategy, pw0.N, pw0.K, pw0.qn, pw0.qk, pw0.idx.clone(),
                                     pw0.cb.clone(), cl(pw0.scales), cl(pw0.sidx), cl(pw0.scb), pw0.w_tscale, pw0.ds)
                    for _ in range(n - 1)]


def prefill_leg(dev, stream, capture, time_graph, steps, world, with_cpu):
    """Config 3: prefill GEMM, PreScale E8M0-B32, M=8192, K=4096, N=9216, 256x256
    QBlocks, BF16 output.  One step = activation quantization + MXCode linear (decode
    once into the workspace, then the native block-scaled GEMM).  The dominant kernel
    is the GEMM; its duration is taken from the native linear on the decoded weight,
    which launches exactly that kernel on the same operands."""
    import torch
    from vector_quantized_mx_b200 import mxc, synth
    w, x = synth.config3()
    M, N, K = x.shape[0], w.N, w.K
    copies = rotated(mxc.pack_weight(w, device=dev), N_COPIES)
    x_dev = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    act = mxc.empty_act(M, K, w.fmt, dev)
    qws = torch.zeros(256, dtype=torch.uint8, device=dev)
    lws = mxc.linear_workspace(M, N, K, w.fmt, dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    with torch.cuda.stream(stream):
        nat0 = mxc.decode_weight(copies[0], stream=stream)
        nats = [nat0] + [mxc.MXTensor(nat0.q.clone(), nat0.sf.clone(), nat0.tscale.clone(), N, K, w.fmt)
                         for _ in range(N_COPIES - 1)]
        mxc.quantize_act(x_dev, w.fmt, out=act, ws=qws, stream=stream)
        mxc.linear(act, copies[0], y=y, ws=lws, stream=stream)
        yn = mxc.native_linear(act, nats[0], out_dtype=torch.bfloat16, ws=lws, stream=stream)
    stream.synchronize()
    if mxc.get_device_error(stream) != 0:
        raise SystemExit("bench: the prefill step failed")
    same = bool(torch.equal(y, yn))

    def step(i):
        mxc.quantize_act(x_dev, w.fmt, out=act, ws=qws, stream=stream)
        mxc.linear(act, copies[i % N_COPIES], y=y, ws=lws, stream=stream)

    def lin(i):
        mxc.linear(act, copies[i % N_COPIES], y=y, ws=lws, stream=stream)

    def nat_lin(i):
        mxc.native_linear(act, nats[i % N_COPIES], y=yn, ws=lws, stream=stream)

    def nat_step(i):
        mxc.quantize_act(x_dev, w.fmt, out=act, ws=qws, stream=stream)
        mxc.native_linear(act, nats[i % N_COPIES], y=yn, ws=lws, stream=stream)
    n = max(10, steps // 4)
    ms = {name: time_graph(capture(n, fn)) / n for name, fn in
          (("step", step), ("linear", lin), ("native_linear", nat_lin), ("native_step", nat_step))}
    flops = 2.0 * M * N * K
    peak, peak_kind = fp4_peak()
    wbytes = copies[0].storage_bytes()
    out = {"workload": "prefill GEMM: PreScale E8M0-B32-FP4, M=8192, K=4096, N=9216, 256x256 QBlocks, BF16 out",
           "ms_per_step": ms["step"], "ms_linear": ms["linear"],
           "tflops": world * flops / (ms["linear"] * 1e-3) / 1e12,
           "tflops_step": world * flops / (ms["step"] * 1e-3) / 1e12,
           "weight_GBps": world * wbytes / (ms["linear"] * 1e-3) / 1e9,
           "roofline": {"bound": "tensor", "unit": "TFLOP/s", "peak": peak, "peak_kind": peak_kind,
                        "kernel": "gemm_pair_kernel<E8M0> (persistent CTA-pair native GEMM of the decode-once path)",
                        "ms_per_launch": ms["native_linear"], "flops_per_launch": flops,
                        "achieved": flops / (ms["native_linear"] * 1e-3) / 1e12,
                        "frac": flops / (ms["native_linear"] * 1e-3) / 1e12 / peak,
                        "layer_frac": flops / (ms["linear"] * 1e-3) / 1e12 / peak,
                        "traffic": measured_traffic("prefill_pair_gemm_bytes_per_launch")},
           "native_fp4": {"ms_linear": ms["native_linear"], "ms_per_step": ms["native_step"],
                          "mxcode_speedup": ms["native_linear"] / ms["linear"],
                          "mxcode_step_speedup": ms["native_step"] / ms["step"],
                          "bitwise_equal_outputs": same},
           "gpu_launches_per_step": 3, "l2": f"rotating {N_COPIES} weight copies; 151 MB BF16 output per step"}
    if with_cpu:
        yh = y.float().cpu().numpy()
        rng = np.random.default_rng(3)
        tiles = []
        for _ in range(8):
            r0, c0 = int(rng.integers(0, M // 256)) * 256, int(rng.integers(0, N // 256)) * 256
            tiles.append((slice(r0, r0 + 256), slice(c0, c0 + 256), True))
        v, nt, t = tile_baseline(w, x, tiles, yh, budget_s=8.0)
        out["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                               "sample": f"{nt} seeded 256x256 output tiles (K=4096) of the prefill layer, "
                                         f"each compared with the GPU output, {t:.1f} s"}
    return out


def moe_leg(dev, stream, capture, time_graph, steps, world, with_cpu):
    """Config 4: MoE, PreScale+ E4M3-B16, 128 experts with gate/up [3072, 4096] and
    down [4096, 1536], 2048 tokens routed top-8 by Zipf(1.1) = 16384 expert-sorted
    rows, BF16 outputs.  One step = grouped quantization + MXCode grouped linear,
    for gate/up and then for down (whose input is synthetic: the SwiGLU between the
    two is not part of the layer).  Roofline per projection: the aggregate bound
    max(compressed weight bytes / HBM, flops / FP4 peak)."""
    import torch
    from vector_quantized_mx_b200 import mxc, synth
    row_tok, off = synth.config4_routing()
    E = synth.MOE_EXPERTS
    offd = torch.from_numpy(off.astype(np.int32)).to(dev)
    M = int(off[-1])
    proj = {}
    for name in ("gate_up", "down"):
        x = synth.config4_activations(name, row_tok)
        ws = [synth.config4_expert(e, name) for e in range(E)]
        packed = [mxc.pack_weight(w, device=dev) for w in ws]
        K, N = ws[0].K, ws[0].N
        proj[name] = {"x": x, "w": ws, "packed": packed, "K": K, "N": N,
                      "x_dev": torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev),
                      "act": mxc.empty_act_grouped(M, K, E, "e4m3_b16", dev),
                      "qws": torch.zeros(256 + 4 * (E + 1), dtype=torch.uint8, device=dev),
                      "mws": torch.zeros(max(16, mxc.lib().mxc_moe_workspace_bytes(M, E, N, K, 1)),
                                         dtype=torch.uint8, device=dev),
                      "y": torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                      "bytes": sum(p.storage_bytes() for p in packed), "flops": 2.0 * M * N * K}

    def quant(p):
        mxc.quantize_act_grouped(p["x_dev"], "e4m3_b16", offd, out=p["act"], ws=p["qws"], stream=stream)

    def moe(p):
        mxc.moe_linear(p["act"], offd, p["packed"], y=p["y"], ws=p["mws"], stream=stream)

    with torch.cuda.stream(stream):
        for p in proj.values():
            quant(p)
            moe(p)
    stream.synchronize()
    if mxc.get_device_error(stream) != 0:
        raise SystemExit("bench: the MoE step failed")

    def step(i):
        for p in proj.values():
            quant(p)
            moe(p)
    n = max(5, steps // 8)
    ms_step = time_graph(capture(n, step)) / n
    hbm, hbm_kind = peaks()
    peak, peak_kind = fp4_peak()
    out = {"workload": "MoE: PreScale+ E4M3-B16-FP4, 128 experts (gate/up 3072x4096, down 4096x1536), "
                       "2048 tokens top-8 Zipf(1.1) = 16384 rows, 256x256 QBlocks, BF16 out",
           "ms_per_step": ms_step, "rows": M, "gpu_launches_per_step": 4 * 2}
    for name, p in proj.items():
        n_l = max(5, steps // 8)
        ms_lin = time_graph(capture(n_l, lambda i, p=p: moe(p))) / n_l
        t_bw = p["bytes"] / (hbm * 1e9) * 1e3
        t_fl = p["flops"] / (peak * 1e12) * 1e3
        out[name] = {"ms_linear": ms_lin, "tflops": world * p["flops"] / (ms_lin * 1e-3) / 1e12,
                     "weight_GBps": world * p["bytes"] / (ms_lin * 1e-3) / 1e9, "weight_bytes": p["bytes"],
                     "roofline": {"bound": "hbm" if t_bw >= t_fl else "tensor",
                                  "kernel": "moe_round_kernel<E4M3, VQ scale-VQ> (persistent) + group prologue",
                                  "target_ms": max(t_bw, t_fl), "frac": max(t_bw, t_fl) / ms_lin,
                                  "hbm_peak_GBps": hbm, "hbm_kind": hbm_kind,
                                  "fp4_peak_TFLOPs": peak, "fp4_kind": peak_kind,
                                  "traffic": measured_traffic(f"moe_{name}_bytes_per_launch")}}
    # The MoE FFN with SwiGLU fused into the gate/up epilogue, which writes the down
    # projection's FP4 activation directly: grouped quantization -> gate/up + SwiGLU
    # -> down.  h's E4M3 tensor scale is calibrated once from a torch evaluation of
    # SwiGLU on the gate/up output (plumbing, outside the timed region).
    pg, pd = proj["gate_up"], proj["down"]
    F = pg["N"] // 2
    with torch.cuda.stream(stream):
        ygu = mxc.moe_linear(pg["act"], offd, pg["packed"], stream=stream)
        hcal = torch.nn.functional.silu(ygu[:, :F]) * ygu[:, F:]
        h_ts = (hcal.abs().max() / 2688.0).reshape(1).to(torch.float32)
        h_act = mxc.moe_gate_up_swiglu(pg["act"], offd, pg["packed"], h_tscale=h_ts, ws=pg["mws"], stream=stream)
    stream.synchronize()
    del ygu, hcal

    def ffn(i):
        quant(pg)
        mxc.moe_gate_up_swiglu(pg["act"], offd, pg["packed"], h_tscale=h_ts, out=h_act, ws=pg["mws"], stream=stream)
        mxc.moe_linear(h_act, offd, pd["packed"], y=pd["y"], ws=pd["mws"], stream=stream)
    n_f = max(5, steps // 8)
    ms_ffn = time_graph(capture(n_f, ffn)) / n_f
    ms_gus = time_graph(capture(n_f, lambda i: mxc.moe_gate_up_swiglu(
        pg["act"], offd, pg["packed"], h_tscale=h_ts, out=h_act, ws=pg["mws"], stream=stream))) / n_f
    if mxc.get_device_error(stream) != 0:
        raise SystemExit("bench: the fused MoE FFN failed")
    out["ffn_swiglu_fused"] = {"ms_per_step": ms_ffn, "ms_gate_up_swiglu": ms_gus,
                               "tflops": world * (pg["flops"] + pd["flops"]) / (ms_ffn * 1e-3) / 1e12,
                               "steps": "grouped quantization, gate/up + SwiGLU + FP4 quantization of h, down",
                               "gpu_launches_per_step": 2 + 2 + 2}
    if with_cpu:
        from oracle import mxcode_oracle as O
        counts = np.diff(off)
        p = proj["gate_up"]
        yh = p["y"].float().cpu().numpy()
        s = O.tensor_scale_e4m3(p["x"])
        t_tot, flops, nt = 0.0, 0.0, 0
        for e in [int(counts.argmax()), 0, 17, 64, 127]:
            r0, r1 = int(off[e]), min(int(off[e + 1]), int(off[e]) + 128)
            if r1 <= r0:
                continue
            dt, ref, sabs = oracle_tile(p["w"][e], p["x"][r0:r1], slice(1024, 1280), s)
            got = yh[r0:r1, 1024:1280]
            if not np.all(np.abs(got - ref) <= 1e-4 * sabs + np.abs(ref) * 2.0 ** -8):
                raise SystemExit(f"bench: MoE expert {e} does not match the oracle")
            t_tot += dt
            flops += 2.0 * (r1 - r0) * 256 * p["K"]
            nt += 1
        out["cpu_baseline"] = {"value": flops / t_tot / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
                               "kind": "oracle",
                               "sample": f"{nt} expert tiles (<=128 rows x 256 columns, K=4096) of gate/up, "
                                         f"each compared with the GPU output, {t_tot:.1f} s"}
    return out


def sweep_leg(dev, stream, capture, time_graph, steps, world):
    """Config 5: K = N = 8192; M in {1, 16, 128, 1024, 16384} x QBlock in {full tensor,
    1024^2, 256^2, 128^2} x {PostScale, PreScale, PreScale+} x {E8M0-B32, E4M3-B16}
    (120 MXCode points), plus native FP4 (4.25 / 4.50 bits per weight) on the same
    decoded values of the PreScale 256^2 weights for each format and M (10 points).
    Each point times the linear layer alone, over 6 rotating weight copies (>= 100 MB,
    so M <= 128 streams its weights from HBM).  Bound: HBM for M <= 16, FP4 tensor
    for M >= 1024, both reported at M = 128; frac is against the bound's peak."""
    import torch
    from vector_quantized_mx_b200 import mxc, synth
    K = N = 8192
    n_copies = 6
    hbm, hbm_kind = peaks()
    fp4, fp4_kind = fp4_peak()
    acts = {}
    for M in synth.SWEEP_M:
        x = torch.from_numpy(synth.config5_activations(M).view(np.int16)).view(torch.bfloat16).to(dev)
        for fmt in synth.FORMATS:
            with torch.cuda.stream(stream):
                acts[(M, fmt)] = mxc.quantize_act(x, fmt, stream=stream)
        del x
    stream.synchronize()
    ws = {M: mxc.linear_workspace(M, N, K, "e4m3_b16", dev) for M in synth.SWEEP_M}
    ys = {M: torch.empty((M, N), dtype=torch.bfloat16, device=dev) for M in synth.SWEEP_M}
    cols = ["M", "qblock", "strategy", "format", "ms", "tflops", "weight_GBps", "bound", "frac", "x_native"]
    rows, native = [], {}

    def timed(fn):
        n = max(5, steps // 4)
        return time_graph(capture(n, fn)) / n

    for fmt in synth.FORMATS:
        for strat in synth.STRATEGIES:
            for qb in synth.SWEEP_QB:
                w = synth.config5_weight(qb, strat, fmt)
                copies = rotated(mxc.pack_weight(w, device=dev), n_copies)
                wbytes = copies[0].storage_bytes()
                nats = None
                if strat == "prescale" and qb == 256:
                    with torch.cuda.stream(stream):
                        nat0 = mxc.decode_weight(copies[0], stream=stream)
                    nats = [nat0] + [mxc.MXTensor(nat0.q.clone(), nat0.sf.clone(), nat0.tscale.clone(), N, K, fmt)
                                     for _ in range(n_copies - 1)]
                for M in synth.SWEEP_M:
                    a, y, wk = acts[(M, fmt)], ys[M], ws[M]
                    ms = timed(lambda i: mxc.linear(a, copies[i % n_copies], y=y, ws=wk, stream=stream))
                    if nats is not None:
                        native[(fmt, M)] = timed(lambda i: mxc.native_linear(a, nats[i % n_copies], y=y, ws=wk,
                                                                             stream=stream))
                    flops = 2.0 * M * N * K
                    io = wbytes + M * K // 2 + M * K // (32 if fmt == "e8m0_b32" else 16) + M * N * 2
                    f_hbm = io / (ms * 1e-3) / 1e9 / hbm
                    f_fp4 = flops / (ms * 1e-3) / 1e12 / fp4
                    bound = "hbm" if M <= 16 else "tensor" if M >= 1024 else "both"
                    frac = f_hbm if M <= 16 else f_fp4 if M >= 1024 else [f_hbm, f_fp4]
                    rows.append([M, qb or "full", strat, fmt, ms, world * flops / (ms * 1e-3) / 1e12,
                                 world * wbytes / (ms * 1e-3) / 1e9, bound, frac, None])
                del copies, nats
    if mxc.get_device_error(stream) != 0:
        raise SystemExit("bench: a sweep point failed")
    for r in rows:
        r[9] = native[(r[3], r[0])] / r[4]
    nat_rows = [[M, fmt, native[(fmt, M)], world * 2.0 * M * N * K / (native[(fmt, M)] * 1e-3) / 1e12]
                for fmt in synth.FORMATS for M in synth.SWEEP_M]
    return {"workload": "K=N=8192 sweep: M x QBlock x strategy x format, BF16 out", "columns": cols,
            "points": rows, "native_columns": ["M", "format", "ms", "tflops"], "native": nat_rows,
            "peaks": {"hbm_GBps": hbm, "hbm_kind": hbm_kind, "fp4_TFLOPs": fp4, "fp4_kind": fp4_kind},
            "l2": f"{n_copies} rotating weight copies per point"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="mxcode", choices=["mxcode", "reference"])
    ap.add_argument("--m", type=int, default=16, choices=[1, 4, 16])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--legs", default="prefill,moe,sweep",
                    help="extra workloads timed after the decode line: prefill (config 3), moe (config 4), "
                         "sweep (config 5)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_gpu(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
