"""Benchmark of the strided-view GEMM library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dg|reference]

Headline step (one pass of the hot path over one batch): the decode GEMV
workload, x[1x4096] * W[4096x14336] and x * K^T with K[128x4096] read in place,
BF16 in, FP32 accumulate, BF16 out, both through dg_gemm.  The metric for
M = 1 is HBM GB/s: algorithmic bytes (every operand byte read once, every
output byte written once) per second.  Weights rotate through three copies
(352 MB, more than the 126 MB L2) so every step streams W from HBM.

Beside the headline the JSON line carries, per workload of the benchmark
definition, TFLOPS, GB/s and the fraction of the roofline
max(FLOPs / tensor peak, bytes / HBM bandwidth) under "per_shape"; the
dominant kernel's roofline ("roofline"); an end-to-end figure through the
same API with host buffers ("e2e"); the FP64 CPU oracle timed on the host
("cpu_baseline"); SM clocks sampled during the timed region ("clocks").

--impl reference times the oracle (the plain CPU implementation the tests
check against) on the same metric and workload, on a bounded sample per step.
Under torchrun with N > 1, ranks run independent replicas (weak scaling, no
collective on the data path); rank 0 prints the line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import shutil
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "GEMM TFLOPS & % of roofline per shape (HBM GB/s for M=1) on 1 B200"
WORKLOAD = ("decode GEMV: x[1x4096]*W[4096x14336] + x*K^T with K[128x4096] read in place; "
            "BF16 in, FP32 accumulate, BF16 out")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0, "source": "fallback"}
ROTATE = 3


# ----------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def flops_bytes(p: W.Problem):
    """Algorithmic FLOPs (2MNK) and bytes: A, B and C written once; C read too
    when beta != 0; the FP8 scales."""
    es = W.ELEM_SIZE
    M, N, K = p.M, p.N, p.K
    b = M * K * es[p.A.dtype] + K * N * es[p.B.dtype] + M * N * es[p.C.dtype]
    if p.beta != 0:
        b += M * N * es[p.C.dtype]
    if p.scale_a is not None:
        b += 4 * M
    if p.scale_b is not None:
        b += 4 * N
    if p.bias is not None:
        b += 4 * N
    return 2.0 * M * N * K, float(b)


def tensor_peak_tflops(dtype: str, peaks) -> float:
    base = peaks["bf16_tflops"]
    return base * 2.0 if dtype == "e4m3" else base  # FP8 dense = 2x BF16 (nominal ratio 4.5/2.25)


def roofline_time_s(p: W.Problem, peaks):
    fl, by = flops_bytes(p)
    t_tc = fl / (tensor_peak_tflops(p.A.dtype, peaks) * 1e12)
    t_mem = by / (peaks["hbm_gbs"] * 1e9)
    return max(t_tc, t_mem), ("tensor" if t_tc >= t_mem else "hbm")


def gpu_smi_id(dev: int) -> str:
    """The GPU's UUID as nvidia-smi and NVML name it ("GPU-..."), so that the
    clock samples come from the GPU this process runs on even when
    CUDA_VISIBLE_DEVICES renumbers the devices; the index as a fallback."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev)


class ClockSampler:
    """nvidia-smi samples (every 100 ms) of SM clock and throttle reasons."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        self.dev = gpu_smi_id(device_index)
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
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
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "nvidia-smi unavailable"}
        rows = []
        for ts, line in self.samples:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9], parts[4]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1]
        window = "timed region"
        if not inside:
            inside = rows
            window = "whole run (timed region shorter than the sampling interval)"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "no samples"}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside), "window": window}


def kernel_traffic(kernel_file: str, summary_file: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel (its sha256 is recorded beside it)."""
    path = os.path.join(ROOT, "profiles", summary_file)
    src = os.path.join(ROOT, "tcgen05_tmem_gemm_b200", "csrc", kernel_file)
    if not os.path.exists(path):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    rec = {}
    for line in open(path):
        if ":" in line and line.strip().startswith(("dram_bytes_per_launch", "kernel_source_sha")):
            k, v = line.split(":", 1)
            rec[k.strip()] = v.split()[0] if v.split() else ""
    if rec.get("kernel_source_sha") != sha:
        return None
    try:
        return float(rec["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------- the dg arm

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's time: every rank's timed region must be over."""
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(bytes_per_step: float, steps: int, world: int, elapsed_max_s: float) -> float:
    """Weak scaling: every rank runs its own replica of the step, so the job
    moves world * steps * bytes_per_step in the slowest rank's time (GB/s)."""
    return bytes_per_step * steps * world / elapsed_max_s / 1e9


def shard_columns(n: int, rank: int, world: int):
    """Columns [lo, hi) of an N-wide output owned by `rank` when one GEMM is
    split across GPUs by columns of B and C (A replicated): the shards are
    independent GEMMs with no exchange on the data path."""
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def hold_gpu(us: float = 150.0):
    """Keep the GPU busy for about `us` microseconds (PyTorch's spin kernel)
    before a timed region is enqueued: the start event and the graphs queue
    up behind it while the host submits them, so the host's submission
    latency of the first graph does not land inside the timed region.  The
    spin kernel itself runs before the start event, outside the region."""
    torch.cuda._sleep(int(us * 2000))  # about 2000 cycles per microsecond at B200 clocks


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def dg_views(p: W.Problem, dg):
    def v(op):
        return dg.make_view(op.base.data_ptr() + op.offset, op.shape, op.stride, op.row_dims, op.dtype)

    return v(p.A), v(p.B), v(p.C)


def time_problem(p_gpu_list, dg, reps: int, warm: int):
    """Per-call times over `reps` calls that rotate through the given
    device-resident copies:
      graph  - the calls captured in one CUDA graph and replayed ten times
               (device time, no host launch cost between kernels): the median
               per call over the replays, and (p10, p90) as the fourth value,
      stream - the same calls enqueued back to back on a stream (includes the
               host cost of each call when the GPU outruns the host),
      host   - host seconds per dg_gemm call while enqueuing."""
    views = [dg_views(p, dg) for p in p_gpu_list]
    s = torch.cuda.Stream()

    epis = [dg.epilogue(q.bias, q.act) if (q.bias is not None or q.act != "none") else None for q in p_gpu_list]

    def calls(n, stream):
        for i in range(n):
            q = p_gpu_list[i % len(views)]
            A, B, C = views[i % len(views)]
            e = epis[i % len(views)]
            if e is None:
                st = dg.dg_gemm(A, B, C, q.alpha, q.beta, q.scale_a, q.scale_b, stream)
            else:
                st = dg.dg_gemm_ex(A, B, C, q.alpha, q.beta, q.scale_a, q.scale_b, e, stream)
            assert st == dg.DG_OK, dg.status_string(st)

    with torch.cuda.stream(s):
        calls(warm, s)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        h0 = time.perf_counter()
        calls(reps, s)
        host = (time.perf_counter() - h0) / reps
        b.record(s)
        torch.cuda.synchronize()
        t_stream = a.elapsed_time(b) * 1e-3 / reps
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
            calls(reps, s)
        g.replay()
        torch.cuda.synchronize()
        # ten replays back to back, each bracketed by its own events: the
        # per-call time is the median over replays, with p10 and p90
        n_rep = 10
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_rep)]
        hold_gpu()
        for ea, eb in evs:
            ea.record(s)
            g.replay()
            eb.record(s)
        torch.cuda.synchronize()
        per_call = sorted(ea.elapsed_time(eb) * 1e-3 / reps for ea, eb in evs)
        t_graph = statistics.median(per_call)
        spread = (per_call[1], per_call[-2])  # p10, p90 of ten
        del g
    assert dg.dg_sync_status(s) == dg.DG_OK
    return t_graph, t_stream, host, spread


# (key, name, workload, rotating copies).  The HBM-bound workloads rotate
# through enough copies that every call reads at least twice the 126 MB L2
# worth of other inputs between two uses of the same copy: gemv 3 x 117 MB,
# gemv_kt 256 x 1 MB, thin 8 x 36 MB, strided 17 x 15 MB.  The square GEMMs are
# compute-bound (2 copies); the small GEMM is launch-bound and L2-resident.
SHAPES = [("small", "small_f16_128x128x256", W.cfg_small, 1),
          ("gemv", "gemv_bf16_1x14336x4096", W.cfg_gemv, ROTATE),
          ("gemv_kt", "gemv_kt_bf16_1x128x4096", W.cfg_gemv_kt, 256),
          ("thin", "thin_f16_64x4096x4096_beta1", W.cfg_thin, 8),
          ("square_bf16", "square_bf16_4096^3", W.cfg_square_bf16, 2),
          ("square_e4m3", "square_e4m3_4096^3", W.cfg_square_e4m3, 2),
          ("strided", "strided_nchw_bf16_3136x1024x256", W.cfg_strided, 17),
          # the fused epilogue (bias per output column + activation, one kernel)
          ("square_bf16_gelu", "square_bf16_4096^3_bias_gelu",
           lambda: W.with_epilogue(W.cfg_square_bf16(), "gelu_tanh"), 2),
          ("thin_gelu", "thin_f16_64x4096x4096_beta1_bias_gelu",
           lambda: W.with_epilogue(W.cfg_thin(), "gelu_tanh"), 8),
          ("strided_nchw_out", "strided_nchw_bf16_3136x1024x256_to_nchw_bias_relu",
           lambda: _strided_nchw_out(), 17)]


def _strided_nchw_out() -> W.Problem:
    """The strided workload with its output written as an NCHW tensor
    [16, 1024, 14, 14] by the epilogue, with a bias and ReLU fused."""
    p = W.with_epilogue(W.cfg_strided(), "relu")
    return W.Problem(p.name + "_nchw_out", p.A, p.B, W.nchw_out(16, 1024, 14, 14), 1.0, 0.0,
                     bias=p.bias, act="relu")


class NvmlClockPoller:
    """SM clock and power-cap state polled through NVML every half millisecond
    in a thread, for timed regions far shorter than nvidia-smi's interval
    (a per-shape timing lasts a few milliseconds).  Reads only."""

    def __init__(self, device_index: int):
        self.samples = []
        self.ok = False
        self.stop_flag = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            gid = gpu_smi_id(device_index)
            self.h = (pynvml.nvmlDeviceGetHandleByUUID(gid) if gid.startswith("GPU-")
                      else pynvml.nvmlDeviceGetHandleByIndex(device_index))
            self.ok = True
        except Exception:  # no NVML: the rows go without a clock
            self.ok = False

    def _run(self):
        nv = self.nv
        cap = getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4)
        while not self.stop_flag.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, bool(reasons & cap)))
            except Exception:
                return
            time.sleep(0.0005)

    def __enter__(self):
        if self.ok:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self.stop_flag.set()
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return None
        return {"sm_mhz_median": statistics.median(m for m, _ in self.samples),
                "sm_mhz_min": min(m for m, _ in self.samples),
                "sw_power_cap_share": sum(1 for _, c in self.samples if c) / len(self.samples),
                "samples": len(self.samples)}


def per_shape(dg, peaks, quick: bool, only=None, tune: bool = False):
    """Every workload of the benchmark definition: time, TFLOPS, GB/s and
    fraction of roofline, with the dispatcher's kernel choice."""
    out = {}
    for key, name, fn, copies in SHAPES:
        if only is not None and key != only:
            continue
        # every copy is used at least once per graph, so the rotation is real;
        # ten replays of 20 calls keep a 4096^3 GEMM's window near 20 ms, short
        # of the power cap that a longer run settles into (the burst peak is
        # the reference)
        reps = max(20, copies)
        base = fn()
        gpus = [base.to("cuda") for _ in range(copies)]
        A, B, C = dg_views(gpus[0], dg)
        pl = dg.dg_plan(A, B, C, base.alpha, base.beta, base.scale_a is not None).as_dict()
        with NvmlClockPoller(torch.cuda.current_device()) as clk:
            t_graph, t_stream, host, spread = time_problem(gpus, dg, reps, warm=5)
        fl, by = flops_bytes(base)
        t_roof, bound = roofline_time_s(base, peaks)
        med = t_graph
        tuned = None
        if tune:
            # the library's autotuner on the same operands: the variant it keeps,
            # then the same graph-replay timing with that variant in force
            q = gpus[0]
            epi = dg.epilogue(q.bias, q.act) if (q.bias is not None or q.act != "none") else None
            st, res = dg.dg_autotune(A, B, C, q.alpha, q.beta, q.scale_a, q.scale_b, epi, None, 5)
            assert st == dg.DG_OK, dg.status_string(st)
            t_tuned, _, _, _ = time_problem(gpus, dg, reps, warm=5)
            chosen = res.plan.as_dict()
            tuned = {"us": t_tuned * 1e6, "frac_of_roofline": t_roof / t_tuned, "candidates": res.candidates,
                     "trial_us_rule": res.default_us, "trial_us_best": res.best_us,
                     "plan": {k: chosen[k] for k in ("kind_name", "block_n", "split_k", "cta_pair", "stream_k_tiles",
                                                     "gather_cluster", "epi_tma_store", "stages", "grid")}}
            dg.dg_tune_clear()
        p10, p90 = spread
        out[name] = {"kernel": pl["kind_name"], "us": med * 1e6, "us_p10": p10 * 1e6, "us_p90": p90 * 1e6,
                     "calls_timed": 10 * reps, "us_stream": t_stream * 1e6,
                     "host_us_per_call": host * 1e6,
                     "tflops": fl / med / 1e12, "gbs": by / med / 1e9, "bound": bound,
                     "roofline_us": t_roof * 1e6, "frac_of_roofline": t_roof / med,
                     "tiles": {k: pl[k] for k in ("block_n", "block_k", "split_k", "swap_ab", "p_gather", "grid")},
                     "timing": ("CUDA-graph replay of the calls, median per call over ten replays (device "
                                "time); us_stream: back-to-back stream calls"),
                     "l2": (f"{copies} rotating input copies, {copies * by / 1e6:.0f} MB"
                            if copies > 1 else "single copy (L2-resident)"),
                     "clocks": clk.summary()}
        if tuned is not None:
            out[name]["autotuned"] = tuned
        del gpus
        torch.cuda.empty_cache()
    return out


def run_one_shape(args):
    torch.cuda.set_device(0)
    import tcgen05_tmem_gemm_b200 as dg

    if args.max_split:
        dg.dg_set_option(dg.DG_OPT_MAX_SPLIT_K, args.max_split)
    if args.stream_k >= 0:
        dg.dg_set_option(dg.DG_OPT_STREAM_K, args.stream_k)
    if args.early_launch >= 0:
        dg.dg_set_option(dg.DG_OPT_EARLY_LAUNCH, args.early_launch)

    res = per_shape(dg, load_peaks(), True, only=args.shape, tune=args.autotune)
    out = {"shape": args.shape, **res}
    if args.trace:
        # one more call with CTA 0's phase timestamps (SM cycles from kernel entry)
        buf = torch.zeros(64, dtype=torch.int64, device="cuda")
        key = [k for k in SHAPES if k[0] == args.shape][0]
        prob = key[2]().to("cuda")
        dg.dg_set_option(dg.DG_OPT_TRACE, buf.data_ptr())
        A, B, C = dg_views(prob, dg)
        assert dg.dg_gemm(A, B, C, prob.alpha, prob.beta, prob.scale_a, prob.scale_b) == dg.DG_OK
        torch.cuda.synchronize()
        dg.dg_set_option(dg.DG_OPT_TRACE, 0)
        t = buf.cpu().tolist()
        t0 = t[0]
        out["trace_cycles"] = {i: (v - t0) for i, v in enumerate(t) if v}
    print(json.dumps(out), flush=True)


def run_dg(args):
    world, rank, local = dist_setup()
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    import tcgen05_tmem_gemm_b200 as dg

    if args.early_launch >= 0:
        dg.dg_set_option(dg.DG_OPT_EARLY_LAUNCH, args.early_launch)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    # graphs are captured on side streams; every call of the step uses them
    stream = torch.cuda.Stream()   # x*W
    side = torch.cuda.Stream()     # x*K^T, concurrent with x*W

    # ---- the step's data: three rotating copies of W and K, one x
    gv = W.cfg_gemv()
    gk = W.cfg_gemv_kt()
    step_bytes = flops_bytes(gv)[1] + flops_bytes(gk)[1]
    copies = []
    for _ in range(ROTATE):
        a = gv.to(dev)
        b = W.Problem(gk.name, a.A, gk.B.to(dev), gk.C.to(dev))  # x shared by both products
        copies.append((a, b, dg_views(a, dg), dg_views(b, dg)))
    torch.cuda.synchronize()

    # A step is the two dg_gemm calls.  They are independent (both read x,
    # each writes its own output), so x*K^T runs on a second stream beside
    # x*W: the 1 MB x*K^T is launch-bound and fits on the SMs next to the two
    # x*W blocks each SM holds.  The timed region replays CUDA graphs of the
    # calls (captured once; the host launch cost of a call does not reach the
    # device timeline) in units of UNIT steps: the unit's x*K^T calls on the
    # side stream, forked from and joined back into the main stream, and its
    # x*W calls on the main stream, bracketed by CUDA events (the roofline's
    # kernel timing covers every x*W launch of the timed region).  UNIT is a
    # multiple of ROTATE, so every unit starts on copy 0.
    UNIT = 16 * ROTATE

    def step(i):
        a, b, va, vb = copies[i % ROTATE]
        st1 = dg.dg_gemm(*va, 1.0, 0.0, None, None, stream)
        st2 = dg.dg_gemm(*vb, 1.0, 0.0, None, None, stream)
        return st1 | st2

    for i in range(args.warmup):
        assert step(i) == 0
    torch.cuda.synchronize()
    assert dg.dg_sync_status(stream) == dg.DG_OK

    def capture(which, n, s):
        """A CUDA graph of n x*W (which=2) or x*K^T (which=3) calls over the
        rotating copies, captured on stream s, and the number of kernels it launches."""
        g = torch.cuda.CUDAGraph()
        n0 = dg.dg_launch_count()
        with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
            for i in range(n):
                assert dg.dg_gemm(*copies[i % ROTATE][which], 1.0, 0.0, None, None, s) == 0
        return g, dg.dg_launch_count() - n0

    graphs = {}
    units = []
    left = args.steps
    while left > 0:
        n = min(UNIT, left)
        if n not in graphs:
            graphs[n] = (capture(2, n, stream), capture(3, n, side))
        units.append(n)
        left -= n
    torch.cuda.synchronize()
    assert dg.dg_sync_status(stream) == dg.DG_OK

    def run_units(evs):
        # the unit's x*W graph is submitted first, so the GPU starts on it at
        # once while the host submits the x*K^T graph; the side stream waits
        # only for the unit's start (the fork event), not for x*W
        launches = 0
        for u, n in enumerate(units):
            (gw, nw), (gk, nk) = graphs[n]
            fork = torch.cuda.Event()
            join = torch.cuda.Event()
            fork.record(stream)
            if evs is not None:
                evs[u][0].record(stream)
            gw.replay()
            if evs is not None:
                evs[u][1].record(stream)
            side.wait_event(fork)
            with torch.cuda.stream(side):
                gk.replay()
            join.record(side)
            stream.wait_event(join)
            launches += nw + nk
        return launches

    # the clock sampler starts first: the warm replay then runs right before
    # the timed region, so the GPU does not idle into it (an idle GPU enters
    # the timed region with its clocks and memory still waking up)
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in units]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        run_units(None)  # warm replay of every graph (untimed)
    barrier(world)
    torch.cuda.synchronize()
    w0 = time.time()
    with torch.cuda.stream(stream):
        hold_gpu()
        t_start.record(stream)
        launches = run_units(evs)
        t_end.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    barrier(world)
    time.sleep(0.25)
    assert dg.dg_sync_status(stream) == dg.DG_OK
    elapsed = t_start.elapsed_time(t_end) * 1e-3
    elapsed_max = max_over_ranks(elapsed, world, dev)
    value = whole_job_value(step_bytes, args.steps, world, elapsed_max)
    gemv_total = sum(a.elapsed_time(b) * 1e-3 for a, b in evs)
    gemv_avg = gemv_total / args.steps  # every x*W launch of the timed region is inside a bracket
    gemv_bytes = flops_bytes(gv)[1]
    achieved = gemv_bytes / gemv_avg / 1e9
    peak_hbm = peaks["hbm_gbs"]
    clocks = sampler.summary(w0, w1)

    # ---- the same kernel over a long window: at least 1000 back-to-back x*W
    # launches (graph replays of UNIT calls), bracketed by CUDA events on its
    # stream, with its own clock samples.  A short timed region weighs its
    # first launch heavily; this one does not.
    (gw_long, nw_long), _ = graphs.get(UNIT) or (capture(2, UNIT, stream), None)
    reps_long = -(-1000 // UNIT)
    with torch.cuda.stream(stream):
        gw_long.replay()
    torch.cuda.synchronize()
    la, lb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    l0 = time.time()
    with torch.cuda.stream(stream):
        hold_gpu()
        la.record(stream)
        for _ in range(reps_long):
            gw_long.replay()
        lb.record(stream)
    torch.cuda.synchronize()
    l1 = time.time()
    time.sleep(0.25)
    sampler.stop()
    assert dg.dg_sync_status(stream) == dg.DG_OK
    long_launches = reps_long * UNIT
    long_avg = la.elapsed_time(lb) * 1e-3 / long_launches
    long_achieved = gemv_bytes / long_avg / 1e9
    traffic = kernel_traffic("gemv.cu", "gemv_n_decode_4096x14336.txt")

    result = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_max / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "bytes_per_step": step_bytes,
                   "l2": f"inputs rotate through {ROTATE} copies of W and K (352 MB > 126 MB L2)",
                   "launch": f"two dg_gemm calls per step, replayed from CUDA graphs in units of {UNIT} steps: "
                             f"the unit's x*K^T calls on a second stream forked from the first, its x*W "
                             f"calls on the first, bracketed by CUDA events",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "kernel": "gemv_n (x*W, 117 MB of W)", "achieved": achieved,
                     "timed_launches": args.steps,
                     "peak": peak_hbm, "unit": "GB/s", "frac": achieved / peak_hbm,
                     "traffic": traffic, "algorithmic_bytes": gemv_bytes, "avg_launch_us": gemv_avg * 1e6,
                     "peak_source": f"{peaks['source']} hbm_gbs (STREAM-style copy)",
                     "long_window": {"launches": long_launches, "avg_launch_us": long_avg * 1e6,
                                     "achieved": long_achieved, "frac": long_achieved / peak_hbm,
                                     "clocks": sampler.summary(l0, l1)}},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if rank == 0:
        if not args.skip_cpu:
            result["e2e"] = e2e(dg, gv, gk, dev, stream, max(3, min(args.steps, 20)))
        if not args.no_per_shape:
            result["per_shape"] = per_shape(dg, peaks, args.quick, tune=args.autotune)
        if not args.skip_cpu:
            result["cpu_baseline"] = cpu_baseline(args.quick)
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist

        barrier(world)
        dist.destroy_process_group()


def run_shard(args):
    """The decode step split over the ranks by columns (strong scaling): x is
    replicated, rank r holds its column block of W and of K^T (rows of K),
    computes its blocks of y = x W and z = x K^T with dg_gemm on its own GPU,
    and one NCCL all-gather per output assembles the whole y and z on every
    rank.  The job is one decode step's bytes per step, whatever the number of
    ranks; the time is the slowest rank's."""
    import datetime

    import torch.distributed as dist

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    if "MASTER_PORT" not in os.environ:
        import socket

        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            os.environ["MASTER_PORT"] = str(sk.getsockname()[1])
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    import tcgen05_tmem_gemm_b200 as dg
    from tcgen05_tmem_gemm_b200 import shard

    dev = torch.device("cuda", local)
    gv, gk = W.cfg_gemv(), W.cfg_gemv_kt()
    step_bytes = flops_bytes(gv)[1] + flops_bytes(gk)[1]
    N, NK = gv.N, gk.N
    x = gv.A.base.to(dev)
    kmat = gk.B.base  # [128, 4096] row-major; K^T's columns are its rows
    blocks = []
    for _ in range(ROTATE):
        wb = shard.local_block(gv.B.base, rank, world, dev)
        kb = shard.local_block(kmat.t(), rank, world, dev)     # [4096, width] block of K^T
        blocks.append((wb, kb))
    yb = torch.zeros(1, shard.shard_width(N, world), dtype=torch.bfloat16, device=dev)
    zb = torch.zeros(1, shard.shard_width(NK, world), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    n_launch = [0]

    def step(i):
        wb, kb = blocks[i % ROTATE]
        n0 = dg.dg_launch_count()
        shard.gemm_block(x, wb, yb, N, rank, world, stream=stream)
        shard.gemm_block(x, kb, zb, NK, rank, world, stream=stream)
        n_launch[0] += dg.dg_launch_count() - n0
        return shard.assemble(yb, N), shard.assemble(zb, NK)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    n_launch[0] = 0
    a.record()
    for i in range(args.steps):
        y, z = step(i)
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    assert dg.dg_sync_status() == dg.DG_OK
    elapsed_max = max_over_ranks(a.elapsed_time(b) * 1e-3, world, dev)
    # the assembled outputs are the single-GPU products (same kernels per column block)
    ref_y = torch.empty(1, N, dtype=torch.bfloat16, device=dev)
    dg.gemm(x, gv.B.base.to(dev), ref_y)
    ok = bool(torch.allclose(y.float(), ref_y.float(), rtol=2e-2, atol=1e-3))
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": step_bytes * args.steps / elapsed_max / 1e9, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_max / args.steps * 1e3, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD + "; split by columns of W and K^T over the ranks",
                       "parallelism": f"column shards x{world}, NCCL all-gather of y and z",
                       "launch": "eager dg_gemm calls and all-gathers on the current stream"},
            "gpu_launches": int(n_launch[0]), "assembled_matches_single_gpu": ok}), flush=True)
    dist.destroy_process_group()


def e2e(dg, gv, gk, dev, stream, steps):
    """Same step through dg_gemm with host buffers: pinned host -> device copies
    of x, W and K, both products, device -> host copies of both outputs, every
    step, timed with CUDA events."""
    hx = gv.A.base.pin_memory()
    hw = gv.B.base.pin_memory()
    hk = gk.B.base.pin_memory()
    hy1 = torch.empty_like(gv.C.base).pin_memory()
    hy2 = torch.empty_like(gk.C.base).pin_memory()
    dx = torch.empty_like(hx, device=dev)
    dw = torch.empty_like(hw, device=dev)
    dk = torch.empty_like(hk, device=dev)
    dy1 = torch.empty_like(hy1, device=dev)
    dy2 = torch.empty_like(hy2, device=dev)
    vx = dg.make_view(dx.data_ptr(), gv.A.shape, gv.A.stride, 1, "bf16")
    vw = dg.make_view(dw.data_ptr(), gv.B.shape, gv.B.stride, 1, "bf16")
    vk = dg.make_view(dk.data_ptr(), gk.B.shape, gk.B.stride, 1, "bf16")
    vy1 = dg.make_view(dy1.data_ptr(), gv.C.shape, gv.C.stride, 1, "bf16")
    vy2 = dg.make_view(dy2.data_ptr(), gk.C.shape, gk.C.stride, 1, "bf16")

    def one():
        dx.copy_(hx, non_blocking=True)
        dw.copy_(hw, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        assert dg.dg_gemm(vx, vw, vy1, 1.0, 0.0, None, None, stream) == dg.DG_OK
        assert dg.dg_gemm(vx, vk, vy2, 1.0, 0.0, None, None, stream) == dg.DG_OK
        hy1.copy_(dy1, non_blocking=True)
        hy2.copy_(dy2, non_blocking=True)

    torch.cuda.synchronize()
    with torch.cuda.stream(stream):  # copies and products in one stream order
        for _ in range(2):
            one()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            one()
        b.record(stream)
        torch.cuda.synchronize()
    t = a.elapsed_time(b) * 1e-3 / steps
    step_bytes = flops_bytes(gv)[1] + flops_bytes(gk)[1]
    h2d = (hx.numel() * hx.element_size() + hw.numel() * hw.element_size() + hk.numel() * hk.element_size())
    d2h = hy1.numel() * hy1.element_size() + hy2.numel() * hy2.element_size()
    return {"value": step_bytes / t / 1e9, "unit": "GB/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": t * 1e3, "steps": steps}


# ---------------------------------------------------------- the CPU oracle

def _oracle_step(orc, gv_s, gk, threads):
    orc.gemm(gv_s, want_bound=False, nthreads=threads)
    orc.gemm(gk, want_bound=False, nthreads=threads)


def _column_sample(gv: W.Problem, cols: int) -> W.Problem:
    """x * W[:, :cols] as a view of the same W (no copy)."""
    B = W.Operand(gv.B.base, (gv.K, cols), gv.B.stride, 1, gv.B.dtype)
    C = W.row_major(torch.empty(1, cols, dtype=torch.bfloat16), "bf16")
    return W.Problem(gv.name + f"_cols{cols}", gv.A, B, C)


def _affinity_cores():
    return sorted(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else list(range(os.cpu_count()))


def cpu_baseline_worker(quick: bool, threads: int, target_s: float = 12.0):
    """The FP64 oracle, as it stands, timed in this process: repeated decode
    steps (x*W and x*K^T) on every core of the affinity set for about
    `target_s` seconds, and the small 128x128x256 GEMM on one core.  Run under
    taskset by cpu_baseline(); touches no GPU."""
    import oracle

    orc = oracle.default()
    gv, gk = W.cfg_gemv(), W.cfg_gemv_kt()
    step_bytes = flops_bytes(gv)[1] + flops_bytes(gk)[1]
    t0 = time.perf_counter()
    _oracle_step(orc, gv, gk, threads)
    one = time.perf_counter() - t0
    reps = 1 if quick else max(1, int(target_s / max(one, 1e-3)))
    t0 = time.perf_counter()
    for _ in range(reps):
        _oracle_step(orc, gv, gk, threads)
    t = (time.perf_counter() - t0) / reps
    small = W.cfg_small()
    fl_small = flops_bytes(small)[0]
    orc.gemm(small, want_bound=False, nthreads=1)
    n_small = 20
    t0 = time.perf_counter()
    for _ in range(n_small):
        orc.gemm(small, want_bound=False, nthreads=1)
    t_small = (time.perf_counter() - t0) / n_small
    return {"value": step_bytes / t / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{reps} full decode steps (x*W 1x4096x14336 and x*K^T 1x4096x128), FP64, "
                      f"{t:.3f} s per step, OpenMP threads bound to the affinity cores",
            "small_1core": {"workload": "small F16 128x128x256 -> FP32", "s_per_call": t_small,
                            "gflops": fl_small / t_small / 1e9, "cores": 1}}


def cpu_baseline(quick: bool):
    """cpu_baseline_worker in a child process pinned with taskset to the cores
    this process may run on (OpenMP threads bound one per core)."""
    cores = _affinity_cores()
    env = dict(os.environ, OMP_PROC_BIND="close", OMP_PLACES="cores", CUDA_VISIBLE_DEVICES="")
    # the parent counts the cores: in the child, the OpenMP runtime binds the
    # initial thread to one core as soon as it is loaded
    cmd = [sys.executable, os.path.abspath(__file__), "--cpu-baseline-worker", str(len(cores))] + \
        (["--quick"] if quick else [])
    if shutil.which("taskset"):
        cmd = ["taskset", "-c", ",".join(str(c) for c in cores)] + cmd
    r = subprocess.run(cmd, capture_output=True, text=True, env=env, timeout=600)
    if r.returncode != 0:
        return {"value": None, "unit": "GB/s", "cores": len(cores), "kind": "oracle",
                "sample": "failed: " + (r.stderr.strip().splitlines() or ["?"])[-1]}
    out = json.loads(r.stdout.strip().splitlines()[-1])
    out["pinning"] = f"taskset -c {cores[0]}-{cores[-1]} ({len(cores)} cores)" if shutil.which("taskset") \
        else "no taskset on this host"
    return out


def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return  # the oracle runs once, on rank 0; the other ranks have no work
    import oracle

    orc = oracle.default()
    threads = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    gv, gk = W.cfg_gemv(), W.cfg_gemv_kt()
    # size each step's sample so the whole run stays within about two minutes
    t0 = time.perf_counter()
    _oracle_step(orc, _column_sample(gv, 1024), gk, threads)
    per_col = (time.perf_counter() - t0) / 1024
    budget = 120.0 / max(1, args.steps + args.warmup)
    cols = int(min(gv.N, max(256, budget / max(per_col, 1e-9))))
    cols -= cols % 8
    sample = _column_sample(gv, cols)
    step_bytes = flops_bytes(sample)[1] + flops_bytes(gk)[1]
    for _ in range(args.warmup):
        _oracle_step(orc, sample, gk, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(orc, sample, gk, threads)
    t = time.perf_counter() - t0
    value = step_bytes * args.steps / t / 1e9
    desc = (f"per step: x*W[:, :{cols}] (of 14336 columns) and x*K^T 1x4096x128, FP64 oracle")
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": desc}, "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["dg", "reference"], default="dg")
    ap.add_argument("--quick", action="store_true", help="fewer repetitions in the side measurements")
    ap.add_argument("--no-per-shape", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true", help="no CPU baseline and no e2e leg (profiling runs)")
    ap.add_argument("--shape", default=None,
                    help="time only this per-shape workload (small, gemv, gemv_kt, thin, square_bf16, "
                         "square_e4m3, strided, square_bf16_gelu, thin_gelu, strided_nchw_out) and print its line")
    ap.add_argument("--max-split", type=int, default=0, help="with --shape: cap the tensor-core split-K")
    ap.add_argument("--stream-k", type=int, default=-1, help="with --shape: 0 or 1 turns the Stream-K tail off or on")
    ap.add_argument("--trace", action="store_true", help="with --shape: phase timestamps of CTA 0")
    ap.add_argument("--cpu-baseline-worker", type=int, default=0, help=argparse.SUPPRESS)
    ap.add_argument("--shard", action="store_true",
                    help="the decode step split over the ranks by columns, with NCCL all-gathers (strong scaling)")
    ap.add_argument("--autotune", action="store_true",
                    help="per-shape rows also report dg_autotune's chosen variant and its time")
    ap.add_argument("--early-launch", type=int, default=-1,
                    help="programmatic dependent launch policy (0 off, 1 at kernel start, 2 near the end, "
                         "3 the library's per-kernel default)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.cpu_baseline_worker:
        print(json.dumps(cpu_baseline_worker(args.quick, args.cpu_baseline_worker)), flush=True)
    elif args.impl == "reference":
        run_reference(args)
    elif args.shape:
        run_one_shape(args)
    elif args.shard:
        run_shard(args)
    else:
        run_dg(args)


if __name__ == "__main__":
    main()
