"""Benchmark of the B200 MACAQ W4A4 MXFP4 linear.

One step = one pass of the whole hot path over one batch of the headline
workload: the dense M=128 MACAQ linear over the five Qwen3-0.6B-shaped
projections (K, N) in {(1024,2048), (1024,1024), (2048,1024), (1024,3072),
(3072,1024)}, bf16 activations with 1% outlier channels x20, MXFP4 weights
prepared offline, BF16 output.  Inputs are seeded and synthetic (synth).

Timing: W warm-up steps, then exactly K steps, each preceded (outside the
timed interval) by a 256 MiB write that flushes the 126 MB L2; device time from
CUDA events on the launching stream; barrier + synchronize around the timed
region; max over ranks.  N > 1 GPUs run independent replicas (the layer needs
no exchange), so scaling is weak.

Also reported: e2e (the same calls with the activations copied from pinned
host memory and the outputs copied back inside the timed interval), the
roofline of the dominant kernel, the clocks seen during the timed region, and,
on one GPU, the per-workload table of all five workloads (us/call, TFLOPS,
fraction of roofline, ALU bound of the activation prologue, unfused ablation,
plain MXFP4, bias + GELU_TANH, eager calls allocating y), the D calibration
times, and the CPU oracle on a bounded sample (all cores, one thread, and a
decoded binary64 GEMM).

`--impl reference` times the CPU oracle (the reference arm) on the same
workload and metric.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "fused W4A4 MXFP4 TFLOPS & µs/call vs FP4/HBM roofline, dense M=16/128/4096 + grouped"
UNIT = "TFLOPS"
WORKLOAD = "dense M=128 MACAQ W4A4 MXFP4 linear x 5 Qwen3-0.6B projections (K,N)=" \
           "(1024,2048),(1024,1024),(2048,1024),(1024,3072),(3072,1024)"
FP4_NOMINAL_TFLOPS = 9000.0   # NVIDIA's published dense FP4 figure for B200
L2_FLUSH_BYTES = 256 << 20


def kernel_source_hash() -> str:
    """Hash of the kernel sources with comments and blank lines removed, so that a
    profile stays matched to its kernels across edits of prose only."""
    import hashlib
    import re
    h = hashlib.sha256()
    d = os.path.join(ROOT, "w4a4_mxfp4_quantize_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"(?m)^\s*//.*$", "", text)        # whole-line comments
        text = re.sub(r"(?m)\s+//[^\"\n]*$", "", text)   # trailing comments (not inside strings)
        text = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
        h.update(f.encode() + b"\0" + text.encode())
    return h.hexdigest()[:16]


def profiled_traffic(summary: str):
    """DRAM bytes per launch recorded by an ncu summary under profiles/, or None
    when the kernels have changed since those counters were taken."""
    path = os.path.join(ROOT, "profiles", summary)
    try:
        fields = dict(line.split(":", 1) for line in open(path) if ":" in line and not line.startswith(("#", "|", " ")))
        if fields.get("kernel_source_sha256_16", "").strip() != kernel_source_hash():
            return None
        return float(fields["dram_bytes_per_launch"].strip())
    except Exception:
        return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        hi = [v for v in sm if v > 0.5 * max(sm)]
        return {"sm_mhz": statistics.median(hi), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def x_dev(xbits, device):
    return torch.from_numpy(np.ascontiguousarray(xbits).view(np.int16)).view(torch.bfloat16).to(device)


def f32(a, device):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


class Prepared:
    """A problem with its weights prepared on the device (untimed, offline) and
    its output and workspace allocated up front (so calls can be captured in a
    CUDA graph)."""

    def __init__(self, p: synth.Problem, device, mq):
        self.p = p
        self.x = x_dev(p.x, device)
        self.x_host = torch.from_numpy(np.ascontiguousarray(p.x).view(np.int16)).view(torch.bfloat16).pin_memory()
        self.D = f32(p.D if p.E > 1 else p.D[0], device)
        W = f32(p.W, device)
        self.Wq, self.Ws = mq.prepare_weights(W, f32(p.D, device))
        del W
        self.y = torch.empty((p.M, p.N), dtype=torch.bfloat16, device=device)
        self.y_host = torch.empty((p.M, p.N), dtype=torch.bfloat16).pin_memory()
        self.gl = None if p.group_list is None else torch.from_numpy(p.group_list.astype(np.int64)).to(device)
        nb = mq.workspace_bytes(p.M, p.N, p.K, p.E)
        self.ws = torch.zeros(nb, dtype=torch.uint8, device=device) if nb else None
        nu = mq.unfused_workspace_bytes(p.M, p.K) if p.E == 1 else 0
        self.ws_unfused = torch.zeros(nu, dtype=torch.uint8, device=device) if nu else None

    def run(self, mq, stream=None):
        if self.gl is None:
            mq.dense_mm(self.x, self.D, self.Wq, self.Ws, self.p.N, out=self.y, stream=stream, ws=self.ws)
        else:
            mq.grouped_mm(self.x, self.D, self.Wq, self.Ws, self.gl, self.p.group_list_type, self.p.N,
                          out=self.y, stream=stream, ws=self.ws)

    def run_alloc(self, mq, stream=None, alt: bool = False):
        """The call as made without a preallocated output: the binding allocates y
        (torch.empty through the caching allocator) on every call.  alt takes a
        second, distinct activation buffer holding the same values."""
        if alt and getattr(self, "x_alt", None) is None:
            self.x_alt = self.x.clone()
        x = self.x_alt if alt else self.x
        if self.gl is None:
            return mq.dense_mm(x, self.D, self.Wq, self.Ws, self.p.N, stream=stream)
        return mq.grouped_mm(x, self.D, self.Wq, self.Ws, self.gl, self.p.group_list_type, self.p.N,
                             stream=stream)

    def run_type2(self, mq, stream=None):
        """The grouped call with the same groups written as group_list_type 2:
        [E, 2] rows of (group index, group size) in expert order."""
        if getattr(self, "gl2", None) is None:
            rows = np.stack([np.arange(self.p.E), self.p.counts], axis=1).astype(np.int64)
            self.gl2 = torch.from_numpy(rows).to(self.y.device)
        mq.grouped_mm(self.x, self.D, self.Wq, self.Ws, self.gl2, 2, self.p.N, out=self.y, stream=stream,
                      ws=self.ws)

    def run_epilogue(self, mq, stream=None):
        """The same call with an fp32 bias and GELU_TANH (npu_grouped_matmul's bias and act_type)."""
        if getattr(self, "bias", None) is None:
            rows = 1 if self.gl is None else self.p.E
            b = np.random.default_rng(3).standard_normal((rows, self.p.N)).astype(np.float32) * 0.5
            self.bias = f32(b[0] if self.gl is None else b, self.y.device)
        if self.gl is None:
            mq.dense_mm(self.x, self.D, self.Wq, self.Ws, self.p.N, out=self.y, stream=stream, ws=self.ws,
                        bias=self.bias, act_type=mq.ACT_GELU_TANH)
        else:
            mq.grouped_mm(self.x, self.D, self.Wq, self.Ws, self.gl, self.p.group_list_type, self.p.N,
                          out=self.y, stream=stream, ws=self.ws, bias=self.bias, act_type=mq.ACT_GELU_TANH)

    def run_fp8(self, mq, stream=None):
        """The same call with the FP8 (E4M3) output (per-tensor output scale 1)."""
        if getattr(self, "y8", None) is None:
            self.y8 = torch.empty((self.p.M, self.p.N), dtype=torch.uint8, device=self.y.device)
            nu = mq.unfused_workspace_bytes(self.p.M, self.p.K) if self.gl is None else 0
            self.ws8 = torch.zeros(nu, dtype=torch.uint8, device=self.y.device) if nu else self.ws
        if self.gl is None:
            mq.dense_mm_fp8(self.x, self.D, self.Wq, self.Ws, self.p.N, 1.0, out=self.y8, stream=stream, ws=self.ws8)
        else:
            mq.grouped_mm_fp8(self.x, self.D, self.Wq, self.Ws, self.gl, self.p.group_list_type, self.p.N, 1.0,
                              out=self.y8, stream=stream, ws=self.ws8)

    def run_unfused(self, mq, stream=None):
        mq.unfused_dense_mm(self.x, self.D, self.Wq, self.Ws, self.p.N, out=self.y, stream=stream,
                            ws=self.ws_unfused)

    def prepare_plain(self, mq, device):
        """Plain MXFP4 weights of the same W (the native baseline)."""
        W = f32(self.p.W, device)
        self.Wq_plain, self.Ws_plain = mq.prepare_weights_plain(W)
        del W

    def run_plain(self, mq, stream=None):
        if self.gl is None:
            mq.dense_mm_plain(self.x, self.Wq_plain, self.Ws_plain, self.p.N, out=self.y, stream=stream,
                              ws=self.ws)
        else:
            mq.grouped_mm_plain(self.x, self.Wq_plain, self.Ws_plain, self.gl, self.p.group_list_type, self.p.N,
                                out=self.y, stream=stream, ws=self.ws)


def layer_nmse(p: synth.Problem, y: torch.Tensor, rows: np.ndarray) -> float:
    """Normalised squared error of output rows against the unquantised layer
    x . W^T in float64 (numpy; the rows' own experts for grouped problems)."""
    yb = y[torch.from_numpy(rows).to(y.device)].float().cpu().numpy().astype(np.float64)
    x = synth.bf16_bits_to_f32(p.x[rows]).astype(np.float64)
    if p.E == 1:
        ref = x @ p.W[0].astype(np.float64).T
    else:
        g = np.searchsorted(np.cumsum(p.counts), rows, side="right")
        ref = np.stack([x[i] @ p.W[g[i]].astype(np.float64).T for i in range(rows.size)])
    return float(np.sum((yb - ref) ** 2) / np.sum(ref ** 2))


def capture(fn, stream):
    """Capture fn() (library calls on the current stream) into a CUDA graph."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()  # warm-up outside capture
    stream.synchronize()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def _trim(t):
    t = np.sort(np.asarray(t))
    cut = len(t) // 10
    q = np.percentile(t, [25, 75])
    return float(np.mean(t[cut:len(t) - cut])), float(q[1] - q[0])


def time_graph(g, flush, stream, reps: int, warm: int = 3, cold: bool = True):
    """Mean (10% trimmed at each end) and IQR of the device time (us) of one graph
    replay, CUDA events on `stream` around the replay; the L2 flush (when `cold`)
    runs before the start event.  Durations measured this way include the graph's
    launch and completion, and for one-call graphs they cluster near multiples of
    about 2.05 us whatever the work inside (per-CTA clock stamps inside the
    kernels show no such grid), so a replay that always follows the same flush
    would always land the same way on that grid.  A GPU-side spin of a seeded
    random 0-4,000 cycles (about 0-2 us, outside the timed interval) before each
    start event spreads the start phase: the mean is then unbiased."""
    rng = np.random.default_rng(12345)
    with torch.cuda.stream(stream):
        for _ in range(warm):
            g.replay()
        evs = []
        for _ in range(reps):
            if cold:
                flush()
            torch.cuda._sleep(int(rng.integers(0, 4000)))
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            evs.append((a, b))
    stream.synchronize()
    return _trim([a.elapsed_time(b) * 1e3 for a, b in evs])


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------
def cpu_oracle_sample(problems, budget_s: float = 12.0, rows: int = 4, prepared=None, nthreads: int = 0):
    """The oracle's hot path (activation quantisation + exact GEMM) on `rows`
    rows of every problem, weights prepared beforehand (offline, untimed, as
    on the GPU), on `nthreads` threads (0: all host cores); returns (TFLOPS,
    seconds, threads, description, prepared)."""
    import oracle
    if prepared is None:
        prepared = [oracle.quantize_weights(p.W[0], p.D[0]) for p in problems]
    threads = nthreads if nthreads > 0 else oracle.num_threads()
    t0 = time.perf_counter()
    flops = 0.0
    n = 0
    while True:
        for p, (qw, sw) in zip(problems, prepared):
            qa, sa = oracle.quantize_act(p.x[:rows], p.D[0], threads)
            oracle.gemm(qa, sa, qw, sw, threads)
            flops += 2.0 * rows * p.N * p.K
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 1000:
            break
    return flops / el / 1e12, el, threads, (
        f"{rows} of {problems[0].M} rows of each of the {len(problems)} projections, {n} passes "
        "(activation quantisation + exact block-scaled GEMM; weights prepared beforehand)"), prepared


def cpu_oracle_detail(problems, prepared, cores: int, budget_s: float = 4.0) -> dict:
    """Two more host-side figures beside the all-core oracle: the same hot path
    on one thread, and a dequantised binary64 GEMM (activation quantisation,
    both operands decoded to their values, one BLAS matmul, the 2^-5 scale;
    weights decoded beforehand) on 4 rows of every problem: the exact GEMM is a
    correctness tool, the decoded one the speed a plain CPU implementation of
    the same arithmetic reaches."""
    import oracle
    v1, el1, _, _, _ = cpu_oracle_sample(problems, budget_s=budget_s, rows=1, prepared=prepared, nthreads=1)
    p0 = problems[0]
    oracle.quantize_act(p0.x[:1], p0.D[0], cores)  # back to every core for later oracle calls
    wdec = [oracle.dequantize(qw, sw) for (qw, sw) in prepared]
    rows = 4
    t0 = time.perf_counter()
    flops, n = 0.0, 0
    while True:
        for p, w in zip(problems, wdec):
            qa, sa = oracle.quantize_act(p.x[:rows], p.D[0], cores)
            _ = (oracle.dequantize(qa, sa) @ w.T) * 2.0 ** -5
            flops += 2.0 * rows * p.N * p.K
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 1000:
            break
    return {
        "single_thread": {"value": v1, "unit": UNIT, "cores": 1, "seconds": el1,
                          "sample": "1 row of each projection, exact GEMM"},
        "dequant_f64_gemm": {"value": flops / el / 1e12, "unit": UNIT, "cores": cores, "seconds": el,
                             "sample": f"{rows} rows of each projection, {n} passes, decoded operands, BLAS matmul"},
    }


def max_over_ranks(total_ms: float, dist, device) -> float:
    """The job's time: the largest of the ranks' timed totals (every rank takes part)."""
    if dist is None:
        return total_ms
    t = torch.tensor([total_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flops_step: float, steps: int, total_ms: float) -> float:
    """Whole-job throughput: every rank runs the same step on its own data
    (replicas), so the job does world x the step's FLOPs in the slowest rank's time."""
    return world * flops_step * steps / (total_ms * 1e-3) / 1e12


def run_reference(args, rank, world):
    if rank != 0:
        return
    problems = synth.config(1)
    steps = []
    prepared = None
    for _ in range(args.warmup):
        *_, prepared = cpu_oracle_sample(problems, budget_s=0.0, rows=1, prepared=prepared)
    for _ in range(args.steps):
        v, el, cores, sample, _ = cpu_oracle_sample(problems, budget_s=min(10.0, 120.0 / max(1, args.steps)),
                                                    rows=4, prepared=prepared)
        steps.append((v, el))
    value = statistics.median(v for v, _ in steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(el for _, el in steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "mxfp4(e2m1,e8m0)->exact->bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": 128 * world, "per_gpu_batch": 128,
                   "parallelism": f"replicas x{world}", "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-table", action="store_true", help="skip the per-workload table")
    ap.add_argument("--table-reps", type=int, default=30)
    ap.add_argument("--only", default=None,
                    help="CFG or CFG:IDX: only run these problems' calls --iters times (for profilers; no JSON)")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--unfused", action="store_true", help="with --only: the unfused ablation instead")
    ap.add_argument("--epilogue", action="store_true", help="with --only: the call with bias and GELU_TANH")
    args = ap.parse_args()
    if args.only is not None:
        run_only(args)
        return
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    if args.impl == "reference":
        run_reference(args, rank, world)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return

    import w4a4_mxfp4_quantize_b200 as mq
    mq.lib()  # fails loudly when the CUDA library is missing

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    stream = torch.cuda.Stream(device)
    hbm_gbs, bf16_tf, peak_kind = load_peaks()
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def flush():
        flush_buf.fill_(1)

    problems = [Prepared(p, device, mq) for p in synth.config(1)]
    # The five projections' activations and outputs live in one device buffer each
    # (every slice starts 16-byte aligned: M K and M N are multiples of 8), so that a
    # step moves its inputs and results with one copy per direction (e2e below).
    x_all = torch.empty(sum(pp.x.numel() for pp in problems), dtype=torch.bfloat16, device=device)
    y_all = torch.empty(sum(pp.y.numel() for pp in problems), dtype=torch.bfloat16, device=device)
    xo = yo = 0
    for pp in problems:
        nx, ny = pp.x.numel(), pp.y.numel()
        x_all[xo:xo + nx].copy_(pp.x.reshape(-1))
        pp.x = x_all[xo:xo + nx].view(pp.x.shape)
        pp.y = y_all[yo:yo + ny].view(pp.y.shape)
        xo, yo = xo + nx, yo + ny
    x_all_host = torch.cat([pp.x_host.reshape(-1) for pp in problems]).pin_memory()
    y_all_host = torch.empty(y_all.numel(), dtype=torch.bfloat16).pin_memory()
    torch.cuda.synchronize()
    flops_step = sum(pp.p.flops() for pp in problems)
    bytes_step = sum(pp.p.algorithmic_bytes() for pp in problems)

    def step():
        for pp in problems:
            pp.run(mq)

    step_graph = capture(step, stream)
    call_graphs = [capture(lambda pp=pp: pp.run(mq), stream) for pp in problems]

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush()
            step_graph.replay()
    stream.synchronize()

    # ---------------- timed region ----------------
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    step_ev = []
    phase = np.random.default_rng(54321)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            flush()
            torch.cuda._sleep(int(phase.integers(0, 4000)))  # start phase spread (time_graph)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            step_graph.replay()
            b.record(stream)
            step_ev.append((a, b))
    stream.synchronize()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clocks = sampler.stop()

    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    total_ms = max_over_ranks(sum(step_ms), dist, device)
    value = job_tflops(world, flops_step, args.steps, total_ms)
    ms_per_step = total_ms / args.steps

    # The dominant kernel is the only one launched in the timed region (one fused
    # launch per projection, back to back), so its average launch duration there
    # is the timed region divided by the launches in it (an upper bound: the
    # interval also holds the graph's own launch and completion, see launch_floor).
    # Standalone single-call graphs (L2 flushed before each) are reported beside
    # it; they carry the launch and completion of a one-kernel graph.
    per_call_us = [time_graph(g, flush, stream, max(args.steps, 30))[0] for g in call_graphs]
    try:  # supplementary: its failure must not cost the line
        floor = launch_floor(device, stream, flush, max(args.steps, 30))
    except Exception as e:  # noqa: BLE001
        floor = {"error": f"{type(e).__name__}: {e}"[:200]}
    launch_s = ms_per_step * 1e-3 / len(problems)
    achieved_gbs = bytes_step / len(problems) / launch_s / 1e9
    roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_gbs, "unit": "GB/s",
                "frac": achieved_gbs / hbm_gbs,
                "traffic": profiled_traffic("fused_small_kernel_dense_M128.md"),
                "traffic_unit": "DRAM bytes per launch (ncu, profiles/fused_small_kernel_dense_M128.md)",
                "peak_kind": f"{peak_kind} copy bandwidth (burst)",
                "kernel": "fused_small_kernel (one launch per projection)",
                "algorithmic_bytes_per_step": bytes_step, "launches_per_step": len(problems),
                "launch_us": launch_s * 1e6,
                "launch_us_from": "timed region / launches in it (the kernel is the only one launched there)",
                "launch_floor": floor}

    # ---------------- e2e: host buffers through the public API (eager calls) ----------------
    h2d = x_all_host.numel() * 2
    d2h = y_all_host.numel() * 2
    e2e_ms = []
    with torch.cuda.stream(stream):
        for it in range(args.warmup + args.steps):
            flush()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            x_all.copy_(x_all_host, non_blocking=True)  # the step's activations, pinned host -> device
            for pp in problems:
                pp.run(mq, stream)
            y_all_host.copy_(y_all, non_blocking=True)  # the step's outputs back to the host
            b.record(stream)
            if it >= args.warmup:
                e2e_ms.append((a, b))
    stream.synchronize()
    e2e_total = max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ms), dist, device)
    e2e = {"value": job_tflops(world, flops_step, args.steps, e2e_total), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "mode": "eager public-API calls, no graph; the five projections' inputs and outputs staged "
                   "contiguously in pinned host memory: one copy per direction per step"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "mxfp4(e2m1,e8m0)->f32->bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": 128 * world, "per_gpu_batch": 128,
                   "parallelism": f"replicas x{world}", "l2": "flushed (256 MiB write) before every timed step"},
        "us_per_call_single_graph": {pp.p.name: us for pp, us in zip(problems, per_call_us)},
        "timing": "CUDA graph of the step replayed; events on the launching stream",
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": len(problems) * args.steps,
        "clocks": clocks,
    }

    if rank == 0:
        if world == 1:
            # CPU oracle on the host cores (bounded sample), and the per-workload tables:
            # one GPU only (at N > 1 the other ranks would wait for them at the barrier)
            v, el, cores, sample, prepared = cpu_oracle_sample([pp.p for pp in problems], budget_s=12.0, rows=4)
            line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                                    "seconds": el}
            try:  # supplementary host figures: their failure must not cost the line
                line["cpu_baseline"].update(cpu_oracle_detail([pp.p for pp in problems], prepared, cores))
            except Exception as e:  # noqa: BLE001
                line["cpu_baseline"]["detail_error"] = f"{type(e).__name__}: {e}"[:200]
            if not args.no_table:
                line["per_workload"] = workload_table(mq, device, stream, flush, hbm_gbs, args.table_reps)
                line["calibration"] = calibration_table(mq, device, stream, flush, hbm_gbs, args.table_reps)
        print(json.dumps(line), flush=True)

    for pp in problems:
        del pp
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_only(args):
    """Run the calls of one workload (or one problem of it) a few times, with
    the L2 flushed before each, so that a profiler can capture them."""
    import w4a4_mxfp4_quantize_b200 as mq
    mq.lib()
    device = torch.device("cuda", 0)
    cfg, _, idx = args.only.partition(":")
    probs = synth.config(int(cfg))
    if idx:
        probs = [probs[int(idx)]]
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    for p in probs:
        pp = Prepared(p, device, mq)
        for _ in range(args.iters):
            flush_buf.fill_(1)
            if args.unfused:
                pp.run_unfused(mq)
            elif args.epilogue:
                pp.run_epilogue(mq)
            else:
                pp.run(mq)
        torch.cuda.synchronize()
        print("ran", p.name, flush=True)
        del pp


# Lane operations per activation element of the quantise-once prologue (scale by
# 1/D, Hadamard butterfly, block maximum, E8M0 and E2M1 encoding, packing, loads
# and stores): ncu counted 2,224,128 warp instructions for quant_tiles_kernel at
# M = 4096, K = 1024, i.e. x 32 lanes / (4096 x 1024) elements.
QUANT_LANE_OPS_PER_ELEMENT = 2224128 * 32 / (4096 * 1024)
SM_MAX_MHZ = 1965.0  # B200 clocks.max.sm


def alu_bound_us(rows: int, K: int, sms: int, mhz: float = SM_MAX_MHZ) -> float:
    """Time the activation prologue needs at full issue rate: rows x K elements x
    lane operations each / (SMs x 128 lanes x clock)."""
    return rows * K * QUANT_LANE_OPS_PER_ELEMENT / (sms * 128 * mhz * 1e6) * 1e6


def time_eager(fn, stream, calls: int = 20, trials: int = 15, warm: int = 20) -> float:
    """Median us per call over `trials` blocks of `calls` eager calls (host launch
    included, L2 not flushed), CUDA events on `stream`; fn(i) is told the call's
    index, so that callers can alternate inputs."""
    out = []
    with torch.cuda.stream(stream):
        for i in range(warm):
            fn(i)
        for _ in range(trials):
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for i in range(calls):
                fn(i)
            t1.record(stream)
            t1.synchronize()
            out.append(t0.elapsed_time(t1) * 1e3 / calls)
    return statistics.median(out)


def workload_table(mq, device, stream, flush, hbm_gbs, reps):
    """us/call (trimmed mean, cold L2), TFLOPS and roofline fraction for every
    problem of the five workloads, fused and unfused (CUDA graph per call), the
    plain MXFP4 baseline's time, the calls with bias + GELU_TANH and with the FP8
    output, and both paths' error against the unquantised layer on sampled rows;
    also eager calls that allocate y on every call, and the ALU bound of the
    activation prologue."""
    rows = []
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    for cfg in range(5):
        for p in synth.config(cfg):
            pp = Prepared(p, device, mq)
            torch.cuda.synchronize()
            g = capture(lambda: pp.run(mq), stream)
            us, iqr = time_graph(g, flush, stream, reps)
            us_warm, _ = time_graph(g, flush, stream, reps, cold=False)
            un = None
            if p.E == 1:
                gu = capture(lambda: pp.run_unfused(mq), stream)
                un, _ = time_graph(gu, flush, stream, reps)
                del gu
            try:  # a supplementary series: its failure must not cost the table
                eager_alloc_us = time_eager(lambda i: pp.run_alloc(mq, stream, alt=bool(i & 1)), stream)
                eager_err = None
            except Exception as e:  # noqa: BLE001
                eager_alloc_us, eager_err = None, f"{type(e).__name__}: {e}"[:200]
                torch.cuda.synchronize()
            type2_us = None
            if p.E > 1:
                try:  # supplementary: its failure must not cost the table
                    g2 = capture(lambda: pp.run_type2(mq), stream)
                    type2_us, _ = time_graph(g2, flush, stream, reps)
                    del g2
                except Exception:  # noqa: BLE001
                    type2_us = None
            ge = capture(lambda: pp.run_epilogue(mq), stream)
            epi_us, _ = time_graph(ge, flush, stream, reps)
            del ge
            try:  # supplementary: its failure must not cost the table
                g8 = capture(lambda: pp.run_fp8(mq), stream)
                fp8_us, _ = time_graph(g8, flush, stream, reps)
                del g8
            except Exception:  # noqa: BLE001
                fp8_us = None
            # accuracy against the unquantised layer on sampled rows, then the plain MXFP4 baseline
            rows_s = np.unique(np.random.default_rng(cfg).integers(0, p.M, min(p.M, 16)))
            pp.run(mq, stream)
            stream.synchronize()
            nmse = layer_nmse(p, pp.y, rows_s)
            pp.prepare_plain(mq, device)
            gp = capture(lambda: pp.run_plain(mq), stream)
            plain_us, _ = time_graph(gp, flush, stream, reps)
            del gp
            pp.run_plain(mq, stream)
            stream.synchronize()
            nmse_plain = layer_nmse(p, pp.y, rows_s)
            t_roof = max(p.algorithmic_bytes() / (hbm_gbs * 1e9), p.flops() / (FP4_NOMINAL_TFLOPS * 1e12))
            rows.append({
                "config": cfg, "name": p.name, "us": us, "iqr_us": iqr, "us_warm_l2": us_warm,

                "tflops": p.flops() / (us * 1e-6) / 1e12, "gbs": p.algorithmic_bytes() / (us * 1e-6) / 1e9,
                "roofline_us": t_roof * 1e6, "frac_roofline": t_roof / (us * 1e-6), "unfused_us": un,
                "plain_us": plain_us, "plain_over_macaq_time": plain_us / us,
                "bias_gelu_tanh_us": epi_us, "fp8_out_us": fp8_us, "eager_alloc_us": eager_alloc_us,
                "group_list_type2_us": type2_us,
                **({"eager_alloc_error": eager_err} if eager_err else {}),
                "alu_bound_us": alu_bound_us(p.M, p.K, sms),
                "nmse": nmse, "nmse_plain": nmse_plain, "nmse_plain_over_macaq": nmse_plain / nmse if nmse else None,
            })
            del g, pp
            torch.cuda.empty_cache()
    return rows


def launch_floor(device, stream, flush, reps: int, launches: int = 5) -> dict:
    """The floor a chain of dependent launches sets, measured the way the step is:
    a CUDA graph of `launches` dependent one-element adds (torch's kernels, no
    work to speak of), L2 flushed before each replay, device time per launch: the
    share of the step's per-launch time that launching and chaining alone cost
    (the step's kernels also use programmatic dependent launch, which can overlap
    a launch with its predecessor's tail)."""
    t = torch.zeros(1, device=device)
    g = capture(lambda: [t.add_(1.0) for _ in range(launches)], stream)
    us, _ = time_graph(g, flush, stream, reps)
    del g
    g1 = capture(lambda: t.add_(1.0), stream)
    us1, _ = time_graph(g1, flush, stream, reps)
    del g1
    return {"us_per_launch": us / launches, "launches": launches, "us_one_launch_graph": us1,
            "what": "CUDA graph of dependent one-element adds (torch's kernels), L2 flushed before each replay, "
                    "events around the replay; us_one_launch_graph: a graph of one such add, the floor of a "
                    "single-call graph figure"}


def calibration_table(mq, device, stream, flush, hbm_gbs, reps):
    """Offline D calibration (macaq_calibrate_d) on 1,024 calibration tokens (the
    MACAQ page's pilot size) for each Qwen3-0.6B-shaped projection: us per call
    (trimmed mean, cold L2) and its bytes (x, W, D) against the HBM bandwidth."""
    out = []
    for (K, N) in synth.QWEN_PAIRS:
        p = synth.dense(1024, K, N, seed=11)
        x, W = x_dev(p.x, device), f32(p.W, device)
        g = capture(lambda: mq.calibrate_d(x, W, stream=stream), stream)
        us, _ = time_graph(g, flush, stream, reps)
        nbytes = 1024 * K * 2 + N * K * 4 + K * 4
        out.append({"name": f"calibrate T=1024 K={K} N={N}", "us": us, "gbs": nbytes / (us * 1e-6) / 1e9,
                    "frac_hbm": nbytes / (us * 1e-6) / 1e9 / hbm_gbs})
        del g, x, W
    return out


if __name__ == "__main__":
    main()
