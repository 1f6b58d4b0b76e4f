"""Benchmark: HQQ quantize+pack and dequantize on B200.

One step = the whole hot path over one matrix: hqq_quantize (min-max init, proximal rounds
with the tensor-wide stop rule, final quantize, bit-packing, fp16 metadata) followed by
hqq_dequantize.  Inputs rotate over enough copies that every step reads its matrix from HBM
(more than twice the 126 MB L2).  Rank 0 prints one JSON line:
  - `ms_per_step`: K steps timed as a whole (CUDA events at the two ends only, so the
    dequantize launch overlaps the quantize call's tail as it does for a user);
  - `value`: quantize+pack Gweights/s, from a second pass of K steps with an event pair
    around every call (all ranks' weights over the max-over-ranks time);
  - `roofline`: the quantize call.  It is bound by instruction issue, not by HBM: `frac` is
    the fraction of the ALU lane-op peak; `hbm_frac` (the target's metric: W read once plus
    codes and metadata written once), `alu_frac` and `issue_frac` (warp instructions from the
    committed ncu summary over 4 issue slots x 148 SMs x the clock) stand beside it;
  - `per_config`: every configuration of the task (256x512 b4 g64; 4096x11008 b2 g16 and b3
    g64; 4096^2 b4 g128 axis 0; the 224-matrix 7B-like stack), each briefly timed;
  - `e2e`: the same metric through the public API with pinned host buffers, copies included;
  - `cpu_baseline`: the CPU oracle on the host, on all cores (OpenMP timing build) and on one;
  - `dequant_back_to_back` and `gemv`: dequantize and the fused forward product, each timed
    back to back by CUDA-graph replay, with the unfused dequantize + matmul beside the latter;
  - `gemm`: the batched forward product (tensor cores) for batches 1, 16, 64 and 256, timed
    the same way, beside the unfused dequantize + matmul.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--workload attn|small|mlp_b2|mlp_b3|attn_ax0|stack] [--no-per-config]

--workload picks the configuration: attn, the default, is the 4096x4096 4-bit group-64
headline; stack quantizes and dequantizes all 224 matrices of the 7B-like stack per step.
--impl reference times the CPU oracle (the plain C reference of the method) on the host on
bounded slices of the same workload.  Under torchrun every rank quantizes its own matrices,
with no data-path communication (weak scaling; stack: the matrices are split, strong scaling).
The reference arm runs on rank 0 only.
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
sys.path.insert(0, ROOT)

METRIC_ATTN = "HQQ quantize+pack Gweights/s at 4096\u00b2 4-bit g64; dequant GB/s; % of HBM peak"
METRIC = METRIC_ATTN
UNIT = "Gweights/s"
ROWS = COLS = 4096
NBITS, GROUP, AXIS, ITERS = 4, 64, 1, 20
WORKLOAD = ("0.02*StudentT(4) clipped to +-1, fp16 4096x4096 (attention-projection-shaped), seed 1; "
            "4-bit, group 64, axis 1, <=20 rounds, p=0.7, beta=10, kappa=1.01")
ROTATE = 8
CASE = None                  # the workloads.Case being timed (set by select())
GEN_DESC = {"outlier_normal": "N(0, 0.02^2) with 0.1% of entries replaced by +-U(0.2, 1.0)",
            "student_t": "0.02*StudentT(4) clipped to +-1",
            "row_lognormal": "N(0, 0.015^2) x per-row LogNormal(0, 0.3)"}
SINGLE = {"small": "SMALL", "attn": "ATTN", "mlp_b2": "MLP_B2", "mlp_b3": "MLP_B3", "attn_ax0": "ATTN_AX0"}


def select(name: str):
    """Point the module's workload constants at one of the single-matrix configurations."""
    global CASE, ROWS, COLS, NBITS, GROUP, AXIS, WORKLOAD, ROTATE, METRIC
    from free_weight_quantization_b200 import workloads as wl
    c = getattr(wl, SINGLE[name])
    CASE = c
    ROWS, COLS, NBITS, GROUP, AXIS = c.rows, c.cols, c.nbits, c.group_size, c.axis
    WORKLOAD = (f"{GEN_DESC[c.gen]}, fp16 {c.rows}x{c.cols}, seed {c.seed}; {c.nbits}-bit, "
                f"group {c.group_size}, axis {c.axis}, <=20 rounds, p=0.7, beta=10, kappa=1.01")
    if name == "attn":
        METRIC = METRIC_ATTN
        WORKLOAD = ("0.02*StudentT(4) clipped to +-1, fp16 4096x4096 (attention-projection-shaped), "
                    "seed 1; 4-bit, group 64, axis 1, <=20 rounds, p=0.7, beta=10, kappa=1.01")
    else:
        METRIC = f"HQQ quantize+pack Gweights/s at {c.rows}x{c.cols} {c.nbits}-bit g{c.group_size} axis {c.axis}; dequant GB/s; % of HBM peak"
    # enough rotating copies that the inputs outgrow twice the 126 MB L2
    ROTATE = max(8, -(-252_000_000 // (2 * c.rows * c.cols)))


ISSUE_LANES_PER_SM = 128     # 4 SM sub-partitions x 32 lanes issue one instruction per clock
ISSUE_SLOTS_PER_SM = 4       # warp instructions per clock per SM (one per sub-partition)
ALU_OPS_INIT, ALU_OPS_ROUND, ALU_OPS_FINAL = 3, 12, 6   # algorithmic ops per weight
HBM_TARGET = 0.60            # the target fraction of the HBM roofline for the headline quantize


PROFILE = os.path.join(ROOT, "profiles", "hqq_stream_kernel_4096x4096_b4g64.md")
# the sources the stream kernel is compiled from: a code change in either withdraws the profile
KERNEL_SRC = [os.path.join(ROOT, "free_weight_quantization_b200", "csrc", "hqq_stream.cu"),
              os.path.join(ROOT, "free_weight_quantization_b200", "csrc", "hqq_common.cuh")]


def code_hash(path) -> str:
    """sha256 of C/CUDA sources (one path or a list) with comments and blank space removed,
    so that only a change of code (not of a comment) makes a recorded profile stale."""
    import hashlib
    import re
    paths = [path] if isinstance(path, str) else list(path)
    parts = []
    for p in paths:
        src = open(p, encoding="utf-8").read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        parts.append("\n".join(line.strip() for line in src.splitlines() if line.strip()))
    return hashlib.sha256("\n".join(parts).encode("utf-8")).hexdigest()


def profiled_fields() -> dict:
    """The per-launch figures of the committed ncu summary of the stream kernel, or {} when
    the kernel's code has changed since that capture."""
    try:
        text = open(PROFILE).read()
        src = code_hash(KERNEL_SRC)
    except OSError:
        return {}
    fields = dict((k.strip(), v.strip()) for k, v in
                  (l.split(":", 1) for l in text.splitlines()
                   if l.startswith(("code-sha256:", "traffic-bytes-per-launch:",
                                    "inst-executed-per-launch:"))))
    if fields.get("code-sha256", "") != src:
        return {}
    out = {}
    for k in ("traffic-bytes-per-launch", "inst-executed-per-launch"):
        try:
            out[k] = float(fields[k])
        except (KeyError, ValueError):
            pass
    return out


def profiled_traffic():
    """DRAM bytes per launch of the stream kernel from the committed ncu summary, or None."""
    return profiled_fields().get("traffic-bytes-per-launch")


def peaks():
    p = {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "src": "fallback"}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        p.update(hbm_gbs=float(m["hbm_gbs"]), sm_max_mhz=float(m.get("sm_max_mhz", 1965.0)),
                 src="measured")
    except (OSError, KeyError, ValueError):
        pass
    return p


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms in the background."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return self
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        win = [p for t, p in self.samples if t0 <= t <= t1]
        window = "timed"
        if len(win) < 3:
            win = [p for _, p in self.samples]
            window = "whole run"
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[1]) for p in win if num(p[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for p in win for n, v in zip(names, p[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(win[0][2]), "reasons": reasons, "samples": len(win),
                "window": window, "power_w_max": max((num(p[3]) or 0.0) for p in win)}


def launches_per_step(nbits: int, group: int, axis: int, n: int) -> int:
    """Kernels one quantize + dequantize step launches: the zero kernel, the stream or search
    kernel and the fixup kernel, a pack kernel when an axis-0 layout's groups do not fill
    whole packed words, and the dequant kernel."""
    cpw = {2: 16, 3: 10, 4: 8}[nbits]
    pack = axis == 0 and (n // group) % cpw != 0
    return 4 + (1 if pack else 0)


def shard(items, rank: int, ws: int):
    """This rank's share of independent work items (every item on exactly one rank)."""
    return items[rank::ws]


def max_over_ranks(values, device, ws: int):
    """Element-wise maximum of per-rank timings (a no-op on one rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if ws > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def run_reference(args, ws, rank):
    """The CPU oracle, as it stands, on a bounded slice of the workload."""
    if rank != 0:
        return
    import numpy as np

    import oracle
    from free_weight_quantization_b200 import workloads as wl
    oracle.build()
    W = CASE.make()
    # each step is a slice of up to 256 rows, fewer for long runs, so the whole run stays
    # within about two minutes: the oracle needs about 2 ms per 4096 weights of a row
    budget_rows = int(60000 * 4096 / COLS)
    rows = max(1, min(256, ROWS, budget_rows // (args.warmup + args.steps)))
    times = []
    for i in range(args.warmup + args.steps):
        nsl = ROWS // rows
        sl = np.ascontiguousarray(W[(i % nsl) * rows:(i % nsl + 1) * rows])
        t0 = time.perf_counter()
        r = oracle.quantize(sl, NBITS, GROUP, AXIS, iters=ITERS)
        oracle.dequant(r["packed"], r["scale"], r["zero"], rows, COLS, NBITS, GROUP, AXIS)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    n = rows * COLS
    value = n * len(times) / sum(times) / 1e9
    sample = (f"{args.steps} slices of {rows}x{COLS} of the {ROWS}x{COLS} workload, "
              "quantize+pack+dequant")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample_rows": rows},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline(W, nbits, group, axis, iters, rows, cols, budget_s=3.0):
    """The oracle on the host: its all-core timing build (OpenMP over groups; exact integer
    round sums, so the same results) and the single-threaded oracle, each repeated over the
    full matrix until about budget_s seconds have passed (at least one pass)."""
    cores = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    import oracle
    oracle.build()
    oracle.build_parallel()

    def timed(parallel):
        reps, t0 = 0, time.perf_counter()
        while True:
            r = oracle.quantize(W, nbits, group, axis, iters=iters, parallel=parallel)
            oracle.dequant(r["packed"], r["scale"], r["zero"], rows, cols, nbits, group, axis)
            reps += 1
            dt = time.perf_counter() - t0
            if dt >= budget_s:
                return reps, dt

    reps_p, dt_p = timed(True)
    reps_1, dt_1 = timed(False)
    n = rows * cols
    return {"value": reps_p * n / dt_p / 1e9, "unit": UNIT, "cores": int(os.environ["OMP_NUM_THREADS"]),
            "kind": "oracle",
            "sample": f"{reps_p} pass(es) over the {rows}x{cols} matrix of the workload, "
                      f"quantize+pack+dequant, {dt_p:.1f} s on {os.environ['OMP_NUM_THREADS']} "
                      "threads (the oracle's OpenMP timing build: same source, its round loop "
                      "spread over threads)",
            "single_core": {"value": reps_1 * n / dt_1 / 1e9, "unit": UNIT, "cores": 1,
                            "sample": f"{reps_1} pass(es), {dt_1:.1f} s single-threaded"}}


class Rig:
    """Rotating device inputs and outputs of one single-matrix configuration, and the calls
    that time it (the library's kernels only: no host work inside the timed regions)."""

    def __init__(self, case, dev, rotate=None):
        import torch

        from free_weight_quantization_b200 import hqq
        self.hqq, self.torch, self.case, self.dev = hqq, torch, case, dev
        c = case
        self.N = c.rows * c.cols
        self.G = self.N // c.group_size
        self.rotate = rotate or max(8, -(-252_000_000 // (2 * self.N)))
        self.W0 = torch.from_numpy(c.make())
        self.Ws = [self.W0.to(dev) for _ in range(self.rotate)]
        self.outs = [hqq.hqq_quantize(self.Ws[0], c.nbits, c.group_size, c.axis, iters=ITERS)
                     for _ in range(self.rotate)]
        self.deqs = [torch.empty_like(self.Ws[0]) for _ in range(self.rotate)]
        self.wsb = hqq.hqq_quantize_workspace_bytes(c.rows, c.cols, c.nbits, c.group_size, c.axis, ITERS)
        self.work = torch.empty(max(16, self.wsb), dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        dbg = hqq.hqq_quantize(self.Ws[0], c.nbits, c.group_size, c.axis, iters=ITERS, debug=True)
        torch.cuda.synchronize()
        self.iters_run = int(dbg.iters_run.item())
        self.rounds = int(dbg.rounds.to(torch.int64).sum().item())
        self.packed_bytes = hqq.hqq_packed_bytes(self.N, c.nbits)
        # W read once + packed codes and fp16 metadata written once (dequantize: the reverse)
        self.alg_bytes = 2 * self.N + self.packed_bytes + 4 * self.G

    def quantize(self, i):
        c = self.case
        k = i % self.rotate
        self.hqq.hqq_quantize(self.Ws[k], c.nbits, c.group_size, c.axis, iters=ITERS, out=self.outs[k],
                              workspace=self.work)

    def dequantize(self, i):
        k = i % self.rotate
        self.hqq.hqq_dequantize(self.outs[k], out=self.deqs[k])

    def quant_ms(self, steps):
        """Average quantize call time: an event pair around every call."""
        torch = self.torch
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            evs[i][0].record(self.stream)
            self.quantize(i)
            evs[i][1].record(self.stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs) / steps

    def per_call_ms(self, loop, n):
        """Per-call time of n back-to-back calls captured in a CUDA graph and replayed (the
        host's per-call launch cost is not what gets measured); plain loop without graphs."""
        torch = self.torch
        loop(2 * self.rotate)  # warm-up (library modules, cuBLAS handles)
        torch.cuda.synchronize()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        try:
            side = torch.cuda.Stream(self.dev)
            side.wait_stream(torch.cuda.current_stream(self.dev))
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.stream(side):
                with torch.cuda.graph(graph, stream=side):
                    loop(n)
            torch.cuda.current_stream(self.dev).wait_stream(side)
            graph.replay()
            torch.cuda.synchronize()
            b0.record(self.stream)
            for _ in range(4):
                graph.replay()
            b1.record(self.stream)
            torch.cuda.synchronize()
            del graph
            return b0.elapsed_time(b1) / (4 * n), "cuda graph replay"
        except RuntimeError:
            torch.cuda.synchronize()
            b0.record(self.stream)
            loop(n)
            b1.record(self.stream)
            torch.cuda.synchronize()
            return b0.elapsed_time(b1) / n, "plain loop"

    def dequant_b2b_ms(self, n):
        def loop(m):
            for i in range(m):
                self.dequantize(i)
        return self.per_call_ms(loop, n)

    def fractions(self, quant_s, deq_s, pk):
        """HBM and ALU fractions of a quantize time and a dequantize time (seconds)."""
        alu_peak = 148 * ISSUE_LANES_PER_SM * pk["sm_max_mhz"] * 1e6 / 1e12   # T ops/s
        ops = self.N * (ALU_OPS_INIT + ALU_OPS_FINAL) + self.case.group_size * self.rounds * ALU_OPS_ROUND
        return {"quant_hbm_frac": self.alg_bytes / quant_s / 1e9 / pk["hbm_gbs"],
                "quant_alu_frac": ops / quant_s / 1e12 / alu_peak,
                "dequant_hbm_frac": self.alg_bytes / deq_s / 1e9 / pk["hbm_gbs"],
                "alg_ops_per_launch": ops}


def measure_config(name, dev, pk, steps=30):
    """One single-matrix configuration, briefly: quantize per call, dequantize back to back."""
    from free_weight_quantization_b200 import workloads as wl
    c = getattr(wl, SINGLE[name])
    rig = Rig(c, dev)
    for i in range(3):
        rig.quantize(i)
        rig.dequantize(i)
    q_ms = rig.quant_ms(steps)
    d_ms, how = rig.dequant_b2b_ms(max(2 * rig.rotate, 100))
    out = {"workload": f"{GEN_DESC[c.gen]}, fp16 {c.rows}x{c.cols}, seed {c.seed}; {c.nbits}-bit, "
                       f"group {c.group_size}, axis {c.axis}, <=20 rounds",
           "quant_us": q_ms * 1e3, "quant_gweights_s": rig.N / (q_ms / 1e3) / 1e9,
           "dequant_b2b_us": d_ms * 1e3, "dequant_timed_by": how,
           "iters_run": rig.iters_run, "group_rounds": rig.rounds,
           "alg_bytes_per_launch": rig.alg_bytes, "quant_steps": steps}
    out.update(rig.fractions(q_ms / 1e3, d_ms / 1e3, pk))
    del rig
    return out


def measure_stack_config(dev, pk, steps=2):
    """The 224-matrix 7B-like stack: quantize every matrix, then dequantize every matrix."""
    import torch

    from free_weight_quantization_b200 import hqq
    from free_weight_quantization_b200 import workloads as wl
    keys = [(l, i) for l in range(wl.STACK_LAYERS) for i in range(len(wl.STACK_SHAPES))]
    Ws = [wl.stack_matrix_torch(l, i, dev) for l, i in keys]
    outs = [hqq.hqq_quantize(W, NBITS, GROUP, AXIS, iters=ITERS, debug=True) for W in Ws]
    torch.cuda.synchronize()
    rounds = sum(int(q.rounds.to(torch.int64).sum().item()) for q in outs)
    iters = [int(q.iters_run.item()) for q in outs]
    for q in outs:
        q.iters_run = q.s = q.z = q.err_trace = q.rounds = None
    deqs = [torch.empty_like(W) for W in Ws]
    work = {}
    for W in Ws:
        r, c = W.shape
        if (r, c) not in work:
            work[(r, c)] = torch.empty(max(16, hqq.hqq_quantize_workspace_bytes(r, c, NBITS, GROUP, AXIS, ITERS)),
                                       dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def quant_all():
        for W, q in zip(Ws, outs):
            hqq.hqq_quantize(W, NBITS, GROUP, AXIS, iters=ITERS, out=q, workspace=work[tuple(W.shape)])

    def deq_all():
        for q, d in zip(outs, deqs):
            hqq.hqq_dequantize(q, out=d)

    quant_all()
    deq_all()
    torch.cuda.synchronize()
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    qt = dt = 0.0
    for _ in range(steps):
        e[0].record(stream)
        quant_all()
        e[1].record(stream)
        deq_all()
        e[2].record(stream)
        torch.cuda.synchronize()
        qt += e[0].elapsed_time(e[1])
        dt += e[1].elapsed_time(e[2])
    n = sum(W.numel() for W in Ws)
    G = n // GROUP
    alg = 2 * n + n // 2 + 4 * G
    q_s, d_s = qt / 1e3 / steps, dt / 1e3 / steps
    alu_peak = 148 * ISSUE_LANES_PER_SM * pk["sm_max_mhz"] * 1e6 / 1e12
    ops = n * (ALU_OPS_INIT + ALU_OPS_FINAL) + GROUP * rounds * ALU_OPS_ROUND
    del Ws, outs, deqs, work
    torch.cuda.empty_cache()
    return {"workload": STACK_WORKLOAD, "matrices": len(keys), "weights": n,
            "quant_ms": q_s * 1e3, "dequant_ms": d_s * 1e3,
            "quant_gweights_s": n / q_s / 1e9, "dequant_gbs": alg / d_s / 1e9,
            "quant_hbm_frac": alg / q_s / 1e9 / pk["hbm_gbs"],
            "quant_alu_frac": ops / q_s / 1e12 / alu_peak,
            "dequant_hbm_frac": alg / d_s / 1e9 / pk["hbm_gbs"],
            "iters_run_min_max": [min(iters), max(iters)], "group_rounds": rounds, "steps": steps,
            "timed_by": "CUDA events around all 224 quantize calls, then around all 224 dequantize calls"}


STACK_WORKLOAD = ("synthetic 7B-like stack: 32 layers x (4 x 4096x4096 + 3 x 4096x11008) fp16, "
                  "0.02*StudentT(4) clipped to +-1 drawn on the GPU from per-matrix seeds; 4-bit, "
                  "group 64, axis 1, per-tensor early stop; quantize all then dequantize all")


def run_stack(args, ws, rank, local):
    """One step = quantize+pack every matrix of the stack, then dequantize every matrix.
    Under torchrun the 224 matrices are split across ranks (no communication: strong scaling)."""
    import torch
    import torch.distributed as dist

    from free_weight_quantization_b200 import hqq
    from free_weight_quantization_b200 import workloads as wl

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        dist.init_process_group("nccl", device_id=dev,
                                timeout=__import__("datetime").timedelta(seconds=120))
    keys = [(l, i) for l in range(wl.STACK_LAYERS) for i in range(len(wl.STACK_SHAPES))]
    mine = shard(keys, rank, ws)
    Ws = [wl.stack_matrix_torch(l, i, dev) for l, i in mine]
    outs = [hqq.hqq_quantize(W, NBITS, GROUP, AXIS, iters=ITERS, debug=True) for W in Ws]
    torch.cuda.synchronize()
    rounds = sum(int(q.rounds.to(torch.int64).sum().item()) for q in outs)
    iters = [int(q.iters_run.item()) for q in outs]
    for q in outs:
        q.iters_run = q.s = q.z = q.err_trace = q.rounds = None
    deqs = [torch.empty_like(W) for W in Ws]
    work = {}
    for W in Ws:
        r, c = W.shape
        if (r, c) not in work:
            work[(r, c)] = torch.empty(max(16, hqq.hqq_quantize_workspace_bytes(r, c, NBITS, GROUP, AXIS, ITERS)),
                                       dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        for W, q in zip(Ws, outs):
            hqq.hqq_quantize(W, NBITS, GROUP, AXIS, iters=ITERS, out=q, workspace=work[tuple(W.shape)])
        for q, d in zip(outs, deqs):
            hqq.hqq_dequantize(q, out=d)

    for _ in range(args.warmup):
        step()
    sampler = ClockSampler(local).start()
    time.sleep(0.3)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tw0 = time.time()
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    tw1 = time.time()
    if ws > 1:
        dist.barrier()
    ms = a.elapsed_time(b) / args.steps
    sampler.stop()
    clocks = sampler.summary(tw0, tw1)
    ms, = max_over_ranks([ms], dev, ws)
    n_all = sum(r * c for r, c in (wl.STACK_SHAPES[i] for _, i in keys))
    n_mine = sum(W.numel() for W in Ws)
    if rank == 0:
        pk = peaks()
        alu_peak = 148 * ISSUE_LANES_PER_SM * pk["sm_max_mhz"] * 1e6 / 1e12
        alg_ops = n_mine * (ALU_OPS_INIT + ALU_OPS_FINAL) + GROUP * rounds * ALU_OPS_ROUND
        ach = alg_ops / (ms / 1e3) / 1e12 * ws
        line = {
            "metric": METRIC, "value": n_all / (ms / 1e3) / 1e9, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": STACK_WORKLOAD, "matrices": len(keys), "weights": n_all,
                       "iters_run_min_max": [min(iters), max(iters)],
                       "l2": "inputs larger than L2 (12.95 GB stack)",
                       "parallelism": f"matrices split across {ws} rank(s)"},
            "roofline": {"bound": "alu", "kernel": "hqq_quantize + hqq_dequantize over the stack",
                         "achieved": ach, "peak": alu_peak, "unit": "Tops/s", "frac": ach / alu_peak,
                         "traffic": None, "alg_ops_per_step": alg_ops * ws},
            "e2e": None,
            "gpu_launches": launches_per_step(NBITS, GROUP, AXIS, 4096 * 4096) * len(Ws) * args.steps,
            "clocks": clocks,
        }
        if not args.no_cpu_baseline:
            Wh = Ws[0].cpu().numpy()
            import oracle
            oracle.build()
            t0 = time.perf_counter()
            r = oracle.quantize(Wh, NBITS, GROUP, AXIS, iters=ITERS)
            oracle.dequant(r["packed"], r["scale"], r["zero"], Wh.shape[0], Wh.shape[1], NBITS, GROUP, AXIS)
            dt = time.perf_counter() - t0
            line["cpu_baseline"] = {"value": Wh.size / dt / 1e9, "unit": UNIT, "cores": 1,
                                    "kind": "oracle",
                                    "sample": f"layer 0 matrix 0 (4096x4096) of the stack, {dt:.1f} s "
                                              "single-threaded; the stack is 247x its size"}
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--workload", default="attn", choices=list(SINGLE) + ["stack"],
                    help="attn: the 4096x4096 headline matrix (default); small, mlp_b2, mlp_b3, "
                         "attn_ax0: the other single-matrix configurations; stack: the 7B-like "
                         "224-matrix stack")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the brief timing of the other configurations")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.steps is None:
        args.steps = {"attn": 2000, "small": 5000, "attn_ax0": 1000, "stack": 20}.get(args.workload, 500)
    if args.workload != "stack":
        select(args.workload)
    ws, rank, local = dist_setup()

    if args.impl == "reference":
        run_reference(args, ws, rank)
        return
    if args.workload == "stack":
        run_stack(args, ws, rank, local)
        return

    import torch
    import torch.distributed as dist

    from free_weight_quantization_b200 import hqq

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        dist.init_process_group("nccl", device_id=dev,
                                timeout=__import__("datetime").timedelta(seconds=120))

    # every rank quantizes its own copies of the workload matrix
    rig = Rig(CASE, dev, rotate=ROTATE if CASE.name.startswith("student-t 4096x4096 b4 g64") else None)
    N, G = rig.N, rig.G
    stream = rig.stream
    K = args.steps

    def step(i):
        rig.quantize(i)
        rig.dequantize(i)

    for i in range(args.warmup):
        step(i)
    sampler = ClockSampler(local).start()
    time.sleep(0.3)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tw0 = time.time()
    # the K timed steps: events at the two ends only
    start.record(stream)
    for i in range(K):
        step(i)
    end.record(stream)
    torch.cuda.synchronize()
    total_ms = start.elapsed_time(end)
    # the same K steps with an event pair around every call, for the quantize / dequantize split
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for i in range(K):
        evs[i][0].record(stream)
        rig.quantize(i)
        evs[i][1].record(stream)
        rig.dequantize(i)
        evs[i][2].record(stream)
    torch.cuda.synchronize()
    tw1 = time.time()
    if ws > 1:
        dist.barrier()
    q_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    d_ms = sum(e[1].elapsed_time(e[2]) for e in evs)

    # Dequantize alone and the fused forward product y = W_hat @ x, each timed back to back over
    # the rotating buffers, plus the unfused path the fused one replaces: dequantize, then the
    # library's fp16 x @ W_hat.T.
    nb2b = max(2 * rig.rotate, min(K, 400))
    xv = torch.randn(COLS, device=dev).to(torch.float16)
    yv = [torch.empty(ROWS, dtype=torch.float32, device=dev) for _ in range(rig.rotate)]
    yl = [torch.empty(1, ROWS, dtype=torch.float16, device=dev) for _ in range(rig.rotate)]

    def loop_gemv(n):
        for i in range(n):
            hqq.hqq_gemv(rig.outs[i % rig.rotate], xv, out=yv[i % rig.rotate])

    def loop_unfused(n):
        for i in range(n):
            k = i % rig.rotate
            rig.dequantize(i)
            torch.matmul(xv.unsqueeze(0), rig.deqs[k].t(), out=yl[k])

    d_b2b_ms, b2b_how = rig.dequant_b2b_ms(nb2b)
    gemv_ms, _ = rig.per_call_ms(loop_gemv, nb2b)
    unfused_ms, _ = rig.per_call_ms(loop_unfused, nb2b)

    # The batched forward product Y = X @ W_hat.T (hqq_gemm: the tcgen05 tensor-core kernel on
    # this layout) for a few batch sizes, beside the unfused dequantize + library fp16 matmul.
    gemm = {}
    for batch in (1, 16, 64, 256):
        Xb = torch.randn(batch, COLS, device=dev).to(torch.float16)
        Yb = [torch.empty(batch, ROWS, dtype=torch.float32, device=dev) for _ in range(rig.rotate)]
        Yh = [torch.empty(batch, ROWS, dtype=torch.float16, device=dev) for _ in range(rig.rotate)]

        def loop_gemm(n, Xb=Xb, Yb=Yb):
            for i in range(n):
                hqq.hqq_gemm(rig.outs[i % rig.rotate], Xb, out=Yb[i % rig.rotate])

        def loop_gemm_unfused(n, Xb=Xb, Yh=Yh):
            for i in range(n):
                k = i % rig.rotate
                rig.dequantize(i)
                torch.matmul(Xb, rig.deqs[k].t(), out=Yh[k])

        ng = max(2 * rig.rotate, min(K, 200))
        g_ms, _ = rig.per_call_ms(loop_gemm, ng)
        u_ms, _ = rig.per_call_ms(loop_gemm_unfused, ng)
        gb = rig.packed_bytes + 4 * G + 2 * batch * COLS + 4 * batch * ROWS
        gemm[str(batch)] = {"us": g_ms * 1e3, "tflops": 2 * ROWS * COLS * batch / (g_ms / 1e3) / 1e12,
                            "gbs": gb / (g_ms / 1e3) / 1e9, "alg_bytes_per_launch": gb,
                            "unfused_dequant_then_matmul_us": u_ms * 1e3}

    # end to end through the public API: pinned host W in, packed codes + metadata + dequantized
    # W out, copies inside the timed region.  Two slots, each with its own stream, device
    # buffers, workspace and pinned host outputs, alternate steps, so one step's upload overlaps
    # the previous step's download on the full-duplex PCIe link.
    Wh = rig.W0.pin_memory()
    nslot = 2
    streams = [torch.cuda.Stream(dev) for _ in range(nslot)]
    works = [rig.work] + [torch.empty(max(16, rig.wsb), dtype=torch.uint8, device=dev) for _ in range(nslot - 1)]
    host_out = [dict(p=torch.empty(rig.outs[0].packed.numel(), dtype=torch.uint8).pin_memory(),
                     s=torch.empty(G, dtype=torch.float16).pin_memory(),
                     z=torch.empty(G, dtype=torch.float16).pin_memory(),
                     d=torch.empty(ROWS, COLS, dtype=torch.float16).pin_memory()) for _ in range(nslot)]
    e2e_steps = max(4, min(K, 50))

    def e2e_step(i):
        k = i % nslot
        st, ho = streams[k], host_out[k]
        with torch.cuda.stream(st):
            rig.Ws[k].copy_(Wh, non_blocking=True)
            hqq.hqq_quantize(rig.Ws[k], NBITS, GROUP, AXIS, iters=ITERS, out=rig.outs[k], workspace=works[k],
                             stream=st)
            hqq.hqq_dequantize(rig.outs[k], out=rig.deqs[k], stream=st)
            ho["p"].copy_(rig.outs[k].packed, non_blocking=True)
            ho["s"].copy_(rig.outs[k].scale, non_blocking=True)
            ho["z"].copy_(rig.outs[k].zero, non_blocking=True)
            ho["d"].copy_(rig.deqs[k], non_blocking=True)

    for i in range(2 * nslot):
        e2e_step(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for st in streams:
        st.wait_event(a)
    for i in range(e2e_steps):
        e2e_step(i)
    for st in streams:
        stream.wait_stream(st)
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / e2e_steps
    # the last slot's outputs arrived on the host intact (one quick check of the copies)
    assert torch.equal(host_out[(e2e_steps - 1) % nslot]["p"], rig.outs[(e2e_steps - 1) % nslot].packed.cpu())
    sampler.stop()
    clocks = sampler.summary(tw0, tw1)

    # max over ranks
    total_ms, q_ms, d_ms, e2e_ms, d_b2b_ms, gemv_ms, unfused_ms = max_over_ranks(
        [total_ms, q_ms, d_ms, e2e_ms, d_b2b_ms, gemv_ms, unfused_ms], dev, ws)

    if rank == 0:
        pk = peaks()
        packed_bytes = rig.packed_bytes
        alg_bytes = rig.alg_bytes
        q_s = q_ms / 1e3 / K
        d_s = d_ms / 1e3 / K
        value = ws * N / q_s / 1e9
        fr = rig.fractions(q_s, d_b2b_ms / 1e3, pk)
        sm_mhz = clocks.get("sm_mhz") or pk["sm_max_mhz"]
        alu_peak = 148 * ISSUE_LANES_PER_SM * pk["sm_max_mhz"] * 1e6 / 1e12   # T ops/s
        stream_engine = AXIS == 1 and NBITS != 3 and GROUP in (16, 32, 64, 128) and GROUP * NBITS % 32 == 0
        kname = ("hqq_quantize (hqq_stream_kernel + hqq_stream_fixup_kernel)" if stream_engine else
                 "hqq_quantize (hqq_search_kernel + hqq_fixup_kernel)")
        headline = CASE.name.startswith("student-t 4096x4096 b4 g64")
        prof = profiled_fields() if headline else {}
        inst = prof.get("inst-executed-per-launch")
        issue_frac = (inst / (ISSUE_SLOTS_PER_SM * 148 * sm_mhz * 1e6 * q_s)) if inst else None
        roofline = {"bound": "alu", "kernel": kname,
                    "achieved": fr["alg_ops_per_launch"] / q_s / 1e12, "peak": alu_peak,
                    "unit": "Tops/s", "frac": fr["quant_alu_frac"],
                    "traffic": prof.get("traffic-bytes-per-launch"),
                    "peak_src": f"148 SMs x 128 lanes x {pk['sm_max_mhz']:.0f} MHz (max clock)",
                    "hbm_frac": fr["quant_hbm_frac"], "hbm_peak_gbs": pk["hbm_gbs"],
                    "hbm_peak_src": pk["src"], "hbm_target": HBM_TARGET,
                    "hbm_target_met": fr["quant_hbm_frac"] >= HBM_TARGET,
                    "alu_frac": fr["quant_alu_frac"], "issue_frac": issue_frac,
                    "issue_src": ("warp instructions per launch from the committed ncu summary / "
                                  f"(4 issue slots x 148 SMs x {sm_mhz:.0f} MHz x the call time)"
                                  if inst else "no ncu summary of this kernel code"),
                    "alg_ops_per_launch": fr["alg_ops_per_launch"], "group_rounds": rig.rounds,
                    "alg_bytes_per_launch": alg_bytes}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": K,
            "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "rows": ROWS, "cols": COLS, "nbits": NBITS,
                       "group_size": GROUP, "axis": AXIS, "iters": ITERS,
                       "iters_run": rig.iters_run,
                       "l2": f"inputs larger than L2: {rig.rotate} rotating copies "
                             f"({rig.rotate * 2 * N / 1e6:.0f} MB > 126 MB)",
                       "parallelism": f"independent matrices per rank x{ws}"},
            "quant_us": q_s * 1e6, "dequant_us": d_s * 1e6,
            "quant_hbm_gbs": alg_bytes / q_s / 1e9, "quant_hbm_frac": fr["quant_hbm_frac"],
            "dequant_gbs": alg_bytes / d_s / 1e9, "dequant_hbm_frac": alg_bytes / d_s / 1e9 / pk["hbm_gbs"],
            "dequant_back_to_back": {"us": d_b2b_ms * 1e3, "gbs": alg_bytes / (d_b2b_ms / 1e3) / 1e9,
                                     "hbm_frac": alg_bytes / (d_b2b_ms / 1e3) / 1e9 / pk["hbm_gbs"],
                                     "launches": nb2b, "timed_by": b2b_how},
            "gemv": {"us": gemv_ms * 1e3,
                     "gbs": (packed_bytes + 4 * G + 2 * COLS + 4 * ROWS) / (gemv_ms / 1e3) / 1e9,
                     "hbm_frac": (packed_bytes + 4 * G + 2 * COLS + 4 * ROWS) / (gemv_ms / 1e3) / 1e9 / pk["hbm_gbs"],
                     "alg_bytes_per_launch": packed_bytes + 4 * G + 2 * COLS + 4 * ROWS,
                     "unfused_dequant_then_matmul_us": unfused_ms * 1e3, "launches": nb2b,
                     "timed_by": b2b_how},
            "gemm": {"batches": gemm, "timed_by": b2b_how,
                     "kernel": "tcgen05 (A = dequantized W from tensor memory, B = X by TMA)"},
            "hbm_peak_gbs": pk["hbm_gbs"], "hbm_peak_src": pk["src"],
            "alg_bytes_per_launch": alg_bytes,
            "roofline": roofline,
            "e2e": {"value": ws * N / (e2e_ms / 1e3) / 1e9, "unit": UNIT,
                    "h2d_bytes_per_step": 2 * N,
                    "d2h_bytes_per_step": packed_bytes + 4 * G + 2 * N},
            "gpu_launches": 2 * launches_per_step(NBITS, GROUP, AXIS, N) * K,
            "clocks": clocks,
        }
        if not args.no_per_config and ws == 1 and headline:
            pc = {"attn": {"workload": WORKLOAD, "quant_us": q_s * 1e6,
                           "quant_gweights_s": N / q_s / 1e9, "dequant_b2b_us": d_b2b_ms * 1e3,
                           "iters_run": rig.iters_run, "group_rounds": rig.rounds,
                           "alg_bytes_per_launch": alg_bytes, **fr}}
            del rig
            for name in ("small", "mlp_b2", "mlp_b3", "attn_ax0"):
                pc[name] = measure_config(name, dev, pk)
            pc["stack"] = measure_stack_config(dev, pk)
            line["per_config"] = pc
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(CASE.make(), NBITS, GROUP, AXIS, ITERS, ROWS, COLS)
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
