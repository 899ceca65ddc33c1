"""Benchmark of the block-quantized matmul on B200.

One step = one pass of the decode hot path over one batch of synthetic input:
the Q4_0 GEMV y = x . dequant(Wq)^T with N=11008, K=4096 and fp32
activations, at M = 1, 4 and 8 (three calls).  `value` is the whole-job
throughput in GB/s of packed weights + activations + outputs, timed on the
device with CUDA events, inputs resident in HBM, each call reading a
different copy of the weights from a rotation larger than 4x L2.  The calls
are made with LWQ_FLAG_OVERLAP (the weights are constant, as in a decode
loop), so each kernel may begin streaming its weights while the previous one
drains; the end-to-end leg, whose weights are copied in every step, does not
use it.  The other
workloads (Q8_0 4096x4096, the Q4_K 7B decode layer and the Q4_0 prefill
GEMMs) are measured in the same run and reported under "workloads"; the
decode-attention workloads (the pages' 512-token example and 7B-shaped
batches) under "attention".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lwq|reference]

Under torchrun every rank runs the same workload on its own GPU (the path
has no exchange step: replicas, weak scaling) and rank 0 prints one JSON line
with the max-over-ranks time.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_quantized_matmul_lwq_b200 import inputs  # noqa: E402

METRIC = "quantized matmul: decode GEMV weight GB/s (% of HBM); prefill GEMM TFLOP/s"
HEADLINE = "q4_0_gemv_11008x4096"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers

def csrc_sha256() -> str:
    """Hash of the CUDA sources (every .cu/.cuh under the package's csrc/)."""
    import glob
    import hashlib
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "block_quantized_matmul_lwq_b200", "csrc", "*.cu*"))):
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def profiled_traffic(workload: str) -> int | None:
    """DRAM bytes (read + write) of one step of `workload`, from the ncu counters recorded in
    profiles/traffic.json, or None when none are recorded or the CUDA sources changed since."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f).get(workload)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("csrc_sha256") != csrc_sha256():
        return None
    return int(rec["bytes_per_step"])


def load_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def step_calls(workload: str):
    """[(fmt, act, M, N, K, seed)] of one step of a workload.  A tuple seed is a
    weight of concatenated rows: equal parts, one per seed (see call_weights)."""
    spec = inputs.WORKLOADS[workload]
    calls = []
    if len(spec["shapes"]) > 1:
        # one call per shape (a single M serves every shape)
        Ms = spec["Ms"] if len(spec["Ms"]) == len(spec["shapes"]) else spec["Ms"] * len(spec["shapes"])
        for M, (N, K), seed in zip(Ms, spec["shapes"], spec["seeds"]):
            calls.append((spec["fmt"], spec["act"], M, N, K, seed))
    else:
        (N, K), = spec["shapes"]
        for M in spec["Ms"]:
            calls.append((spec["fmt"], spec["act"], M, N, K, spec["seeds"][0]))
    return calls


def call_weights(fmt: str, N: int, K: int, seed):
    """Packed weights of one call: seed s gives make_weights(fmt, rng(s), N, K); a
    tuple of seeds stacks that many equal row blocks, each generated as its own tensor."""
    if isinstance(seed, tuple):
        n = N // len(seed)
        return np.concatenate([inputs.make_weights(fmt, inputs.rng(s), n, K) for s in seed], axis=0)
    return inputs.make_weights(fmt, inputs.rng(seed), N, K)


def call_path(lwq, fmt: str, act: str, M: int, N: int, K: int) -> str:
    """The kernel family the library picks for a call."""
    return {1: "gemv", 2: "gemm", 3: "simple"}[lwq.lwq_select_config(call_fmt(lwq, fmt, act), M, N, K).path]


def base_act(act: str) -> str:
    """Activation dtype of a call; "f32:i8" is fp32 activations taken as int8 blocks (LWQ_FLAG_ACT_I8)."""
    return act.split(":")[0]


def call_fmt(lwq, fmt: str, act: str) -> int:
    """The C ABI's fmt of a call."""
    code = lwq.fmt_code(fmt, base_act(act))
    return code | lwq.LWQ_FLAG_ACT_I8 if act.endswith(":i8") else code


def call_activations(act: str, M: int, K: int, seed):
    """Activations of one call (a fused call takes those of its first part)."""
    s = seed[0] if isinstance(seed, tuple) else seed
    return inputs.activations(inputs.rng(s + 1000003), M, K, base_act(act))


def call_bytes(fmt, act, M, N, K) -> int:
    xe = 4 if base_act(act) == "f32" else 2
    return N * inputs.row_bytes(fmt, K) + M * K * xe + M * N * 4


def call_flops(M, N, K) -> int:
    return 2 * M * N * K


def reduce_max(value: float, dist_on: bool, device=None) -> float:
    """Max of a float over all ranks (identity without torch.distributed)."""
    if not dist_on:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, dist_on: bool, device=None) -> float:
    if not dist_on:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while active."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="lwq_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) == len(self.FIELDS):
                        rows.append(parts)
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[0]) for r in rows if num(r[0]) is not None]
        smax = [num(r[1]) for r in rows if num(r[1]) is not None]
        power = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower().startswith("active")})
        # samples under load: power at least half the largest seen (the set-up before the timed
        # region idles)
        pmax = max(power) if power else None
        loaded = [num(r[0]) for r in rows if num(r[0]) is not None and num(r[2]) is not None and pmax
                  and num(r[2]) >= 0.5 * pmax]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "sm_mhz_under_load": statistics.median(loaded) if loaded else None,
                "power_w_max": pmax, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- GPU arm

class Problem:
    """Device-resident inputs of one workload: rotating weight copies, x, y per call."""

    def __init__(self, workload: str, dev, rotate_min_bytes: int):
        import torch
        self.calls = step_calls(workload)
        self.host = []
        self.dev_calls = []
        cache = {}
        for fmt, act, M, N, K, seed in self.calls:
            key = (fmt, N, K, seed)
            if key not in cache:
                cache[key] = call_weights(fmt, N, K, seed)
            Wq = cache[key]
            x = call_activations(act, M, K, seed)
            self.host.append((Wq, x))
        self.step_weight_bytes = sum(N * inputs.row_bytes(f, K) for f, a, M, N, K, s in self.calls)
        # every call of a step reads its own weight copy; R steps cycle through
        # all copies, so a copy is re-read only after >= rotate_min_bytes of other weights
        self.R = max(3, -(-rotate_min_bytes // max(1, self.step_weight_bytes)))
        uses = {}
        self.use_index = []
        for fmt, act, M, N, K, seed in self.calls:
            key = (fmt, N, K, seed)
            self.use_index.append(uses.get(key, 0))
            uses[key] = uses.get(key, 0) + 1
        self.uses = uses
        self.weights = {}
        for (fmt, act, M, N, K, seed), (Wq, x) in zip(self.calls, self.host):
            key = (fmt, N, K, seed)
            if key not in self.weights:
                base = torch.from_numpy(Wq).to(dev)
                self.weights[key] = [base] + [base.clone() for _ in range(self.R * uses[key] - 1)]
            xd = torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).to(dev)
            yd = torch.empty((M, N), dtype=torch.float32, device=dev)
            self.dev_calls.append((fmt, act, M, N, K, seed, xd, yd))
        self.copies_bytes = sum(len(v) * v[0].numel() for v in self.weights.values())
        self.bytes_per_step = sum(call_bytes(f, a, M, N, K) for f, a, M, N, K, s in self.calls)
        self.flops_per_step = sum(call_flops(M, N, K) for f, a, M, N, K, s in self.calls)

    def enqueue_call(self, lwq, i: int, r: int, stream) -> int:
        """Enqueue call i of the step on `stream`, reading weight copy r; returns launches enqueued."""
        fmt, act, M, N, K, seed, xd, yd = self.dev_calls[i]
        key = (fmt, N, K, seed)
        W = self.weights[key][(r * self.uses[key] + self.use_index[i]) % len(self.weights[key])]
        # the weight copies are never written while timed, so each call may start
        # streaming its weights while the previous call finishes (LWQ_FLAG_OVERLAP)
        lwq.lwq_matmul(call_fmt(lwq, fmt, act) | lwq.LWQ_FLAG_OVERLAP, W, xd, yd, M, N, K, stream=stream)
        return lwq.lwq_last_launch_count()

    def enqueue_step(self, lwq, r: int, stream) -> int:
        """Enqueue one step on `stream`, reading weight copy r; returns launches enqueued."""
        return sum(self.enqueue_call(lwq, i, r, stream) for i in range(len(self.dev_calls)))


def replay_steps(graphs, full, n: int, first: int = 0) -> None:
    """Replay n steps, step i reading weight copy (first + i) mod R: whole
    rotations (from copy 0) through `full`, which holds all R steps in one
    graph, and the other steps one graph each."""
    R = len(graphs)
    i, c = 0, first % R
    while i < n:
        if c == 0 and n - i >= R:
            full.replay()
            i += R
        else:
            graphs[c].replay()
            i += 1
            c = (c + 1) % R


def time_workload(lwq, workload: str, dev, steps: int, warmup: int, dist_on: bool, per_call: bool = True):
    """Device time of `steps` steps (graph-replayed, rotating weights), max over ranks.

    The R steps of one weight rotation are captured in one graph, as a decode
    loop captures its calls: a graph launch costs the device several
    microseconds and ends the overlap of one call with the next, which one
    graph per step would add to every step."""
    import torch
    import torch.distributed as dist
    prob = Problem(workload, dev, rotate_min_bytes=4 * L2_BYTES)
    stream = torch.cuda.Stream(device=dev)
    graphs = []
    launches_per_step = 0
    with torch.cuda.stream(stream):
        for r in range(prob.R):   # eager warm-up of every copy, then one graph per copy
            prob.enqueue_step(lwq, r, stream)
        stream.synchronize()
        for r in range(prob.R):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                launches_per_step = prob.enqueue_step(lwq, r, stream)
            graphs.append(g)
        full = torch.cuda.CUDAGraph()
        with torch.cuda.graph(full, stream=stream):
            for r in range(prob.R):
                prob.enqueue_step(lwq, r, stream)
        full.replay()   # first launch uploads the graph; not a timed or warm-up step
    stream.synchronize()
    with torch.cuda.stream(stream):
        # the warm-up ends on copy R-1, so the timed steps start on the copy read longest ago
        replay_steps(graphs, full, warmup, first=-warmup)
    stream.synchronize()
    if dist_on:
        dist.barrier()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        replay_steps(graphs, full, steps)
        end.record(stream)
    stream.synchronize()
    torch.cuda.synchronize(dev)
    if dist_on:
        dist.barrier()
    ms = start.elapsed_time(end)
    ms_max = reduce_max(ms, dist_on, dev)

    # per-call device durations: one graph per call running it on every weight copy
    per = None
    if per_call:
        per = []
        for i, c in enumerate(prob.calls):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    for r in range(prob.R):
                        prob.enqueue_call(lwq, i, r, stream)
                g.replay()
            stream.synchronize()
            reps = max(2, min(50, steps // (4 * prob.R) or 2))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(reps):
                    g.replay()
                e1.record(stream)
            stream.synchronize()
            per.append({"call": c, "ms_mean": e0.elapsed_time(e1) / (reps * prob.R)})
            del g
    return prob, ms, ms_max, launches_per_step, per


def e2e_workload(lwq, workload: str, dev, steps: int, dist_on: bool):
    """End to end through the public API: pinned host inputs -> device -> lwq_matmul -> host result."""
    import torch
    import torch.distributed as dist
    calls = step_calls(workload)
    host = []
    for fmt, act, M, N, K, seed in calls:
        Wq = call_weights(fmt, N, K, seed)
        x = call_activations(act, M, K, seed)
        Wp = torch.from_numpy(Wq).pin_memory()
        xp = torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).pin_memory()
        yp = torch.empty((M, N), dtype=torch.float32).pin_memory()
        Wd = torch.empty_like(Wp, device=dev)
        xd = torch.empty_like(xp, device=dev)
        yd = torch.empty((M, N), dtype=torch.float32, device=dev)
        host.append((fmt, act, M, N, K, Wp, xp, yp, Wd, xd, yd))
    stream = torch.cuda.Stream(device=dev)
    h2d = sum(h[5].numel() * h[5].element_size() + h[6].numel() * h[6].element_size() for h in host)
    d2h = sum(h[7].numel() * 4 for h in host)

    def one_step():
        for fmt, act, M, N, K, Wp, xp, yp, Wd, xd, yd in host:
            Wd.copy_(Wp, non_blocking=True)
            xd.copy_(xp, non_blocking=True)
            lwq.lwq_matmul(call_fmt(lwq, fmt, act), Wd, xd, yd, M, N, K, stream=stream)
            yp.copy_(yd, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(2):
            one_step()
    stream.synchronize()
    if dist_on:
        dist.barrier()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(steps):
            one_step()
        end.record(stream)
    stream.synchronize()
    if dist_on:
        dist.barrier()
    ms = reduce_max(start.elapsed_time(end), dist_on, dev)
    nbytes = sum(call_bytes(c[0], c[1], c[2], c[3], c[4]) for c in calls)
    return ms, nbytes, h2d, d2h


def cpu_baseline(workload: str, budget_s: float = 15.0) -> dict:
    """The oracle as it stands, on the host cores, for about budget_s seconds of CPU work:
    two thirds with every core (the line's value), one third with one thread."""
    import oracle
    calls = step_calls(workload)
    threads = oracle.max_threads()

    def make(rows):
        data = []
        for fmt, act, M, N, K, seed in calls:
            n = min(rows, N)
            Wq = call_weights(fmt, N, K, seed)[:n] if isinstance(seed, tuple) else \
                inputs.make_weights(fmt, inputs.rng(seed), n, K)
            x = call_activations(act, M, K, seed)
            data.append((fmt, act, M, n, K, Wq, x))
        return data

    def run(data, reps, nthreads):
        t0 = time.perf_counter()
        for _ in range(reps):
            for fmt, act, M, n, K, Wq, x in data:
                oracle.matmul(fmt, Wq, x, act=act, nthreads=nthreads)
        return time.perf_counter() - t0

    def measure(nthreads, budget):
        full_rows = max(c[3] for c in calls)
        data = make(64)
        t_row = run(data, 1, nthreads) / 64
        if t_row * full_rows <= budget / 4:
            data = make(full_rows)
            t_step = run(data, 1, nthreads)
            reps = max(1, min(10000, int(budget / max(t_step, 1e-9))))
            sample = f"{reps} repetitions of one whole step (every weight row of every call; fp64 C oracle)"
        else:
            rows = max(16, min(full_rows, int(budget / max(t_row, 1e-9))))
            data = make(rows)
            reps = 1
            sample = f"first {rows} weight rows of every call of one step (fp64 C oracle)"
        total_s = run(data, reps, nthreads)
        total_bytes = reps * sum(call_bytes(fmt, act, M, n, K) for fmt, act, M, n, K, Wq, x in data)
        return total_bytes / total_s / 1e9, sample, total_s

    v_all, s_all, t_all = measure(threads, budget_s * 2 / 3)
    v_one, s_one, t_one = measure(1, budget_s / 3)
    return {"value": round(v_all, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": s_all + f", OpenMP on {threads} threads", "seconds": round(t_all, 2),
            "single_thread": {"value": round(v_one, 4), "unit": "GB/s", "cores": 1, "sample": s_one,
                              "seconds": round(t_one, 2)}}


def host_enqueue_cost(lwq, dev, n: int = 10000, batch: int = 200) -> dict:
    """Host time of one lwq_matmul call (the headline's M=1 call) through the C ABI: median
    over n calls, timed in batches with the stream drained between batches so that no call
    waits for room in the launch queue; the same calls with M = 0, which the first argument check
    refuses, give what ctypes costs for each signature."""
    import torch
    fmt, act, M, N, K, seed = step_calls(HEADLINE)[0]
    W = torch.from_numpy(call_weights(fmt, N, K, seed)).to(dev)
    x = torch.from_numpy(call_activations(act, M, K, seed)).to(dev)
    y = torch.empty((M, N), dtype=torch.float32, device=dev)
    lib = lwq.lib()
    code = call_fmt(lwq, fmt, act) | lwq.LWQ_FLAG_OVERLAP
    stream = torch.cuda.Stream(device=dev)
    sp = stream.cuda_stream
    args = (code, W.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K, sp)
    import ctypes
    cfg = lwq.lwq_config()
    plan_args = (code, M, N, K, ctypes.byref(cfg))
    # the same entry points with the same arguments except M = 0, refused by their first check:
    # what ctypes itself costs for each signature
    call0_args = (code, W.data_ptr(), x.data_ptr(), y.data_ptr(), 0, N, K, sp)
    plan0_args = (code, 0, N, K, ctypes.byref(cfg))
    launches = 0
    per_call, per_call0, per_plan, per_plan0 = [], [], [], []
    for i in range(-2, n // batch):
        stream.synchronize()
        t0 = time.perf_counter()
        for _ in range(batch):
            lib.lwq_matmul(*args)
        t1 = time.perf_counter()
        launches = lib.lwq_last_launch_count()
        stream.synchronize()
        t2 = time.perf_counter()
        for _ in range(batch):
            lib.lwq_matmul(*call0_args)
        t3 = time.perf_counter()
        for _ in range(batch):
            lib.lwq_select_config(*plan_args)
        t4 = time.perf_counter()
        for _ in range(batch):
            lib.lwq_select_config(*plan0_args)
        t5 = time.perf_counter()
        if i >= 0:
            per_call.append((t1 - t0) / batch * 1e6)
            per_call0.append((t3 - t2) / batch * 1e6)
            per_plan.append((t4 - t3) / batch * 1e6)
            per_plan0.append((t5 - t4) / batch * 1e6)
    med, call0 = statistics.median(per_call), statistics.median(per_call0)
    plan, plan0 = statistics.median(per_plan), statistics.median(per_plan0)
    # the library's own host work per call (argument checks, the tile choice, the cached tensor-map
    # lookup and the CUDA launch), and of it the checks and the tile choice alone (lwq_select_config
    # runs the same checks and planner), each less its refused call's cost
    return {"median_us_per_call": round(med, 3), "ctypes_us_per_call": round(call0, 3),
            "library_us_per_call": round(med - call0, 3), "dispatch_us_per_call": round(plan - plan0, 3),
            "calls": n, "kernels_per_call": launches,
            "call": {"fmt": fmt, "act": act, "M": M, "N": N, "K": K}}


def sweep_points(lwq, dev, peaks: dict, fmts=None, shapes=None, Ms=None) -> list:
    """The format x batch sweep (fp16 activations, LWQ_FLAG_OVERLAP, rotating weight copies),
    each point against its binding roofline min(P_tc, BW * I), I = 2MNK / bytes."""
    import torch
    fmts = fmts or inputs.SWEEP_FMTS
    shapes = shapes or inputs.SWEEP_SHAPES_KN
    Ms = Ms or inputs.SWEEP_MS
    bw, ptc = peaks["hbm_gbs"] * 1e9, peaks["bf16_tflops"] * 1e12
    stream = torch.cuda.Stream(device=dev)
    out = []
    for fmt in fmts:
        for K, N in shapes:
            Wq = inputs.make_weights(fmt, inputs.rng(11), N, K)
            R = max(3, -(-(4 * L2_BYTES) // Wq.nbytes))
            base = torch.from_numpy(Wq).to(dev)
            Ws = [base] + [base.clone() for _ in range(R - 1)]
            for M in Ms:
                x = inputs.activations(inputs.rng(12), M, K, "f16")
                xd = torch.from_numpy(x.view(np.int16)).to(dev)
                yd = torch.empty((M, N), dtype=torch.float32, device=dev)
                code = lwq.fmt_code(fmt, "f16") | lwq.LWQ_FLAG_OVERLAP
                cfg = lwq.lwq_select_config(lwq.fmt_code(fmt, "f16"), M, N, K)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.stream(stream):
                    for W in Ws:
                        lwq.lwq_matmul(code, W, xd, yd, M, N, K, stream=stream)
                    stream.synchronize()
                    with torch.cuda.graph(g, stream=stream):
                        for W in Ws:
                            lwq.lwq_matmul(code, W, xd, yd, M, N, K, stream=stream)
                    g.replay()
                    stream.synchronize()
                    reps = max(3, min(50, int(2e-3 / max(1e-6, 1e-5 * len(Ws)))))
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    for _ in range(reps):
                        g.replay()
                    e1.record(stream)
                stream.synchronize()
                ms = e0.elapsed_time(e1) / (reps * len(Ws))
                nbytes, flops = call_bytes(fmt, "f16", M, N, K), call_flops(M, N, K)
                t = ms / 1e3
                attain = min(ptc, bw * flops / nbytes)
                bound = "hbm" if bw * flops / nbytes < ptc else "tensor"
                out.append({"fmt": fmt, "M": M, "K": K, "N": N, "ms": round(ms, 5),
                            "path": {1: "gemv", 2: "gemm", 3: "simple"}[cfg.path],
                            "GB/s": round(nbytes / t / 1e9, 1), "TFLOP/s": round(flops / t / 1e12, 2),
                            "bound": bound, "frac": round(flops / t / attain, 4)})
                del g
            del Ws, base
    return out


def time_attention(lwq, dev, name: str, reps: int, peaks: dict) -> dict:
    """Decode attention through the C ABI: CUDA events around ``reps`` calls, the caches rotated
    over copies that together exceed 4x L2 (every call streams its K and V from HBM)."""
    import torch
    spec = inputs.ATTENTION_WORKLOADS[name]
    B, H, Hkv, L, D = spec["B"], spec["H"], spec["Hkv"], spec["L"], spec["D"]
    q, k, v, lens = inputs.attention_problem(B, H, Hkv, L, D, spec["act"], seed=0)
    dq = torch.from_numpy(q).to(dev)
    cache_bytes = 2 * k.nbytes
    copies = max(1, -(-4 * L2_BYTES // cache_bytes))
    ks = [torch.from_numpy(k).to(dev)]
    vs = [torch.from_numpy(v).to(dev)]
    for _ in range(copies - 1):
        ks.append(ks[0].clone())
        vs.append(vs[0].clone())
    out = torch.empty((B, H, D), dtype=torch.float32, device=dev)
    code = lwq.LWQ_ACT_F16 if spec["act"] == "f16" else lwq.LWQ_ACT_BF16
    scale = D ** -0.5
    n = max(reps, 3 * copies)
    for i in range(3):
        lwq.lwq_attention_decode(code, dq, ks[i % copies], vs[i % copies], None, out, B, H, Hkv, L, D, scale)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n):
        lwq.lwq_attention_decode(code, dq, ks[i % copies], vs[i % copies], None, out, B, H, Hkv, L, D, scale)
    e1.record()
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) * 1e3 / n
    nbytes = cache_bytes + q.nbytes + out.numel() * 4
    gbs = nbytes / us / 1e3
    return {"shape": {"B": B, "H": H, "Hkv": Hkv, "L": L, "D": D, "dtype": spec["act"]}, "calls": n,
            "us_per_call": round(us, 2), "launches_per_call": lwq.lwq_last_launch_count(),
            "bytes_per_call": int(nbytes), "value": round(gbs, 1), "unit": "GB/s",
            "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4), "cache_copies": copies}


def run_gpu_arm(args):
    import torch
    import torch.distributed as dist
    import block_quantized_matmul_lwq_b200 as lwq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if dist_on:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    peaks, peak_src = load_peaks()
    ws_bytes = 0
    for wl in [HEADLINE] + args.extra:
        for fmt, act, M, N, K, seed in step_calls(wl):
            ws_bytes = max(ws_bytes, lwq.lwq_workspace_size(call_fmt(lwq, fmt, act), M, N, K))
    if not args.no_sweep:
        ws_bytes = max([ws_bytes] + [lwq.lwq_workspace_size(lwq.fmt_code(f, "f16"), max(inputs.SWEEP_MS), n, k)
                                     for f in inputs.SWEEP_FMTS for k, n in inputs.SWEEP_SHAPES_KN])
    if not args.no_attention:
        ws_bytes = max([ws_bytes] + [lwq.lwq_attention_workspace_size(s["B"], s["H"], s["Hkv"], s["L"], s["D"])
                                     for s in inputs.ATTENTION_WORKLOADS.values()])
    ws = torch.zeros(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    lwq.lwq_init(ws, ws.numel())

    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    sampler = ClockSampler(gpu_index)
    with sampler:
        prob, ms_local, ms, lps, per = time_workload(lwq, HEADLINE, dev, args.steps, args.warmup, dist_on)
    clocks = sampler.summary()

    bytes_all = reduce_sum(float(prob.bytes_per_step * args.steps), dist_on, dev)
    value = bytes_all / (ms / 1e3) / 1e9
    # roofline: every launch in the timed region is the headline kernel (tensor-core GEMV,
    # Q4_0 x fp32); achieved = algorithmic bytes per step / device time per step on this rank
    achieved = prob.bytes_per_step / (ms_local / args.steps / 1e3) / 1e9
    traffic = args.traffic if args.traffic is not None else profiled_traffic(HEADLINE)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                "algorithmic_bytes_per_step": prob.bytes_per_step, "per": "step (three launches: M=1, 4, 8)",
                "peak_source": peak_src,
                "kernel": "lwq::gemv_kernel<Q4_0, fp32 x> (M=1: one column tile, M=4: two, M=8: three)",
                "per_call_ms": [{"M": p["call"][2], "ms": round(p["ms_mean"], 5),
                                 "GB/s": round(call_bytes(*p["call"][:5]) / p["ms_mean"] / 1e6, 1)} for p in per]}

    e2e_ms, e2e_bytes, h2d, d2h = e2e_workload(lwq, HEADLINE, dev, args.e2e_steps, dist_on)
    e2e_all = reduce_sum(float(e2e_bytes * args.e2e_steps), dist_on, dev)
    e2e = {"value": round(e2e_all / (e2e_ms / 1e3) / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": args.e2e_steps}

    extra = {}
    for wl in args.extra:
        gemm = wl.endswith("prefill_gemm")
        # the prefill GEMMs run long enough (about a second) for the clocks to settle under the
        # power cap, sampled meanwhile: the sustained bf16 peak is their denominator
        nsteps = max(args.extra_steps, args.gemm_steps) if gemm else args.extra_steps
        wl_sampler = ClockSampler(gpu_index)
        with wl_sampler:
            p2, _, ms2, lps2, per2 = time_workload(lwq, wl, dev, nsteps, 3, dist_on)
        rec = {"steps": nsteps, "ms_per_step": round(ms2 / nsteps, 5), "launches_per_step": lps2}
        if gemm:
            tflops = p2.flops_per_step * nsteps / (ms2 / 1e3) / 1e12
            rec.update({"value": round(tflops, 2), "unit": "TFLOP/s",
                        "frac_of_bf16_sustained": round(tflops / peaks["bf16_tflops_sustained"], 4),
                        "frac_of_bf16_peak": round(tflops / peaks["bf16_tflops"], 4),
                        "clocks": wl_sampler.summary(),
                        "per_call": [{"M": p["call"][2], "N": p["call"][3], "K": p["call"][4],
                                      "ms": round(p["ms_mean"], 4),
                                      "TFLOP/s": round(call_flops(*p["call"][2:5]) / p["ms_mean"] / 1e9, 1)}
                                     for p in per2]})
        else:
            gbs = p2.bytes_per_step * nsteps / (ms2 / 1e3) / 1e9
            rec.update({"value": round(gbs, 1), "unit": "GB/s", "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
                        "per_call": [{"M": p["call"][2], "N": p["call"][3], "K": p["call"][4],
                                      "ms": round(p["ms_mean"], 5),
                                      "GB/s": round(call_bytes(*p["call"][:5]) / p["ms_mean"] / 1e6, 1),
                                      "path": call_path(lwq, *p["call"][:5])}
                                     for p in per2]})
        extra[wl] = rec

    attention = None
    if not args.no_attention:
        attention = {name: time_attention(lwq, dev, name, args.extra_steps, peaks)
                     for name in inputs.ATTENTION_WORKLOADS}

    host = host_enqueue_cost(lwq, dev) if not args.no_host_cost else None
    sweep = None
    if not args.no_sweep:
        sweep = {"act": "f16", "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"],
                                         "source": peak_src},
                 "frac": "achieved / min(P_tc, BW * I), I = 2MNK / (packed W + x + y bytes)",
                 "points": sweep_points(lwq, dev, peaks)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(HEADLINE, budget_s=args.cpu_budget)

    torch.cuda.synchronize(dev)
    err = lwq.lwq_get_device_error()
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 6), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": HEADLINE, "weights": "q4_0 (codes q - 8 exact, block scale in fp32)",
                       "activations": "f32, all 24 significand bits (three exact bf16 parts)",
                       "mma": "bf16 x bf16 products (exact), f32 accumulation",
                       "accumulate": "f32", "M": [1, 4, 8], "N": 11008, "K": 4096, "seed": 0,
                       "l2": f"inputs larger than L2: every call reads its own weight copy, "
                             f"{prob.copies_bytes / 1e6:.0f} MB of copies in rotation",
                       "parallelism": f"replicas x{world}", "timing": "CUDA graphs of one weight rotation (R steps), CUDA events",
                       "launch": "LWQ_FLAG_OVERLAP: programmatic dependent launches, weights constant"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": lps * args.steps, "clocks": clocks, "workloads": extra, "attention": attention,
            "host_enqueue": host, "sweep": sweep,
            "device_error": err,
        }
        print(json.dumps(line), flush=True)
    if dist_on:
        dist.barrier()
        dist.destroy_process_group()
    lwq.lwq_shutdown()


def run_sweep(args):
    """The format x batch sweep alone: one JSON line per point."""
    import torch
    import block_quantized_matmul_lwq_b200 as lwq
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    ws_bytes = max(lwq.lwq_workspace_size(lwq.fmt_code(f, "f16"), 1024, n, k)
                   for f in inputs.SWEEP_FMTS for k, n in inputs.SWEEP_SHAPES_KN)
    ws = torch.zeros(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    lwq.lwq_init(ws, ws.numel())
    for rec in sweep_points(lwq, dev, peaks):
        rec.update({"sweep": True, "act": "f16", "peak_source": peak_src})
        print(json.dumps(rec), flush=True)
    torch.cuda.synchronize(dev)
    err = lwq.lwq_get_device_error()
    print(json.dumps({"sweep_done": True, "device_error": err}), flush=True)
    lwq.lwq_shutdown()


def run_reference_arm(args):
    """The oracle (the deliberately slow CPU definition) on the host cores, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    calls = step_calls(HEADLINE)
    threads = oracle.max_threads()
    # size each step's row sample so that warmup + steps fit the budget
    budget = args.reference_budget
    probe_rows = 32
    t0 = time.perf_counter()
    data = []
    for fmt, act, M, N, K, seed in calls:
        g = inputs.rng(seed)
        Wq = inputs.make_weights(fmt, g, probe_rows, K)
        x = inputs.activations(inputs.rng(seed + 1000003), M, K, act)
        data.append((fmt, act, M, K, Wq, x))
    t_probe = time.perf_counter()
    for fmt, act, M, K, Wq, x in data:
        oracle.matmul(fmt, Wq, x, act=act)
    per_row = (time.perf_counter() - t_probe) / probe_rows
    rows = int(budget / max(1, args.steps + args.warmup) / max(per_row, 1e-9))
    rows = max(1, min(rows, 11008))
    data = []
    for fmt, act, M, N, K, seed in calls:
        g = inputs.rng(seed)
        Wq = inputs.make_weights(fmt, g, rows, K)
        x = inputs.activations(inputs.rng(seed + 1000003), M, K, act)
        data.append((fmt, act, M, K, Wq, x))
    for _ in range(args.warmup):
        for fmt, act, M, K, Wq, x in data:
            oracle.matmul(fmt, Wq, x, act=act)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for fmt, act, M, K, Wq, x in data:
            oracle.matmul(fmt, Wq, x, act=act)
    dt = time.perf_counter() - t0
    step_bytes = sum(call_bytes(fmt, act, M, rows, K) for fmt, act, M, K, Wq, x in data)
    value = step_bytes * args.steps / dt / 1e9
    sample = f"first {rows} of 11008 weight rows of every call of a step (M=1,4,8; K=4096)"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus":
            int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": HEADLINE, "weights": "q4_0", "activations": "f32", "M": [1, 4, 8], "N": 11008,
                   "K": 4096, "seed": 0},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=60)
    ap.add_argument("--impl", choices=["lwq", "reference"], default="lwq")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--extra-steps", type=int, default=400)
    ap.add_argument("--gemm-steps", type=int, default=4000,
                    help="steps of each prefill GEMM workload (about a second, so the clocks settle)")
    ap.add_argument("--extra", nargs="*", default=["q8_0_gemv_4096x4096", "q4_k_7b_layer_decode",
                                                   "q4_k_7b_layer_decode_fused", "q4_0_gemv_11008x4096_act_i8",
                                                   "q4_k_7b_layer_decode_act_i8",
                                                   "q4_0_prefill_gemm", "q6_k_7b_layer_decode",
                                                   "q5_k_7b_layer_decode", "q2_k_7b_layer_decode",
                                                   "q6_k_prefill_gemm", "q5_k_prefill_gemm", "q2_k_prefill_gemm"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="leave the format x batch sweep out of the line")
    ap.add_argument("--no-host-cost", action="store_true", help="leave the host enqueue timing out")
    ap.add_argument("--no-attention", action="store_true", help="leave the decode-attention workloads out")
    ap.add_argument("--sweep", action="store_true",
                    help="time the format x batch sweep instead (one JSON line per point)")
    ap.add_argument("--case", default=None,
                    help="time one workload alone (a name from inputs.WORKLOADS or inputs.ATTENTION_WORKLOADS) "
                         "and print its own JSON line: a small command for profilers")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--reference-budget", type=float, default=60.0)
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu DRAM bytes per step of the headline kernels (default: profiles/traffic.json, "
                         "when the CUDA sources still match it)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    return args


def run_case(args):
    """One workload alone, on one GPU (the command the ncu captures under profiles/ run)."""
    import torch
    import block_quantized_matmul_lwq_b200 as lwq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, _ = load_peaks()
    if args.case in inputs.ATTENTION_WORKLOADS:
        spec = inputs.ATTENTION_WORKLOADS[args.case]
        need = lwq.lwq_attention_workspace_size(spec["B"], spec["H"], spec["Hkv"], spec["L"], spec["D"])
        ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
        lwq.lwq_init(ws, ws.numel())
        rec = time_attention(lwq, dev, args.case, args.steps, peaks)
    else:
        need = max(lwq.lwq_workspace_size(call_fmt(lwq, f, a), M, N, K) for f, a, M, N, K, _ in step_calls(args.case))
        ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
        lwq.lwq_init(ws, ws.numel())
        prob, ms_local, ms, lps, per = time_workload(lwq, args.case, dev, args.steps, args.warmup, False)
        rec = {"ms_per_step": round(ms / args.steps, 5), "launches_per_step": lps,
               "per_call_ms": [round(p["ms_mean"], 5) for p in per]}
    print(json.dumps({"case": args.case, **rec}), flush=True)
    lwq.lwq_shutdown()


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference_arm(args)
    elif args.sweep:
        run_sweep(args)
    elif args.case:
        run_case(args)
    else:
        run_gpu_arm(args)


if __name__ == "__main__":
    main()
