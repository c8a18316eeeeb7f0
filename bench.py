"""Benchmark of the B200 FP8 block-scaled NT GEMM (dense sweep + grouped forms).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One STEP is one pass over the dense sweep of the DeepGEMM performance table:
M in {64, 128, 4096} x (N, K) in {(2112,7168), (24576,1536), (32768,512),
(7168,16384), (4096,7168), (7168,2048)}, e4m3 inputs with 1x128 / 128x128 FP32
scales, bf16 output -- 18 GEMMs through the C ABI.  Inputs are larger than L2:
each shape cycles over enough copies of its operands (>= 3 x the 126 MB L2 in
total) that every launch reads operands last touched at least 3 x L2 of other
traffic ago.  The K launches of each shape are captured in one CUDA graph and
timed with CUDA events around its replay on the capture stream (after one
untimed replay that uploads the graph), so host launch overhead stays out of
microsecond-scale decode shapes.  ``value`` is the
aggregate TFLOP/s of the sweep (sum of flops / sum of kernel times), max over
ranks for N > 1 (each rank runs the same sweep on its own GPU: weak scaling, no
collective on the data path).  Per shape, ``us_flushed`` is also given: a
single eager launch timed with events after a 512 MiB L2-flush write (dirty
L2, launch overhead included).  The grouped contiguous and masked workloads are
timed like the sweep and reported under ``grouped``.  ``e2e`` is the same sweep measured around
pinned-host -> device copies of every input, the GEMM and the device -> host
copy of D, with the three on their own streams so that the copies of one
shape overlap the GEMM of another (``serial_value``: all on one stream).  ``cpu_baseline`` times the CPU oracle on a bounded row sample.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as wl  # noqa: E402

SPEC_FP8_TFLOPS = 4500.0    # B200 dense FP8 datasheet figure
SPEC_HBM_GBS = 8000.0       # HBM3e datasheet figure used by the target
FP8_PER_BF16 = 2.0          # nominal dense FP8 : BF16 tensor ratio (4.5 : 2.25 PF)
L2_FLUSH_BYTES = 512 << 20
L2_BYTES = 126_000_000      # B200 L2 capacity
ROTATE_FACTOR = 3           # other traffic between two reads of one input copy, in L2 sizes


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            m = json.load(f)
        return {"hbm_gbs": float(m["hbm_gbs"]), "bf16_tflops": float(m["bf16_tflops"]),
                "bf16_tflops_sustained": float(m.get("bf16_tflops_sustained", m["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------ distributed ---

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def dist_init(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate(total_flops_per_rank: float, seconds_max: float, world: int) -> float:
    """Whole-job TFLOP/s: the work of all ranks over the slowest rank's time."""
    return total_flops_per_rank * world / seconds_max / 1e12


# ---------------------------------------------------------------- clocks ----

class ClockSampler:
    """Samples SM clock, max clock, power and clock-event reasons every 5 ms
    through NVML (read-only queries, the data nvidia-smi prints) while active."""

    REASONS = {"sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, gpu_index: int, period_s: float = 0.005):
        self.gpu, self.period = gpu_index, period_s
        self.samples, self.thread, self.stop = [], None, None
        self.nvml = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.gpu]) if vis and vis.split(",")[0].isdigit() else self.gpu
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None
            return self
        self.stop = threading.Event()

        def loop():
            n = self.nvml
            while not self.stop.is_set():
                try:
                    sm = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
                    rs = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                    pw = n.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                    self.samples.append((sm, rs, pw))
                except Exception:
                    pass
                self.stop.wait(self.period)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=2)

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        n = self.nvml
        reasons = sorted({name for _, rs, _ in self.samples for name, attr in self.REASONS.items()
                          if rs & getattr(n, attr, 0)})
        sm = [x[0] for x in self.samples]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "sm_mhz_min": min(sm),
                "power_w_max": round(max(x[2] for x in self.samples), 1), "reasons": reasons,
                "samples": len(self.samples), "source": "nvml, every 5 ms during the timed steps"}


# ------------------------------------------------------------------ ours ----

class Problem:
    def __init__(self, case: wl.Case, dg):
        self.case = case
        self.dg = dg
        c = case
        if c.mode == "masked":
            self.D = torch.empty(c.G, c.M, c.N, dtype=torch.bfloat16, device="cuda")
        else:
            self.D = torch.empty(c.M, c.N, dtype=torch.bfloat16, device="cuda")
        self.flops = c.flops()
        self.bytes = c.bytes()
        mode = {"dense": 0, "contiguous": 1, "masked": 2}[c.mode]
        self.plan = dg.dg_make_plan(mode, c.M, c.N, c.K, c.G, dg.dg_get_num_sms())
        pl = self.plan
        # Names of the C++ template instances the call launches.
        if pl["swap_ab"]:
            self.kernel = f"fp8_gemm_swapab_kernel<{pl['block_m']}, {mode}>"
        else:
            self.kernel = f"fp8_gemm_kernel<{pl['block_n']}, {pl['stages']}, {mode}, 0>"

    def run(self, case=None, D=None):
        c = case or self.case
        D = self.D if D is None else D
        if c.mode == "dense":
            self.dg.dg_fp8_gemm_nt(D, c.A, c.sa, c.sa_stride, c.B, c.sb)
        elif c.mode == "contiguous":
            self.dg.dg_grouped_contiguous_nt(D, c.A, c.sa, c.sa_stride, c.B, c.sb, c.m_indices)
        else:
            self.dg.dg_grouped_masked_nt(D, c.A, c.sa, c.sa_stride, c.B, c.sb, c.masked_m)


def kernel_source_sha() -> str:
    """Hash of the device code that defines the dominant kernel instance (the
    persistent GEMM kernel and the PTX helpers it uses)."""
    import hashlib
    h = hashlib.sha256()
    for f in [os.path.join(ROOT, "moe_grouped_gemm_weight_b200", "csrc", n) for n in ("dg_kernel.cuh", "dg_ptx.cuh")]:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch recorded by ncu under profiles/ for `kernel`, if the
    kernel sources have not changed since the capture (else None)."""
    import glob
    for path in glob.glob(os.path.join(ROOT, "profiles", "dram_traffic_*.txt")):
        kv = {}
        with open(path) as f:
            for line in f:
                if "=" in line and not line.startswith("#") and " " not in line.split("=")[0].strip():
                    k, v = line.split("=", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("kernel") == kernel and kv.get("kernel_source_sha") == kernel_source_sha():
            return int(kv["traffic_per_launch"]), os.path.relpath(path, ROOT)
    return None, None


def roof_time_s(flops, byts, tflops, gbs):
    return max(flops / (tflops * 1e12), byts / (gbs * 1e9))


def time_problems(problems, flush, reps: int):
    """Per-problem list of kernel times (s), L2 flushed before every launch."""
    stream = torch.cuda.current_stream()
    times = [[] for _ in problems]
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in problems]
    for _ in range(reps):
        for i, p in enumerate(problems):
            flush.zero_()
            evs[i][0].record(stream)
            p.run()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        for i in range(len(problems)):
            times[i].append(evs[i][0].elapsed_time(evs[i][1]) * 1e-3)
    return times


def footprint(c: wl.Case) -> int:
    """Device bytes of one launch's operands, scales, index arrays and output."""
    ts = [c.A, c.sa, c.B, c.sb] + [t for t in (c.m_indices, c.masked_m) if t is not None]
    out = (c.G if c.mode == "masked" else 1) * c.M * c.N * 2
    return sum(t.numel() * t.element_size() for t in ts) + out


def copies_needed(c: wl.Case) -> int:
    return min(64, max(2, -(-ROTATE_FACTOR * L2_BYTES // footprint(c))))


class RotatingGraph:
    """`launches` calls of one problem captured in a CUDA graph, cycling over
    copies of its inputs (distinct buffers, same values) and outputs."""

    def __init__(self, p: Problem, launches: int, warmup: int, stream):
        c = p.case
        self.p, self.launches, self.stream = p, launches, stream
        self.copies = copies_needed(c)
        self.reps = [(c, p.D)]
        for _ in range(self.copies - 1):
            cc = wl.Case(c.mode, c.M, c.N, c.K, c.G, c.A.clone(), c.sa.clone(), c.sa_stride, c.B.clone(),
                         c.sb.clone(), m_indices=c.m_indices, masked_m=c.masked_m)
            self.reps.append((cc, torch.empty_like(p.D)))
        with torch.cuda.stream(stream):
            # eager warm-up on the capture stream: first-call set-up of every
            # kernel instance and of the stream's K-split workspace
            for i in range(max(warmup, 1) * self.copies):
                rc, rd = self.reps[i % self.copies]
                p.run(case=rc, D=rd)
        stream.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=stream):
            for i in range(launches):
                rc, rd = self.reps[i % self.copies]
                p.run(case=rc, D=rd)
        self.ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        # The first replay of a graph also uploads it (about 2 us per launch
        # for microsecond kernels): do it untimed.
        with torch.cuda.stream(stream):
            self.graph.replay()
        stream.synchronize()

    def replay(self):
        # CUDAGraph.replay launches on the current stream: make it the one the
        # events are recorded on
        with torch.cuda.stream(self.stream):
            self.ev[0].record(self.stream)
            self.graph.replay()
            self.ev[1].record(self.stream)

    def seconds_per_launch(self) -> float:
        return self.ev[0].elapsed_time(self.ev[1]) * 1e-3 / self.launches


class Ue8m0Problem(Problem):
    """A dense problem with power-of-two scales, run through a chosen entry
    point: "promote" (dg_fp8_gemm_nt), "ue8m0" (dg_fp8_gemm_nt_ue8m0, routed)
    or "block_scaled" (the same call with DG_FORCE_BLOCK_SCALED=1)."""

    def __init__(self, case, dg, path):
        super().__init__(case, dg)
        self.path = path

    def run(self, case=None, D=None):
        c = case or self.case
        D = self.D if D is None else D
        if self.path == "promote":
            self.dg.dg_fp8_gemm_nt(D, c.A, c.sa, c.sa_stride, c.B, c.sb)
        else:
            prev = os.environ.pop("DG_FORCE_BLOCK_SCALED", None)
            if self.path == "block_scaled":
                os.environ["DG_FORCE_BLOCK_SCALED"] = "1"
            try:
                self.dg.dg_fp8_gemm_nt_ue8m0(D, c.A, c.sa, c.sa_stride, c.B, c.sb)
            finally:
                os.environ.pop("DG_FORCE_BLOCK_SCALED", None)
                if prev is not None:
                    os.environ["DG_FORCE_BLOCK_SCALED"] = prev


# The block-scaled comparison shapes; the last two are the stress workload
# (heavy-tailed activations with power-of-two scales, workloads.STRESS_SHAPES).
UE8M0_SHAPES = [(4096, 32768, 512), (4096, 24576, 1536), (4096, 7168, 2048)] + list(wl.STRESS_SHAPES)


def time_ue8m0(dg, launches: int, warmup: int, stream) -> list:
    """Power-of-two scales (the stress generator): each shape through the three
    paths, each as a CUDA graph over input copies larger than L2."""
    out = []
    for (m, n, k) in UE8M0_SHAPES:
        case = wl.dense_case(m, n, k, seed=0, stress=True, device="cuda")
        row = {"M": m, "N": n, "K": k, "flops": case.flops(), "bytes": case.bytes()}
        for path in ("promote", "ue8m0", "block_scaled"):
            pr = Ue8m0Problem(case, dg, path)
            gr = RotatingGraph(pr, launches, warmup, stream)
            gr.replay()
            torch.cuda.synchronize()
            t = gr.seconds_per_launch()
            row[f"us_{path}"] = round(t * 1e6, 2)
            row[f"tflops_{path}"] = round(pr.flops / t / 1e12, 1)
            del gr
        out.append(row)
    return out


class LayoutProblem(Problem):
    """A dense problem run with its operands stored in another order (the same
    values, transposed copies): "nt", "nn", "tn" or "tt"."""

    def __init__(self, case, dg, layout):
        super().__init__(case, dg)
        self.layout = layout
        self.kernel = self.kernel.replace(", 0>", f", {dict(nt=0, tt=1, nn=2, tn=3)[layout]}>")

    def run(self, case=None, D=None):
        c = case or self.case
        D = self.D if D is None else D
        a_t, b_t = self.layout[0] == "t", self.layout[1] == "n"
        key = (c.A.data_ptr(), c.B.data_ptr())
        cache = self.__dict__.setdefault("_stored", {})
        if key not in cache:  # transposed copies, made once per input copy (untimed warm-up)
            cache[key] = (c.A.t().contiguous() if a_t else c.A, c.B.t().contiguous() if b_t else c.B)
        A, B = cache[key]
        getattr(self.dg, f"dg_fp8_gemm_{self.layout}")(D, A, c.sa, c.sa_stride, B, c.sb)


LAYOUT_SHAPES = [(4096, 7168, 16384), (4096, 4096, 7168)]


def time_layouts(dg, launches: int, warmup: int, stream) -> list:
    out = []
    for (m, n, k) in LAYOUT_SHAPES:
        case = wl.dense_case(m, n, k, seed=0, device="cuda")
        row = {"M": m, "N": n, "K": k}
        for layout in ("nt", "nn", "tn", "tt"):
            pr = LayoutProblem(case, dg, layout)
            gr = RotatingGraph(pr, launches, warmup, stream)
            gr.replay()
            torch.cuda.synchronize()
            t = gr.seconds_per_launch()
            row[f"us_{layout}"] = round(t * 1e6, 2)
            row[f"tflops_{layout}"] = round(pr.flops / t / 1e12, 1)
            del gr, pr
        out.append(row)
    return out


# K-grouped GEMM (MoE weight gradient): experts x tokens per expert, M x N.
KGROUPED = {"M": 7168, "N": 2048, "tokens": [4096, 4096, 4096, 4096]}


def time_k_grouped(dg, launches: int, warmup: int, stream) -> dict:
    """The K-grouped GEMM as a CUDA graph over input copies larger than L2."""
    M, N, counts = KGROUPED["M"], KGROUPED["N"], KGROUPED["tokens"]
    K = sum(counts)
    case = wl.dense_case(M, N, K, seed=0, device="cuda")
    offsets = torch.tensor([0] + list(torch.tensor(counts).cumsum(0).tolist()), dtype=torch.int32, device="cuda")
    G = len(counts)
    footprint = 2 * M * K + N * K + 2 * G * M * N
    copies = min(64, max(2, -(-ROTATE_FACTOR * L2_BYTES // footprint)))
    reps = [(case.A.t().contiguous(), case.B.t().contiguous(),
             torch.empty(G, M, N, dtype=torch.bfloat16, device="cuda")) for _ in range(copies)]

    def call(i):
        At, Bt, D = reps[i % copies]
        dg.dg_k_grouped_fp8_gemm_tn(D, At, case.sa, case.sa_stride, Bt, case.sb, offsets)

    with torch.cuda.stream(stream):
        for i in range(max(warmup, 1) * copies):
            call(i)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(launches):
            call(i)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        graph.replay()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) * 1e-3 / launches
    flops = 2.0 * M * N * K
    nbytes = M * K + N * K + 2 * G * M * N + 4 * M * (K // 128) + 4 * (-(-N // 128)) * (K // 128)
    del graph, reps
    return {"workload": f"K-grouped (weight gradient) G={G} tokens={counts} M={M} N={N}", "us": round(t * 1e6, 2),
            "tflops": round(flops / t / 1e12, 1), "gbs": round(nbytes / t / 1e9, 1), "input_copies": copies}


# FP8 cast workloads: (kind, rows, K); "1x128" = activations, "128x128" = weights.
CAST_SHAPES = [("1x128", 4096, 7168), ("1x128", 32768, 7168), ("1x128", 128, 7168), ("1x128", 64, 7168),
               ("128x128", 7168, 16384), ("128x128", 4096, 7168)]


def time_casts(dg, launches: int, warmup: int, stream) -> list:
    """Each cast shape as a CUDA graph of `launches` calls over input copies
    larger than L2 (like the GEMMs); one untimed replay first."""
    out = []
    for kind, R, K in CAST_SHAPES:
        in_bytes = R * K * 2
        copies = min(64, max(2, -(-ROTATE_FACTOR * L2_BYTES // (in_bytes + R * K))))
        g = torch.Generator(device="cuda").manual_seed(R + K)
        X0 = torch.randn(R, K, generator=g, device="cuda").to(torch.bfloat16)
        bufs = []
        for _ in range(copies):
            nsc = (K // 128) * R if kind == "1x128" else -(-R // 128) * (K // 128)
            bufs.append((X0.clone(), torch.empty(R, K, dtype=torch.uint8, device="cuda"),
                         torch.empty(nsc, dtype=torch.float32, device="cuda")))

        def call(i):
            X, Q, sc = bufs[i % copies]
            if kind == "1x128":
                dg.dg_to_fp8_1x128(Q, sc, R, X)
            else:
                dg.dg_to_fp8_128x128(Q, sc, X)

        with torch.cuda.stream(stream):
            for i in range(max(warmup, 1) * copies):
                call(i)
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(launches):
                call(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            graph.replay()
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) * 1e-3 / launches
        nbytes = R * K * 3 + 4 * R * (K // 128) if kind == "1x128" else R * K * 3 + 4 * (-(-R // 128)) * (K // 128)
        out.append({"cast": kind, "rows": R, "K": K, "us": round(t * 1e6, 2), "gbs": round(nbytes / t / 1e9, 1),
                    "algorithmic_bytes": nbytes, "input_copies": copies})
        del graph, bufs
    return out


def oracle_rows_sample(c: wl.Case, nrows: int, salt: int = 0):
    """A deterministic spread of nrows distinct row indices of a case."""
    import numpy as np
    n = min(nrows, c.M)
    return np.array(sorted({(salt + i * 9973) % c.M for i in range(n)}), dtype=np.int64)


def cpu_baseline(problems, budget_s: float = 15.0) -> dict:
    """The CPU oracle, as it stands, on a bounded row sample of every shape.

    The oracle parallelises over output rows, so each call gets one row per
    host thread; calls repeat per shape until that shape's share of the budget
    is spent."""
    import oracle
    threads = oracle.num_threads()
    flops, t_total = 0.0, 0.0
    sample = []
    per_shape_budget = budget_s / len(problems)
    for p in problems:
        c = p.case
        A, sa, B, sb = c.A.cpu().numpy(), c.sa.cpu().numpy(), c.B.cpu().numpy(), c.sb.cpu().numpy()
        spent, nrows, calls = 0.0, 0, 0
        while spent < per_shape_budget:
            rows = oracle_rows_sample(c, threads, salt=calls)
            t0 = time.perf_counter()
            oracle.gemm_nt(A, sa, c.sa_stride, B, sb, c.M, c.N, c.K, rows=rows, want_d64=False, want_mag=False)
            spent += time.perf_counter() - t0
            nrows += len(rows)
            calls += 1
        flops += 2.0 * nrows * c.N * c.K
        t_total += spent
        sample.append(f"{c.M}x{c.N}x{c.K}:{nrows}rows")
    return {"value": flops / t_total / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": "all N columns of a few rows of every dense-sweep shape (" + ", ".join(sample) + ")",
            "seconds": round(t_total, 2)}


def run_ours(args, rank, world, local):
    torch.cuda.set_device(local)
    dist_init(world, "nccl")
    from moe_grouped_gemm_weight_b200 import build as dgbuild
    dgbuild.build()
    import moe_grouped_gemm_weight_b200 as dg

    peaks = load_peaks()
    # Each shape's timed launches are one CUDA-graph replay of a few to tens
    # of milliseconds, about as long as the measured burst GEMM: fractions are
    # taken against the burst peak, with the sustained one (a seconds-long run
    # under the power cap) reported beside it.
    p_fp8_burst = peaks["bf16_tflops"] * FP8_PER_BF16
    p_fp8_sust = peaks["bf16_tflops_sustained"] * FP8_PER_BF16
    dev = torch.device("cuda", local)

    shapes = wl.DENSE_SWEEP
    if args.shape:
        shapes = [tuple(int(x) for x in args.shape.lower().split("x"))]
    problems = [Problem(wl.dense_case(m, n, k, seed=0, device="cuda"), dg) for (m, n, k) in shapes]
    grouped = [] if args.no_grouped else [
        Problem(wl.contiguous_case(device="cuda", seed=0, **wl.CONTIGUOUS_MAIN), dg),
        Problem(wl.masked_case(device="cuda", seed=0, **wl.MASKED_MAIN), dg),
        Problem(wl.masked_case(device="cuda", seed=0, **wl.MASKED_SINGLE), dg)]
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    step_flops = float(sum(p.flops for p in problems))

    # untimed: W warm-up launches per shape, then capture of the K timed launches
    cap_stream = torch.cuda.Stream(device=dev)
    graphs = [RotatingGraph(p, args.steps, args.warmup, cap_stream) for p in problems]
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps (K launches of each of the 18 shapes) ----
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    with ClockSampler(local) as clk:
        for gr in graphs:
            gr.replay()
        torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall0
    barrier(world)
    clocks = clk.summary()
    times = [gr.seconds_per_launch() for gr in graphs]   # mean kernel time per launch

    kernel_s = sum(times) * args.steps                   # K steps of kernel time
    kernel_s_max = max_over_ranks(kernel_s, world, dev)
    value = aggregate(step_flops * args.steps, kernel_s_max, world)
    ms_per_step = kernel_s_max / args.steps * 1e3

    # for comparison: single eager launches after an L2-flush write (untimed region)
    flushed = time_problems(problems, flush, max(3, min(args.steps, 20)))

    per_shape = []
    for p, tm, gr, tf in zip(problems, times, graphs, flushed):
        c = p.case
        per_shape.append({
            "M": c.M, "N": c.N, "K": c.K, "us": round(tm * 1e6, 2),
            "tflops": round(p.flops / tm / 1e12, 1), "gbs": round(p.bytes / tm / 1e9, 1),
            "frac_roof_spec": round(roof_time_s(p.flops, p.bytes, SPEC_FP8_TFLOPS, SPEC_HBM_GBS) / tm, 3),
            "frac_roof_measured": round(roof_time_s(p.flops, p.bytes, p_fp8_burst, peaks["hbm_gbs"]) / tm, 3),
            "frac_roof_measured_sustained": round(roof_time_s(p.flops, p.bytes, p_fp8_sust, peaks["hbm_gbs"]) / tm, 3),
            "bound": "tensor" if p.flops / p_fp8_burst / 1e12 > p.bytes / peaks["hbm_gbs"] / 1e9 else "hbm",
            "kernel": p.kernel, "input_copies": gr.copies,
            "us_flushed": round(statistics.median(tf) * 1e6, 2),
            "frac_roof_measured_flushed": round(
                roof_time_s(p.flops, p.bytes, p_fp8_burst, peaks["hbm_gbs"]) / statistics.median(tf), 3),
        })
    del graphs

    # dominant kernel instance: the one with the largest share of step time
    by_kernel = {}
    for p, t in zip(problems, times):
        d = by_kernel.setdefault(p.kernel, {"flops": 0.0, "bytes": 0.0, "s": 0.0, "launches": 0})
        d["flops"] += p.flops * args.steps
        d["bytes"] += p.bytes * args.steps
        d["s"] += t * args.steps
        d["launches"] += args.steps
    dom_name, dom = max(by_kernel.items(), key=lambda kv: kv[1]["s"])
    tensor_bound = dom["flops"] / (p_fp8_burst * 1e12) > dom["bytes"] / (peaks["hbm_gbs"] * 1e9)
    if tensor_bound:
        ach = dom["flops"] / dom["s"] / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": round(p_fp8_burst, 1), "unit": "TFLOP/s",
                "frac": round(ach / p_fp8_burst, 3), "peak_sustained": round(p_fp8_sust, 1),
                "frac_sustained": round(ach / p_fp8_sust, 3)}
    else:
        ach = dom["bytes"] / dom["s"] / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / peaks["hbm_gbs"], 3)}
    traffic, traffic_src = recorded_traffic(dom_name)
    roof.update({"traffic": traffic, "traffic_source": traffic_src,
                 "algorithmic_bytes_per_launch": int(dom["bytes"] / dom["launches"]),
                 "kernel": dom_name, "share": round(dom["s"] / kernel_s, 3),
                 "peak_source": f"{peaks['source']} burst (fp8 = {FP8_PER_BF16:g} x bf16 burst); sustained beside it"
                 if tensor_bound else peaks["source"]})

    # grouped workloads (same method, reported alongside; untimed region)
    g_launches = max(3, min(args.steps, 20))
    gtimes, gflushed = [], []
    for p in grouped:
        gr = RotatingGraph(p, g_launches, args.warmup, cap_stream)
        gr.replay()
        torch.cuda.synchronize()
        gtimes.append(gr.seconds_per_launch())
        del gr
    gflushed = time_problems(grouped, flush, g_launches) if grouped else []
    grouped_out = []
    for p, tm, tf in zip(grouped, gtimes, gflushed):
        c = p.case
        grouped_out.append({
            "workload": c.mode + (f" G={c.G} rows={p.case.rows_computed()}" if c.mode == "masked" else
                                  f" G={c.G} M_total={c.M}"),
            "N": c.N, "K": c.K, "us": round(tm * 1e6, 2), "tflops": round(p.flops / tm / 1e12, 1),
            "gbs": round(p.bytes / tm / 1e9, 1),
            "frac_roof_spec": round(roof_time_s(p.flops, p.bytes, SPEC_FP8_TFLOPS, SPEC_HBM_GBS) / tm, 3),
            "frac_roof_measured": round(roof_time_s(p.flops, p.bytes, p_fp8_burst, peaks["hbm_gbs"]) / tm, 3),
            "bound": "tensor" if p.flops / p_fp8_burst / 1e12 > p.bytes / peaks["hbm_gbs"] / 1e9 else "hbm",
            "kernel": p.kernel, "us_flushed": round(statistics.median(tf) * 1e6, 2)})

    casts = [] if args.no_grouped else time_casts(dg, max(3, min(args.steps, 20)), args.warmup, cap_stream)
    ue8m0 = [] if args.no_grouped else time_ue8m0(dg, max(3, min(args.steps, 10)), args.warmup, cap_stream)
    layouts = [] if args.no_grouped else time_layouts(dg, max(3, min(args.steps, 10)), args.warmup, cap_stream)
    kgrouped = None if args.no_grouped else time_k_grouped(dg, max(3, min(args.steps, 10)), args.warmup, cap_stream)
    if kgrouped:
        kgrouped["frac_roof_measured"] = round(kgrouped["tflops"] / p_fp8_burst, 3)
    for row in ue8m0:
        for path in ("promote", "ue8m0", "block_scaled"):
            t = row[f"us_{path}"] * 1e-6
            row[f"frac_{path}"] = round(roof_time_s(row["flops"], row["bytes"], p_fp8_burst, peaks["hbm_gbs"]) / t, 3)
    for c in casts:
        c["frac_hbm_measured"] = round(c["gbs"] / peaks["hbm_gbs"], 3)

    e2e = None
    if not args.no_e2e:
        # end to end: pinned host inputs -> device, GEMM, D -> pinned host
        host = []
        for p in problems:
            c = p.case
            host.append({k: getattr(c, k).cpu().pin_memory() for k in ("A", "sa", "B", "sb")})
        dev_bufs = [{k: torch.empty_like(getattr(p.case, k)) for k in ("A", "sa", "B", "sb")} for p in problems]
        d_host = [torch.empty(p.D.shape, dtype=p.D.dtype).pin_memory() for p in problems]
        h2d = sum(t.numel() * t.element_size() for h in host for t in h.values())
        d2h = sum(t.numel() * t.element_size() for t in d_host)
        # Three streams, one per engine: copies in, GEMMs, copies out.  Shape i's
        # GEMM waits for its inputs; its copy-out waits for the GEMM; the next
        # step's copy into shape i's inputs waits until this step's GEMM has
        # read them, and the next GEMM into D until D has been copied out.
        s_in, s_mm, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in problems]
        ev_mm = [torch.cuda.Event() for _ in problems]
        ev_out = [torch.cuda.Event() for _ in problems]

        def e2e_step():
            for i, (p, h, db, dh) in enumerate(zip(problems, host, dev_bufs, d_host)):
                with torch.cuda.stream(s_in):
                    s_in.wait_event(ev_mm[i])
                    for k in ("A", "sa", "B", "sb"):
                        db[k].copy_(h[k], non_blocking=True)
                    ev_in[i].record(s_in)
                with torch.cuda.stream(s_mm):
                    s_mm.wait_event(ev_in[i])
                    s_mm.wait_event(ev_out[i])
                    c = p.case
                    p.run(case=wl.Case(c.mode, c.M, c.N, c.K, c.G, db["A"], db["sa"], c.sa_stride, db["B"], db["sb"]))
                    ev_mm[i].record(s_mm)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_mm[i])
                    dh.copy_(p.D, non_blocking=True)
                    ev_out[i].record(s_out)

        def e2e_step_serial():
            # the same work in order on one stream, for comparison
            for p, h, db, dh in zip(problems, host, dev_bufs, d_host):
                for k in ("A", "sa", "B", "sb"):
                    db[k].copy_(h[k], non_blocking=True)
                c = p.case
                p.run(case=wl.Case(c.mode, c.M, c.N, c.K, c.G, db["A"], db["sa"], c.sa_stride, db["B"], db["sb"]))
                dh.copy_(p.D, non_blocking=True)

        e2e_steps = max(1, min(args.steps, 3))
        e2e_step()
        torch.cuda.synchronize()
        e2e_step_serial()
        torch.cuda.synchronize()
        barrier(world)
        # pipelined: the timed region opens on the copy-in stream, before the
        # first copy, and closes on the copy-out stream after the last copy,
        # which depends on every earlier copy and GEMM
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        s_mm.wait_event(e0)
        s_out.wait_event(e0)
        for _ in range(e2e_steps):
            e2e_step()
        s_out.wait_stream(s_in)
        s_out.wait_stream(s_mm)
        e1.record(s_out)
        torch.cuda.synchronize()
        e2e_s = max_over_ranks(e0.elapsed_time(e1) * 1e-3, world, dev)
        stream = torch.cuda.current_stream()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(e2e_steps):
            e2e_step_serial()
        f1.record(stream)
        torch.cuda.synchronize()
        serial_s = max_over_ranks(f0.elapsed_time(f1) * 1e-3, world, dev)
        e2e = {"value": round(aggregate(step_flops * e2e_steps, e2e_s, world), 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "pipelined": "copy-in, GEMM and copy-out on three streams, ordered by events",
               "serial_value": round(aggregate(step_flops * e2e_steps, serial_s, world), 3)}

    cpu = cpu_baseline(problems) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None

    # Compact per-workload summary, printed last in the line: [us, fraction of
    # the measured roofline] per shape (fractions against the burst FP8 peak or
    # the measured HBM copy bandwidth, whichever bounds the shape).
    summary = {
        "dense": {f"{r['M']}x{r['N']}x{r['K']}": [r["us"], r["frac_roof_measured"]] for r in per_shape},
        "grouped": {r["workload"]: [r["us"], r["frac_roof_measured"]] for r in grouped_out},
        "stress": {f"{r['M']}x{r['N']}x{r['K']} {path}": [r[f"us_{path}"], r[f"frac_{path}"]]
                   for r in ue8m0 if (r["M"], r["N"], r["K"]) in set(map(tuple, wl.STRESS_SHAPES))
                   for path in ("promote", "ue8m0")},
        "k_grouped": [kgrouped["us"], kgrouped["frac_roof_measured"]] if kgrouped else None,
        "dominant": {"kernel": roof["kernel"], "frac": roof["frac"], "frac_sustained": roof.get("frac_sustained")},
        "frac_is": "of measured roofline: burst FP8 (2 x bf16 burst) or HBM copy bandwidth",
    }
    detail = {"per_shape": per_shape, "grouped": grouped_out, "cast": casts, "ue8m0": ue8m0, "layouts": layouts,
              "k_grouped": kgrouped}
    out = {
        "metric": "FP8 scaled-GEMM TFLOPS per shape; % of B200 FP8 peak or HBM roofline",
        "value": round(value, 1), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 x e4m3 -> f32 accumulate -> bf16",
        "data": "synthetic (seeded randn inputs quantised to e4m3 with 1x128 / 128x128 FP32 scales)",
        "config": {"workload": "dense FP8 NT GEMM sweep, 18 shapes: M in {64,128,4096} x (N,K) in "
                               "{(2112,7168),(24576,1536),(32768,512),(7168,16384),(4096,7168),(7168,2048)}",
                   "l2": "inputs larger than L2: each shape cycles over copies of its inputs totalling "
                         ">= 3 x 126 MB; its K launches run as one CUDA graph, CUDA events around the replay "
                         "(us_flushed per shape: single eager launch after a 512 MiB L2-flush write)",
                   "parallelism": f"replicas x{world} (weak scaling, no data-path collective)",
                   "wall_ms_per_step": round(t_wall / args.steps * 1e3, 3)},
        "clocks": clocks,
        "gpu_launches": len(problems) * args.steps,
        "peaks": {"fp8_tflops_burst": p_fp8_burst, "fp8_tflops_sustained": p_fp8_sust,
                  "hbm_gbs": peaks["hbm_gbs"], "source": peaks["source"],
                  "spec_fp8_tflops": SPEC_FP8_TFLOPS, "spec_hbm_gbs": SPEC_HBM_GBS},
        "detail": args.detail or "not written (pass --detail PATH)",
        "cpu_baseline": cpu,
        "e2e": e2e,
        "roofline": roof,
        "summary": summary,
    }
    if rank == 0:
        if args.detail:
            with open(args.detail, "w") as f:
                json.dump(detail, f, indent=1)
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------- reference ----

def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: each step computes one row per host
    thread of every shape of the sweep (all N columns), a bounded sample."""
    if rank != 0:
        return
    import oracle
    threads = oracle.num_threads()
    cases = [wl.dense_case(m, n, k, seed=0) for (m, n, k) in wl.DENSE_SWEEP]
    arrays = [(c.A.numpy(), c.sa.numpy(), c.B.numpy(), c.sb.numpy()) for c in cases]

    def step(i):
        fl = 0.0
        for c, (A, sa, B, sb) in zip(cases, arrays):
            rows = oracle_rows_sample(c, threads, salt=i)
            oracle.gemm_nt(A, sa, c.sa_stride, B, sb, c.M, c.N, c.K, rows=rows, want_d64=False, want_mag=False)
            fl += 2.0 * len(rows) * c.N * c.K
        return fl

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    fl = sum(step(args.warmup + i) for i in range(args.steps))
    dt = time.perf_counter() - t0
    v = fl / dt / 1e12
    out = {"impl": "reference", "metric": "FP8 scaled-GEMM TFLOPS per shape; % of B200 FP8 peak or HBM roofline",
           "value": v, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": "dense FP8 NT GEMM sweep, 18 shapes: M in {64,128,4096} x (N,K) in "
                                  "{(2112,7168),(24576,1536),(32768,512),(7168,16384),(4096,7168),(7168,2048)}"},
           "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                            "sample": f"{threads} full output rows (all N columns) of each of the 18 shapes "
                                      "per step"},
           "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-grouped", action="store_true", help="skip the grouped workloads")
    ap.add_argument("--shape", default="", help="run one dense shape MxNxK instead of the sweep")
    ap.add_argument("--detail", default="", help="write the per-shape, grouped, cast, block-scaled, layout and "
                                                 "K-grouped tables to this JSON file")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)  # at least 3 untimed warm-up steps
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
