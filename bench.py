"""Benchmark of the W8A8 INT8 linear hot path on B200, one JSON line on rank 0.

One step = the whole path on one batch of the Llama-2-7B-shaped MLP up-projection
(X bf16 [2048, 4096] with 0.1% of the columns scaled x60, W bf16 [11008, 4096]):
  SmoothQuant linear: channel absmax of X -> smoothing factors (alpha 0.5) -> smoothed
  per-channel int8 weight -> smoothed per-token int8 activation -> INT8 GEMM + dequant;
  LLM.int8() linear on the same X and W (threshold 6.0): per-channel int8 of the
  unsmoothed weight -> decomposed linear (column absmax, outlier mask, masked per-token
  quantization, gathers, INT8 GEMM with the bf16 outlier product in the same tiles).
The metric counts the tensor-core work of the two linears (2*M*N*K each, plus
2*M*N*K_o for the outlier product) per unit of time, whole job over all ranks.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU (torchrun, one rank per GPU): each rank runs its own replica of the workload
(independent token batches, weak scaling); there is no collective in the data path.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from w8a8_quantized_gemm_b200 import workloads as wl  # noqa: E402

METRIC = "W8A8 linear TOPS and % of B200 INT8 peak; quantize-kernel GB/s vs HBM peak"
ALPHA = 0.5
THRESHOLD = 6.0
N_SETS = 4  # rotating input sets: 4 x (16.8 MB X + 90.2 MB W) = 428 MB > 126 MB L2

# DRAM traffic of one int8 GEMM launch on this workload (dram__bytes_read.sum +
# dram__bytes_write.sum of `ncu --clock-control none --metrics gpu__time_duration.sum,
# dram__bytes_read.sum,dram__bytes_write.sum -k regex:w8a8_gemm -s 1 -c 1 python -m
# w8a8_quantized_gemm_b200.profile_cases gemm`), valid while the GEMM source's code (comments
# aside) hashes to GEMM_SRC_SHA. The reads are Xq + Wq once (53.6 MB); most of Y's 45 MB of
# writes are still in L2 when the kernel ends, so the write figure is below Y's size.
NCU_GEMM_TRAFFIC_BYTES = 53614336 + 13162496
GEMM_SRC_SHA = "e385499f0733b73e"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def _gemm_src_sha():
    """SHA-256 (16 hex digits) of the GEMM source with its // comments and blank lines dropped:
    editing a comment does not invalidate the recorded traffic, changing the code does."""
    lines = []
    with open(os.path.join(ROOT, "w8a8_quantized_gemm_b200", "csrc", "sq_gemm.cu")) as f:
        for line in f:
            code = line.split("//", 1)[0].rstrip()
            if code:
                lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:16]


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Polls NVML (SM clock, clock-event reasons) in a thread during the timed region."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            import torch
            handle = None
            try:
                props = torch.cuda.get_device_properties(device_index)
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.h = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()

    def _reasons_now(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(fn(self.h))

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self._reasons_now()
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml_unavailable"], "samples": 0}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- distributed
def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _init_pg(ws, local):
    import datetime

    import torch
    import torch.distributed as dist
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return ws > 1


def _max_over_ranks(x: float, use_dist: bool, local) -> float:
    """Maximum of x over the ranks (x itself on one rank). `local` is the CUDA device index
    (NCCL) or None for a CPU process group (gloo)."""
    if not use_dist:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cpu" if local is None else f"cuda:{local}")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(use_dist: bool, local):
    if use_dist:
        import torch.distributed as dist
        if local is None:
            dist.barrier()
        else:
            dist.barrier(device_ids=[local])


def whole_job_rate(units_per_step: float, steps: int, world: int, ms_max: float) -> float:
    """Units per second of the whole job: every rank processed `steps` steps of its own replica
    in at most `ms_max` milliseconds (the slowest rank's time)."""
    return units_per_step * world * steps / (ms_max * 1e-3)


# ----------------------------------------------------------------------------- our arm
class Path:
    """Device buffers and one step of the hot path through the C ABI."""

    def __init__(self, p, dev, n_sets):
        import torch

        from w8a8_quantized_gemm_b200 import sq
        self.torch, self.sq, self.p = torch, sq, p
        M, N, K = p.M, p.N, p.K
        self.M, self.N, self.K = M, N, K

        def up(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

        self.X = [up(p.X) for _ in range(n_sets)]
        self.W = [up(p.W) for _ in range(n_sets)]
        f32, i8 = torch.float32, torch.int8
        self.amax = torch.empty(K, dtype=f32, device=dev)
        self.s = torch.empty(K, dtype=f32, device=dev)
        self.inv_s = torch.empty(K, dtype=f32, device=dev)
        self.Wq = torch.empty((N, K), dtype=i8, device=dev)
        self.e = torch.empty(N, dtype=f32, device=dev)
        self.Xq = torch.empty((M, K), dtype=i8, device=dev)
        self.d = torch.empty(M, dtype=f32, device=dev)
        self.Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.Wq0 = torch.empty((N, K), dtype=i8, device=dev)
        self.e0 = torch.empty(N, dtype=f32, device=dev)
        self.Y2 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.cnt = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ws_gemm = sq.workspace(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K, dev)
        self.ws_llm = sq.workspace(sq.SQ_OP_LLMINT8, M, N, K, dev)
        self.names = ["act_channel_absmax", "smooth_scale", "smooth_quant_weight", "quant_act_per_token",
                      "int8_gemm_dequant", "quant_weight_unsmoothed", "llmint8_decomposed_linear"]
        self.times = {n: 0.0 for n in self.names}
        self.ev_pool = []

    def step(self, i, record=None, external=False):
        sq, X, W = self.sq, self.X[i % len(self.X)], self.W[i % len(self.W)]
        ev = []

        def mark():
            if record is not None:
                e = self.torch.cuda.Event(enable_timing=True, external=external)
                e.record()
                ev.append(e)

        mark()
        sq.sq_act_channel_absmax(X, self.amax)
        mark()
        sq.sq_smooth_scale(self.amax, W, ALPHA, self.s, self.inv_s)
        mark()
        sq.sq_smooth_quant_weight(W, self.s, sq.SQ_PER_CHANNEL, self.Wq, self.e)
        mark()
        sq.sq_quant_act_per_token(X, self.inv_s, self.Xq, self.d)
        mark()
        sq.sq_int8_gemm_dequant(self.Xq, self.Wq, self.d, self.e, sq.SQ_PER_CHANNEL, None, self.Y, None, self.ws_gemm)
        mark()
        sq.sq_smooth_quant_weight(W, None, sq.SQ_PER_CHANNEL, self.Wq0, self.e0)
        mark()
        sq.llmint8_decomposed_linear(X, W, self.Wq0, self.e0, THRESHOLD, None, self.Y2, None, self.cnt, None,
                                     self.ws_llm)
        mark()
        if record is not None:
            record.append(ev)

    def isolated_times(self, reps=5):
        """Each operation of the step alone: its calls over the rotating input sets captured
        `reps` times round in one CUDA graph, mean device time per call (no event nodes)."""
        sq = self.sq
        ops = {
            "act_channel_absmax": lambda X, W: sq.sq_act_channel_absmax(X, self.amax),
            "smooth_scale": lambda X, W: sq.sq_smooth_scale(self.amax, W, ALPHA, self.s, self.inv_s),
            "smooth_quant_weight": lambda X, W: sq.sq_smooth_quant_weight(W, self.s, sq.SQ_PER_CHANNEL, self.Wq,
                                                                          self.e),
            "quant_act_per_token": lambda X, W: sq.sq_quant_act_per_token(X, self.inv_s, self.Xq, self.d),
            "int8_gemm_dequant": lambda X, W: sq.sq_int8_gemm_dequant(self.Xq, self.Wq, self.d, self.e,
                                                                      sq.SQ_PER_CHANNEL, None, self.Y, None,
                                                                      self.ws_gemm),
            "quant_weight_unsmoothed": lambda X, W: sq.sq_smooth_quant_weight(W, None, sq.SQ_PER_CHANNEL, self.Wq0,
                                                                              self.e0),
            "llmint8_decomposed_linear": lambda X, W: sq.llmint8_decomposed_linear(
                X, W, self.Wq0, self.e0, THRESHOLD, None, self.Y2, None, self.cnt, None, self.ws_llm),
        }
        out = {}
        for n, fn in ops.items():
            fns = [(lambda X=X, W=W, fn=fn: fn(X, W)) for X, W in zip(self.X, self.W)]
            out[n] = _graph_time_us(self.torch, fns, reps) * 1e-3  # ms
        return out

    def collect(self, records):
        self.torch.cuda.synchronize()
        for ev in records:
            for j, n in enumerate(self.names):
                self.times[n] += ev[j].elapsed_time(ev[j + 1])
        return {n: t / max(len(records), 1) for n, t in self.times.items()}


def run_ours(args):
    import torch

    from w8a8_quantized_gemm_b200 import sq
    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    use_dist = _init_pg(ws, local)
    dev = f"cuda:{local}"
    hbm, bf16, bf16_sus, peak_kind = _peaks()
    int8_peak = 2.0 * bf16  # nominal dense int8 : bf16 ratio of 2 (4.5 / 2.25 PFLOP/s)

    p = wl.llama7b_mlp_up()
    M, N, K = p.M, p.N, p.K
    path = Path(p, dev, N_SETS)

    for i in range(args.warmup):
        path.step(i)
    sq.sq_sync_status()
    k_o = int(path.cnt.item())
    ops_step = 2.0 * M * N * K * 2 + 2.0 * M * N * k_o

    # ---------------------------------------------------------------- timed region
    # The K timed steps are captured once as one CUDA graph (launch overhead out of the way,
    # as a serving loop would run them); every SAMPLE_EVERY-th step carries timing events
    # between its operations (an event node costs a few microseconds inside a graph, so
    # instrumenting every step would inflate the step time). The graph is replayed once
    # untimed and once timed.
    records = []
    mode = "cuda_graph"
    stream = torch.cuda.Stream()
    graph = None
    launches0 = sq.sq_kernel_launch_count()
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(args.steps):
                path.step(i, records if i % args.sample_every == 0 else None, external=True)
        launches = sq.sq_kernel_launch_count() - launches0
        with torch.cuda.stream(stream):
            graph.replay()
        torch.cuda.synchronize()
    except Exception as exc:  # capture unsupported here: time the same steps eagerly
        mode = f"eager ({type(exc).__name__})"
        graph, records = None, []
        torch.cuda.synchronize()
    torch.cuda.synchronize()
    _barrier(use_dist, local)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            if graph is not None:
                t_start.record()
                graph.replay()
                t_end.record()
            else:
                launches0 = sq.sq_kernel_launch_count()
                t_start.record()
                for i in range(args.steps):
                    path.step(i, records if i % args.sample_every == 0 else None)
                t_end.record()
                launches = sq.sq_kernel_launch_count() - launches0
        torch.cuda.synchronize()
    _barrier(use_dist, local)
    torch.cuda.synchronize()
    ms_total = t_start.elapsed_time(t_end)
    ms_total = _max_over_ranks(ms_total, use_dist, local)
    sq.sq_sync_status()
    per_kernel = path.collect(records)
    del graph
    iso = path.isolated_times()

    ms_step = ms_total / args.steps
    value = whole_job_rate(ops_step, args.steps, ws, ms_total) / 1e12

    # ---------------------------------------------------------------- kernel rooflines
    gemm_ms = per_kernel["int8_gemm_dequant"]
    gemm_tops = 2.0 * M * N * K / (gemm_ms * 1e-3) / 1e12
    traffic = NCU_GEMM_TRAFFIC_BYTES if (NCU_GEMM_TRAFFIC_BYTES and GEMM_SRC_SHA == _gemm_src_sha()) else None
    roofline = {"kernel": "w8a8_gemm_kernel (sq_int8_gemm_dequant)", "bound": "tensor",
                "achieved": round(gemm_tops, 1), "peak": round(int8_peak, 1), "unit": "TFLOP/s",
                "frac": round(gemm_tops / int8_peak, 4), "traffic": traffic,
                "peak_note": f"int8 dense = 2 x {peak_kind} bf16 burst {bf16} TFLOP/s (nominal int8:bf16 = 2); "
                             f"vs 4500 datasheet: {gemm_tops / 4500.0:.3f}"}
    hbm_bytes = {
        "act_channel_absmax": 2.0 * M * K + 4 * K,
        "smooth_scale": 2.0 * N * K + 12 * K,
        "smooth_quant_weight": 3.0 * N * K + 4 * N + 4 * K,
        "quant_act_per_token": 3.0 * M * K + 4 * M + 4 * K,
        "quant_weight_unsmoothed": 3.0 * N * K + 4 * N,
    }
    kernels = {}
    for n, t in per_kernel.items():
        # rates from the operation timed alone (event nodes inside the step add a few us to
        # the short operations); the in-step time beside it
        ti = iso[n]
        ent = {"us": round(ti * 1e3, 2), "us_in_step": round(t * 1e3, 2)}
        if n in hbm_bytes:
            gbs = hbm_bytes[n] / (ti * 1e-3) / 1e9
            ent.update({"GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4)})
        elif n == "int8_gemm_dequant":
            tops_i = 2.0 * M * N * K / (ti * 1e-3) / 1e12
            ent.update({"TOPS": round(tops_i, 1), "frac_int8_peak": round(tops_i / int8_peak, 4)})
        else:
            tops = (2.0 * M * N * K + 2.0 * M * N * k_o) / (ti * 1e-3) / 1e12
            ent.update({"TOPS": round(tops, 1), "frac_int8_peak": round(tops / int8_peak, 4), "k_outliers": k_o})
        kernels[n] = ent

    # the library's kernels inside the step (several per call), from the profiler's records;
    # the masked LLM.int8 quantization is rated on the bytes it must move: X read, codes and
    # row scales written, both gathered outlier operands (zero-padded to 64 columns) written
    # and the outlier columns of W read
    pad = (k_o + 63) // 64 * 64
    masked_bytes = 3.0 * M * K + 4 * M + 2.0 * (M + N) * pad + 2.0 * N * k_o
    ktimes_note = ("avg device time per launch over 4 untimed steps (CUDA profiler activity records); "
                   f"the masked quantization of the LLM.int8 linear moves {masked_bytes / 1e6:.1f} MB "
                   f"(X read, codes, row scales, both gathered outlier operands, the {k_o} outlier columns of W)")

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = run_e2e(path, p, args, ops_step, use_dist, local, ws)

    # the profiler pass comes after every timed part of the line
    try:
        ktimes = measure_kernel_times(path)
    except Exception as exc:  # the profiler's activity records are a diagnostic: keep the line
        ktimes = {"error": f"{type(exc).__name__}: {exc}"}

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TOPS", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic (seeded numpy PCG64, bf16)",
        "config": {"workload": f"llama7b_mlp_up X[{M},{K}] W[{N},{K}]: SmoothQuant W8A8 linear (alpha {ALPHA}, "
                               f"per-token act, per-channel weight) + LLM.int8 linear (threshold {THRESHOLD})",
                   "M": M, "N": N, "K": K, "outlier_columns": k_o, "ops_per_step": ops_step,
                   "l2": f"{N_SETS} rotating input sets ({N_SETS * (2 * M * K + 2 * N * K) / 1e6:.0f} MB) > L2",
                   "parallelism": f"replica x{ws}"},
        "roofline": roofline, "kernels": kernels, "kernel_times_in_step": ktimes,
        "kernel_times_note": ktimes_note, "gpu_launches": int(launches), "launch_mode": mode,
        "kernel_timing": f"roofline: CUDA event nodes around each operation of every {args.sample_every}th timed "
                         f"step ({len(records)} steps sampled); kernels: us / rate / frac from each operation "
                         f"timed alone over the {N_SETS} input sets in its own CUDA graph, us_in_step from the "
                         f"sampled event nodes",
        "clocks": clk.summary(), "e2e": e2e, "peaks": {"hbm_gbs": hbm, "bf16_tflops": bf16, "kind": peak_kind},
    }
    if rank == 0 and ws == 1 and not args.no_configs:
        del path
        torch.cuda.empty_cache()
        try:
            line["other_workloads"] = measure_configs(dev, hbm, int8_peak)
        except Exception as exc:  # keep the main line; say what failed
            line["other_workloads"] = {"error": f"{type(exc).__name__}: {exc}"}
        torch.cuda.empty_cache()
        try:
            pk = measure_int8_peak(dev, iso["int8_gemm_dequant"] * 1e3)
            line["int8_peak_measured"] = pk
            burst = pk["cublas_int8_8192^3"]["burst_TOPS"]
            roofline["frac_of_cublas_int8_burst"] = round(gemm_tops / burst, 4)
        except Exception as exc:
            line["int8_peak_measured"] = {"error": f"{type(exc).__name__}: {exc}"}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(p, args.cpu_budget)
    if use_dist:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def _graph_time_us(torch, fns, reps):
    """Mean device time of one call, the calls captured `reps` times round in one CUDA graph
    (so launch overhead stays out) and the graph replayed once untimed, once timed."""
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for f in fns:
            f()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(reps):
            for f in fns:
                f()
    with torch.cuda.stream(s):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) * 1e3 / (reps * len(fns))


def _entries(hbm, int8_peak):
    def hbm_entry(us, nbytes):
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"us": round(us, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4)}

    def tops_entry(us, ops):
        t = ops / (us * 1e-6) / 1e12
        return {"us": round(us, 2), "TOPS": round(t, 1), "frac_int8_peak": round(t / int8_peak, 4)}
    return hbm_entry, tops_entry


def measure_int8_peak(dev, gemm_us_7b):
    """cuBLAS's int8 GEMM (torch._int_mm, int32 output) as a measured int8 tensor-core rate:
    8192^3 best of ten graph replays (burst) and back to back for about two seconds
    (sustained, under the power cap), and on the 2048 x 11008 x 4096 shape beside this
    library's GEMM (which also dequantizes and writes bf16). A library kernel, timed here as a
    reference rate only; it is not on the hot path."""
    import torch
    gen = torch.Generator(device=dev)
    gen.manual_seed(1)
    out = {}
    n = 8192
    A = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=gen)
    B = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=gen)
    C = torch.empty((n, n), dtype=torch.int32, device=dev)
    Bt = B.t()
    fn = [lambda: torch._int_mm(A, Bt, out=C)]
    best = min(_graph_time_us(torch, fn, 3) for _ in range(10))
    reps = max(3, int(2.0e6 / best))
    sustained = _graph_time_us(torch, fn, reps)
    ops = 2.0 * n ** 3
    out["cublas_int8_8192^3"] = {"burst_us": round(best, 1), "burst_TOPS": round(ops / best / 1e6, 1),
                                 "sustained_us": round(sustained, 1),
                                 "sustained_TOPS": round(ops / sustained / 1e6, 1),
                                 "sustained_reps": reps}
    del A, B, C, Bt
    M, N, K = 2048, 11008, 4096
    Xq = [torch.randint(-127, 128, (M, K), dtype=torch.int8, device=dev, generator=gen) for _ in range(4)]
    Wq = [torch.randint(-127, 128, (N, K), dtype=torch.int8, device=dev, generator=gen) for _ in range(4)]
    C = torch.empty((M, N), dtype=torch.int32, device=dev)
    us = _graph_time_us(torch, [(lambda x=x, w=w: torch._int_mm(x, w.t(), out=C)) for x, w in zip(Xq, Wq)], 10)
    burst = ops / best / 1e6
    out["cublas_int8_2048x11008x4096"] = {"us": round(us, 2), "TOPS": round(2.0 * M * N * K / us / 1e6, 1)}
    out["w8a8_gemm_2048x11008x4096"] = {"us": round(gemm_us_7b, 2),
                                        "TOPS": round(2.0 * M * N * K / gemm_us_7b / 1e6, 1),
                                        "frac_of_cublas_int8_burst": round(2.0 * M * N * K / gemm_us_7b / 1e6 / burst,
                                                                           4)}
    out["note"] = ("cuBLAS writes int32 (4 bytes per output); the library's GEMM dequantizes and writes bf16 "
                   "(2 bytes); both are timed in CUDA graphs over rotated inputs")
    return out


def measure_configs(dev, hbm, int8_peak):
    """The other workloads, each timed alone after the main timed region (not part of the
    step): the tiny config's latency, the decode sweep (M in {1,4,16,64}, 4096 x 4096, eight
    weight copies rotated so the weight streams from HBM; the GEMM alone and the decode step
    quantization + GEMM), the LLM.int8 sweep (X [4096, 8192] with 0 / 8 / 82 outlier columns,
    W [8192, 8192]), the 70B-shaped FFN path (8192 x 28672 x 8192: calibration, smoothing,
    both quantizations and the GEMM at alpha 0.3 / 0.5 / 0.7, and the GEMM forms) and the
    reductions and variants on large inputs (X [8192, 8192], two rotated copies, 268 MB > L2;
    timed first). Random device inputs of those shapes and distributions; the parity tests
    cover the values."""
    import torch

    from w8a8_quantized_gemm_b200 import sq
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    out = {}
    hbm_entry, tops_entry = _entries(hbm, int8_peak)

    out["tiny_latency"] = measure_tiny_latency(dev)

    # reductions and variants on X [8192, 8192]: algorithmic bytes read X once (+ write codes once).
    # Timed before the GEMM-heavy workloads: after seconds of GEMMs under the power cap the SM
    # clock stays lowered for a while, and the latency-bound fused norm follows the SM clock
    # (85 / 78 us fresh against 123-132 / 84-121 us right after 3 s of 70B GEMMs, one box).
    M = K = 8192
    Xs = [(1.5 * torch.randn(M, K, device=dev, generator=gen) + 0.2).to(torch.bfloat16) for _ in range(2)]
    inv = torch.rand(K, device=dev, generator=gen) + 0.5
    g = (torch.rand(K, device=dev, generator=gen) + 0.5).to(torch.bfloat16)
    b = (0.1 * torch.randn(K, device=dev, generator=gen)).to(torch.bfloat16)
    Xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    d, z = torch.empty(M, device=dev), torch.empty(M, dtype=torch.int32, device=dev)
    d1, clip, thr = torch.empty(1, device=dev), torch.full((1,), 4.0, device=dev), torch.empty(1, device=dev)
    amax = torch.empty(K, device=dev)
    wpt = sq.workspace(sq.SQ_OP_QUANT_ACT_PER_TENSOR, M, 0, K, device=dev)
    wms = sq.workspace(sq.SQ_OP_MEAN_STD_THRESHOLD, M, 0, K, device=dev)
    wpc = sq.workspace(sq.SQ_OP_ABS_PERCENTILE, M, 0, K, device=dev)
    n = M * K
    var = {}
    cases = [
        ("act_channel_absmax", 2 * n + 4 * K, lambda X: sq.sq_act_channel_absmax(X, amax)),
        ("quant_act_per_token", 3 * n, lambda X: sq.sq_quant_act_per_token(X, inv, Xq, d)),
        ("layernorm_smooth_quant", 3 * n, lambda X: sq.sq_norm_smooth_quant(X, sq.SQ_NORM_LAYER, g, b, 1e-5, inv, Xq,
                                                                            d)),
        ("rmsnorm_smooth_quant", 3 * n, lambda X: sq.sq_norm_smooth_quant(X, sq.SQ_NORM_RMS, g, None, 1e-5, inv, Xq,
                                                                          d)),
        ("quant_act_per_token_asym", 3 * n, lambda X: sq.sq_quant_act_per_token_asym(X, inv, Xq, d, z)),
        ("quant_act_per_tensor_dynamic", 3 * n, lambda X: sq.sq_quant_act_per_tensor(X, inv, Xq, d1, None, wpt)),
        ("quant_act_per_tensor_static_clip", 3 * n, lambda X: sq.sq_quant_act_per_tensor(X, inv, Xq, d1, clip)),
        ("act_mean_std_threshold", 2 * n, lambda X: sq.sq_act_mean_std_threshold(X, 6.0, thr, None, wms)),
        ("act_abs_percentile", 2 * n, lambda X: sq.sq_act_abs_percentile(X, 99.99, d1, wpc)),
    ]
    for name, nbytes, fn in cases:
        us = _graph_time_us(torch, [(lambda X=X: fn(X)) for X in Xs], 5)
        var[name] = hbm_entry(us, nbytes)
    var["note"] = ("X bf16 [8192, 8192]; GB/s on the bytes of one read of X (+ one write of the int8 codes); the "
                   "dynamic per-tensor form reads X twice by design (global maximum first); timed before the "
                   "GEMM-heavy workloads")
    out["variants_8192x8192"] = var
    del Xs, Xq

    # decode sweep: bytes N*K + M*K + 2*M*N + 4*(M+N) per GEMM call; the step adds the
    # activation rows (2*M*K read, M*K + 4*M written)
    N = K = 4096
    Wqs = [torch.randint(-127, 128, (N, K), dtype=torch.int8, device=dev, generator=gen) for _ in range(8)]
    e = torch.rand(N, device=dev, generator=gen) * 1e-3
    inv_s = torch.rand(K, device=dev, generator=gen) + 0.5
    dec, dec_path = {}, {}
    for M in (1, 4, 16, 64):
        Xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=dev, generator=gen)
        d = torch.rand(M, device=dev, generator=gen) * 1e-2
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = sq.workspace(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K, device=dev)
        us = _graph_time_us(torch, [(lambda w=w: sq.sq_int8_gemm_dequant(Xq, w, d, e, sq.SQ_PER_CHANNEL, None, Y,
                                                                         None, ws)) for w in Wqs], 10)
        gemm_bytes = N * K + M * K + 2 * M * N + 4 * (M + N)
        dec[f"M{M}"] = hbm_entry(us, gemm_bytes)
        Xs = [torch.randn(M, K, device=dev, generator=gen) for _ in range(8)]
        for x in Xs:
            x[:, :6] += 40.0
        Xs = [x.to(torch.bfloat16) for x in Xs]
        Xq2, d2 = torch.empty((M, K), dtype=torch.int8, device=dev), torch.empty(M, device=dev)

        def step(x, w, Xq2=Xq2, d2=d2, Y=Y, ws=ws):
            sq.sq_quant_act_per_token(x, inv_s, Xq2, d2)
            sq.sq_int8_gemm_dequant(Xq2, w, d2, e, sq.SQ_PER_CHANNEL, None, Y, None, ws)
        us2 = _graph_time_us(torch, [(lambda x=x, w=w: step(x, w)) for x, w in zip(Xs, Wqs)], 10)
        ent = hbm_entry(us2, gemm_bytes + 3 * M * K + 4 * M)
        ent["launches"] = 2
        dec_path[f"M{M}"] = ent
    out["decode_4096x4096"] = dec
    out["decode_step_quant_gemm_4096x4096"] = dec_path
    del Wqs

    # LLM.int8 sweep
    M, N, K = 4096, 8192, 8192
    base = (0.5 * torch.randn(M, K, device=dev, generator=gen)).clamp_(-5.5, 5.5)
    W = (0.015 * torch.randn(N, K, device=dev, generator=gen)).to(torch.bfloat16)
    Wq, ew = torch.empty((N, K), dtype=torch.int8, device=dev), torch.empty(N, device=dev)
    sq.sq_smooth_quant_weight(W, None, sq.SQ_PER_CHANNEL, Wq, ew)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = sq.workspace(sq.SQ_OP_LLMINT8, M, N, K, device=dev)
    cnt = torch.empty(1, dtype=torch.int32, device=dev)
    llm = {}
    for k_o in (0, 8, 82):
        X = base.clone()
        if k_o:
            cols = torch.randperm(K, device=dev, generator=gen)[:k_o]
            mag = 20.0 + 180.0 * torch.rand(k_o, device=dev, generator=gen)
            X[:, cols] += mag * torch.where(torch.rand(k_o, device=dev, generator=gen) < 0.5, -1.0, 1.0)
        X = X.to(torch.bfloat16)
        us = _graph_time_us(torch, [lambda: sq.llmint8_decomposed_linear(X, W, Wq, ew, 6.0, None, Y, None, cnt, None,
                                                                         ws)], 5)
        found = int(cnt.item())
        ent = tops_entry(us, 2.0 * M * N * K + 2.0 * M * N * found)
        ent["k_outliers"] = found
        llm[f"K_o={k_o}"] = ent
    out["llmint8_4096x8192x8192"] = llm
    del base, W, Wq, Y, ws, X

    out.update(measure_ffn70b(dev, hbm, int8_peak, gen))

    sq.sq_sync_status()
    return out


def measure_ffn70b(dev, hbm, int8_peak, gen):
    """The 70B-shaped FFN path, X [8192, 8192] ~N(0,1) with 4 columns x100, W [28672, 8192]
    ~N(0,0.01), bias ~N(0,0.1): for alpha in {0.3, 0.5, 0.7} each call of the SmoothQuant path
    (channel absmax of X, smoothing factors from W, smoothed per-channel weight quantization,
    smoothed per-token activation quantization, GEMM + dequant + bias) timed alone, and the
    whole path as one graph; then the GEMM with asymmetric activations, with a per-tensor
    activation scale, and the weight row sums."""
    import torch

    from w8a8_quantized_gemm_b200 import sq
    hbm_entry, tops_entry = _entries(hbm, int8_peak)
    out = {}
    M, N, K = 8192, 28672, 8192
    X = torch.randn(M, K, device=dev, generator=gen)
    cols = torch.randperm(K, device=dev, generator=gen)[:4]
    X[:, cols] *= 100.0
    X = X.to(torch.bfloat16)
    W = (0.01 * torch.randn(N, K, device=dev, generator=gen)).to(torch.bfloat16)
    bias = (0.1 * torch.randn(N, device=dev, generator=gen)).to(torch.bfloat16)
    amax, s, inv_s = (torch.empty(K, device=dev) for _ in range(3))
    Wq, e = torch.empty((N, K), dtype=torch.int8, device=dev), torch.empty(N, device=dev)
    Xq, d = torch.empty((M, K), dtype=torch.int8, device=dev), torch.empty(M, device=dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ops = 2.0 * M * N * K
    path = {}
    for alpha in (0.3, 0.5, 0.7):
        steps = {
            "act_channel_absmax": (lambda: sq.sq_act_channel_absmax(X, amax), hbm, 2 * M * K + 4 * K),
            "smooth_scale": (lambda: sq.sq_smooth_scale(amax, W, alpha, s, inv_s), hbm, 2 * N * K + 12 * K),
            "smooth_quant_weight": (lambda: sq.sq_smooth_quant_weight(W, s, sq.SQ_PER_CHANNEL, Wq, e), hbm,
                                    3 * N * K + 4 * N + 4 * K),
            "quant_act_per_token": (lambda: sq.sq_quant_act_per_token(X, inv_s, Xq, d), hbm, 3 * M * K + 4 * M + 4 * K),
            "int8_gemm_dequant_bias": (lambda: sq.sq_int8_gemm_dequant(Xq, Wq, d, e, sq.SQ_PER_CHANNEL, bias, Y),
                                       None, ops),
        }
        ent = {}
        total = 0.0
        for name, (fn, bw, work) in steps.items():
            us = _graph_time_us(torch, [fn], 3)
            total += us
            ent[name] = hbm_entry(us, work) if bw is not None else tops_entry(us, work)

        def whole():
            for fn, _, _ in steps.values():
                fn()
        us = _graph_time_us(torch, [whole], 3)
        ent["whole_path"] = tops_entry(us, ops)
        ent["whole_path"]["sum_of_calls_us"] = round(total, 1)
        path[f"alpha={alpha}"] = ent
    out["ffn70b_path_8192x28672x8192"] = path
    us = _graph_time_us(torch, [lambda: sq.sq_int8_gemm_dequant(Xq, Wq, d, e, sq.SQ_PER_CHANNEL, bias, Y)], 3)
    out["ffn70b_gemm_8192x28672x8192"] = tops_entry(us, ops)
    z = torch.randint(-128, 128, (M,), dtype=torch.int32, device=dev, generator=gen)
    rs = torch.empty(N, dtype=torch.int32, device=dev)
    sq.sq_weight_row_sums(Wq, rs)
    us = _graph_time_us(torch, [lambda: sq.sq_int8_gemm_dequant_ex(Xq, Wq, d, sq.SQ_PER_CHANNEL, z, e,
                                                                   sq.SQ_PER_CHANNEL, rs, bias, Y)], 3)
    out["gemm_asymmetric_8192x28672x8192"] = tops_entry(us, ops)
    us = _graph_time_us(torch, [lambda: sq.sq_int8_gemm_dequant_ex(Xq, Wq, d[:1], sq.SQ_PER_TENSOR, None, e,
                                                                   sq.SQ_PER_CHANNEL, None, bias, Y)], 3)
    out["gemm_per_tensor_x_8192x28672x8192"] = tops_entry(us, ops)
    us = _graph_time_us(torch, [lambda: sq.sq_weight_row_sums(Wq, rs)], 5)
    out["weight_row_sums_28672x8192"] = hbm_entry(us, N * K + 4 * N)
    return out


def measure_tiny_latency(dev):
    """The tiny config's whole SmoothQuant path (channel absmax, smoothing factors, per-tensor
    weight quantization, per-token activation quantization, GEMM) and its LLM.int8 linear,
    X [16, 256], W [256, 256]: launch-to-result latency of one eager call sequence (host clock
    from the first launch to the end of a stream synchronize, median of 50) and the device
    time of the same sequence replayed as a CUDA graph."""
    import torch

    from w8a8_quantized_gemm_b200 import sq
    p = wl.tiny()
    M, N, K = p.M, p.N, p.K

    def up(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    X, W = up(p.X), up(p.W)
    amax, s, inv_s = (torch.empty(K, device=dev) for _ in range(3))
    Wq, e = torch.empty((N, K), dtype=torch.int8, device=dev), torch.empty(1, device=dev)
    Xq, d = torch.empty((M, K), dtype=torch.int8, device=dev), torch.empty(M, device=dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    wsw = sq.workspace(sq.SQ_OP_SMOOTH_QUANT_WEIGHT, 0, N, K, dev)
    wsg = sq.workspace(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K, dev)
    Wq1, e1 = torch.empty((N, K), dtype=torch.int8, device=dev), torch.empty(N, device=dev)
    sq.sq_smooth_quant_weight(W, None, sq.SQ_PER_CHANNEL, Wq1, e1)
    Y1 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    wsl = sq.workspace(sq.SQ_OP_LLMINT8, M, N, K, dev)

    def smoothquant():
        sq.sq_act_channel_absmax(X, amax)
        sq.sq_smooth_scale(amax, W, p.alpha, s, inv_s)
        sq.sq_smooth_quant_weight(W, s, sq.SQ_PER_TENSOR, Wq, e, wsw)
        sq.sq_quant_act_per_token(X, inv_s, Xq, d)
        sq.sq_int8_gemm_dequant(Xq, Wq, d, e, sq.SQ_PER_TENSOR, None, Y, None, wsg)

    def llmint8():
        sq.llmint8_decomposed_linear(X, W, Wq1, e1, p.threshold, None, Y1, None, None, None, wsl)

    out = {}
    for name, fn in (("smoothquant_path", smoothquant), ("llmint8_linear", llmint8)):
        stream = torch.cuda.current_stream()
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        lat = []
        for _ in range(50):
            t0 = time.perf_counter()
            fn()
            stream.synchronize()
            lat.append((time.perf_counter() - t0) * 1e6)
        out[name] = {"eager_launch_to_result_us": round(statistics.median(lat), 2),
                     "graph_device_us": round(_graph_time_us(torch, [fn], 20), 2)}
    out["config"] = f"tiny X[{M},{K}] W[{N},{K}]; SmoothQuant alpha {p.alpha} per-tensor weight; LLM.int8 6.0"
    return out


def measure_kernel_times(path, steps=4):
    """Device time of every kernel of the step, from the CUDA profiler's activity records
    (torch.profiler over `steps` untimed steps): the library launches several kernels inside
    one call (the LLM.int8 linear: column absmax, outlier mask, masked quantization with the
    gathers, GEMM), which CUDA events around the calls cannot separate."""
    import torch
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for i in range(steps):
            path.step(i)
        torch.cuda.synchronize()
    out = {}
    for ev in prof.key_averages():
        if getattr(ev, "device_type", None) != torch.autograd.DeviceType.CUDA:
            continue
        t = getattr(ev, "self_device_time_total", None) or getattr(ev, "self_cuda_time_total", 0.0)
        key = ev.key.replace("(anonymous namespace)::", "").replace("unnamed>::", "").replace("void ", "")
        key = key.split("(")[0].replace("sq::", "")
        out[key] = {"launches_per_step": ev.count / steps, "avg_us": round(t / max(ev.count, 1), 2)}
    return out


def run_e2e(path, p, args, ops_step, use_dist, local, ws):
    """Same step through the C ABI with the inputs in pinned HOST memory: every step copies its
    X and W host-to-device and both outputs device-to-host, all inside the timed region. The
    copies run on their own streams, so step i's outputs go back and step i+1's inputs come in
    while step i+1 computes (inputs in the rotating device sets, outputs double-buffered)."""
    import torch
    steps = max(3, min(args.steps, args.e2e_steps))
    hX = torch.from_numpy(np.ascontiguousarray(p.X).view(np.int16)).view(torch.bfloat16).pin_memory()
    hW = torch.from_numpy(np.ascontiguousarray(p.W).view(np.int16)).view(torch.bfloat16).pin_memory()
    hY = [torch.empty(path.Y.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    hY2 = [torch.empty(path.Y2.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    dY = [path.Y, torch.empty_like(path.Y)]
    dY2 = [path.Y2, torch.empty_like(path.Y2)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    nsets = len(path.X)

    def run(n):
        ev_in, ev_comp, ev_out = {}, {}, {}
        for i in range(n):
            k, b = i % nsets, i % 2
            with torch.cuda.stream(s_in):
                if i >= nsets:
                    s_in.wait_event(ev_comp[i - nsets])  # set k no longer in use
                path.X[k].copy_(hX, non_blocking=True)
                path.W[k].copy_(hW, non_blocking=True)
                ev_in[i] = torch.cuda.Event()
                ev_in[i].record()
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[i])
                if i >= 2:
                    s_comp.wait_event(ev_out[i - 2])  # output buffers b copied out
                path.Y, path.Y2 = dY[b], dY2[b]
                path.step(k)
                ev_comp[i] = torch.cuda.Event()
                ev_comp[i].record()
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[i])
                hY[b].copy_(dY[b], non_blocking=True)
                hY2[b].copy_(dY2[b], non_blocking=True)
                ev_out[i] = torch.cuda.Event()
                ev_out[i].record()

    run(2)
    torch.cuda.synchronize()
    _barrier(use_dist, local)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    run(steps)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_comp)
    b.record(s_out)
    torch.cuda.synchronize()
    path.Y, path.Y2 = dY[0], dY2[0]
    ms = _max_over_ranks(a.elapsed_time(b), use_dist, local)
    bi = hX.numel() * 2 + hW.numel() * 2
    bo = hY[0].numel() * 2 + hY2[0].numel() * 2
    return {"value": round(whole_job_rate(ops_step, steps, ws, ms) / 1e12, 3), "unit": "TOPS",
            "h2d_bytes_per_step": int(bi), "d2h_bytes_per_step": int(bo), "steps": steps,
            "ms_per_step": round(ms / steps, 3),
            "mode": "copy-in / compute / copy-out on three streams, overlapped across steps"}


# ----------------------------------------------------------------------------- oracle on the host
def _sample(p, R, Nr):
    """A sub-problem of the workload: R token rows of X and Nr output rows of W (seeded)."""
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(p.M, R, replace=False)) if R < p.M else np.arange(p.M)
    wrows = np.sort(rng.choice(p.N, Nr, replace=False)) if Nr < p.N else np.arange(p.N)
    return np.ascontiguousarray(p.X[rows]), np.ascontiguousarray(p.W[wrows])


def _oracle_step(X, W, oracle):
    """The whole step on the host oracle for the linear X [R,K] x W [Nr,K]: both linears,
    calibration and weight preparation included. Returns (tensor ops, K_o)."""
    amax = oracle.act_channel_absmax(X)
    s, inv_s = oracle.smooth_scale(amax, W, ALPHA)
    Wq, e = oracle.smooth_quant_weight(W, s, oracle.PER_CHANNEL)
    xq, d = oracle.quant_act_per_token(X, inv_s)
    oracle.dequant(oracle.int8_gemm(xq, Wq), d, e, None)
    mask, idx, k_o = oracle.outlier_columns(amax, THRESHOLD)
    Wq0, e0 = oracle.smooth_quant_weight(W, None, oracle.PER_CHANNEL)
    xq0, d0 = oracle.quant_act_per_token(X, None, mask)
    o = oracle.outlier_product(X, W, idx)
    oracle.dequant(oracle.int8_gemm(xq0, Wq0), d0, e0, None, o)
    R, K = X.shape
    Nr = W.shape[0]
    return 2.0 * R * Nr * K * 2 + 2.0 * R * Nr * k_o, k_o


def cpu_baseline(p, budget_s):
    """The oracle, as it stands, on the whole step of the workload (all rows), repeated until
    about `budget_s` seconds of host work (at most 3 repetitions)."""
    import oracle
    X, W = p.X, p.W
    reps, ops, t = 0, 0.0, 0.0
    while reps < 3 and (reps == 0 or t < budget_s):
        t0 = time.perf_counter()
        o, _ = _oracle_step(X, W, oracle)
        t += time.perf_counter() - t0
        ops += o
        reps += 1
    return {"value": round(ops / t / 1e12, 6), "unit": "TOPS", "cores": oracle.num_threads(), "kind": "oracle",
            "seconds": round(t, 3),
            "sample": f"the whole step on the full workload ({p.M} token rows, {p.N} output channels), {reps} run(s)"}


def run_reference(args):
    """The oracle as the reference arm: each step is the whole path on a seeded sub-problem of
    the workload (a subset of token rows and output channels, full K), sized so that the
    --steps/--warmup run ends within a couple of minutes."""
    ws, rank, local = _dist()
    if rank != 0:
        return
    import oracle
    p = wl.llama7b_mlp_up()
    R = min(args.ref_rows, p.M)
    Nr = min(1024, p.N)
    X, W = _sample(p, R, Nr)
    t0 = time.perf_counter()
    _oracle_step(X, W, oracle)
    t1 = time.perf_counter()
    per_step_target = min(1.0, 120.0 / max(1, args.steps + args.warmup))
    Nr = int(min(p.N, max(64, Nr * per_step_target / max(t1 - t0, 1e-4))))
    X, W = _sample(p, R, Nr)
    for _ in range(args.warmup):
        _oracle_step(X, W, oracle)
    ops = 0.0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        o, k_o = _oracle_step(X, W, oracle)
        ops += o
    t1 = time.perf_counter()
    value = ops / (t1 - t0) / 1e12
    sample = (f"whole step (calibration, smoothing, both weight quantizations, both linears) on {R} of {p.M} "
              f"token rows x {Nr} of {p.N} output channels, K={p.K}")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TOPS", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round((t1 - t0) * 1e3 / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic (seeded numpy PCG64, bf16)",
            "config": {"workload": f"llama7b_mlp_up X[{p.M},{p.K}] W[{p.N},{p.K}] (sub-problem {R}x{Nr})",
                       "M": p.M, "N": p.N, "K": p.K},
            "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--sample-every", type=int, default=10, help="timed steps per step carrying event nodes")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip timing the other workloads and the variants")
    ap.add_argument("--ref-rows", type=int, default=64, help="token rows per reference-arm step")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
