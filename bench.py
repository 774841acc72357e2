#!/usr/bin/env python
"""Benchmark of the weight-only quantized product on B200.

Headline workload: the decode GEMV y (1 x 4096) = x (1 x 4096) @ dequant(W_q),
W_q 4-bit K-major words, group 128, fp16 scales and zero points.  One *step*
is one decode pass over a stack of L distinct weight sets of that shape (each
with its own x and y: independent products, as the projections of one token),
launched back to back with WQ_FLAG_PDL_INPUTS_READY and replayed as one CUDA
graph.  ``chained`` reports the same stack run as a dependency chain (each x
is the previous y, WQ_FLAG_PDL).  The stack's weights exceed twice the L2 size, so every
launch reads its words from HBM.  ``value`` is the algorithmic HBM bytes of
the products (packed words + s + z + x + y) per second, whole job.

Also measured on the same box, in the same run:
* ``gemm``: the batched product M=512, K=4096, N=2048 (4-bit, group 128) in TFLOP/s;
* ``workloads``: every synthetic workload (bit-width sweep, 3-bit planes, M=4/16),
  with fp16 and with bf16 x, scales, zeros and y;
* ``e2e``: the headline metric through the Python API with host buffers (x copied
  in and y copied out every step);
* ``cpu_baseline``: the CPU oracle (plain C, fp64) on a bounded sample.

``--impl reference`` times the CPU oracle as the reference arm.
``--gpus N`` (under torchrun) runs N independent replicas, one per GPU.
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
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import wq_inputs  # noqa: E402

HEADLINE = "decode_gemv_m1"
GEMM_WL = "prefill_gemm"
# the kernels those two launch, as ncu names them (spaces as underscores)
HEADLINE_KERNEL = "gemv_decode_kernel<16>"
GEMM_KERNEL = "gemm_kernel<4,_0,_1>"
METRIC = "packed-int GEMV HBM GB/s and % of peak at M=1; wq_gemm TFLOPS at M=512"
FALLBACK_HBM, FALLBACK_TF = 6650.0, 1590.0
# Nominal B200 figures, reported beside the measured ones: HBM3e ~8 TB/s,
# dense fp16 / bf16 tensor cores 2.25 PFLOP/s.
NOMINAL_HBM, NOMINAL_TF = 8000.0, 2250.0


def algo_bytes(wl) -> int:
    """Algorithmic bytes of one product: packed words, s, z, x and y."""
    return wl.K * wl.N * wl.bits // 8 + 2 * 2 * wl.groups * wl.N + 2 * wl.M * wl.K + 2 * wl.M * wl.N


def algo_flops(wl) -> int:
    return 2 * wl.M * wl.N * wl.K


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    return FALLBACK_HBM, FALLBACK_TF, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks (NVML)
class ClockSampler:
    """Samples SM clock and clock-event reasons of one GPU on a thread (NVML)."""

    NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
             0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
             0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def start(self):
        if self.nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self.nv and self._t:
            self._stop.set()
            self._t.join()
            self._sample()

    def report(self):
        if not self.nv or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for b, n in self.NAMES.items() if self.reasons & b and b != 0x1]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------------ replicas
def replica_max(v: float, dist=None, device=None) -> float:
    """The largest of every rank's `v` (a time: the job ends with its slowest
    replica); `v` itself without a process group."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_step: float, steps: int, world: int, elapsed_s: float) -> float:
    """Whole-job throughput: every replica processes `units_per_step` per step
    (weak scaling), timed by the slowest replica's `elapsed_s`."""
    return units_per_step * steps * world / elapsed_s


# ------------------------------------------------------------------ helpers
# Sources that no timed kernel is built from (the failure-path self-test).
# the device code of the timed kernels (the decode GEMV and the prefill GEMM)
DIGEST_SOURCES = ("wq_gemv_lean.cu", "wq_gemm.cu", "wq_ptx.cuh", "wq_dequant.cuh")


def src_digest() -> str:
    """Digest of the files the timed kernels' device code is built from: an ncu
    figure taken on other kernel sources does not count for this build."""
    h = hashlib.sha1()
    for name in DIGEST_SOURCES:
        h.update((ROOT / "gemm_wq_gemv_b200" / "csrc" / name).read_bytes())
    return h.hexdigest()[:12]


def ncu_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch from profiles/ncu_traffic.txt, if taken on this source."""
    p = ROOT / "profiles" / "ncu_traffic.txt"
    if not p.exists():
        return None
    for line in p.read_text().splitlines():
        if line.startswith("#") or not line.strip():
            continue
        kv = dict(t.split("=", 1) for t in line.split() if "=" in t)
        if kv.get("kernel") == kernel and kv.get("workload") == workload and kv.get("src") == src_digest():
            return float(kv["dram_bytes_per_launch"])
    return None


class Stack:
    """L distinct weight sets of one workload on the device, plus x / y per set."""

    def __init__(self, wq, torch, wl, L, dev, seed0=0, dtype="fp16"):
        import numpy as np
        self.wl, self.L = wl, L
        base = wq_inputs.draw(wl, seed=seed0, dtype=dtype)
        codes = torch.from_numpy(base.codes).to(dev)
        w_q, w_lo = wq.pack_kmajor(codes, wl.bits)

        def dev_array(a):  # bf16 inputs are uint16 bit patterns on the host
            if dtype == "bf16":
                return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
            return torch.from_numpy(a).to(dev)

        s = dev_array(base.scales)
        z = dev_array(base.zeros)
        del codes
        self.sets = []
        for i in range(L):
            x = dev_array(wq_inputs.x_batch(wl.M, wl.K, seed=1000 + i, dtype=dtype))
            y = torch.empty((wl.M, wl.N), dtype=x.dtype, device=dev)
            self.sets.append((x, w_q.clone() if i else w_q, None if w_lo is None else (w_lo.clone() if i else w_lo),
                              s.clone() if i else s, z.clone() if i else z, y))
        self.np = np

    def run(self, wq, fn, pdl=False, inputs_ready=False):
        wl = self.wl
        for (x, a, b, s, z, y) in self.sets:
            fn(x, a, b, s, z, wl.bits, wl.group_size, out=y, pdl=pdl, inputs_ready=inputs_ready)

    def run_chain(self, wq):
        """Each product's x is the previous product's y (square K = N): a true
        dependency chain, launched with WQ_FLAG_PDL."""
        wl = self.wl
        x = self.sets[0][0]
        for (_, a, b, s, z, y) in self.sets:
            wq.gemv(x, a, b, s, z, wl.bits, wl.group_size, out=y, pdl=True)
            x = y


def time_graph(torch, graph, stream, steps, warmup, barrier=None, sampler=None):
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.start()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.stop()
    if barrier:
        barrier()
    return e0.elapsed_time(e1) / 1e3  # seconds


def capture(torch, fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        fn()  # first run outside the graph (lazy set-up)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.synchronize()
    return g, s


def layers_for(wl, L2):
    """Weight sets per step: enough distinct sets to exceed twice the L2 (at most 1024)."""
    return min(1024, max(2, int(2 * L2 // algo_bytes(wl)) + 2))


def cpu_model() -> str:
    try:
        for line in Path("/proc/cpuinfo").read_text().splitlines():
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(seconds: float = 10.0):
    """The CPU oracle (plain C fp64) on full decode GEMVs: OpenMP over all host
    threads for ~`seconds`, then one thread for ~`seconds` / 4."""
    import oracle
    wl = wq_inputs.WORKLOADS[HEADLINE]
    case = wq_inputs.draw(wl, 0)
    wq_, wlo = oracle.pack(case.codes, wl.bits)

    def run(limit):
        reps, t0 = 0, time.perf_counter()
        while True:
            oracle.wq_matmul(case.x, wq_, wlo, case.scales, case.zeros, wl.bits, wl.group_size)
            reps += 1
            el = time.perf_counter() - t0
            if el >= limit or reps >= 2000:
                return reps, el

    cores = oracle.threads()
    reps, el = run(seconds)
    single = None
    try:
        oracle.set_threads(1)
        r1, e1 = run(seconds / 4)
        single = {"value": round(algo_bytes(wl) * r1 / e1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                  "sample": f"{r1} full decode GEMVs in {e1:.1f} s"}
    except AttributeError:
        pass
    finally:
        if hasattr(oracle, "set_threads"):
            oracle.set_threads(cores)
    return {"value": round(algo_bytes(wl) * reps / el / 1e9, 3), "unit": "GB/s", "cores": cores,
            "kind": "oracle", "cpu": cpu_model(), "single_thread": single,
            "numpy": numpy_baseline(seconds / 4),
            "sample": f"{reps} full decode GEMVs (M=1, K=N=4096, 4-bit, g128) in {el:.1f} s, fp64 C, OpenMP"}


def numpy_baseline(seconds: float):
    """The NumPy twin of the oracle (unpack, dequantise, fp64 matmul through the
    BLAS NumPy links) on full decode GEMVs, with the BLAS thread count."""
    import oracle
    wl = wq_inputs.WORKLOADS[HEADLINE]
    case = wq_inputs.draw(wl, 0)
    wq_, wlo = oracle.numpy_oracle.pack(case.codes, wl.bits)
    try:
        from threadpoolctl import threadpool_info
        blas = [{"api": d.get("internal_api"), "threads": d.get("num_threads")} for d in threadpool_info()
                if d.get("user_api") == "blas"]
    except Exception:  # threadpoolctl missing: the count is unknown
        blas = None
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.numpy_oracle.wq_matmul(case.x, wq_, wlo, case.scales, case.zeros, wl.bits, wl.group_size)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds or reps >= 200:
            break
    return {"value": round(algo_bytes(wl) * reps / el / 1e9, 4), "unit": "GB/s", "blas": blas,
            "sample": f"{reps} full decode GEMVs in {el:.1f} s, NumPy fp64 (dequantise, then x @ w)"}


def mse_bench(wq, torch, dev, reps: int = 5):
    """Times wq_mse_search on the page's workload shape with synthetic weights
    drawn like an nn.Linear initialisation (uniform in +-1/sqrt(4096)), and the
    NumPy oracle on a bounded sample of the same shape's rows."""
    import numpy as np
    R, C, G, bits = 14336, 4096, 16, 4
    gen = torch.Generator(device=dev)
    gen.manual_seed(42)
    w = (torch.rand((R, C), generator=gen, device=dev) * 2 - 1) / 64.0
    out = {"workload": f"W {R}x{C} fp32, group {G}, {bits}-bit, 20 candidates (maxshrink 0.2, grid 100), norm 2.4"}
    for name, pat in (("patience_5", 5), ("exhaustive", None)):
        for _ in range(2):
            wq.mse_search(w, bits, G, norm=2.4, patience=pat)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            r = wq.mse_search(w, bits, G, norm=2.4, patience=pat)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        out[name] = {"ms": round(ms, 4), "groups_per_s": round(R * C / G / (ms * 1e-3), 1),
                     "weight_GBps": round(R * C * 4 / (ms * 1e-3) / 1e9, 1)}
    # the oracle (NumPy, fp32 steps and fp64 errors) on 1024 rows of the same shape
    import oracle.mse_observer as mo
    sample = w[:1024].cpu().numpy()
    t0 = time.perf_counter()
    mo.search(sample, bits, G, maxshrink=0.2, grid=100, norm=2.4, patience=5)
    el = time.perf_counter() - t0
    out["cpu_baseline"] = {"groups_per_s": round(1024 * C / G / el, 1), "cores": 1, "kind": "oracle",
                           "sample": f"1024 of the {R} rows ({1024 * C // G} groups) in {el:.2f} s, NumPy"}
    del w, r
    return out


def gptq_bench(wq, torch, dev, reps: int = 3):
    """Times wq_gptq_quantize on the GPTQ page's benchmark problem: W 8192 x 8192
    fp32 drawn like an nn.Linear initialisation, H = A A^T + I (A ~ N(0, 1)),
    symmetric 8-bit arguments with groups of 128 (absolute-maximum scales),
    blocks of 128, percdamp 0.01; and the oracle (NumPy fp32) on a 2048 x 2048
    problem of the same recipe, beside the CUDA path on that problem."""
    import numpy as np

    def problem(n, seed):
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed)
        w = (torch.rand((n, n), generator=gen, device=dev) * 2 - 1) / float(np.sqrt(n))
        a = torch.randn((n, n), generator=gen, device=dev)
        prev = torch.backends.cuda.matmul.allow_tf32
        torch.backends.cuda.matmul.allow_tf32 = False  # the page's fp32 Hessian, not TF32
        h = a @ a.T
        torch.backends.cuda.matmul.allow_tf32 = prev
        h += torch.eye(n, device=dev)
        s = (w.abs().reshape(n, n // 128, 128).amax(-1) / 127.5).contiguous()
        return w, h, s, torch.zeros_like(s)

    def timed(n, k):
        w, h, s, z = problem(n, 42)
        wq.gptq_quantize(w, h, s, z, 128, 8)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(k):
            r = wq.gptq_quantize(w, h, s, z, 128, 8)
        e1.record()
        torch.cuda.synchronize()
        if wq.device_status() != 0:
            raise RuntimeError("wq_gptq_quantize reported a device status")
        return e0.elapsed_time(e1) / k, (w, h, s, z, r)

    n = 8192
    ms, _ = timed(n, reps)
    flops = n ** 3 / 3 + n * n * n  # one Cholesky factorisation + the column updates (R C^2)
    peak = 148 * 128 * 2 * 1.965e9 / 1e12  # fp32 FMA lanes x 2 flop x max SM clock, TFLOP/s
    out = {"workload": f"W {n}x{n} fp32, H = A A^T + I, symmetric 8-bit, group 128, blocks of 128, "
                       "percdamp 0.01 (the GPTQ page's benchmark defaults)",
           "ms": round(ms, 3),
           "roofline": {"bound": "alu", "achieved": round(flops / (ms * 1e-3) / 1e12, 2), "peak": round(peak, 1),
                        "unit": "TFLOP/s", "frac": round(flops / (ms * 1e-3) / 1e12 / peak, 4),
                        "flops": "C^3/3 (one Cholesky) + R C^2 (each column's error times every later column)",
                        "peak_how": "148 SMs x 128 fp32 FMA lanes x 2 x 1965 MHz"},
           "page_context": "the page prints 135 ms for its Triton variant (2191 ms eager) on its own, unnamed GPU"}
    small = 2048
    ms_small, (w, h, s, z, r) = timed(small, reps)
    from oracle import gptq as og
    W, H, S, Z = (t.cpu().numpy() for t in (w, h, s, z))
    t0 = time.perf_counter()
    ref = og.quantize_weight(W, H, S, Z, 128, 8)
    el = time.perf_counter() - t0
    agree = float(np.mean(r["codes"].cpu().numpy().T.astype(np.int32) - 128 == ref["codes"]))
    out["small"] = {"workload": f"{small}x{small}, same recipe", "ms": round(ms_small, 3),
                    "codes_equal_to_oracle": round(agree, 6)}
    out["cpu_baseline"] = {"ms": round(el * 1e3, 1), "kind": "oracle", "cores": os.cpu_count(),
                           "sample": f"the whole {small}x{small} problem, NumPy fp32 with its BLAS/LAPACK threads"}
    del w, h, s, z, r
    return out


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    """The CPU oracle timed as the reference arm, on the headline config and metric."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    import oracle
    wl = wq_inputs.WORKLOADS[HEADLINE]
    case = wq_inputs.draw(wl, 0)
    wq_, wlo = oracle.pack(case.codes, wl.bits)
    # one step = the product for a slice of 256 output columns (1/16 of the GEMV)
    cols = 256
    rng = np.random.default_rng(0)
    def step(i):
        n0 = (i * cols) % wl.N
        ms = np.zeros(cols, np.int32)
        ns = np.arange(n0, n0 + cols, dtype=np.int32)
        oracle.wq_matmul_sampled(case.x, wq_, wlo, case.scales, case.zeros, wl.bits, wl.group_size, ms, ns)
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    el = time.perf_counter() - t0
    frac = cols / wl.N
    bytes_step = algo_bytes(wl) * frac
    v = bytes_step * args.steps / el / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "decode GEMV M=1 K=4096 N=4096 4-bit g128 (fp16 x, s, z)",
                       "parallelism": "cpu oracle"},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
                             "sample": f"each step: {cols} of the {wl.N} output columns of the decode GEMV, "
                                       "each output computed on its own from the packed words (fp64 C)"},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ profiler case
def run_case(name: str, reps: int) -> int:
    """Launch one workload's product `reps` times on one weight set, untimed: the
    command the profiler summaries under profiles/ capture."""
    import torch
    from gemm_wq_gemv_b200 import build as wq_build
    wq_build.build()
    import gemm_wq_gemv_b200 as wq
    dev = torch.device("cuda", 0)
    if name.startswith("gptq_"):  # GPTQ of an n x n problem of the page's recipe, e.g. gptq_2048
        n = int(name.split("_")[1])
        gen = torch.Generator(device=dev)
        gen.manual_seed(42)
        w = (torch.rand((n, n), generator=gen, device=dev) * 2 - 1) / float(n) ** 0.5
        a = torch.randn((n, n), generator=gen, device=dev)
        torch.backends.cuda.matmul.allow_tf32 = False
        h = a @ a.T + torch.eye(n, device=dev)
        s = (w.abs().reshape(n, -1, 128).amax(-1) / 127.5).contiguous()
        for _ in range(reps):
            wq.gptq_quantize(w, h, s, torch.zeros_like(s), 128, 8)
        torch.cuda.synchronize()
        assert wq.device_status() == 0
        print(json.dumps({"case": name, "reps": reps, "kernel": "gptq"}))
        return 0
    wl = wq_inputs.WORKLOADS[name]
    stack = Stack(wq, torch, wl, 1, dev)
    fn = wq.gemv if wl.M <= 16 else wq.gemm
    for _ in range(reps):  # the launch flag of the timed runs, so the same CTA shape
        stack.run(wq, fn, inputs_ready=True)
    torch.cuda.synchronize()
    assert wq.device_status() == 0
    print(json.dumps({"case": name, "reps": reps, "kernel": "gemv" if fn is wq.gemv else "gemm"}))
    return 0


# ------------------------------------------------------------------ GPU arm
def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["wq", "reference"], default="wq")
    ap.add_argument("--no-secondary", action="store_true", help="skip the per-workload table")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ncu-case", metavar="WORKLOAD", default=None,
                    help="only launch WORKLOAD's kernel --reps times, untimed (for profiler captures)")
    ap.add_argument("--reps", type=int, default=6)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.ncu_case:
        return run_case(args.ncu_case, args.reps)

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if dist:
            dist.barrier()

    def max_over_ranks(v):
        return replica_max(v, dist, dev)

    from gemm_wq_gemv_b200 import build as wq_build
    wq_build.build()
    import gemm_wq_gemv_b200 as wq

    props = torch.cuda.get_device_properties(dev)
    L2 = props.L2_cache_size
    hbm_peak, tf_peak, tf_sust, peak_kind = peaks()

    # ---- headline: decode GEMV stack
    wl = wq_inputs.WORKLOADS[HEADLINE]
    L = layers_for(wl, L2)
    stack = Stack(wq, torch, wl, L, dev)
    g, s = capture(torch, lambda: stack.run(wq, wq.gemv, inputs_ready=True))
    sampler = ClockSampler(local)
    el = time_graph(torch, g, s, args.steps, args.warmup, barrier, sampler)
    el = max_over_ranks(el)
    bytes_step = algo_bytes(wl) * L
    value = job_rate(bytes_step, args.steps, world, el) / 1e9
    per_launch_s = el / (args.steps * L)
    achieved = algo_bytes(wl) / per_launch_s / 1e9
    traffic = ncu_traffic(HEADLINE_KERNEL, HEADLINE)

    # ---- the same stack as a dependency chain (x of each product = y of the previous)
    cg, cs = capture(torch, lambda: stack.run_chain(wq))
    c_steps = max(3, min(args.steps, 500))
    c_el = max_over_ranks(time_graph(torch, cg, cs, c_steps, args.warmup, barrier))
    c_launch_s = c_el / (c_steps * L)
    chained = {"us_per_launch": round(c_launch_s * 1e6, 3),
               "GBps": round(algo_bytes(wl) / c_launch_s / 1e9, 1),
               "frac": round(algo_bytes(wl) / c_launch_s / 1e9 / hbm_peak, 4),
               "how": "same stack, x of each product = y of the previous, WQ_FLAG_PDL (wait before reading x)"}
    del cg

    # ---- e2e: the same stack through the API with host buffers
    xs_host = torch.empty((L, wl.M, wl.K), dtype=torch.float16, pin_memory=True)
    for i, st in enumerate(stack.sets):
        xs_host[i].copy_(st[0].cpu())
    ys_host = torch.empty((L, wl.M, wl.N), dtype=torch.float16, pin_memory=True)
    xs_dev = torch.empty((L, wl.M, wl.K), dtype=torch.float16, device=dev)
    ys_dev = torch.empty((L, wl.M, wl.N), dtype=torch.float16, device=dev)
    e2e_steps = max(3, min(args.steps, 200))

    # the layers as a decode loop holds them: one prepared product (wq.GemvPlan)
    # per weight set, and views of the step's x and y buffers
    plans = [wq.GemvPlan(a, b, sc, z, wl.bits, wl.group_size, wl.M, inputs_ready=True)
             for (x, a, b, sc, z, y) in stack.sets]
    x_views = [xs_dev[i] for i in range(L)]
    y_views = [ys_dev[i] for i in range(L)]

    def e2e_step():
        xs_dev.copy_(xs_host, non_blocking=True)
        for plan, xv, yv in zip(plans, x_views, y_views):
            plan(xv, out=yv)
        ys_host.copy_(ys_dev, non_blocking=True)
        torch.cuda.current_stream().synchronize()

    def e2e_step_calls():  # the same through wq.gemv, every argument checked and resolved per call
        xs_dev.copy_(xs_host, non_blocking=True)
        for i, (x, a, b, sc, z, y) in enumerate(stack.sets):
            wq.gemv(xs_dev[i], a, b, sc, z, wl.bits, wl.group_size, out=ys_dev[i], inputs_ready=True)
        ys_host.copy_(ys_dev, non_blocking=True)
        torch.cuda.current_stream().synchronize()

    def time_steps(fn):
        for _ in range(3):
            fn()
        barrier()
        t0 = time.perf_counter()
        for _ in range(e2e_steps):
            fn()
        return max_over_ranks(time.perf_counter() - t0)

    e2e_el = time_steps(e2e_step)
    e2e_value = job_rate(bytes_step, e2e_steps, world, e2e_el) / 1e9
    e2e_calls_value = job_rate(bytes_step, e2e_steps, world, time_steps(e2e_step_calls)) / 1e9

    # the same step (copy in, 31 API calls, copy out) captured once as a CUDA
    # graph and replayed, as a decode loop that captures its step would run it
    def e2e_graph_body():
        xs_dev.copy_(xs_host, non_blocking=True)
        for i, (x, a, b, sc, z, y) in enumerate(stack.sets):
            wq.gemv(xs_dev[i], a, b, sc, z, wl.bits, wl.group_size, out=ys_dev[i], inputs_ready=True)
        ys_host.copy_(ys_dev, non_blocking=True)

    eg, es = capture(torch, e2e_graph_body)
    with torch.cuda.stream(es):
        for _ in range(3):
            eg.replay()
    torch.cuda.synchronize()
    barrier()
    t0 = time.perf_counter()
    with torch.cuda.stream(es):
        for _ in range(e2e_steps):
            eg.replay()
            es.synchronize()
    eg_el = max_over_ranks(time.perf_counter() - t0)
    e2e_graph_value = job_rate(bytes_step, e2e_steps, world, eg_el) / 1e9
    del stack, g, eg, plans

    # ---- GEMM: M=512 prefill product
    gwl = wq_inputs.WORKLOADS[GEMM_WL]
    GL = layers_for(gwl, L2)
    gstack = Stack(wq, torch, gwl, GL, dev)
    gg, gs = capture(torch, lambda: gstack.run(wq, wq.gemm, inputs_ready=True))
    gsteps = max(3, min(args.steps, 200))
    gel = max_over_ranks(time_graph(torch, gg, gs, gsteps, args.warmup, barrier))
    g_launch_s = gel / (gsteps * GL)
    g_tflops = algo_flops(gwl) / g_launch_s / 1e12
    g_traffic = ncu_traffic(GEMM_KERNEL, GEMM_WL)
    del gstack, gg

    # ---- context: the same kernel on a large product (no split-K, many k blocks),
    # where fixed per-launch costs vanish; not a configured workload
    big = None
    if not args.no_secondary:
        # timing only: random packed words (every bit pattern is a valid 4-bit code),
        # drawn on the device; two weight sets (310 MB) so that each call reads HBM
        bM, bK, bN = 256, 16384, 18944
        gen = torch.Generator(device=dev)
        gen.manual_seed(7)
        bx = torch.randn((bM, bK), generator=gen, device=dev).half()
        bsets = []
        for _ in range(2):
            bw = torch.randint(-2**31, 2**31 - 1, (bK // 8, bN), generator=gen, device=dev, dtype=torch.int32)
            bsc = (torch.rand((bK // 128, bN), generator=gen, device=dev) * 0.015 + 0.005).half()
            bz = torch.randint(0, 16, (bK // 128, bN), generator=gen, device=dev).half()
            bsets.append((bw, bsc, bz, torch.empty((bM, bN), dtype=torch.float16, device=dev)))

        def big_run():
            for (bw, bsc, bz, by) in bsets:
                wq.gemm(bx, bw, None, bsc, bz, 4, 128, out=by, inputs_ready=True)

        bg, bs = capture(torch, big_run)
        b_el = time_graph(torch, bg, bs, 10, 3)
        b_us = b_el / (10 * len(bsets)) * 1e6
        b_tf = 2.0 * bM * bK * bN / (b_us * 1e-6) / 1e12
        big = {"workload": f"M={bM} K={bK} N={bN} 4-bit g128 (context, not a configured workload)",
               "us": round(b_us, 2), "TFLOPS": round(b_tf, 1), "frac_of_burst": round(b_tf / tf_peak, 4),
               "frac_of_sustained": round(b_tf / tf_sust, 4) if tf_sust else None}
        del bg, bsets, bx

    # ---- the MSE-observer search (the step that chooses s and z) on the page's
    # benchmark shape: a 14336 x 4096 fp32 weight, group 16, 4 bits, 20 shrink
    # candidates (maxshrink 0.2, grid 100), patience 5, norm 2.4
    mse = None
    if not args.no_secondary:
        mse = mse_bench(wq, torch, dev)

    # ---- GPTQ block quantisation (the step that chooses the codes) on the page's
    # benchmark problem
    gq = None
    if not args.no_secondary:
        gq = gptq_bench(wq, torch, dev)

    # ---- every workload once (rank-local, for the table)
    table = []
    if not args.no_secondary:
        for dtype, (name, w) in [(d, nw) for d in ("fp16", "bf16") for nw in wq_inputs.WORKLOADS.items()]:
            fn = wq.gemm if w.M > 16 else wq.gemv
            n_l = layers_for(w, L2)
            stk = Stack(wq, torch, w, n_l, dev, dtype=dtype)
            gr, st_ = capture(torch, lambda: stk.run(wq, fn, inputs_ready=True))
            reps = 20
            t = time_graph(torch, gr, st_, reps, 3)
            us = t / (reps * n_l) * 1e6
            row = {"workload": name, "dtype": dtype, "M": w.M, "K": w.K, "N": w.N, "bits": w.bits,
                   "group": w.group_size, "kernel": "gemm" if fn is wq.gemm else "gemv", "us": round(us, 3)}
            if fn is wq.gemm:
                tfl = algo_flops(w) / (us * 1e-6) / 1e12
                row.update({"TFLOPS": round(tfl, 1), "frac": round(tfl / tf_peak, 4)})
            else:
                gbs = algo_bytes(w) / (us * 1e-6) / 1e9
                row.update({"GBps": round(gbs, 1), "frac": round(gbs / hbm_peak, 4)})
            table.append(row)
            del stk, gr

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16xf16->f32 (4-bit codes dequantised to f16)",
        "data": "synthetic (seeded: x ~ N(0,1), codes U[0,15], s ~ U[0.005,0.02], integer z U[0,15])",
        "config": {"workload": f"decode GEMV M=1 K=4096 N=4096 4-bit g128, stack of {L} weight sets per step",
                   "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: {bytes_step / 1e6:.0f} MB of distinct weights per step "
                         f"> 2 x {L2 / 1e6:.0f} MB L2",
                   "launch": "one CUDA graph per step; independent products launched with "
                             "WQ_FLAG_PDL_INPUTS_READY (each waits for the previous only before writing y)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                     "nominal_peak": NOMINAL_HBM, "frac_of_nominal": round(achieved / NOMINAL_HBM, 4),
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback",
                     "algorithmic_bytes_per_launch": algo_bytes(wl), "launch_us": round(per_launch_s * 1e6, 3)},
        "gemm": {"workload": "M=512 K=4096 N=2048 4-bit g128", "TFLOPS": round(g_tflops, 1),
                 "us": round(g_launch_s * 1e6, 3),
                 "roofline": {"bound": "tensor", "achieved": round(g_tflops, 1), "peak": tf_peak, "unit": "TFLOP/s",
                              "frac": round(g_tflops / tf_peak, 4), "traffic": g_traffic,
                              "nominal_peak": NOMINAL_TF, "frac_of_nominal": round(g_tflops / NOMINAL_TF, 4),
                              "peak_source": "measured bf16 burst (fp16 nominal ratio 1:1)"},
                 "l2": f"{GL} rotating input sets ({algo_bytes(gwl) * GL / 1e6:.0f} MB) per graph"},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": L * wl.M * wl.K * 2, "d2h_bytes_per_step": L * wl.M * wl.N * 2,
                "how": "python API per layer, one prepared product per weight set (wq.GemvPlan), x copied "
                       "in from pinned host memory and y copied back every step; weights resident",
                "per_call_api": round(e2e_calls_value, 2),
                "per_call_api_how": "the same step through wq.gemv, every argument checked and resolved per call",
                "graph_replay": round(e2e_graph_value, 2),
                "graph_replay_how": "the same step (copies included) captured once as a CUDA graph through "
                                    "the API and replayed, host-synchronised every step"},
        "chained": chained,
        "gemm_large": big,
        "clocks": sampler.report(),
        "gpu_launches": args.steps * L * world,
        "workloads": table,
        "mse_search": mse,
        "gptq": gq,
        "source": src_digest(),
    }
    if rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
