#!/usr/bin/env python
"""Benchmark of the H-BitLinear forward (BitNet v2) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one whole forward -- LayerNorm, Hadamard transform, INT4 absmean
quantization, ternary int8 GEMM on the tensor cores, dequantisation -- over
one batch of the 7B-like Wdown workload (M=8192 tokens, K=16384, N=4096, bf16
in and out).  Ternarising the weight happens once before timing (weights are
static at inference).  The input (268 MB of bf16) is larger than the 126 MB
L2, so no step finds the previous step's activations in cache.

Rank 0 prints one JSON line.  `value` is tokens/s of the whole job (every rank
runs its own replica of the workload: the path shards over tokens with no
collective, so scaling is weak), from CUDA events on the launching stream,
max over ranks.  Extra keys: the roofline of the dominant kernel (the GEMM,
timed per launch with CUDA events on its stream through the stage entry
points), the LN+FHT+quant kernel's HBM figure, an end-to-end figure through
host memory, the oracle on host cores, and SM clocks sampled during timing.

`--impl reference` times the CPU oracle (the pages publish no code to run) on
bounded samples of the same workload, on rank 0 only.
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

METRIC = "H-BitLinear fwd tokens/s + INT8-MMA TOPS (7B Wdown); FHT+quant HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0  # nominal dense ratio on B200: 4.5 POPS int8 vs 2.25 PFLOP/s bf16
INT8_NOMINAL_TOPS = 4500.0  # nominal dense INT8 of one B200


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="wdown_7b")
    ap.add_argument("--bits", type=int, default=4, choices=[4, 8])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the per-config numbers, the size sweeps and the sustained block")
    ap.add_argument("--sustained-seconds", type=float, default=3.0)
    ap.add_argument("--sweep", choices=["k1", "fwd", "k1_noh", "bwd", "kv", "lib"], default=None,
                    help="instead of the step line: the LN+FHT+INT4 kernel alone at M=65536 for each K, "
                         "or the whole forward at K=N=4096 for each M (one JSON line per point)")
    ap.add_argument("--shape", default=None,
                    help="with --sweep k1 or k1_noh: one point M,K instead of the sweep (e.g. for a profiler); "
                         "with --sweep lib: one shape M,K,N")
    a = ap.parse_args(argv)
    a.warmup = max(3, a.warmup)
    return a


def source_digest(paths):
    """sha256 over the named source files (the counters in profiles/ name the kernel source they measured)."""
    import hashlib
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(key):
    """DRAM bytes per launch from the committed ncu summary, or None if the kernel changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f).get(key)
    if not d:
        return None
    if source_digest(d["sources"]) != d["source_sha256"]:
        return None
    return d["dram_bytes_per_launch"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ ranks

class Ranks:
    """torch.distributed plumbing: barrier and max-over-ranks, nothing on the data path."""

    def __init__(self, backend: str):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=180))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, v: float, device=None) -> float:
        if self.pg is None:
            return v
        import torch
        t = torch.tensor([float(v)], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def aggregate_value(tokens_per_rank: int, world: int, max_seconds_per_step: float) -> float:
    """Whole-job throughput: all ranks' tokens over the slowest rank's step time."""
    return tokens_per_rank * world / max_seconds_per_step


# ------------------------------------------------------------------ clocks

# Throttle reasons that make a timed region unusable: the GPU slowed itself
# down for protection (power-cap throttling, sw_power_cap, is normal for a
# dense GEMM on a 1 kW part and is kept and reported).
BAD_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clocks_rejected(clk) -> bool:
    """True if a clock record disqualifies its timed region: a hardware or
    thermal slowdown was active, or the SM clock under load sat well below its
    maximum (under 70%) with no reason reported (a clock lock left behind by
    someone else).  Such a region is measured once more."""
    if not clk or clk.get("sm_mhz") is None:
        return False
    if any(r in BAD_REASONS for r in clk.get("reasons", [])):
        return True
    mx = clk.get("sm_max_mhz")
    return bool(mx) and not clk.get("reasons") and clk["sm_mhz"] < 0.7 * mx

class ClockSampler:
    """SM clock, power and clock-event reasons sampled while timing: NVML every
    millisecond (a timed region of a few milliseconds still gets samples),
    else nvidia-smi every 100 ms.  Reading only; no setting is changed."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, gpu_id: str, period_s: float = 0.001):
        self.gpu_id = gpu_id
        self.period = period_s
        self.proc = None
        self.lines = []
        self.samples = []      # (sm_mhz, max_mhz, reason bitmask) from NVML
        self.t = None
        self.nvml = None
        self._stop = threading.Event()
        self.source = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id)
            self.nvml = (pynvml, h)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.source = "nvml, %.0f ms period" % (self.period * 1e3)
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi, 100 ms period"
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _poll(self):
        pynvml, h = self.nvml
        get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), self.max_mhz,
                                     int(get_reasons(h))))
            except Exception:
                pass
            time.sleep(self.period)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def wait_first_sample(self, timeout=5.0):
        t0 = time.time()
        while time.time() - t0 < timeout and not (self.samples or self.lines):
            time.sleep(0.01)

    def stop(self):
        sm, mx, counts = [], [], {}
        if self.nvml is not None:
            self._stop.set()
            self.t.join(timeout=2)
            for c, m, r in self.samples:
                sm.append(float(c))
                mx.append(float(m))
                for n, bit in self.REASONS:
                    if r & bit:
                        counts[n] = counts.get(n, 0) + 1
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)
            names = [n for n, _ in self.REASONS]
            for ln in self.lines:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        counts[n] = counts.get(n, 0) + 1
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"], "samples": 0}
        load = [s for s in sm if mx and s > 0.3 * max(mx)] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(counts), "reason_samples": counts, "samples": len(sm), "source": self.source}


# ------------------------------------------------------------------ CPU baseline (oracle)

def oracle_rows_per_second(wl, bits: int, seconds: float, max_rows: int = 512):
    """Time the oracle's forward on consecutive seeded rows until `seconds` pass."""
    import numpy as np
    import oracle
    from ternary_gemm_b200.inputs import make_w, make_x_rows
    oracle.build()
    w, a = oracle.ternary(make_w(wl))
    rows = np.arange(min(max_rows, wl.M), dtype=np.int64)
    x = make_x_rows(wl, rows)
    done, t0 = 0, time.perf_counter()
    while done < rows.size:
        oracle.forward_rows(x[done:done + 1], w, a, bits)
        done += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return done / dt, done, dt


def oracle_rows_per_second_all_cores(wl, bits: int, seconds: float, max_rows: int = 2048):
    """The same oracle forward, rows spread over every host core: one thread per
    core, each calling the single-threaded C oracle on its own rows (ctypes
    releases the GIL during the call).  Returns (rows/s, rows, seconds, threads)."""
    import concurrent.futures as cf
    import numpy as np
    import oracle
    from ternary_gemm_b200.inputs import make_w, make_x_rows
    oracle.build()
    w, a = oracle.ternary(make_w(wl))
    threads = max(1, os.cpu_count() or 1)
    rows = np.arange(min(max_rows, wl.M), dtype=np.int64)
    x = make_x_rows(wl, rows)
    deadline = time.perf_counter() + seconds
    counter = {"next": 0}
    lock = threading.Lock()

    def work():
        done = 0
        while time.perf_counter() < deadline:
            with lock:
                i = counter["next"]
                counter["next"] += 1
            if i >= rows.size:
                break
            oracle.forward_rows(x[i:i + 1], w, a, bits)
            done += 1
        return done

    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        done = sum(ex.map(lambda _: work(), range(threads)))
    dt = time.perf_counter() - t0
    return done / dt, done, dt, threads


def run_reference(args):
    """The reference arm: the CPU oracle on bounded samples, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    import oracle
    from ternary_gemm_b200.inputs import WORKLOADS, make_w, make_x_rows
    wl = WORKLOADS[args.workload]
    oracle.build()
    w, a = oracle.ternary(make_w(wl))
    per_step = 1
    x = make_x_rows(wl, np.arange((args.warmup + args.steps) * per_step, dtype=np.int64) % wl.M)
    for s in range(args.warmup):
        oracle.forward_rows(x[s:s + 1], w, a, args.bits)
    t0 = time.perf_counter()
    for s in range(args.warmup, args.warmup + args.steps):
        oracle.forward_rows(x[s:s + 1], w, a, args.bits)
    dt = time.perf_counter() - t0
    value = args.steps * per_step / dt
    sample = ("%d rows of %s (M=%d K=%d N=%d, INT%d), one row per step: LN+FHT+quant+GEMM+dequant in the "
              "single-threaded C oracle" % (args.steps, wl.name, wl.M, wl.K, wl.N, args.bits))
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": wl.name, "M": wl.M, "K": wl.K, "N": wl.N, "bits": args.bits,
                       "x_dtype": wl.dtype, "parallelism": "replicas"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ ours

def _to_device(a):
    import numpy as np
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


# ------------------------------------------------------------------ measurement helpers (ours)

def _events_timed(torch, fn, n, stream, warm=3):
    """Mean seconds per call of fn over n back-to-back calls (CUDA events on `stream`)."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        fn()
    b.record(stream)
    b.synchronize()
    return a.elapsed_time(b) / n / 1e3


def _graph_timed(torch, fn, n):
    """Device seconds per call: n calls captured in one CUDA graph on a side stream, replayed
    (median of 5 replays); the host launch cost is not in it."""
    gs = torch.cuda.Stream()
    with torch.cuda.stream(gs):
        for _ in range(3):
            fn(gs)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=gs):
        for _ in range(n):
            fn(gs)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(gs)
        with torch.cuda.stream(gs):
            g.replay()
        b.record(gs)
        b.synchronize()
        ts.append(a.elapsed_time(b) / n / 1e3)
    del g
    return sorted(ts)[2]


def measure_int8_peak(torch, dev, reps=10):
    """Dense INT8 tensor throughput of this GPU, measured now: the library's int8 GEMM
    (torch._int_mm, cuBLASLt, int32 out) at the 7B Wdown shape, best of `reps` launches."""
    M, K, N = 8192, 16384, 4096
    g = torch.Generator(device=dev).manual_seed(11)
    A = torch.randint(-8, 8, (M, K), device=dev, generator=g, dtype=torch.int8)
    w = torch.randint(-1, 2, (N, K), device=dev, generator=g, dtype=torch.int8)
    try:
        for _ in range(3):
            torch._int_mm(A, w.t())
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            torch._int_mm(A, w.t())
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b) / 1e3)
    except RuntimeError as e:
        return {"tops": None, "error": str(e).splitlines()[0]}
    finally:
        del A, w
        torch.cuda.empty_cache()
    t = min(ts)
    return {"tops": 2.0 * M * N * K / t / 1e12, "us": t * 1e6, "shape": [M, K, N],
            "how": "torch._int_mm (cuBLASLt int8 GEMM, int32 out) at M=%d K=%d N=%d, best of %d, CUDA events"
                   % (M, K, N, reps)}


def stage_times(torch, hbl, x, packed, alpha, N, bits, y, stream, n):
    """Mean seconds per launch of the forward's stages, through the stage entry points
    (the same kernels hbl_forward runs): the quantizer, the weight widening and the GEMM."""
    M, K = x.shape
    dev = x.device
    sc = torch.empty((M,), dtype=torch.float32, device=dev)
    q = torch.empty((M, K), dtype=torch.int8, device=dev)
    Wi = torch.empty((N, K), dtype=torch.int8, device=dev)
    stages = [lambda: hbl.hbl_fht_quant_i8(x, bits, codes=q, scales=sc),
              lambda: hbl.hbl_widen_ternary(packed, K, w=Wi),
              lambda: hbl.hbl_gemm_dequant(q, Wi, sc, alpha, y=y)]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
    for _ in range(3):
        for f in stages:
            f()
    torch.cuda.synchronize()
    for i in range(n):
        for j, f in enumerate(stages):
            evs[i][j].record(stream)
            f()
        evs[i][3].record(stream)
    torch.cuda.synchronize()
    t_k1 = statistics.mean(e[0].elapsed_time(e[1]) for e in evs) / 1e3
    t_wd = statistics.mean(e[1].elapsed_time(e[2]) for e in evs) / 1e3
    t_gm = statistics.mean(e[2].elapsed_time(e[3]) for e in evs) / 1e3
    return t_k1, t_wd, t_gm


def stage_graph_times(torch, hbl, x, packed, alpha, N, bits, y, n):
    """Device seconds per launch of the forward's stages (quantizer, widening, GEMM),
    each captured n times in a CUDA graph: no host launch cost, which small shapes
    would otherwise measure."""
    M, K = x.shape
    dev = x.device
    sc = torch.empty((M,), dtype=torch.float32, device=dev)
    q = torch.empty((M, K), dtype=torch.int8, device=dev)
    Wi = torch.empty((N, K), dtype=torch.int8, device=dev)
    hbl.hbl_fht_quant_i8(x, bits, codes=q, scales=sc)
    hbl.hbl_widen_ternary(packed, K, w=Wi)
    t_k1 = _graph_timed(torch, lambda st: hbl.hbl_fht_quant_i8(x, bits, codes=q, scales=sc, stream=st), n)
    t_wd = _graph_timed(torch, lambda st: hbl.hbl_widen_ternary(packed, K, w=Wi, stream=st), n)
    t_gm = _graph_timed(torch, lambda st: hbl.hbl_gemm_dequant(q, Wi, sc, alpha, y=y, stream=st), n)
    del q, Wi, sc
    return t_k1, t_wd, t_gm


def k1_bytes_of(M, K, x_bytes, bits):
    """Algorithmic bytes of the forward's quantizer launch: x read, codes (one int8 per
    element, the GEMM's operand) and scales written."""
    return M * K * x_bytes + M * K + 4 * M


def config_numbers(torch, hbl, wl, bits, peaks, int8_peak, stream, x=None, packed=None, alpha=None):
    """One workload: tokens/s of hbl_forward, and its GEMM's TOPS and quantizer's GB/s
    from the stage entry points."""
    from ternary_gemm_b200.inputs import make_w, make_x
    if x is None:
        x = _to_device(make_x(wl))
    if packed is None:
        packed, alpha = hbl.hbl_pack_ternary(_to_device(make_w(wl)))
    M, K = x.shape
    N = wl.N
    y = torch.empty((M, N), dtype=x.dtype, device=x.device)
    ws = torch.empty((hbl.hbl_forward_workspace_bytes(M, K, N, bits),), dtype=torch.uint8, device=x.device)
    n = 50 if M * K <= (1 << 25) else 20
    t_eager = _events_timed(torch, lambda: hbl.hbl_forward(x, packed, alpha, N, bits, y=y, workspace=ws), n,
                            stream)
    t = _graph_timed(torch, lambda st: hbl.hbl_forward(x, packed, alpha, N, bits, y=y, workspace=ws, stream=st), n)
    t_k1, t_wd, t_gm = stage_graph_times(torch, hbl, x, packed, alpha, N, bits, y, n)
    ops = 2.0 * M * N * K
    k1_bytes = k1_bytes_of(M, K, x.element_size(), bits)
    out = {"workload": wl.name, "M": M, "K": K, "N": N, "bits": bits, "x_dtype": wl.dtype,
           "tokens_per_s": M / t, "ms_per_forward": t * 1e3, "ms_per_forward_eager": t_eager * 1e3,
           "gemm_tops": ops / t_gm / 1e12, "gemm_frac": ops / t_gm / 1e12 / int8_peak, "gemm_ms": t_gm * 1e3,
           "k1_gbs": k1_bytes / t_k1 / 1e9, "k1_frac": k1_bytes / t_k1 / 1e9 / peaks["hbm_gbs"],
           "k1_ms": t_k1 * 1e3, "widen_ms": t_wd * 1e3,
           "timing": "device time: n launches captured in one CUDA graph (eager: host launches included)"}
    del y, ws
    return out


def k1_sweep(torch, hbl, peaks, stream, M=65536, ks=None):
    """The fused LN+FHT+INT4 kernel alone (packed nibbles out) at M rows for each K."""
    from ternary_gemm_b200.inputs import SWEEP_K1_KS, WORKLOADS, make_x
    base = WORKLOADS["sweep"]
    out = []
    for K in (ks or SWEEP_K1_KS):
        distinct = min(4096, M)               # seeded rows, repeated to M on the device
        x = _to_device(make_x(base.with_shape(distinct, K, 256))).repeat(M // distinct, 1)
        codes = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
        sc = torch.empty((M,), dtype=torch.float32, device=x.device)
        t = _events_timed(torch, lambda: hbl.hbl_fht_quant(x, 4, codes=codes, scales=sc), 20, stream)
        nbytes = M * K * 2 + M * K // 2 + 4 * M
        out.append({"M": M, "K": K, "ms": t * 1e3, "GB/s": nbytes / t / 1e9,
                    "frac": nbytes / t / 1e9 / peaks["hbm_gbs"]})
        del x, codes, sc
        torch.cuda.empty_cache()
    return out


def fwd_sweep(torch, hbl, stream):
    """The whole forward at K = N = 4096 for each token count: device time (CUDA graph)
    and eager time (host launch cost included)."""
    from ternary_gemm_b200.inputs import SWEEP_FWD_MS, WORKLOADS, make_w, make_x
    base = WORKLOADS["sweep"]
    K = N = 4096
    packed, alpha = hbl.hbl_pack_ternary(_to_device(make_w(base.with_shape(1, K, N))))
    out = []
    for M in SWEEP_FWD_MS:
        x = _to_device(make_x(base.with_shape(M, K, N)))
        y = torch.empty((M, N), dtype=x.dtype, device=x.device)
        ws = torch.empty((hbl.hbl_forward_workspace_bytes(M, K, N, 4),), dtype=torch.uint8, device=x.device)
        te = _events_timed(torch, lambda: hbl.hbl_forward(x, packed, alpha, N, 4, y=y, workspace=ws), 50, stream)
        tg = _graph_timed(torch, lambda st: hbl.hbl_forward(x, packed, alpha, N, 4, y=y, workspace=ws, stream=st),
                          20)
        out.append({"M": M, "us_gpu": tg * 1e6, "tokens_per_s_gpu": M / tg, "us_eager": te * 1e6,
                    "path": "one kernel: quantizer + packed-weight product" if M <= 4 else "quantizer + tcgen05 GEMM"})
        del x, y, ws
    return out


def bench_ours(args):
    import numpy as np
    import torch
    from ternary_gemm_b200 import build as hbl_build
    hbl_build.build()
    import ternary_gemm_b200 as hbl
    from ternary_gemm_b200.inputs import WORKLOADS, make_w, make_x

    ranks = Ranks("nccl")
    torch.cuda.set_device(ranks.local)
    dev = torch.device("cuda", ranks.local)
    wl = WORKLOADS[args.workload]
    M, K, N, bits = wl.M, wl.K, wl.N, args.bits
    peaks, peak_kind = load_peaks()

    # CPU baseline first, before any GPU work in this process (rank 0, N = 1 only)
    cpu = cpu_all = None
    if ranks.rank == 0 and ranks.world == 1 and not args.no_cpu_baseline:
        v, n, dt = oracle_rows_per_second(wl, bits, args.cpu_seconds)
        cpu = {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": "%d rows of %s (K=%d, N=%d, INT%d) through LN+FHT+quant+GEMM+dequant, single-threaded C "
                         "oracle, %.1f s" % (n, wl.name, K, N, bits, dt)}
        va, na, dta, nt = oracle_rows_per_second_all_cores(wl, bits, args.cpu_seconds / 2)
        cpu_all = {"value": va, "unit": "tokens/s", "cores": nt, "kind": "oracle",
                   "sample": "%d rows of %s through the same C oracle, one thread per host core, %.1f s"
                             % (na, wl.name, dta)}

    x = _to_device(make_x(wl))
    W = _to_device(make_w(wl))
    stream = torch.cuda.current_stream()
    packed, alpha = hbl.hbl_pack_ternary(W)
    del W
    y = torch.empty((M, N), dtype=x.dtype, device=dev)
    ws = torch.empty((hbl.hbl_forward_workspace_bytes(M, K, N, bits),), dtype=torch.uint8, device=dev)

    def step():
        hbl.hbl_forward(x, packed, alpha, N, bits, y=y, workspace=ws)

    gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # -------- headline: K whole forwards
    def timed_region():
        clocks = ClockSampler(gpu_uuid)
        clocks.start()
        clocks.wait_first_sample()
        ranks.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        e1.synchronize()
        ranks.barrier()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps, clocks.stop()

    ms, clk = timed_region()
    ms_max = ranks.max(ms, dev)
    # a region that any rank's clock record disqualifies is measured once more
    # (every rank takes the same decision: the flag is maxed over ranks)
    rejected = None
    if ranks.max(1.0 if clocks_rejected(clk) else 0.0, dev) > 0:
        rejected = {"ms_per_step": ms_max, "clocks": clk}
        ms, clk = timed_region()
        ms_max = ranks.max(ms, dev)
    value = aggregate_value(M, ranks.world, ms_max / 1e3)

    # -------- per-kernel times through the stage entry points (same kernels as hbl_forward)
    nst = max(20, min(args.steps, 200))
    sclocks = ClockSampler(gpu_uuid)
    sclocks.start()
    sclocks.wait_first_sample()
    t_k1, t_wd, t_gm = stage_times(torch, hbl, x, packed, alpha, N, bits, y, stream, nst)
    stage_clk = sclocks.stop()
    t_gm = ranks.max(t_gm, dev)
    t_k1 = ranks.max(t_k1, dev)

    # -------- the INT8 denominator, measured now on this GPU
    i8 = measure_int8_peak(torch, dev)
    int8_peak = max(i8["tops"] or 0.0, INT8_NOMINAL_TOPS)
    ops = 2.0 * M * N * K
    achieved_tops = ops / t_gm / 1e12
    k1_bytes = k1_bytes_of(M, K, 2 if wl.dtype == "bf16" else 4, bits)
    k1_gbs = k1_bytes / t_k1 / 1e9
    gemm_kernel = "gemm_i8_2sm_kernel (tcgen05 kind::i8, cta_group::2, dequant epilogue)"
    roofline = {"bound": "tensor", "kernel": gemm_kernel,
                "achieved": achieved_tops, "peak": int8_peak, "unit": "TFLOP/s", "frac": achieved_tops / int8_peak,
                "traffic": measured_traffic("gemm_7b_wdown"),
                "peak_source": "larger of the library int8 GEMM measured in this run (%s TOPS) and the nominal "
                               "dense %.0f TOPS" % ("%.1f" % i8["tops"] if i8["tops"] else "n/a",
                                                    INT8_NOMINAL_TOPS),
                "int8_measured": i8,
                "frac_of_bf16_burst_x2": achieved_tops / (peaks["bf16_tflops"] * INT8_OVER_BF16),
                "bf16_burst_kind": peak_kind,
                "algorithmic_ops_per_launch": ops, "launch_ms": t_gm * 1e3}
    if roofline["frac"] > 1.0:
        roofline["peak_suspect"] = "achieved above the peak: the denominator does not bound this kernel"
    k1 = {"bound": "hbm", "kernel": "ln_fht_quant_tc_kernel (tcgen05 high Hadamard factor; INT%d, %s out)"
          % (bits, "int8 codes"), "achieved": k1_gbs,
          "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": k1_gbs / peaks["hbm_gbs"],
          "traffic": measured_traffic("k1_7b_wdown"),
          "algorithmic_bytes_per_launch": k1_bytes, "launch_ms": t_k1 * 1e3}

    # -------- end to end through host memory (pinned), the public call.  The
    # batch goes in row chunks over three streams -- upload, hbl_forward,
    # download -- so PCIe transfers in both directions overlap each other and
    # the GPU work (rows are independent through the whole layer).
    e2e = None
    if not args.no_e2e:
        chunks = 8 if M % 8 == 0 else 1
        cm = M // chunks
        xh = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
        xh.copy_(x)
        yh = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
        xd = torch.empty_like(x)
        s_up, s_cmp, s_dn = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        wsc = torch.empty((hbl.hbl_forward_workspace_bytes(cm, K, N, bits),), dtype=torch.uint8, device=dev)

        def e2e_step():
            for c in range(chunks):
                r0, r1 = c * cm, (c + 1) * cm
                with torch.cuda.stream(s_up):
                    xd[r0:r1].copy_(xh[r0:r1], non_blocking=True)
                    up = torch.cuda.Event()
                    up.record(s_up)
                s_cmp.wait_event(up)
                hbl.hbl_forward(xd[r0:r1], packed, alpha, N, bits, y=y[r0:r1], workspace=wsc, stream=s_cmp)
                done = torch.cuda.Event()
                done.record(s_cmp)
                s_dn.wait_event(done)
                with torch.cuda.stream(s_dn):
                    yh[r0:r1].copy_(y[r0:r1], non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        ranks.barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(s_up)
        s_cmp.wait_event(f0)
        s_dn.wait_event(f0)
        for _ in range(args.e2e_steps):
            e2e_step()
        s_dn.wait_stream(s_up)
        s_dn.wait_stream(s_cmp)
        f1.record(s_dn)
        f1.synchronize()
        ranks.barrier()
        e2e_ms = ranks.max(f0.elapsed_time(f1) / args.e2e_steps, dev)
        e2e = {"value": aggregate_value(M, ranks.world, e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": x.numel() * x.element_size(),
               "d2h_bytes_per_step": y.numel() * y.element_size(), "ms_per_step": e2e_ms,
               "pipeline": "%d row chunks, upload / hbl_forward / download on three streams" % chunks}

    # -------- every workload, the size sweeps and a sustained run (rank 0's GPU, one at a time)
    extras = {}
    if not args.no_extras and ranks.world == 1:
        from ternary_gemm_b200.inputs import WORKLOADS as WL
        cfgs = []
        for name, b in (("tiny", 4), ("wo_1p3b", 4), ("wo_1p3b", 8), ("wdown_3b", 4), ("wdown_7b", 8)):
            same = name == wl.name
            cfgs.append(config_numbers(torch, hbl, WL[name], b, peaks, int8_peak, stream,
                                       x=x if same else None, packed=packed if same else None,
                                       alpha=alpha if same else None))
            torch.cuda.empty_cache()
        extras["configs"] = cfgs
        extras["k1_sweep"] = {"what": "LN+FHT+INT4 alone (hbl_fht_quant, packed nibbles), M=65536, seeded "
                                      "N(0,1) rows with 1% outlier channels x30; GB/s of 2 K + K/2 + 4 bytes per row",
                              "peak_gbs": peaks["hbm_gbs"], "points": k1_sweep(torch, hbl, peaks, stream)}
        extras["fwd_sweep"] = {"what": "hbl_forward at K=N=4096, INT4, bf16 in/out",
                               "points": fwd_sweep(torch, hbl, stream)}
        # sustained: the headline forward for a few seconds, with its own clock record
        ms_est = ms
        nsus = max(1000, int(args.sustained_seconds * 1e3 / ms_est))
        sclk = ClockSampler(gpu_uuid, period_s=0.02)
        sclk.start()
        sclk.wait_first_sample()
        ts = _events_timed(torch, step, nsus, stream)
        sc = sclk.stop()
        extras["sustained"] = {"steps": nsus, "ms_per_step": ts * 1e3, "tokens_per_s": M / ts,
                               "seconds": nsus * ts, "sm_mhz": sc["sm_mhz"], "sm_max_mhz": sc["sm_max_mhz"],
                               "clock_samples": sc["samples"],
                               "sw_power_cap_samples": sc["reason_samples"].get("sw_power_cap", 0),
                               "reasons": sc["reasons"]}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ranks.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": wl.name, "M": M, "K": K, "N": N, "bits": bits, "x_dtype": wl.dtype,
                       "y_dtype": wl.dtype, "l2": "inputs larger than L2 (x is %d MB per step)"
                       % (x.numel() * x.element_size() // 2 ** 20), "parallelism": "replicas"},
            "roofline": roofline, "k1": k1, "int8_tops": achieved_tops,
            "stages_ms": {"ln_fht_quant": t_k1 * 1e3, "widen_ternary": t_wd * 1e3, "gemm_dequant": t_gm * 1e3,
                          "clocks": stage_clk},
            "cpu_baseline": cpu, "cpu_baseline_all_cores": cpu_all, "e2e": e2e, "gpu_launches": 2 * args.steps,
            "clocks": clk}
    if rejected is not None:
        line["remeasured"] = {"why": "the first timed region's clock record showed a slowdown", "first": rejected}
    line.update(extras)
    if ranks.rank == 0:
        print(json.dumps(line), flush=True)
    ranks.barrier()
    ranks.close()
    return 0


def bench_sweep(args):
    """Size sweeps (one JSON line per point, rank 0 / one GPU)."""
    import numpy as np
    import torch
    from ternary_gemm_b200 import build as hbl_build
    hbl_build.build()
    import ternary_gemm_b200 as hbl
    from ternary_gemm_b200.inputs import SWEEP_FWD_MS, SWEEP_K1_KS, WORKLOADS, make_w, make_x
    peaks, peak_kind = load_peaks()
    base = WORKLOADS["sweep"]
    reps = max(3, min(args.steps, 50))
    stream = torch.cuda.current_stream()

    def timed(fn, n):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        b.synchronize()
        return a.elapsed_time(b) / n / 1e3

    def graph_timed(fn, n):
        # device time per call: n calls captured in one CUDA graph on a side stream, replayed
        gs = torch.cuda.Stream()
        with torch.cuda.stream(gs):
            for _ in range(3):
                fn(gs)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=gs):
            for _ in range(n):
                fn(gs)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(gs)
            with torch.cuda.stream(gs):
                g.replay()
            b.record(gs)
            b.synchronize()
            ts.append(a.elapsed_time(b) / n / 1e3)
        del g
        return sorted(ts)[2]

    if args.sweep == "bwd":
        return bench_backward(args, hbl, peaks, peak_kind, timed)
    if args.sweep == "kv":
        # QKV states of 8192 tokens, 32 heads of 128 (the 7B shape), three tensors, bf16
        rows, D = 3 * 8192 * 32, 128
        g = torch.Generator(device="cuda").manual_seed(7)
        x = (torch.randn((rows, D), device="cuda", generator=g) * 2.0).to(torch.bfloat16)
        codes = torch.empty((rows, D), dtype=torch.uint8, device="cuda")
        sc = torch.empty((rows,), dtype=torch.float32, device="cuda")
        for bits in (3, 4, 8):
            t = timed(lambda: hbl.hbl_kv_quant(x, bits, codes=codes, scales=sc), reps)
            nbytes = rows * D * 2 + rows * D + 4 * rows
            gbs = nbytes / t / 1e9
            print(json.dumps({"sweep": "kv_quant", "rows": rows, "D": D, "bits": bits, "ms": t * 1e3, "GB/s": gbs,
                              "frac_hbm": gbs / peaks["hbm_gbs"], "peak_kind": peak_kind,
                              "bytes_per_launch": nbytes, "input": "seeded N(0, 4) bf16 head vectors"}),
                  flush=True)
        return 0
    if args.sweep == "lib":
        # the int8 GEMM beside the library's (torch._int_mm, cuBLASLt) and a bf16 GEMM of
        # the same shape (torch.matmul, cuBLAS), on INT4-range codes and ternary weights;
        # the arms alternate in blocks of launches so that clock drift hits them alike
        g = torch.Generator(device="cuda").manual_seed(11)
        shapes = (("wo_1p3b", (4096, 2048, 2048)), ("wdown_3b", (8192, 8192, 2560)), ("wdown_7b", (8192, 16384, 4096)))
        if args.shape:
            shape = tuple(int(v) for v in args.shape.split(","))
            if len(shape) != 3:
                raise SystemExit("--shape with --sweep lib: M,K,N")
            shapes = (("%dx%dx%d" % shape, shape),)
        for name, (M, K, N) in shapes:
            A = torch.randint(-8, 8, (M, K), device="cuda", generator=g, dtype=torch.int8)
            w = torch.randint(-1, 2, (N, K), device="cuda", generator=g, dtype=torch.int8)
            acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
            Ab, wb = A.to(torch.bfloat16), w.to(torch.bfloat16)
            sc = torch.rand((M,), device="cuda", generator=g)
            al = torch.full((1,), 0.01, device="cuda")
            y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            # ours: int32 sums (the library's output type) and the forward's GEMM (dequantised bf16 y)
            arms = {"ours": lambda: hbl.hbl_gemm_i8_i32(A, w, acc=acc),
                    "ours_dequant_bf16": lambda: hbl.hbl_gemm_dequant(A, w, sc, al, y=y),
                    "cublas_bf16": lambda: torch.matmul(Ab, wb.t())}
            arm_unit = {"ours": "_int8_tops", "ours_dequant_bf16": "_int8_tops", "cublaslt": "_int8_tops",
                        "cublas_bf16": "_tflops"}
            same = None
            try:
                same = bool(torch.equal(torch._int_mm(A, w.t()), hbl.hbl_gemm_i8_i32(A, w, acc=acc)))
                arms["cublaslt"] = lambda: torch._int_mm(A, w.t())
            except RuntimeError as e:     # no int8 library GEMM for this device or shape
                same = str(e).splitlines()[0]
            n = 10 if K >= 8192 else 40
            ts = {k: [] for k in arms}
            clocks = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(0).uuid))
            clocks.start()
            for r in range(16):
                for k in (list(arms) if r % 2 == 0 else list(arms)[::-1]):
                    ts[k].append(timed(arms[k], n))
            clk = clocks.stop()
            ops = 2.0 * M * N * K
            out = {"sweep": "gemm_vs_library", "workload": name, "M": M, "K": K, "N": N}
            for k, v in ts.items():
                t = sorted(v)[len(v) // 2]
                out[k + "_us"] = t * 1e6
                out[k + arm_unit[k]] = ops / t / 1e12
            out["int32_results_identical"] = same
            out["clocks"] = clk
            out["timing"] = "CUDA events; median of 16 blocks of %d launches, the arms alternating" % n
            print(json.dumps(out), flush=True)
            del A, w, acc, Ab, wb, arms, y
            torch.cuda.empty_cache()
        return 0
    if args.sweep in ("k1", "k1_noh"):
        M, ks = 65536, SWEEP_K1_KS
        if args.shape:
            M, K1 = (int(v) for v in args.shape.split(","))
            ks = [K1]
        for K in ks:
            distinct = min(4096, M)              # seeded rows, repeated to M on the device
            if M % distinct:
                raise SystemExit("--shape: M must be a multiple of 4096 or below it")
            x = _to_device(make_x(base.with_shape(distinct, K, 256))).repeat(M // distinct, 1)
            codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
            sc = torch.empty((M,), dtype=torch.float32, device="cuda")
            if args.sweep == "k1":
                t = timed(lambda: hbl.hbl_fht_quant(x, 4, codes=codes, scales=sc), reps)
            else:   # the same LayerNorm + INT4 path without the Hadamard transform
                t = timed(lambda: hbl.hbl_norm_quant(x, 4, hbl.HBL_NORM_LAYER, codes=codes, scales=sc), reps)
            nbytes = M * K * 2 + M * K // 2 + 4 * M
            gbs = nbytes / t / 1e9
            name = "k1_ln_fht_int4" if args.sweep == "k1" else "ln_int4_no_transform"
            print(json.dumps({"sweep": name, "M": M, "K": K, "ms": t * 1e3, "GB/s": gbs,
                              "frac_hbm": gbs / peaks["hbm_gbs"], "peak_kind": peak_kind,
                              "bytes_per_launch": nbytes,
                              "input": "%d seeded rows repeated to %d" % (distinct, M)}),
                  flush=True)
            del x, codes, sc
            torch.cuda.empty_cache()
    else:
        K = N = 4096
        W = _to_device(make_w(base.with_shape(1, K, N)))
        packed, alpha = hbl.hbl_pack_ternary(W)
        for M in SWEEP_FWD_MS:
            x = _to_device(make_x(base.with_shape(M, K, N)))
            y = torch.empty((M, N), dtype=x.dtype, device="cuda")
            ws = torch.empty((hbl.hbl_forward_workspace_bytes(M, K, N, 4),), dtype=torch.uint8, device="cuda")
            t = timed(lambda: hbl.hbl_forward(x, packed, alpha, N, 4, y=y, workspace=ws), reps)
            tg = graph_timed(lambda st: hbl.hbl_forward(x, packed, alpha, N, 4, y=y, workspace=ws, stream=st), 20)
            print(json.dumps({"sweep": "fwd_int4", "M": M, "K": K, "N": N,
                              "path": "packed-weight kernel" if M <= 4 else "widen + tcgen05 GEMM",
                              "us": t * 1e6, "tokens/s": M / t, "int8_tops": 2.0 * M * N * K / t / 1e12,
                              "us_gpu": tg * 1e6, "tokens/s_gpu": M / tg,
                              "timing": "us: eager calls back to back (host launch cost included); "
                                        "us_gpu: 20 calls captured in one CUDA graph, replayed"}), flush=True)
    return 0


def bench_backward(args, hbl, peaks, peak_kind, timed):
    """The straight-through-estimator backward at the step workload (one JSON line):
    tokens/s of hbl_backward, and the roofline of its dominant kernel, the bf16
    tensor-core GEMM (two per call, 2 M N K flops each), timed alone through its
    stage entry point against the measured bf16 peak."""
    import numpy as np
    import torch
    from ternary_gemm_b200.inputs import WORKLOADS, make_w, make_x
    wl = WORKLOADS[args.workload]
    M, K, N = wl.M, wl.K, wl.N
    reps = max(3, min(args.steps, 20))
    x = _to_device(make_x(wl))
    packed, alpha = hbl.hbl_pack_ternary(_to_device(make_w(wl)))
    rng = np.random.default_rng(17)
    gy = _to_device((rng.standard_normal((M, N)).astype(np.float32) * 0.01).view(np.uint32).__rshift__(16)
                    .astype(np.uint16))
    gx = torch.empty_like(x)
    gW = torch.empty((N, K), dtype=torch.float32, device="cuda")
    ws = torch.empty((hbl.hbl_backward_workspace_bytes(M, K, N, args.bits),), dtype=torch.uint8, device="cuda")
    t = timed(lambda: hbl.hbl_backward(x, packed, alpha, N, args.bits, gy, g_x=gx, g_W=gW, workspace=ws), reps)
    # stages alone (same shapes; operand values do not change the timing)
    w16 = torch.randint(-1, 2, (N, K), device="cuda").to(torch.bfloat16)
    q16 = torch.randint(-8, 8, (M, K), device="cuda").to(torch.bfloat16)
    gt = torch.randn((M, K), dtype=torch.float32, device="cuda")
    t_gt = timed(lambda: hbl.hbl_gemm_bf16_f32(gy, w16, scale=alpha, D=gt), reps)
    t_gw = timed(lambda: hbl.hbl_gemm_bf16_f32(gy, q16, a_mn=True, D=gW), reps)
    t_fht = timed(lambda: hbl.hbl_fht_ln_backward(gt, x, g_x=gx), reps)
    flops = 2.0 * M * N * K
    gemm_t = min(t_gt, t_gw)
    achieved = flops / gemm_t / 1e12
    peak = peaks["bf16_tflops"]
    esz = x.element_size()
    print(json.dumps({
        "sweep": "bwd", "metric": "H-BitLinear backward tokens/s (straight-through estimator)",
        "value": M / t, "unit": "tokens/s", "ms": t * 1e3, "dtype": "bf16",
        "config": {"workload": args.workload, "M": M, "K": K, "N": N, "bits": args.bits},
        "roofline": {"bound": "tensor", "kernel": "gemm_bf16_2sm_kernel (tcgen05 kind::f16, cta_group::2)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": "%s bf16 burst" % peak_kind,
                     "algorithmic_flops_per_launch": flops},
        "stages_ms": {"gemm_g_t": t_gt * 1e3, "gemm_g_W": t_gw * 1e3, "fht_ln_backward": t_fht * 1e3},
        "stage_gbs": {"fht_ln_backward": (4.0 + 2.0 * esz) * M * K / t_fht / 1e9},
        "hbm_gbs_peak": peaks["hbm_gbs"],
        "data": "synthetic", "timing": "CUDA events, %d calls after 3 warm-ups, each stage alone" % reps}),
        flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.sweep:
        return bench_sweep(args)
    if args.impl == "reference":
        return run_reference(args)
    return bench_ours(args)


if __name__ == "__main__":
    sys.exit(main())
