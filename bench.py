#!/usr/bin/env python
"""Throughput of the KroQuant online activation quantizer (kq_quantize) on B200.

One step = one kq_quantize call over the whole bandwidth-stress activation
(16384 x 12288 bf16, Student-t(3), 0.5% outlier channels x100): Kronecker
block transform, E8M0 scale and E2M1 codes for every 32-element block.
Reported as algorithmic GB/s (2 B read + 0.5 B + 1/32 B written per element)
and as a fraction of the measured HBM bandwidth.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 it runs under torch.distributed.run, one rank per GPU; every rank
quantizes its own 16384-row shard of one larger batch (weak scaling, no
collective on the data path); the time is the maximum over ranks.
``--impl reference`` times the float64 CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import collections
import hashlib
import json
import multiprocessing as mp
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "kq_quantize GB/s (bf16 in→MXFP4 out) and % of B200 HBM peak"
UNIT = "GB/s"
GEMM_METRIC = "W4A4 MXFP4 GEMM TFLOP/s on the transformed layer (M x d x d)"
WORKLOAD = "stress"
FALLBACK_HBM_GBS = 6650.0
# Nominal B200 HBM3e bandwidth (8 TB/s): the spec figure, reported beside the
# fraction of the measured copy bandwidth.
SPEC_HBM_GBS = 8000.0
CPU_SAMPLE_ROWS = 4096
REFERENCE_BUDGET_S = 60.0
E2E_WORKSPACE_BYTES = 64 << 20


# ------------------------------------------------------------------ helpers
def dist_env():
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_row0(rank: int, rows_per_rank: int) -> int:
    """First row of this rank's shard in the global batch (weak scaling)."""
    return rank * rows_per_rank


def aggregate_gbs(bytes_per_rank_step: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job GB/s: bytes every rank moved over the slowest rank's time."""
    return bytes_per_rank_step * world * steps / (max_ms * 1e-3) / 1e9


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# Dense FP4 : BF16 tensor throughput on B200, nominal (9 : 2.25 PFLOP/s).
FP4_PER_BF16 = 4.0
FALLBACK_BF16_TFLOPS = 1590.0


def measured_fp4_peak():
    """FP4 tensor peak in TFLOP/s: the measured burst bf16 GEMM rate times
    the nominal FP4 : BF16 ratio."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return FP4_PER_BF16 * float(json.load(f)["bf16_tflops"]), "measured bf16 x 4"
    except (OSError, KeyError, ValueError):
        return FP4_PER_BF16 * FALLBACK_BF16_TFLOPS, "fallback bf16 x 4"


KERNEL_SOURCES = ("kq_kernels.cu", "kq_device.cuh")


def _code_only(text: str) -> str:
    """C++ source without comments and whitespace."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return re.sub(r"\s+", "", text)


def kernel_source_hash() -> str:
    """Hash of the code (comments and whitespace aside) that defines the timed
    kernel: a committed ncu traffic figure is reported only while it holds."""
    h = hashlib.sha256()
    src = os.path.join(ROOT, "w4a4_post_quantization_b200", "csrc")
    for f in KERNEL_SOURCES:
        with open(os.path.join(src, f)) as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_hash: str, name: str):
    """DRAM bytes per launch from a committed ncu record (JSON under
    ``profiles/``), if it was taken on the current kernel sources (else
    None)."""
    path = os.path.join(ROOT, "profiles", name)
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if not isinstance(rec, dict) or rec.get("kernel_source_hash") != kernel_hash:
        return None
    try:
        return float(rec["dram_bytes_per_full_launch"])
    except (KeyError, TypeError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, local_rank: int, period_s: float = 0.0):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            ids = [v for v in vis.split(",") if v.strip()] if vis else []
            ident = ids[local_rank] if local_rank < len(ids) else str(local_rank)
            if ident.startswith("GPU-") or ident.startswith("MIG-"):
                self.h = pynvml.nvmlDeviceGetHandleByUUID(ident)
            else:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(int(ident))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:            # no NVML on this host
            self.nvml, self.error = None, repr(e)
        self._arm()

    def _run(self):
        # Polls from construction on, so that the thread and NVML are warm
        # when the timed region starts; every poll is kept with the times
        # its queries started and ended.
        n = self.nvml
        while not self._stop.is_set():
            t0 = time.perf_counter()
            try:
                mhz = n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM)
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception as e:
                self.error = repr(e)
                return
            self._polls.append((t0, time.perf_counter(), mhz, mask))
            time.sleep(self.period)

    def _arm(self):
        self._polls = collections.deque(maxlen=100000)
        self._t_start = self._t_end = None
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def start(self):
        """Marks the start of the timed region (call right before it)."""
        if self._thread is not None:
            # A short interpreter switch interval lets the sampling thread
            # run between the launching thread's calls.
            self._switch = sys.getswitchinterval()
            sys.setswitchinterval(5e-5)
        self._t_start = time.perf_counter()

    def stop(self):
        """Ends the region.  A poll counts when its queries overlap the region
        (an NVML query can take longer than a short region lasts)."""
        self._t_end = time.perf_counter()
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            if hasattr(self, "_switch"):
                sys.setswitchinterval(self._switch)
        ts, te = self._t_start, self._t_end
        polls = [p for p in self._polls
                 if ts is not None and p[1] >= ts and p[0] <= te]
        self.samples = [p[2] for p in polls]
        for _, _, _, mask in polls:
            for k, bit in self.REASONS.items():
                if mask & bit:
                    self.reasons.add(k)
        durs = [p[1] - p[0] for p in self._polls]
        return {
            "sm_mhz": statistics.median(self.samples) if self.samples else None,
            "sm_max_mhz": self.max_mhz,
            "reasons": sorted(self.reasons),
            "samples": len(self.samples),
            "region_ms": round((te - ts) * 1e3, 3) if ts is not None else None,
            "poll_ms": round(statistics.median(durs) * 1e3, 3) if durs else None,
            "source": "nvml" if self.nvml is not None else f"unavailable: {self.error}",
        }


# -------------------------------------------------------- oracle (CPU) leg
def _oracle_chunk(args):
    """Runs in a spawned worker with one BLAS thread: oracle on a row chunk."""
    bits, params = args
    from oracle import kq_oracle as o
    t0 = time.perf_counter()
    o.quantize(bits, params)
    return time.perf_counter() - t0


def _cpu_workers() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(32, n))


def _worker_ready(pause: float):
    """Imports the oracle in a spawned worker, then holds it briefly so that
    every worker of the pool takes one of these tasks."""
    from oracle import kq_oracle  # noqa: F401
    time.sleep(pause)
    return os.getpid()


def oracle_pool(workers: int):
    """A spawned pool whose workers have all started and imported the
    oracle before it is returned, so that their start-up does not compete
    with the timed GPU launches for the host cores."""
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"
    pool = mp.get_context("spawn").Pool(workers)
    pool.map(_worker_ready, [0.2] * workers, chunksize=1)
    return pool


def time_oracle(pool, case, rows: int, chunk: int = 128, per_chunk=None):
    """Wall time of the oracle over the first ``rows`` rows, split in chunks
    over the pool's workers; ``per_chunk`` (a list) receives each chunk's own
    compute time on its one core."""
    bits = case.x_bits()[:rows]
    jobs = [(bits[r:r + chunk], case.params) for r in range(0, rows, chunk)]
    t0 = time.perf_counter()
    times = pool.map(_oracle_chunk, jobs)
    if per_chunk is not None:
        per_chunk.extend(times)
    return time.perf_counter() - t0


def run_reference(args):
    import workloads as w
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    workers = _cpu_workers()
    pool = oracle_pool(workers)
    M_full = w.CONFIGS[WORKLOAD]["M"]
    probe = w.make_case(WORKLOAD, M=min(M_full, 64 * workers))
    d = probe.d
    # Oracle rate on this host, then rows per step so that all K + W steps
    # take about REFERENCE_BUDGET_S.
    sec = time_oracle(pool, probe, probe.M, chunk=64)
    rate_rows = probe.M / sec
    per_step = REFERENCE_BUDGET_S / (args.steps + args.warmup)
    rows = int(max(workers, min(M_full, rate_rows * per_step)))
    case = w.make_case(WORKLOAD, M=rows)
    chunk = max(1, -(-rows // workers))
    for _ in range(args.warmup):
        time_oracle(pool, case, rows, chunk)
    elapsed = [time_oracle(pool, case, rows, chunk) for _ in range(args.steps)]
    pool.close()
    total = sum(elapsed)
    gbs = w.algorithmic_bytes(rows, d) * args.steps / total / 1e9
    sample = (f"rows 0-{rows - 1} of the {M_full}x{d} stress input per step, "
              f"float64 numpy oracle in {workers} spawned processes, 1 BLAS thread each")
    line = {
        "metric": METRIC, "value": gbs, "unit": UNIT, "impl": "reference",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(_config(d, M_full, "oracle"), sample_rows_per_step=rows),
        "cpu_baseline": {"value": gbs, "unit": UNIT, "cores": workers, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": gbs, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


L2_BYTES = 126e6


def _config(d, M, impl, block=32, case=None):
    x_mb = M * d * 2 / 1e6
    return {
        "workload": (f"bandwidth stress: M={M} tokens x d={d} bf16, Student-t(3), "
                     "0.5% outlier channels x100, learned Kronecker-LU block params"
                     if case is None else
                     f"{case} (seeded DiT-shaped stand-in): M={M} tokens x d={d} bf16"),
        "M": M, "d": d, "block": block,
        "format": f"MXFP4 (E2M1 codes + E8M0 scale per {block})",
        "impl": impl,
        "l2": (f"inputs larger than L2 ({x_mb:.0f} MB x vs 126 MB L2); no flush"
               if M * d * 2 > L2_BYTES else
               f"x ({x_mb:.0f} MB) fits in L2: not a bandwidth measurement"),
    }


# Per-config table: the three quantizers at every config (C0..C4, first gain
# input), per-launch CUDA events with L2 flushed before every launch.
PER_CONFIG_REPS = 50          # single-launch samples per quantizer and config
PER_CONFIG_BLOCKS = 5         # back-to-back blocks per quantizer and config
PER_CONFIG_BLOCK = 100        # launches per block (at least one pass over the copies)
PER_CONFIG_MAX_COPIES = 512
LATENCY_BOUND_US = 10.0     # roofline time below this: launch latency dominates
HOST_AHEAD_CYCLES = 40_000_000   # about 20 ms of device sleep, far longer than queueing 50 launches


def gemm_kernel_name() -> str:
    """The 32-element tiled-scale product kernel the library selects: the
    persistent kernel unless KQ_GEMM_PERSISTENT=0, the CTA pair with
    KQ_GEMM_PAIR=1 (the same switches the library reads)."""
    def flag(var, default):           # the library's reading: atoi(value) != 0
        v = os.environ.get(var)
        if v is None:
            return default
        m = re.match(r"\s*[+-]?\d+", v)
        return bool(m) and int(m.group()) != 0

    if flag("KQ_GEMM_PAIR", False):
        name = "gemm_mxf4_pair"
    elif not flag("KQ_GEMM_PERSISTENT", True):
        name = "gemm_mxf4_kernel"
    else:
        name = "gemm_mxf4_persistent"
    return f"{name}<tiled scales> (tcgen05.mma kind::mxf4)"


def per_config_table(dev, peak, stress=None):
    """kq_quantize, kq_quantize_hadamard and kq_quantize_smooth at every config,
    two ways.  Back to back: blocks of launches cycle over enough copies of x
    (and of the outputs) that every launch reads x from HBM (each copy was
    last touched three L2 sizes of traffic earlier); one event pair around a
    block, the median over blocks.  Single launch: a buffer of twice the L2
    size is overwritten before each launch and an event pair brackets it;
    this includes the event and launch overhead (about 6 us for an empty
    kernel timed the same way).  Configs whose roofline time is under
    LATENCY_BOUND_US are labelled latency-bound.  ``stress`` = (x, params,
    inv_s) already on the device reuses C4's input."""
    import numpy as np
    import torch
    import workloads as w
    import w4a4_post_quantization_b200 as kq
    flush = torch.empty(int(2 * L2_BYTES) // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def block_us(fns, n):
        torch.cuda.synchronize()
        torch.cuda._sleep(HOST_AHEAD_CYCLES)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n):
            fns[i % len(fns)]()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / n

    def single_us(fn):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(PER_CONFIG_REPS)]
        torch.cuda.synchronize()
        torch.cuda._sleep(HOST_AHEAD_CYCLES)
        for e0, e1 in ev:
            flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        return float(np.median([e0.elapsed_time(e1) * 1e3 for e0, e1 in ev]))

    rows = []
    for name, cfg in w.CONFIGS.items():
        for di in range(len(cfg["d"])):
            if name == "stress" and stress is not None:
                x, params, inv_s = stress
            else:
                c = w.make_case(name, di, 0)
                x = c.x.to(dev)
                params = torch.from_numpy(c.params).to(dev)
                inv_s = torch.from_numpy(c.inv_s).to(dev)
            M, d = x.shape
            alg = w.algorithmic_bytes(M, d)
            ncopy = min(PER_CONFIG_MAX_COPIES, max(1, int(np.ceil(3 * L2_BYTES / alg))))
            xs = [x] + [x.clone() for _ in range(ncopy - 1)]
            qs = [torch.empty((M, d // 2), dtype=torch.uint8, device=dev) for _ in range(ncopy)]
            ss = [torch.empty((M, d // 32), dtype=torch.uint8, device=dev) for _ in range(ncopy)]
            seed = w.case_seed(name, di, 0)
            p16 = torch.from_numpy(w.draw_params16(d, seed)).to(dev)
            s16s = [torch.empty((M, d // 16), dtype=torch.uint8, device=dev) for _ in range(ncopy)]
            tokens = w.TOKENS_PER_SAMPLE[name]
            a_sh, a_sc = (t.to(dev) for t in w.draw_adaln(-(-M // tokens), d, seed))
            fams = {"kron": [lambda i=i: kq.quantize(xs[i], params, qs[i], ss[i]) for i in range(ncopy)],
                    "hadamard": [lambda i=i: kq.quantize_hadamard(xs[i], qs[i], ss[i])
                                 for i in range(ncopy)],
                    "smooth": [lambda i=i: kq.quantize_smooth(xs[i], inv_s, qs[i], ss[i])
                               for i in range(ncopy)],
                    "kron_tcgen05": [lambda i=i: kq.quantize(xs[i], params, qs[i], ss[i],
                                                             impl=kq.KQ_IMPL_MMA)
                                     for i in range(ncopy)],
                    "kron16": [lambda i=i: kq.quantize16(xs[i], p16, qs[i], s16s[i])
                               for i in range(ncopy)],
                    "adaln": [lambda i=i: kq.quantize_adaln(xs[i], a_sh, a_sc, tokens, params, 1e-6,
                                                            qs[i], ss[i])
                              for i in range(ncopy)]}
            n = max(PER_CONFIG_BLOCK, ncopy)
            row = {"config": f"{name} d={d}", "M": M, "d": d, "algorithmic_bytes": alg,
                   "copies": ncopy, "launches_per_block": n,
                   "regime": ("latency-bound" if alg / (peak * 1e9) * 1e6 < LATENCY_BOUND_US
                              else "bandwidth")}
            for vname, fns in fams.items():
                # The block-16 variant writes twice the scale bytes.
                b = M * d * (2.0 + 0.5 + 1.0 / 16) if vname == "kron16" else alg
                for f in fns:
                    f()
                blocks = [block_us(fns, n) for _ in range(PER_CONFIG_BLOCKS)]
                med = float(np.median(blocks))
                row[vname] = {"us": med, "min_us": float(min(blocks)), "max_us": float(max(blocks)),
                              "gbs": b / (med * 1e-6) / 1e9,
                              "frac": b / (med * 1e-6) / 1e9 / peak,
                              "frac_spec": b / (med * 1e-6) / 1e9 / SPEC_HBM_GBS,
                              "single_launch_us": single_us(fns[0])}
            rows.append(row)
            del xs, qs, ss, s16s
    del flush
    return {"blocks": PER_CONFIG_BLOCKS, "single_launch_reps": PER_CONFIG_REPS,
            "l2": "back to back over rotating copies of x (3x L2 of traffic between two uses "
                  "of a copy); single launch after overwriting a 2x L2 buffer",
            "host": "launches queued behind a device sleep: events time the device only",
            "latency_bound_below_us": LATENCY_BOUND_US, "rows": rows}


# The W4A4 layer at DiT shapes (M tokens x N out x K in): the square layer
# of the stress input, PixArt-Sigma's MLP up-projection and FLUX.1's.
LAYER_SHAPES = (("stress square", 16384, 12288, 12288), ("pixart_sigma mlp", 8192, 4608, 1152),
                ("flux_schnell mlp", 4608, 12288, 3072))


def queued_ms(fn, n: int, stream, warmup: int = 3) -> float:
    """Average device time of back-to-back calls, queued behind a device
    sleep so that the host's per-call cost (argument checks, the launch) does
    not leave the GPU idle between short kernels; CUDA events on ``stream``.
    At least ``n`` calls and about 2 ms of work are timed, after a few
    untimed calls queued behind the sleep that bring the clocks back up."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    fn()
    torch.cuda.synchronize()
    est = max(time.perf_counter() - t0, 1e-6)
    n = max(n, min(2000, int(2e-3 / est) + 1))
    torch.cuda._sleep(HOST_AHEAD_CYCLES)
    for _ in range(max(warmup, n // 4)):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n


def layer_table(dev, stream, steps: int):
    """Per shape: the block-scaled product alone (TFLOP/s and its fraction of
    the FP4 peak) and the layer as a user runs it (activations quantized on
    the fly into the tiled scale layout, then the product), beside the same
    product in bf16 through torch.matmul."""
    import torch
    import workloads as w
    import w4a4_post_quantization_b200 as kq
    fp4_peak, fp4_src = measured_fp4_peak()
    out = {"peak_tflops": fp4_peak, "peak_source": fp4_src, "kernel": gemm_kernel_name(),
           "out": "bf16", "steps": steps,
           "timing": "back to back, queued behind a device sleep (host cost hidden)",
           "rows": []}
    for label, M, N, K in LAYER_SHAPES:
        # Each shape starts from an idle GPU: right after the square shape's
        # bf16 products (tens of ms at the power cap) the short-K product
        # measured a third slower than on its own.
        torch.cuda.synchronize()
        time.sleep(0.5)
        seed = 4242 + K
        p = torch.from_numpy(w.draw_params(K, seed)).to(dev)
        wt = w.device_randn_bf16((N, K), seed + 7, dev)
        xa = w.device_randn_bf16((M, K), seed + 11, dev)
        qw, sw = kq.quantize_weight_tiled(wt, p)
        qa, sa = kq.quantize_tiled(xa, p)
        c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        flops = 2.0 * M * N * K
        ms_g = queued_ms(lambda: kq.gemm_mxfp4_tiled(qa, sa, qw, sw, out=c,
                                                     out_dtype=torch.bfloat16), steps, stream)

        def layer():
            kq.quantize_tiled(xa, p, qa, sa)
            kq.gemm_mxfp4_tiled(qa, sa, qw, sw, out=c, out_dtype=torch.bfloat16)
        ms_l = queued_ms(layer, steps, stream)
        ms_b = queued_ms(lambda: torch.matmul(xa, wt.t(), out=c), steps, stream)
        tf = flops / (ms_g * 1e-3) / 1e12
        out["rows"].append({"layer": label, "shape_mnk": [M, N, K], "gemm_ms": ms_g,
                            "gemm_tflops": tf, "gemm_frac": tf / fp4_peak,
                            "layer_ms": ms_l, "layer_tflops": flops / (ms_l * 1e-3) / 1e12,
                            "bf16_matmul_ms": ms_b, "layer_speedup_over_bf16": ms_b / ms_l})
        del qw, sw, qa, sa, c, wt, xa
    return out


CONFIG_LABELS = {"tiny d=1152": "C0", "pixart_sigma d=1152": "C1a", "pixart_sigma d=4608": "C1b",
                 "sana d=2240": "C2a", "sana d=5600": "C2b", "flux_schnell d=3072": "C3a",
                 "flux_schnell d=12288": "C3b", "stress d=12288": "C4"}
SUMMARY_COLS = ("kron", "hadamard", "smooth", "kron_tcgen05", "kron16", "adaln")


def compact_summary(variants):
    """The headline figures of the variants, rounded, in a few hundred
    characters (the end of the line): fraction of the measured HBM peak per
    config and quantizer (back to back), the per-config microseconds of
    kq_quantize, and the layer's fraction of the FP4 peak per shape."""
    summ = {}
    pc = variants.get("per_config")
    if pc:
        summ["per_config_cols"] = list(SUMMARY_COLS)
        summ["frac_of_measured_hbm"] = {
            CONFIG_LABELS.get(r["config"], r["config"]):
                [round(r[c]["frac"], 3) if c in r else None for c in SUMMARY_COLS]
            for r in pc["rows"]}
        summ["kron_us"] = {CONFIG_LABELS.get(r["config"], r["config"]): round(r["kron"]["us"], 1)
                           for r in pc["rows"]}
    lt = variants.get("layers")
    if lt:
        summ["gemm_frac_of_fp4"] = {r["layer"]: round(r["gemm_frac"], 3) for r in lt["rows"]}
        summ["layer_speedup_over_bf16"] = {r["layer"]: round(r["layer_speedup_over_bf16"], 2)
                                           for r in lt["rows"]}
    return summ


# --------------------------------------------------------------- GPU leg
def time_steps(fn, steps: int, warmup: int, stream, sampler=None):
    """Average ms per step over exactly ``steps`` calls, CUDA events on
    ``stream``, barrier + synchronize on both sides.  (Queuing the calls
    behind a device sleep measured 1-1.5 % slower at 20 steps on two boxes,
    so the host enqueues them as they run.)"""
    import torch
    import torch.distributed as dist
    for _ in range(warmup):
        fn()
    sync = (lambda: dist.barrier()) if dist.is_initialized() else (lambda: None)
    torch.cuda.synchronize()
    sync()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if sampler is not None:
        sampler.start()
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler is not None else None
    sync()
    return start.elapsed_time(end) / steps, clocks


def run_gpu(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import w4a4_post_quantization_b200 as kq
    import workloads as w

    world, rank, local = dist_env()
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")

    # CPU baseline pool first (spawned, rank 0 at N=1 only).
    pool = None
    if world == 1 and not args.no_cpu_baseline and args.op == "kron":
        pool = oracle_pool(_cpu_workers())

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    if args.case:
        # Another config's input (profiling): name:d_index, full size.
        cname, cdi = args.case.split(":")
        case = w.make_case(cname, int(cdi))
        M = case.M
    else:
        M = args.rows or w.CONFIGS[WORKLOAD]["M"]
        case = w.make_case(WORKLOAD, M=M,
                           row0=shard_row0(rank, -(-M // w.ROW_CHUNK) * w.ROW_CHUNK))
    d = case.d
    x = case.x.to(dev)
    params = torch.from_numpy(case.params).to(dev)
    inv_s = torch.from_numpy(case.inv_s).to(dev)
    q = torch.empty((M, d // 2), dtype=torch.uint8, device=dev)
    s = torch.empty((M, d // 32), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    alg_bytes = w.algorithmic_bytes(M, d)
    # 16-element variant: [d/16, 4, 3] parameters, one scale byte per 16.
    p16 = torch.from_numpy(w.draw_params16(d, case.seed)).to(dev)
    s16 = torch.empty((M, d // 16), dtype=torch.uint8, device=dev)
    bytes16 = M * d * (2.0 + 0.5 + 1.0 / 16)
    if args.op == "kron16":
        alg_bytes = bytes16
    # AdaLN modulation of the batch's samples (bf16 [B, d], read once per
    # CTA and sample: not counted in the algorithmic bytes).
    tokens = w.TOKENS_PER_SAMPLE[args.case.split(":")[0] if args.case else WORKLOAD]
    ada_shift, ada_scale = (t.to(dev) for t in w.draw_adaln(-(-M // tokens), d, case.seed))

    gemm_flops = 2.0 * M * d * d
    gemm_mnk = [M, d, d]
    if args.op == "gemm" and args.gemm_shape:
        # Another layer shape M x N x K (profiling): N(0, 1) activations and
        # weights drawn on the device, parameters of the stress distribution.
        gm, gn, gk = gemm_mnk = args.gemm_shape
        pg = torch.from_numpy(w.draw_params(gk, case.seed)).to(dev)
        Wg = w.device_randn_bf16((gn, gk), case.seed + 7, dev)
        qw, sw = kq.quantize_weight_tiled(Wg, pg)
        xg = w.device_randn_bf16((gm, gk), case.seed + 11, dev)
        qt, st_ = kq.quantize_tiled(xg, pg)
        cg = torch.empty((gm, gn), dtype=torch.bfloat16, device=dev)
        layer_in = (xg, Wg, pg)
        gemm_flops = 2.0 * gm * gn * gk
    elif args.op == "gemm":
        # The layer the codes feed, as the timed step: C = Q(x T) Q(W T^-T)^T
        # with a square synthetic weight (d x d), bf16 output; both
        # quantizers write their scales in the tensor cores' tiled layout.
        Wg = w.device_randn_bf16((d, d), case.seed + 7, dev)
        qw, sw = kq.quantize_weight_tiled(Wg, params)
        qt, st_ = kq.quantize_tiled(x, params)
        cg = torch.empty((M, d), dtype=torch.bfloat16, device=dev)
        layer_in = (x, Wg, params)

    if args.op == "gemm":
        def step():
            kq.gemm_mxfp4_tiled(qt, st_, qw, sw, out=cg, out_dtype=torch.bfloat16)
    elif args.op == "kron":
        def step():
            kq.quantize(x, params, q, s)
    elif args.op == "kron_mma":
        def step():
            kq.quantize(x, params, q, s, impl=kq.KQ_IMPL_MMA)
    elif args.op == "kron16":
        def step():
            kq.quantize16(x, p16, q, s16)
    elif args.op == "adaln":
        def step():
            kq.quantize_adaln(x, ada_shift, ada_scale, tokens, params, 1e-6, q, s)
    elif args.op == "hadamard":
        def step():
            kq.quantize_hadamard(x, q, s)
    else:
        def step():
            kq.quantize_smooth(x, inv_s, q, s)

    # Clock ramp: untimed launches for ~0.3 s so the timed region starts warm.
    t_end = time.perf_counter() + 0.3
    while time.perf_counter() < t_end:
        step()
        torch.cuda.synchronize()
    sampler = ClockSampler(local)
    eager_ms, eager_clocks = time_steps(step, args.steps, args.warmup, stream,
                                        None if args.launch == "graph" else sampler)
    if args.launch == "graph":
        # The K timed steps captured once into a CUDA graph and replayed once:
        # the same K kernel launches without the host's per-launch cost.
        graph, gstream = torch.cuda.CUDAGraph(), torch.cuda.Stream(dev)
        gstream.wait_stream(stream)
        with torch.cuda.graph(graph, stream=gstream):
            for _ in range(args.steps):
                step()
        torch.cuda.synchronize()
        ms, clocks = time_steps(graph.replay, 1, max(args.warmup // args.steps, 3), stream, sampler)
        ms /= args.steps
    else:
        ms, clocks = eager_ms, eager_clocks
    ms_max = max_over_ranks(ms, dev)
    eager_max = max_over_ranks(eager_ms, dev)
    value = aggregate_gbs(alg_bytes, world, args.steps, ms_max * args.steps)
    if args.op == "gemm":
        value = gemm_flops * world / (ms_max * 1e-3) / 1e12

    # Comparators and the copy ceiling on the same input (context, same GPU).
    variants = {}
    if args.op == "gemm" and not args.quick:
        # The linear layer as a user runs it: activations quantized on the fly
        # (the weight offline), then the W4A4 product; against the same
        # product in bf16 through torch.matmul (cuBLAS).
        xl, wl, pl = layer_in
        cb = torch.empty_like(cg)
        n_l = max(3, min(args.steps, 20))
        ms_b, _ = time_steps(lambda: torch.matmul(xl, wl.t(), out=cb), n_l, 3, stream)
        ms_qa, _ = time_steps(lambda: kq.quantize_tiled(xl, pl, qt, st_), n_l, 3, stream)

        def layer_step():
            kq.quantize_tiled(xl, pl, qt, st_)
            kq.gemm_mxfp4_tiled(qt, st_, qw, sw, out=cg, out_dtype=torch.bfloat16)
        ms_l, _ = time_steps(layer_step, n_l, 3, stream)
        ms_b, ms_qa, ms_l = (max_over_ranks(v, dev) for v in (ms_b, ms_qa, ms_l))
        variants["layer"] = {
            "shape_mnk": gemm_mnk, "out": "bf16", "steps": n_l,
            "bf16_matmul": {"ms": ms_b, "tflops": gemm_flops / (ms_b * 1e-3) / 1e12},
            "w4a4": {"ms": ms_l, "quantize_activations_ms": ms_qa,
                     "tflops": gemm_flops / (ms_l * 1e-3) / 1e12},
            "speedup_over_bf16": ms_b / ms_l}
    if not args.quick and args.op != "gemm":
        ms_h, _ = time_steps(lambda: kq.quantize_hadamard(x, q, s), args.steps, args.warmup, stream)
        ms_s, _ = time_steps(lambda: kq.quantize_smooth(x, inv_s, q, s), args.steps, args.warmup,
                             stream)
        ms_max_h = max_over_ranks(ms_h, dev)
        ms_max_s = max_over_ranks(ms_s, dev)
        ms_16, _ = time_steps(lambda: kq.quantize16(x, p16, q, s16), args.steps, args.warmup,
                              stream)
        ms_max_16 = max_over_ranks(ms_16, dev)
        ms_a, _ = time_steps(
            lambda: kq.quantize_adaln(x, ada_shift, ada_scale, tokens, params, 1e-6, q, s),
            args.steps, args.warmup, stream)
        ms_max_a = max_over_ranks(ms_a, dev)
        buf = torch.empty_like(x)
        ms_c, _ = time_steps(lambda: buf.copy_(x), args.steps, args.warmup, stream)
        ms_max_c = max_over_ranks(ms_c, dev)
        impls = {}
        for name, code in (("panel", kq.KQ_IMPL_PANEL), ("tma_flat", kq.KQ_IMPL_TMA),
                           ("direct", kq.KQ_IMPL_DIRECT), ("tcgen05_dense_k", kq.KQ_IMPL_MMA),
                           ("warp_shuffle", kq.KQ_IMPL_WARP)):
            ms_i, _ = time_steps(lambda: kq.quantize(x, params, q, s, impl=code), args.steps,
                                 args.warmup, stream)
            impls[name] = alg_bytes / (max_over_ranks(ms_i, dev) * 1e-3) / 1e9
        variants.update({
            "eager_gbs": aggregate_gbs(alg_bytes, world, 1, eager_max),
            "kq_quantize_impl_gbs": impls,
            "hadamard": {"gbs": alg_bytes / (ms_max_h * 1e-3) / 1e9, "ms": ms_max_h},
            "smooth": {"gbs": alg_bytes / (ms_max_s * 1e-3) / 1e9, "ms": ms_max_s},
            "block16": {"gbs": bytes16 / (ms_max_16 * 1e-3) / 1e9, "ms": ms_max_16,
                        "bytes_per_launch": bytes16},
            "adaln_fused": {"gbs": alg_bytes / (ms_max_a * 1e-3) / 1e9, "ms": ms_max_a,
                            "tokens_per_sample": tokens,
                            "op": "LayerNorm + AdaLN modulate + transform + MXFP4, one pass"},
            "kronecker_over_smooth_speed": ms_max_s / ms_max,
            "d2d_copy_gbs": 2 * x.numel() * 2 / (ms_max_c * 1e-3) / 1e9,
        })
        del buf
        if world == 1 and args.op == "kron" and M == w.CONFIGS[WORKLOAD]["M"] and not args.case:
            variants["per_config"] = per_config_table(dev, measured_peak()[0],
                                                      (x, params, inv_s))
            # The layer the codes feed, C = Q(x T) Q(W T^-T)^T, on the block-
            # scaled tensor cores at three DiT shapes.
            variants["layers"] = layer_table(dev, stream, max(3, min(args.steps, 40)))

    # End to end through the public API: pinned host x in, pinned host codes
    # and scales out, streamed through a device workspace (kq_quantize_host).
    e2e = None
    if not args.no_e2e and args.op == "kron":
        x_host = case.x.pin_memory()
        p_host = torch.from_numpy(case.params).pin_memory()
        q_host = torch.empty((M, d // 2), dtype=torch.uint8).pin_memory()
        s_host = torch.empty((M, d // 32), dtype=torch.uint8).pin_memory()
        p_dev = torch.empty_like(params)
        ws = torch.empty(E2E_WORKSPACE_BYTES, dtype=torch.uint8, device=dev)

        def e2e_step():
            p_dev.copy_(p_host, non_blocking=True)
            kq.quantize_host(x_host, p_dev, q_host, s_host, ws)

        e2e_steps = min(args.steps, 20)
        ms_e, _ = time_steps(e2e_step, e2e_steps, min(args.warmup, 3), stream)
        ms_max_e = max_over_ranks(ms_e, dev)
        h2d = x_host.numel() * 2 + p_host.numel() * 4
        d2h = q_host.numel() + s_host.numel()
        e2e = {"value": aggregate_gbs(alg_bytes, world, 1, ms_max_e), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "ms_per_step": ms_max_e, "api": "kq_quantize_host",
               "workspace_bytes": E2E_WORKSPACE_BYTES}
        kq.quantize(x, params, q, s)
        torch.cuda.synchronize()
        assert torch.equal(q_host, q.cpu()) and torch.equal(s_host, s.cpu())
        del ws

    peak, peak_src = measured_peak()
    per_launch_gbs = alg_bytes / (ms * 1e-3) / 1e9
    khash = kernel_source_hash()
    if args.op == "gemm":
        fp4_peak, fp4_src = measured_fp4_peak()
        tf = gemm_flops / (ms * 1e-3) / 1e12
        roof_gemm = {"bound": "tensor", "achieved": tf, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": tf / fp4_peak, "peak_source": fp4_src, "traffic": None,
                     "algorithmic_flops_per_launch": gemm_flops,
                     "kernel": gemm_kernel_name()}
    roof = {"bound": "hbm", "achieved": per_launch_gbs, "peak": peak, "unit": "GB/s",
            "frac": per_launch_gbs / peak, "peak_source": peak_src,
            # The capture is of one full-size stress launch: other row counts
            # get no traffic figure.
            "traffic": (profiled_traffic(khash, "kq_quantize_stress_traffic.json")
                        if args.op == "kron" and M == w.CONFIGS[WORKLOAD]["M"] and not args.case
                        else None),
            "algorithmic_bytes_per_launch": alg_bytes,
            "kernel": {"kron": "panel_kernel<kron, mx4>", "kron16": "panel_kernel<kron16, mx4>",
                       "gemm": gemm_kernel_name(),
                       "kron_mma": "mma_kernel", "adaln": "adaln_kernel<mx4>",
                       "hadamard": "panel_kernel<hadamard, mx4>",
                       "smooth": "panel_kernel<smooth, mx4>"}[args.op],
            "kernel_source_hash": khash}

    cpu = None
    if pool is not None and rank == 0:
        rows = CPU_SAMPLE_ROWS
        chunk_s = []
        sec = time_oracle(pool, case, rows, per_chunk=chunk_s)
        pool.close()
        cpu = {"value": w.algorithmic_bytes(rows, d) / sec / 1e9, "unit": UNIT,
               "cores": _cpu_workers(), "kind": "oracle",
               "sample": f"rows 0-{rows - 1} of the {M}x{d} stress input, float64 numpy "
                         f"oracle in {_cpu_workers()} spawned processes, 1 BLAS thread each, "
                         f"{sec:.2f} s wall",
               # One core: the same chunks' compute times inside their workers.
               "single_core_value": w.algorithmic_bytes(rows, d) / sum(chunk_s) / 1e9}

    if args.op == "gemm":
        roof = roof_gemm
    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC if args.op != "gemm" else GEMM_METRIC, "value": value,
            "unit": UNIT if args.op != "gemm" else "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32" if args.op != "gemm" else "mxfp4 x mxfp4, f32 accumulate",
            "data": "synthetic",
            "config": dict(_config(d, M, {"kron": "panel", "gemm": "tcgen05 kind::mxf4", "kron16": "panel", "hadamard": "panel",
                                          "smooth": "panel", "kron_mma": "tcgen05 dense K",
                                          "adaln": "fused rows"}[args.op],
                                   16 if args.op == "kron16" else 32,
                                   args.case or None), op=args.op,
                           launch=("cuda_graph: the K steps captured once, replayed once"
                                   if args.launch == "graph" else "eager: one call per step"), global_batch_rows=M * world,
                           parallelism=f"row shards x{world}", clock_ramp_s=0.3,
                           **({"gemm_shape_mnk": gemm_mnk} if args.op == "gemm" else {})),
            "hbm_frac": value / world / peak if args.op != "gemm" else None,
            "hbm_frac_spec": value / world / SPEC_HBM_GBS if args.op != "gemm" else None,
            "spec_hbm_gbs": SPEC_HBM_GBS,
            # Absolute throughput beside the bytes: elements of x per second, all ranks.
            "elements_per_s": (M * d * world / (ms_max * 1e-3)) if args.op != "gemm" else None,
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
            "gpu_launches": args.steps, "variants": variants,
            # Last, so that the end of the line carries the headline figures.
            "summary": dict(compact_summary(variants), hbm_frac=round(value / world / peak, 4),
                            hbm_frac_spec=round(value / world / SPEC_HBM_GBS, 4)),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------- calibration leg
CALIB_LAYER = dict(M=2048, d=1152, N=1152)   # a PixArt-Sigma-width projection


def _calib_inputs(kind: str, seed: int):
    """Synthetic calibration activations [M, d] (N(0, 1) rows) and an
    N(0, 1/d) weight; ``kind`` places two outlier channels (x40 and x25) in
    one 32-block ("inside") or 97 channels apart ("apart", the review's
    falsifier: no 32x32 block can mix them)."""
    import torch
    import workloads as w
    M, d, N = CALIB_LAYER["M"], CALIB_LAYER["d"], CALIB_LAYER["N"]
    x = w.random_bf16((M, d), seed=seed).float()
    chans = (37, 45) if kind == "inside" else (37, 134)
    x[:, chans[0]] *= 40.0
    x[:, chans[1]] *= 25.0
    return x.to(torch.bfloat16), w.draw_weight(N, d, seed)


def _output_loss_at(kc, x, wt, params):
    cal = kc.LayerCalibrator(x, wt, params)
    return cal.losses()[0]


def _smooth_output_loss(kq, x, wt):
    """SmoothQuant's output loss on the GPU: s_c = sqrt(max|x_c| / max|w_c|),
    x diag(s)^-1 and W diag(s) through the per-channel quantizer, the W4A4
    product on the tensor cores, the residual against x W^T."""
    import torch
    ax = x.float().abs().amax(dim=0)
    aw = wt.float().abs().amax(dim=0)
    s = torch.where((ax > 0) & (aw > 0), torch.sqrt(ax / aw.clamp_min(1e-30)),
                    torch.ones_like(ax)).contiguous()
    qa, sa = kq.quantize_smooth(x, (1.0 / s).contiguous())
    qb, sb = kq.quantize_smooth(wt, s)
    y = kq.gemm_mxfp4(qa, sa, qb, sb)
    y_ref = torch.matmul(x.float(), wt.float().t())
    ws = torch.zeros((kq.residual_workspace_bytes(),), dtype=torch.uint8, device=x.device)
    _, ss = kq.residual(y, y_ref, 1.0, ws)
    _, s0 = kq.residual(y_ref, torch.zeros_like(y_ref), 1.0, ws)
    return float(ss.item()) / float(s0.item())


def run_calibration(args):
    """Calibration of the transform on one synthetic layer: time per Adam
    step (the loss, its straight-through gradient and the update, all in the
    library's kernels) and the output error it reaches, beside SmoothQuant,
    the Hadamard initialization and no transform; with the review's two
    falsifiers (outliers more than 32 channels apart; the learned transform
    on jointly permuted channels)."""
    import torch
    import w4a4_post_quantization_b200 as kq
    from w4a4_post_quantization_b200 import calibrate as kc
    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("--op calibrate runs on one GPU")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    steps = 100
    quality = {}
    ms_step = None
    for kind in ("inside", "apart"):
        x, wt = _calib_inputs(kind, seed=2026)
        x, wt = x.to(dev), wt.to(dev)
        nb = x.shape[1] // 32
        ident = torch.zeros((nb, 5, 3), dtype=torch.float32, device=dev)
        ident[:, :, 1] = 1.0
        cal = kc.LayerCalibrator(x, wt)
        l_init = cal.losses()[0]
        cal.run(3)                                    # warm-up steps
        cal = kc.LayerCalibrator(x, wt)
        cal.losses()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        hist = cal.run(steps)
        e1.record()
        torch.cuda.synchronize()
        if kind == "inside":
            ms_step = e0.elapsed_time(e1) / steps
        l_cal = cal.losses()[0]
        perm = torch.randperm(x.shape[1], generator=torch.Generator().manual_seed(7)).to(dev)
        l_perm = _output_loss_at(kc, x[:, perm].contiguous(), wt[:, perm].contiguous(),
                                 cal.params)
        quality[kind] = {
            "output_mse_rel": {"no_transform": _output_loss_at(kc, x, wt, ident),
                               "smoothquant": _smooth_output_loss(kq, x, wt),
                               "hadamard_init": l_init, "kronecker_calibrated": l_cal,
                               "calibrated_on_permuted_channels": l_perm},
            "total_loss_first_last": [hist[0], hist[-1]]}
    M, d, N = CALIB_LAYER["M"], CALIB_LAYER["d"], CALIB_LAYER["N"]
    cpu = None
    if not args.no_cpu_baseline:
        import numpy as np
        from oracle import kq_calibration as oc
        from oracle import kq_oracle as oo
        x, wt = _calib_inputs("inside", seed=2026)
        bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
        x64, w64 = oo.bf16_bits_to_float64(bits(x)), oo.bf16_bits_to_float64(bits(wt))
        t0 = time.perf_counter()
        oc.calibrate(x64, w64, steps=2)
        sec = (time.perf_counter() - t0) / 2
        cpu = {"value": 1000.0 * sec, "unit": "ms per step", "cores": 1, "kind": "oracle",
               "sample": f"2 Adam steps of the float64 oracle on the same {M}x{d}x{N} layer"}
    line = {
        "metric": "transform calibration: ms per Adam step (loss, straight-through "
                  "gradient, update)", "value": ms_step, "unit": "ms", "n_gpus": 1,
        "steps": steps, "warmup": 3, "higher_is_better": False, "data": "synthetic",
        "config": {"workload": f"one linear layer M={M} tokens x d={d} -> N={N}, "
                               "N(0,1) activations with two outlier channels (x40, x25), "
                               "N(0,1/d) weight; Hadamard init, Adam lr 1e-2",
                   **CALIB_LAYER},
        "quality": quality, "cpu_baseline": cpu, "dtype": "f32", "vs_baseline": None}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quick", action="store_true", help="skip the comparator timings")
    ap.add_argument("--launch", default="eager", choices=["graph", "eager"],
                    help="time the K steps as K calls (default) or as one CUDA graph replay")
    ap.add_argument("--op", default="kron", choices=["kron", "kron_mma", "kron16", "adaln", "gemm", "calibrate", "hadamard",
                             "smooth"],
                    help="quantizer timed as the step (kron = kq_quantize, the metric; "
                         "the comparators are for profiling)")
    ap.add_argument("--gemm-shape", type=lambda v: [int(t) for t in v.split(",")], default=None,
                    metavar="M,N,K",
                    help="with --op gemm: time this layer shape instead of the stress "
                         "input's square layer (profiling)")
    ap.add_argument("--case", default="", metavar="NAME:D_INDEX",
                    help="time the quantizer on another config's full-size input, e.g. "
                         "flux_schnell:0 (profiling only)")
    ap.add_argument("--rows", type=int, default=0,
                    help="rows of the stress input per GPU (default: its 16384); "
                         "smaller values are for profiling captures only")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "calibrate":
        return run_calibration(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
