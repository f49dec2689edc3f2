#!/usr/bin/env python
"""Throughput of MoE dispatch + combine on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill]
    python bench.py --impl reference ...   # the CPU oracle, timed on host cores

A step is one pass of the hot path over one batch of synthetic tokens that is
already resident in HBM: route (top-k + counts + scan) -> dispatch -> combine,
three kernel launches (two up to 1024 tokens, where route and dispatch run as
one launch).  The expert output Y that combine reads is produced
once before timing by the identity expert (FP8 rows dequantised to bf16);
it is an input of the dispatch+combine metric, like x.  No step finds its
inputs in L2: a step moves more than 4x the L2 size, or else enough buffer
sets rotate that 4x L2 of traffic separates two uses of a set.  Steps run
back to back; the K-step region is timed with CUDA events on the launching
stream and reduced with MAX across ranks.  Kernel durations (for the
roofline) come from a separate pass with events between the kernels, which
would otherwise break the programmatic-launch overlap between them.  With
N > 1 every rank runs an independent replica on its own GPU (the path has no cross-GPU step on one GPU's virtual
ranks), so scaling is weak and value = all ranks' tokens / max time.

`e2e` times the public call a user makes, moe_layer, with pinned host
buffers: host->device copies of logits, x and scales, the layer (route,
dispatch, identity expert, combine) and the device->host copy of out.

`--workload layer` and `--workload layer_fp8` time the MoE layer with SwiGLU
experts instead (bf16, or FP8 with 128-column row scales and 128x128 weight-tile
scales): route + dispatch -> grouped GEMMs on the tensor cores -> combine.
Their roofline line is the grouped GEMMs against HBM or the tensor peak,
whichever binds at the batch.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import workloads  # noqa: E402

METRIC = "dispatch+combine tokens/s and achieved HBM GB/s (% of B200 peak) on 1 GPU"
L2_BYTES = 126 << 20
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ accounting
def algorithmic_bytes(cfg, n: int) -> dict:
    """Bytes each step must move (index maps included; capacity, padding and
    weights excluded)."""
    xb = workloads.DTYPE_BYTES[cfg.x_dtype]
    yb = workloads.DTYPE_BYTES[cfg.y_dtype]
    ob = workloads.DTYPE_BYTES[cfg.out_dtype]
    k, d, e = cfg.top_k, cfg.hidden, cfg.n_experts
    row = d * xb + cfg.scale_cols * 4
    route = n * e * 4 + n * k * 8
    dispatch = n * row + n * k * row + n * k * 8
    combine = n * k * d * yb + n * k * 8 + n * d * ob
    return {"route": route, "dispatch": dispatch, "route_dispatch": route + dispatch,
            "combine": combine, "step": route + dispatch + combine}


# moe_route_dispatch runs route and dispatch as one launch up to this batch
# (the library's documented limit; the binding carries the same constant)
FUSED_MAX_TOKENS = 1024


def describe(cfg, n: int) -> str:
    s = (f"{cfg.name}: N={n}, D={cfg.hidden}, E={cfg.n_experts}, k={cfg.top_k}, "
         f"R={cfg.n_ranks}, x={cfg.x_dtype}")
    if cfg.scale_block:
        s += f" + fp32 scale per {cfg.scale_block} cols"
    s += f", Y={cfg.y_dtype}, out={cfg.out_dtype}, logits={cfg.logits}"
    return s


def step_config(cfg, n: int, n_sets: int, world: int, graph: bool = False,
                two_kernel: bool = False, warm: bool = False) -> dict:
    """The `config` object shared by both arms' JSON lines."""
    step_bytes = algorithmic_bytes(cfg, n)["step"]
    return {"workload": describe(cfg, n), "parallelism": f"replicas{world}",
            "launch": "one CUDA graph per step, replayed" if graph else "eager stream launches",
            "l2": (f"warm: one buffer set reused by every step ({step_bytes / 1e6:.0f} MB, "
                   f"{'inside' if step_bytes < L2_BYTES else 'larger than'} the L2)" if warm else
                   f"no flush: {n_sets} buffer set(s) rotate so a step's data was last touched "
                   f">= 4x L2 ({step_bytes * max(1, n_sets - 1) / 1e6:.0f} MB of traffic) "
                   f"earlier; steps run back to back"),
            "timed": ("moe_route_topk + moe_dispatch + moe_combine: 3 launches/step"
                      if two_kernel else
                      "moe_route_dispatch (route: top-k + counts + scan, then dispatch) + "
                      "moe_combine: " + ("2 launches/step (route and dispatch fused)"
                                         if n <= FUSED_MAX_TOKENS else "3 launches/step")),
            "y_source": "identity expert output, produced once before timing"}


def buffer_sets(cfg, n: int) -> int:
    step = algorithmic_bytes(cfg, n)["step"]
    return 1 if step >= 4 * L2_BYTES else max(1, min(32, -(-4 * L2_BYTES // step) + 1))


def read_peaks() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def _strip_comments(code: bytes) -> bytes:
    """C/C++ source without its comments and blank-line and trailing-space
    differences: what the compiler sees of it (string literals in these
    files hold no comment markers)."""
    code = re.sub(rb"/\*.*?\*/", b" ", code, flags=re.S)
    code = re.sub(rb"//[^\n]*", b"", code)
    lines = [ln.rstrip() for ln in code.split(b"\n")]
    return b"\n".join(ln for ln in lines if ln)


def _device_part(name: str, start: bytes = b"", end: bytes = b"") -> bytes:
    """The code of a source file between two markers (whole ends if absent),
    comments stripped, so that a record stays tied to the code it was taken
    on and not to its comments."""
    with open(os.path.join(ROOT, "combine_moe_route_11_b200", "csrc", name), "rb") as f:
        text = f.read()
    a = text.find(start) if start and start in text else 0
    b = text.find(end) if end and end in text else len(text)
    return _strip_comments(text[a:b])


_HELPERS = b"// ------------------------------------------------------------------ device helpers"


def kernel_source_hash() -> str:
    """Hash of the source the combine kernel is compiled from: combine.cu and
    the device-helper part of the internal header (host-side declarations
    there do not change the kernel)."""
    h = hashlib.sha256()
    h.update(_device_part("combine.cu"))
    h.update(_device_part("moe_internal.cuh", start=_HELPERS))
    return h.hexdigest()[:16]


def gemm_source_hash() -> str:
    """Hash of the device code of the grouped GEMM kernels: swiglu_gemm.cu up to
    its host side, and the device-helper part of the internal header."""
    h = hashlib.sha256()
    h.update(_device_part("swiglu_gemm.cu",
                          end=b"// ---------------------------------------------------------------- host side"))
    h.update(_device_part("moe_internal.cuh", start=_HELPERS))
    return h.hexdigest()[:16]


def fp8_gemm_source_hash() -> str:
    """Hash of the device code of the FP8 grouped GEMM and H quantisation
    kernels: fp8_gemm.cu up to its host side, and the device-helper part of
    the internal header."""
    h = hashlib.sha256()
    h.update(_device_part("fp8_gemm.cu",
                          end=b"// ---------------------------------------------------------------- host side"))
    h.update(_device_part("moe_internal.cuh", start=_HELPERS))
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, source_hash=kernel_source_hash):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f).get(workload)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_hash") != source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock and throttle reasons sampled while the GPU works: through NVML
    every 5 ms (read-only queries; the calls release the GIL), else
    `nvidia-smi -lms 100`.  A timed region shorter than the period reports the
    samples nearest to it and says so."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    # NVML clock-event reason bits, in the order of NAMES
    BITS = [0x8, 0x40, 0x20, 0x4]

    def __init__(self, device_index: int):
        self.samples = []  # (time, sm MHz, max MHz, set of reasons)
        self.proc = None
        self.thread = None
        self.running = False
        self.source = None
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                nvml_index = torch.cuda._get_nvml_device_index(device_index)
            except Exception:
                nvml_index = device_index
            handle = pynvml.nvmlDeviceGetHandleByIndex(nvml_index)
            max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

            def poll():
                while self.running:
                    try:
                        mhz = pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM)
                        bits = get_reasons(handle)
                    except Exception:
                        break
                    active = {nm for nm, bit in zip(self.NAMES, self.BITS) if bits & bit}
                    self.samples.append((time.time(), float(mhz), float(max_mhz), active))
                    time.sleep(0.005)

            self.running = True
            self.source = "nvml, 5 ms"
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.running = False
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(device_index), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.source = "nvidia-smi, 100 ms"
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm, mx = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            active = {nm for nm, v in zip(self.NAMES, parts[2:]) if v.lower().startswith("active")}
            self.samples.append((time.time(), sm, mx, active))

    def wait_first(self, timeout=5.0):
        t0 = time.time()
        while (self.proc or self.running) and not self.samples and time.time() - t0 < timeout:
            time.sleep(0.01)

    def stop(self, t_start: float, t_end: float):
        if self.source is None:
            return None
        if self.running:
            self.running = False
            self.thread.join(timeout=2)
        else:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        all_samples = list(self.samples)
        window = [x for x in all_samples if t_start <= x[0] <= t_end]
        where = "during the timed region"
        if not window and all_samples:
            # a region shorter than the period: the samples closest to it
            mid = 0.5 * (t_start + t_end)
            window = sorted(all_samples, key=lambda x: abs(x[0] - mid))[:2]
            where = "nearest to the timed region (shorter than the sampling period)"
        if not window:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": self.source}
        sm = [x[1] for x in window]
        reasons = set()
        for x in window:
            reasons |= x[3]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[2] for x in window),
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source,
                "window": where}


# ------------------------------------------------------------------ distributed
def init_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def reduce_max(value: float, device) -> float:
    """Max over ranks (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_max_list(values, device) -> list:
    """Element-wise max over ranks of a list of floats."""
    if not (dist.is_available() and dist.is_initialized()):
        return list(values)
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_throughput(world: int, tokens_per_rank: int, max_ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank / (max_ms_per_step * 1e-3)


def barrier(device):
    if dist.is_available() and dist.is_initialized():
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------ CPU oracle timing
def host_cpu() -> dict:
    """The host CPU the oracle runs on: model name and cores."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        avail = len(os.sched_getaffinity(0))
    except AttributeError:
        avail = os.cpu_count() or 1
    return {"cpu_model": model, "cores_available": avail, "nproc": os.cpu_count()}


# most oracle worker processes started at once (each holds its slice's buffers)
MAX_ORACLE_WORKERS = 64

_CFG_FIELDS = ("n_experts", "top_k", "n_ranks", "inter", "x_dtype", "y_dtype", "out_dtype",
               "scale_block")


class OracleCores:
    """The CPU oracle on several host cores at once: one worker process per
    core (oracle/timing_worker.py), each running the unchanged
    single-threaded oracle on its own contiguous slice of the batch's tokens
    as an independent sub-batch.  Workers load their slice first; a step
    sends "go" to all of them and lasts until the slowest one answers."""

    def __init__(self, cfg, inp_np: dict, workers: int):
        import tempfile
        import numpy as np
        n = inp_np["logits"].shape[0]
        self.workers = max(1, min(workers, n))
        self.tokens = n
        self.tmp = tempfile.TemporaryDirectory(prefix="moe_oracle_")
        cfg_path = os.path.join(self.tmp.name, "cfg.json")
        with open(cfg_path, "w") as f:
            json.dump({k: getattr(cfg, k) for k in _CFG_FIELDS}, f)
        bounds = [n * i // self.workers for i in range(self.workers + 1)]
        self.procs = []
        for i in range(self.workers):
            path = os.path.join(self.tmp.name, f"slice{i}.npz")
            np.savez(path, **{k: inp_np[k][bounds[i]:bounds[i + 1]]
                              for k in ("logits", "x", "x_scale") if inp_np.get(k) is not None})
            self.procs.append(subprocess.Popen(
                [sys.executable, "-m", "oracle.timing_worker", path, cfg_path], cwd=ROOT,
                stdin=subprocess.PIPE, stdout=subprocess.PIPE, text=True))
        for p in self.procs:
            if p.stdout.readline().strip() != "ready":
                self.close()
                raise RuntimeError("an oracle worker failed to start")

    def step(self) -> float:
        """Wall seconds of one pass of every worker over its slice."""
        t0 = time.perf_counter()
        for p in self.procs:
            p.stdin.write("go\n")
            p.stdin.flush()
        for p in self.procs:
            float(p.stdout.readline())
        return time.perf_counter() - t0

    def close(self):
        for p in self.procs:
            try:
                p.stdin.write("quit\n")
                p.stdin.flush()
                p.wait(timeout=30)
            except (OSError, subprocess.TimeoutExpired, ValueError):
                p.kill()
        self.tmp.cleanup()


def oracle_inputs(cfg, n: int, seed: int = 0) -> dict:
    return {k: workloads.as_numpy_bits(v) for k, v in
            workloads.make_inputs(cfg, seed=seed, n=n).items()}


def oracle_seconds_per_token(cfg, n_cal: int = 16) -> float:
    """Single-core seconds per token of the oracle's whole path (calibration)."""
    import oracle
    inp = oracle_inputs(cfg, n_cal)
    t0 = time.perf_counter()
    oracle.run_path(cfg, inp)
    return (time.perf_counter() - t0) / n_cal


def time_oracle(cfg, budget_s: float, max_tokens: int, seed: int = 0):
    """Tokens/s of the CPU oracle (route, dispatch, identity expert, combine)
    on one core, on a sample sized to take about budget_s seconds."""
    import oracle
    per_tok = oracle_seconds_per_token(cfg)
    n = int(max(1, min(max_tokens, budget_s / max(per_tok, 1e-9))))
    inp = oracle_inputs(cfg, n, seed)
    t0 = time.perf_counter()
    oracle.run_path(cfg, inp)
    dt = time.perf_counter() - t0
    return n, dt


def cpu_baseline_leg(cfg, n: int) -> dict:
    """The oracle timed on the host: single-threaded on a ~6 s sample, and on
    all host cores (up to MAX_ORACLE_WORKERS) over the whole N-token batch."""
    host = host_cpu()
    nt1, dt1 = time_oracle(cfg, budget_s=6.0, max_tokens=n)
    workers = min(host["cores_available"], MAX_ORACLE_WORKERS)
    pool = OracleCores(cfg, oracle_inputs(cfg, n), workers)
    try:
        pool.step()  # first touch of every buffer
        walls = [pool.step() for _ in range(3)]
    finally:
        pool.close()
    wall = statistics.median(walls)
    path = ("the oracle's whole path (route, counts, offsets, slots, dispatch, identity "
            "expert, combine), unchanged single-threaded C")
    return {"value": n / wall, "unit": "tokens/s", "cores": pool.workers, "kind": "oracle",
            "sample": (f"all {n} tokens of the batch, split into {pool.workers} contiguous "
                       f"slices run as independent sub-batches by {pool.workers} worker "
                       f"processes at once; median of 3 passes ({wall:.2f} s each) after one "
                       f"untimed pass; {path}"),
            **host,
            "single_thread": {"value": nt1 / dt1, "unit": "tokens/s", "cores": 1,
                              "sample": f"{nt1} of the {n} tokens in one process, one pass "
                                        f"in {dt1:.1f} s"}}


def run_reference(args, cfg):
    """The oracle as the reference arm, on the host cores: every step runs a
    bounded sample of the batch's tokens split over the workers, and the
    line reports the measured time of those steps."""
    world, rank, _ = init_dist()
    if rank != 0:
        return
    host = host_cpu()
    workers = min(host["cores_available"], MAX_ORACLE_WORKERS)
    n_steps = args.steps + args.warmup
    per_step_budget = max(0.05, 90.0 / max(1, n_steps))
    per_tok = oracle_seconds_per_token(cfg)
    n = int(max(1, min(cfg.n, per_step_budget * workers / max(per_tok, 1e-9))))
    pool = OracleCores(cfg, oracle_inputs(cfg, n), workers)
    try:
        for _ in range(args.warmup):
            pool.step()
        walls = [pool.step() for _ in range(args.steps)]
    finally:
        pool.close()
    dt = sum(walls)
    value = n * args.steps / dt
    sample = (f"{n} of the {cfg.n} tokens per step (the first {n} of the seed-0 batch), split "
              f"into {pool.workers} contiguous slices run as independent sub-batches by "
              f"{pool.workers} worker processes at once; the oracle's whole path (route, counts, "
              f"offsets, slots, dispatch, identity expert, combine), unchanged single-threaded C")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "tokens_per_step": n,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64 (oracle arithmetic)", "data": "synthetic",
            "config": step_config(cfg, cfg.n, buffer_sets(cfg, cfg.n), args.gpus),
            "step_ms": percentiles([w * 1e3 for w in walls]),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": pool.workers,
                             "kind": "oracle", "sample": sample, **host},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def percentiles(xs) -> dict:
    """p10 / median / p90 of a list (nearest-rank on the sorted values)."""
    v = sorted(xs)
    if not v:
        return {}
    pick = lambda q: v[min(len(v) - 1, max(0, int(round(q * (len(v) - 1)))))]  # noqa: E731
    return {"n": len(v), "p10": pick(0.1), "p50": statistics.median(v), "p90": pick(0.9),
            "min": v[0], "max": v[-1]}


# ------------------------------------------------------------------ GPU arm
# The K-step region repeats back to back until this much work was timed, so
# that the clock sampler sees the GPU under load and regions can be compared.
MIN_WINDOW_S = 0.1
MAX_REPEATS = 2000


def timed_regions(region, stream, dev, steps: int):
    """Time region() -- K steps -- R times back to back, one CUDA event pair
    per region on the launching stream, bracketed by a barrier and a device
    synchronisation on both sides.  R is chosen from one untimed region so
    that the R regions last at least MIN_WINDOW_S.  Returns the regions'
    milliseconds (each the max over ranks) and the wall-clock window."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    region()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    one_ms = reduce_max(e0.elapsed_time(e1), dev)
    repeats = int(min(MAX_REPEATS, max(1, -(-MIN_WINDOW_S * 1e3 // max(one_ms, 1e-3)))))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(repeats + 1)]
    barrier(dev)
    torch.cuda.synchronize(dev)
    t_start = time.time()
    ev[0].record(stream)
    for r in range(repeats):
        region()
        ev[r + 1].record(stream)
    torch.cuda.synchronize(dev)
    t_end = time.time()
    barrier(dev)
    times = reduce_max_list([ev[r].elapsed_time(ev[r + 1]) for r in range(repeats)], dev)
    return times, t_start, t_end


def path_dtype(cfg) -> str:
    """What the path computes in: the row encoding it moves, the expert-output
    and output types, and the accumulation type of the combine."""
    rows = {"f32": "fp32", "bf16": "bf16", "fp8_e4m3": "fp8_e4m3"}[cfg.x_dtype]
    if cfg.scale_block:
        rows += f" + fp32 scale per {cfg.scale_block} cols"
    names = {"f32": "fp32", "bf16": "bf16"}
    return (f"{rows} rows moved as bytes, {names[cfg.y_dtype]} Y / {names[cfg.out_dtype]} out, "
            f"fp32 accumulate")


def time_e2e(mr, plan, inp, n, out_dtype, dev, stream, steps, world):
    """Steps through the public moe_layer call, each with the host->device
    copy of its inputs from pinned memory and the device->host copy of its
    output.  Two buffer slots let the copies run on their own streams: the
    copy-in of step i+1 and the copy-out of step i-1 overlap step i's
    compute (PCIe moves data both ways at once).  Timed with events from the
    first copy-in to the last copy-out, max over ranks."""
    lws = plan.new_workspace(dev, layer=True)
    logits_h = inp["logits"].pin_memory()
    x_h = inp["x"].pin_memory()
    xs_h = inp["x_scale"].pin_memory() if inp["x_scale"] is not None else None
    slots = []
    for _ in range(2):
        slots.append({
            "logits": torch.empty(logits_h.shape, dtype=logits_h.dtype, device=dev),
            "x": torch.empty(x_h.shape, dtype=x_h.dtype, device=dev),
            "xs": torch.empty(xs_h.shape, dtype=xs_h.dtype, device=dev) if xs_h is not None
            else None,
            "out": torch.empty(n, plan.hidden, dtype=out_dtype, device=dev),
            "ev_in": torch.cuda.Event(), "ev_comp": torch.cuda.Event(), "ev_out": torch.cuda.Event()})
    for sl in slots:
        sl["out_h"] = torch.empty(sl["out"].shape, dtype=sl["out"].dtype).pin_memory()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def step(i):
        sl = slots[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(sl["ev_comp"])  # step i-2 has consumed this slot's inputs
            sl["logits"].copy_(logits_h, non_blocking=True)
            sl["x"].copy_(x_h, non_blocking=True)
            if xs_h is not None:
                sl["xs"].copy_(xs_h, non_blocking=True)
            sl["ev_in"].record(s_in)
        stream.wait_event(sl["ev_in"])
        if i >= 2:
            stream.wait_event(sl["ev_out"])  # step i-2's output has left the device
        mr.moe_layer(plan, sl["logits"], sl["x"], sl["xs"], None, None, sl["out"], lws, stream)
        sl["ev_comp"].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(sl["ev_comp"])
            sl["out_h"].copy_(sl["out"], non_blocking=True)
            sl["ev_out"].record(s_out)

    for i in range(4):
        step(i)
    torch.cuda.synchronize(dev)
    barrier(dev)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        step(i)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    if mr.moe_get_status(plan, lws, stream) != 0:
        raise RuntimeError("device status set during e2e")
    e2e_ms = reduce_max(e0.elapsed_time(e1) / steps, dev)
    h2d = logits_h.numel() * 4 + x_h.numel() * x_h.element_size() + \
        (xs_h.numel() * 4 if xs_h is not None else 0)
    d2h = slots[0]["out_h"].numel() * slots[0]["out_h"].element_size()
    return {"value": world * n / (e2e_ms * 1e-3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
            "steps": steps, "call": "moe_layer (identity experts)",
            "pipeline": "two slots: copy-in, moe_layer and copy-out on three streams"}


def run_ours(args, cfg):
    world, rank, local = init_dist()
    import combine_moe_route_11_b200 as mr
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    n = cfg.n
    plan = mr.Plan.from_config(cfg, n_max=n)
    nb = algorithmic_bytes(cfg, n)
    # Buffer sets rotate so that a step never finds its data in L2: the other
    # sets' traffic between two uses of a set is at least 4x the L2 size.
    n_sets = 1 if args.warm_l2 else buffer_sets(cfg, n)
    sets = []
    for si in range(n_sets):
        inp = workloads.make_inputs(cfg, seed=rank * 1000 + si, n=n)
        st = {"inp": inp, "logits": inp["logits"].to(dev), "x": inp["x"].to(dev),
              "xs": inp["x_scale"].to(dev) if inp["x_scale"] is not None else None,
              "ws": plan.new_workspace(dev), "b": plan.new_buffers(n, dev)}
        sets.append(st)

    def cur():
        return torch.cuda.current_stream(dev)

    def route(st):
        b = st["b"]
        mr.moe_route_topk(plan, st["logits"], b["topk_idx"], b["topk_w"], b["counts"],
                          b["expert_off"], st["ws"], cur())

    def dispatch(st):
        b = st["b"]
        mr.moe_dispatch(plan, st["x"], st["xs"], b["topk_idx"], b["recv"], b["recv_scale"],
                        b["slot_of"], b["src_of"], st["ws"], cur())

    def route_dispatch(st):
        b = st["b"]
        mr.moe_route_dispatch(plan, st["logits"], st["x"], st["xs"], b["topk_idx"], b["topk_w"],
                              b["counts"], b["expert_off"], b["recv"], b["recv_scale"],
                              b["slot_of"], b["src_of"], st["ws"], cur())

    def combine(st):
        b = st["b"]
        mr.moe_combine(plan, st["y"], b["topk_w"], b["slot_of"], b["out"], st["ws"], cur())

    # expert output read by combine: identity expert, produced once per set
    for st in sets:
        route(st)
        dispatch(st)
        b = st["b"]
        if cfg.x_dtype == "fp8_e4m3":
            mr.moe_expert_dequant(plan, n, b["recv"], b["recv_scale"], b["slot_of"], b["y"],
                                  st["ws"], stream)
            st["y"] = b["y"]
        else:
            st["y"] = b["recv"]
    torch.cuda.synchronize(dev)
    for st in sets:
        if mr.moe_get_status(plan, st["ws"], stream) != 0:
            raise RuntimeError("device status set before timing")

    # The step is what moe_route_dispatch + moe_combine launch: one fused
    # route + dispatch kernel for small batches, else the route and dispatch
    # kernels (the very launches moe_route_dispatch makes at that size).
    if n <= mr.FUSED_MAX_TOKENS and not args.two_kernel:
        stages = [("route_dispatch", route_dispatch), ("combine", combine)]
    else:
        stages = [("route", route), ("dispatch", dispatch), ("combine", combine)]

    def step(st, evs=None):
        for j, (_, f) in enumerate(stages):
            if evs:
                evs[j].record(cur())
            f(st)
        if evs:
            evs[len(stages)].record(cur())

    for i in range(args.warmup):
        step(sets[i % n_sets])
    # pass 1: per-kernel CUDA events inside every step (kernel durations)
    k_steps = min(args.steps, 200)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
          for _ in range(k_steps)]
    torch.cuda.synchronize(dev)
    for i in range(k_steps):
        step(sets[i % n_sets], ev[i])
    torch.cuda.synchronize(dev)
    kern_ms = {name: sum(e[j].elapsed_time(e[j + 1]) for e in ev) / k_steps
               for j, (name, _) in enumerate(stages)}
    # pass 2: the K-step region back to back, events only around each region;
    # the region repeats until >= MIN_WINDOW_S of timed work, so that the
    # clock samples fall inside it and the spread between regions shows
    sampler = ClockSampler(local)
    sampler.wait_first()
    for i in range(args.warmup):
        step(sets[i % n_sets])
    graphs = None
    if args.graph:
        # one CUDA graph per buffer set holding one whole step; replayed K times
        graphs = []
        for st in sets:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(st)
            graphs.append(g)
        for i in range(args.warmup):
            graphs[i % n_sets].replay()

    def region():
        for i in range(args.steps):
            if graphs:
                graphs[i % n_sets].replay()
            else:
                step(sets[i % n_sets])

    region_ms, t_start, t_end = timed_regions(region, stream, dev, args.steps)
    clocks = sampler.stop(t_start, t_end)
    # per-step distribution: >= 100 steps with an event after every step (the
    # events cut the launch overlap across step boundaries, so these read a
    # little above the back-to-back steps)
    n_dist = max(100, min(args.steps, 1000))
    dev_ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_dist + 1)]
    torch.cuda.synchronize(dev)
    dev_ev[0].record(stream)
    for i in range(n_dist):
        if graphs:
            graphs[i % n_sets].replay()
        else:
            step(sets[i % n_sets])
        dev_ev[i + 1].record(stream)
    torch.cuda.synchronize(dev)
    per_step = [dev_ev[i].elapsed_time(dev_ev[i + 1]) for i in range(n_dist)]
    for st in sets:
        if mr.moe_get_status(plan, st["ws"], stream) != 0:
            raise RuntimeError("device status set during timing")
    ms_step = statistics.median(region_ms) / args.steps
    peak, peak_kind = read_peaks()
    dom = max((k for k in kern_ms if k != "route"), key=lambda k: kern_ms[k])
    achieved = nb[dom] / (kern_ms[dom] * 1e-3) / 1e9
    step_gbs = nb["step"] / (ms_step * 1e-3) / 1e9
    inp = sets[0]["inp"]
    logits, x, xs, b = sets[0]["logits"], sets[0]["x"], sets[0]["xs"], sets[0]["b"]

    # ---- end to end through moe_layer with pinned host buffers
    e2e = None
    if not args.no_e2e:
        e2e = time_e2e(mr, plan, inp, n, sets[0]["b"]["out"].dtype, dev, stream,
                       max(3, min(args.steps, 50)), world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_leg(cfg, n)

    if rank == 0:
        line = {
            "metric": METRIC, "value": job_throughput(world, n, ms_step), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": path_dtype(cfg), "data": "synthetic",
            "config": step_config(cfg, n, n_sets, world, args.graph, args.two_kernel,
                                  args.warm_l2),
            "repeats": len(region_ms),
            "region_ms_per_step": percentiles([r / args.steps for r in region_ms]),
            "step_ms": dict(percentiles(per_step), how="one event after every step"),
            "hbm_gbs": step_gbs, "hbm_pct_of_peak": 100.0 * step_gbs / peak,
            "kernel_us": {k: v * 1e3 for k, v in kern_ms.items()},
            "algorithmic_bytes": nb,
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": recorded_traffic(cfg.name) if dom == "combine" else None},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": len(stages) * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


def run_layer(args, cfg):
    """The MoE layer with SwiGLU experts: route -> dispatch -> grouped GEMMs
    (tcgen05) -> combine.  The roofline line is the grouped GEMM against
    whichever peak bounds it: the weight stream (HBM) at small batches, the
    tensor cores once enough rows share each expert's weights.  Expert
    weights (5.6 GB in bf16, 2.8 GB in FP8 at the layer shape) are drawn on
    the device from a seeded generator with the workload's N(0, w_std)
    distribution, and for FP8 experts quantised per 128x128 tile there;
    parity tests draw them on the host."""
    world, rank, local = init_dist()
    import combine_moe_route_11_b200 as mr
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    n, E, D, I, k = cfg.n, cfg.n_experts, cfg.hidden, cfg.inter, cfg.top_k
    plan = mr.Plan.from_config(cfg, n_max=n)
    fp8 = plan.fp8_experts
    inp = workloads.make_inputs(cfg, seed=rank, n=n, with_weights=False)
    logits, x = inp["logits"].to(dev), inp["x"].to(dev)
    xs = inp["x_scale"].to(dev) if inp["x_scale"] is not None else None
    gen = torch.Generator(device=dev).manual_seed(1000 + rank)
    wdt = torch.uint8 if fp8 else torch.bfloat16
    wgu = torch.empty(E, 2 * I, D, dtype=wdt, device=dev)
    wd = torch.empty(E, D, I, dtype=wdt, device=dev)
    sgu = torch.empty(E, 2 * I // 128, D // 128, device=dev) if fp8 else None
    sd = torch.empty(E, D // 128, I // 128, device=dev) if fp8 else None
    for e in range(E):
        a = torch.randn(2 * I, D, generator=gen, device=dev) * cfg.w_std
        c = torch.randn(D, I, generator=gen, device=dev) * cfg.w_std
        if fp8:
            wgu[e], sgu[e] = workloads.quantise_fp8_tiles(a, 128)
            wd[e], sd[e] = workloads.quantise_fp8_tiles(c, 128)
        else:
            wgu[e], wd[e] = a.to(torch.bfloat16), c.to(torch.bfloat16)
    del a, c
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)

    def route_dispatch():
        # the call moe_layer makes: one launch at n <= 1024, else two
        mr.moe_route_dispatch(plan, logits, x, xs, b["topk_idx"], b["topk_w"], b["counts"],
                              b["expert_off"], b["recv"], b.get("recv_scale"), b["slot_of"],
                              b["src_of"], ws, stream)

    def expert():
        if fp8:
            mr.moe_expert_swiglu_fp8(plan, n, b["recv"], b["recv_scale"], b["counts"],
                                     b["expert_off"], b["slot_of"], wgu, sgu, wd, sd, b["h"],
                                     b["hq"], b["h_scale"], b["y"], ws, stream)
        else:
            mr.moe_expert_swiglu(plan, n, b["recv"], b["counts"], b["expert_off"], wgu, wd,
                                 b["h"], b["y"], ws, stream)

    def combine():
        mr.moe_combine(plan, b["y"], b["topk_w"], b["slot_of"], b["out"], ws, stream)

    stages = [route_dispatch, expert, combine]
    for _ in range(args.warmup):
        for f in stages:
            f()
    k_steps = min(args.steps, 50)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
          for _ in range(k_steps)]
    torch.cuda.synchronize(dev)
    for i in range(k_steps):
        for j, f in enumerate(stages):
            ev[i][j].record(stream)
            f()
        ev[i][len(stages)].record(stream)
    torch.cuda.synchronize(dev)
    names = ["route_dispatch", "expert_gemm", "combine"]
    kern_ms = {nm: sum(e[j].elapsed_time(e[j + 1]) for e in ev) / k_steps
               for j, nm in enumerate(names)}
    sampler = ClockSampler(local)
    sampler.wait_first()

    def region():
        for _ in range(args.steps):
            for f in stages:
                f()

    region_ms, t_start, t_end = timed_regions(region, stream, dev, args.steps)
    clocks = sampler.stop(t_start, t_end)
    if mr.moe_get_status(plan, ws, stream) != 0:
        raise RuntimeError("device status set during timing")
    ms_step = statistics.median(region_ms) / args.steps
    rows = n * k
    flops = 2.0 * rows * (2 * I * D + D * I)
    if fp8:
        # e4m3 weights plus one fp32 scale per 128x128 tile
        wbytes = wgu.numel() + wd.numel() + (sgu.numel() + sd.numel()) * 4
        # activations the layer must move: X codes + scales read, Hq codes +
        # scales written and read, Y written (the bf16 H that GEMM1 hands to
        # the quantisation kernel is this implementation's extra round trip
        # and is not counted)
        abytes = rows * (D + D // 32 + 2 * (I + I // 32) + D * 2)
        kernel = "expert_gemm (GEMM1 + H quantisation + GEMM2)"
    else:
        wbytes = (wgu.numel() + wd.numel()) * 2
        # activations the two GEMMs must move: X rows read, H written and read, Y written
        abytes = rows * (D * 2 + 2 * I * 2 + D * 2)
        kernel = "expert_gemm (GEMM1 + GEMM2)"
    t_gemm = kern_ms["expert_gemm"] * 1e-3
    tfs = flops / t_gemm / 1e12
    gbs = (wbytes + abytes) / t_gemm / 1e9
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except OSError:
        pass
    peak = float(peaks.get("bf16_tflops_sustained", 1400.0))
    peak_kind = "measured sustained" if peaks else "fallback"
    if fp8:
        # no measured e4m3 peak: the bf16 one times the nominal e4m3 / bf16 ratio (4.5 / 2.25)
        peak *= 2.0
        peak_kind += " bf16 x 2 (nominal e4m3/bf16 ratio)"
    hbm_peak, _ = read_peaks()
    # the roofline is whichever resource needs longer at its measured peak
    tensor_line = {"bound": "tensor", "kernel": kernel,
                   "achieved": tfs, "peak": peak, "peak_kind": peak_kind,
                   "unit": "TFLOP/s", "frac": tfs / peak, "traffic": None}
    base = workloads.CONFIGS[cfg.name]
    full_shape = (n, E, D, I) == (base.n, base.n_experts, base.hidden, base.inter)
    record = ("layer_fp8", fp8_gemm_source_hash) if fp8 else ("layer", gemm_source_hash)
    hbm_line = {"bound": "hbm", "kernel": kernel,
                "achieved": gbs, "peak": hbm_peak,
                "peak_kind": "measured" if peaks else "fallback",
                "unit": "GB/s", "frac": gbs / hbm_peak,
                "traffic": recorded_traffic(*record) if full_shape else None,
                "algorithmic_bytes": wbytes + abytes}
    hbm_bound = (wbytes + abytes) / (hbm_peak * 1e9) >= flops / (peak * 1e12)
    roofline, other = (hbm_line, tensor_line) if hbm_bound else (tensor_line, hbm_line)
    if rank == 0:
        line = {
            "metric": "MoE layer tokens/s (route + dispatch + SwiGLU grouped GEMM + combine)",
            "value": world * n / (ms_step * 1e-3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("fp8_e4m3 rows and weights with fp32 block scales, bf16 H/Y/out, fp32 "
                      "accumulate" if fp8 else "bf16 rows, weights, H, Y and out, fp32 accumulate"),
            "data": "synthetic (expert weights drawn on the device, seeded)",
            "repeats": len(region_ms),
            "region_ms_per_step": percentiles([r / args.steps for r in region_ms]),
            "config": {"workload": describe(cfg, n) + f", SwiGLU I={I}, W~N(0,{cfg.w_std})"
                       + (" as e4m3 with an fp32 scale per 128x128 tile" if fp8 else ""),
                       "l2": f"each step streams {wbytes / 1e9:.1f} GB of weights (> 20x L2)"},
            "kernel_us": {kk: v * 1e3 for kk, v in kern_ms.items()},
            "roofline": roofline,
            "roofline_other": other,
            "weight_stream_gbs": wbytes / (kern_ms["expert_gemm"] * 1e-3) / 1e9,
            "weight_stream_frac_of_hbm": wbytes / (kern_ms["expert_gemm"] * 1e-3) / 1e9 / hbm_peak,
            # route(+dispatch), GEMM1, [H quantisation,] GEMM2, combine
            "gpu_launches": ((4 if n <= mr.FUSED_MAX_TOKENS else 5) + (1 if fp8 else 0))
            * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


def run_router(args, cfg):
    """The router GEMM with the top-k fused (moe_router_topk) on the
    workload's routing shape: bf16 hidden rows x [N, D] (drawn ~N(0,1)) and
    router weights [E, D] (~N(0, 0.02)), one call per step (the GEMM with
    the top-k epilogue, then the counts / offsets kernel).  The roofline
    line is the call against whichever of the tensor peak (2 N E D flops)
    and the HBM peak (x and the weights read once, the picks and maps
    written) needs longer."""
    world, rank, local = init_dist()
    import combine_moe_route_11_b200 as mr
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    n, E, D, k = cfg.n, cfg.n_experts, cfg.hidden, cfg.top_k
    rcfg = cfg.replace(x_dtype="bf16", y_dtype="bf16", out_dtype="bf16", scale_block=0)
    plan = mr.Plan.from_config(rcfg, n_max=n)
    gen = torch.Generator(device=dev).manual_seed(2000 + rank)
    # enough buffer sets that a set's x was last read >= 4x L2 earlier
    x_bytes = n * D * 2
    n_sets = max(1, min(16, -(-4 * L2_BYTES // x_bytes) + 1)) if x_bytes < 4 * L2_BYTES else 1
    xs = [torch.randn(n, D, generator=gen, device=dev).to(torch.bfloat16) for _ in range(n_sets)]
    w = (torch.randn(E, D, generator=gen, device=dev) * 0.02).to(torch.bfloat16)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)

    def step(i):
        mr.moe_router_topk(plan, xs[i % n_sets], w, None, b["topk_idx"], b["topk_w"],
                           b["counts"], b["expert_off"], ws, stream)

    for i in range(args.warmup):
        step(i)
    sampler = ClockSampler(local)
    sampler.wait_first()

    def region():
        for i in range(args.steps):
            step(i)

    region_ms, t_start, t_end = timed_regions(region, stream, dev, args.steps)
    clocks = sampler.stop(t_start, t_end)
    if mr.moe_get_status(plan, ws, stream) != 0:
        raise RuntimeError("device status set during timing")
    ms_step = statistics.median(region_ms) / args.steps
    flops = 2.0 * n * E * D
    nbytes = x_bytes + E * D * 2 + n * k * 8 + n * k * 4 + (2 * E + 1) * 4
    t = ms_step * 1e-3
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except OSError:
        pass
    tpeak = float(peaks.get("bf16_tflops", 1590.0))
    hpeak, hkind = read_peaks()
    tensor_line = {"bound": "tensor", "kernel": "moe_router_topk (router GEMM + top-k, counts)",
                   "achieved": flops / t / 1e12, "peak": tpeak,
                   "peak_kind": "measured burst" if peaks else "fallback",
                   "unit": "TFLOP/s", "frac": flops / t / 1e12 / tpeak, "traffic": None}
    hbm_line = {"bound": "hbm", "kernel": "moe_router_topk (router GEMM + top-k, counts)",
                "achieved": nbytes / t / 1e9, "peak": hpeak, "peak_kind": hkind, "unit": "GB/s",
                "frac": nbytes / t / 1e9 / hpeak, "traffic": None, "algorithmic_bytes": nbytes}
    hbm_bound = nbytes / (hpeak * 1e9) >= flops / (tpeak * 1e12)
    roofline, other = (hbm_line, tensor_line) if hbm_bound else (tensor_line, hbm_line)
    if rank == 0:
        print(json.dumps({
            "metric": "router GEMM + top-k tokens/s (moe_router_topk)",
            "value": world * n / t, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 hidden rows and router weights, fp32 accumulate and logits",
            "data": "synthetic (x ~ N(0,1), router weights ~ N(0, 0.02), drawn on the device)",
            "config": {"workload": f"{cfg.name} routing shape: N={n}, D={D}, E={E}, k={k}, "
                                   f"R={cfg.n_ranks}, bf16 hidden rows",
                       "l2": f"{n_sets} x buffer set(s) rotate"},
            "repeats": len(region_ms),
            "region_ms_per_step": percentiles([r / args.steps for r in region_ms]),
            "roofline": roofline, "roofline_other": other,
            "gpu_launches": 2 * args.steps, "clocks": clocks}), flush=True)
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="prefill", choices=sorted(workloads.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--router", action="store_true",
                    help="time the router GEMM with the top-k fused (moe_router_topk) on the "
                         "workload's routing shape instead")
    ap.add_argument("--two-kernel", action="store_true",
                    help="time the route and dispatch kernels (moe_route_topk + moe_dispatch) "
                         "even where moe_route_dispatch would run them as one launch")
    ap.add_argument("--warm-l2", action="store_true",
                    help="reuse one buffer set in every step, so a step that fits in L2 finds "
                         "its data there (the default rotates sets so that it never does)")
    ap.add_argument("--graph", action="store_true",
                    help="replay each step as one captured CUDA graph")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override N (smaller batches for profiler captures, larger ones for "
                         "the supplementary tensor-bound layer runs)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override E (smaller weight sets for profiler captures only)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    cfg = workloads.CONFIGS[args.workload]
    if args.tokens:
        cfg = cfg.replace(n=args.tokens)
    if args.experts:
        cfg = cfg.replace(n_experts=args.experts)
    if args.impl == "reference":
        if cfg.inter > 0 or args.router:
            ap.error("the reference arm times the identity-expert path")
        run_reference(args, cfg)
    elif args.router:
        run_router(args, cfg)
    elif cfg.inter > 0:
        run_layer(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
