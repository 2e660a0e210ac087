#!/usr/bin/env python
"""Throughput benchmark of the attention hot path: one step = forward +
backward of one batch of the workload (default: B=2, H=16, N=8192, d=128,
causal, Q and K drawn with gain 2), inputs resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
    python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N ...

With --workload set to an FP8 workload (fwd_fp8_*), a step is one FP8-mode
forward on inputs quantized to e4m3 beforehand (quantization is in the e2e
leg, not in the kernel timing), against twice the measured bf16 peak (the
nominal FP8 : bf16 ratio of the tensor cores).

With --workload set to a decode workload (decode_*), a step is one decode
call (Nq new queries per head against an Nk-key KV cache) and the metric is
algorithmic bytes moved per second, bound by HBM.

Prints one JSON line (rank 0). Multi-GPU runs are weak scaling: every rank
runs its own batch of the same per-GPU size (attention over independent
(batch, head) slices needs no exchange), timed on the device between
barriers, maximum over ranks. FLOPs are algorithmic: 4*B*Hq*N^2*d for the
forward (half when causal) and 2.5x that for the backward.
"""

from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOP/s (bf16) and fraction of B200 dense BF16 peak"
FP8_METRIC = "attention forward TFLOP/s in FP8 mode (e4m3 operands, block scales) and fraction of B200 dense FP8 peak"
DECODE_METRIC = "decode attention: algorithmic HBM bytes per second (read q, K/V cache; write o, lse)"
DEFAULT_WORKLOAD = "fwdbwd_b2_h16_n8192_d128_causal_peaky"
L2_BYTES = 126 << 20     # B200 L2
FLUSH_BYTES = 512 << 20  # written before each timed step when the inputs do not exceed 2x L2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["native", "reference"], default="native")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--e2e-steps", type=int, default=None,
                   help="end-to-end steps through the public API (default: --steps; 0 skips them)")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    args = p.parse_args(argv)
    if args.e2e_steps is None:
        args.e2e_steps = args.steps
    return args


# ----------------------------------------------------------------- ranks

def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(
        os.environ.get("LOCAL_RANK", "0"))


def init_dist(backend: str):
    import torch.distributed as dist

    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def max_over_ranks(x: float, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (identity without a group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        if isinstance(pk, dict):
            return pk, "measured"
    except (OSError, ValueError):
        pass
    return dict(FALLBACK_PEAKS), "fallback"


def peak_value(key: str):
    """(value, source) of one roofline denominator: the measured figure when
    MEASURED_PEAKS.json holds a positive number under ``key``, else the
    fallback figure, labelled as such."""
    pk, src = load_peaks()
    v = pk.get(key)
    if isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0:
        return float(v), src
    return float(FALLBACK_PEAKS[key]), "fallback"


def captured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of ``kernel`` on ``workload`` from the ncu
    capture table profiles/traffic.json, or None when there is no entry or
    the kernel's sources changed since the capture (sha256 of their
    concatenation, first 16 hex digits)."""
    import hashlib

    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            captures = json.load(f)["captures"]
    except (OSError, ValueError, KeyError):
        return None
    for c in captures:
        if c.get("kernel") != kernel or c.get("workload") != workload:
            continue
        m = hashlib.sha256()
        try:
            for src in c["sources"]:
                with open(os.path.join(ROOT, "exact_io_aware_56_b200", "csrc", src), "rb") as f:
                    m.update(f.read())
        except (OSError, KeyError):
            return None
        if m.hexdigest()[:16] != c.get("sha256_16"):
            return None
        return int(c["traffic_bytes"])
    return None


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clocks and clock-event (throttle) reasons while the timed
    region runs. Polls NVML from a thread every ~1 ms (read-only queries;
    nothing is set), falling back to ``nvidia-smi -lms 20``; the summary keeps
    only the samples taken between ``begin()`` and ``end()`` (host time),
    and the nearest one if the region is shorter than the polling period."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.device = device
        self.samples = []  # (host time, sm MHz, max sm MHz, set of reason names)
        self.t_begin = self.t_end = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None

    def _bus_id(self):
        """PCI bus id of the CUDA device (unaffected by CUDA_VISIBLE_DEVICES)."""
        import torch

        p = torch.cuda.get_device_properties(self.device)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        bus = self._bus_id()
        for arg in (bus, bus.encode()):
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(arg)
            except Exception:
                pass
        if "CUDA_VISIBLE_DEVICES" not in os.environ:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.device.index)
        raise RuntimeError(f"no NVML device with PCI bus id {bus}")

    def _poll_nvml(self, pynvml, h):
        reasons_of = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or getattr(
            pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self._stop.is_set():
            sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
            bits = reasons_of(h)
            names = {n for b, n in self.REASONS.items() if bits & b}
            self.samples.append((time.monotonic(), float(sm), float(mx), names))
            self._stop.wait(0.001)

    def _poll_smi(self):
        for line in self._proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            names = {n for n, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                      parts[5:9]) if v.lower() == "active"}
            self.samples.append((time.monotonic(), sm, mx, names))

    def __enter__(self):
        try:
            pynvml, h = self._nvml_handle()
            self._thread = threading.Thread(target=self._poll_nvml, args=(pynvml, h), daemon=True)
        except Exception as exc:
            print(f"bench.py: NVML clock sampling unavailable ({exc}); using nvidia-smi", file=sys.stderr)
            # nvidia-smi numbers GPUs physically; the torch index is not that
            # number under CUDA_VISIBLE_DEVICES, the PCI bus id always is.
            try:
                target = self._bus_id()
            except Exception:
                target = None if "CUDA_VISIBLE_DEVICES" in os.environ else str(self.device.index)
            self._thread = None
            if target is not None:
                try:
                    self._proc = subprocess.Popen(
                        ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "20",
                         "-i", target], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                    self._thread = threading.Thread(target=self._poll_smi, daemon=True)
                except OSError:
                    self._thread = None
        if self._thread is not None:
            self._thread.start()
        return self

    def begin(self):
        # The sampler must be running before the timed region starts.
        t0 = time.monotonic()
        while not self.samples and self._thread is not None and time.monotonic() - t0 < 3.0:
            time.sleep(0.01)
        self.t_begin = time.monotonic()

    def end(self):
        self.t_end = time.monotonic()

    def __exit__(self, *exc):
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        b = self.t_begin if self.t_begin is not None else self.samples[0][0]
        e = self.t_end if self.t_end is not None else self.samples[-1][0]
        inside = [x for x in self.samples if b <= x[0] <= e]
        if not inside:  # region shorter than the polling period: the sample nearest its middle
            mid = 0.5 * (b + e)
            inside = [min(self.samples, key=lambda x: abs(x[0] - mid))]
        reasons = set().union(*(x[3] for x in inside))
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": inside[-1][2],
                "reasons": sorted(reasons), "samples": len(inside)}


# ------------------------------------------------------ end to end

def pipelined_e2e(dev, compute_stream, host_in, make_set, run, steps):
    """Times ``steps`` end-to-end steps through the public API, pipelined the
    way a caller streaming batches would: two sets of device buffers
    alternate; step k copies its inputs from pinned host memory into set k % 2
    on a copy-in stream, computes on ``compute_stream`` once they are in, and
    copies every output back to pinned host memory on a copy-out stream, so
    that the next step's inputs and the previous step's outputs cross the
    host link while this step computes (in both directions at once). Every
    step moves all its input and output bytes. Returns the device time in ms
    from the first copy-in to the last copy-out.

    ``make_set()`` returns (device inputs in the order of ``host_in``, device
    outputs); ``run(dev_in, dev_out, stream)`` enqueues one step's compute."""
    import torch

    sets = [make_set() for _ in range(2)]
    host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs] for _, outs in sets]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=False)
    in_done = [ev() for _ in range(steps)]
    comp_done = [ev() for _ in range(steps)]
    out_done = [ev() for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    t0.record(s_in)
    for k in range(steps):
        dins, douts = sets[k % 2]
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(comp_done[k - 2])  # set k % 2's inputs were read by step k - 2
            for d, h in zip(dins, host_in):
                d.copy_(h, non_blocking=True)
            in_done[k].record(s_in)
        compute_stream.wait_event(in_done[k])
        if k >= 2:
            compute_stream.wait_event(out_done[k - 2])  # set k % 2's outputs were copied out
        run(dins, douts, compute_stream)
        comp_done[k].record(compute_stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[k])
            for h, d in zip(host_out[k % 2], douts):
                h.copy_(d, non_blocking=True)
            out_done[k].record(s_out)
    s_out.wait_event(out_done[steps - 1])
    t1.record(s_out)
    torch.cuda.synchronize(dev)
    return t0.elapsed_time(t1)


# ------------------------------------------------------------ CPU oracle

# A (batch, head) slice whose forward costs more than this many algorithmic
# FLOPs is sampled by query rows instead of whole (the 131072-token forward:
# ~4.4 TFLOP per slice, hours of fp64 work).
ROW_SAMPLE_ABOVE_FLOPS = 200e9


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info

        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover - threadpoolctl missing
        return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def oracle_sample(w, seconds: float, max_slices: int = 64):
    """Times the fp64 oracle (as it stands) on whole (batch, head) slices of
    the workload until about ``seconds`` have passed. Returns
    (algorithmic FLOPs done, wall seconds, units done, threads, unit name).

    A forward-only workload whose slice is too large for that (more than
    ROW_SAMPLE_ABOVE_FLOPS) is timed on chunks of 64 seeded query rows of
    one slice instead (``attn_fwd_rows``), each row counted at its
    algorithmic cost 4 * (visible keys) * d."""
    import numpy as np

    import oracle
    from exact_io_aware_56_b200 import make_inputs, sample_rows, to_f64

    threads = _blas_threads()
    flops_slice = (w.fwd_flops() + w.bwd_flops()) / (w.B * w.Hq)
    done, elapsed, n = 0.0, 0.0, 0
    if not w.backward and w.fwd_flops() / (w.B * w.Hq) > ROW_SAMPLE_ABOVE_FLOPS:
        host = make_inputs(1, 1, 1, w.N, w.d, w.seed + 7919, w.qk_gain, False)
        ref = {k: to_f64(v) for k, v in host.items()}
        order = sample_rows(w.N, min(w.N, 64 * 4096), w.seed + 7919)
        np.random.default_rng(w.seed).shuffle(order)
        while n < max_slices * 64 and (elapsed < seconds or n == 0):
            rows = np.sort(order[n * 64:(n + 1) * 64])
            t0 = time.perf_counter()
            oracle.attn_fwd_rows(ref["q"], ref["k"], ref["v"], w.causal, w.scale, 0, 0, rows)
            elapsed += time.perf_counter() - t0
            keys = (rows + 1) if w.causal else np.full(len(rows), w.N)
            done += float(4.0 * keys.sum() * w.d)
            n += 1
        return done, elapsed, n, threads, "chunks of 64 query rows of one (batch, head) slice"
    while n < max_slices and (elapsed < seconds or n == 0):
        host = make_inputs(1, 1, 1, w.N, w.d, w.seed + 7919 * (n + 1), w.qk_gain, w.backward)
        ref = {k: to_f64(v) for k, v in host.items()}
        t0 = time.perf_counter()
        oracle.attn_fwd_ref(ref["q"], ref["k"], ref["v"], w.causal, w.scale)
        if w.backward:
            oracle.attn_bwd_ref(ref["q"], ref["k"], ref["v"], ref["dout"], w.causal, w.scale)
        elapsed += time.perf_counter() - t0
        done += flops_slice
        n += 1
    return done, elapsed, n, threads, "whole (batch, head) slices"


def decode_oracle_sample(w, seconds: float, max_batches: int = 64):
    """Times the fp64 decode oracle (as it stands) on whole batches of the
    workload until about ``seconds`` have passed. Returns (algorithmic bytes
    of the batches done, wall seconds, batches, threads)."""
    import oracle
    from exact_io_aware_56_b200 import make_decode_inputs, to_f64

    threads = _blas_threads()
    bytes_batch = w.bytes_moved() / w.B
    done, elapsed, n = 0.0, 0.0, 0
    while n < max_batches and (elapsed < seconds or n == 0):
        host = make_decode_inputs(1, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.seed + 7919 * (n + 1))
        ref = {k: to_f64(v) for k, v in host.items()}
        t0 = time.perf_counter()
        oracle.attn_decode_ref(ref["q"], ref["k"], ref["v"], w.scale, w.causal)
        elapsed += time.perf_counter() - t0
        done += bytes_batch
        n += 1
    return done, elapsed, n, threads


def decode_config(w, world):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
            "causal": w.causal, "global_batch": w.B * world,
            "parallelism": f"replicas{world}" if world > 1 else "single"}


def decode_reference_arm(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    times, threads = [], 1
    for it in range(args.warmup + args.steps):
        _, el, _, threads = decode_oracle_sample(w, 0.0, max_batches=1)
        if it >= args.warmup:
            times.append(el)
    ms = 1e3 * sum(times) / len(times)
    value = w.bytes_moved() / w.B / (ms * 1e-3) / 1e9
    sample = f"one batch of {w.name} (fp64 decode oracle) per step"
    line = {
        "impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(decode_config(w, 1), sample=sample),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def fp8_oracle_sample(w, seconds: float, max_slices: int = 64):
    """Times the fp64 FP8-mode oracle (quantize with the oracle, then attention
    on the dequantized tensors) on whole (batch, head) slices. Returns
    (algorithmic FLOPs done, wall seconds, slices, threads)."""
    import oracle
    from exact_io_aware_56_b200 import make_inputs, to_f64

    threads = _blas_threads()
    flops_slice = w.fwd_flops() / (w.B * w.Hq)
    done, elapsed, n = 0.0, 0.0, 0
    while n < max_slices and (elapsed < seconds or n == 0):
        host = make_inputs(1, 1, 1, w.N, w.d, w.seed + 7919 * (n + 1), w.qk_gain, False)
        ref = {k: to_f64(v) for k, v in host.items()}
        t0 = time.perf_counter()
        q8, sq = oracle.quantize_blocks(ref["q"])
        k8, sk = oracle.quantize_blocks(ref["k"])
        v8, sv = oracle.quantize_blocks(ref["v"], None)
        oracle.attn_fwd_fp8_ref(q8, sq, k8, sk, v8, sv, w.causal, w.scale)
        elapsed += time.perf_counter() - t0
        done += flops_slice
        n += 1
    return done, elapsed, n, threads


def fp8_reference_arm(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    times, threads = [], 1
    for it in range(args.warmup + args.steps):
        _, el, _, threads = fp8_oracle_sample(w, 0.0, max_slices=1)
        if it >= args.warmup:
            times.append(el)
    ms = 1e3 * sum(times) / len(times)
    value = w.fwd_flops() / (w.B * w.Hq) / (ms * 1e-3) / 1e12
    sample = f"one (batch, head) slice of {w.name} (fp64 FP8-mode oracle: quantize + attention) per step"
    line = {
        "impl": "reference", "metric": FP8_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                   "causal": w.causal, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def reference_arm(args):
    from exact_io_aware_56_b200 import DECODE_WORKLOADS, FP8_WORKLOADS, WORKLOADS

    if args.workload in DECODE_WORKLOADS:
        return decode_reference_arm(args, DECODE_WORKLOADS[args.workload])
    if args.workload in FP8_WORKLOADS:
        return fp8_reference_arm(args, FP8_WORKLOADS[args.workload])

    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    times, flops = [], []
    threads, unit = 1, ""
    for it in range(args.warmup + args.steps):
        f, el, _, threads, unit = oracle_sample(w, 0.0, max_slices=1)
        if it >= args.warmup:
            times.append(el)
            flops.append(f)
    ms = 1e3 * sum(times) / len(times)
    value = sum(flops) / (sum(times) or 1e-30) / 1e12
    passes = "fwd+bwd" if w.backward else "fwd"
    sample = f"one of the {unit} of {w.name} ({passes}, fp64 oracle) per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                   "causal": w.causal, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ native arm

def native_arm(args):
    import torch

    from exact_io_aware_56_b200 import WORKLOADS, fa, make_inputs

    w = WORKLOADS[args.workload]
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device; there is no CPU path")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist("nccl")
    fa.lib()

    host = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed + rank, w.qk_gain, w.backward)
    q, k, v = (host[n].to(dev) for n in ("q", "k", "v"))
    dout = host["dout"].to(dev) if w.backward else None
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    o_resid = None
    if w.backward:
        # Training path: the forward also keeps o's rounding residual for D.
        o_resid = torch.empty_like(q)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(fa.fa_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        fa.fa_fwd(q, k, v, o, lse, w.causal, w.scale, stream, o_resid=o_resid)
        if ev is not None:
            ev[1].record(stream)
        if w.backward:
            fa.fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, w.causal, w.scale, ws, stream, o_resid=o_resid)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.fa_check_device_error(stream) != fa.FA_OK:
        raise RuntimeError("device watchdog fired during warm-up")

    # Per-step events: [fwd start, fwd end, bwd pre end, bwd main end, step end].
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for e in evs:  # torch creates the CUDA event on first record; the hook needs real handles
        e[2].record(stream)
        e[3].record(stream)
    # Inputs smaller than twice L2: L2 is flushed (a buffer larger than L2
    # is written) before every timed step, outside its events, and the time
    # is the sum of the steps' own event intervals.
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v) + ((dout,) if w.backward else ()))
    flush = in_bytes < 2 * L2_BYTES
    scratch = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clocks:
        time.sleep(0.05)
        clocks.begin()
        t_start.record(stream)
        for s in range(args.steps):
            if flush:
                scratch.fill_(s & 0xFF)
            if w.backward:
                fa.fa_profile_set_bwd_events(evs[s][2], evs[s][3])
            step(evs[s])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        clocks.end()
    fa.fa_profile_set_bwd_events(None, None)
    barrier(dev)
    if fa.fa_check_device_error(stream) != fa.FA_OK:
        raise RuntimeError("device watchdog fired during the timed steps")
    ms_local = sum(e[0].elapsed_time(e[4]) for e in evs) if flush else t_start.elapsed_time(t_end)
    ms_total = max_over_ranks(ms_local, dev)
    step_flops = w.fwd_flops() + w.bwd_flops()
    value = step_flops * args.steps * world / (ms_total * 1e-3) / 1e12

    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    kernels = {"fwd": {"ms": fwd_ms, "flops": w.fwd_flops(), "launches_per_step": 1}}
    if w.backward:
        kernels["bwd_main"] = {"ms": statistics.mean(e[2].elapsed_time(e[3]) for e in evs),
                               "flops": w.bwd_flops(), "launches_per_step": 1}
        kernels["bwd_pre"] = {"ms": statistics.mean(e[1].elapsed_time(e[2]) for e in evs)}
        kernels["bwd_post"] = {"ms": statistics.mean(e[3].elapsed_time(e[4]) for e in evs)}
    peak, peak_src = peak_value("bf16_tflops")
    for kn in ("fwd", "bwd_main"):
        if kn in kernels:
            kk = kernels[kn]
            kk["tflops"] = kk["flops"] / (kk["ms"] * 1e-3) / 1e12
            kk["frac"] = kk["tflops"] / peak
    dom = max((kn for kn in ("fwd", "bwd_main") if kn in kernels), key=lambda kn: kernels[kn]["ms"])
    roofline = {
        "bound": "tensor", "kernel": dom, "achieved": kernels[dom]["tflops"], "peak": peak, "unit": "TFLOP/s",
        "frac": kernels[dom]["frac"], "traffic": captured_traffic(dom, w.name),
        "traffic_algorithmic": "fwd: q, k, v read, o (+ o_resid), lse written; "
                               "bwd: q, k, v, dO, L, D read, dk, dv written, dQ fp32 accumulator",
        "peak_source": f"{peak_src} bf16 dense (burst)",
        "kernels": {kn: {x: kernels[kn][x] for x in ("ms", "tflops", "frac") if x in kernels[kn]}
                    for kn in kernels},
    }

    # End to end through the public API: pinned host inputs copied in, both
    # passes run, every output copied back, all inside the timed region
    # (pipelined across steps, see pipelined_e2e).
    e2e = None
    if args.e2e_steps > 0:
        names = ["q", "k", "v"] + (["dout"] if w.backward else [])
        hin = [host[n].pin_memory() for n in names]

        def make_set():
            dins = [torch.empty(t.shape, dtype=t.dtype, device=dev) for t in hin]
            douts = [torch.empty_like(o), torch.empty_like(lse)]
            if w.backward:
                douts += [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
            return dins, douts

        def run(dins, douts, st):
            eq, ek, ev_ = dins[0], dins[1], dins[2]
            fa.fa_fwd(eq, ek, ev_, douts[0], douts[1], w.causal, w.scale, st, o_resid=o_resid)
            if w.backward:
                fa.fa_bwd(eq, ek, ev_, douts[0], dins[3], douts[1], douts[2], douts[3], douts[4], w.causal,
                          w.scale, ws, st, o_resid=o_resid)

        h2d = sum(t.numel() * t.element_size() for t in hin)
        d2h = sum(t.numel() * t.element_size() for t in [o, lse] + ([q, k, v] if w.backward else []))
        pipelined_e2e(dev, stream, hin, make_set, run, 2)  # warm-up of the streams and buffers
        barrier(dev)
        e2e_ms = max_over_ranks(pipelined_e2e(dev, stream, hin, make_set, run, args.e2e_steps), dev)
        e2e = {"value": step_flops * args.e2e_steps * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipelined": "inputs of step k+1 and outputs of step k-1 cross the host link while step k computes"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        flops, secs, n, threads, unit = oracle_sample(w, args.cpu_seconds)
        passes = "fwd+bwd" if w.backward else "fwd"
        cpu = {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} {unit} of {w.name}, {passes}, fp64 oracle, {secs:.1f} s"}

    l2_note = (f"inputs {in_bytes / 2**20:.0f} MiB per rank, L2 flushed before every step "
               f"({FLUSH_BYTES >> 20} MiB write, outside the step's events)" if flush else
               f"inputs larger than L2 ({in_bytes / 2**20:.0f} MiB per rank), no flush")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                   "causal": w.causal, "qk_gain": w.qk_gain, "global_batch": w.B * world,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": l2_note},
        "fraction_of_peak": value / world / peak,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * (4 if w.backward else 1),
        "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


def fp8_native_arm(args, w):
    """One step = one fa_fwd_fp8 call on e4m3 codes and scales resident in
    HBM (quantized once by fa_quantize_fp8 before the timed region)."""
    import torch

    from exact_io_aware_56_b200 import fa, make_inputs

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device; there is no CPU path")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist("nccl")
    fa.lib()
    host = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed + rank, w.qk_gain, False)
    q, k, v = (host[n].to(dev) for n in ("q", "k", "v"))
    stream = torch.cuda.current_stream(dev)
    q8, sq = fa.quantize_fp8(q, False, stream)
    k8, sk = fa.quantize_fp8(k, False, stream)
    v8, sv = fa.quantize_fp8(v, True, stream)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)

    def step():
        fa.fa_fwd_fp8(q8, sq, k8, sk, v8, sv, o, lse, w.causal, w.scale, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.fa_check_device_error(stream) != fa.FA_OK:
        raise RuntimeError("device watchdog fired during warm-up")
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clocks:
        time.sleep(0.05)
        clocks.begin()
        t_start.record(stream)
        for _ in range(args.steps):
            step()
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        clocks.end()
    barrier(dev)
    if fa.fa_check_device_error(stream) != fa.FA_OK:
        raise RuntimeError("device watchdog fired during the timed steps")
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), dev)
    value = w.fwd_flops() * args.steps * world / (ms_total * 1e-3) / 1e12
    peak, peak_src = peak_value("bf16_tflops")
    peak *= 2.0
    achieved = w.fwd_flops() / (ms_total / args.steps * 1e-3) / 1e12
    roofline = {
        "bound": "tensor", "kernel": "fwd_fp8", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
        "frac": achieved / peak, "traffic": captured_traffic("fwd_fp8", w.name),
        "peak_source": f"{peak_src} bf16 dense (burst) x 2, the nominal FP8 : bf16 ratio",
    }
    e2e = None
    if args.e2e_steps > 0:
        # bf16 q, k, v in from pinned host memory, quantized and attended on
        # the device, o and lse back, pipelined as the training step's e2e
        # (see pipelined_e2e). The codes and scales are one set: quantization
        # and attention of consecutive steps run in order on one stream.
        hin = [host[n].pin_memory() for n in ("q", "k", "v")]

        def make_set():
            return [torch.empty(t.shape, dtype=t.dtype, device=dev) for t in hin], [torch.empty_like(o),
                                                                                    torch.empty_like(lse)]

        def run(dins, douts, st):
            fa.fa_quantize_fp8(dins[0], q8, sq, False, st)
            fa.fa_quantize_fp8(dins[1], k8, sk, False, st)
            fa.fa_quantize_fp8(dins[2], v8, sv, True, st)
            fa.fa_fwd_fp8(q8, sq, k8, sk, v8, sv, douts[0], douts[1], w.causal, w.scale, st)

        h2d = sum(t.numel() * t.element_size() for t in hin)
        d2h = sum(t.numel() * t.element_size() for t in (o, lse))
        pipelined_e2e(dev, stream, hin, make_set, run, 2)  # warm-up of the streams and buffers
        barrier(dev)
        e2e_ms = max_over_ranks(pipelined_e2e(dev, stream, hin, make_set, run, args.e2e_steps), dev)
        e2e = {"value": w.fwd_flops() * args.e2e_steps * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipelined": "inputs of step k+1 and outputs of step k-1 cross the host link while step k computes"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        flops, secs, n, threads = fp8_oracle_sample(w, args.cpu_seconds)
        cpu = {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} whole (batch, head) slices of {w.name}, fp64 FP8-mode oracle, {secs:.1f} s"}
    in_bytes = sum(t.numel() for t in (q8, k8, v8))
    line = {
        "metric": FP8_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                   "causal": w.causal, "qk_gain": w.qk_gain, "global_batch": w.B * world,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": f"e4m3 inputs {in_bytes / 2**20:.0f} MiB per rank, compute-bound, no flush"},
        "fraction_of_peak": value / world / peak,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


def decode_native_arm(args, w):
    """One step = one fa_decode call on the resident cache; the decode
    kernel's own time (split kernel, through the decode timing hook) gives
    the roofline, the whole call (split + merge) the value."""
    import torch

    from exact_io_aware_56_b200 import fa, make_decode_inputs

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device; there is no CPU path")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist("nccl")
    fa.lib()
    host = make_decode_inputs(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.seed + rank)
    q, k, v = (host[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.fa_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.fa_decode(q, k, v, o, lse, w.causal, w.scale, ws, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.fa_check_device_error(stream) != fa.FA_OK:
        raise RuntimeError("device watchdog fired during warm-up")
    # Per-step events: [start, after the split kernel, end].
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for e in evs:  # torch creates the CUDA event on first record; the hook needs real handles
        e[1].record(stream)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clocks:
        time.sleep(0.05)
        clocks.begin()
        t_start.record(stream)
        for s in range(args.steps):
            evs[s][0].record(stream)
            fa.fa_profile_set_decode_event(evs[s][1])
            step()
            evs[s][2].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        clocks.end()
    fa.fa_profile_set_decode_event(None)
    barrier(dev)
    if fa.fa_check_device_error(stream) != fa.FA_OK:
        raise RuntimeError("device watchdog fired during the timed steps")
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), dev)
    value = w.bytes_moved() * args.steps * world / (ms_total * 1e-3) / 1e9
    peak, peak_src = peak_value("hbm_gbs")
    main_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    merge_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    # The split kernel's algorithmic bytes: it reads q and the K/V cache
    # (its partial results are working storage, not algorithmic traffic).
    kv_q = 2 * w.B * w.Hkv * w.Nk * w.d * 2 + w.B * w.Hq * w.Nq * w.d * 2
    achieved = kv_q / (main_ms * 1e-3) / 1e9
    roofline = {
        "bound": "hbm", "kernel": "decode_kernel", "achieved": achieved, "peak": peak, "unit": "GB/s",
        "frac": achieved / peak, "traffic": captured_traffic("decode_kernel", w.name),
        "peak_source": f"{peak_src} copy bandwidth",
        "algorithmic_bytes_per_launch": kv_q,
        "kernels": {"decode_kernel": {"ms": main_ms}, "decode_merge": {"ms": merge_ms}},
    }
    e2e = None
    if args.e2e_steps > 0:
        hin = {n: host[n].pin_memory() for n in host}
        hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (o, lse)]
        h2d = sum(t.numel() * t.element_size() for t in hin.values())
        d2h = sum(t.numel() * t.element_size() for t in (o, lse))
        dins = {"q": q, "k": k, "v": v}

        def e2e_step():
            for n, t in dins.items():
                t.copy_(hin[n], non_blocking=True)
            step()
            for src, dst in zip((o, lse), hout):
                dst.copy_(src, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        barrier(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(a.elapsed_time(b), dev)
        e2e = {"value": w.bytes_moved() * args.e2e_steps * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        done, secs, n, threads = decode_oracle_sample(w, args.cpu_seconds)
        cpu = {"value": done / secs / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} whole batches of {w.name}, fp64 decode oracle, {secs:.1f} s"}
    line = {
        "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(decode_config(w, world),
                       l2=f"K/V cache larger than L2 ({kv_q / 2**20:.0f} MiB per rank), no flush"),
        "fraction_of_peak": value / world / peak,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * 2,
        "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return reference_arm(args)
    from exact_io_aware_56_b200 import DECODE_WORKLOADS, FP8_WORKLOADS

    if args.workload in DECODE_WORKLOADS:
        return decode_native_arm(args, DECODE_WORKLOADS[args.workload])
    if args.workload in FP8_WORKLOADS:
        return fp8_native_arm(args, FP8_WORKLOADS[args.workload])
    return native_arm(args)


if __name__ == "__main__":
    sys.exit(main())
