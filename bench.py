#!/usr/bin/env python3
"""Throughput benchmark of the B200 per-token dynamic quantization path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--graph]

One step = one call of the hot path over one batch of the workload (default:
symmetric INT8 with fp32 smooth scales, bf16 x [8192, 4096], the size the
headline metric is quoted on). The metric is GB/s of algorithmic HBM traffic
(x read + codes and scales written + side tables read), with rows/s and the
fraction of the measured HBM copy bandwidth alongside.

Timing: one untimed step on each buffer set, W untimed warm-up steps, then
exactly K steps between a barrier + device synchronize on both sides, timed
with CUDA events on the launching stream; the max over ranks is reported.
Consecutive steps rotate over several input/output buffer sets whose total is
at least 12 x the 126 MB L2, so no step reads data an earlier one left in L2
(with 3 x the L2, some lines survived a rotation: 8192 x 4096 bf16 ran 0.5 us
per call faster and read 6 % less from DRAM than it moves); tiny workloads
stop at 1024 sets, still above the L2. SM clocks and throttle reasons are
sampled through NVML during the timed region.

Multi-GPU (torchrun, one process per GPU): rows are independent, so each rank
quantizes its own full batch with no collective on the data path (weak
scaling); only the timing uses a MAX all-reduce.

--impl reference times the CPU oracle (the plain sequential implementation of
the same formulas) on the same metric, on the host cores of rank 0.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "sym_int8_smooth_bf16_8192x4096"
METRIC = "DynamicQuant GB/s and % of B200 HBM roofline (rows/s at 8192x4096 bf16)"
L2_BYTES = 126 * 1024 * 1024
L2_ROTATION = 12  # the rotating buffer sets hold at least this many L2 capacities
MAX_SETS = 1024  # (at most this many sets: tiny workloads stop at a few L2 capacities)
FALLBACK_HBM_GBS = 6650.0
PRE_ROLL_CYCLES = 2_000_000  # device sleep queued ahead of the timed launches (~1 ms at 1.9 GHz)
PRE_ROLL_CYCLES_PER_STEP = 20_000  # and ~10 us more per timed step, so the host stays ahead of the device


# ---------------------------------------------------------------- helpers

METRIC_W8A8 = "W8A8 product TFLOP/s (int8 tensor ops, per-token x per-channel scales) and % of the tensor roofline"


def work(wl):
    """(units per step, divisor to the reported unit, unit, metric): HBM bytes for
    the bandwidth-bound operations, tensor ops (2 M N K) for the W8A8 product."""
    if wl.kind == "w8a8_gemm":
        m, k = (int(v) for v in wl.tensors["a"].shape)
        n = int(wl.tensors["b"].shape[0])
        return 2 * m * n * k, 1e12, "TFLOP/s", METRIC_W8A8
    return algorithmic_bytes(wl), 1e9, "GB/s", METRIC


def algorithmic_bytes(wl) -> int:
    """HBM bytes one call must move: x read, codes + per-row floats written, side tables read."""
    t = wl.tensors
    rows, cols = wl.rows, wl.cols
    if wl.kind == "w8a8_gemm":
        return int(sum(v.numel() * v.element_size() for v in t.values()) + rows * int(t["b"].shape[0]) * 2)
    if wl.kind.startswith("dequant"):
        # codes + scale (and offset) tables read, [rows, cols] outputs written
        total = sum(v.numel() * v.element_size() for v in t.values() if v is not None)
        return int(total + rows * cols * {"f32": 4, "f16": 2, "bf16": 2}[wl.out_dtype])
    x = t["x"]
    total = x.numel() * x.element_size()
    if wl.kind == "dynamic_quant":
        code_bytes = rows * cols if wl.y_dtype == "int8" else rows * cols // 2
        per_row = 4 * (2 if wl.mode == "asymmetric" else 1)
        total += code_bytes + rows * per_row
        for k in ("smooth", "group_index"):
            if t.get(k) is not None:
                total += t[k].numel() * t[k].element_size()
    else:
        total += rows * cols + rows * 4
        for k in ("ada_scale", "ada_shift", "weight", "bias", "smooth"):
            if t.get(k) is not None:
                total += t[k].numel() * t[k].element_size()
    return int(total)


def workload_config(wl) -> dict:
    """The config keys that describe a workload's operation and types."""
    if wl.kind == "w8a8_gemm":
        return {"operation": "w8a8_gemm", "m": int(wl.tensors["a"].shape[0]), "n": int(wl.tensors["b"].shape[0]),
                "k": int(wl.tensors["a"].shape[1]), "out_dtype": wl.out_dtype, "scales": "per-token x per-channel"}
    if wl.kind.startswith("dequant"):
        c = {"operation": wl.kind, "rows": wl.rows, "cols": wl.cols, "y_dtype": wl.y_dtype,
             "scale_dtype": str(wl.tensors["scale"].dtype).replace("torch.", ""), "out_dtype": wl.out_dtype,
             "offset": wl.tensors.get("offset") is not None}
        if wl.kind == "dequant_per_group":
            c.update(group_size=wl.group_size, k_dim=wl.k_dim)
        return c
    return {"operation": wl.kind, "x_dtype": "bf16" if "bf16" in wl.name else "f16", "rows": wl.rows,
            "cols": wl.cols, "mode": wl.mode if wl.kind == "dynamic_quant" else "symmetric", "y_dtype": wl.y_dtype}


SMS = 148


def ada_table_staged(wl) -> bool:
    """Whether the library's AdaLayerNormQuant launch takes the ring kernel
    that folds the affine table rows of its CTA's batches in shared memory
    (hidden a multiple of 8, and those rows within 64 KB): one launch per
    call. Otherwise the affine-table kernel runs first: two launches."""
    b, s, h = wl.primary.shape
    rows = b * s
    if h % 8 or rows == 0:
        return False
    grid = min(rows, SMS)
    per_cta = -(-rows // grid)
    nb = min((per_cta - 1) // s + 2, b)
    return nb * h * 8 <= 64 * 1024


def launches_per_call(wl) -> int:
    """Kernels one C-ABI call launches: DynamicQuant, the dequantizers and the
    W8A8 product one; AdaLayerNormQuant one when its ring kernel folds the
    affine table itself, else two (the affine table, then the row kernel)."""
    if wl.kind == "ada_layernorm_quant":
        return 1 if ada_table_staged(wl) else 2
    return 1


def timed_kernel(wl) -> str:
    """The kernel the timed region runs (the roofline's subject)."""
    if wl.kind == "dynamic_quant":
        # few short rows (one warp each, at most 2 per SM) take the warp kernel
        nvec = wl.cols // 8
        one_warp = wl.cols % 8 == 0 and any(nvec == 32 * v for v in (2, 4, 6, 7, 8))
        return "dynamic_quant_warp_kernel" if one_warp and wl.rows <= 2 * SMS else "dynamic_quant_ring_kernel"
    if wl.kind == "ada_layernorm_quant":
        return ("ada_layernorm_quant_ring_kernel (one launch per call: the affine table folded in the kernel)"
                if ada_table_staged(wl) else
                "ada_layernorm_quant_ring_kernel (time of the whole call: affine-table kernel included)")
    if wl.kind == "w8a8_gemm":
        return "w8a8_gemm_persistent_kernel"
    return {"dequant_per_token": "dequant_vec_kernel (per-token layout)",
            "dequant_per_group": "dequant_vec_kernel (per-group layout)"}[wl.kind]


def measured_peaks(tensor: bool = False):
    """(peak, kind): the measured HBM copy bandwidth (GB/s), or for the int8
    tensor product the measured bf16 burst GEMM rate x 2 (the nominal int8 :
    bf16 ratio, 4.5 : 2.25 PFLOP/s dense)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        if tensor:
            return 2.0 * float(d["bf16_tflops"]), "measured"
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return (2.0 * 1590.0 if tensor else FALLBACK_HBM_GBS), "fallback"


# The sources each operation's kernels are built from (a profile's traffic
# figure stays valid while these are unchanged).
KERNEL_SOURCES = {
    "dynamic_quant": ("dynamic_quant_kernels.cuh", "dynamic_quant_ring.cuh", "dq_device.cuh", "tma_pipeline.cuh",
                      "ring_prefetch.cuh", "dq_args.cuh", "quant_launch.cuh", "dq_launch.cuh"),
    "ada_layernorm_quant": ("ada_layernorm_quant_kernels.cuh", "ada_layernorm_quant_ring.cuh", "dq_device.cuh",
                            "tma_pipeline.cuh", "ring_prefetch.cuh", "dq_args.cuh", "ada_launch.cu", "dq_launch.cuh"),
    "dequant_per_token": ("dequant_kernels.cuh", "dq_device.cuh", "dq_args.cuh", "dequant_launch.cu", "dq_launch.cuh"),
    "dequant_per_group": ("dequant_kernels.cuh", "dq_device.cuh", "dq_args.cuh", "dequant_launch.cu", "dq_launch.cuh"),
    "w8a8_gemm": ("w8a8_gemm.cu", "tma_pipeline.cuh"),
}


def source_hash(kind: str) -> str:
    """Hash of the code in those sources: comments and blank lines are left
    out, so a comment edit does not void a capture."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "token_dynamic_quantization_b200", "csrc")
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
        h.update(name.encode())
        h.update(code.encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kind: str):
    """dram read+write bytes per launch from the committed ncu summary, if it
    was taken on the current sources of the workload's kernels (else None)."""
    path = os.path.join(ROOT, "profiles", f"ncu_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"source_hash:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != source_hash(kind):
        return None
    return int(m_bytes.group(1))


class ClockSampler:
    """NVML sampling of SM clock, power and throttle reasons in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples = []  # (t, sm_mhz, max_mhz, reasons_mask)
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                try:
                    mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    mask = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.samples.append((time.perf_counter(), sm, mask))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._thread.start()

    def stop(self):
        self._stop.set()
        if self.ok:
            self._thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "NVML unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed"
        if len(inside) < 3:
            inside = [s for s in self.samples if s[0] <= t1]
            inside = inside[-max(3, len(inside) // 4):] if inside else []
            window = "timed+warmup (timed region shorter than the sampling period)"
        reasons = set()
        for _, _, mask in inside:
            for bit, name in self.REASONS.items():
                if mask & bit and name != "gpu_idle":
                    reasons.add(name)
        sm = [s[1] for s in inside]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(inside), "window": window}


# ---------------------------------------------------------------- distributed plumbing

def relaunch_under_torchrun(argv, n_gpus: int) -> int:
    """`--gpus N` (N > 1) started as a plain process: run this same command
    under torch.distributed.run with N local ranks (one per GPU) and return
    its exit status."""
    import socket
    import subprocess

    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    # the ranks' process group ends a stuck collective after 120 s; as the last
    # bound, well above it, the whole run is stopped after an hour
    cmd = ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n_gpus}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != n_gpus:
        raise SystemExit(f"bench.py: --gpus {n_gpus} but WORLD_SIZE={world}; start one rank per requested GPU")
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- the CUDA arm

class Launcher:
    """Pointer-level calls of the C ABI over a ring of buffer sets on one stream."""

    def __init__(self, dq, wl, device, sets: int):
        import torch

        self.dq, self.wl = dq, wl
        t = wl.tensors
        self.stream = torch.cuda.Stream(device)
        self.sptr = self.stream.cuda_stream
        self.sets = []
        xs = wl.primary.to(device)
        for i in range(sets):
            x = xs if i == 0 else xs.clone()
            if wl.kind == "w8a8_gemm":
                out = torch.empty((wl.rows, int(t["b"].shape[0])), dtype=torch.bfloat16, device=device)
                self.sets.append(dict(x=x, out=out))
            elif wl.kind.startswith("dequant"):
                out = torch.empty((wl.rows, wl.cols), dtype={"f32": torch.float32, "f16": torch.float16,
                                                              "bf16": torch.bfloat16}[wl.out_dtype], device=device)
                self.sets.append(dict(x=x, out=out))
            elif wl.kind == "dynamic_quant":
                cols = wl.cols
                ycols = cols if wl.y_dtype == "int8" else (cols // 2 if wl.y_dtype == "int4" else cols // 8)
                ydt = {"int8": torch.int8, "int4": torch.uint8, "int32": torch.int32}[wl.y_dtype]
                y = torch.empty((wl.rows, ycols), dtype=ydt, device=device)
                scale = torch.empty(wl.rows, dtype=torch.float32, device=device)
                offset = torch.empty(wl.rows, dtype=torch.float32, device=device) if wl.mode == "asymmetric" else None
                self.sets.append(dict(x=x, y=y, scale=scale, offset=offset))
            else:
                out = torch.empty(tuple(t["x"].shape), dtype=torch.int8, device=device)
                qs = torch.empty(tuple(t["x"].shape[:2]), dtype=torch.float32, device=device)
                self.sets.append(dict(x=x, out=out, qs=qs))
        self.side = {k: (v.to(device) if v is not None else None) for k, v in t.items() if k not in ("x", "y", "a")}
        if wl.kind.startswith("dequant") or wl.kind == "w8a8_gemm":
            self.ws_bytes, self.ws = 0, None
        elif wl.kind == "dynamic_quant":
            gi = self.side.get("group_index")
            self.ngroups = int(gi.numel()) if gi is not None else 0
            x_dt = dq.DQ_BF16 if t["x"].dtype == torch.bfloat16 else dq.DQ_F16
            self.ws_bytes = dq.dq_get_workspace_size(wl.rows, wl.cols, x_dt,
                                                     dq.DQ_ASYMMETRIC if wl.mode == "asymmetric" else dq.DQ_SYMMETRIC,
                                                     {"int8": dq.DQ_INT8, "int4": dq.DQ_INT4X2,
                                                      "int32": dq.DQ_INT32}[wl.y_dtype], self.ngroups)
            self.ws = torch.zeros(max(1, self.ws_bytes // 4), dtype=torch.int32, device=device)
        else:
            x = t["x"]
            self.ws_bytes = dq.dq_ada_layernorm_quant_get_workspace_size(
                int(x.shape[0]), int(x.shape[1]), int(x.shape[2]),
                dq.DQ_BF16 if x.dtype == torch.bfloat16 else dq.DQ_F16,
                {torch.float32: dq.DQ_F32, torch.float16: dq.DQ_F16, torch.bfloat16: dq.DQ_BF16}[t["ada_scale"].dtype])
            self.ws = torch.zeros(max(4, (self.ws_bytes + 15) // 16 * 4), dtype=torch.float32, device=device)
        self._prepare_args()

    def _prepare_args(self):
        import torch

        dq, wl = self.dq, self.wl
        p = lambda t: None if t is None else t.data_ptr()
        code = {torch.float32: dq.DQ_F32, torch.float16: dq.DQ_F16, torch.bfloat16: dq.DQ_BF16}
        self.calls = []
        ycode = {"int8": dq.DQ_INT8, "int4": dq.DQ_INT4X2, "int32": dq.DQ_INT32}
        for s in self.sets:
            if wl.kind == "w8a8_gemm":
                d = self.side
                args = (p(s["x"]), p(d["b"]), wl.rows, int(d["b"].shape[0]), int(s["x"].shape[1]), p(d["a_scale"]),
                        p(d["b_scale"]), p(s["out"]), code[s["out"].dtype], 0, self.sptr)
                self.calls.append((dq.dq_w8a8_gemm, args))
            elif wl.kind == "dequant_per_token":
                sc, off = self.side["scale"], self.side.get("offset")
                args = (p(s["x"]), ycode[wl.y_dtype], wl.rows, wl.cols, p(sc), p(off), code[sc.dtype],
                        p(s["out"]), code[s["out"].dtype], self.sptr)
                self.calls.append((dq.dq_dequant_per_token, args))
            elif wl.kind == "dequant_per_group":
                sc, off = self.side["scale"], self.side.get("offset")
                args = (p(s["x"]), ycode[wl.y_dtype], wl.rows, wl.cols, p(sc), p(off), code[sc.dtype], wl.group_size,
                        wl.k_dim, p(s["out"]), code[s["out"].dtype], self.sptr)
                self.calls.append((dq.dq_dequant_per_group, args))
            elif wl.kind == "dynamic_quant":
                sm = self.side.get("smooth")
                gi = self.side.get("group_index")
                args = (p(s["x"]), code[s["x"].dtype], wl.rows, wl.cols, p(sm), code[sm.dtype] if sm is not None
                        else dq.DQ_F32, p(gi), self.ngroups,
                        dq.DQ_ASYMMETRIC if wl.mode == "asymmetric" else dq.DQ_SYMMETRIC,
                        {"int8": dq.DQ_INT8, "int4": dq.DQ_INT4X2, "int32": dq.DQ_INT32}[wl.y_dtype],
                        p(s["y"]), p(s["scale"]), p(s["offset"]), p(self.ws) if self.ws_bytes else None,
                        self.ws_bytes, self.sptr)
                self.calls.append((dq.dq_dynamic_quant, args))
            else:
                d = self.side
                b, sq, h = (int(v) for v in s["x"].shape)
                args = (p(s["x"]), code[s["x"].dtype], b, sq, h, p(d["ada_scale"]), p(d["ada_shift"]),
                        p(d.get("weight")), p(d.get("bias")), p(d.get("smooth")), code[d["ada_scale"].dtype],
                        float(wl.epsilon), p(s["out"]), p(s["qs"]), p(self.ws), self.ws_bytes, self.sptr)
                self.calls.append((dq.dq_ada_layernorm_quant, args))

    def step(self, i: int):
        fn, args = self.calls[i % len(self.calls)]
        st = fn(*args)
        if st != 0:
            raise RuntimeError(f"launch failed: {self.dq.dq_status_string(st)}")


def rotation_sets(per_set: int) -> int:
    """Buffer sets the timed steps rotate over: at least L2_ROTATION L2
    capacities in all (two sets at least, MAX_SETS at most)."""
    return min(MAX_SETS, max(2, math.ceil(L2_ROTATION * L2_BYTES / per_set)))


def run_ours(args, world, rank, local):
    import torch

    from token_dynamic_quantization_b200 import dq
    from token_dynamic_quantization_b200 import workloads

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = workloads.make(args.workload, rows=args.rows)
    nbytes = algorithmic_bytes(wl)
    per_set = wl.primary.numel() * wl.primary.element_size() + nbytes
    sets = rotation_sets(per_set)
    L = Launcher(dq, wl, device, sets)
    torch.cuda.synchronize(device)

    sampler = ClockSampler(local)
    sampler.start()
    graph = None
    with torch.cuda.stream(L.stream):
        # every buffer set once, then the W warm-up steps: the first launch on
        # a set is slower (per-token dequantization over 12 sets: 18.6 us per
        # call in a 20-step window after 5 warm-up steps, 17.9 after 24)
        for i in range(sets):
            L.step(i)
        for i in range(args.warmup):
            L.step(i)
        if args.graph:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=L.stream):
                for i in range(args.steps):
                    L.step(i)
    torch.cuda.synchronize(device)
    barrier(world)
    torch.cuda.synchronize(device)

    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    with torch.cuda.stream(L.stream):
        # the device sleeps ~1 ms (+ ~10 us per step) before the start event,
        # while the host queues the K launches: the host's launch latency stays
        # outside the timed region, which holds exactly the K steps (a 2 us
        # call would otherwise wait on the host's ~4 us per launch)
        torch.cuda._sleep(PRE_ROLL_CYCLES + PRE_ROLL_CYCLES_PER_STEP * args.steps)
        start.record(L.stream)
        if graph is not None:
            graph.replay()  # replays on the current stream, i.e. L.stream
        else:
            for i in range(args.steps):
                L.step(i)
        end.record(L.stream)
    torch.cuda.synchronize(device)
    t1 = time.perf_counter()
    barrier(world)
    sampler.stop()
    ms_local = start.elapsed_time(end)
    ms = max_over_ranks(ms_local, world, device)
    clocks = sampler.summary(t0, t1)
    if graph is not None:
        del graph

    ms_per_step = ms / args.steps
    units, divisor, unit, metric = work(wl)
    value = units * world / (ms_per_step * 1e-3) / divisor  # every rank did `units` per step (max over ranks)
    rows_per_s = wl.rows * world / (ms_per_step * 1e-3)

    # end to end through the public API with host buffers: H2D of the step's
    # inputs, the call, D2H of its outputs, all inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(dq, wl, device, nbytes, world, min(args.steps, 20))

    tensor = wl.kind == "w8a8_gemm"
    peak, peak_kind = measured_peaks(tensor)
    achieved = units / (ms_local / args.steps * 1e-3) / divisor
    result = None
    if rank == 0:
        traffic = profiled_traffic(args.workload, wl.kind)
        result = {
            "metric": metric,
            "value": round(value, 2),
            "unit": unit,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 6),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "s8 x s8 -> s32, f32 scales" if tensor else "f32",
            "data": "synthetic",
            "config": {
                "workload": args.workload,
                **workload_config(wl),
                "algorithmic_bytes_per_step": nbytes,
                "rows_per_s": round(rows_per_s, 1),
                "parallelism": f"dp{world} (independent row batches, no collective)",
                "l2": f"inputs larger than L2: {sets} rotating buffer sets, {sets * per_set / 1e6:.0f} MB "
                      f"> 126 MB (target {L2_ROTATION} x)",
                "priming": f"{sets} untimed steps, one per buffer set, before the W warm-up steps",
                "launch": "cuda graph of K launches" if args.graph else
                          "eager C-ABI launches, queued behind a ~1 ms device sleep (host launch latency untimed)",
            },
            "roofline": {
                "bound": "tensor" if tensor else "hbm",
                "achieved": round(achieved, 2),
                "peak": peak,
                "unit": unit,
                "frac": round(achieved / peak, 4),
                "peak_kind": ("measured bf16 burst GEMM (MEASURED_PEAKS.json bf16_tflops) x 2, the nominal int8 ratio"
                              if tensor else "measured (MEASURED_PEAKS.json hbm_gbs, copy kernel)")
                if peak_kind == "measured" else "fallback",
                "traffic": traffic,
                "kernel": timed_kernel(wl),
            },
            "clocks": clocks,
            "gpu_launches": args.steps * launches_per_call(wl),
        }
        if e2e is not None:
            result["e2e"] = e2e
        if not args.no_cpu_baseline and world == 1:
            result["cpu_baseline"] = cpu_baseline(wl, nbytes, target_s=args.cpu_seconds)
    return result


def run_e2e(dq, wl, device, nbytes, world, steps):
    """End to end through the public API with host buffers.

    Every step copies its inputs from pinned host memory to the device, calls
    the library, and copies the step's results (codes, scales, offsets) back
    to pinned host memory. Steps are pipelined over three buffer sets on three
    streams (host->device copies, the call, device->host copies), so one
    step's copies overlap its neighbours' work, as a serving loop would run
    them. The time is from before the first upload to after the last download.
    """
    import torch

    t = wl.tensors
    host_in = {k: (v.pin_memory() if v is not None else None) for k, v in t.items()}
    nsets = 3
    s_in, s_call, s_out = (torch.cuda.Stream(device) for _ in range(3))
    sets = []
    for _ in range(nsets):
        d_in = {k: (v.to(device) if v is not None else None) for k, v in host_in.items()}  # outputs sized by a real call
        odt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[wl.out_dtype]
        if wl.kind == "w8a8_gemm":
            o = dq.w8a8_gemm(d_in["a"], d_in["b"], d_in["a_scale"], d_in["b_scale"], out_dtype=odt,
                             stream=s_call.cuda_stream)
            outs = (o,)
        elif wl.kind == "dequant_per_token":
            o = dq.dequant_per_token(d_in["y"], d_in["scale"], d_in.get("offset"), y_dtype=wl.y_dtype, cols=wl.cols,
                                     out_dtype=odt, stream=s_call.cuda_stream)
            outs = (o,)
        elif wl.kind == "dequant_per_group":
            o = dq.dequant_per_group(d_in["y"], d_in["scale"], d_in.get("offset"), group_size=wl.group_size,
                                     k_dim=wl.k_dim, y_dtype=wl.y_dtype, cols=wl.cols, out_dtype=odt,
                                     stream=s_call.cuda_stream)
            outs = (o,)
        elif wl.kind == "dynamic_quant":
            y, sc, off, ws = dq.dynamic_quant(d_in["x"], d_in.get("smooth"), d_in.get("group_index"), mode=wl.mode,
                                              y_dtype=wl.y_dtype, check=False, stream=s_call.cuda_stream)
            outs = (y, sc, off, ws)
        else:
            y, sc = dq.ada_layernorm_quant(d_in["x"], d_in["ada_scale"], d_in["ada_shift"], d_in.get("weight"),
                                           d_in.get("bias"), d_in.get("smooth"), epsilon=wl.epsilon,
                                           stream=s_call.cuda_stream, check=False)
            ws_bytes = dq.dq_ada_layernorm_quant_get_workspace_size(*d_in["x"].shape, dq._dtype_code(d_in["x"]),
                                                                     dq._dtype_code(d_in["ada_scale"]))
            ws = torch.empty((ws_bytes + 15) // 16 * 4, dtype=torch.float32, device=device) if ws_bytes else None
            outs = (y, sc, ws)
        keep = {"dynamic_quant": 3, "ada_layernorm_quant": 2, "dequant_per_token": 1, "dequant_per_group": 1,
                "w8a8_gemm": 1}[wl.kind]
        results = [o for o in outs[:keep] if o is not None]
        h_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in results]
        ev = {n: torch.cuda.Event() for n in ("in", "call", "out")}
        sets.append({"in": d_in, "outs": outs, "results": results, "h_out": h_out, "ev": ev, "used": False})
    torch.cuda.synchronize(device)

    def step(i):
        st = sets[i % nsets]
        ev = st["ev"]
        if st["used"]:
            s_in.wait_event(ev["call"])    # the call that last read this set's inputs is done
            s_call.wait_event(ev["out"])   # this set's last results are on the host
        with torch.cuda.stream(s_in):
            for k, v in host_in.items():
                if v is not None:
                    st["in"][k].copy_(v, non_blocking=True)
            ev["in"].record(s_in)
        s_call.wait_event(ev["in"])
        d = st["in"]
        if wl.kind == "w8a8_gemm":
            dq.w8a8_gemm(d["a"], d["b"], d["a_scale"], d["b_scale"], out=st["outs"][0], stream=s_call.cuda_stream)
        elif wl.kind == "dequant_per_token":
            dq.dequant_per_token(d["y"], d["scale"], d.get("offset"), y_dtype=wl.y_dtype, cols=wl.cols,
                                 out=st["outs"][0], stream=s_call.cuda_stream)
        elif wl.kind == "dequant_per_group":
            dq.dequant_per_group(d["y"], d["scale"], d.get("offset"), group_size=wl.group_size, k_dim=wl.k_dim,
                                 y_dtype=wl.y_dtype, cols=wl.cols, out=st["outs"][0], stream=s_call.cuda_stream)
        elif wl.kind == "dynamic_quant":
            dq.dynamic_quant(d["x"], d.get("smooth"), d.get("group_index"), mode=wl.mode, y_dtype=wl.y_dtype,
                             out=st["outs"], stream=s_call.cuda_stream)
        else:
            y, sc, ws = st["outs"]
            dq.ada_layernorm_quant(d["x"], d["ada_scale"], d["ada_shift"], d.get("weight"), d.get("bias"),
                                   d.get("smooth"), epsilon=wl.epsilon, out=(y, sc), workspace=ws,
                                   stream=s_call.cuda_stream)
        ev["call"].record(s_call)
        s_out.wait_event(ev["call"])
        with torch.cuda.stream(s_out):
            for h, o in zip(st["h_out"], st["results"]):
                h.copy_(o, non_blocking=True)
            ev["out"].record(s_out)
        st["used"] = True

    for i in range(2 * nsets):
        step(i)
    torch.cuda.synchronize(device)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    s_call.wait_event(start)  # the timed pipeline starts behind the start event
    s_out.wait_event(start)
    for i in range(steps):
        step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_call)
    end.record(s_out)
    torch.cuda.synchronize(device)
    ms = max_over_ranks(start.elapsed_time(end), world, device) / steps
    h2d = sum(v.numel() * v.element_size() for v in host_in.values() if v is not None)
    d2h = sum(o.numel() * o.element_size() for o in sets[0]["results"])
    units, divisor, unit, _ = work(wl)
    return {"value": round(units * world / (ms * 1e-3) / divisor, 3), "unit": unit, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 4), "steps": steps,
            "note": "every step: pinned host inputs -> device, C-ABI call, results -> pinned host; "
                    "pipelined over 3 buffer sets on separate copy / compute streams"}


# ---------------------------------------------------------------- the oracle (CPU) arm

def _oracle_rows(wl, r0, r1):
    import oracle

    t = wl.tensors
    if wl.kind == "w8a8_gemm":
        return oracle.w8a8_gemm(t["a"][r0:r1].numpy(), t["b"].numpy(), t["a_scale"][r0:r1].numpy(),
                                t["b_scale"].numpy(), out_dtype=wl.out_dtype)
    if wl.kind == "dequant_per_group":
        off = t.get("offset")
        if wl.k_dim == 1:
            tr = slice(r0, r1)
        else:  # column groups: start the sample on a group boundary
            r0 -= r0 % wl.group_size
            tr = slice(r0 // wl.group_size, -(-r1 // wl.group_size))
        return oracle.dequant_per_group(t["y"][r0:r1].numpy(), t["scale"][tr], None if off is None else off[tr],
                                        group_size=wl.group_size, k_dim=wl.k_dim, y_dtype=wl.y_dtype, cols=wl.cols,
                                        out_dtype=wl.out_dtype)
    if wl.kind == "dequant_per_token":
        off = t.get("offset")
        return oracle.dequant_per_token(t["y"][r0:r1].numpy(), t["scale"][r0:r1],
                                        None if off is None else off[r0:r1], y_dtype=wl.y_dtype, cols=wl.cols,
                                        out_dtype=wl.out_dtype)
    if wl.kind == "dynamic_quant":
        gi = t.get("group_index")
        smooth = t.get("smooth")
        if gi is not None:
            # rows [r0, r1) with their experts: rebase the cumulative end rows
            g = gi.numpy().astype("int64") - r0
            g = g.clip(0, r1 - r0).astype("int32")
            return oracle.dynamic_quant(t["x"][r0:r1], smooth=smooth, group_index=g, mode=wl.mode,
                                        y_dtype=wl.y_dtype)
        return oracle.dynamic_quant(t["x"][r0:r1], smooth=smooth, mode=wl.mode, y_dtype=wl.y_dtype)
    b, s, h = t["x"].shape
    x = t["x"].reshape(b * s, h)
    # rows of one batch entry at a time (the adaptive parameters are per batch)
    bi = r0 // s
    r1 = min(r1, (bi + 1) * s)
    xs = x[r0:r1].reshape(1, r1 - r0, h)
    return oracle.ada_layernorm_quant(xs, t["ada_scale"][bi:bi + 1], t["ada_shift"][bi:bi + 1], t.get("weight"),
                                      t.get("bias"), t.get("smooth"), epsilon=wl.epsilon)


def cpu_baseline(wl, nbytes, target_s: float = 10.0):
    """The oracle as it stands, single-threaded, on a bounded sample of rows."""
    rows = wl.rows
    units, divisor, unit, _ = work(wl)
    bytes_per_row = units / rows  # work units (bytes, or tensor ops) per row
    # calibrate on a small slice, then size the sample to ~target_s of CPU work
    n0 = min(rows, 64)
    t0 = time.perf_counter()
    _oracle_rows(wl, 0, n0)
    dt = max(time.perf_counter() - t0, 1e-6)
    per_row = dt / n0
    n = int(min(rows, max(n0, target_s / per_row)))
    passes, elapsed, done = 0, 0.0, 0
    while elapsed < target_s and passes < 1000:
        t0 = time.perf_counter()
        _oracle_rows(wl, 0, n)
        elapsed += time.perf_counter() - t0
        done += n
        passes += 1
    gbs = done * bytes_per_row / elapsed / divisor
    return {"value": round(gbs, 6), "unit": unit, "cores": 1, "kind": "oracle",
            "sample": f"first {n} of {rows} rows x {passes} pass(es) ({elapsed:.1f} s), "
                      f"single-threaded C++ oracle, {unit} of the same algorithmic work",
            "host_cpus": os.cpu_count()}


def run_reference(args, world, rank):
    from token_dynamic_quantization_b200 import workloads

    if rank != 0:
        return None
    wl = workloads.make(args.workload, rows=args.rows)
    units, divisor, unit, metric = work(wl)
    rows = wl.rows
    bytes_per_row = units / rows  # work units (bytes, or tensor ops) per row
    # size each step so that warmup + steps take about args.cpu_seconds in total
    n0 = min(rows, 64)
    t0 = time.perf_counter()
    _oracle_rows(wl, 0, n0)
    per_row = max(time.perf_counter() - t0, 1e-6) / n0
    budget = args.cpu_seconds * 3
    n = int(max(1, min(rows, budget / (per_row * max(1, args.steps + args.warmup)))))
    for _ in range(args.warmup):
        _oracle_rows(wl, 0, n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_rows(wl, 0, n)
    elapsed = time.perf_counter() - t0
    ms_per_step = elapsed / args.steps * 1e3
    gbs = n * bytes_per_row * args.steps / elapsed / divisor
    sample = f"first {n} of {rows} rows per step, single-threaded C++ oracle"
    return {
        "impl": "reference",
        "metric": metric,
        "value": round(gbs, 6),
        "unit": unit,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "s8 x s8 -> s32, f32 scales" if wl.kind == "w8a8_gemm" else "f32",
        "data": "synthetic",
        "config": {"workload": args.workload, **workload_config(wl), "rows_per_step": n,
                   "rows_per_s": round(n * args.steps / elapsed, 1)},
        "cpu_baseline": {"value": round(gbs, 6), "unit": unit, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": "reference arm = the CPU oracle (the pages ship no runnable implementation)",
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--rows", type=int, default=None,
                    help="smaller row count of the same workload (for quick profiler captures)")
    ap.add_argument("--graph", action="store_true", help="replay the K timed launches as one CUDA graph")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        raise SystemExit(relaunch_under_torchrun(sys.argv[1:] if argv is None else list(argv), args.gpus))

    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            res = run_reference(args, world, rank)
        else:
            res = run_ours(args, world, rank, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
