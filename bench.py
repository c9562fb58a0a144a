#!/usr/bin/env python
"""Benchmark of the W4A16 decode path on B200.

A step is one decode pass (M = 1 token) through the seven linears of a
LLaMA-2-7B-shaped block (q/k/v/o 4096x4096, gate/up 4096->11008, down
11008->4096), 4-bit asymmetric, group 128, packed by this library. Steps
rotate over copies of the block whose packed weights together exceed the L2
cache, so every step streams its weights from HBM. Each block copy's seven
launches are one CUDA graph.

The headline `value` is the effective bandwidth of the step: algorithmic bytes
(packed weights + fp16 steps + fp16 zeros + X + Y) / device time. The last
stdout line is that headline with `roofline` (against the measured HBM copy
bandwidth, with the DRAM traffic ncu recorded for the kernel's current
source), `e2e` (the public calls from pinned host buffers), `cpu_baseline`
(the oracle on 1 and all host cores), `clocks` and `gpu_launches`. The line
before it carries `rows`, the other hot-path rows measured in the same run:
quantize + pack, the block with q|k|v and gate|up packed, single-shape GEMVs
(3-bit, groups of 32/64, 8192x28672), the small-M sweep with and without the
GEMM workspace, dense fp16 matmuls for context, W4A8, the AWQ search (fused,
two-kernel, 3-bit pipeline), the scale fold and GPTQ.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank runs its own replicas (weak scaling, no
collective on the data path); rank 0 prints the max-over-ranks timing.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A16 GEMV effective GB/s & % of B200 HBM peak; small-M GEMM TFLOP/s"
WORKLOAD = "llama2_7b_block_decode_M1_w4_asym_g128"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def gemm_bytes(M: int, N: int, K: int, bits: int) -> int:
    """Algorithmic bytes of one W{bits}A16 matmul: packed weight, fp16 steps and
    zeros (one each per 128 input channels of a row), X and Y."""
    return N * K * bits // 8 + N * (K // 128) * 4 + M * K * 2 + M * N * 2


def quantize_bytes(N: int, K: int, bits: int) -> int:
    return N * K * 2 + N * K * bits // 8 + N * (K // 128) * 4


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# Source files of each kernel whose DRAM traffic the bench reports.
KERNEL_SOURCES = {"gemv_rows_kernel": ("wq_gemv_rows.cu", "wq_common.cuh")}


def _code_only(text: str) -> str:
    """C++ source without comments and whitespace."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return re.sub(r"\s+", "", text)


def kernel_source_hash(kernel: str = "gemv_rows_kernel") -> str:
    """Hash of the code (comments and whitespace dropped) of the files that
    define `kernel`: a stored traffic figure is used only while it is
    unchanged."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "weight_only_quantization_group_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(d, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, if the
    kernel's sources have not changed since it was captured."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or kernel not in KERNEL_SOURCES or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


def gpu_uuid(index: int) -> str | None:
    """The CUDA device's UUID (to find the same GPU through NVML), or None."""
    try:
        import torch
        u = getattr(torch.cuda.get_device_properties(index), "uuid", None)
        return str(u) if u is not None else None
    except Exception:
        return None


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank reports its own device time and all
    take the maximum (the same collective on every rank, in the same order)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """SM clocks and throttle reasons while the timed steps run: nvidia-smi
    every 200 ms, one nvidia-smi reading on each side of the region, and an
    NVML thread reading the clock and the active event reasons every 100 us
    (a timed region of a millisecond sees no periodic nvidia-smi sample).
    Read-only: nothing here changes a setting of the GPU."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clocks-event reason bits (nvml.h, nvmlClocksEventReason*), by the
    # names the summary reports
    NVML_REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                    "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, gpu_index: int, uuid: str | None = None, nvml=None, period_s: float = 100e-6):
        self.gpu = gpu_index
        self.uuid = uuid
        self.proc = None
        self.lines = []
        self.nvml = nvml            # the pynvml module (injected by tests), else imported on entry
        self.period = period_s
        self.nvml_sm = []           # SM MHz per NVML sample
        self.nvml_reasons = set()
        self.nvml_max = None
        self._thread = None
        self._stop = None

    def _once(self):
        """One immediate sample (a short timed region may see no periodic one)."""
        try:
            r = subprocess.run(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=10)
            self.lines += [ln for ln in r.stdout.splitlines() if ln.strip()]
        except (OSError, subprocess.SubprocessError):
            pass

    def _nvml_handle(self, nv):
        """The NVML device of this rank's CUDA device: matched by UUID (NVML
        does not follow CUDA_VISIBLE_DEVICES), else by index."""
        if self.uuid:
            want = self.uuid.lower().removeprefix("gpu-")
            for i in range(nv.nvmlDeviceGetCount()):
                h = nv.nvmlDeviceGetHandleByIndex(i)
                u = nv.nvmlDeviceGetUUID(h)
                u = (u.decode() if isinstance(u, bytes) else u).lower().removeprefix("gpu-")
                if u == want:
                    return h
        return nv.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll(self, nv, h):
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            except Exception:
                return
            self.nvml_sm.append(float(sm))
            for nm, b in self.NVML_REASONS.items():
                if bits & b:
                    self.nvml_reasons.add(nm)
            time.sleep(self.period)

    def _start_nvml(self):
        import threading
        nv = self.nvml
        try:
            if nv is None:
                import pynvml as nv
            nv.nvmlInit()
            h = self._nvml_handle(nv)
            self.nvml_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:
            return
        self.nvml = nv
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
        self._thread.start()

    def __enter__(self):
        self._once()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        self._start_nvml()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines += [ln for ln in out.splitlines() if ln.strip()]
        self._once()
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        smi_samples = len(sm)
        sm += self.nvml_sm
        reasons |= self.nvml_reasons
        if mx is None:
            mx = self.nvml_max
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
               "samples": len(sm), "nvml_samples": len(self.nvml_sm), "smi_samples": smi_samples}
        if self.nvml_sm:
            out["sm_mhz_min"] = min(self.nvml_sm)
        return out


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    from weight_only_quantization_group_b200 import build
    build.build()
    import weight_only_quantization_group_b200 as wq
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks = load_peaks()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    def dt(t):
        return torch.from_numpy(np.ascontiguousarray(t)).to(dev)

    # -- the block: quantize + pack each linear on the GPU -------------------
    cases = synth.config_llama7b_decode(1)
    block = []
    for c in cases:
        N, K = c.W.shape
        Wd = dt(c.W)
        packed, steps, zeros = wq.wq_quantize_pack(Wd, bits=4)
        block.append({"name": c.name, "N": N, "K": K, "X": dt(c.X), "W": Wd, "q": (packed, steps, zeros),
                      "Xh": c.X})
    assert wq.wq_get_last_device_error() == 0
    step_bytes = sum(gemm_bytes(1, b["N"], b["K"], 4) for b in block)
    block_w_bytes = sum(b["N"] * b["K"] // 2 for b in block)
    n_copies = max(2, math.ceil(4 * L2_BYTES / block_w_bytes))

    # -- rotating block copies and one graph per copy -------------------------
    copies = [block]
    for _ in range(n_copies - 1):
        copies.append([{**b, "q": tuple(t.clone() for t in b["q"])} for b in block])
    Ys = [[torch.empty((1, b["N"]), dtype=torch.float16, device=dev) for b in block] for _ in copies]
    s_cap = torch.cuda.Stream(device=dev)
    graphs = []
    for ci, blk in enumerate([] if args.eager else copies):
        # warm the launch path (function attributes) before capture
        for b, y in zip(blk, Ys[ci]):
            wq.wq_w4a16_gemm(b["X"], *b["q"], b["N"], bits=4, out=y)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s_cap):
            for b, y in zip(blk, Ys[ci]):
                wq.wq_w4a16_gemm(b["X"], *b["q"], b["N"], bits=4, out=y)
        graphs.append(g)
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()

    def run_step(i):
        if args.eager:  # same launches without graphs (for profilers)
            ci = i % n_copies
            for b, y in zip(copies[ci], Ys[ci]):
                wq.wq_w4a16_gemm(b["X"], *b["q"], b["N"], bits=4, out=y)
        else:
            graphs[i % n_copies].replay()

    for i in range(args.warmup):
        run_step(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank, gpu_uuid(local_rank)) as clk:
        ev0.record(stream)
        for i in range(args.steps):
            run_step(i)
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    assert wq.wq_get_last_device_error() == 0
    ms_per_step = ms / args.steps
    value = world * step_bytes * args.steps / (ms * 1e-3) / 1e9  # GB/s, all ranks

    # -- e2e: the public call with host buffers, copies inside the timed region.
    # The seven inputs travel in one pinned host buffer (one copy in), the
    # seven outputs in one device buffer (one copy out), as a serving loop would
    # stage them.
    k_off = np.cumsum([0] + [b["K"] for b in block])
    n_off = np.cumsum([0] + [b["N"] for b in block])
    xh_all = torch.from_numpy(np.concatenate([b["Xh"].reshape(-1) for b in block])).pin_memory()
    yh_all = torch.empty(int(n_off[-1]), dtype=torch.float16).pin_memory()
    x_all = torch.empty(int(k_off[-1]), dtype=torch.float16, device=dev)
    y_all = torch.empty(int(n_off[-1]), dtype=torch.float16, device=dev)
    x_views = [x_all[int(k_off[i]):int(k_off[i + 1])].view(1, -1) for i in range(len(block))]
    y_views = [y_all[int(n_off[i]):int(n_off[i + 1])].view(1, -1) for i in range(len(block))]
    e2e_steps = max(20, min(2000, args.steps // 10))
    h2d = xh_all.numel() * 2
    d2h = yh_all.numel() * 2

    def e2e_calls(blk):
        x_all.copy_(xh_all, non_blocking=True)
        for b, x, y in zip(blk, x_views, y_views):
            wq.wq_w4a16_gemm(x, *b["q"], b["N"], bits=4, out=y)
        yh_all.copy_(y_all, non_blocking=True)

    # As a decode loop runs it: the step's calls (copy in, seven GEMVs, copy
    # out) captured once per weight copy and replayed, then a host sync on the
    # result; eagerly issued calls are timed too (row e2e_eager).
    e2e_graphs = []
    if not args.eager:
        for blk in copies:
            e2e_calls(blk)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s_cap):
                e2e_calls(blk)
            e2e_graphs.append(g)
        torch.cuda.synchronize()

    def e2e_step(i, graphs):
        if graphs:
            graphs[i % n_copies].replay()
        else:
            e2e_calls(copies[i % n_copies])
        torch.cuda.current_stream().synchronize()

    def time_e2e(graphs):
        for i in range(3):
            e2e_step(i, graphs)
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(e2e_steps):
            e2e_step(i, graphs)
        e1.record()
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), world, dev)

    e2e_ms = time_e2e(e2e_graphs)
    e2e_value = world * step_bytes * e2e_steps / (e2e_ms * 1e-3) / 1e9
    e2e_eager_ms = time_e2e([]) if e2e_graphs else e2e_ms
    del e2e_graphs

    rows = {}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if rank == 0 and world == 1 and not args.no_rows:
        # the same graphs' step time with programmatic dependent launch off
        wq.wq_set_option(wq.WQ_OPT_PDL, 0)
        try:
            g_off = []
            for ci, blk in enumerate(copies[:2]):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=s_cap):
                    for b, y in zip(blk, Ys[ci]):
                        wq.wq_w4a16_gemm(b["X"], *b["q"], b["N"], bits=4, out=y)
                g_off.append(g)
            torch.cuda.synchronize()
            for i in range(20):
                g_off[i % 2].replay()
            e0.record()
            for i in range(400):
                g_off[i % 2].replay()
            e1.record()
            torch.cuda.synchronize()
            rows["block_step_pdl_off"] = {"us": e0.elapsed_time(e1) / 400 * 1e3,
                                          "note": "2 block copies only (L2 may hold part)"}
            del g_off
        finally:
            wq.wq_set_option(wq.WQ_OPT_PDL, 1)
        # the same seven linears with the ones that share an input concatenated
        # along N (q|k|v, gate|up): four launches per step, identical codes and
        # outputs (groups never cross rows)
        fused_copies = []
        for blk in copies[:n_copies]:
            by = {b["name"].split("_")[2]: b for b in blk}
            f = []
            for names in (("q", "k", "v"), ("o",), ("gate", "up"), ("down",)):
                parts = [by[n] for n in names]
                q = tuple(torch.cat([p["q"][i] for p in parts], 0) for i in range(3))
                N = sum(p["N"] for p in parts)
                f.append((parts[0]["X"], q, N, torch.empty((1, N), dtype=torch.float16, device=dev)))
            fused_copies.append(f)
        g_fused = []
        for f in fused_copies:
            for X, q, N, y in f:
                wq.wq_w4a16_gemm(X, *q, N, bits=4, out=y)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s_cap):
                for X, q, N, y in f:
                    wq.wq_w4a16_gemm(X, *q, N, bits=4, out=y)
            g_fused.append(g)
        torch.cuda.synchronize()
        for i in range(20):
            g_fused[i % n_copies].replay()
        e0.record()
        for i in range(400):
            g_fused[i % n_copies].replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / 400 * 1e3
        rows["block_step_fused_4_launches"] = {"us": us, "GB/s": step_bytes / (us * 1e-6) / 1e9,
                                               "frac_hbm": step_bytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                                               "note": "q|k|v and gate|up concatenated along N"}
        del g_fused, fused_copies
        rows = {**rows, **measure_rows(wq, torch, synth, dev, block, peaks)}

    del graphs
    if rank != 0:
        return None, None

    clocks = clk.summary()
    traffic = profiled_traffic("gemv_rows_kernel")
    achieved = step_bytes / (ms_per_step * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic",
        "config": {
            "workload": WORKLOAD,
            "linears": [f"{b['name']}" for b in block],
            "bytes_per_step": step_bytes,
            "block_copies": n_copies,
            "l2": f"inputs larger than L2: {n_copies} block copies, {n_copies * block_w_bytes / 1e6:.0f} MB of packed weight rotate",
            "graph": "eager launches" if args.eager else "one CUDA graph of 7 launches per block copy",
            "parallelism": f"replicas x{world}",
        },
        "roofline": {
            "bound": "hbm",
            "kernel": "gemv_rows_kernel (ActHalf offset sums; R4 C32 S2 for K=4096, R4 C64 S2 for K=11008)",
            "achieved": round(achieved, 2),
            "peak": peaks["hbm_gbs"],
            "peak_source": f"{peaks['source']} HBM copy bandwidth",
            "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": traffic,
            "note": "achieved = algorithmic bytes of the 7 launches / device time of the step (graph gaps included)",
        },
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                "path": ("CUDA graph of the step's public calls: one pinned copy of the 7 inputs in, "
                         "wq_w4a16_gemm per linear, one copy of the 7 outputs out; host sync on the result per step"
                         if not args.eager else
                         "one pinned copy of the 7 inputs in, wq_w4a16_gemm per linear, one copy of the 7 outputs "
                         "out, stream sync per step"),
                "eager_value": round(world * step_bytes * e2e_steps / (e2e_eager_ms * 1e-3) / 1e9, 2),
                "eager_ms_per_step": e2e_eager_ms / e2e_steps},
        "gpu_launches": 7 * args.steps * world,  # all ranks' launches in the timed region
        "clocks": clocks,
        "rows_line": ("printed on the line before this one" if rows else
                      "measured at N = 1 only" if world > 1 else "not measured (--no-rows)"),
    }
    if "block_step_fused_4_launches" in rows:
        f = rows["block_step_fused_4_launches"]
        line["packed_4_launches"] = {
            "value": round(f["GB/s"], 2), "unit": "GB/s", "ms_per_step": f["us"] / 1e3,
            "frac": round(f["frac_hbm"], 4),
            "note": "the same 7 linears and bytes, q|k|v and gate|up each packed as one weight (they share an "
                    "input): 4 launches per step"}
    if not args.no_cpu_baseline and world == 1:  # the host baseline: rank 0 at N = 1 only
        line["cpu_baseline"] = cpu_baseline(cases, args.cpu_seconds)
    return line, rows


def _time_graph(torch, fn_list, reps: int = 5, inner: int = 1):
    """Median ms of one pass over fn_list, captured as one graph and replayed."""
    s = torch.cuda.Stream()
    for f in fn_list:
        f()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(inner):
            for f in fn_list:
                f()
    g.replay()
    torch.cuda.synchronize()
    out = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        out.append(a.elapsed_time(b) / inner)
    del g
    return statistics.median(out)


def measure_rows(wq, torch, synth, dev, block, peaks):
    rows = {}

    def dt(t):
        return torch.from_numpy(np.ascontiguousarray(t)).to(dev)

    # S3 quantize + pack over the block (W fp16 read 404 MB > L2)
    fns = [lambda b=b: wq.wq_quantize_pack(b["W"], bits=4, out=b["q"]) for b in block]
    ms = _time_graph(torch, fns)
    qb = sum(quantize_bytes(b["N"], b["K"], 4) for b in block)
    rows["quantize_pack_block_w4"] = {"ms": ms, "GB/s": qb / (ms * 1e-3) / 1e9,
                                      "frac_hbm": qb / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                      "weights": sum(b["N"] * b["K"] for b in block)}

    # single-shape GEMVs, rotating copies >= 4x L2
    def gemv_row(name, N, K, bits, W16, X16, M=1, ws=True):
        """ws: pass the GEMM workspace (the tensor-core kernel's stream-K
        schedule where it applies), as a caller that has one would."""
        packed, steps, zeros = wq.wq_quantize_pack(dt(W16), bits=bits)
        wbytes = N * K * bits // 8
        nc = max(2, math.ceil(4 * L2_BYTES / wbytes))
        qs = [(packed, steps, zeros)] + [tuple(t.clone() for t in (packed, steps, zeros)) for _ in range(nc - 1)]
        X = dt(X16)
        Y = torch.empty((M, N), dtype=torch.float16, device=dev)
        nws = wq.wq_gemm_workspace_bytes(M, N, K, bits=bits) if ws else 0
        W = torch.zeros(nws, dtype=torch.uint8, device=dev) if nws else None  # zero-filled once
        fns = [lambda q=q: wq.wq_w4a16_gemm(X, *q, N, bits=bits, out=Y, workspace=W) for q in qs]
        ms = _time_graph(torch, fns) / nc
        by = gemm_bytes(M, N, K, bits)
        fl = 2.0 * M * N * K
        rows[name] = {"M": M, "N": N, "K": K, "bits": bits, "us": ms * 1e3, "GB/s": by / (ms * 1e-3) / 1e9,
                      "frac_hbm": by / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "TFLOP/s": fl / (ms * 1e-3) / 1e12}
        del qs

    c1 = synth.config_small_linear(0)
    gemv_row("gemv_small_linear_K256_N128", 128, 256, 4, c1.W, c1.X)
    for b in block[:1] + block[4:5] + block[6:7]:
        gemv_row(f"gemv_{b['name']}", b["N"], b["K"], 4, b["W"].cpu().numpy(), b["Xh"])
    for bits in (4, 3):
        c = synth.config_llama65b_decode(bits)
        gemv_row(f"gemv_llama65b_8192x8192_w{bits}", 8192, 8192, bits, c.W, c.X)
        if bits == 3:  # 3-bit rows with two rows per batch
            wq.wq_set_option(wq.WQ_OPT_GEMV_ROWS_SHAPE, 3)
            try:
                gemv_row("gemv_llama65b_8192x8192_w3_rows_r2", 8192, 8192, bits, c.W, c.X)
            finally:
                wq.wq_set_option(wq.WQ_OPT_GEMV_ROWS_SHAPE, 0)
        for tag, var in (("tiled", wq.WQ_GEMV_OFFSET_SUMS), ("tiled_exact", wq.WQ_GEMV_EXACT)):
            wq.wq_set_option(wq.WQ_OPT_GEMV_KERNEL, wq.WQ_GEMV_KERNEL_TILED)
            wq.wq_set_option(wq.WQ_OPT_GEMV_VARIANT, var)
            try:
                gemv_row(f"gemv_llama65b_8192x8192_w{bits}_{tag}", 8192, 8192, bits, c.W, c.X)
            finally:
                wq.wq_set_option(wq.WQ_OPT_GEMV_KERNEL, wq.WQ_GEMV_KERNEL_AUTO)
                wq.wq_set_option(wq.WQ_OPT_GEMV_VARIANT, wq.WQ_GEMV_OFFSET_SUMS)
    big = synth.config_smallm_sweep(1)
    # row-streaming kernel shapes (rows per batch, channels per lane)
    c65 = synth.config_llama65b_decode(4)
    # and the two ways of forming lane sums (int: integer digits, half: fp32
    # offset sums), and the grid rule (g0 / g1)
    shapes = {1: "r4x32s2", 2: "r4x64s2", 3: "r2x64s2", 4: "r4x32s3"}
    sweep = [("half", wq.WQ_GEMV_OFFSET_SUMS, sh, 1) for sh in shapes]
    sweep += [("int", wq.WQ_GEMV_INT_DIGITS, sh, 1) for sh in (2, 4)]
    sweep += [("half", wq.WQ_GEMV_OFFSET_SUMS, sh, 0) for sh in (2, 4)]
    for vtag, var, shape, gm in sweep:
        wq.wq_set_option(wq.WQ_OPT_GEMV_ROWS_SHAPE, shape)
        wq.wq_set_option(wq.WQ_OPT_GEMV_VARIANT, var)
        wq.wq_set_option(wq.WQ_OPT_GEMV_GRID, gm)
        try:
            tag2 = f"{shapes[shape]}_{vtag}_g{gm}"
            gemv_row(f"gemv_rows_{tag2}_8192x8192_w4", 8192, 8192, 4, c65.W, c65.X)
            gemv_row(f"gemv_rows_{tag2}_8192x28672_w4", 28672, 8192, 4, big.W, synth.smallm_activations(1))
            for b in (block[0], block[4], block[6]):
                gemv_row(f"gemv_rows_{tag2}_{b['name']}", b["N"], b["K"], 4, b["W"].cpu().numpy(), b["Xh"])
            if shape in (1, 2, 3):
                gemv_row(f"gemv_rows_{tag2}_M2_8192x28672_w4", 28672, 8192, 4, big.W, synth.smallm_activations(2),
                         M=2)
        finally:
            wq.wq_set_option(wq.WQ_OPT_GEMV_ROWS_SHAPE, 0)
            wq.wq_set_option(wq.WQ_OPT_GEMV_VARIANT, wq.WQ_GEMV_OFFSET_SUMS)
            wq.wq_set_option(wq.WQ_OPT_GEMV_GRID, 1)
    for M in synth.SMALLM_SWEEP:
        gemv_row(f"smallm_M{M}_8192x28672_w4", 28672, 8192, 4, big.W, synth.smallm_activations(M), M=M)
        if M >= 3:  # the same call without a workspace: one CTA per row tile
            gemv_row(f"smallm_M{M}_8192x28672_w4_nows", 28672, 8192, 4, big.W, synth.smallm_activations(M), M=M,
                     ws=False)
    # context: the dense fp16 matmul of the same shape (cuBLAS through torch),
    # reading the 470 MB fp16 weight
    Wd16 = dt(big.W)
    for M in (1, 16, 128):
        Xd = dt(synth.smallm_activations(M))
        Yd = torch.empty((M, 28672), dtype=torch.float16, device=dev)
        ms = _time_graph(torch, [lambda: torch.matmul(Xd, Wd16.t(), out=Yd)])
        fl = 2.0 * M * 28672 * 8192
        by = 28672 * 8192 * 2 + M * 8192 * 2 + M * 28672 * 2
        rows[f"torch_fp16_dense_M{M}_8192x28672"] = {
            "us": ms * 1e3, "TFLOP/s": fl / (ms * 1e-3) / 1e12, "frac_bf16_peak": fl / (ms * 1e-3) / 1e12 /
            peaks["bf16_tflops"], "GB/s": by / (ms * 1e-3) / 1e9, "note": "torch.matmul, dense fp16 weight (context)"}
    del Wd16
    # tensor-core kernel: dequantizing warps, channels per stage, ring depth (0 = library choice)
    for M in (4, 16, 64, 128):
        for dw, bk, S in ((8, 128, 0), (4, 128, 0), (4, 128, 5), (4, 64, 0), (8, 64, 5), (8, 128, 5)):
            wq.wq_set_option(wq.WQ_OPT_TC_STAGES, S)
            wq.wq_set_option(wq.WQ_OPT_TC_BK, bk)
            wq.wq_set_option(wq.WQ_OPT_TC_DEQUANT_WARPS, dw)
            name = f"smallm_M{M}_8192x28672_w4_tc_dw{dw}_bk{bk}_s{S}"
            try:
                gemv_row(name, 28672, 8192, 4, big.W, synth.smallm_activations(M), M=M)
            except wq.WQError as e:
                rows[name] = {"error": str(e)}
            finally:
                wq.wq_set_option(wq.WQ_OPT_TC_STAGES, 0)
                wq.wq_set_option(wq.WQ_OPT_TC_BK, 0)
                wq.wq_set_option(wq.WQ_OPT_TC_DEQUANT_WARPS, 0)
    c4 = synth.config_llama65b_decode(4)
    # the other kernel on each side of the crossover, for the record
    for M in (2, 3, 4, 8, 16):
        path = wq.WQ_PATH_TENSOR_CORE if M < 3 else wq.WQ_PATH_GEMV
        if M in (3, 4):  # both kernels at M = 3, 4 on the narrower weights (the default picks the row kernel)
            for p2, t2 in ((wq.WQ_PATH_GEMV, "gemv"), (wq.WQ_PATH_TENSOR_CORE, "tc")):
                wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, p2)
                try:
                    gemv_row(f"smallm4_M{M}_8192x8192_w4_{t2}", 8192, 8192, 4, c4.W, synth.smallm_activations(M),
                             M=M)
                    for b in (block[0], block[4], block[6]):
                        Xm = synth.activations(synth.rng(77 + M), M, b["K"])
                        gemv_row(f"M{M}_{b['name'].replace('_M1', '')}_{t2}", b["N"], b["K"], 4,
                                 b["W"].cpu().numpy(), Xm, M=M)
                finally:
                    wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, wq.WQ_PATH_AUTO)
        wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, path)
        try:
            tag = "tc" if path == wq.WQ_PATH_TENSOR_CORE else "gemv"
            gemv_row(f"smallm_M{M}_8192x28672_w4_{tag}", 28672, 8192, 4, big.W, synth.smallm_activations(M), M=M)
        finally:
            wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, wq.WQ_PATH_AUTO)
    # small-M sweeps on the LLaMA-65B-shaped 8192 x 8192 weight, 4- and 3-bit
    # (64 row tiles: M >= 3 splits K over clusters of CTAs)
    for bits in (4, 3):
        cb = synth.config_llama65b_decode(bits)
        for M in synth.SMALLM_SWEEP:
            gemv_row(f"smallm{bits}_M{M}_8192x8192_w{bits}", 8192, 8192, bits, cb.W, synth.smallm_activations(M), M=M)
    # the K split forced, M = 16, 8192 x 8192 4-bit
    for ks in (1, 2, 4, 8):
        wq.wq_set_option(wq.WQ_OPT_TC_KSPLIT, ks)
        try:
            gemv_row(f"smallm4_M16_8192x8192_w4_ksplit{ks}", 8192, 8192, 4, c4.W, synth.smallm_activations(16), M=16)
        except wq.WQError as e:
            rows[f"smallm4_M16_8192x8192_w4_ksplit{ks}"] = {"error": str(e)}
        finally:
            wq.wq_set_option(wq.WQ_OPT_TC_KSPLIT, 0)
    # groups of 32 and 64 channels (8192 x 28672, 4-bit): decode GEMV and M = 16
    for group in (32, 64):
        for M in (1, 16):
            name = f"group{group}_M{M}_8192x28672_w4"
            W16 = big.W
            packed, steps, zeros = wq.wq_quantize_pack(dt(W16), bits=4, group_size=group)
            nc = max(2, math.ceil(4 * L2_BYTES / (28672 * 8192 // 2)))
            qs = [(packed, steps, zeros)] + [tuple(t.clone() for t in (packed, steps, zeros)) for _ in range(nc - 1)]
            X = dt(synth.smallm_activations(M))
            Y = torch.empty((M, 28672), dtype=torch.float16, device=dev)
            fns = [lambda q=q: wq.wq_w4a16_gemm(X, *q, 28672, bits=4, group_size=group, out=Y) for q in qs]
            ms = _time_graph(torch, fns) / nc
            by = 28672 * 8192 // 2 + 28672 * (8192 // group) * 4 + M * 8192 * 2 + M * 28672 * 2
            rows[name] = {"M": M, "group": group, "us": ms * 1e3, "GB/s": by / (ms * 1e-3) / 1e9,
                          "frac_hbm": by / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
            del qs
    # S1/S2/S4 AWQ scale search over one LLaMA-2-7B block (4 search places,
    # T=512 calibration rows, 20 alphas), then packing with the chosen scales
    groups = synth.config_awq_block(5)
    flops = sum(2.0 * X.shape[0] * sum(W.shape[0] for _, W in named) * X.shape[1] * 20 for _, X, named in groups)

    def awq_block(bits, loss_path):
        old = wq.wq_get_option(wq.WQ_OPT_AWQ_LOSS)
        wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, loss_path)
        try:
            prepared = []
            for gname, X, named in groups:
                Xd = dt(X)
                Wd = [dt(W) for _, W in named]
                need = wq.wq_awq_workspace_bytes(X.shape[0], X.shape[1], [W.shape[0] for W in Wd], 20, bits=bits)
                prepared.append((gname, Xd, Wd, torch.empty(need, dtype=torch.uint8, device=dev)))
            outs = [wq.wq_awq_scale_search(Xd, Wd, bits=bits, workspace=ws) for _, Xd, Wd, ws in prepared]
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            outs = [wq.wq_awq_scale_search(Xd, Wd, bits=bits, workspace=ws) for _, Xd, Wd, ws in prepared]
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b)
            assert wq.wq_get_last_device_error() == 0
            return prepared, outs, ms
        finally:
            wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, old)

    # default: the error tiles built inside the loss GEMM (no E in HBM)
    prepared, outs, ms = awq_block(4, wq.WQ_AWQ_LOSS_FUSED)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    packs4 = [wq.wq_quantize_pack(W, o["s"], bits=4) for (_, Xd, Wd, _), o in zip(prepared, outs) for W in Wd]
    a.record()
    i = 0
    for (_, Xd, Wd, _), o in zip(prepared, outs):
        for W in Wd:
            wq.wq_quantize_pack(W, o["s"], bits=4, out=packs4[i])
            i += 1
    b.record()
    torch.cuda.synchronize()
    assert wq.wq_get_last_device_error() == 0
    rows["awq_search_llama7b_block"] = {
        "ms": ms, "loss_gemm_TFLOP/s": flops / (ms * 1e-3) / 1e12,
        "frac_bf16_peak": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
        "best_alpha": {g: int(o["best"].item()) / 20 for (g, _, _, _), o in zip(prepared, outs)},
        "pack_with_s_ms": a.elapsed_time(b)}
    # the option: E written to global memory in fp16 and read back by a second kernel
    _, outs2, ms2 = awq_block(4, wq.WQ_AWQ_LOSS_TWO_KERNELS)
    rows["awq_search_llama7b_block_two_kernels"] = {
        "ms": ms2, "loss_gemm_TFLOP/s": flops / (ms2 * 1e-3) / 1e12,
        "same_alpha_as_default": all(int(f["best"].item()) == int(o["best"].item()) for f, o in zip(outs2, outs))}
    del prepared, outs, outs2

    # the 3-bit group-128 pipeline at block scale: AWQ search, pack with s,
    # then one decode step (7 GEMVs, X diag(s)^-1 prepared once)
    prepared, outs, ms3 = awq_block(3, wq.WQ_AWQ_LOSS_FUSED)
    packs = []
    for (_, Xd, Wd, _), o in zip(prepared, outs):  # outputs allocated once, untimed
        for W in Wd:
            packs.append((W.shape[0], W.shape[1], o["s"], wq.wq_quantize_pack(W, o["s"], bits=3)))
    a.record()
    i = 0
    for (_, Xd, Wd, _), o in zip(prepared, outs):
        for W in Wd:
            wq.wq_quantize_pack(W, o["s"], bits=3, out=packs[i][3])
            i += 1
    b.record()
    torch.cuda.synchronize()
    pack3_ms = a.elapsed_time(b)
    xs = [torch.randn((1, K), device=dev).half() / s for N, K, s, _ in packs]
    ys = [torch.empty((1, N), dtype=torch.float16, device=dev) for N, _, _, _ in packs]
    fns = [lambda i=i: wq.wq_w4a16_gemm(xs[i], *packs[i][3], packs[i][0], bits=3, out=ys[i]) for i in range(len(packs))]
    step3 = _time_graph(torch, fns)
    by3 = sum(gemm_bytes(1, N, K, 3) for N, K, _, _ in packs)
    assert wq.wq_get_last_device_error() == 0
    rows["awq_pipeline_llama7b_block_w3"] = {
        "search_ms": ms3, "pack_with_s_ms": pack3_ms, "decode_step_us": step3 * 1e3,
        "decode_step_GB/s": by3 / (step3 * 1e-3) / 1e9,
        "note": "decode step: the block's 7 linears once (weights L2-resident after packing, not rotated)",
        "best_alpha": {g: int(o["best"].item()) / 20 for (g, _, _, _), o in zip(prepared, outs)}}
    del prepared, outs, packs

    # W4A8 (Lab 5's linear): int8 activation codes per group of 32, dp4a
    # group dot products, 8192 x 28672 (weights rotated through > 4x L2)
    for M in (1, 4):
        packed, steps, zeros = wq.wq_quantize_pack(dt(big.W), bits=4, group_size=32)
        nc = max(2, math.ceil(4 * L2_BYTES / (28672 * 8192 // 2)))
        qs = [(packed, steps, zeros)] + [tuple(t.clone() for t in (packed, steps, zeros)) for _ in range(nc - 1)]
        qx, mult = wq.wq_quantize_act_int8(dt(synth.smallm_activations(M)), group_size=32)
        Y = torch.empty((M, 28672), dtype=torch.float16, device=dev)
        fns = [lambda q=q: wq.wq_w4a8_gemm(qx, mult, *q, 28672, group_size=32, out=Y) for q in qs]
        ms = _time_graph(torch, fns) / nc
        by = 28672 * 8192 // 2 + 28672 * (8192 // 32) * 4 + M * 8192 * 5 + M * 28672 * 2
        rows[f"w4a8_g32_M{M}_8192x28672"] = {"us": ms * 1e3, "GB/s": by / (ms * 1e-3) / 1e9,
                                             "frac_hbm": by / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
        del qs

    # GPTQ (fp64 Hessian, factorizations, column loop with error feedback)
    # on LLaMA-2-7B-shaped linears with 512 calibration tokens, 4-bit g128
    for name, N, K in (("q_proj", 4096, 4096), ("gate_proj", 11008, 4096)):
        g0 = synth.rng(90)
        Wg = dt(synth.weight(g0, N, K, 0.02))
        Xg = dt(synth.activations(g0, 512, K, channel_frac=0.01, channel_mult=20.0))
        wsg = torch.empty(wq.wq_gptq_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
        wq.wq_gptq_quantize_pack(Wg, Xg, workspace=wsg)
        torch.cuda.synchronize()
        a.record()
        wq.wq_gptq_quantize_pack(Wg, Xg, workspace=wsg)
        b.record()
        torch.cuda.synchronize()
        assert wq.wq_get_last_device_error() == 0
        rows[f"gptq_llama7b_{name}_T512_w4"] = {"ms": a.elapsed_time(b), "N": N, "K": K,
                                                "workspace_MB": wsg.numel() / 1e6}
        del wsg

    # AWQ scale folding over the block: s_qkv into the first norm's weight,
    # s_o into v_proj's rows, s_gate_up into the second norm's weight,
    # s_down into up_proj's rows (fp16 in, fp16 out: 4 bytes per element)
    g0 = synth.rng(77)
    gam = dt((1.0 + 0.1 * g0.standard_normal(4096)).astype(np.float16))
    sv = dt(np.exp(0.3 * g0.standard_normal(11008)).astype(np.float16))
    Wv, Wu = block[2]["W"], block[5]["W"]
    outv, outu, outg = torch.empty_like(Wv), torch.empty_like(Wu), torch.empty_like(gam)
    fns = [lambda: wq.wq_awq_fold_norm(gam, sv[:4096], out=outg),
           lambda: wq.wq_awq_fold_linear_rows(Wv, sv[:4096], out=(outv, None)),
           lambda: wq.wq_awq_fold_norm(gam, sv[:4096], out=outg),
           lambda: wq.wq_awq_fold_linear_rows(Wu, sv, out=(outu, None))]
    fms = _time_graph(torch, fns)
    fby = 4 * (2 * 4096 + Wv.numel() + Wu.numel())
    assert wq.wq_get_last_device_error() == 0
    rows["awq_fold_llama7b_block"] = {"us": fms * 1e3, "GB/s": fby / (fms * 1e-3) / 1e9,
                                      "frac_hbm": fby / (fms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    return rows


def _oracle_rows(task):
    """Oracle GEMV of one block of output rows (unpack, fp64 dequantize, fp64
    matmul); a process-pool task of the all-cores baseline."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_limits
        lim = threadpool_limits(limits=1)
    except ImportError:  # pragma: no cover
        lim = None
    X, words, st, z, K, reps = task
    for _ in range(reps):
        O.gemm_ref(X, O.unpack_codes(words, 4, K), st, z, 128)
    if lim is not None:
        lim.__exit__(None, None, None)
    return reps


def _oracle_sample(cases, frac: int):
    """The first 1/frac of each linear's output rows, quantized and packed by
    the oracle: (X, packed words, steps, zeros, rows, K) per linear."""
    import oracle as O
    out = []
    for c in cases:
        N, K = c.W.shape
        rows = max(1, N // frac)
        codes, st, z = O.quantize_groups(c.W[:rows], 4, 128, False)
        out.append((c.X, O.pack_codes(codes, 4), st, z, rows, K))
    return out


class OraclePool:
    """The oracle GEMV over output rows on every host core: a spawn-started
    process pool (safe after CUDA initialisation), one row block per core and
    linear. Every worker runs the oracle single-threaded."""

    def __init__(self):
        import multiprocessing as mp
        self.cores = os.cpu_count() or 1
        self.pool = mp.get_context("spawn").Pool(self.cores)

    def run(self, prepared, reps: int) -> int:
        tasks = []
        for X, words, st, z, rows, K in prepared:
            bounds = np.linspace(0, rows, self.cores + 1).astype(int)
            for a, b in zip(bounds[:-1], bounds[1:]):
                if b > a:
                    tasks.append((X, words[a:b], st[a:b], z[a:b], K, reps))
        self.pool.map(_oracle_rows, tasks, chunksize=1)
        return sum(gemm_bytes(1, rows, K, 4) for _, _, _, _, rows, K in prepared) * reps

    def close(self):
        self.pool.close()
        self.pool.join()


def cpu_baseline(cases, seconds: float):
    """The oracle (numpy, fp64 dequantize + matmul), as it stands, on a sample of
    each linear's output rows: single-threaded, and over output rows on every
    host core, each for about `seconds`."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:  # pragma: no cover
        threadpool_limits = None
    frac = 16
    prepared = _oracle_sample(cases, frac)
    ctx = threadpool_limits(limits=1) if threadpool_limits else None
    t0 = time.perf_counter()
    done_bytes, reps = 0, 0
    if ctx:
        ctx.__enter__()
    try:
        while True:
            for X, words, st, z, rows, K in prepared:
                codes = O.unpack_codes(words, 4, K)
                O.gemm_ref(X, codes, st, z, 128)
                done_bytes += gemm_bytes(1, rows, K, 4)
            reps += 1
            if time.perf_counter() - t0 >= seconds:
                break
    finally:
        if ctx:
            ctx.__exit__(None, None, None)
    el = time.perf_counter() - t0
    one = done_bytes / el / 1e9
    pool = OraclePool()
    try:
        pool.run(prepared, 1)  # workers started and warm
        t0 = time.perf_counter()
        by = pool.run(prepared, reps)
        el_all = time.perf_counter() - t0
    finally:
        pool.close()
    sample = f"1/{frac} of the output rows of each of the 7 linears (unpack + fp64 dequantize + fp64 matmul)"
    return {"value": round(by / el_all / 1e9, 4), "unit": "GB/s", "cores": pool.cores, "kind": "oracle",
            "sample": f"{sample}, {reps} passes in {el_all:.1f} s over output rows on {pool.cores} host cores "
                      f"(spawned processes, one thread each)",
            "single_thread": {"value": round(one, 4), "unit": "GB/s", "cores": 1,
                              "sample": f"{sample}, {reps} passes in {el:.1f} s, one thread"}}


def _oracle_gemv_task(task):
    """Oracle GEMV of one block of output rows, `reps` times (one thread)."""
    import oracle as O
    from threadpoolctl import threadpool_limits
    X, words, st, z, K, bits, reps = task
    with threadpool_limits(limits=1):
        for _ in range(reps):
            O.gemm_ref(X, O.unpack_codes(words, bits, K), st, z, 128)
    return reps


def oracle_table(path: str):
    """The oracle, as it stands, timed on the host cores for each workload of
    the result table: one thread, and over output rows on every core (one
    single-threaded spawned process per core; the AWQ search over numpy's own
    BLAS threads). Each cell runs on a sample of output rows and is scaled to
    the whole workload by the sampled fraction (every step is linear in the
    rows). Writes milliseconds per workload to `path`."""
    import multiprocessing as mp

    import oracle as O
    import synth
    from threadpoolctl import threadpool_limits
    cores = os.cpu_count() or 1
    pool = mp.get_context("spawn").Pool(cores)
    out = {"cores": cores, "unit": "ms per workload (scaled from the sampled rows)", "cells": {}}

    def gemv_cell(name, cases, bits, frac):
        prepared = []
        for X, W in cases:
            N, K = W.shape
            rows = max(1, N // frac)
            codes, st, z = O.quantize_groups(W[:rows], bits, 128, False)
            prepared.append((X, O.pack_codes(codes, bits), st, z, rows, K))
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            for X, words, st, z, rows, K in prepared:
                O.gemm_ref(X, O.unpack_codes(words, bits, K), st, z, 128)
            one = time.perf_counter() - t0
        tasks = []
        for X, words, st, z, rows, K in prepared:
            b = np.linspace(0, rows, cores + 1).astype(int)
            tasks += [(X, words[i:j], st[i:j], z[i:j], K, bits, 1) for i, j in zip(b[:-1], b[1:]) if j > i]
        pool.map(_oracle_gemv_task, tasks, chunksize=1)  # workers warm
        t0 = time.perf_counter()
        pool.map(_oracle_gemv_task, tasks, chunksize=1)
        allc = time.perf_counter() - t0
        out["cells"][name] = {"one_core_ms": one * frac * 1e3, "all_cores_ms": allc * frac * 1e3,
                              "sample": f"1/{frac} of the output rows"}
        print(name, out["cells"][name], flush=True)

    try:
        c1 = synth.config_small_linear(0)
        gemv_cell("small_linear_K256_N128_M1_w4", [(c1.X, c1.W)], 4, 1)
        gemv_cell("llama2_7b_block_M1_w4", [(c.X, c.W) for c in synth.config_llama7b_decode(1)], 4, 16)
        for bits in (4, 3):
            c = synth.config_llama65b_decode(bits)
            gemv_cell(f"llama65b_8192x8192_M1_w{bits}", [(c.X, c.W)], bits, 32)
        W = synth.config_smallm_sweep(1).W
        for M in synth.SMALLM_SWEEP:
            gemv_cell(f"smallm_8192x28672_M{M}_w4", [(synth.smallm_activations(M), W)], 4, 64)
        # AWQ search over the block: every search place on 1/16 of its rows
        frac = 16
        places = [(X, [Wl[: max(1, Wl.shape[0] // frac)] for _, Wl in named])
                  for _, X, named in synth.config_awq_block(5)]
        cell = {}
        for label, lim in (("one_core_ms", 1), ("all_cores_ms", None)):
            with threadpool_limits(limits=lim):
                t0 = time.perf_counter()
                for X, Ws in places:
                    O.awq_search(X, Ws, 4, 128, False)
                cell[label] = (time.perf_counter() - t0) * frac * 1e3
        cell["sample"] = f"1/{frac} of the output rows of every search place; all cores = numpy's BLAS threads"
        out["cells"]["awq_search_llama7b_block_w4"] = cell
        print("awq_search_llama7b_block_w4", cell, flush=True)
    finally:
        pool.close()
        pool.join()
    with open(path, "w") as f:
        json.dump(out, f, indent=1)


# ---------------------------------------------------------------------------
# reference arm: the oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args, rank: int, world: int):
    """The reference arm: the oracle as it stands, over output rows on every
    host core (one single-threaded process per core), on a sample of each
    linear's rows sized so the whole run takes about --ref-seconds."""
    if rank != 0:
        return None
    import oracle as O
    import synth
    cases = synth.config_llama7b_decode(1)
    budget = float(args.ref_seconds)
    pool = OraclePool()
    try:
        # calibrate the sample so the whole run fits the budget
        probe = _oracle_sample(cases, 64)
        pool.run(probe, 1)
        t0 = time.perf_counter()
        pool.run(probe, 1)
        per_step_1_64 = time.perf_counter() - t0
        steps_total = args.steps + args.warmup
        frac = max(1, int(math.ceil(64 * steps_total * per_step_1_64 / budget)))
        frac = 1 << max(0, (frac - 1).bit_length())  # a power of two >= the estimate
        prepared = _oracle_sample(cases, frac) if frac != 64 else probe
        for _ in range(args.warmup):
            pool.run(prepared, 1)
        t0 = time.perf_counter()
        by = 0
        for _ in range(args.steps):
            by += pool.run(prepared, 1)
        el = time.perf_counter() - t0
    finally:
        pool.close()
    value = by / el / 1e9
    sample = (f"1/{frac} of the output rows of each of the 7 linears per step (unpack + fp64 dequantize + fp64 "
              f"matmul), over output rows on {pool.cores} host cores (spawned processes, one thread each)")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 5),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": el * 1e3 / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "parallelism": "host cores (rank 0 only)"},
        "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": pool.cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------
# single-case mode (a small, bounded run of one kernel, e.g. under ncu)
# ---------------------------------------------------------------------------

def run_case(args):
    import torch

    from weight_only_quantization_group_b200 import build
    build.build()
    import weight_only_quantization_group_b200 as wq
    import synth

    dev = torch.device("cuda", 0)
    g = synth.rng(77)
    W = torch.from_numpy(synth.weight(g, args.N, args.K, 0.02)).to(dev)
    X = torch.from_numpy(synth.activations(g, args.M, args.K)).to(dev)
    opts = {"auto": wq.WQ_PATH_AUTO, "gemv": wq.WQ_PATH_GEMV, "tc": wq.WQ_PATH_TENSOR_CORE}
    wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, opts[args.path])
    wq.wq_set_option(wq.WQ_OPT_GEMV_VARIANT, {"int": wq.WQ_GEMV_INT_DIGITS, "exact": wq.WQ_GEMV_EXACT}.get(
        args.gemv_variant, wq.WQ_GEMV_OFFSET_SUMS))
    wq.wq_set_option(wq.WQ_OPT_GEMV_KERNEL, wq.WQ_GEMV_KERNEL_TILED if args.gemv_variant == "tiled"
                     else wq.WQ_GEMV_KERNEL_AUTO)
    wq.wq_set_option(wq.WQ_OPT_GEMV_ROWS_SHAPE, args.rows_shape)
    wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, wq.WQ_AWQ_LOSS_TWO_KERNELS if args.awq_loss == "two"
                     else wq.WQ_AWQ_LOSS_FUSED)
    q = wq.wq_quantize_pack(W, bits=args.bits, group_size=args.group)
    Y = torch.empty((args.M, args.N), dtype=torch.float16, device=dev)
    ws = None
    if args.case == "gemm" and args.workspace:
        n = wq.wq_gemm_workspace_bytes(args.M, args.N, args.K, bits=args.bits, group_size=args.group)
        ws = torch.zeros(max(n, 1), dtype=torch.uint8, device=dev) if n else None
    if args.case == "awq":  # M calibration rows, one linear of N outputs, 20 alphas
        ws = torch.empty(wq.wq_awq_workspace_bytes(args.M, args.K, [args.N], 20, bits=args.bits),
                         dtype=torch.uint8, device=dev)
    if args.case == "gptq":  # M calibration rows
        ws = torch.empty(wq.wq_gptq_workspace_bytes(args.N, args.K, bits=args.bits, group_size=args.group),
                         dtype=torch.uint8, device=dev)
    if args.case == "w4a8":
        qx, mult = wq.wq_quantize_act_int8(X, group_size=args.group)
    if args.case == "fold":
        sv = torch.from_numpy(synth.activations(g, 1, args.N, std=0.2).reshape(-1)).abs().add_(0.5).to(dev)
        Wo = torch.empty_like(W)
    torch.cuda.synchronize()
    times = []
    for _ in range(args.reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        if args.case == "gemm":
            wq.wq_w4a16_gemm(X, *q, args.N, bits=args.bits, group_size=args.group, out=Y, workspace=ws)
        elif args.case == "awq":
            wq.wq_awq_scale_search(X, [W], bits=args.bits, workspace=ws)
        elif args.case == "gptq":
            wq.wq_gptq_quantize_pack(W, X, bits=args.bits, group_size=args.group, workspace=ws, out=q)
        elif args.case == "w4a8":
            wq.wq_w4a8_gemm(qx, mult, *q, args.N, group_size=args.group, out=Y)
        elif args.case == "fold":
            wq.wq_awq_fold_linear_rows(W, sv, out=(Wo, None))
        else:
            wq.wq_quantize_pack(W, bits=args.bits, out=q)
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) * 1e3)
    st = wq.wq_get_last_device_error()
    print(json.dumps({"case": args.case, "M": args.M, "N": args.N, "K": args.K, "bits": args.bits,
                      "path": args.path, "us": times, "device_status": st}))
    if st != 0:
        sys.exit(1)


# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row measurements")
    ap.add_argument("--rows-out", default=None, help="also write the per-row measurements to this JSON file")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch eagerly instead of replaying CUDA graphs")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-seconds", type=float, default=60.0)
    ap.add_argument("--case", choices=["gemm", "quantize", "awq", "gptq", "w4a8", "fold"], default=None,
                    help="run one small kernel configuration --reps times (for profiling)")
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--N", type=int, default=8192)
    ap.add_argument("--K", type=int, default=8192)
    ap.add_argument("--bits", type=int, default=4)
    ap.add_argument("--group", type=int, default=128)
    ap.add_argument("--workspace", action="store_true", help="--case gemm: pass the GEMM workspace")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--path", choices=["auto", "gemv", "tc"], default="auto")
    ap.add_argument("--gemv-variant", choices=["int", "offset", "exact", "tiled"], default="offset")
    ap.add_argument("--rows-shape", type=int, default=0, choices=list(range(5)))
    ap.add_argument("--awq-loss", choices=["fused", "two"], default="fused",
                    help="--case awq: loss GEMM with on-chip error tiles, or error matrix + loss GEMM")
    ap.add_argument("--oracle-table", default=None,
                    help="only time the oracle on the host cores for each workload of the result table "
                         "and write the milliseconds to this JSON file")
    args = ap.parse_args()
    if args.oracle_table:
        oracle_table(args.oracle_table)
        return
    if args.case:
        run_case(args)
        return
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line, rows = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if line is not None:
        if rows:
            # the other hot-path rows: their own line (and file), so that the
            # last line stays a compact headline
            if args.rows_out:
                with open(args.rows_out, "w") as f:
                    json.dump(rows, f, indent=1)
            print(json.dumps({"rows": rows}), flush=True)
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
