"""Benchmark of the Atom W4A4 hot path on B200.

One step = the online path of one quantized linear layer over one batch:
atom_reorder_quant of the fp16 activations (reorder + INT4/INT8 quantize) then
atom_w4a4_gemm against weights quantized once beforehand (the weights are
quantized offline in the method, so their quantization is outside the step).

Workload: the Llama-70B-shaped MLP up-projection, A fp16 [8192, 8192]
(Student-t(4), 128 outlier channels x30), W fp16 [28672, 8192] (N(0, 0.01)),
seeded synthetic inputs (w4a4_mixed_precision_b200.inputs).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl atom|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs its own batch against
its own replica of the quantized weights: there is no data exchange on the
path, so the scaling is weak and `value` sums the ranks' work over the slowest
rank's time. `--impl reference` times the CPU oracle (test infrastructure) on
the host cores on a bounded row sample of the same workload.
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
sys.path.insert(0, ROOT)

WORKLOAD_INDEX = 4
METRIC = "W4A4 GEMM TOPS and % int tensor peak; quantize GB/s and % HBM (1 B200)"
INT8_OVER_BF16 = 2.0     # nominal dense int8 : bf16 tensor throughput on B200 (4.5 : 2.25 P)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def _kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "w4a4_mixed_precision_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


L2_BYTES = 126e6


def _l2_note(w) -> str:
    """How the workload's bytes compare with the 126 MB L2 (timing-hygiene note)."""
    a_mb = w.M * w.K * 2 / 1e6
    w_mb = w.N * ((w.K - 128) // 2 + 128 + 4 * (w.K // 128)) / 1e6
    y_mb = w.M * w.N * 2 / 1e6
    if max(a_mb, y_mb) * 1e6 > L2_BYTES:
        return (f"larger than L2: each step reads A fp16 {a_mb:.0f} MB and writes Y {y_mb:.0f} MB "
                f"(packed W {w_mb:.0f} MB), which evicts L2 between steps")
    if (a_mb + w_mb + y_mb) * 1e6 > L2_BYTES:
        return (f"A fp16 {a_mb:.1f} MB, packed W {w_mb:.1f} MB and Y {y_mb:.1f} MB: more than L2 in "
                f"total, but part of it may stay in L2 between steps")
    return (f"small case: A fp16 {a_mb:.1f} MB, packed W {w_mb:.1f} MB and Y {y_mb:.1f} MB fit in "
            f"L2, so its timings are warm-L2 (a parity and profiling case, not a bench line)")


def _profiled_traffic(kernel: str):
    """DRAM bytes per launch (read + write) from the committed ncu summary
    profiles/traffic.md, if it was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    try:
        with open(path) as f:
            lines = f.read().splitlines()
    except OSError:
        return None
    for line in lines:
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 5 and cells[0] == kernel:
            if cells[1] != _kernel_source_hash():
                return None
            try:
                return int(cells[4])
            except ValueError:
                return None
    return None


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._period = period_s
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:                                   # noqa: BLE001 (no NVML: no clocks)
            self._h = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                bits = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:                               # noqa: BLE001
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._h is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._h is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- CPU oracle


def cpu_oracle_run(w, A, W, idx, budget_s: float, min_rows: int = 8):
    """Times the CPU oracle on a growing row sample of the workload until the
    sample takes at least `budget_s`; returns (ops_per_s, rows, seconds, cores)."""
    from oracle import c_oracle
    cores = len(os.sched_getaffinity(0))
    c_oracle.set_threads(cores)
    qw = c_oracle.quantize(W, idx)                      # offline weights, not timed
    rows = min_rows
    while True:
        t0 = time.perf_counter()
        qa = c_oracle.quantize(np.ascontiguousarray(A[:rows]), idx)
        c_oracle.gemm(*qa, *qw, w.K)
        dt = time.perf_counter() - t0
        if dt >= budget_s or rows >= w.M:
            break
        rows = min(w.M, max(rows * 2, int(rows * budget_s / max(dt, 1e-3) * 1.1)))
    return 2.0 * rows * w.N * w.K / dt, rows, dt, cores


# ----------------------------------------------------------------------------- per-config legs


def _time_cycle(fns, n, stream):
    """Average ms per call of `fns` called round-robin n times back to back on
    `stream` (three untimed calls first), timed with CUDA events on that stream."""
    import torch
    for i in range(3):
        fns[i % len(fns)]()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        fns[i % len(fns)]()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n


def _time_graph(fns, n, stream):
    """Average ms per call of the same round-robin sequence of n calls, captured
    once in a CUDA graph on `stream` and replayed (one untimed replay first):
    the device time of the calls without the host's per-call launch cost."""
    import torch
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            fns[i % len(fns)]()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):   # replay() launches on the current stream
        g.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    del g
    return ms


def _copies_for(bytes_per_set: float, cap: int = 16) -> int:
    """Input sets to rotate through so that consecutive calls never find their
    operands in the 126 MB L2 (at least two sets, and more than twice L2)."""
    return int(min(cap, max(2, -(-2 * L2_BYTES // max(bytes_per_set, 1)))))


def int8_probe_tops(stream, groups: int = 4096, reps: int = 5):
    """Dense INT8 tensor-core rate measured by the library's probe loop
    (atom_probe_mma_i8: the GEMM's 2-SM MMA shape back to back, no data
    movement); the median of `reps` timed launches after two untimed ones."""
    import torch
    from w4a4_mixed_precision_b200 import atom
    ops = 0
    for _ in range(2):
        ops = atom.atom_probe_mma_i8(groups, stream=stream)
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        atom.atom_probe_mma_i8(groups, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    if atom.atom_device_status(clear=True) != 0:
        raise RuntimeError("device status set by the INT8 probe")
    return ops / (ms * 1e-3) / 1e12, ms


def per_config_legs(configs, dev, stream, n_calls, int8_peak, int8_probe, hbm_gbs):
    """Throughput of the other Llama-shaped workloads, each on its own seeded
    inputs, with input sets rotated so that no call finds its operands in L2:
    the decode GEMM (latency and GB/s of its algorithmic bytes against HBM), the
    prefill and down-projection GEMMs (TOPS against the int8 denominators), the
    quantizer (GB/s against HBM), and fp16 cuBLAS of the same shape beside each."""
    import torch
    from w4a4_mixed_precision_b200 import atom, inputs
    out = {}
    for c in configs:
        w = inputs.workload(c)
        Kd, G = w.K - 128, w.K // 128
        A_h, W_h, idx_h = inputs.activations(c), inputs.weights(c), inputs.outlier_channels(c)
        A = torch.from_numpy(A_h.view(np.uint16)).to(dev).view(torch.float16)
        W16 = torch.from_numpy(W_h.view(np.uint16)).to(dev).view(torch.float16)
        idx = torch.from_numpy(idx_h).to(dev)
        del A_h, W_h
        qw0 = atom.atom_quant_weights(W16, idx)
        qa0 = atom.atom_reorder_quant(A, idx)
        packed_row = Kd // 2 + 128 + 4 * G
        gemm_bytes = (w.M + w.N) * packed_row + w.M * w.N * 2
        quant_bytes = w.M * (2 * w.K + packed_row)
        ops = 2.0 * w.M * w.N * w.K
        n_sets = _copies_for(gemm_bytes)
        qas = [qa0] + [atom.Quantized(*(t.clone() for t in qa0)) for _ in range(n_sets - 1)]
        qws = [qw0] + [atom.Quantized(*(t.clone() for t in qw0)) for _ in range(n_sets - 1)]
        ys = [torch.empty((w.M, w.N), dtype=torch.float16, device=dev) for _ in range(n_sets)]
        wss = [atom.gemm_workspace(w.M, w.N, w.K, dev) for _ in range(n_sets)]

        gs = torch.cuda.Stream()   # graph capture needs a stream other than the default one

        def gemm_fn(i, st):
            return lambda: atom.atom_w4a4_gemm(qas[i], qws[i], w.K, y=ys[i], stream=st,
                                               workspace=wss[i])
        g_ms = _time_cycle([gemm_fn(i, stream) for i in range(n_sets)], n_calls, stream)
        g_ms_graph = _time_graph([gemm_fn(i, gs) for i in range(n_sets)], n_calls, gs)
        n_qsets = _copies_for(quant_bytes)
        As = [A] + [A.clone() for _ in range(n_qsets - 1)]
        qouts = [atom.empty_quantized(w.M, w.K, dev) for _ in range(n_qsets)]

        def quant_fn(i, st):
            return lambda: atom.atom_reorder_quant(As[i], idx, out=qouts[i], stream=st)
        q_ms = _time_cycle([quant_fn(i, stream) for i in range(n_qsets)], n_calls, stream)
        q_ms_graph = _time_graph([quant_fn(i, gs) for i in range(n_qsets)], n_calls, gs)

        # one layer's online step: quantize A, then the GEMM on those codes
        def step_fn(i, st):
            qo, j = qouts[i % n_qsets], i % n_sets

            def f():
                atom.atom_reorder_quant(As[i % n_qsets], idx, out=qo, stream=st)
                atom.atom_w4a4_gemm(qo, qws[j], w.K, y=ys[j], stream=st, workspace=wss[j])
            return f
        st_ms_graph = _time_graph([step_fn(i, gs) for i in range(max(n_sets, n_qsets))],
                                  n_calls, gs)
        del As, qouts, qas, ys, wss
        n_csets = _copies_for(2.0 * (w.M + w.N) * w.K + 2.0 * w.M * w.N)
        Ws = [W16] + [W16.clone() for _ in range(n_csets - 1)]
        yc = torch.empty((w.M, w.N), dtype=torch.float16, device=dev)
        c_fns = [(lambda Wi: (lambda: torch.matmul(A, Wi.t(), out=yc)))(Wi) for Wi in Ws]
        c_ms = _time_cycle(c_fns, n_calls, stream)
        with torch.cuda.stream(gs):
            c_ms_graph = _time_graph(c_fns, n_calls, gs)
        del Ws, yc, W16, A
        if atom.atom_device_status(clear=True) != 0:
            raise RuntimeError(f"device status set on workload {c}")
        g_tops = ops / (g_ms * 1e-3) / 1e12
        entry = {
            "workload": f"{w.name} M={w.M} N={w.N} K={w.K}",
            "gemm_us": round(g_ms * 1e3, 2),
            "gemm_us_graph": round(g_ms_graph * 1e3, 2),
            "gemm_gbs_graph": round(gemm_bytes / (g_ms_graph * 1e-3) / 1e9, 1),
            "gemm_tops": round(g_tops, 2),
            "gemm_frac_int8_peak": round(g_tops / int8_peak, 4),
            "gemm_frac_int8_probe": round(g_tops / int8_probe, 4) if int8_probe else None,
            "gemm_algorithmic_bytes": gemm_bytes,
            "gemm_gbs": round(gemm_bytes / (g_ms * 1e-3) / 1e9, 1),
            "gemm_frac_hbm": round(gemm_bytes / (g_ms * 1e-3) / 1e9 / hbm_gbs, 4),
            "gemm_splits_workspace_bytes": atom.atom_gemm_workspace_bytes(w.M, w.N, w.K),
            "quant_us": round(q_ms * 1e3, 2),
            "quant_us_graph": round(q_ms_graph * 1e3, 2),
            "step_us_graph": round(st_ms_graph * 1e3, 2),
            "quant_bytes": quant_bytes,
            "quant_gbs": round(quant_bytes / (q_ms * 1e-3) / 1e9, 1),
            "quant_frac_hbm": round(quant_bytes / (q_ms * 1e-3) / 1e9 / hbm_gbs, 4),
            "fp16_cublas_us": round(c_ms * 1e3, 2),
            "fp16_cublas_us_graph": round(c_ms_graph * 1e3, 2),
            "fp16_cublas_tflops": round(ops / (c_ms * 1e-3) / 1e12, 2),
            "w4a4_gemm_speedup_vs_fp16": round(c_ms / g_ms, 3),
            "calls": n_calls,
            "timing": "*_us: CUDA events around `calls` calls issued back to back from Python "
                      "(host launch cost included); *_us_graph: the same calls captured in one "
                      "CUDA graph and replayed (device time per call); step_us_graph: quantize "
                      "then GEMM, one layer's online step, per step in a graph",
            "l2": f"GEMM rotates {n_sets} input sets, quantizer {n_qsets}, cuBLAS {n_csets} "
                  f"weight copies (each rotation more than twice the 126 MB L2, or 16 sets)",
            "bound": "hbm" if c == 1 else "tensor",
        }
        out[w.name] = entry
    return out


# ----------------------------------------------------------------------------- main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["atom", "reference"], default="atom")
    ap.add_argument("--workload", type=int, default=WORKLOAD_INDEX)
    ap.add_argument("--cpu-budget", type=float, default=10.0,
                    help="seconds of CPU oracle work for the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cublas", action="store_true",
                    help="skip the fp16 cuBLAS GEMM of the same shape reported beside the result")
    ap.add_argument("--no-w8a8", action="store_true",
                    help="skip the W8A8 comparator GEMM (and torch._int_mm) of the same shape")
    ap.add_argument("--no-w4a8", action="store_true",
                    help="skip the W4A8 variant (INT8 activations, the same INT4 weights)")
    ap.add_argument("--no-gemm-quant", action="store_true",
                    help="skip the GEMM with the next layer's quantization in its epilogue")
    ap.add_argument("--no-kv", action="store_true",
                    help="skip the INT4 KV-cache quantize/dequantize measurement")
    ap.add_argument("--m", type=int, default=None,
                    help="use only the first M activation rows (small profiling cases)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the decode / prefill / down-projection workloads (1, 2, 3)")
    ap.add_argument("--no-probe", action="store_true",
                    help="skip the INT8 tensor-core peak probe (second GEMM denominator)")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    from w4a4_mixed_precision_b200 import inputs
    w = inputs.workload(args.workload)
    if args.m is not None:
        import dataclasses
        w = dataclasses.replace(w, M=args.m, name=f"{w.name}_m{args.m}")
    workload_cfg = {"workload": f"{w.name} M={w.M} N={w.N} K={w.K}", "M": w.M, "N": w.N, "K": w.K,
                    "group": 128, "n_outlier": 128, "activations": w.describe(),
                    "parallelism": f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU",
                    "l2": _l2_note(w)}

    if args.impl == "reference":
        return run_reference(args, w, workload_cfg, rank)

    import torch
    import torch.distributed as dist
    from w4a4_mixed_precision_b200 import atom, parallel

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    A_h = inputs.activations(args.workload, rows=w.M)
    W_h = inputs.weights(args.workload)
    idx_h = inputs.outlier_channels(args.workload)

    A = torch.from_numpy(A_h.view(np.uint16)).to(dev).view(torch.float16)
    idx = torch.from_numpy(idx_h).to(dev)
    qw = atom.atom_quant_weights(torch.from_numpy(W_h.view(np.uint16)).to(dev).view(torch.float16),
                                 idx)
    qa = atom.empty_quantized(w.M, w.K, dev)
    y = torch.empty((w.M, w.N), dtype=torch.float16, device=dev)
    torch.cuda.synchronize()
    atom.atom_device_status(clear=True)

    stream = torch.cuda.current_stream()
    n_steps = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_steps)]

    def step(i=None):
        if i is not None:
            ev[i][0].record(stream)
        atom.atom_reorder_quant(A, idx, out=qa, stream=stream)
        if i is not None:
            ev[i][1].record(stream)
        atom.atom_w4a4_gemm(qa, qw, w.K, y=y, stream=stream)
        if i is not None:
            ev[i][2].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        t_start.record(stream)
        for i in range(n_steps):
            step(i)
        t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    status = atom.atom_device_status(clear=True)
    if status != 0:
        raise RuntimeError(f"device status {atom.STATUS.get(status, status)} during the timed run")

    elapsed_ms = t_start.elapsed_time(t_end)
    quant_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(n_steps)]
    gemm_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(n_steps)]

    # the quantizer alone: 20 launches back to back on two alternating inputs
    # (each larger than L2), with no GEMM in between whose Y write-backs share
    # the quantizer's HBM time
    A2, qa2 = A.clone(), atom.empty_quantized(w.M, w.K, dev)
    quant_alone_ms = _time_cycle(
        [lambda: atom.atom_reorder_quant(A, idx, out=qa, stream=stream),
         lambda: atom.atom_reorder_quant(A2, idx, out=qa2, stream=stream)], 20, stream)
    del A2, qa2
    elapsed_ms = parallel.max_over_ranks(elapsed_ms, dev)   # the slowest rank's time

    # -------- end-to-end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        # Consecutive steps overlap: the host-to-device copy of step i+1 and the
        # device-to-host copy of step i-1 run on their own streams while step i
        # computes; device buffers alternate between two sets, and events keep
        # each buffer from being overwritten before its previous use is done.
        A_pin = torch.from_numpy(A_h.view(np.uint16)).view(torch.float16).pin_memory()
        y_pin = [torch.empty((w.M, w.N), dtype=torch.float16).pin_memory() for _ in range(2)]
        a_dev = [torch.empty_like(A) for _ in range(2)]
        qa2 = [qa, atom.empty_quantized(w.M, w.K, dev)]
        y2 = [y, torch.empty_like(y)]
        s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
        ev_h2d = [torch.cuda.Event() for _ in range(2)]
        ev_quant = [torch.cuda.Event() for _ in range(2)]
        ev_gemm = [torch.cuda.Event() for _ in range(2)]
        ev_d2h = [torch.cuda.Event() for _ in range(2)]
        e2e_steps = max(10, min(20, n_steps // 2))

        def e2e_step(i):
            b = i % 2
            s_h2d.wait_event(ev_quant[b])       # a_dev[b]'s previous contents are quantized
            with torch.cuda.stream(s_h2d):
                a_dev[b].copy_(A_pin, non_blocking=True)
            ev_h2d[b].record(s_h2d)
            stream.wait_event(ev_h2d[b])
            atom.atom_reorder_quant(a_dev[b], idx, out=qa2[b], stream=stream)
            ev_quant[b].record(stream)
            stream.wait_event(ev_d2h[b])        # y2[b] of two steps ago has been copied out
            atom.atom_w4a4_gemm(qa2[b], qw, w.K, y=y2[b], stream=stream)
            ev_gemm[b].record(stream)
            s_d2h.wait_event(ev_gemm[b])
            with torch.cuda.stream(s_d2h):
                y_pin[b].copy_(y2[b], non_blocking=True)
            ev_d2h[b].record(s_d2h)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_h2d.wait_event(e0)
        s_d2h.wait_event(e0)
        for i in range(e2e_steps):
            e2e_step(i)
        stream.wait_event(ev_d2h[(e2e_steps - 1) % 2])   # the last result is on the host
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / e2e_steps
        e2e_ms = parallel.max_over_ranks(e2e_ms, dev)
        e2e = {"value": round(2.0 * w.M * w.N * w.K * world / (e2e_ms * 1e-3) / 1e12, 2),
               "unit": "TOPS", "h2d_bytes_per_step": A_h.nbytes,
               "d2h_bytes_per_step": w.M * w.N * 2, "ms_per_step": round(e2e_ms, 4),
               "steps": e2e_steps,
               "pipelining": "host-to-device copy, compute and device-to-host copy of "
                             "consecutive steps on three streams, two device buffer sets"}

    # The library's own legs run first, before the dense library comparators,
    # which leave the GPU at its power cap for a while.
    # -------- the GEMM with the next layer's activation quantization in its epilogue
    # (atom_w4a4_gemm_quant), against the unfused pair it replaces: the unsplit GEMM
    # to fp16 Y, then atom_reorder_quant of Y with its last 128 columns as outliers
    gemm_quant = None
    if not args.no_gemm_quant and w.N % 128 == 0 and w.N >= 256:
        out_f = atom.empty_quantized(w.M, w.N, dev)
        out_u = atom.empty_quantized(w.M, w.N, dev)
        y_u = torch.empty((w.M, w.N), dtype=torch.float16, device=dev)
        tail = torch.arange(w.N - 128, w.N, dtype=torch.int32, device=dev)
        n_gq = max(3, min(10, n_steps // 20))

        def time_gq(fn):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(n_gq):
                fn()
            a1.record(stream)
            torch.cuda.synchronize()
            return a0.elapsed_time(a1) / n_gq

        def unfused():
            atom.atom_w4a4_gemm(qa, qw, w.K, y=y_u, stream=stream, split=False)
            atom.atom_reorder_quant(y_u, tail, out=out_u, stream=stream)

        f_ms = time_gq(lambda: atom.atom_w4a4_gemm_quant(qa, qw, w.K, out=out_f, stream=stream))
        u_ms = time_gq(unfused)
        ops = 2.0 * w.M * w.N * w.K
        gemm_quant = {"value": round(ops / (f_ms * 1e-3) / 1e12, 2), "unit": "TOPS",
                      "ms": round(f_ms, 4), "steps": n_gq,
                      "unfused_ms": round(u_ms, 4),
                      "output_bytes": w.M * ((w.N - 128) // 2 + 128 + 4 * (w.N // 128)),
                      "unfused_output_bytes": w.M * w.N * 2,
                      "kind": "atom_w4a4_gemm_quant: the same GEMM writing the next layer's "
                              "INT4/INT8 codes and scales of Y instead of fp16 Y; unfused = "
                              "atom_w4a4_gemm (no K split) then atom_reorder_quant of Y"}
        del out_f, out_u, y_u
        if atom.atom_device_status(clear=True) != 0:
            raise RuntimeError("device status set by the quantizing GEMM")

    # -------- W4A8 variant: INT8 activations in every group, the same INT4 weights
    w4a8 = None
    if not args.no_w4a8:
        qa_a8 = atom.atom_reorder_quant_a8(A, idx, stream=stream)
        y_a8 = torch.empty((w.M, w.N), dtype=torch.float16, device=dev)
        n_a8 = max(3, min(10, n_steps // 20))
        for _ in range(3):
            atom.atom_w4a8_gemm(qa_a8, qw, w.K, y=y_a8, stream=stream)
        torch.cuda.synchronize()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(n_a8):
            atom.atom_w4a8_gemm(qa_a8, qw, w.K, y=y_a8, stream=stream)
        a1.record(stream)
        torch.cuda.synchronize()
        a8_ms = a0.elapsed_time(a1) / n_a8
        w4a8 = {"value": round(2.0 * w.M * w.N * w.K / (a8_ms * 1e-3) / 1e12, 2), "unit": "TOPS",
                "ms": round(a8_ms, 4), "steps": n_a8,
                "kind": "atom_w4a8_gemm: INT8 activations (atom_reorder_quant_a8 of the same A) "
                        "x the same INT4/INT8 weights, fp16 out, no K split"}
        del qa_a8, y_a8
        if atom.atom_device_status(clear=True) != 0:
            raise RuntimeError("device status set by the W4A8 variant")

    # -------- the dense INT8 tensor-core rate (second denominator) and the other workloads
    peaks, peak_kind = _peaks()
    int8_peak = peaks["bf16_tflops"] * INT8_OVER_BF16
    probe = None
    if not args.no_probe:
        probe_tops, probe_ms = int8_probe_tops(stream)
        probe = {"value": round(probe_tops, 1), "unit": "TOPS", "ms": round(probe_ms, 4),
                 "kind": "atom_probe_mma_i8: tcgen05.mma.cta_group::2.kind::i8 M=256 N=256 "
                         "K=32 back to back on every CTA pair (one CTA per SM), zero operands "
                         "in shared memory, no loads or dequantization; median of 5 launches"}
    per_config = None
    if not args.no_per_config and args.m is None and args.workload == WORKLOAD_INDEX:
        with ClockSampler(torch.cuda.current_device()) as pc_clocks:
            per_config = per_config_legs((1, 2, 3), dev, stream, max(10, min(50, n_steps)),
                                         int8_peak, probe["value"] if probe else None,
                                         peaks["hbm_gbs"])
        per_config["clocks"] = pc_clocks.summary()

    # -------- fp16 cuBLAS GEMM of the same shape (torch.matmul), a library baseline
    cublas = None
    if not args.no_cublas:
        W16 = torch.from_numpy(W_h.view(np.uint16)).to(dev).view(torch.float16)
        y16 = torch.empty((w.M, w.N), dtype=torch.float16, device=dev)
        for _ in range(3):
            torch.matmul(A, W16.t(), out=y16)
        torch.cuda.synchronize()
        n_cb = max(3, min(20, n_steps // 10))
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(n_cb):
            torch.matmul(A, W16.t(), out=y16)
        c1.record(stream)
        torch.cuda.synchronize()
        cb_ms = c0.elapsed_time(c1) / n_cb
        cublas = {"value": round(2.0 * w.M * w.N * w.K / (cb_ms * 1e-3) / 1e12, 2),
                  "unit": "TFLOP/s", "ms": round(cb_ms, 4), "steps": n_cb,
                  "kind": "torch.matmul fp16 x fp16 -> fp16 (cuBLAS), same M, N, K, "
                          "operands resident in HBM"}
        del W16, y16

    # -------- W8A8 comparator of the same shape, and torch._int_mm (cuBLASLt int8)
    w8a8 = None
    if not args.no_w8a8:
        qa8_h, qw8_h, sa8_h, sw8_h = inputs.int8_case(4000 + args.workload, w.M, w.N, w.K)
        qa8 = torch.from_numpy(qa8_h).to(dev)
        qw8 = torch.from_numpy(qw8_h).to(dev)
        sa8 = torch.from_numpy(sa8_h).to(dev)
        sw8 = torch.from_numpy(sw8_h).to(dev)
        y8 = torch.empty((w.M, w.N), dtype=torch.float16, device=dev)
        n_w8 = max(3, min(20, n_steps // 10))

        def time_it(fn):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(n_w8):
                fn()
            a1.record(stream)
            torch.cuda.synchronize()
            return a0.elapsed_time(a1) / n_w8

        w8_ms = time_it(lambda: atom.atom_w8a8_gemm(qa8, sa8, qw8, sw8, y=y8, stream=stream))
        mm_ms = time_it(lambda: torch._int_mm(qa8, qw8.t()))
        ops8 = 2.0 * w.M * w.N * w.K
        w8a8 = {"value": round(ops8 / (w8_ms * 1e-3) / 1e12, 2), "unit": "TOPS",
                "ms": round(w8_ms, 4), "steps": n_w8,
                "kind": "atom_w8a8_gemm: int8 x int8, per-row x per-column fp32 scales, fp16 out, "
                        "same M, N, K, seeded uniform int8 operands resident in HBM",
                "torch_int_mm": {"value": round(ops8 / (mm_ms * 1e-3) / 1e12, 2),
                                 "unit": "TOPS", "ms": round(mm_ms, 4),
                                 "kind": "torch._int_mm int8 x int8 -> int32 (cuBLASLt), "
                                         "no scales"}}
        del qa8, qw8, y8
        if atom.atom_device_status(clear=True) != 0:
            raise RuntimeError("device status set by the W8A8 comparator")

    # -------- INT4 KV cache: 131072 tokens x 8 KV heads x head_dim 128 (268 MB fp16)
    kv = None
    if not args.no_kv:
        kv_tokens, kv_heads = 131072, 8
        kv_x = [torch.from_numpy(inputs.kv_cache(5000 + i, kv_tokens, kv_heads).view(np.uint16))
                .to(dev).view(torch.float16) for i in range(2)]
        kv_q = [atom.atom_kv_quant(x, stream=stream) for x in kv_x]
        kv_y = [torch.empty_like(x) for x in kv_x]
        n_kv = max(3, min(20, n_steps // 10))

        def time_kv(fn):
            for i in range(3):
                fn(i)
            torch.cuda.synchronize()
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for i in range(n_kv):
                fn(i)
            a1.record(stream)
            torch.cuda.synchronize()
            return a0.elapsed_time(a1) / n_kv

        q_ms = time_kv(lambda i: atom.atom_kv_quant(kv_x[i % 2], q4=kv_q[i % 2][0],
                                                     scales=kv_q[i % 2][1], stream=stream))
        d_ms = time_kv(lambda i: atom.atom_kv_dequant(kv_q[i % 2][0], kv_q[i % 2][1],
                                                       out=kv_y[i % 2], stream=stream))
        kv_groups = kv_tokens * kv_heads
        kv_bytes = kv_groups * (256 + 64 + 4)   # fp16 vectors + packed codes + scales
        kv = {"shape": f"{kv_tokens} tokens x {kv_heads} heads x 128", "groups": kv_groups,
              "bytes_per_call": kv_bytes,
              "quant": {"value": round(kv_bytes / (q_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                        "ms": round(q_ms, 4)},
              "dequant": {"value": round(kv_bytes / (d_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                          "ms": round(d_ms, 4)},
              "l2": "two caches of 268 MB alternate, larger than L2"}
        del kv_x, kv_q, kv_y
        if atom.atom_device_status(clear=True) != 0:
            raise RuntimeError("device status set by the KV-cache kernels")

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    ops = 2.0 * w.M * w.N * w.K
    ms_per_step = elapsed_ms / n_steps
    value = ops * world / (ms_per_step * 1e-3) / 1e12
    gemm_avg = statistics.mean(gemm_ms)
    quant_avg = statistics.mean(quant_ms)
    gemm_tops = ops / (gemm_avg * 1e-3) / 1e12
    Kd = w.K - 128
    quant_bytes = w.M * (2 * w.K + Kd // 2 + 128 + 4 * (w.K // 128))
    quant_gbs = quant_bytes / (quant_avg * 1e-3) / 1e9
    gemm_bytes = (w.M + w.N) * (Kd // 2 + 128 + 4 * (w.K // 128)) + w.M * w.N * 2

    # profiles/traffic.md was captured on the full default workload only
    profiled_shape = args.workload == WORKLOAD_INDEX and args.m is None
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": n_steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic (seeded; see w4a4_mixed_precision_b200/inputs.py)",
        "config": workload_cfg,
        "gemm_tops": round(gemm_tops, 2),
        "gemm_frac_int8_peak": round(gemm_tops / int8_peak, 4),
        "gemm_frac_int8_probe": round(gemm_tops / probe["value"], 4) if probe else None,
        "quant_gbs": round(quant_gbs, 1),
        "quant_frac_hbm": round(quant_gbs / peaks["hbm_gbs"], 4),
        "kernel_ms": {"reorder_quant": round(quant_avg, 4), "w4a4_gemm": round(gemm_avg, 4)},
        "roofline": {
            "kernel": "w4a4_gemm_kernel",
            "bound": "tensor",
            "achieved": round(gemm_tops, 2),
            "peak": round(int8_peak, 1),
            "unit": "TOPS",
            "frac": round(gemm_tops / int8_peak, 4),
            "traffic": _profiled_traffic("w4a4_gemm_kernel") if profiled_shape else None,
            "algorithmic_bytes": gemm_bytes,
            "peak_source": f"{peak_kind} bf16 burst {peaks['bf16_tflops']} TFLOP/s x "
                           f"{INT8_OVER_BF16} (nominal int8:bf16 ratio)",
            "frac_of_int8_probe": round(gemm_tops / probe["value"], 4) if probe else None,
        },
        "roofline_quant": {
            "kernel": "reorder_quant_kernel",
            "bound": "hbm",
            "achieved": round(quant_gbs, 1),
            "peak": peaks["hbm_gbs"],
            "unit": "GB/s",
            "frac": round(quant_gbs / peaks["hbm_gbs"], 4),
            "traffic": _profiled_traffic("reorder_quant_kernel") if profiled_shape else None,
            "algorithmic_bytes": quant_bytes,
            "peak_source": f"{peak_kind} HBM copy",
            "alone": {
                "achieved": round(quant_bytes / (quant_alone_ms * 1e-3) / 1e9, 1),
                "frac": round(quant_bytes / (quant_alone_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                "ms": round(quant_alone_ms, 4),
                "how": "20 launches back to back on two alternating copies of A, no GEMM between",
            },
        },
        "clocks": clocks.summary(),
        "gpu_launches": 2 * n_steps,
        "e2e": e2e,
    }
    if probe is not None:
        line["int8_probe"] = probe
    if per_config is not None:
        line["per_config"] = per_config
    if cublas is not None:
        cublas["w4a4_gemm_speedup"] = round(cublas["ms"] / gemm_avg, 3)
        line["fp16_cublas"] = cublas
    if w8a8 is not None:
        w8a8["frac_int8_peak"] = round(w8a8["value"] / int8_peak, 4)
        line["w8a8"] = w8a8
    if gemm_quant is not None:
        line["gemm_quant"] = gemm_quant
    if w4a8 is not None:
        line["w4a8"] = w4a8
    if kv is not None:
        kv["quant"]["frac_hbm"] = round(kv["quant"]["value"] / peaks["hbm_gbs"], 4)
        kv["dequant"]["frac_hbm"] = round(kv["dequant"]["value"] / peaks["hbm_gbs"], 4)
        line["kv_int4"] = kv
    if world == 1 and not args.no_cpu_baseline:
        ops_s, rows, dt, cores = cpu_oracle_run(w, A_h, W_h, idx_h, args.cpu_budget)
        line["cpu_baseline"] = {"value": round(ops_s / 1e12, 6), "unit": "TOPS", "cores": cores,
                                "kind": "oracle",
                                "sample": f"first {rows} of {w.M} activation rows x all {w.N} "
                                          f"weight rows (quantize + GEMM, {dt:.1f} s; weights "
                                          f"quantized beforehand, untimed)"}
    print(json.dumps(line), flush=True)


def run_reference(args, w, workload_cfg, rank):
    """The CPU oracle as the reference arm: one bounded row sample per step."""
    if rank != 0:
        return
    from w4a4_mixed_precision_b200 import inputs
    from oracle import c_oracle
    cores = len(os.sched_getaffinity(0))
    c_oracle.set_threads(cores)
    A = inputs.activations(args.workload, rows=w.M)
    W = inputs.weights(args.workload)
    idx = inputs.outlier_channels(args.workload)
    qw = c_oracle.quantize(W, idx)
    # size the per-step sample so that warmup + steps stay within a few minutes
    t0 = time.perf_counter()
    probe = 4
    qa = c_oracle.quantize(np.ascontiguousarray(A[:probe]), idx)
    c_oracle.gemm(*qa, *qw, w.K)
    per_row = (time.perf_counter() - t0) / probe
    total_steps = args.steps + max(3, args.warmup)
    rows = int(max(1, min(w.M, 120.0 / total_steps / max(per_row, 1e-6))))
    times = []
    for i in range(total_steps):
        t0 = time.perf_counter()
        qa = c_oracle.quantize(np.ascontiguousarray(A[:rows]), idx)
        c_oracle.gemm(*qa, *qw, w.K)
        dt = time.perf_counter() - t0
        if i >= max(3, args.warmup):
            times.append(dt)
    ms = statistics.mean(times) * 1e3
    value = 2.0 * rows * w.N * w.K / (ms * 1e-3) / 1e12
    sample = (f"first {rows} of {w.M} activation rows x all {w.N} weight rows per step "
              f"(quantize + GEMM; weights quantized once beforehand)")
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded; see w4a4_mixed_precision_b200/inputs.py)",
        "config": workload_cfg, "impl": "reference",
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
