#!/usr/bin/env python
"""MoE expert layer, forward + backward, tokens/s on B200 (one GPU per process; N independent replicas).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is the whole hot path over one batch: routing metadata, row-wise dispatch, grouped GEMM1 +
SwiGLU, grouped GEMM2, combine, combine backward, GEMM2 dgrad + SwiGLU backward, GEMM2 wgrad, GEMM1
dgrad, GEMM1 wgrad, token reduce (plus router scores / top-k / router backward for learned-router
workloads). Inputs are resident in HBM when the timed region starts; the e2e figure repeats the
measurement through the public layer API with host-resident inputs and outputs copied each step
(on copy streams that overlap the neighbouring steps' compute).
Rank 0 prints one JSON line.
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
sys.path.insert(0, ROOT)

METRIC = "MoE layer fwd+bwd tokens/s at E=128 top-4; grouped GEMM % tensor-core peak"
DEFAULT_WORKLOAD = "e128_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}


def max_over_ranks(x: float, device=None) -> float:
    """The slowest rank's value (the job's time): all-reduce MAX over the process group, if any."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS)


# ------------------------------------------------------------------------------------------------
# algorithmic work per op (bytes moved once, flops of the definition); R = routed rows = T*k
# ------------------------------------------------------------------------------------------------

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch, taken from a committed ncu
# capture of the kernel as it is now; an entry is removed whenever its kernel changes, so a kernel or
# workload not listed reports null.
MEASURED_TRAFFIC = {
    # e128_bf16, ncu capture of the full-size launch of the current kernel
    # (dram__bytes_read.sum + dram__bytes_write.sum)
    ("e128_bf16", "gemm_wgrad1"): 286.59e6 + 1.0129e9,
    ("e128_bf16", "gemm_fwd1_swiglu"): 1.23e9 + 198.25e6,
}
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal


def op_work_mx(w):
    """Per-op algorithmic (bytes, flops) of the MXFP8 layer step: fp8 codes + 1/32 scale bytes for GEMM
    operands, bf16 for everything stored."""
    T, d, F, E, k = w.T, w.d, w.F, w.E, w.k
    R = T * k
    Rp = R + 127 * E                   # 128-row groups in MXFP8 mode
    q = lambda n: n + n // 32          # codes + scales of n elements
    ops = {}
    ops["route_metadata"] = (T * k * 4 * 3 + Rp * 4, 0)
    # the routed input, a, dy and dh13 exist only in their two quantised forms: their producers read
    # bf16 once and write the row-block and the column-block codes + scales
    ops["dispatch_quant"] = (T * d * 2 + R * 4 + 2 * q(R * d), 0)
    ops["gemm_fwd1_swiglu_quant"] = (q(R * d) + q(E * 2 * F * d) + R * 2 * F * 2 + 2 * q(R * F),
                                     4 * R * d * F)
    ops["gemm_fwd2"] = (q(R * F) + q(E * d * F) + R * d * 2, 2 * R * F * d)
    ops["combine"] = ((R * d + T * d) * 2 + T * k * 8, 0)
    ops["combine_bwd_quant"] = ((T * d + R * d) * 2 + T * k * 8 + R * 4 + 2 * q(R * d), 0)
    ops["gemm_dgrad2_swiglu_quant"] = (q(R * d) + q(E * d * F) + R * 2 * F * 2 + 2 * q(R * 2 * F),
                                       2 * R * d * F)
    ops["gemm_wgrad2"] = (q(R * d) + q(R * F) + E * d * F * 2, 2 * R * d * F)
    ops["gemm_dgrad1"] = (q(R * 2 * F) + q(E * 2 * F * d) + R * d * 2, 4 * R * F * d)
    ops["gemm_wgrad1"] = (q(R * 2 * F) + q(R * d) + E * 2 * F * d * 2, 4 * R * F * d)
    ops["token_reduce"] = ((R * d + T * d) * 2, 0)
    return ops


def weight_quant_work(w):
    n = w.E * 2 * w.F * w.d + w.E * w.d * w.F  # W13 + W2 elements
    return 2 * (n * 2 + n + n // 32)            # two orientations: read bf16, write codes + scales


def op_work(w, es=2, recompute=False):
    if w.dtype == "mxfp8":
        return op_work_mx(w)
    T, d, F, E, k = w.T, w.d, w.F, w.E, w.k
    R = T * k
    Rp = R + 31 * E  # upper bound of padded rows written (pad rows are written as zeros)
    ops = {}
    if w.routing == "learned":
        ops["router_logits"] = (T * d * es + E * d * es + T * E * 4, 2 * T * d * E)
        ops["route_topk"] = (T * E * 4 + T * k * 8, 0)
    ops["route_metadata"] = (T * k * 4 * 3 + Rp * 4, 0)
    ops["dispatch"] = ((T + R) * d * es, 0)
    fwd1 = ((R * d + E * 2 * F * d + R * 2 * F + R * F) * es, 2 * R * d * 2 * F)
    # with activation recompute the forward's GEMM1 writes only a; the backward runs it again in full
    ops["gemm_fwd1_swiglu"] = (fwd1[0] - R * 2 * F * es, fwd1[1]) if recompute else fwd1
    ops["gemm_fwd2"] = ((R * F + E * d * F + R * d) * es, 2 * R * F * d)
    ops["combine"] = ((R * d + T * d) * es + T * k * 8, 0)
    ops["combine_bwd"] = ((T * d + 2 * R * d) * es + T * k * 12, 0)
    if recompute:
        ops["gemm_fwd1_recompute"] = fwd1
    # in the order moe_layer_bwd issues them
    ops["gemm_dgrad2_swiglu"] = ((R * d + E * d * F + 2 * R * 2 * F) * es, 2 * R * d * F)
    ops["gemm_dgrad1"] = ((R * 2 * F + E * 2 * F * d + R * d) * es, 2 * R * 2 * F * d)
    ops["token_reduce"] = ((R * d + T * d) * es + (T * k * 8 if w.routing == "learned" else 0), 0)
    ops["gemm_wgrad2"] = ((R * d + R * F + E * d * F) * es, 2 * R * d * F)
    ops["gemm_wgrad1"] = ((R * 2 * F + R * d + E * 2 * F * d) * es, 2 * R * 2 * F * d)
    if w.routing == "learned":
        ops["router_wgrad"] = ((T * E + T * d + E * d) * es, 2 * T * E * d)
    return ops


class Step:
    """The layer's kernels issued op by op through the C ABI (the same sequence moe_layer_fwd /
    moe_layer_bwd enqueue), with CUDA events between ops for a per-kernel breakdown."""

    def __init__(self, layer, w, inp):
        import torch
        from mixture_experts_layer_row_b200 import _lib as L
        self.L, self.layer, self.w, self.inp = L, layer, w, inp
        self.learned = w.routing == "learned"
        lay = layer
        if self.learned:
            self.dlsel = torch.zeros((w.T, w.k), dtype=torch.float32, device=lay.device)
            self.dlogits = torch.zeros((w.T, w.E), dtype=lay.act, device=lay.device)
        else:
            lay.idx.copy_(inp["idx"])
            lay.gates.copy_(inp["gates"])
        self.names = list(op_work(w, recompute=layer.recompute).keys())
        self.ev = None
        self.only = None  # record only the boundaries of this op (None: every op boundary)

    def events(self, n_steps, only=None):
        """Events for the next n_steps runs: at every op boundary (the per-op breakdown), or only
        around op `only` (every other boundary is left free, so consecutive kernels overlap their
        launch and prologue through programmatic dependent launch)."""
        import torch
        self.only = only
        self.ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(self.names) + 1)]
                   for _ in range(n_steps)]

    def op_ms(self, i, name):
        j = self.names.index(name)
        return self.ev[i][j].elapsed_time(self.ev[i][j + 1])

    @property
    def only_idx(self):
        j = self.names.index(self.only)
        return (j, j + 1)

    def run(self, i=None):
        if self.layer.mx:
            return self.run_mx(i)
        L, lay, w, inp = self.L, self.layer, self.w, self.inp
        ev = self.ev[i] if (i is not None and self.ev is not None) else None
        c = lay.cfg
        n = 0

        def mark():
            nonlocal n
            if ev is not None and (self.only is None or n in self.only_idx):
                ev[n].record()
            n += 1

        if self.learned:
            mark(); L.router_logits(c, inp["x"], inp["W_r"], inp["bias"], lay.logits, lay.ws)
            mark(); L.route_topk(c, lay.logits, None, lay.idx, lay.gates, lay.ws)
        mark(); L.route_metadata(c, lay.idx, lay.counts, lay.offsets, lay.poff, lay.perm, lay.prow,
                                 lay.row_token, lay.ws)
        mark(); L.dispatch(c, inp["x"], lay.prow, lay.counts, lay.poff, lay.x_perm)
        mark(); L.grouped_gemm(c, L.GEMM_FWD1_SWIGLU, lay.x_perm, inp["W13"], lay.h13, lay.a, None,
                               lay.counts, lay.poff, lay.ws)
        mark(); L.grouped_gemm(c, L.GEMM_FWD2, lay.a, inp["W2"], lay.y, None, None, lay.counts, lay.poff,
                               lay.ws)
        mark(); L.combine(c, lay.y, lay.gates, lay.prow, lay.out)
        dls = self.dlsel if self.learned else None
        dlg = self.dlogits if self.learned else None
        mark(); L.combine_bwd(c, inp["dout"], lay.y, lay.gates, lay.prow, lay.idx, lay.counts, lay.poff,
                              lay.dy, lay.dgates, dls, dlg)
        h13 = lay.h13
        if lay.recompute:
            mark(); L.grouped_gemm(c, L.GEMM_FWD1_SWIGLU, lay.x_perm, inp["W13"], lay.dh13, lay.a, None,
                                   lay.counts, lay.poff, lay.ws)
            h13 = lay.dh13
        mark(); L.grouped_gemm(c, L.GEMM_DGRAD2_SWIGLU, lay.dy, inp["W2"], lay.dh13, None, h13,
                               lay.counts, lay.poff, lay.ws)
        mark(); L.grouped_gemm(c, L.GEMM_DGRAD1, lay.dh13, inp["W13"], lay.dx_perm, None, None,
                               lay.counts, lay.poff, lay.ws)
        mark(); L.token_reduce(c, lay.dx_perm, lay.prow, lay.dx, dls,
                               lay.idx if self.learned else None, inp["W_r"] if self.learned else None)
        mark(); L.grouped_gemm(c, L.GEMM_WGRAD2, lay.dy, lay.a, lay.dW2, None, None, lay.counts,
                               lay.poff, lay.ws)
        mark(); L.grouped_gemm(c, L.GEMM_WGRAD1, lay.dh13, lay.x_perm, lay.dW13, None, None,
                               lay.counts, lay.poff, lay.ws)
        if self.learned:
            mark(); L.router_wgrad(c, self.dlogits, inp["x"], lay.dW_r, lay.ws)
        mark()


    def run_mx(self, i=None):
        """The kernels of moe_layer_fwd_mxfp8 / moe_layer_bwd_mxfp8, op by op (uniform routing): the
        routed input, a, dy and dh13 leave their producers only as their two quantised forms."""
        L, lay, w, inp = self.L, self.layer, self.w, self.inp
        ev = self.ev[i] if (i is not None and self.ev is not None) else None
        c, qa, qw = lay.cfg, lay.qa_t, lay.qw_t
        n = 0

        def mark():
            nonlocal n
            if ev is not None and (self.only is None or n in self.only_idx):
                ev[n].record()
            n += 1

        cnt, po, ws, ops = lay.counts, lay.poff, lay.ws, lay.q_ops
        mark(); L.route_metadata(c, lay.idx, lay.counts, lay.offsets, lay.poff, lay.perm, lay.prow,
                                 lay.row_token, ws)
        mark(); L.dispatch_mxfp8(c, inp["x"], lay.row_token, po, ops["x"])
        mark(); L.grouped_gemm_mxfp8_quant(c, L.GEMM_FWD1_SWIGLU, qa["xq"], qa["xs"], qw["W13q"],
                                           qw["W13s"], lay.h13, None, ops["a"], cnt, po, ws)
        mark(); L.grouped_gemm_mxfp8(c, L.GEMM_FWD2, qa["aq"], qa["as"], qw["W2q"], qw["W2s"], lay.y,
                                     None, None, cnt, po, ws)
        mark(); L.combine(c, lay.y, lay.gates, lay.prow, lay.out)
        mark(); L.combine_bwd_mxfp8(c, inp["dout"], lay.y, lay.gates, lay.row_token, po, lay.dgates,
                                    ops["dy"])
        mark(); L.grouped_gemm_mxfp8_quant(c, L.GEMM_DGRAD2_SWIGLU, qa["dyq"], qa["dys"], qw["W2tq"],
                                           qw["W2ts"], None, lay.h13, ops["dh"], cnt, po, ws)
        mark(); L.grouped_gemm_mxfp8(c, L.GEMM_WGRAD2, qa["dytq"], qa["dyts"], qa["atq"], qa["ats"],
                                     lay.dW2, None, None, cnt, po, ws)
        mark(); L.grouped_gemm_mxfp8(c, L.GEMM_DGRAD1, qa["dhq"], qa["dhs"], qw["W13tq"], qw["W13ts"],
                                     lay.dx_perm, None, None, cnt, po, ws)
        mark(); L.grouped_gemm_mxfp8(c, L.GEMM_WGRAD1, qa["dhtq"], qa["dhts"], qa["xtq"], qa["xts"],
                                     lay.dW13, None, None, cnt, po, ws)
        mark(); L.token_reduce(c, lay.dx_perm, lay.prow, lay.dx)
        mark()


class ClockSampler:
    """SM clock and throttle reasons around and during the timed region: NVML reads from a background
    thread, one when sampling starts, then every 50 ms, and one more when the region ends (so even a
    region of a few tens of milliseconds is bracketed); `nvidia-smi -lms 200` where NVML cannot be
    used. Polling NVML every few milliseconds slowed the measured step by 10 %, so the period stays
    long."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None
        self.nvml = None
        self.thread = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(getattr(torch.cuda.get_device_properties(self.index), "uuid", "") or "")
        for u in (uuid, "GPU-" + uuid):
            try:
                if u and u != "GPU-":
                    return pynvml, pynvml.nvmlDeviceGetHandleByUUID(u)
            except pynvml.NVMLError:
                pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.nvml = (nv, h, nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            nv, h, _ = self.nvml
            self.rows, self.stop_evt = [], threading.Event()

            def run():
                while True:
                    try:
                        self.rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                          nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
                    except nv.NVMLError:
                        break
                    if self.stop_evt.wait(0.05):
                        break
            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.rows and self.thread.is_alive() and time.time() - t0 < 2.0:
                time.sleep(0.001)
            return
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)  # its start-up, before the timed region
        except (OSError, FileNotFoundError):
            self.proc = None

    @staticmethod
    def _summary(sm, mx, reasons, n, source):
        loaded = [v for v in sm if mx and v > 0.3 * mx] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": n, "source": source}

    def stop(self):
        if self.nvml is not None:
            nv, h, mx = self.nvml
            self.stop_evt.set()
            self.thread.join(timeout=2)
            try:  # the region's end
                self.rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                  nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except nv.NVMLError:
                pass
            rows = list(self.rows)
            try:
                nv.nvmlShutdown()
            except Exception:
                pass
            if not rows:
                return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["no samples"], "source": "nvml"}
            bits = (("hw_slowdown", nv.nvmlClocksEventReasonHwSlowdown),
                    ("hw_thermal_slowdown", nv.nvmlClocksEventReasonHwThermalSlowdown),
                    ("sw_thermal_slowdown", nv.nvmlClocksEventReasonSwThermalSlowdown),
                    ("sw_power_cap", nv.nvmlClocksEventReasonSwPowerCap))
            reasons = {name for _, r in rows for name, b in bits if r & b}
            return self._summary([float(c) for c, _ in rows], float(mx), reasons, len(rows),
                                 "nvml at start, every 50 ms and at the end")
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        reasons = set()
        for r in rows:
            for name, col in (("hw_slowdown", 5), ("hw_thermal_slowdown", 6),
                              ("sw_thermal_slowdown", 7), ("sw_power_cap", 8)):
                if r[col].lower().startswith("active"):
                    reasons.add(name)
        return self._summary(sm, max(mx) if mx else None, reasons, len(rows), "nvidia-smi every 200 ms")


class ExpertSample:
    """The fp64 oracle's per-expert forward + backward (MXFP8-emulated for the MXFP8 workload) over
    every routed row of a subset of experts. The experts' weights are converted to fp64 once, outside
    the timed region. Throughput = processed routed rows / k per second."""

    def __init__(self, w, inp, n_experts):
        import numpy as np
        import torch
        f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
        self.w, self.mx = w, w.dtype == "mxfp8"
        idx = inp["idx"].cpu().numpy().astype(np.int64)
        gates, x, dout = f64(inp["gates"]), f64(inp["x"]), f64(inp["dout"])
        self.work = []
        for e in range(n_experts):
            tj = np.argwhere(idx == e)
            self.work.append((x[tj[:, 0]], gates[tj[:, 0], tj[:, 1]][:, None] * dout[tj[:, 0]],
                              f64(inp["W13"][e]), f64(inp["W2"][e])))
        self.rows = sum(len(wk[0]) for wk in self.work)

    def run(self):
        from oracle import moe as O
        t0 = time.perf_counter()
        for X, dY, W13e, W2e in self.work:
            h13, a, _ = O.expert_fwd(X, W13e, W2e, self.mx)
            O.expert_bwd(X, W13e, W2e, h13, a, dY, self.mx)
        return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([int(i.get("num_threads", 1)) for i in threadpool_info()] or [1])
    except Exception:
        return 1


def cpu_baseline_experts(w, inp, n_experts, label):
    smp = ExpertSample(w, inp, n_experts)
    dt = smp.run()
    return {"value": smp.rows / w.k / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{label}: experts 0..{n_experts - 1}, all {smp.rows} of their routed rows "
                      f"({'MXFP8-emulated ' if smp.mx else ''}fp64 per-expert forward + backward), "
                      f"{dt:.1f} s; tokens/s = rows / k / s"}


def cpu_baseline(w, inp, n_tokens, label):
    if w.E * 3 * w.F * w.d > 1_500_000_000 or w.dtype == "mxfp8":
        return cpu_baseline_experts(w, inp, 6, label)
    """The fp64 oracle, as it stands, on the first n_tokens tokens of the workload (their routing,
    the full expert weights), forward + backward; returns tokens/s and what was run."""
    import numpy as np
    import torch
    from oracle import moe as O
    f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
    x = f64(inp["x"][:n_tokens])
    dout = f64(inp["dout"][:n_tokens])
    W13, W2 = f64(inp["W13"]), f64(inp["W2"])
    learned = w.routing == "learned"
    Wr = f64(inp["W_r"]) if learned else None
    bias = f64(inp["bias"]) if inp["bias"] is not None else None
    if not learned:
        idx = inp["idx"][:n_tokens].cpu().numpy().astype(np.int64)
        gates = f64(inp["gates"][:n_tokens])
    t0 = time.perf_counter()
    if learned:
        lg = O.router_logits(x, Wr, bias)
        idx, gates = O.route(lg, w.k)
    out, saved = O.layer_fwd(x, W13, W2, idx, gates)
    O.layer_bwd(dout, x, W13, W2, idx, gates, saved, W_r=Wr)
    dt = time.perf_counter() - t0
    return {"value": n_tokens / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{label}: first {n_tokens} tokens ({n_tokens * w.k} routed rows), full expert "
                      f"weights, fp64 forward + backward, {dt:.1f} s"}


def run_reference(args, w):
    """The oracle timed as it stands on the host cores (rank 0 only). Each step is the oracle's
    per-expert forward + backward over the routed rows of a subset of experts, the subset sized from
    a one-expert probe so that warm-up + timed steps take about two and a half minutes."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from moe_workloads import make_inputs
    import torch
    if w.routing == "learned":  # the oracle routes from its own fp64 router scores
        from oracle import moe as O
        import numpy as np
        inp = make_inputs(w, seed=0, device="cpu")
        f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
        lg = O.router_logits(f64(inp["x"]), f64(inp["W_r"]), None if inp["bias"] is None else f64(inp["bias"]))
        idx, g = O.route(lg, w.k)
        inp["idx"], inp["gates"] = torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(g)
    else:
        inp = make_inputs(w, seed=0, device="cpu")
    probe = ExpertSample(w, inp, 1)
    t1 = max(probe.run(), 1e-3)
    budget = min(30.0, 150.0 / max(1, args.steps + args.warmup))
    m = max(1, min(w.E, int(budget / t1)))
    smp = ExpertSample(w, inp, m)
    times = []
    for i in range(args.warmup + args.steps):
        dt = smp.run()
        if i >= args.warmup:
            times.append(dt)
    per = statistics.mean(times)
    val = smp.rows / w.k / per
    sample = (f"{w.name}: per step the fp64 oracle's per-expert forward + backward over experts "
              f"0..{m - 1} ({smp.rows} routed rows = {smp.rows / w.k:.0f} token-equivalents), "
              f"{'MXFP8-emulated, ' if smp.mx else ''}{per:.2f} s per step")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": dict(workload_config(w), parallelism=f"replicas x{args.gpus}"),
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def gemm_peak(args):
    """Dense throughput of this library's own tcgen05 grouped GEMM on one square problem (one expert
    holding every row: M = N = K = 8192), forward GEMM2 op (K-major operands, plain bf16 store): bf16
    on CTA pairs, or MXFP8 block-scaled (E4M3 operands, UE8M0 scales). CUDA events around 20 launches
    after 5 warm-up launches, nvidia-smi clocks sampled meanwhile. Prints one JSON line."""
    import torch
    from mixture_experts_layer_row_b200 import _lib as L
    torch.cuda.set_device(0)
    n = 8192
    mx = args.gemm_peak == "mxfp8"
    cfg = L.make_config(n, n, n, 1, 1, L.DTYPE_MXFP8 if mx else L.DTYPE_BF16)
    R = L.max_rows(cfg)
    dev = torch.device("cuda", 0)
    ws = torch.zeros(L.workspace_size(cfg), dtype=torch.uint8, device=dev)
    counts = torch.tensor([n], dtype=torch.int32, device=dev)
    poff = torch.tensor([0, n], dtype=torch.int32, device=dev)
    g = torch.Generator(device=dev).manual_seed(0)
    A = torch.zeros((R, n), dtype=torch.bfloat16, device=dev)
    A[:n] = torch.randn((n, n), generator=g, device=dev).to(torch.bfloat16)
    B = (torch.randn((n, n), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    C = torch.empty((R, n), dtype=torch.bfloat16, device=dev)
    if mx:
        q = lambda t: (torch.empty(t.shape, dtype=torch.uint8, device=dev),
                       torch.empty(t.numel() // 32, dtype=torch.uint8, device=dev))
        (Aq, As), (Bq, Bs) = q(A), q(B)
        L.quantize_mxfp8(A, Aq, As, L.QUANT_ROW_TILED)
        L.quantize_mxfp8(B, Bq, Bs, L.QUANT_ROW_TILED)
        run = lambda: L.grouped_gemm_mxfp8(cfg, L.GEMM_FWD2, Aq, As, Bq, Bs, C, None, None, counts, poff, ws)
    else:
        run = lambda: L.grouped_gemm(cfg, L.GEMM_FWD2, A, B, C, None, None, counts, poff, ws)
    for _ in range(5):
        run()
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(20):
        run()
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / 20
    flops = 2.0 * n * n * n
    print(json.dumps({"gemm_peak": args.gemm_peak, "M": n, "N": n, "K": n, "ms": ms,
                      "tflops": flops / (ms / 1e3) / 1e12, "clocks": clk,
                      "error_flags": L.get_error(ws)}), flush=True)
    return 0


def workload_config(w):
    return {"workload": f"{w.name}: T={w.T} d={w.d} F={w.F} E={w.E} k={w.k} {w.dtype}, "
                        f"{w.routing} routing" + (f", skew bias {w.skew}*ln(1/rank)" if w.skew else ""),
            "T": w.T, "d_model": w.d, "ffn": w.F, "experts": w.E, "top_k": w.k,
            "routing": w.routing, "seed": 0,
            "l2": "no flush: every step streams inputs larger than the 126 MB L2 "
                  "(expert weights alone are read twice and their gradients written once per step)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=8192, help="oracle sample for cpu_baseline (capped at T)")
    ap.add_argument("--ref-tokens", type=int, default=256, help="oracle sample per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--experts", type=int, default=0,
                    help="expert-count sweep: the workload's shapes with E experts, uniform routing")
    ap.add_argument("--tokens", type=int, default=0,
                    help="the workload's shapes with T tokens (smaller cases for ncu captures)")
    ap.add_argument("--gemm-peak", default="",
                    choices=["", "bf16", "mxfp8"],
                    help="time this library's grouped GEMM on one large square group (E=1) and print its "
                         "TFLOP/s instead of the layer step")
    ap.add_argument("--recompute", action="store_true",
                    help="activation recompute: the layer keeps no h13 and the backward regenerates it; "
                         "also times it against stored activations through the layer API")
    args = ap.parse_args()

    from moe_workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.experts:
        w = w.scaled(E=args.experts, routing="uniform", skew=0.0, name=f"{w.name}_E{args.experts}")
    if args.tokens:
        w = w.scaled(T=args.tokens, name=f"{w.name}_T{args.tokens}")
    if args.gemm_peak:
        return gemm_peak(args)
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    from moe_workloads import make_inputs
    from mixture_experts_layer_row_b200 import MoELayer
    from mixture_experts_layer_row_b200 import _lib as L

    inp = make_inputs(w, seed=0, device="cuda")
    learned = w.routing == "learned"
    if args.recompute and w.dtype == "mxfp8":
        raise SystemExit("--recompute: activation recompute is implemented for the bf16 / fp32 layer")
    layer = MoELayer(w.T, w.d, w.F, w.E, w.k, dtype=w.dtype, learned_router=learned,
                     recompute=args.recompute)
    layer.set_weights(inp["W13"], inp["W2"], inp["W_r"] if learned else None)
    step = Step(layer, w, inp)

    # the op-by-op sequence computes exactly what the public layer API computes
    step.run()
    torch.cuda.synchronize()
    ref = (layer.out.clone(), layer.dx.clone(), layer.dW13.clone(), layer.dW2.clone())
    layer.forward(inp["x"], bias=inp["bias"], idx=inp["idx"], gates=inp["gates"])
    layer.backward(inp["dout"])
    torch.cuda.synchronize()
    same = all(torch.equal(a, b) for a, b in zip(ref, (layer.out, layer.dx, layer.dW13, layer.dW2)))
    assert same, "op-by-op sequence differs from moe_layer_fwd/bwd"
    assert layer.error_flags() == 0, "device error flag set"

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step.run()
    # per-op breakdown: an instrumented pass of K steps with an event at every op boundary (each event
    # also serialises the two kernels around it, so these per-op times include launch gaps)
    step.events(args.steps)
    for i in range(args.steps):
        step.run(i)
    torch.cuda.synchronize()
    per_op = {n: 0.0 for n in step.names}
    for i in range(args.steps):
        for n in step.names:
            per_op[n] += step.op_ms(i, n)
    per_op = {n: v / args.steps for n, v in per_op.items()}
    ms_instrumented = sum(step.ev[i][0].elapsed_time(step.ev[i][-1]) for i in range(args.steps)) / args.steps
    dom = max(per_op, key=lambda n: per_op[n])
    # timed region: K steps issued back to back as the layer API issues them, with events only around
    # the dominant kernel (its duration for the roofline)
    step.events(args.steps, only=dom)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    n0 = L.launch_count()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record()
    for i in range(args.steps):
        step.run(i)
    t_end.record()
    torch.cuda.synchronize()
    launches = L.launch_count() - n0
    clk = clocks.stop()
    barrier()
    ms = max_over_ranks(t_start.elapsed_time(t_end), "cuda")
    ms_per_step = ms / args.steps
    value = world * w.T / (ms_per_step / 1e3)

    # device memory high-water mark of the run so far: inputs, weights, gradients, the layer's saved
    # activations and scratch (the MXFP8 path adds the quantised copies)
    peak_mem_gb = torch.cuda.max_memory_allocated() / 1e9

    # the dominant kernel's duration inside the timed region
    dom_ms = sum(step.op_ms(i, dom) for i in range(args.steps)) / args.steps

    peaks = load_peaks()
    work = op_work(w, 4 if w.dtype == "fp32" else 2, recompute=layer.recompute)
    bw = peaks["hbm_gbs"]
    # tensor peak of the GEMMs' own dtype: the measured bf16 figure times the nominal dense ratio
    # (tf32 1.1 / bf16 2.25 PFLOP/s; fp8 4.5 / 2.25)
    ratio = {"fp32": 0.5, "bf16": 1.0, "mxfp8": 2.0}[w.dtype]
    tc = peaks["bf16_tflops"] * ratio
    roof_time = 0.0
    for n, (b, f) in work.items():
        roof_time += max(b / (bw * 1e9), f / (tc * 1e12))
    # every HBM-bound kernel's achieved bandwidth against the measured copy peak and the nominal 8 TB/s
    hbm_ops = {}
    for n, (b, f) in work.items():
        if b / (bw * 1e9) >= f / (tc * 1e12):
            gbs = b / (per_op[n] / 1e3) / 1e9
            hbm_ops[n] = {"GB/s": round(gbs, 1), "frac_measured": round(gbs / bw, 3),
                          "frac_nominal": round(gbs / NOMINAL_HBM_GBS, 3)}
    gemm_ops = [n for n in work if n.startswith("gemm_")]
    gemm_flops = sum(work[n][1] for n in gemm_ops)
    gemm_ms = sum(per_op[n] for n in gemm_ops)
    b, f = work[dom]
    t_dom = dom_ms / 1e3
    if b / (bw * 1e9) >= f / (tc * 1e12) or f == 0:
        roof = {"kernel": dom, "bound": "hbm", "achieved": b / t_dom / 1e9, "peak": bw, "unit": "GB/s",
                "frac": (b / t_dom / 1e9) / bw, "traffic": MEASURED_TRAFFIC.get((w.name, dom)),
                "algorithmic_bytes": b, "flops": f, "ms": dom_ms,
                "peak_source": f"{peaks['source']} hbm_gbs"}
    else:
        roof = {"kernel": dom, "bound": "tensor", "achieved": f / t_dom / 1e12, "peak": tc,
                "unit": "TFLOP/s", "frac": (f / t_dom / 1e12) / tc,
                "traffic": MEASURED_TRAFFIC.get((w.name, dom)),
                "algorithmic_bytes": b, "flops": f, "ms": dom_ms,
                "peak_source": f"{peaks['source']} bf16_tflops (burst) x {ratio} ({w.dtype})"}

    # activation memory kept between the forward and the backward (the layer's own buffers)
    nb = lambda t: t.numel() * t.element_size()
    if layer.mx:
        kept = sum(nb(layer.qa_t[n]) for n in ("xtq", "xts", "atq", "ats")) + nb(layer.h13) + nb(layer.y)
        # the bf16 layer of the same shapes keeps x_perm [R, d], h13 [R, 2F], a [R, F] and y [R, d],
        # with its own routed-row count (its groups are padded to 32 rows, the MXFP8 layer's to 128)
        R_bf16 = L.max_rows(L.make_config(w.T, w.d, w.F, w.E, w.k, L.DTYPE_BF16))
        kept_bf16 = R_bf16 * (2 * w.d + 3 * w.F) * 2
        act_mem = {"kept_between_passes_bytes": kept, "bf16_layer_same_shapes_bytes": kept_bf16,
                   "ratio": kept / kept_bf16,
                   "note": "MXFP8 keeps the column forms of x and a (codes + scales), h13 and y"}
    else:
        # with activation recompute neither h13 nor a is kept (a is scratch the backward rewrites)
        kept = nb(layer.x_perm) + nb(layer.y) + (0 if layer.recompute else nb(layer.h13) + nb(layer.a))
        act_mem = {"kept_between_passes_bytes": kept}

    wq = None
    if layer.mx:  # weights are quantised once per update: timed on their own, not in the step
        q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        layer.quantize_weights()
        q0.record()
        for _ in range(5):
            layer.quantize_weights()
        q1.record()
        torch.cuda.synchronize()
        wq_ms = q0.elapsed_time(q1) / 5
        wq = {"ms": wq_ms, "GB/s": weight_quant_work(w) / (wq_ms / 1e3) / 1e9,
              "tokens_per_s_including_it": world * w.T / ((ms_per_step + wq_ms) / 1e3),
              "note": "once per weight update (optimizer step), outside the timed layer step"}

    # end to end through the public layer API: host inputs in, host results out, every step. The
    # loop is the one a training job runs: step i+1's inputs are copied host -> device on one copy
    # stream while step i computes (two device input buffers), and step i's out / dx are read back
    # on another copy stream while the next step's work proceeds. out and dx alternate between two
    # device buffers (the layer API writes into the caller's), so a step never waits for the
    # previous step's read-back; a buffer is only rewritten after its own read-back has finished.
    e2e = None
    if not args.no_e2e:
        hx = inp["x"].cpu().pin_memory()
        hd = inp["dout"].cpu().pin_memory()
        hi = inp["idx"].cpu().pin_memory() if not learned else None
        hg = inp["gates"].cpu().pin_memory() if not learned else None
        bx = [torch.empty_like(inp["x"]) for _ in range(2)]
        bd = [torch.empty_like(inp["dout"]) for _ in range(2)]
        bi = [torch.empty_like(inp["idx"]) for _ in range(2)] if not learned else [None, None]
        bg = [torch.empty_like(inp["gates"]) for _ in range(2)] if not learned else [None, None]
        bo = [torch.empty_like(layer.out) for _ in range(2)]
        bdx = [torch.empty_like(layer.dx) for _ in range(2)]
        ho = [torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory() for _ in range(2)]
        hdx = [torch.empty(layer.dx.shape, dtype=layer.dx.dtype).pin_memory() for _ in range(2)]
        h2d = hx.numel() * hx.element_size() + hd.numel() * hd.element_size()
        if not learned:
            h2d += hi.numel() * 4 + hg.numel() * 4
        d2h = ho[0].numel() * ho[0].element_size() + hdx[0].numel() * hdx[0].element_size()
        comp = torch.cuda.current_stream()
        up, down = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        loaded, consumed = [ev(), ev()], [ev(), ev()]
        out_read, dx_read, fwd_done, bwd_done = [ev(), ev()], [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def upload(j):
            with torch.cuda.stream(up):
                up.wait_event(consumed[j])  # the step that last used buffer j has finished with it
                bx[j].copy_(hx, non_blocking=True)
                bd[j].copy_(hd, non_blocking=True)
                if not learned:
                    bi[j].copy_(hi, non_blocking=True)
                    bg[j].copy_(hg, non_blocking=True)
                loaded[j].record(up)

        def e2e_run(n):
            upload(0)
            for i in range(n):
                j = i % 2
                comp.wait_event(loaded[j])
                if i + 1 < n:
                    upload(1 - j)
                comp.wait_event(out_read[j])  # bo[j]'s read-back (two steps ago) has finished
                layer.forward(bx[j], bias=inp["bias"], idx=bi[j], gates=bg[j], out=bo[j])
                fwd_done[j].record(comp)
                with torch.cuda.stream(down):
                    down.wait_event(fwd_done[j])
                    ho[j].copy_(bo[j], non_blocking=True)
                    out_read[j].record(down)
                comp.wait_event(dx_read[j])
                layer.backward(bd[j], dx=bdx[j])
                consumed[j].record(comp)
                bwd_done[j].record(comp)
                with torch.cuda.stream(down):
                    down.wait_event(bwd_done[j])
                    hdx[j].copy_(bdx[j], non_blocking=True)
                    dx_read[j].record(down)
            for j in range(2):  # the timed region ends with every result on the host
                comp.wait_event(out_read[j])
                comp.wait_event(dx_read[j])

        e2e_run(args.warmup)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        e2e_run(args.steps)
        e1.record(comp)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), "cuda")
        e2e = {"value": world * w.T / (ems / args.steps / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": ems / args.steps,
               "api": "MoELayer.forward/backward -> moe_layer_fwd/bwd into alternating out / dx "
                      "buffers; copies on two streams overlap the neighbouring steps' compute"}
        jl = (args.steps - 1) % 2
        assert torch.equal(ho[jl].cuda(), ref[0]) and torch.equal(hdx[jl].cuda(), ref[1])

    # activation recompute against stored activations, both through the public layer API on the
    # same device-resident inputs, timed in alternation (so clock and power drift hit both alike),
    # with the activation memory each keeps between the two passes
    rc = None
    if layer.recompute:
        lay_st = MoELayer(w.T, w.d, w.F, w.E, w.k, dtype=w.dtype, learned_router=learned)
        lay_st.set_weights(inp["W13"], inp["W2"], inp["W_r"] if learned else None)

        def api_ms(lay):
            def one():
                lay.forward(inp["x"], bias=inp["bias"], idx=inp["idx"], gates=inp["gates"])
                lay.backward(inp["dout"])
            for _ in range(args.warmup):
                one()
            torch.cuda.synchronize()
            barrier()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record()
            for _ in range(args.steps):
                one()
            a1.record()
            torch.cuda.synchronize()
            return max_over_ranks(a0.elapsed_time(a1), "cuda") / args.steps

        t_st, t_rc = [], []
        for _ in range(3):
            t_st.append(api_ms(lay_st))
            t_rc.append(api_ms(layer))
        ms_st, ms_rc = sorted(t_st)[1], sorted(t_rc)[1]
        same = all(torch.equal(a, b) for a, b in zip(
            (lay_st.out, lay_st.dx, lay_st.dW13, lay_st.dW2), (layer.out, layer.dx, layer.dW13, layer.dW2)))
        assert same and layer.error_flags() == 0, "recompute differs from stored activations"
        es, R = layer.act.itemsize, layer.R
        # kept from forward to backward: x_perm and y, plus h13 and a when stored (with recompute a
        # is scratch that the backward rewrites)
        kept_st = R * (2 * w.d + 2 * w.F + w.F) * es
        kept_rc = R * 2 * w.d * es
        rc = {"ms_per_step_stored": ms_st, "ms_per_step_recompute": ms_rc,
              "value_stored": world * w.T / (ms_st / 1e3), "value_recompute": world * w.T / (ms_rc / 1e3),
              "throughput_ratio": ms_st / ms_rc,
              "kept_activation_bytes": {"stored": kept_st, "recompute": kept_rc},
              "kept_activation_ratio": kept_rc / kept_st, "bit_identical": same,
              "timing": "layer API, device-resident inputs, median of 3 alternating runs of K steps"}
        del lay_st

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, inp, min(args.cpu_tokens, w.T), w.name)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded; shapes and distributions of the workload)",
            "config": dict(workload_config(w), parallelism=f"replicas x{world}",
                           **({"activation_recompute": True} if layer.recompute else {})),
            "tflops": 18 * w.d * w.F * w.T * w.k * world / (ms_per_step / 1e3) / 1e12,
            "grouped_gemm_tensor_frac": (gemm_flops / (gemm_ms / 1e3) / 1e12) / tc,
            "layer_roofline": {"roofline_ms": roof_time * 1e3, "frac": roof_time * 1e3 / ms_per_step,
                               "peaks": peaks},
            "roofline": roof,
            "per_op_ms": {n: round(v, 4) for n, v in per_op.items()},
            "per_op_note": "instrumented pass of K steps with an event at every op boundary, run before "
                           "the timed region (each event serialises the kernels around it)",
            "ms_per_step_instrumented": ms_instrumented,
            "per_op_hbm": hbm_ops,
            "weight_quantisation": wq,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
            "peak_mem_gb": round(peak_mem_gb, 2),
            "activation_memory": act_mem,
        }
        if rc is not None:
            line["recompute"] = rc
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
