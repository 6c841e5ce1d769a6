"""Benchmark of the scaled FP8 GEMM hot path on B200.

Headline workload (one "step" = the whole per-call hot path on one batch):
  ffn_up: X bf16 [8192, 8192] -> mxfp8_quantize -> mxfp8_gemm against the
  pre-quantized W [22016, 8192] (MXFP8, 1x32 UE8M0 blocks) -> C bf16.
  This is the FFN up-projection shape of the "从 DeepGEMM 到 vLLM" page's
  benchmark_gemm listing, and the largest single-GPU configuration.
  value = 2*M*N*K per step / step time, in TFLOPS.

The other hot-path rows (per-row quantizer, rowwise GEMM, Q.K^T MX GEMM,
the decode sweep) are measured in the "rows" object of the same JSON line.

Multi-GPU (torchrun): every rank runs its own replica on its own GPU (no
data-path collective; weak scaling); time = max over ranks.

--impl reference: the CPU oracle as it stands, on a bounded sample of the
same workload, on the host cores (rank 0 only).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP8 GEMM TFLOPS & % of B200 FP8 peak; quantize/decode GB/s & % of HBM"
M, N, K = 8192, 22016, 8192
FLOPS_PER_STEP = 2.0 * M * N * K
CPU_SAMPLE_ROWS = 256        # cpu_baseline: this many full rows of C
REF_ROWS_PER_STEP = 16       # reference arm: a 16 x 2752 block of C per step
REF_COLS_PER_STEP = N // 8


# ---------------------------------------------------------------- helpers

def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _src_hash():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "mxfp8_block_scaled_fp8_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _ncu_traffic(kernel_key: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        e = t[kernel_key]
        return e["bytes_per_launch"] if e.get("src_hash") == _src_hash() else None
    except Exception:
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {"gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
               "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100}

    def __init__(self, index: int, period_s: float = 0.01, pci_bus_id: str | None = None):
        self.index, self.period, self.pci = index, period_s, pci_bus_id
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = None
            if self.pci:
                try:
                    self._h = pynvml.nvmlDeviceGetHandleByPciBusId(self.pci)
                except Exception:
                    self._h = None
            if self._h is None:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self._nv = None
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def max_over_ranks(value: float, device=None) -> float:
    """Largest value over all ranks (the slowest rank sets the job time)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def percentiles(xs):
    """p10 / p50 / p90 of a list of per-step times (nearest rank)."""
    v = sorted(xs)
    if not v:
        return None
    pick = lambda q: v[min(len(v) - 1, max(0, int(round(q * (len(v) - 1)))))]
    return {"p10": pick(0.10), "p50": pick(0.50), "p90": pick(0.90), "mean": sum(v) / len(v)}


def job_tflops(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank runs `steps` steps of its own replica."""
    return flops_per_step * steps * world / (max_ms * 1e-3) / 1e12


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ---------------------------------------------------------------- GPU timing utilities

def _graph_time(calls, reps: int = 10) -> float:
    """Device time (ms) per call: `calls` (one zero-argument function per
    call, each touching its own copy of the large operand so that together
    they exceed L2) are captured once into a CUDA graph and replayed `reps`
    times between two CUDA events.  This times the kernels back to back, as a
    serving engine replays them, without host launch latency."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for f in calls:                      # first calls: per-device setup happens here
            f()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in calls:
            f()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    b.synchronize()
    ms = a.elapsed_time(b) / (reps * len(calls))
    del g
    return ms


def _copies(nbytes: int, min_total: int = 320 << 20) -> int:
    return max(2, -(-min_total // max(nbytes, 1)))


def _rows_measurements(fp8mm, synthetic, peaks, only=None):
    """Per-row measurements of the other hot-path steps (each its own unit),
    timed by CUDA-graph replay over rotated operand copies (> L2 in total)."""
    import re
    import torch
    dev = torch.device("cuda")
    out = {}
    hbm = peaks["hbm_gbs"]
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    want = (lambda name: re.search(only, name) is not None) if only else (lambda name: True)

    if want("quantize_rowwise_8192x8192") or want("fp8_gemm_8192x2048x8192"):
        a, bt = synthetic.attn()
        a, bt = a.to(dev), bt.to(dev)
        R, Kq = a.shape
        if want("quantize_rowwise_8192x8192"):
            xs = [a] + [a.clone() for _ in range(_copies(a.numel() * 2) - 1)]
            qa = torch.empty(a.shape, dtype=torch.uint8, device=dev)
            sa = torch.empty(R, dtype=torch.float32, device=dev)
            t = _graph_time([lambda x=x: fp8mm.fp8_quantize_rowwise(x, qa, sa) for x in xs])
            gbs = (3.0 * R * Kq + 4 * R) / (t * 1e-3) / 1e9
            out["quantize_rowwise_8192x8192"] = {"ms": t, "GB/s": gbs, "frac_hbm": gbs / hbm}
            del xs
        if want("fp8_gemm_8192x2048x8192"):
            qa, sa = fp8mm.fp8_quantize_rowwise(a)
            qb, sb = fp8mm.fp8_quantize_rowwise(bt)
            c = torch.empty((R, bt.shape[0]), dtype=torch.bfloat16, device=dev)
            ws = torch.zeros(fp8mm.workspace_bytes(R, bt.shape[0], Kq), dtype=torch.uint8, device=dev)
            t = _graph_time([lambda: fp8mm.fp8_gemm(qa, qb, sa, sb, c, workspace=ws)] * 4)
            tf = 2.0 * 8192 * 2048 * 8192 / (t * 1e-3) / 1e12
            out["fp8_gemm_8192x2048x8192"] = {"ms": t, "TFLOPS": tf, "frac_fp8_peak": tf / fp8_peak}
        del a, bt

    if want("tensor_scale_8192x8192") or want("quantize_static_8192x8192") or want("fp8_gemm_e4m3_out_8192x2048x8192"):
        # per-tensor calibration scale, static-scale quantizer, GEMM with E4M3 output
        a, bt = synthetic.attn()
        a, bt = a.to(dev), bt.to(dev)
        R, Kq = a.shape
        xs = [a] + [a.clone() for _ in range(_copies(a.numel() * 2) - 1)]
        s_dev = torch.empty(1, dtype=torch.float32, device=dev)
        if want("tensor_scale_8192x8192"):
            t = _graph_time([lambda x=x: fp8mm.fp8_tensor_scale(x, s_dev) for x in xs])
            gbs = 2.0 * R * Kq / (t * 1e-3) / 1e9
            out["tensor_scale_8192x8192"] = {"ms": t, "GB/s": gbs, "frac_hbm": gbs / hbm}
        fp8mm.fp8_tensor_scale(a, s_dev)
        qa = torch.empty(a.shape, dtype=torch.uint8, device=dev)
        if want("quantize_static_8192x8192"):
            t = _graph_time([lambda x=x: fp8mm.fp8_quantize_static(x, s_dev, qa) for x in xs])
            gbs = 3.0 * R * Kq / (t * 1e-3) / 1e9
            out["quantize_static_8192x8192"] = {"ms": t, "GB/s": gbs, "frac_hbm": gbs / hbm}
        del xs
        if want("fp8_gemm_e4m3_out_8192x2048x8192"):
            qa, sa = fp8mm.fp8_quantize_rowwise(a)
            qb, sb = fp8mm.fp8_quantize_rowwise(bt)
            c8 = torch.empty((R, bt.shape[0]), dtype=torch.uint8, device=dev)
            so = torch.ones(1, dtype=torch.float32, device=dev)
            ws = torch.zeros(fp8mm.workspace_bytes(R, bt.shape[0], Kq), dtype=torch.uint8, device=dev)
            t = _graph_time([lambda: fp8mm.fp8_gemm_e4m3_out(qa, qb, sa, sb, so, c8, workspace=ws)] * 4)
            tf = 2.0 * 8192 * 2048 * 8192 / (t * 1e-3) / 1e12
            out["fp8_gemm_e4m3_out_8192x2048x8192"] = {"ms": t, "TFLOPS": tf, "frac_fp8_peak": tf / fp8_peak}
        del a, bt

    if want("concat_mla_k_16384x128"):
        # MLA key assembly in FP8: 16384 tokens x 128 heads, nope 128 + rope 64 (one per token)
        T, H = 16384, 128
        g = torch.Generator(device=dev).manual_seed(5)
        sets = []
        per = T * H * 128 + T * 64
        for _ in range(_copies(per)):
            nope = torch.randint(0, 256, (T, H, 128), device=dev, dtype=torch.uint8, generator=g)
            rope = torch.randint(0, 256, (T, 1, 64), device=dev, dtype=torch.uint8, generator=g)
            sets.append((nope.view(torch.float8_e4m3fn), rope.view(torch.float8_e4m3fn)))
        kout = torch.empty((T, H, 192), dtype=torch.float8_e4m3fn, device=dev)
        t = _graph_time([lambda n_=n_, r_=r_: fp8mm.concat_mla_k(n_, r_, kout) for n_, r_ in sets])
        byts = T * H * 128 + T * 64 + T * H * 192
        out["concat_mla_k_16384x128"] = {"ms": t, "GB/s": byts / (t * 1e-3) / 1e9,
                                         "frac_hbm": byts / (t * 1e-3) / 1e9 / hbm}
        del sets, kout

    if want("mxfp8_gemm_2048x1024x4096"):
        # Q.K^T shape: 64 output tiles, fewer than the 148 SMs
        a, bt = synthetic.qk()
        qa, sfa = fp8mm.mxfp8_quantize(a.to(dev))
        qb, sfb = fp8mm.mxfp8_quantize(bt.to(dev))
        c = torch.empty((2048, 1024), dtype=torch.bfloat16, device=dev)
        t = _graph_time([lambda: fp8mm.mxfp8_gemm(qa, sfa, qb, sfb, c)] * 8)
        tf = 2.0 * 2048 * 1024 * 4096 / (t * 1e-3) / 1e12
        out["mxfp8_gemm_2048x1024x4096"] = {"ms": t, "TFLOPS": tf, "frac_fp8_peak": tf / fp8_peak}

    if want("mxfp8_quantize_8192x8192"):
        # MX quantizer on the step's activation shape, standalone (inside the
        # step it follows the GEMM and shares HBM with the write-back of C)
        x, _ = synthetic.ffn_up()
        x = x.to(dev)
        xs = [x] + [x.clone() for _ in range(_copies(x.numel() * 2) - 1)]
        qx = torch.empty(x.shape, dtype=torch.uint8, device=dev)
        sfx = torch.empty(fp8mm.sf_bytes(*x.shape), dtype=torch.uint8, device=dev)
        t = _graph_time([lambda x_=x_: fp8mm.mxfp8_quantize(x_, qx, sfx) for x_ in xs])
        R, Kq = x.shape
        gbs = (3.0 * R * Kq + R * Kq / 32) / (t * 1e-3) / 1e9
        out["mxfp8_quantize_8192x8192"] = {"ms": t, "GB/s": gbs, "frac_hbm": gbs / hbm}
        del x, xs, qx, sfx

    if want("mxfp8_quantize_22016x8192"):
        # MX quantizer on the FFN weight (done once at load), standalone
        _, w = synthetic.ffn_up()
        w = w.to(dev)
        qw = torch.empty(w.shape, dtype=torch.uint8, device=dev)
        sfw = torch.empty(fp8mm.sf_bytes(*w.shape), dtype=torch.uint8, device=dev)
        t = _graph_time([lambda: fp8mm.mxfp8_quantize(w, qw, sfw)] * 2)
        R, Kq = w.shape
        gbs = (3.0 * R * Kq + R * Kq / 32) / (t * 1e-3) / 1e9
        out["mxfp8_quantize_22016x8192"] = {"ms": t, "GB/s": gbs, "frac_hbm": gbs / hbm}
        del w, qw, sfw

    # decode sweep: quantize X per call + small-M GEMM against a resident weight
    ws_, xs = synthetic.decode()
    sweep = {}
    for name, w in ws_.items():
        n, k = synthetic.DECODE_SHAPES[name]
        if not any(want(f"{name}_{n}x{k}_m{m}") for m in synthetic.DECODE_M):
            continue
        qw0, sfw0 = fp8mm.mxfp8_quantize(w.to(dev))
        copies = _copies(qw0.numel())
        wq = [(qw0, sfw0)] + [(qw0.clone(), sfw0.clone()) for _ in range(copies - 1)]
        for m in synthetic.DECODE_M:
            key = f"{name}_{n}x{k}_m{m}"
            if not want(key):
                continue
            x = xs[k][:m].contiguous().to(dev)
            qx = torch.empty((m, k), dtype=torch.uint8, device=dev)
            sfx = torch.empty(fp8mm.sf_bytes(m, k), dtype=torch.uint8, device=dev)
            c = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
            wsp = torch.zeros(fp8mm.workspace_bytes(m, n, k), dtype=torch.uint8, device=dev)

            # weights are quantized once, at load: the GEMM may stream them
            # while the activation quantizer before it is still running
            def call(qw, sfw):
                fp8mm.mxfp8_quantize(x, qx, sfx)
                fp8mm.mxfp8_gemm(qx, sfx, qw, sfw, c, workspace=wsp, weights_ready=True)
            t = _graph_time([lambda qw=qw, sfw=sfw: call(qw, sfw) for qw, sfw in wq])
            tg = _graph_time([lambda qw=qw, sfw=sfw: fp8mm.mxfp8_gemm(qx, sfx, qw, sfw, c, workspace=wsp,
                                                                      weights_ready=True)
                              for qw, sfw in wq])
            # the same step as one launch: activation quantized inside the GEMM
            wsq = torch.zeros(fp8mm.quantize_gemm_workspace_bytes(m, n, k), dtype=torch.uint8, device=dev)
            tf_ = _graph_time([lambda qw=qw, sfw=sfw: fp8mm.mxfp8_quantize_gemm(x, qw, sfw, c, workspace=wsq,
                                                                                weights_ready=True)
                               for qw, sfw in wq])
            e2e_bytes = n * k + n * k / 32 + 2 * m * k + 2 * m * n
            gemm_bytes = n * k + n * k / 32 + m * k + 128 * k / 32 + 2 * m * n
            sweep[key] = {"ms": t, "GB/s": e2e_bytes / (t * 1e-3) / 1e9, "frac_hbm": e2e_bytes / (t * 1e-3) / 1e9 / hbm,
                          "gemm_ms": tg, "gemm_GB/s": gemm_bytes / (tg * 1e-3) / 1e9,
                          "gemm_frac_hbm": gemm_bytes / (tg * 1e-3) / 1e9 / hbm,
                          "fused_ms": tf_, "fused_GB/s": e2e_bytes / (tf_ * 1e-3) / 1e9,
                          "fused_frac_hbm": e2e_bytes / (tf_ * 1e-3) / 1e9 / hbm}
        del wq
    if sweep:
        out["decode"] = sweep
    out["timing"] = "CUDA-graph replay, operands rotated over copies totalling > 320 MiB (no L2 reuse)"
    return out


def _rows_summary(rows):
    """The per-row roofline fractions at a glance: each quantizer and GEMM row's
    fraction, and the decode sweep's range per way of calling it."""
    out = {}
    for name, r in rows.items():
        if isinstance(r, dict) and "frac_hbm" in r:
            out[name] = {"frac_hbm": r["frac_hbm"]}
        elif isinstance(r, dict) and "frac_fp8_peak" in r:
            out[name] = {"frac_fp8_peak": r["frac_fp8_peak"]}
    dec = rows.get("decode")
    if dec:
        for key, label in (("gemm_frac_hbm", "decode_gemm_alone"), ("frac_hbm", "decode_quantize_then_gemm"),
                           ("fused_frac_hbm", "decode_quantize_gemm")):
            v = [c[key] for c in dec.values()]
            out[label] = {"frac_hbm_min": min(v), "frac_hbm_max": max(v), "cases": len(v)}
    return out


def _sustained(step, gemm, stream, local, pci, seconds: float = 3.0, k: int = 100):
    """The headline step back to back for `seconds` (the GPU settles at its
    power cap); then k more steps and k GEMM calls, each timed alone with CUDA
    events, with the clocks sampled meanwhile."""
    import torch
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < seconds:
        for _ in range(50):
            step()
        torch.cuda.synchronize()
        n += 50
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    def timed(f):
        out = []
        for _ in range(k):
            ev[0].record(stream)
            f()
            ev[1].record(stream)
            ev[1].synchronize()
            out.append(ev[0].elapsed_time(ev[1]))
        return out

    with ClockSampler(local, pci_bus_id=pci) as clocks:
        s_list = timed(step)
        g_list = timed(gemm)
    st, gm = percentiles(s_list), percentiles(g_list)
    return {"warm_seconds": seconds, "warm_steps": n, "calls_timed": k, "step_ms": st, "gemm_ms": gm["p50"],
            "gemm_ms_pct": gm, "TFLOPS_per_step": FLOPS_PER_STEP / (st["p50"] * 1e-3) / 1e12,
            "clocks": clocks.summary(),
            "note": "after several seconds of back-to-back steps (power cap); each call timed alone, median"}


def _best_of(torch, f, reps: int = 10):
    for _ in range(3):
        f()
    torch.cuda.synchronize()
    best = None
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        f()
        e1.record()
        e1.synchronize()
        t = e0.elapsed_time(e1)
        best = t if best is None else min(best, t)
    return best


def _yardstick(torch, dev, mx=None):
    """torch._scaled_mm (cuBLASLt FP8) on the same GPU in the same run: a
    library yardstick, not a target and not the roofline denominator.  mx =
    (qx, sfx, qw, sfw, ours): the step's own MXFP8 operands, whose scale
    layout is the one cuBLASLt reads for 1x32 UE8M0 block scales, timed
    through cuBLASLt and through our call `ours` in the same protocol."""
    out = {"what": "torch._scaled_mm e4m3 x e4m3 -> bf16, best of 10 calls after 3 warm-up calls; "
                   "a library yardstick, not a target"}
    if mx is not None:
        try:
            qx, sfx, qw, sfw, ours = mx
            m, k = qx.shape
            n = qw.shape[0]
            a8, b8 = qx.view(torch.float8_e4m3fn), qw.view(torch.float8_e4m3fn)
            sa, sb = sfx.view(torch.float8_e8m0fnu), sfw.view(torch.float8_e8m0fnu)
            f = lambda: torch._scaled_mm(a8, b8.t(), scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)
            ref = f()
            c = ours()
            torch.cuda.synchronize()
            diff = float((ref.float() - c.float()).abs().max())
            tl, to = _best_of(torch, f), _best_of(torch, ours)
            fl = 2.0 * m * n * k
            out[f"{m}x{n}x{k}_mxfp8_cublaslt"] = {"ms": tl, "TFLOPS": fl / (tl * 1e-3) / 1e12,
                                                  "max_abs_diff_vs_ours": diff}
            out[f"{m}x{n}x{k}_mxfp8_ours_same_protocol"] = {"ms": to, "TFLOPS": fl / (to * 1e-3) / 1e12}
            del ref, c
        except Exception as e:  # a library limitation is reported, not fatal
            out["mxfp8_error"] = f"{type(e).__name__}: {e}"[:200]
    try:
        shapes = {"8192x8192x8192_per_tensor": (8192, 8192, 8192, False),
                  "8192x22016x8192_rowwise": (8192, 22016, 8192, True),
                  "8192x2048x8192_rowwise": (8192, 2048, 8192, True)}
        for name, (m, n, k, rowwise) in shapes.items():
            a = torch.randn((m, k), device=dev).to(torch.float8_e4m3fn)
            b = torch.randn((n, k), device=dev).to(torch.float8_e4m3fn)
            sa = torch.ones((m, 1) if rowwise else (), device=dev)
            sb = torch.ones((1, n) if rowwise else (), device=dev)
            f = lambda: torch._scaled_mm(a, b.t(), scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)
            best = _best_of(torch, f)
            out[name] = {"ms": best, "TFLOPS": 2.0 * m * n * k / (best * 1e-3) / 1e12}
            del a, b
    except Exception as e:  # a library limitation is reported, not fatal
        out["error"] = f"{type(e).__name__}: {e}"[:200]
    return out


# ---------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    import torch.distributed as dist

    import mxfp8_block_scaled_fp8_b200 as fp8mm
    from mxfp8_block_scaled_fp8_b200 import synthetic

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))
    peaks = _peaks()

    x_cpu, w_cpu = synthetic.ffn_up()
    x = x_cpu.to(dev)
    w = w_cpu.to(dev)
    qw, sfw = fp8mm.mxfp8_quantize(w)              # weights quantized once, at load
    del w
    qx = torch.empty((M, K), dtype=torch.uint8, device=dev)
    sfx = torch.empty(fp8mm.sf_bytes(M, K), dtype=torch.uint8, device=dev)
    c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    # split-K workspace (zeroed once, reused by every call): the tiles of the
    # GEMM's last, partly filled wave of SM pairs run as K parts
    gws = torch.zeros(fp8mm.workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        fp8mm.mxfp8_quantize(x, qx, sfx)
        fp8mm.mxfp8_gemm(qx, sfx, qw, sfw, c, workspace=gws)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    pci = None
    if hasattr(props, "pci_bus_id"):
        pci = f"{getattr(props, 'pci_domain_id', 0):08X}:{props.pci_bus_id:02X}:{getattr(props, 'pci_device_id', 0):02X}.0"
    with ClockSampler(local, pci_bus_id=pci) as clocks:
        t_start.record(stream)
        for e0, e1, e2 in evs:
            e0.record(stream)
            fp8mm.mxfp8_quantize(x, qx, sfx)
            e1.record(stream)
            fp8mm.mxfp8_gemm(qx, sfx, qw, sfw, c, workspace=gws)
            e2.record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    q_list = [e0.elapsed_time(e1) for e0, e1, _ in evs]
    g_list = [e1.elapsed_time(e2) for _, e1, e2 in evs]
    s_list = [e0.elapsed_time(e2) for e0, _, e2 in evs]
    q_ms = sum(q_list) / args.steps
    g_ms = sum(g_list) / args.steps
    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps
    value = job_tflops(FLOPS_PER_STEP, args.steps, ws, total_ms)

    # end to end through the public API with host buffers, pipelined the way a
    # serving loop runs it: every step copies its X in from pinned host memory,
    # runs mxfp8_quantize + mxfp8_gemm, and copies its full C back to pinned
    # host memory, all inside the timed region.  The copies and the kernels
    # are on three streams with two device buffer sets, so step i+1's upload
    # and step i-1's readback overlap step i's kernels (PCIe is full duplex).
    e2e_steps = max(4, min(args.steps, 10))
    x_host = x_cpu.pin_memory()
    c_hosts = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_devs = [x, torch.empty_like(x)]
    c_devs = [c, torch.empty_like(c)]
    s_h2d, s_cmp, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n):
        h2d_ev = [torch.cuda.Event() for _ in range(n)]
        cmp_ev = [torch.cuda.Event() for _ in range(n)]
        d2h_ev = [torch.cuda.Event() for _ in range(n)]
        for i in range(n):
            b = i % 2
            if i >= 2:
                s_h2d.wait_event(cmp_ev[i - 2])            # x_devs[b] no longer read
            with torch.cuda.stream(s_h2d):
                x_devs[b].copy_(x_host, non_blocking=True)
                h2d_ev[i].record(s_h2d)
            s_cmp.wait_event(h2d_ev[i])
            if i >= 2:
                s_cmp.wait_event(d2h_ev[i - 2])            # c_devs[b] read back
            with torch.cuda.stream(s_cmp):
                fp8mm.mxfp8_quantize(x_devs[b], qx, sfx)
                fp8mm.mxfp8_gemm(qx, sfx, qw, sfw, c_devs[b], workspace=gws)
                cmp_ev[i].record(s_cmp)
            s_d2h.wait_event(cmp_ev[i])
            with torch.cuda.stream(s_d2h):
                c_hosts[b].copy_(c_devs[b], non_blocking=True)
                d2h_ev[i].record(s_d2h)

    torch.cuda.synchronize()
    e2e_run(2)                                          # warm-up
    torch.cuda.synchronize()
    a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a_ev.record(s_h2d)
    e2e_run(e2e_steps)
    b_ev.record(s_d2h)                                  # after every readback (each waited for its step)
    torch.cuda.synchronize()
    e2e_ms = a_ev.elapsed_time(b_ev) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dev)
    del x_devs, c_devs

    # the same step back to back for a few seconds: the GPU settles at its
    # power cap, where the short timed region above runs at burst clocks
    sustained = None
    if not args.no_sustained:
        sustained = _sustained(step, lambda: fp8mm.mxfp8_gemm(qx, sfx, qw, sfw, c, workspace=gws), stream, local,
                               pci)
    yard = None
    if rank == 0 and not args.no_rows:
        yard = _yardstick(torch, dev, (qx, sfx, qw, sfw, lambda: fp8mm.mxfp8_gemm(qx, sfx, qw, sfw, c, workspace=gws)))

    rows = None
    if rank == 0 and not args.no_rows:
        rows = _rows_measurements(fp8mm, synthetic, peaks, args.only)

    fp8_peak = 2.0 * peaks["bf16_tflops"]
    achieved = FLOPS_PER_STEP / (g_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": ws, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic (seeded N(0,1) X, N(0,0.02^2) W, 0.1% x20 outliers)",
        "config": {"workload": "ffn_up: X [8192,8192] bf16 -> mxfp8_quantize -> mxfp8_gemm with W [22016,8192] "
                               "pre-quantized MXFP8 (1x32 UE8M0), bf16 out",
                   "M": M, "N": N, "K": K, "parallelism": f"dp{ws} (independent replicas)",
                   "workspace": "split-K workspace given: the last partly filled wave of tiles runs as K parts",
                   "l2": "inputs larger than L2: X 128 MiB bf16 and Wq 172 MiB are re-read every step"},
        "e2e": {"value": job_tflops(FLOPS_PER_STEP, 1, ws, e2e_ms), "unit": "TFLOPS",
                "h2d_bytes_per_step": x_host.numel() * 2, "d2h_bytes_per_step": c_hosts[0].numel() * 2,
                "ms_per_step": e2e_ms, "steps": e2e_steps,
                "pipelining": "H2D, kernels and D2H on three streams with two device buffer sets"},
        "gpu_launches": 2 * args.steps,
        "kernels": {"mxfp8_quantize_ms": q_ms, "mxfp8_gemm_ms": g_ms},
        "per_step_ms": {"step": percentiles(s_list), "mxfp8_quantize": percentiles(q_list),
                        "mxfp8_gemm": percentiles(g_list),
                        "note": "CUDA events around each call of every timed step (nearest-rank percentiles)"},
        "roofline": {"bound": "tensor", "kernel": "gemm_pair_kernel<mx> (mxfp8_gemm, 256x256 tiles on 2-CTA clusters)", "achieved": achieved,
                     "peak": fp8_peak, "unit": "TFLOP/s", "frac": achieved / fp8_peak,
                     "traffic": _ncu_traffic("mxfp8_gemm_ffn_up"),
                     "frac_of_sustained": achieved / (2.0 * peaks["bf16_tflops_sustained"]),
                     "peak_note": f"FP8 dense = 2 x {peaks['source']} bf16 burst {peaks['bf16_tflops']} TFLOP/s "
                                  f"(nominal FP8/BF16 ratio); sustained-based peak "
                                  f"{2.0 * peaks['bf16_tflops_sustained']:.0f}",
                     "algorithmic": "2*M*N*K flops per launch"},
        "quantize_roofline": {"bound": "hbm", "achieved": (3.0 * M * K + M * K / 32) / (q_ms * 1e-3) / 1e9,
                              "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": (3.0 * M * K + M * K / 32) / (q_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                              "traffic": _ncu_traffic("mxfp8_quantize_x")},
        "clocks": clocks.summary(),
    }
    if sustained is not None:
        sustained["gemm_frac_of_burst_peak"] = FLOPS_PER_STEP / (sustained["gemm_ms"] * 1e-3) / 1e12 / fp8_peak
        sustained["gemm_frac_of_sustained_peak"] = (FLOPS_PER_STEP / (sustained["gemm_ms"] * 1e-3) / 1e12
                                                    / (2.0 * peaks["bf16_tflops_sustained"]))
        line["sustained"] = sustained
    if yard is not None:
        line["yardstick"] = yard
    if rank == 0 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(CPU_SAMPLE_ROWS, _oracle_workload(x_cpu, w_cpu))
        if not args.no_rows:
            line["cpu_baseline"]["per_config"] = cpu_per_config()
    if rows is not None:
        line["rows"] = rows
        line["rows_summary"] = _rows_summary(rows)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------- CPU oracle

def _oracle_workload(x=None, w=None):
    import oracle
    from mxfp8_block_scaled_fp8_b200 import synthetic
    if x is None:
        x, w = synthetic.ffn_up()
    qw, sfw = oracle.mx_quantize(synthetic.bits(w))   # weights quantized once (untimed, as on the GPU)
    return oracle, synthetic, x, qw, sfw


def _oracle_step(oracle, synthetic, x, qw, sfw, r0, rows, c0=0, cols=N):
    qx, sfx = oracle.mx_quantize(synthetic.bits(x[r0:r0 + rows]))
    oracle.gemm_mx(qx, sfx, qw[c0:c0 + cols], sfw[c0:c0 + cols], want_bound=False)


def cpu_baseline(rows: int, prepared=None):
    import oracle as _o
    oracle, synthetic, x, qw, sfw = prepared or _oracle_workload()
    t = time.perf_counter()
    _oracle_step(oracle, synthetic, x, qw, sfw, 0, rows)
    dt = time.perf_counter() - t
    return {"value": 2.0 * rows * N * K / dt / 1e12, "unit": "TFLOPS", "cores": min(_o.default_threads(), rows),
            "kind": "oracle", "seconds": dt,
            "sample": f"{rows} of {M} rows of the ffn_up step (mx-quantize those rows of X, then their full "
                      f"rows of C against all {N} columns, fp64 exact accumulation); W quantized beforehand"}


def cpu_per_config(gemm_sample_rows: int = 16):
    """The oracle timed on every configuration shape: the quantizer of each
    mode on every operand (rowwise for the per-token configurations, MX for
    the block-scaled ones; decode weights once, each activation per case), the
    GEMM in full for tiny, qk and every decode case, and on `gemm_sample_rows`
    full rows of C for attn and ffn_up (their full GEMMs take minutes)."""
    import oracle
    from mxfp8_block_scaled_fp8_b200 import synthetic as S
    out = {}

    def timed(name, f, units, unit, **extra):
        t = time.perf_counter()
        r = f()
        dt = time.perf_counter() - t
        out[name] = {"seconds": dt, unit: units / dt / 1e6 if unit == "Melem/s" else units / dt / 1e9, **extra}
        return r

    def rowwise_case(name, a, bt, sample):
        qa, sa = timed(f"{name}.quantize_rowwise_A", lambda: oracle.quantize_rowwise(S.bits(a)), a.numel(), "Melem/s")
        qb, sb = timed(f"{name}.quantize_rowwise_B", lambda: oracle.quantize_rowwise(S.bits(bt)), bt.numel(), "Melem/s")
        r = qa.shape[0] if sample is None else sample
        timed(f"{name}.gemm", lambda: oracle.gemm_rowwise(qa[:r], qb, sa[:r], sb, want_bound=False),
              r * qb.shape[0] * qa.shape[1], "GMAC/s", rows=f"{r} of {qa.shape[0]}")

    def mx_case(name, a, bt, sample):
        qa, sfa = timed(f"{name}.mx_quantize_A", lambda: oracle.mx_quantize(S.bits(a)), a.numel(), "Melem/s")
        qb, sfb = timed(f"{name}.mx_quantize_B", lambda: oracle.mx_quantize(S.bits(bt)), bt.numel(), "Melem/s")
        r = qa.shape[0] if sample is None else sample
        timed(f"{name}.gemm", lambda: oracle.gemm_mx(qa[:r], sfa[:r], qb, sfb, want_bound=False),
              r * qb.shape[0] * qa.shape[1], "GMAC/s", rows=f"{r} of {qa.shape[0]}")

    rowwise_case("tiny", *S.tiny(), None)
    mx_case("qk", *S.qk(), None)
    rowwise_case("attn", *S.attn(), gemm_sample_rows)
    mx_case("ffn_up", *S.ffn_up(), gemm_sample_rows)
    ws_, xs = S.decode()
    for name, w in ws_.items():
        n, k = S.DECODE_SHAPES[name]
        qw, sfw = timed(f"decode.{name}.mx_quantize_W", lambda: oracle.mx_quantize(S.bits(w)), w.numel(), "Melem/s")
        for m in S.DECODE_M:
            x = xs[k][:m]
            qx, sfx = timed(f"decode.{name}_m{m}.mx_quantize_X", lambda: oracle.mx_quantize(S.bits(x)), x.numel(),
                            "Melem/s")
            timed(f"decode.{name}_m{m}.gemm", lambda: oracle.gemm_mx(qx, sfx, qw, sfw, want_bound=False),
                  m * n * k, "GMAC/s", rows=f"{m} of {m}")
    out["_about"] = ("CPU oracle (plain C, fp64 exact accumulation) on the host cores; the same seeded bf16 inputs "
                     "as the GPU rows; 'rows' gives how much of C was computed")
    out["_cores"] = oracle.default_threads()
    return out


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    prepared = _oracle_workload()
    oracle, synthetic, x, qw, sfw = prepared
    def ref_step(i):
        r0 = (i * REF_ROWS_PER_STEP) % M
        c0 = (i * REF_COLS_PER_STEP) % (N - REF_COLS_PER_STEP + 1)
        _oracle_step(oracle, synthetic, x, qw, sfw, r0, REF_ROWS_PER_STEP, c0, REF_COLS_PER_STEP)

    for i in range(args.warmup):
        ref_step(i)
    t = time.perf_counter()
    for i in range(args.steps):
        ref_step(args.warmup + i)
    dt = time.perf_counter() - t
    value = 2.0 * REF_ROWS_PER_STEP * REF_COLS_PER_STEP * K * args.steps / dt / 1e12
    sample = (f"each step: a {REF_ROWS_PER_STEP} x {REF_COLS_PER_STEP} block of C of the ffn_up step "
              f"(mx-quantize those rows of X, exact fp64 dot products over all K = {K})")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": "ffn_up 8192x22016x8192 MXFP8 (CPU oracle, sampled rows)",
                                            "M": M, "N": N, "K": K},
            "cpu_baseline": {"kind": "oracle", "cores": min(oracle.default_threads(), REF_ROWS_PER_STEP),
                             "sample": sample, "value": value,
                             "unit": "TFLOPS"},
            "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-sustained", action="store_true", help="skip the sustained (power-cap) loop")
    ap.add_argument("--only", default=None, help="regex: measure only the matching per-row cases")
    ap.add_argument("--rows-only", action="store_true", help="skip the headline step (profiling of single rows)")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.rows_only:
        import torch
        import mxfp8_block_scaled_fp8_b200 as fp8mm
        from mxfp8_block_scaled_fp8_b200 import synthetic
        torch.cuda.set_device(0)
        print(json.dumps({"rows": _rows_measurements(fp8mm, synthetic, _peaks(), args.only)}), flush=True)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
