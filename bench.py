#!/usr/bin/env python
"""Throughput of the blockwise FP8 W8A8 linear layer on B200.

One step = one pass of the whole hot path over the prefill workload (X bf16 [8192, 4096] with an
RMSNorm weight, W bf16 [24576, 4096]):
    per-step weight requant (128x128 blocks, fp32 scales)  ->  fused RMSNorm + 1x128 token quant
    ->  block-scaled FP8 GEMM (bf16 out).
`value` is the linear layer's 2*M*N*K FLOPs per step over the device-timed step, summed over
ranks (each rank runs its own replica: weak scaling, no collective on the data path).  The other
rows of the path (E8M0 requant, requant sweep of a 36-layer model, decode GEMM, MoE grouped GEMM)
are timed separately and reported under "rows".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-rows]

`--impl reference` times the CPU oracle (plain C, all host cores) on a bounded sample of the same
workload; it is the deliberately slow baseline, not a GPU implementation.
"""
import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M_, N_, K_ = 8192, 24576, 4096
FLOPS = 2.0 * M_ * N_ * K_
GEMM_BYTES = M_ * K_ + N_ * K_ + (K_ // 128) * M_ * 4 + (N_ // 128) * (K_ // 128) * 4 + M_ * N_ * 2
METRIC = "blockwise W8A8 FP8 GEMM TFLOP/s (% FP8 peak); quant-kernel HBM GB/s (% peak)"
WORKLOAD = "prefill linear: RMSNorm+1x128 quant of X[8192,4096] -> GEMM with W[24576,4096] requantized (128x128, fp32 scales) every step"
L2_BYTES = 126 * 2 ** 20


def max_over_ranks(x, dist, device):
    """The maximum of a per-rank float over all ranks (identity on one rank).  Every rank must call
    it at the same point: it is a collective."""
    if dist is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world, ms_per_step):
    """Whole-job throughput: every rank runs one step of the workload (weak scaling), so the job
    does world x FLOPS per step in the slowest rank's step time."""
    return world * FLOPS / (ms_per_step / 1e3) / 1e12


def gemm_traffic_recorded():
    """DRAM bytes per launch of the dense GEMM on the bench's workload, as RECORDED from an ncu
    capture in profiles/k_gemm_w8a8_block_prefill.md (not a live counter of this run) -- only
    while the kernel source is the one that capture measured (else None)."""
    import hashlib
    here = os.path.dirname(os.path.abspath(__file__))
    src = os.path.join(here, "fp8_blockwise_w8a8_b200", "csrc", "gemm_kernel.cuh")
    prof = os.path.join(here, "profiles", "k_gemm_w8a8_block_prefill.md")
    try:
        text = open(prof).read()
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    vals = dict(line.split(":", 1) for line in text.splitlines()
                if line.startswith(("traffic_bytes_per_launch:", "source_sha256:")))
    if vals.get("source_sha256", "").strip() != sha:
        return None
    return int(vals["traffic_bytes_per_launch"].strip())


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm": p["hbm_gbs"], "bf16": p["bf16_tflops"],
                "bf16_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and clock-event reasons sampled during a timed window: through NVML every
    2 ms in a background thread (nvidia-smi every 20 ms where NVML is unavailable).  start()
    returns once the first sample is in; stop(window) keeps the samples whose timestamps fall
    inside the window (host epoch seconds)."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown"}

    def __init__(self, device):
        p = torch.cuda.get_device_properties(device)
        self.bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        self.proc = None
        self.file = None
        self.thread = None
        self.samples = []
        self.source = None

    def _nvml_loop(self, nv, h, mx):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = get_reasons(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
            except Exception:
                break
            self.samples.append((time.time(), float(sm), float(mx),
                                 {n for b, n in self.REASONS.items() if bits & b}, pw))
            time.sleep(0.002)

    def start(self):
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByPciBusId(self.bus)
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._stop = False
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h, mx), daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 5.0:
                time.sleep(0.001)
            if self.samples:
                self.source = "nvml, 2 ms"
                return
            self._stop = True
            self.thread.join()
            self.thread = None
        except Exception:
            self.thread = None
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.bus, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.file, stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi, 20 ms"
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        t0 = time.time()
        while time.time() - t0 < 10.0 and self.proc.poll() is None:
            if os.path.getsize(self.file.name) > 0:
                break
            time.sleep(0.01)

    def _smi_samples(self):
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.file.seek(0)
        rows = [ln.split(",") for ln in self.file.read().strip().splitlines() if ln.strip()]
        os.unlink(self.file.name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        parsed = []
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                parsed.append((ts, float(r[2]), float(r[3]),
                               {n for n, v in zip(names, r[6:10]) if v.lower() == "active"},
                               float(r[4]) if r[4].replace(".", "", 1).isdigit() else None))
            except ValueError:
                continue
        return parsed

    def stop(self, window=None):
        """window = (t_begin, t_end) in host epoch seconds: only samples inside it are used (all
        samples, flagged, if none falls inside)."""
        if self.thread is not None:
            self._stop = True
            self.thread.join()
            parsed = list(self.samples)
        elif self.proc is not None:
            parsed = self._smi_samples()
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        inside = parsed if window is None else \
            [p for p in parsed if window[0] - 0.001 <= p[0] <= window[1] + 0.001]
        out = {}
        if window is not None and not inside:
            inside = parsed
            out["window"] = "no sample inside the timed window; all samples"
        sm = [p[1] for p in inside]
        pw = [p[4] for p in inside if p[4] is not None]
        out.update({"sm_mhz": statistics.median(sm) if sm else None,
                    "sm_max_mhz": inside[-1][2] if inside else None,
                    "reasons": sorted(set().union(*[p[3] for p in inside])) if inside else [],
                    "samples": len(sm), "source": self.source,
                    "power_w_max": max(pw) if pw else None})
        return out


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------
def dev_bf16(a, device):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


class LinearStep:
    """Device buffers and the three calls of one step; every call goes through the C ABI."""

    def __init__(self, fq, x, gamma, w, eps):
        self.fq = fq
        self.x, self.gamma, self.w, self.eps = x, gamma, w, eps
        dev = x.device
        self.wq = torch.empty((N_, K_), dtype=torch.uint8, device=dev)
        self.sw = torch.empty((N_ // 128, K_ // 128), dtype=torch.float32, device=dev)
        self.aq = torch.empty((M_, K_), dtype=torch.uint8, device=dev)
        self.sa = torch.empty((K_ // 128, M_), dtype=torch.float32, device=dev)
        self.out = torch.empty((M_, N_), dtype=torch.bfloat16, device=dev)

    def run(self, ev=None):
        fq = self.fq
        if ev is not None:
            ev[0].record()
        fq.quant_weight_block(self.w, fq.FP8Q_SCALE_F32, out_q=self.wq, out_s=self.sw)
        if ev is not None:
            ev[1].record()
        fq.rmsnorm_quant_token(self.x, self.gamma, self.eps, out_q=self.aq, out_sa=self.sa)
        if ev is not None:
            ev[2].record()
        fq.gemm_w8a8_block(self.aq, self.sa, self.wq, self.sw, fq.FP8Q_SCALE_F32, out=self.out)
        if ev is not None:
            ev[3].record()


def e2e_pipelined(step, xh, wh, gh, oh, steps, warmup):
    """End-to-end step time (ms) through the public API with host buffers, double-buffered over
    three streams: step i+1's inputs (X, W, gamma) go host -> device on one stream and step i's
    output device -> host on another while step i's three calls run on the compute stream.  Every
    step moves its own inputs in and its whole output out; the timed span covers all three
    streams from the first copy-in to the last copy-out."""
    fq = step.fq
    dev = step.x.device
    bufs = [(step.x, step.w, step.gamma, step.out),
            (torch.empty_like(step.x), torch.empty_like(step.w), torch.empty_like(step.gamma),
             torch.empty_like(step.out))]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    cmp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]

    def launch(i):
        b = i & 1
        x, w, g, out = bufs[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(cmp_done[b])        # step i-2 has consumed this input set
            x.copy_(xh, non_blocking=True)
            w.copy_(wh, non_blocking=True)
            g.copy_(gh, non_blocking=True)
            h2d_done[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(h2d_done[b])
            if i >= 2:
                s_cmp.wait_event(d2h_done[b])       # step i-2's output has reached the host
            fq.quant_weight_block(w, fq.FP8Q_SCALE_F32, out_q=step.wq, out_s=step.sw)
            fq.rmsnorm_quant_token(x, g, step.eps, out_q=step.aq, out_sa=step.sa)
            fq.gemm_w8a8_block(step.aq, step.sa, step.wq, step.sw, fq.FP8Q_SCALE_F32, out=out)
            cmp_done[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[b])
            oh[b].copy_(out, non_blocking=True)
            d2h_done[b].record(s_out)

    def run(n):
        main = torch.cuda.current_stream()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        hold_gpu()
        t0.record(main)
        for s in (s_in, s_cmp, s_out):
            s.wait_event(t0)
        for i in range(n):
            launch(i)
        for s in (s_in, s_cmp, s_out):
            main.wait_stream(s)
        t1.record(main)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)
    run(max(2, warmup))
    ms = run(steps) / steps
    del bufs
    return ms


def hold_gpu():
    """Keep the GPU busy for ~25 ms so that the host can enqueue a timed batch ahead of it; the
    events then time device work only, never host launch overhead."""
    torch.cuda._sleep(50_000_000)


def timed_loop(fn, steps, warmup, flush=None):
    """Mean device time (ms) of fn over `steps` calls after `warmup`, with an event pair around
    each call on the current stream; `flush` (if given) runs between calls, outside the timed
    spans.  All calls are enqueued behind hold_gpu() and synchronized once at the end."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    hold_gpu()
    for a, b in ev:
        if flush is not None:
            flush()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) for a, b in ev]
    return statistics.mean(times), times


def measure_rows(fq, device, steps, warmup, pk):
    """The remaining rows of the hot path, each timed on its own workload."""
    from fp8_blockwise_w8a8_b200 import inputs
    rows = {}
    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    flush_rd = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=device)

    def flush():
        # write a buffer twice the size of L2, then read another one: the timed kernel starts
        # with none of its inputs in L2 and no dirty lines left to write back on its account
        flush_buf.fill_(1.0)
        flush_rd.sum()

    hbm = pk["hbm"]
    fp8_peak = 2.0 * pk["bf16"]

    # a1 / a2 on the prefill weight alone, L2 flushed between calls (inside the step the requant
    # also absorbs the write-back of the previous step's GEMM output)
    wp = torch.randn((N_, K_), device=device).mul_(0.02).to(torch.bfloat16)
    for fmt, name in ((fq.FP8Q_SCALE_F32, "a1_requant_f32_prefill_W_flushed"),
                      (fq.FP8Q_SCALE_E8M0, "a2_requant_e8m0_prefill_W_flushed")):
        qp, sp = fq.quant_weight_block(wp, fmt)
        ms, _ = timed_loop(lambda: fq.quant_weight_block(wp, fmt, out_q=qp, out_s=sp), steps,
                           warmup, flush)
        byts = N_ * K_ * 3 + sp.numel() * sp.element_size()
        rows[name] = {"ms": ms, "GB/s": byts / ms / 1e6, "frac": byts / ms / 1e6 / hbm,
                      "workload": "W [24576, 4096] alone"}
        del qp, sp
    del wp

    # requant sweep: all 252 weights of the 36-layer model, fp32 and E8M0 scales
    ws = [inputs.sweep_matrix(l, i, device) for l in range(inputs.SWEEP_LAYERS)
          for i in range(len(inputs.SWEEP_MATRICES))]
    qs = [torch.empty(w.shape, dtype=torch.uint8, device=device) for w in ws]
    elems = sum(w.numel() for w in ws)
    for fmt, name in ((fq.FP8Q_SCALE_F32, "a1_requant_sweep_f32"),
                      (fq.FP8Q_SCALE_E8M0, "a2_requant_sweep_e8m0")):
        ss = [torch.empty((w.shape[0] // 128, w.shape[1] // 128), device=device,
                          dtype=torch.float32 if fmt == fq.FP8Q_SCALE_F32 else torch.uint8)
              for w in ws]
        sbytes = sum(s.numel() * s.element_size() for s in ss)

        def sweep():
            for w, q, s in zip(ws, qs, ss):
                fq.quant_weight_block(w, fmt, out_q=q, out_s=s)
        ms, _ = timed_loop(sweep, max(3, steps // 4), max(1, warmup // 2))
        byts = elems * 3 + sbytes
        rows[name] = {"ms": ms, "bytes": byts, "GB/s": byts / ms / 1e6,
                      "frac": byts / ms / 1e6 / hbm, "launches": len(ws),
                      "workload": "36 layers x {q,k,v,o,gate,up,down}, 6.946 G bf16 weights"}
        del ss
    del qs
    torch.cuda.empty_cache()
    # the same sweep as one batched launch over all 252 weights
    for fmt, name in (("f32", "a1_requant_sweep_f32_batched"),
                      ("e8m0", "a2_requant_sweep_e8m0_batched")):
        batch = fq.WeightBatch(ws, fmt)
        sbytes = sum(s.numel() * s.element_size() for s in batch.s)
        ms, _ = timed_loop(batch.run, max(3, steps // 4), max(1, warmup // 2))
        byts = elems * 3 + sbytes
        rows[name] = {"ms": ms, "bytes": byts, "GB/s": byts / ms / 1e6,
                      "frac": byts / ms / 1e6 / hbm, "launches": 1,
                      "workload": "36 layers x {q,k,v,o,gate,up,down}, 6.946 G bf16 weights, "
                                  "one launch"}
        del batch
        torch.cuda.empty_cache()
    del ws
    torch.cuda.empty_cache()

    # decode: token quant of A [128, 4096] and GEMM with W [12288, 4096]
    d = inputs.decode_linear()
    a = dev_bf16(d["A"], device)
    w = dev_bf16(d["W"], device)
    wq, sw = fq.quant_weight_block(w, "f32")
    aq, sa = fq.rmsnorm_quant_token(a)
    out = torch.empty((128, 12288), dtype=torch.bfloat16, device=device)
    byts = 12288 * 4096 + 128 * 4096 + 128 * 32 * 4 + 96 * 32 * 4 + 128 * 12288 * 2
    fl = 2.0 * 128 * 12288 * 4096
    ms, _ = timed_loop(lambda: fq.gemm_w8a8_block(aq, sa, wq, sw, out=out), steps, warmup, flush)
    rows["a5_gemm_decode"] = {"ms": ms, "TFLOP/s": fl / ms / 1e9, "GB/s": byts / ms / 1e6,
                              "frac_hbm": byts / ms / 1e6 / hbm, "bound": "hbm", "splits": 1,
                              "workload": "M=128 N=12288 K=4096"}
    # decode down projection (long K, few tiles): split-K with the library's choice vs unsplit
    Md, Nd, Kd = 128, 4096, 12288
    ad = dev_bf16(inputs.randn_bf16((Md, Kd), 1.0, 90, 0), device)
    wd = dev_bf16(inputs.randn_bf16((Nd, Kd), 0.02, 90, 1), device)
    wqd, swd = fq.quant_weight_block(wd, "f32")
    aqd, sad = fq.rmsnorm_quant_token(ad)
    outd = torch.empty((Md, Nd), dtype=torch.bfloat16, device=device)
    wsd = fq.splitk_workspace(Md, Nd, Kd, 0, device=device)
    splits = max(1, wsd.numel() // (16 * 128 * 256 * 4))
    bd = Nd * Kd + Md * Kd + Md * (Kd // 128) * 4 + (Nd // 128) * (Kd // 128) * 4 + Md * Nd * 2
    fd = 2.0 * Md * Nd * Kd
    for name, fn, sp in (("a5_gemm_decode_down_splitk",
                          lambda: fq.gemm_w8a8_block_splitk(aqd, sad, wqd, swd, splits=0,
                                                            workspace=wsd, out=outd), splits),
                         ("a5_gemm_decode_down_unsplit",
                          lambda: fq.gemm_w8a8_block(aqd, sad, wqd, swd, out=outd), 1)):
        ms, _ = timed_loop(fn, steps, warmup, flush)
        rows[name] = {"ms": ms, "TFLOP/s": fd / ms / 1e9, "GB/s": bd / ms / 1e6,
                      "frac_hbm": bd / ms / 1e6 / hbm, "bound": "hbm", "splits": sp,
                      "workload": f"M={Md} N={Nd} K={Kd}"}
    del ad, wd, wqd, swd, aqd, sad, outd, wsd
    ms, _ = timed_loop(lambda: fq.rmsnorm_quant_token(a, out_q=aq, out_sa=sa), steps, warmup,
                       flush)
    byts = 128 * 4096 * 3 + 128 * 32 * 4
    rows["a3_token_quant_decode"] = {"ms": ms, "GB/s": byts / ms / 1e6,
                                     "frac": byts / ms / 1e6 / hbm, "workload": "A [128, 4096]"}
    del a, w, wq, sw, aq, sa, out

    # per-token x per-channel variant of the prefill linear: per-channel requant of W, fused
    # RMSNorm + per-token quant of X, and the per-channel GEMM (no per-K-block promotion)
    d = inputs.prefill_linear()
    x = dev_bf16(d["X"], device)
    gam = dev_bf16(d["gamma"], device)
    w = dev_bf16(d["W"], device)
    wq, sw = fq.quant_rowwise(w)
    aq, sa = fq.quant_rowwise(x, gam, d["eps"])
    out = torch.empty((M_, N_), dtype=torch.bfloat16, device=device)
    ms, _ = timed_loop(lambda: fq.quant_rowwise(w, out_q=wq, out_s=sw), steps, warmup)
    byts = N_ * K_ * 3 + N_ * 4
    rows["ptpc_weight_quant_prefill_W"] = {"ms": ms, "GB/s": byts / ms / 1e6,
                                           "frac": byts / ms / 1e6 / hbm,
                                           "workload": "W [24576, 4096], one scale per output channel"}
    ms, _ = timed_loop(lambda: fq.quant_rowwise(x, gam, d["eps"], out_q=aq, out_s=sa), steps,
                       warmup, flush)
    byts = M_ * K_ * 3 + M_ * 4 + K_ * 2
    rows["ptpc_rmsnorm_quant_prefill_X"] = {"ms": ms, "GB/s": byts / ms / 1e6,
                                            "frac": byts / ms / 1e6 / hbm,
                                            "workload": "X [8192, 4096], RMSNorm + one scale per token"}
    # residual add + RMSNorm + quant: x and the residual read, the new residual written, codes
    res = dev_bf16(inputs.randn_bf16((M_, K_), 1.0, 2, 7), device)
    for per_token, tag in ((False, "1x128"), (True, "per_token")):
        aq2 = torch.empty((M_, K_), dtype=torch.uint8, device=device)
        sa2 = (torch.empty((M_,), dtype=torch.float32, device=device) if per_token else
               torch.empty((K_ // 128, M_), dtype=torch.float32, device=device))
        ms, _ = timed_loop(lambda: fq.add_rmsnorm_quant(x, res, gam, d["eps"], per_token,
                                                        out_q=aq2, out_sa=sa2), steps, warmup,
                           flush)
        byts = M_ * K_ * 7 + sa2.numel() * 4 + K_ * 2
        rows[f"add_rmsnorm_quant_{tag}_prefill_X"] = {
            "ms": ms, "GB/s": byts / ms / 1e6, "frac": byts / ms / 1e6 / hbm,
            "workload": f"X, residual [8192, 4096] -> residual, codes ({tag} scales)"}
        del aq2, sa2
    del res
    ms, _ = timed_loop(lambda: fq.gemm_w8a8_rowwise(aq, sa, wq, sw, out=out), steps, warmup)
    rows["ptpc_gemm_prefill"] = {"ms": ms, "TFLOP/s": FLOPS / ms / 1e9,
                                 "frac_fp8": FLOPS / ms / 1e9 / fp8_peak,
                                 "frac_fp8_sustained": FLOPS / ms / 1e9 / (2.0 * pk["bf16_sustained"]),
                                 "workload": "M=8192 N=24576 K=4096, per-token x per-channel scales"}

    def ptpc_step():
        fq.quant_rowwise(w, out_q=wq, out_s=sw)
        fq.quant_rowwise(x, gam, d["eps"], out_q=aq, out_s=sa)
        fq.gemm_w8a8_rowwise(aq, sa, wq, sw, out=out)
    ms, _ = timed_loop(ptpc_step, steps, warmup)
    rows["ptpc_prefill_step"] = {"ms": ms, "TFLOP/s": FLOPS / ms / 1e9,
                                 "workload": "the prefill step with per-channel W and per-token X scales"}
    del x, gam, w, wq, sw, aq, sa, out
    torch.cuda.empty_cache()

    # MoE: token quant of the routed rows and the two grouped GEMMs
    mo = inputs.moe()
    off = torch.from_numpy(mo["offsets"]).to(device)
    R = int(mo["offsets"][-1])
    for key, wkey, name in (("A_gateup", "W_gateup", "gateup"), ("A_down", "W_down", "down")):
        a = dev_bf16(mo[key], device)
        W = dev_bf16(mo[wkey], device)
        E, N, K = W.shape
        wq, sw = fq.quant_weight_block(W.view(E * N, K), "f32")
        wq = wq.view(E, N, K)
        sw = sw.view(E, N // 128, K // 128)
        aq, sa = fq.rmsnorm_quant_token(a)
        ms_q, _ = timed_loop(lambda: fq.rmsnorm_quant_token(a, out_q=aq, out_sa=sa), steps,
                             warmup, flush)
        qbytes = R * K * 3 + R * (K // 128) * 4
        rows[f"a3_token_quant_moe_{name}"] = {"ms": ms_q, "GB/s": qbytes / ms_q / 1e6,
                                              "frac": qbytes / ms_q / 1e6 / hbm,
                                              "workload": f"A [{R}, {K}]"}
        out = torch.empty((R, N), dtype=torch.bfloat16, device=device)
        ms, _ = timed_loop(lambda: fq.grouped_gemm_w8a8_block(aq, sa, wq, sw, off, out=out),
                           steps, warmup, flush)
        fl = 2.0 * R * N * K
        byts = E * N * K + R * K + R * N * 2 + R * (K // 128) * 4 + E * (N // 128) * (K // 128) * 4
        rows[f"a6_grouped_gemm_moe_{name}"] = {
            "ms": ms, "TFLOP/s": fl / ms / 1e9, "frac_fp8": fl / ms / 1e9 / fp8_peak,
            "GB/s": byts / ms / 1e6, "frac_hbm": byts / ms / 1e6 / hbm,
            "workload": f"128 experts, {R} routed rows, N={N} K={K}"}
        del a, W, wq, sw, aq, sa, out
    torch.cuda.empty_cache()

    # the MoE FFN chain: quant of the routed rows -> grouped gate/up GEMM -> SiLU-and-mul + 1x128
    # quant -> grouped down GEMM (all on the device, in this library's kernels)
    a = dev_bf16(mo["A_gateup"], device)
    Wgu = dev_bf16(mo["W_gateup"], device)
    Wd = dev_bf16(mo["W_down"], device)
    E, Ngu, Kgu = Wgu.shape
    _, Nd, Kd = Wd.shape
    wq_gu, sw_gu = fq.quant_weight_block(Wgu.view(E * Ngu, Kgu), "f32")
    wq_gu, sw_gu = wq_gu.view(E, Ngu, Kgu), sw_gu.view(E, Ngu // 128, Kgu // 128)
    wq_d, sw_d = fq.quant_weight_block(Wd.view(E * Nd, Kd), "f32")
    wq_d, sw_d = wq_d.view(E, Nd, Kd), sw_d.view(E, Nd // 128, Kd // 128)
    aq, sa = fq.rmsnorm_quant_token(a)
    hgu = torch.empty((R, Ngu), dtype=torch.bfloat16, device=device)
    aq_d = torch.empty((R, Kd), dtype=torch.uint8, device=device)
    sa_d = torch.empty((Kd // 128, R), dtype=torch.float32, device=device)
    out_d = torch.empty((R, Nd), dtype=torch.bfloat16, device=device)
    fq.grouped_gemm_w8a8_block(aq, sa, wq_gu, sw_gu, off, out=hgu)
    ms, _ = timed_loop(lambda: fq.silu_mul_quant(hgu, out_q=aq_d, out_sa=sa_d), steps, warmup,
                       flush)
    byts = R * Ngu * 2 + R * Kd + R * (Kd // 128) * 4
    rows["silu_mul_quant_moe"] = {"ms": ms, "GB/s": byts / ms / 1e6, "frac": byts / ms / 1e6 / hbm,
                                  "workload": f"[gate | up] [{R}, {Ngu}] -> codes [{R}, {Kd}]"}
    ms, _ = timed_loop(lambda: fq.silu_mul_quant(hgu, out_q=aq_d, out_sa=sa_d, scale_fmt="e8m0"),
                       steps, warmup, flush)
    rows["silu_mul_quant_moe_e8m0"] = {
        "ms": ms, "GB/s": byts / ms / 1e6, "frac": byts / ms / 1e6 / hbm,
        "workload": f"[gate | up] [{R}, {Ngu}] -> codes [{R}, {Kd}], E8M0 scales"}

    def moe_chain():
        fq.rmsnorm_quant_token(a, out_q=aq, out_sa=sa)
        fq.grouped_gemm_w8a8_block(aq, sa, wq_gu, sw_gu, off, out=hgu)
        fq.silu_mul_quant(hgu, out_q=aq_d, out_sa=sa_d)
        fq.grouped_gemm_w8a8_block(aq_d, sa_d, wq_d, sw_d, off, out=out_d)
    ms, _ = timed_loop(moe_chain, steps, warmup, flush)
    fl = 2.0 * R * Ngu * Kgu + 2.0 * R * Nd * Kd
    rows["moe_ffn_chain"] = {"ms": ms, "TFLOP/s": fl / ms / 1e9,
                             "workload": f"128 experts, {R} routed rows: quant -> gate/up {Ngu}x{Kgu} "
                                         f"-> SiLU-and-mul quant -> down {Nd}x{Kd}",
                             "launches": 4}
    del a, Wgu, Wd, wq_gu, sw_gu, wq_d, sw_d, aq, sa, hgu, aq_d, sa_d, out_d
    torch.cuda.empty_cache()

    # attention output projection (wo_a): inverse RoPE + 1x128 quant, then the block-diagonal
    # GEMM over the head groups (E8M0 scales on both sides, as the page's MX-scaled GEMM)
    wa = inputs.wo_a()
    T, H, D = wa["o"].shape
    G, N_g, K_g = wa["W"].shape
    Kt = H * D
    o_d = dev_bf16(wa["o"], device)
    pos_d = torch.from_numpy(wa["positions"]).to(device)
    cos_d = torch.from_numpy(wa["cos"]).to(device)
    sin_d = torch.from_numpy(wa["sin"]).to(device)
    W = dev_bf16(wa["W"], device)
    wq, sw = fq.quant_weight_block(W.view(G * N_g, K_g), "e8m0")
    wq, sw = wq.view(G, N_g, K_g), sw.view(G, N_g // 128, K_g // 128)
    q_d = torch.empty((T, Kt), dtype=torch.uint8, device=device)
    sa_d = torch.empty((Kt // 128, T), dtype=torch.float32, device=device)
    out_d = torch.empty((T, G * N_g), dtype=torch.bfloat16, device=device)
    byts = T * Kt * 2 + T * Kt + T * (Kt // 128) * 4 + T * 8 + T * 64 * 4
    for fmt, tag in ((fq.FP8Q_SCALE_E8M0, "e8m0"), (fq.FP8Q_SCALE_F32, "f32")):
        ms, _ = timed_loop(lambda: fq.inverse_rope_quant(o_d, pos_d, cos_d, sin_d, 64, True, fmt,
                                                         out_q=q_d, out_sa=sa_d),
                           steps, warmup, flush)
        rows[f"inverse_rope_quant_wo_a_{tag}"] = {
            "ms": ms, "GB/s": byts / ms / 1e6, "frac": byts / ms / 1e6 / hbm,
            "workload": f"o [{T}, {H}, {D}] (64 rotary dims, interleaved) -> codes [{T}, {Kt}]"}
    fq.inverse_rope_quant(o_d, pos_d, cos_d, sin_d, 64, True, fq.FP8Q_SCALE_E8M0, out_q=q_d,
                          out_sa=sa_d)
    fl = 2.0 * T * G * N_g * K_g
    ms, _ = timed_loop(lambda: fq.gemm_w8a8_block_diag(q_d, sa_d, wq, sw, out=out_d), steps,
                       warmup, flush)
    rows["gemm_diag_wo_a"] = {"ms": ms, "TFLOP/s": fl / ms / 1e9,
                              "frac_fp8": fl / ms / 1e9 / fp8_peak,
                              "frac_fp8_sustained": fl / ms / 1e9 / (2.0 * pk["bf16_sustained"]),
                              "workload": f"{G} head groups: [{T}, {K_g}] x [{N_g}, {K_g}] each"}

    def wo_a_chain():
        fq.inverse_rope_quant(o_d, pos_d, cos_d, sin_d, 64, True, fq.FP8Q_SCALE_E8M0,
                              out_q=q_d, out_sa=sa_d)
        fq.gemm_w8a8_block_diag(q_d, sa_d, wq, sw, out=out_d)
    ms, _ = timed_loop(wo_a_chain, steps, warmup, flush)
    rows["wo_a_chain"] = {"ms": ms, "TFLOP/s": fl / ms / 1e9,
                          "workload": f"inverse RoPE quant -> {G}-group GEMM, {T} tokens",
                          "launches": 2}
    # the same GEMM with the scales applied by the tensor core (both scale sets powers of two)
    ms, _ = timed_loop(lambda: fq.gemm_w8a8_mx(q_d, sa_d, wq, sw, out=out_d), steps, warmup,
                       flush)
    rows["gemm_mx_wo_a"] = {"ms": ms, "TFLOP/s": fl / ms / 1e9,
                            "frac_fp8": fl / ms / 1e9 / fp8_peak,
                            "frac_fp8_sustained": fl / ms / 1e9 / (2.0 * pk["bf16_sustained"]),
                            "workload": f"{G} head groups: [{T}, {K_g}] x [{N_g}, {K_g}] each, "
                                        "hardware block scaling"}

    def wo_a_chain_mx():
        fq.inverse_rope_quant(o_d, pos_d, cos_d, sin_d, 64, True, fq.FP8Q_SCALE_E8M0,
                              out_q=q_d, out_sa=sa_d)
        fq.gemm_w8a8_mx(q_d, sa_d, wq, sw, out=out_d)
    ms, _ = timed_loop(wo_a_chain_mx, steps, warmup, flush)
    rows["wo_a_chain_mx"] = {"ms": ms, "TFLOP/s": fl / ms / 1e9,
                             "workload": f"inverse RoPE quant -> {G}-group MX GEMM, {T} tokens",
                             "launches": 2}
    del o_d, pos_d, cos_d, sin_d, W, wq, sw, q_d, sa_d, out_d
    torch.cuda.empty_cache()

    # FP8 KV cache: per-step recalibration of the per-tensor QKV scales, then the cache write
    kv = inputs.kv_cache()
    Hq, Hkv, Dh = kv["Hq"], kv["Hkv"], kv["D"]
    qkv = dev_bf16(kv["qkv"], device)
    T = qkv.shape[0]
    slots = torch.from_numpy(kv["slots"]).to(device)
    kc = torch.zeros((kv["num_slots"], Hkv * Dh), dtype=torch.uint8, device=device)
    vc = torch.zeros_like(kc)
    amax3 = torch.empty(3, dtype=torch.float32, device=device)
    sc3 = torch.empty(3, dtype=torch.float32, device=device)
    qo = torch.empty((T, Hq * Dh), dtype=torch.uint8, device=device)
    ms, _ = timed_loop(lambda: fq.qkv_scales(qkv, Hq, Hkv, Dh, out_amax=amax3, out_scales=sc3),
                       steps, warmup, flush)
    byts = qkv.numel() * 2
    rows["kv_qkv_scales_prefill"] = {"ms": ms, "GB/s": byts / ms / 1e6, "frac": byts / ms / 1e6 / hbm,
                                     "workload": f"QKV [{T}, {qkv.shape[1]}] -> 3 scales",
                                     "launches": 3}
    cached = int((kv["slots"] >= 0).sum())
    byts = qkv.numel() * 2 + T * 8 + T * Hq * Dh + cached * 2 * Hkv * Dh
    ms, _ = timed_loop(lambda: fq.kv_cache_write(qkv, Hq, Hkv, Dh, slots, sc3, kc, vc, out_q=qo),
                       steps, warmup, flush)
    rows["kv_cache_write_prefill"] = {
        "ms": ms, "GB/s": byts / ms / 1e6, "frac": byts / ms / 1e6 / hbm,
        "workload": f"{T} tokens, Q {Hq}x{Dh} quantized, K and V {Hkv}x{Dh} to cache slots"}
    dq = qkv[:256]
    ms, _ = timed_loop(lambda: fq.kv_cache_write(dq, Hq, Hkv, Dh, slots[:256], sc3, kc, vc,
                                                 out_q=qo[:256]), steps, warmup, flush)
    rows["kv_cache_write_decode"] = {"ms": ms, "workload": "256 decode tokens (launch-bound)"}
    del kv, qkv, slots, kc, vc, qo
    torch.cuda.empty_cache()

    # decode attention over the FP8 KV cache (the cache's reader): 64 sequences, contexts
    # U[512, 4096], 32 query / 8 kv heads of 128; the cache is written by the library first
    da = inputs.decode_attention(device=device)
    Hq, Hkv, Dh = da["Hq"], da["Hkv"], da["D"]
    S, Bd = da["num_slots"], da["q"].shape[0]
    rows_c = torch.cat([torch.zeros((S, Hq * Dh), dtype=torch.bfloat16, device=device),
                        da["k"], da["v"]], 1)
    _, s3 = fq.qkv_scales(rows_c, Hq, Hkv, Dh)
    kc = torch.empty((S, Hkv * Dh), dtype=torch.uint8, device=device)
    vc = torch.empty_like(kc)
    fq.kv_cache_write(rows_c, Hq, Hkv, Dh, torch.arange(S, device=device), s3, kc, vc,
                      quantize_q=False)
    del rows_c
    rows_q = torch.cat([da["q"], torch.zeros((Bd, 2 * Hkv * Dh), dtype=torch.bfloat16,
                                             device=device)], 1)
    qc = fq.kv_cache_write(rows_q, Hq, Hkv, Dh, -torch.ones(Bd, dtype=torch.int64, device=device),
                           s3, kc, vc)
    bt = torch.from_numpy(da["block_table"]).to(device)
    sl = torch.from_numpy(da["seq_lens"]).to(device)
    wsa = torch.empty(fq.attention_decode_workspace_bytes(Bd, Hq, Hkv, Dh, da["max_seq_len"]),
                      dtype=torch.uint8, device=device)
    oa = torch.empty((Bd, Hq * Dh), dtype=torch.bfloat16, device=device)
    ms, _ = timed_loop(lambda: fq.attention_decode(qc, kc, vc, s3, bt, sl, Hq, Hkv,
                                                   da["block_size"], da["max_seq_len"],
                                                   workspace=wsa, out=oa), steps, warmup, flush)
    npos = int(da["seq_lens"].sum())
    byts = npos * Hkv * Dh * 2 + Bd * Hq * Dh * 3     # K and V rows read, q codes, bf16 out
    rows["attention_decode_fp8kv"] = {
        "ms": ms, "GB/s": byts / ms / 1e6, "frac": byts / ms / 1e6 / hbm, "launches": 2,
        "workload": f"{Bd} sequences, {npos} cached positions (contexts U[512, 4096]), 32 query "
                    "/ 8 kv heads x 128, paged cache of 16-slot blocks"}
    del da, kc, vc, qc, bt, sl, wsa, oa, rows_q
    torch.cuda.empty_cache()

    # the prefill linear layer with power-of-two (E8M0) scales on both operands: the fused
    # RMSNorm + quant writes E8M0 activation scales, the weight requant E8M0 block scales, and
    # the GEMM applies both in the tensor core (hardware block scaling)
    pf = inputs.prefill_linear()
    X = dev_bf16(pf["X"], device)
    G = dev_bf16(pf["gamma"], device)
    W = dev_bf16(pf["W"], device)
    Mp, Kp = X.shape
    Np = W.shape[0]
    aq, sa = fq.rmsnorm_quant_token(X, G, pf["eps"], scale_fmt="e8m0")
    ms, _ = timed_loop(lambda: fq.rmsnorm_quant_token(X, G, pf["eps"], out_q=aq, out_sa=sa,
                                                      scale_fmt="e8m0"), steps, warmup, flush)
    byts = Mp * Kp * 3 + (Kp // 128) * Mp * 4 + Kp * 2
    rows["a4_rmsnorm_quant_e8m0_prefill_X"] = {
        "ms": ms, "GB/s": byts / ms / 1e6, "frac": byts / ms / 1e6 / hbm,
        "workload": "X [8192, 4096] -> codes + E8M0 1x128 scales (stored as fp32)"}
    xs = X.clone()
    ms, _ = timed_loop(lambda: fq.rmsnorm_quant_token(xs, None, out_q=aq, out_sa=sa,
                                                      scale_fmt="e8m0"), steps, warmup, flush)
    byts = Mp * Kp * 3 + (Kp // 128) * Mp * 4
    rows["a3_token_quant_e8m0_prefill_X"] = {
        "ms": ms, "GB/s": byts / ms / 1e6, "frac": byts / ms / 1e6 / hbm,
        "workload": "plain 1x128 quant of X [8192, 4096], E8M0 scales"}
    del xs
    aq, sa = fq.rmsnorm_quant_token(X, G, pf["eps"], scale_fmt="e8m0")
    wq, sw = fq.quant_weight_block(W, "e8m0")
    out = torch.empty((Mp, Np), dtype=torch.bfloat16, device=device)
    fl = 2.0 * Mp * Np * Kp

    def e8m0_step():
        fq.quant_weight_block(W, "e8m0", out_q=wq, out_s=sw)
        fq.rmsnorm_quant_token(X, G, pf["eps"], out_q=aq, out_sa=sa, scale_fmt="e8m0")
        fq.gemm_w8a8_mx(aq, sa, wq, sw, out=out)
    ms, _ = timed_loop(e8m0_step, steps, warmup)
    rows["e8m0_prefill_step"] = {
        "ms": ms, "TFLOP/s": fl / ms / 1e9, "launches": 3,
        "workload": "prefill linear with E8M0 scales: requant W (E8M0) -> RMSNorm + 1x128 quant "
                    "of X (E8M0) -> hardware block-scaled GEMM, bf16 out"}
    ms, _ = timed_loop(lambda: fq.gemm_w8a8_mx(aq, sa, wq, sw, out=out), steps, warmup)
    rows["gemm_mx_prefill"] = {"ms": ms, "TFLOP/s": fl / ms / 1e9,
                               "frac_fp8": fl / ms / 1e9 / fp8_peak,
                               "frac_fp8_sustained": fl / ms / 1e9 / (2.0 * pk["bf16_sustained"]),
                               "workload": f"M={Mp} N={Np} K={Kp}, E8M0 scales, hardware block "
                                           "scaling"}
    sw32 = torch.ldexp(torch.ones_like(sw, dtype=torch.float32), sw.to(torch.int32) - 127)
    ms, _ = timed_loop(lambda: fq.gemm_w8a8_block(aq, sa, wq, sw32, out=out), steps, warmup)
    rows["gemm_sw_promotion_prefill_pow2"] = {
        "ms": ms, "TFLOP/s": fl / ms / 1e9,
        "workload": f"M={Mp} N={Np} K={Kp}, the same power-of-two scales, software promotion"}
    del X, G, W, aq, sa, wq, sw, sw32, out
    torch.cuda.empty_cache()
    return rows


GEMM_SAMPLE_ROWS = 64      # output rows of the fp64 GEMM reference in the oracle's step sample
QUANT_SAMPLE_ROWS = 1024   # weight rows requantized and token rows normalised + quantized


def cpu_baseline_sample():
    """Time the oracle, as it stands, on a bounded sample of one step of the workload and scale
    it to the step.  Returns (value TFLOP/s, cores, sample description, seconds spent)."""
    import oracle
    from fp8_blockwise_w8a8_b200 import inputs
    oracle.lib()
    n_w = n_x = QUANT_SAMPLE_ROWS
    d = inputs.prefill_linear(M=n_x, N=n_w, K=K_)
    t0 = time.perf_counter()
    wq, sw = oracle.quant_weight_block(d["W"], oracle.SCALE_F32)
    t1 = time.perf_counter()
    aq, sa = oracle.rmsnorm_quant_token(d["X"], d["gamma"], d["eps"])
    t2 = time.perf_counter()
    rows = np.linspace(0, n_x - 1, GEMM_SAMPLE_ROWS).astype(np.int64)
    oracle.gemm_w8a8_block(aq, sa, wq, sw, oracle.SCALE_F32, rows=rows)
    t3 = time.perf_counter()
    step_s = ((t1 - t0) * (N_ / n_w) + (t2 - t1) * (M_ / n_x) +
              (t3 - t2) * (M_ / len(rows)) * (N_ / n_w))
    sample = (f"oracle on a sample of one step: requant of {n_w} of {N_} weight rows, "
              f"RMSNorm+quant of {n_x} of {M_} token rows, fp64 GEMM reference of "
              f"{len(rows)} output rows x {n_w} columns; each part scaled linearly to the full "
              "step (the per-step time is extrapolated from this sample)")
    return FLOPS / step_s / 1e12, oracle.num_threads(), sample, t3 - t0


def cpu_rows():
    """The oracle timed on each configuration as the CPU-baseline plan sets out: the decode
    linear in full, the prefill linear and the MoE FFN on sampled rows, the requant sweep as its
    layer 0 (x 36 layers).  Rates are of the sampled work; the sample is stated per row."""
    import oracle
    from fp8_blockwise_w8a8_b200 import inputs
    oracle.lib()
    out = {"cores": oracle.num_threads()}

    def timed(fn):
        t0 = time.perf_counter()
        r = fn()
        return r, time.perf_counter() - t0

    # decode linear [128, 4096] x [12288, 4096], in full
    d = inputs.decode_linear()
    (aq, sa), ta = timed(lambda: oracle.quant_token_1x128(d["A"]))
    (wq, sw), tw = timed(lambda: oracle.quant_weight_block(d["W"], oracle.SCALE_F32))
    _, tg = timed(lambda: oracle.gemm_w8a8_block(aq, sa, wq, sw, oracle.SCALE_F32))
    M, K = d["A"].shape
    N = d["W"].shape[0]
    out["decode_linear"] = {"sample": "in full", "token_quant_s": ta, "requant_s": tw,
                            "gemm_s": tg, "gemm_GFLOP/s": 2.0 * M * N * K / tg / 1e9,
                            "requant_GB/s": N * K * 3 / tw / 1e9}
    del d, aq, sa, wq, sw
    # prefill linear: quant of 1024 of the rows, GEMM reference of 64 rows x all 24576 columns
    d = inputs.prefill_linear()
    xs = np.ascontiguousarray(d["X"][:QUANT_SAMPLE_ROWS])
    (aq_s, sa_s), tx = timed(lambda: oracle.rmsnorm_quant_token(xs, d["gamma"], d["eps"]))
    (wq, sw), tw = timed(lambda: oracle.quant_weight_block(d["W"], oracle.SCALE_F32))
    rows = np.linspace(0, QUANT_SAMPLE_ROWS - 1, GEMM_SAMPLE_ROWS).astype(np.int64)
    _, tg = timed(lambda: oracle.gemm_w8a8_block(aq_s, sa_s, wq, sw, oracle.SCALE_F32,
                                                 rows=rows))
    out["prefill_linear"] = {
        "sample": f"RMSNorm+quant of {QUANT_SAMPLE_ROWS} of {M_} rows; requant of all of W; "
                  f"GEMM reference of {GEMM_SAMPLE_ROWS} rows x {N_} columns",
        "rmsnorm_quant_GB/s": QUANT_SAMPLE_ROWS * K_ * 3 / tx / 1e9,
        "requant_GB/s": N_ * K_ * 3 / tw / 1e9,
        "gemm_GFLOP/s": 2.0 * GEMM_SAMPLE_ROWS * N_ * K_ / tg / 1e9,
        "step_s_extrapolated": tx * M_ / QUANT_SAMPLE_ROWS + tw + tg * M_ / GEMM_SAMPLE_ROWS}
    del d, wq, sw
    # requant sweep: layer 0 of the 36-layer model in both scale formats, x 36
    ws = [inputs.sweep_matrix(0, i).view(torch.int16).numpy().view(np.uint16)
          for i in range(len(inputs.SWEEP_MATRICES))]
    elems = sum(w.size for w in ws)
    for fmt, name in ((oracle.SCALE_F32, "requant_sweep_f32"),
                      (oracle.SCALE_E8M0, "requant_sweep_e8m0")):
        _, t = timed(lambda: [oracle.quant_weight_block(w, fmt) for w in ws])
        out[name] = {"sample": "layer 0 (7 weights), time x 36 for the sweep",
                     "GB/s": elems * 3 / t / 1e9, "sweep_s_extrapolated": 36 * t}
    del ws
    # MoE FFN: 1024 of the 32768 routed rows through quant -> gate/up -> quant -> down
    d = inputs.moe()
    off = d["offsets"]
    sel = np.linspace(0, int(off[-1]) - 1, QUANT_SAMPLE_ROWS).astype(np.int64)
    t_all = 0.0
    fl = 0.0
    for a_key, w_key in (("A_gateup", "W_gateup"), ("A_down", "W_down")):
        W = d[w_key]
        E, Nm, Km = W.shape
        (aq, sa), t1 = timed(lambda: oracle.quant_token_1x128(np.ascontiguousarray(d[a_key][sel])))
        wq, sw = oracle.quant_weight_block(W.reshape(E * Nm, Km), oracle.SCALE_F32)
        # the sampled rows keep their experts: offsets of the sample within the sorted rows
        soff = np.searchsorted(sel, off).astype(np.int32)
        _, t2 = timed(lambda: oracle.grouped_gemm_w8a8_block(
            aq, sa, wq.reshape(E, Nm, Km), sw.reshape(E, Nm // 128, Km // 128), soff,
            oracle.SCALE_F32))
        t_all += t1 + t2
        fl += 2.0 * len(sel) * Nm * Km
    out["moe_ffn"] = {"sample": f"{QUANT_SAMPLE_ROWS} of {int(off[-1])} routed rows (token quant "
                                "and grouped GEMM, gate/up then down)",
                      "GFLOP/s": fl / t_all / 1e9, "seconds": t_all}
    return out


def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    from fp8_blockwise_w8a8_b200 import build as cuda_build
    if rank == 0 or world == 1:
        cuda_build.build()
    if dist is not None:
        dist.barrier()
    import fp8_blockwise_w8a8_b200 as fq
    from fp8_blockwise_w8a8_b200 import inputs

    pk = peaks()
    d = inputs.prefill_linear()
    x = dev_bf16(d["X"], device)
    gamma = dev_bf16(d["gamma"], device)
    w = dev_bf16(d["W"], device)
    step = LinearStep(fq, x, gamma, w, d["eps"])
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    if fq.check_device_error() != 0:
        raise SystemExit("device error during warm-up")

    # --- device-timed region: inputs resident in HBM; the step's working set (X 67 MB, W 201 MB,
    # codes 134 MB, out 403 MB) exceeds L2, so consecutive steps do not reuse cached data.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(device)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    hold_gpu()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for i in range(args.steps):
        step.run(evs[i])
    t_end.record()
    torch.cuda.synchronize()
    t_host_end = time.time()
    ms_local = t_start.elapsed_time(t_end)
    clk = clocks.stop((t_host_end - ms_local / 1000.0, t_host_end))
    if dist is not None:
        dist.barrier()
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), dist, device)
    ms_step = ms_total / args.steps
    k_req = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    k_rms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    k_gemm = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    if fq.check_device_error() != 0:
        raise SystemExit("device error during the timed region")

    # --- clock soak: the same step back to back for >= 1 s of device time, after the timed
    # region and outside it, so that the clock record covers a window long enough to show
    # power capping (the K-step region above may last only tens of ms).  Reported beside the
    # K-step numbers, never in place of them.
    soak_n = max(args.steps, int(math.ceil(1000.0 / max(ms_step, 1e-3))) + 1)
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(soak_n)]
    sclocks = ClockSampler(device)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sclocks.start()
    hold_gpu()
    s_start = torch.cuda.Event(enable_timing=True)
    s_end = torch.cuda.Event(enable_timing=True)
    s_start.record()
    for i in range(soak_n):
        step.run(sev[i])
    s_end.record()
    torch.cuda.synchronize()
    s_host_end = time.time()
    s_ms = s_start.elapsed_time(s_end)
    sclk = sclocks.stop((s_host_end - s_ms / 1000.0, s_host_end))
    s_ms = max_over_ranks(s_ms, dist, device)
    soak_gemm = statistics.mean(e[2].elapsed_time(e[3]) for e in sev)
    soak_rms = statistics.mean(e[1].elapsed_time(e[2]) for e in sev)
    soak_req = statistics.mean(e[0].elapsed_time(e[1]) for e in sev)
    del sev
    if fq.check_device_error() != 0:
        raise SystemExit("device error during the clock soak")

    # --- end to end through the public API with host buffers
    xh = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    xh.copy_(x)
    wh = torch.empty(w.shape, dtype=w.dtype, pin_memory=True)
    wh.copy_(w)
    gh = torch.empty(gamma.shape, dtype=gamma.dtype, pin_memory=True)
    gh.copy_(gamma)
    oh = [torch.empty(step.out.shape, dtype=step.out.dtype, pin_memory=True) for _ in range(2)]

    def e2e_step():           # the same step with its copies in order on one stream
        x.copy_(xh, non_blocking=True)
        w.copy_(wh, non_blocking=True)
        gamma.copy_(gh, non_blocking=True)
        step.run()
        oh[0].copy_(step.out, non_blocking=True)
    e2e_steps = max(3, args.steps // 2)
    ms_serial, _ = timed_loop(e2e_step, e2e_steps, max(1, args.warmup // 2))
    ms_serial = max_over_ranks(ms_serial, dist, device)
    ms_e2e = e2e_pipelined(step, xh, wh, gh, oh, e2e_steps, args.warmup)
    ms_e2e = max_over_ranks(ms_e2e, dist, device)
    h2d = xh.numel() * 2 + wh.numel() * 2 + gh.numel() * 2
    d2h = oh[0].numel() * 2

    rows = {}
    req_bytes = N_ * K_ * 3 + (N_ // 128) * (K_ // 128) * 4
    rms_bytes = M_ * K_ * 3 + (K_ // 128) * M_ * 4 + K_ * 2
    fp8_peak_burst = 2.0 * pk["bf16"]
    fp8_peak_sus = 2.0 * pk["bf16_sustained"]
    # the K-step window is short; its clocks decide which measured peak applies to it
    capped = bool(clk.get("reasons")) and "sw_power_cap" in clk["reasons"]
    fp8_peak = fp8_peak_sus if capped else fp8_peak_burst
    rows["a1_requant_f32_prefill_W"] = {"ms": k_req, "GB/s": req_bytes / k_req / 1e6,
                                        "frac": req_bytes / k_req / 1e6 / pk["hbm"]}
    rows["a4_rmsnorm_quant_prefill_X"] = {"ms": k_rms, "GB/s": rms_bytes / k_rms / 1e6,
                                          "frac": rms_bytes / k_rms / 1e6 / pk["hbm"]}
    rows["a5_gemm_prefill"] = {"ms": k_gemm, "TFLOP/s": FLOPS / k_gemm / 1e9,
                               "frac": FLOPS / k_gemm / 1e9 / fp8_peak}
    launches = 3 * args.steps
    if args.rows and world == 1:
        rows.update(measure_rows(fq, device, args.steps, args.warmup, pk))
    if dist is not None:
        dist.barrier()

    line = None
    if rank == 0:
        cpu = None
        if world == 1:
            samples = [cpu_baseline_sample() for _ in range(3)]
            cpu_v = statistics.median(v[0] for v in samples)
            cores, sample = samples[0][1], samples[0][2]
            cpu = {"value": cpu_v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                   "sample": sample + "; median of 3 runs",
                   "runs": [v[0] for v in samples]}
            if args.rows:
                cpu["rows"] = cpu_rows()
        gemm_tf = FLOPS / k_gemm / 1e9
        line = {
            "metric": METRIC,
            "value": whole_job_tflops(world, ms_step),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "e4m3 x e4m3 -> f32 accumulate, bf16 in/out",
            "data": "synthetic (seeded N(0,1) activations, U(0.5,1.5) gamma, N(0,0.02) weights)",
            "config": {"workload": WORKLOAD, "M": M_, "N": N_, "K": K_,
                       "weight_scales": "fp32 128x128", "act_scales": "fp32 1x128",
                       "parallelism": f"{world} independent replicas" if world > 1 else "1 GPU",
                       "l2": "inputs larger than L2 (step working set 0.8 GB > 126 MB)",
                       "rows_l2": "rows: between timed calls write 2 x L2 then read another 2 x L2 buffer (flush, no dirty lines left)"},
            "roofline": {"bound": "tensor", "achieved": gemm_tf, "peak": fp8_peak,
                         "unit": "TFLOP/s", "frac": gemm_tf / fp8_peak,
                         "traffic": None,
                         "traffic_recorded": gemm_traffic_recorded(),
                         "traffic_recorded_note": "DRAM bytes per launch recorded from the ncu "
                                                  "capture in profiles/k_gemm_w8a8_block_prefill.md "
                                                  "(read, not measured in this run); null once the "
                                                  "kernel source differs from the captured one",
                         "algorithmic_bytes": GEMM_BYTES,
                         "kernel": "k_gemm_w8a8_block<false>",
                         "peak_source": (f"{pk['source']}: 2 x {'sustained' if capped else 'burst'} "
                                         f"cuBLAS bf16 ({pk['bf16_sustained'] if capped else pk['bf16']}"
                                         " TFLOP/s), the fp8/bf16 nominal ratio; "
                                         + ("sw_power_cap seen in the window" if capped else
                                            "no power cap in the K-step window")),
                         "sustained": {
                             "achieved": FLOPS / soak_gemm / 1e9, "peak": fp8_peak_sus,
                             "frac": FLOPS / soak_gemm / 1e9 / fp8_peak_sus,
                             "window": f"clock soak: {soak_n} steps back to back, "
                                       f"{s_ms / 1000.0:.2f} s of device time",
                             "peak_source": f"{pk['source']}: 2 x sustained cuBLAS bf16 "
                                            f"({pk['bf16_sustained']} TFLOP/s)"}},
            "roofline_quant": {
                "bound": "hbm", "unit": "GB/s", "peak": pk["hbm"],
                "peak_source": f"{pk['source']} HBM copy bandwidth",
                "a4_rmsnorm_quant": {"kernel": "k_rmsnorm_quant_token<true>",
                                     "algorithmic_bytes": rms_bytes, "ms": k_rms,
                                     "achieved": rms_bytes / k_rms / 1e6,
                                     "frac": rms_bytes / k_rms / 1e6 / pk["hbm"]},
                "a1_requant": {"kernel": "k_quant_weight_block<fp32>",
                               "algorithmic_bytes": req_bytes, "ms": k_req,
                               "achieved": req_bytes / k_req / 1e6,
                               "frac": req_bytes / k_req / 1e6 / pk["hbm"]}},
            "soak": {"steps": soak_n, "seconds": s_ms / 1000.0,
                     "ms_per_step": s_ms / soak_n, "gemm_ms": soak_gemm, "a4_ms": soak_rms,
                     "a1_ms": soak_req, "clocks": sclk,
                     "note": "the same step back to back for >= 1 s after the K-step timed "
                             "region (not part of value); its clock record shows the "
                             "sustained state"},
            "e2e": {"value": whole_job_tflops(world, ms_e2e), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": ms_e2e,
                    "pipeline": "double-buffered: copy-in of step i+1 and copy-out of step i "
                                "overlap step i's calls (three streams)",
                    "serial_ms_per_step": ms_serial},
            "cpu_baseline": cpu,
            "clocks": clk,
            "gpu_launches": launches,
            "rows": rows,
        }
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------
# reference arm: the CPU oracle, as it stands
# ---------------------------------------------------------------------------------------------
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    for _ in range(args.warmup):
        cpu_baseline_sample()
    vals, spent = [], 0.0
    for _ in range(args.steps):
        v, cores, sample, s = cpu_baseline_sample()
        vals.append(v)
        spent += s
    value = statistics.mean(vals)
    ms_step = FLOPS / (value * 1e12) * 1e3
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64 reference (E4M3 codes, fp32 scales)",
        "data": "synthetic (seeded, same recipe as the GPU arm)",
        "config": {"workload": WORKLOAD, "M": M_, "N": N_, "K": K_,
                   "weight_scales": "fp32 128x128", "act_scales": "fp32 1x128",
                   "parallelism": "host cores (rank 0 only)",
                   "timing": "each step is a bounded sample of the workload timed on the host "
                             "cores; ms_per_step is extrapolated linearly from it (see "
                             "cpu_baseline.sample), it is not a measured full step"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ncu_case(name):
    """A few launches of one kernel on a case sized for an Nsight Compute capture (inputs larger
    than L2, a few hundred MB on the device): 2 warm-up launches, then 3 more."""
    import fp8_blockwise_w8a8_b200 as fq
    from fp8_blockwise_w8a8_b200 import inputs
    fq._lib.lib()
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(7)

    def randn(shape, std):
        return (torch.randn(shape, generator=g, device=dev) * std).to(torch.bfloat16)
    if name == "gemm_prefill":           # M=4096 of the prefill GEMM: A 16 MB, W 100 MB, out 201 MB
        aq, sa = fq.rmsnorm_quant_token(randn((4096, K_), 1.0))
        wq, sw = fq.quant_weight_block(randn((N_, K_), 0.02), "f32")
        out = torch.empty((4096, N_), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.gemm_w8a8_block(aq, sa, wq, sw, out=out)
    elif name == "gemm_prefill_full":    # the bench's GEMM launch: M=8192 (A 34 MB, W 101 MB, out 403 MB)
        aq, sa = fq.rmsnorm_quant_token(randn((M_, K_), 1.0))
        wq, sw = fq.quant_weight_block(randn((N_, K_), 0.02), "f32")
        out = torch.empty((M_, N_), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.gemm_w8a8_block(aq, sa, wq, sw, out=out)
    elif name == "gemm_decode":
        aq, sa = fq.rmsnorm_quant_token(randn((128, K_), 1.0))
        wq, sw = fq.quant_weight_block(randn((12288, K_), 0.02), "f32")
        out = torch.empty((128, 12288), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.gemm_w8a8_block(aq, sa, wq, sw, out=out)
    elif name == "gemm_decode_splitk":
        aq, sa = fq.rmsnorm_quant_token(randn((128, K_), 1.0))
        wq, sw = fq.quant_weight_block(randn((12288, K_), 0.02), "f32")
        out = torch.empty((128, 12288), dtype=torch.bfloat16, device=dev)
        ws = fq.splitk_workspace(128, 12288, K_, 0, device=dev)
        fn = lambda: fq.gemm_w8a8_block_splitk(aq, sa, wq, sw, splits=0, workspace=ws, out=out)
    elif name == "rmsnorm_prefill":      # X [8192, 4096]: 67 MB in, 35 MB out
        x = randn((M_, K_), 1.0)
        gam = randn((K_,), 0.5) + 1.0
        fn = lambda: fq.rmsnorm_quant_token(x, gam, 1e-6)
    elif name == "token_prefill":        # plain 1x128 token quant of X [8192, 4096]
        x = randn((M_, K_), 1.0)
        fn = lambda: fq.rmsnorm_quant_token(x)
    elif name == "rmsnorm_prefill_e8m0":  # the fused front end with E8M0 activation scales
        x = randn((M_, K_), 1.0)
        gam = randn((K_,), 0.5) + 1.0
        fn = lambda: fq.rmsnorm_quant_token(x, gam, 1e-6, scale_fmt="e8m0")
    elif name == "token_prefill_e8m0":   # plain 1x128 token quant with E8M0 scales
        x = randn((M_, K_), 1.0)
        fn = lambda: fq.rmsnorm_quant_token(x, scale_fmt="e8m0")
    elif name == "requant_prefill":      # W [24576, 4096]: 201 MB in, 101 MB out
        w = randn((N_, K_), 0.02)
        fn = lambda: fq.quant_weight_block(w, "f32")
    elif name == "requant_prefill_e8m0":
        w = randn((N_, K_), 0.02)
        fn = lambda: fq.quant_weight_block(w, "e8m0")
    elif name == "grouped_gateup":
        tok, off = inputs.moe_routing()
        R = int(off[-1])
        aq, sa = fq.rmsnorm_quant_token(randn((R, 2048), 1.0))
        wq, sw = fq.quant_weight_block(randn((128 * 1536, 2048), 0.02), "f32")
        offd = torch.from_numpy(off).to(dev)
        out = torch.empty((R, 1536), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.grouped_gemm_w8a8_block(aq, sa, wq.view(128, 1536, 2048),
                                                sw.view(128, 12, 16), offd, out=out)
    elif name == "silu_moe":              # [gate | up] [32768, 1536] -> codes [32768, 768]
        hgu = randn((32768, 1536), 2.0)
        fn = lambda: fq.silu_mul_quant(hgu)
    elif name == "ptpc_gemm_prefill":     # M=4096 of the per-channel GEMM: A 17 MB, W 101 MB, out 201 MB
        aq, sa = fq.quant_rowwise(randn((4096, K_), 1.0))
        wq, sw = fq.quant_rowwise(randn((N_, K_), 0.02))
        out = torch.empty((4096, N_), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.gemm_w8a8_rowwise(aq, sa, wq, sw, out=out)
    elif name == "grouped_down":
        tok, off = inputs.moe_routing()
        R = int(off[-1])
        aq, sa = fq.rmsnorm_quant_token(randn((R, 768), 1.0))
        wq, sw = fq.quant_weight_block(randn((128 * 2048, 768), 0.02), "f32")
        offd = torch.from_numpy(off).to(dev)
        out = torch.empty((R, 2048), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.grouped_gemm_w8a8_block(aq, sa, wq.view(128, 2048, 768),
                                                sw.view(128, 16, 6), offd, out=out)
    elif name in ("inverse_rope_wo_a", "inverse_rope_wo_a_f32"):   # o [8192, 32, 512]: 268 MB in
        o = randn((8192, 32, 512), 1.0)
        pos = torch.randint(0, 16384, (8192,), generator=g, device=dev)
        cs = torch.rand((16384, 32), generator=g, device=dev)
        sn = torch.rand((16384, 32), generator=g, device=dev)
        fmt = "f32" if name.endswith("f32") else "e8m0"
        fn = lambda: fq.inverse_rope_quant(o, pos, cs, sn, 64, True, fmt)
    elif name == "gemm_diag_wo_a":       # 4 head groups: [8192, 4096] x [1024, 4096] each
        o = randn((8192, 32, 512), 1.0)
        aq, sa = fq.inverse_rope_quant(o, None, None, None, 0)
        wq, sw = fq.quant_weight_block(randn((4096, 4096), 0.02), "e8m0")
        out = torch.empty((8192, 4096), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.gemm_w8a8_block_diag(aq, sa, wq.view(4, 1024, 4096),
                                             sw.view(4, 8, 32), out=out)
    elif name == "attention_decode":     # 64 sequences, 153K cached positions: K+V 314 MB
        da = inputs.decode_attention(device=dev)
        Hq, Hkv, Dh = da["Hq"], da["Hkv"], da["D"]
        S, Bd = da["num_slots"], da["q"].shape[0]
        rows_c = torch.cat([torch.zeros((S, Hq * Dh), dtype=torch.bfloat16, device=dev),
                            da["k"], da["v"]], 1)
        _, s3 = fq.qkv_scales(rows_c, Hq, Hkv, Dh)
        kc = torch.empty((S, Hkv * Dh), dtype=torch.uint8, device=dev)
        vc = torch.empty_like(kc)
        fq.kv_cache_write(rows_c, Hq, Hkv, Dh, torch.arange(S, device=dev), s3, kc, vc,
                          quantize_q=False)
        del rows_c
        rows_q = torch.cat([da["q"], torch.zeros((Bd, 2 * Hkv * Dh), dtype=torch.bfloat16,
                                                 device=dev)], 1)
        qc = fq.kv_cache_write(rows_q, Hq, Hkv, Dh,
                               -torch.ones(Bd, dtype=torch.int64, device=dev), s3, kc, vc)
        bt = torch.from_numpy(da["block_table"]).to(dev)
        sl = torch.from_numpy(da["seq_lens"]).to(dev)
        wsa = torch.empty(fq.attention_decode_workspace_bytes(Bd, Hq, Hkv, Dh, da["max_seq_len"]),
                          dtype=torch.uint8, device=dev)
        oa = torch.empty((Bd, Hq * Dh), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.attention_decode(qc, kc, vc, s3, bt, sl, Hq, Hkv, da["block_size"],
                                         da["max_seq_len"], workspace=wsa, out=oa)
    elif name == "gemm_mx_prefill":      # the prefill GEMM with E8M0 scales, hardware block scaling
        x = randn((M_, K_), 1.0)
        aq, sa = fq.inverse_rope_quant(x.view(M_, 1, K_), None, None, None, 0, True, "e8m0")
        wq, sw = fq.quant_weight_block(randn((N_, K_), 0.02), "e8m0")
        out = torch.empty((M_, N_), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.gemm_w8a8_mx(aq, sa, wq, sw, out=out)
    else:
        raise SystemExit(f"unknown --ncu-case {name}")
    torch.cuda.synchronize()
    for _ in range(5):
        fn()
    torch.cuda.synchronize()
    if fq.check_device_error() != 0:
        raise SystemExit("device error")
    print(f"ncu case {name}: ok")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-rows", dest="rows", action="store_false")
    ap.add_argument("--ncu-case", default=None,
                    help="run a few launches of one kernel on a small case (for ncu) and exit")
    args = ap.parse_args()
    if args.ncu_case:
        run_ncu_case(args.ncu_case)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
