"""Benchmark of the wave-round hot path on B200: fused append + chunk-causal attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one wave round of one layer: wf_qk_norm_rope_append (per-head Q/K
RMSNorm, 3D RoPE, K/V into the ring) followed by wf_chunk_causal_attn, with
the ring advancing one chunk per step (steady state, full history).  Inputs
are seeded synthetic bf16 N(0,1) tensors resident in HBM before timing.

Prints ONE JSON line (rank 0).  `value` is useful attention TFLOP/s over all
ranks (QK^T + PV over visible, unpadded query/key pairs / step time).  Under
torchrun every rank runs its own replica of the workload on its own GPU (the
path shards by independent problems; no data-path collective).

--impl reference times the fp64 CPU oracle (the parity reference) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from chunk_causal_dit_b200 import inputs as wi  # noqa: E402

METRIC = "wave-round chunk-causal attention useful TFLOP/s & chunks/s on 1 B200; % of peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
BAD_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


# nominal dense bf16 tensor peak and HBM3e bandwidth of one B200 (for the second
# fraction next to the measured-peak one)
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def strip_c_comments(text: str) -> str:
    """C/C++ source without // and /* */ comments or blank lines (string
    literals of the kernel sources contain no comment markers)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_hash(read=None):
    """Hash of the attention kernel's code (comments excluded), used to tell
    whether the committed ncu traffic record still describes this kernel."""
    h = hashlib.sha256()
    for name in ("attn_kernel.cu", "sm100.cuh", "wf_internal.h"):
        path = os.path.join("chunk_causal_dit_b200", "csrc", name)
        if read is None:
            with open(os.path.join(ROOT, path)) as f:
                text = f.read()
        else:
            text = read(path)
        h.update(strip_c_comments(text).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload):
    """Per-launch DRAM bytes of the attention kernel from the committed ncu summary,
    or None when the summary is missing or was taken on another kernel source."""
    path = os.path.join(ROOT, "profiles", "attn_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("kernel_hash") != kernel_source_hash():
        return None
    return d.get("per_launch_bytes", {}).get(workload)


class ClockSampler:
    """SM clock, power and clock-event reasons sampled in-process through NVML
    (read-only queries) every few milliseconds from a background thread, with
    host timestamps, so that even a timed region of tens of milliseconds gets
    several samples.  Nothing is set or reset."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, device_index, interval_s=0.002):
        import threading
        self.samples = []                 # (t, sm_mhz, power_w, reasons_mask)
        self.sm_max = None
        self.error = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = self._handle(pynvml, device_index)
            self.sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM))
        except Exception as e:            # no NVML: the record says so
            self.error = "nvml unavailable: %s" % e
            return
        self.interval = interval_s
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()

    @staticmethod
    def _handle(pynvml, device_index):
        """NVML handle of the CUDA device (matched by PCI bus id when torch exposes it)."""
        try:
            import torch
            pr = torch.cuda.get_device_properties(device_index)
            bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            ids = [x for x in vis.split(",") if x.strip().isdigit()]
            idx = int(ids[device_index]) if device_index < len(ids) else device_index
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        nv, h = self._nvml, self._h
        while not self._stop.is_set():
            try:
                t = time.time()
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((t, float(sm), pw, int(rs)))
            except Exception as e:
                self.error = str(e)
                return
            self._stop.wait(self.interval)

    def wait_ready(self, n=3, timeout_s=2.0):
        """Wait (at most timeout_s) until the sampler has taken n samples, so that a
        slow first NVML query on a fresh process cannot leave a short timed region
        without any sample."""
        t_end = time.time() + timeout_s
        while self._thread is not None and len(self.samples) < n and self.error is None \
                and time.time() < t_end:
            time.sleep(0.002)

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def summary(self, t0, t1):
        inside = [x for x in self.samples if t0 <= x[0] <= t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": ["no samples"],
                    "samples": 0, "source": "nvml", **({"error": self.error} if self.error else {})}
        reasons = sorted({n for _, _, _, m in inside for n, bit in self.REASONS if m & bit})
        return {"sm_mhz": statistics.median(x[1] for x in inside),
                "sm_mhz_min": min(x[1] for x in inside),
                "sm_max_mhz": self.sm_max, "reasons": reasons, "samples": len(inside),
                "power_w_max": round(max(x[2] for x in inside), 1),
                "window_s": round(t1 - t0, 4), "source": "nvml, in-process, every %g ms" % (
                    1e3 * self.interval)}


def l2_note(working_set_mb):
    if working_set_mb > 126:
        return "no flush: per-step working set %.0f MB > 126 MB L2" % working_set_mb
    return ("no flush: per-step working set %.2f MB fits in L2 (latency-bound workload, "
            "no roofline claim)" % working_set_mb)


def dist_setup(gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != gpus and world > 1:
        raise SystemExit("--gpus %d but WORLD_SIZE %d" % (gpus, world))
    return rank, world, local


def make_group(world, backend):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def barrier(dist, device=None):
    if dist is not None:
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def allreduce_max(dist, value, device=None):
    """Max of a per-rank scalar over all ranks (host-side timing reduction only)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world, flops_per_rank_step, ms_step_max):
    """Whole-job useful TFLOP/s: every rank's work over the slowest rank's time."""
    return world * flops_per_rank_step / (ms_step_max * 1e-3) / 1e12


# ------------------------------------------------------------------ ours --

def run_ours(args, rank, world, local):
    import torch
    from chunk_causal_dit_b200 import wf

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = make_group(world, "nccl")
    w = wi.WORKLOADS[args.workload]
    peaks, peak_src = load_peaks()

    plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
    x = wi.wave_inputs(w, seed=rank)
    hk, hv = wi.history_prefill(w, seed=rank)
    q, k, v = x.q.to(dev), x.k.to(dev), x.v.to(dev)
    gq, gk = x.gamma_q.to(dev), x.gamma_k.to(dev)
    kc = torch.empty((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    for j in range(w.n_hist):
        kc[j % w.R].copy_(hk[j])
        vc[j % w.R].copy_(hv[j])
    q_out = torch.empty_like(q)
    o = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)
    r0 = w.n_hist
    flops_step = wf.wf_useful_flops(plan, r0)
    tensor_bytes = w.T * w.H * w.D * 2
    fp8 = args.attn == "fp8qk"
    # bf16: read q, k, v, write q', K', V; fused FP8: the q' write is one code byte
    append_bytes = (11 if fp8 else 12) * w.T * w.H * w.D
    if fp8:
        # E4M3 copies of q_out (per row) and of the key ring (per 128-row tile);
        # the history chunks were quantized when they were appended
        nt = (w.L + 127) // 128
        q8 = torch.empty((w.T, w.H, w.D), dtype=torch.uint8, device=dev)
        q_scale = torch.empty((w.H, w.T), dtype=torch.float32, device=dev)
        k8 = torch.empty((w.R, w.L, w.H, w.D), dtype=torch.uint8, device=dev)
        k_scale = torch.empty((w.R, nt, w.H), dtype=torch.float32, device=dev)
        wf.wf_quantize_k_fp8(plan, 0, w.n_hist, kc, k8, k_scale, stream)

    def step(r):
        if fp8:
            # the append writes q's E4M3 codes; the wave's K chunks are quantized after it
            wf.wf_qk_norm_rope_append_fp8q(plan, r, q, k, v, None, gq, gk, None, q8, q_scale,
                                           kc, vc, stream)
            wf.wf_quantize_k_fp8(plan, r, w.n_wave, kc, k8, k_scale, stream)
            wf.wf_chunk_causal_attn_fp8qk(plan, r, q8, q_scale, k8, k_scale, vc, o, None, stream)
        else:
            wf.wf_qk_norm_rope_append(plan, r, q, k, v, None, gq, gk, q_out, kc, vc, stream)
            wf.wf_chunk_causal_attn(plan, r, q_out, kc, vc, o, None, stream)

    rnd = r0
    for _ in range(args.warmup):
        step(rnd)
        rnd += 1
    torch.cuda.synchronize(dev)
    if wf.wf_sync_status(plan, stream) != wf.WF_OK:
        raise SystemExit("device status error during warm-up")

    # ---- device-timed steps (kernel events inside give the roofline) ----
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.wait_ready()
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    start.record(stream)
    for i in range(args.steps):
        e0, e1, eq, e2 = ev[i]
        e0.record(stream)
        if fp8:
            wf.wf_qk_norm_rope_append_fp8q(plan, rnd, q, k, v, None, gq, gk, None, q8, q_scale,
                                           kc, vc, stream)
        else:
            wf.wf_qk_norm_rope_append(plan, rnd, q, k, v, None, gq, gk, q_out, kc, vc, stream)
        e1.record(stream)
        if fp8:
            wf.wf_quantize_k_fp8(plan, rnd, w.n_wave, kc, k8, k_scale, stream)
            eq.record(stream)
            wf.wf_chunk_causal_attn_fp8qk(plan, rnd, q8, q_scale, k8, k_scale, vc, o, None,
                                          stream)
        else:
            eq.record(stream)
            wf.wf_chunk_causal_attn(plan, rnd, q_out, kc, vc, o, None, stream)
        e2.record(stream)
        rnd += 1
    stop.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier(dist, dev)
    clocks.stop()
    status = wf.wf_sync_status(plan, stream)
    if status != wf.WF_OK:
        raise SystemExit("device status %d (%s)" % (status, wf.status_string(status)))
    ms_total = allreduce_max(dist, start.elapsed_time(stop), dev)
    ms_step = ms_total / args.steps
    t_append = [a.elapsed_time(b) for a, b, _, _ in ev]
    t_quant = [b.elapsed_time(c) for _, b, c, _ in ev]
    t_attn = [c.elapsed_time(d) for _, _, c, d in ev]
    attn_ms = statistics.mean(t_attn)
    append_ms = statistics.mean(t_append)
    quant_ms = statistics.mean(t_quant)

    # ---- end to end through the API: pinned host in, pinned host out ----
    # Every round copies its q, k, v from pinned host memory and its O back;
    # HostRoundPipeline overlaps those copies with the neighbouring rounds'
    # kernels (double-buffered staging, separate copy streams).
    from chunk_causal_dit_b200.pipeline import HostRoundPipeline
    hq = x.q.pin_memory()
    hk_ = x.k.pin_memory()
    hv_ = x.v.pin_memory()
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    e2e_steps = max(3, min(args.steps, 50))
    pipe = HostRoundPipeline(plan, kc, vc, gq, gk, device=dev,
                             fp8=(k8, k_scale) if fp8 else None)
    pipe.run([(rnd + i, hq, hk_, hv_, ho) for i in range(2)])
    rnd += 2
    pipe.synchronize()
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    s2, t2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pipe.run([(rnd + i, hq, hk_, hv_, ho) for i in range(e2e_steps)], start_event=s2,
             end_event=t2)
    rnd += e2e_steps
    pipe.synchronize()
    torch.cuda.synchronize(dev)
    e2e_ms = allreduce_max(dist, s2.elapsed_time(t2), dev) / e2e_steps
    barrier(dist, dev)
    # the PCIe floor of the end-to-end step: the same host bytes copied alone
    # (pinned -> device, one copy per input tensor, CUDA events), best of 3
    h2d_ms = []
    for _ in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for src, dst in ((hq, q), (hk_, k), (hv_, v)):
            dst.copy_(src, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize(dev)
        h2d_ms.append(a.elapsed_time(b))
    h2d_gbs = 3 * tensor_bytes / (min(h2d_ms) * 1e-3) / 1e9

    clk = clocks.summary(t_wall0, t_wall1)
    head_block = plan.head_block(r0, fp8)      # the attention's unit order (steady state)
    block = None
    if not args.no_block and w.H * w.D in wi.BLOCK_WIDTHS:
        del q, k, v, x, hq, hk_, hv_, ho, pipe
        block = run_block(args, plan, w, rnd, flops_step, dev, stream, peaks, dist, fp8)
    plan.destroy()
    legs = fp8_leg = None
    if not args.no_configs and not fp8:
        # every rank runs the legs (no collective inside); rank 0 reports them
        legs, fp8_leg = run_config_legs(args, dev, peaks)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return None

    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_src_note = "%s bf16_tflops (burst)" % peak_src
    if fp8:
        # half the useful FLOPs (Q.K^T) run on E4M3 at twice the bf16 rate
        # (nominal 4.5 vs 2.25 PF dense), half (P.V) on bf16: the contraction's
        # peak is 1 / (0.5 / 2 + 0.5) = 4/3 of the measured bf16 peak
        peak_tf = round(peak_tf * 4.0 / 3.0, 1)
        peak_src_note = ("4/3 x %s bf16_tflops (burst): Q.K^T at the nominal 2x E4M3 rate, "
                         "P.V at bf16" % peak_src)
    attn_tflops = flops_step / (attn_ms * 1e-3) / 1e12
    value = aggregate_tflops(world, flops_step, ms_step)
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    append_gbs = append_bytes / (append_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 q.k^t, bf16 p.v" if fp8 else "bf16",
        "data": "synthetic (seeded bf16 N(0,1) q/k/v and history, gains 1+0.1N(0,1))",
        "config": {
            "workload": w.name,
            "heads": w.H, "head_dim": w.D, "chunk_tokens": w.L, "wave_chunks": w.n_wave,
            "history_chunks": w.n_hist, "wave_tokens": w.T, "attention": args.attn,
            "attn_unit_order": "heads in blocks of %d" % head_block,
            "parallelism": "replica%d (independent wave rounds, no data-path collective)" % world,
            "l2": l2_note((append_bytes + 2 * w.R * w.L * w.H * w.D * 2) / 1e6),
        },
        # query chunks per second of attention (W / t_attn) and of the whole step
        "chunks_per_s": round(world * w.n_wave / (attn_ms * 1e-3), 2),
        "chunks_per_s_step": round(world * w.n_wave / (ms_step * 1e-3), 2),
        "pct_peak": round(100.0 * value / world / peak_tf, 2),
        "roofline": {
            "kernel": "chunk_causal_attn_kernel<128, fp8>" if fp8 else "chunk_causal_attn_kernel",
            "bound": "tensor",
            "achieved": round(attn_tflops, 2),
            "peak": peak_tf,
            "unit": "TFLOP/s",
            "frac": round(attn_tflops / peak_tf, 4),
            "frac_nominal": round(attn_tflops / (NOMINAL_BF16_TFLOPS * (4.0 / 3.0 if fp8 else 1.0)),
                                  4),
            # the sustained GEMM figure (seconds under the power cap) applies only
            # to a timed region that long; a short region runs at burst clocks
            "frac_sustained": (round(attn_tflops / (peaks.get("bf16_tflops_sustained", 1374.1) *
                                                    (4.0 / 3.0 if fp8 else 1.0)), 4)
                               if t_wall1 - t_wall0 >= 1.0 else None),
            "timed_region_s": round(t_wall1 - t_wall0, 4),
            "peak_source": peak_src_note,
            "traffic": profiled_traffic(args.workload + ("/fp8qk" if fp8 else "")),
            "ms_per_launch": round(attn_ms, 5),
            "useful_flop_per_launch": flops_step,
        },
        "append": {
            "kernel": "qk_norm_rope_append_kernel" + ("<128, q8>" if fp8 else ""),
            "bound": "hbm",
            "ms_per_launch": round(append_ms, 5),
            "achieved": round(append_gbs, 1),
            "peak": hbm,
            "unit": "GB/s",
            "frac": round(append_gbs / hbm, 4),
            "frac_nominal": round(append_gbs / NOMINAL_HBM_GBS, 4),
            "bytes_per_launch": append_bytes,
        },
        **({"quantize": {
            "kernels": "quantize_tiles_kernel (the wave's key chunks; q is quantized in the "
                       "append)",
            "bound": "hbm",
            "ms_per_step": round(quant_ms, 5),
            "achieved": round(3 * w.T * w.H * w.D / (quant_ms * 1e-3) / 1e9, 1),
            "peak": hbm,
            "unit": "GB/s",
            "frac": round(3 * w.T * w.H * w.D / (quant_ms * 1e-3) / 1e9 / hbm, 4),
            "bytes_per_step": 3 * w.T * w.H * w.D,
        }} if fp8 else {}),
        "e2e": {
            "value": round(aggregate_tflops(world, flops_step, e2e_ms), 3),
            "unit": "TFLOP/s",
            "ms_per_step": round(e2e_ms, 4),
            "h2d_bytes_per_step": 3 * tensor_bytes,
            "d2h_bytes_per_step": tensor_bytes,
            # a step cannot be shorter than its host-to-device copy (the D2H of the
            # previous round overlaps it on the other copy engine)
            "h2d_gbs_measured": round(h2d_gbs, 2),
            "pcie_floor_ms": round(3 * tensor_bytes / (h2d_gbs * 1e9) * 1e3, 4),
        },
        "gpu_launches": (3 if fp8 else 2) * args.steps,
        "clocks": clk,
    }
    if block is not None:
        line["block"] = block
    if legs is not None:
        line["configs"] = legs
        line["fp8qk"] = fp8_leg
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
    return line


# ----------------------------------------- the other configurations (legs) --

def measure_single_layer(w, steps, warmup, dev, peaks, fp8=False, seed=0):
    """A short timed loop of one single-layer workload (append, then attention;
    with fp8 the two quantizers and the FP8 attention), ring advancing one chunk
    per step, CUDA events around every kernel, its own clock record.  Returns
    per-kernel times, the attention's roofline fraction (burst peak: the region
    lasts well under a second) and the append's GB/s."""
    import torch
    from chunk_causal_dit_b200 import wf
    stream = torch.cuda.current_stream(dev)
    plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
    x = wi.wave_inputs(w, seed=seed)
    hk, hv = wi.history_prefill(w, seed=seed)
    q, k, v = x.q.to(dev), x.k.to(dev), x.v.to(dev)
    gq, gk = x.gamma_q.to(dev), x.gamma_k.to(dev)
    kc = torch.empty((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    for j in range(w.n_hist):
        kc[j % w.R].copy_(hk[j])
        vc[j % w.R].copy_(hv[j])
    q_out, o = torch.empty_like(q), torch.empty_like(q)
    if fp8:
        nt = (w.L + 127) // 128
        q8 = torch.empty((w.T, w.H, w.D), dtype=torch.uint8, device=dev)
        q_scale = torch.empty((w.H, w.T), dtype=torch.float32, device=dev)
        k8 = torch.empty((w.R, w.L, w.H, w.D), dtype=torch.uint8, device=dev)
        k_scale = torch.empty((w.R, nt, w.H), dtype=torch.float32, device=dev)
        wf.wf_quantize_k_fp8(plan, 0, w.n_hist, kc, k8, k_scale, stream)
    r0 = w.n_hist
    flops = wf.wf_useful_flops(plan, r0)

    def step(r, e=None):
        if e is not None:
            e[0].record(stream)
        if fp8:
            wf.wf_qk_norm_rope_append_fp8q(plan, r, q, k, v, None, gq, gk, None, q8, q_scale,
                                           kc, vc, stream)
        else:
            wf.wf_qk_norm_rope_append(plan, r, q, k, v, None, gq, gk, q_out, kc, vc, stream)
        if e is not None:
            e[1].record(stream)
        if fp8:
            wf.wf_quantize_k_fp8(plan, r, w.n_wave, kc, k8, k_scale, stream)
        if e is not None:
            e[2].record(stream)
        if fp8:
            wf.wf_chunk_causal_attn_fp8qk(plan, r, q8, q_scale, k8, k_scale, vc, o, None, stream)
        else:
            wf.wf_chunk_causal_attn(plan, r, q_out, kc, vc, o, None, stream)
        if e is not None:
            e[3].record(stream)

    rnd = r0
    for _ in range(warmup):
        step(rnd)
        rnd += 1
    torch.cuda.synchronize(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    clocks = ClockSampler(dev.index)
    clocks.wait_ready()
    torch.cuda.synchronize(dev)
    t0 = time.time()
    for i in range(steps):
        step(rnd, ev[i])
        rnd += 1
    torch.cuda.synchronize(dev)
    t1 = time.time()
    clocks.stop()
    status = wf.wf_sync_status(plan, stream)
    plan.destroy()
    if status != wf.WF_OK:
        raise SystemExit("device status %d (%s) in the %s leg" % (status, wf.status_string(status),
                                                                 w.name))
    app = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    qnt = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    att = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
    stp = statistics.mean(e[0].elapsed_time(e[3]) for e in ev)
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * (4.0 / 3.0 if fp8 else 1.0)
    append_bytes = (11 if fp8 else 12) * w.T * w.H * w.D
    d = {"workload": w.name, "heads": w.H, "head_dim": w.D, "chunk_tokens": w.L,
         "wave_chunks": w.n_wave, "history_chunks": w.n_hist, "steps": steps, "warmup": warmup,
         "attention_ms": round(att, 5), "append_us": round(1e3 * app, 2),
         "step_ms": round(stp, 5), "useful_flop_per_launch": flops}
    if w.T * w.H * w.D * 2 * 6 > 126e6:      # beyond L2: a roofline claim holds
        att_tf = flops / (att * 1e-3) / 1e12
        d.update({"attention_tflops": round(att_tf, 2), "attention_frac": round(att_tf / peak_tf, 4),
                  "attention_frac_nominal": round(att_tf / (NOMINAL_BF16_TFLOPS *
                                                            (4.0 / 3.0 if fp8 else 1.0)), 4),
                  "append_gbs": round(append_bytes / (app * 1e-3) / 1e9, 1),
                  "append_frac": round(append_bytes / (app * 1e-3) / 1e9 / hbm, 4),
                  "chunks_per_s": round(w.n_wave / (att * 1e-3), 2),
                  "step_tflops": round(flops / (stp * 1e-3) / 1e12, 2)})
    else:
        d["note"] = "latency only: the working set fits in L2, no roofline claim"
    if fp8:
        qbytes = 3 * w.T * w.H * w.D           # the wave's key chunks (q: in the append)
        d.update({"quantize_us": round(1e3 * qnt, 2),
                  "quantize_gbs": round(qbytes / (qnt * 1e-3) / 1e9, 1),
                  "quantize_frac": round(qbytes / (qnt * 1e-3) / 1e9 / hbm, 4),
                  "attention_peak": round(peak_tf, 1),
                  "peak_source": "4/3 x measured bf16 burst: Q.K^T at 2x (E4M3), P.V at bf16"})
    d["clocks"] = clocks.summary(t0, t1)
    return d


def measure_round_loop(w, rounds, warmup, dev, peaks, seed=0, dist=None):
    """Full rounds of the multi-layer workload: per round, layer after layer, the
    append and the attention of each layer on its own ring, then the ring
    advances.  Returns per-round latency (median, p90), rounds/s, the attention's
    mean launch time and roofline fraction, and its own clock record."""
    import torch
    from chunk_causal_dit_b200 import wf
    stream = torch.cuda.current_stream(dev)
    plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
    sets = [wi.wave_inputs(w, seed=seed, salt=s) for s in range(2)]   # pool of two input sets
    qs = [(x.q.to(dev), x.k.to(dev), x.v.to(dev)) for x in sets]
    gq, gk = sets[0].gamma_q.to(dev), sets[0].gamma_k.to(dev)
    hk, hv = wi.history_prefill(w, seed=seed)
    caches = []
    for _ in range(w.layers):
        kc = torch.empty((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        for j in range(w.n_hist):
            kc[j % w.R].copy_(hk[j])
            vc[j % w.R].copy_(hv[j])
        caches.append((kc, vc))
    q_out = torch.empty_like(qs[0][0])
    o = torch.empty_like(q_out)
    r0 = w.n_hist
    flops_layer = wf.wf_useful_flops(plan, r0)

    def run_round(r, attn_events=None):
        for layer, (kc, vc) in enumerate(caches):
            q, k, v = qs[layer % 2]
            wf.wf_qk_norm_rope_append(plan, r, q, k, v, None, gq, gk, q_out, kc, vc, stream)
            if attn_events is not None:
                attn_events[layer][0].record(stream)
            wf.wf_chunk_causal_attn(plan, r, q_out, kc, vc, o, None, stream)
            if attn_events is not None:
                attn_events[layer][1].record(stream)

    rnd = r0
    for _ in range(warmup):
        run_round(rnd)
        rnd += 1
    torch.cuda.synchronize(dev)
    rev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(rounds)]
    aev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(w.layers)] for _ in range(rounds)]
    clocks = ClockSampler(dev.index)
    clocks.wait_ready()
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    t0 = time.time()
    for i in range(rounds):
        rev[i][0].record(stream)
        run_round(rnd, aev[i])
        rev[i][1].record(stream)
        rnd += 1
    torch.cuda.synchronize(dev)
    t1 = time.time()
    barrier(dist, dev)
    clocks.stop()
    status = wf.wf_sync_status(plan, stream)
    plan.destroy()
    if status != wf.WF_OK:
        raise SystemExit("device status %d (%s) in the round loop" % (status,
                                                                      wf.status_string(status)))
    per_round = [a.elapsed_time(b) for a, b in rev]
    attn_ms = statistics.mean(a.elapsed_time(b) for rr in aev for a, b in rr)
    srt = sorted(per_round)
    # a loop of this length runs under the power cap: the sustained GEMM figure
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    att_tf = flops_layer / (attn_ms * 1e-3) / 1e12
    return {"per_round": per_round, "attn_ms": attn_ms, "flops_layer": flops_layer,
            "clocks": clocks.summary(t0, t1), "timed_region_s": t1 - t0,
            "summary": {
                "workload": w.name, "layers": w.layers, "rounds": rounds, "warmup": warmup,
                "round_ms_median": round(statistics.median(per_round), 4),
                "round_ms_p90": round(srt[min(len(srt) - 1, int(0.9 * len(srt)))], 4),
                "rounds_per_s": round(1e3 * rounds / sum(per_round), 3),
                "chunks_per_s": round(1e3 * rounds / sum(per_round), 3),
                "round_tflops": round(w.layers * flops_layer * rounds / (sum(per_round) * 1e-3)
                                      / 1e12, 2),
                "attention_ms": round(attn_ms, 5),
                "attention_tflops": round(att_tf, 2),
                "attention_frac_sustained": round(att_tf / peak, 4),
                "attention_frac_burst": round(att_tf / peaks.get("bf16_tflops", 1630.1), 4),
                "timed_region_s": round(t1 - t0, 3),
                "clocks": clocks.summary(t0, t1)}}


VAE_STAGE = dict(T=12, H=120, W=208, C=384)


def measure_vae_stage(steps, warmup, dev, peaks, seed=0):
    """The streaming VAE-decode stage: one residual block (RMSNorm + SiLU, causal
    3x3x3 conv, RMSNorm + SiLU, causal conv + residual) per chunk of 12 frames at
    120 x 208 with 384 channels, chunk after chunk, each convolution reading the
    previous chunk's last two input frames as its history (views into the
    previous chunk's buffers: double-buffered, no copies).  CUDA events around
    every kernel; the convolutions' roofline is the bf16 tensor peak (burst)."""
    import torch
    from chunk_causal_dit_b200 import wf
    T, H, W, C = VAE_STAGE["T"], VAE_STAGE["H"], VAE_STAGE["W"], VAE_STAGE["C"]
    stream = torch.cuda.current_stream(dev)
    plan = wf.Plan(64, 1, 0, 1, 128)
    xs = [wi.bf16_normal((T, H, W, C), seed + i, wi.STREAM_X).to(dev) for i in range(2)]
    w1 = wi.bf16_weight(C, 27 * C, seed, 1).reshape(C, 3, 3, 3, C).contiguous().to(dev)
    w2 = wi.bf16_weight(C, 27 * C, seed, 2).reshape(C, 3, 3, 3, C).contiguous().to(dev)
    b1 = wi.f32_vector((C,), 0.02, seed, wi.STREAM_BIAS, 1).to(dev)
    b2 = wi.f32_vector((C,), 0.02, seed, wi.STREAM_BIAS, 2).to(dev)
    g1 = (1 + 0.1 * wi.f32_vector((C,), 1.0, seed, wi.STREAM_GAMMA, 1)).to(dev)
    g2 = (1 + 0.1 * wi.f32_vector((C,), 1.0, seed, wi.STREAM_GAMMA, 2)).to(dev)
    h1 = [torch.empty((T, H, W, C), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    h2 = [torch.empty_like(h1[0]) for _ in range(2)]
    c1 = torch.empty_like(h1[0])
    out = torch.empty_like(h1[0])

    def chunk(i, ev=None):
        a, prev = i % 2, (i + 1) % 2
        hist1 = h1[prev][T - 2:] if i > 0 else None
        hist2 = h2[prev][T - 2:] if i > 0 else None
        x = xs[i % 2]
        if ev is not None:
            ev[0].record(stream)
        wf.wf_rms_norm_silu(plan, x, g1, h1[a], stream)
        if ev is not None:
            ev[1].record(stream)
        wf.wf_causal_conv3d(plan, h1[a], hist1, w1, b1, None, c1, stream)
        if ev is not None:
            ev[2].record(stream)
        wf.wf_rms_norm_silu(plan, c1, g2, h2[a], stream)
        if ev is not None:
            ev[3].record(stream)
        wf.wf_causal_conv3d(plan, h2[a], hist2, w2, b2, x, out, stream)
        if ev is not None:
            ev[4].record(stream)

    for i in range(warmup):
        chunk(i)
    torch.cuda.synchronize(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    clocks = ClockSampler(dev.index)
    clocks.wait_ready()
    torch.cuda.synchronize(dev)
    t0 = time.time()
    for i in range(steps):
        chunk(warmup + i, ev[i])
    torch.cuda.synchronize(dev)
    t1 = time.time()
    clocks.stop()
    status = wf.wf_sync_status(plan, stream)
    plan.destroy()
    if status != wf.WF_OK:
        raise SystemExit("device status %d (%s) in the VAE leg" % (status, wf.status_string(status)))
    conv_flop = 2.0 * T * H * W * C * C * 27      # every tap of the 3x3x3 kernel
    norm_ms = statistics.mean(e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]) for e in ev) / 2
    conv_ms = statistics.mean(e[1].elapsed_time(e[2]) + e[3].elapsed_time(e[4]) for e in ev) / 2
    blk_ms = statistics.mean(e[0].elapsed_time(e[4]) for e in ev)
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    conv_tf = conv_flop / (conv_ms * 1e-3) / 1e12
    norm_bytes = 4 * T * H * W * C
    return {
        "what": "streaming VAE-decode stage: residual block (RMSNorm+SiLU, causal 3x3x3 conv, "
                "RMSNorm+SiLU, causal conv + residual) per chunk, history from the previous chunk",
        "frames_per_chunk": T, "height": H, "width": W, "channels": C,
        "steps": steps, "warmup": warmup,
        "block_ms_per_chunk": round(blk_ms, 4),
        "chunks_per_s": round(1e3 / blk_ms, 2),
        "frames_per_s": round(T * 1e3 / blk_ms, 1),
        "block_tflops": round(2 * conv_flop / (blk_ms * 1e-3) / 1e12, 2),
        "conv": {"kernel": "gemm_pair_kernel<conv, BN=192> (implicit GEMM, K = 27 taps x 384)",
                 "bound": "tensor", "ms_per_launch": round(conv_ms, 5),
                 "achieved": round(conv_tf, 2), "peak": peak, "unit": "TFLOP/s",
                 "frac": round(conv_tf / peak, 4),
                 "frac_nominal": round(conv_tf / NOMINAL_BF16_TFLOPS, 4),
                 "flop_per_launch": conv_flop},
        "norm": {"kernel": "rms_norm_silu_kernel", "bound": "hbm",
                 "ms_per_launch": round(norm_ms, 5),
                 "achieved": round(norm_bytes / (norm_ms * 1e-3) / 1e9, 1), "peak": hbm,
                 "unit": "GB/s", "frac": round(norm_bytes / (norm_ms * 1e-3) / 1e9 / hbm, 4),
                 "bytes_per_launch": norm_bytes},
        "clocks": clocks.summary(t0, t1),
    }


def run_vae(args, rank, world, local):
    """bench.py --workload vae_stage: the VAE-decode stage alone, one replica per GPU."""
    import torch
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = make_group(world, "nccl")
    peaks, _ = load_peaks()
    barrier(dist, dev)
    v = measure_vae_stage(args.steps, args.warmup, dev, peaks, seed=rank)
    ms = allreduce_max(dist, v["block_ms_per_chunk"], dev)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return None
    return {
        "metric": "streaming VAE-decode stage: useful conv TFLOP/s (two causal 3x3x3 convs "
                  "per chunk)",
        "value": round(world * 2 * v["conv"]["flop_per_launch"] / (ms * 1e-3) / 1e12, 3),
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded bf16 N(0,1) chunks, random-init weights)",
        "config": {"workload": "vae_stage", "frames_per_chunk": v["frames_per_chunk"],
                   "height": v["height"], "width": v["width"], "channels": v["channels"],
                   "parallelism": "replica%d" % world,
                   "l2": "no flush: per-chunk working set %.0f MB > 126 MB L2" % (
                       8 * v["frames_per_chunk"] * v["height"] * v["width"] * v["channels"]
                       * 2 / 1e6)},
        "roofline": v["conv"], "vae_stage": v, "gpu_launches": 4 * args.steps,
        "clocks": v["clocks"],
    }


def run_config_legs(args, dev, peaks):
    """The other configurations of the benchmark, each a short leg with its own
    clock record: the tiny wave (latency), the 5-step and 14B waves, the 30-layer
    x 20-round loop, and the FP8 Q.K^T attention on the headline wave."""
    import torch
    legs = {}
    for name, steps in (("tiny", 400), ("wan13b_5step", 20), ("wan14b_4step", 20)):
        # the tiny wave runs ~30 us a step: enough steps for several clock samples
        legs[name] = measure_single_layer(wi.WORKLOADS[name], steps, 5, dev, peaks)
        torch.cuda.empty_cache()
    legs["wan13b_round"] = measure_round_loop(wi.WORKLOADS["wan13b_round"], 20, 3, dev,
                                              peaks)["summary"]
    torch.cuda.empty_cache()
    fp8 = measure_single_layer(wi.WORKLOADS[args.workload], 30, 5, dev, peaks, fp8=True)
    torch.cuda.empty_cache()
    legs["vae_stage"] = measure_vae_stage(10, 3, dev, peaks)
    torch.cuda.empty_cache()
    return legs, fp8


def block_flops(w, hidden, ffn, attn_flops):
    """Useful FLOPs of one DiT block over the wave: the four projections (QKV,
    output, two feed-forward layers) plus the chunk-causal attention."""
    HD = w.H * w.D
    return 2.0 * w.T * (3 * HD * hidden + hidden * HD + 2 * hidden * ffn) + attn_flops


def run_block(args, plan, w, r0, attn_flops, dev, stream, peaks, dist, fp8=False):
    """One DiT block over the wave per step: LayerNorm + modulation, the QKV
    projection with the norm/RoPE/ring append fused in, the chunk-causal
    attention, the output projection with the gated residual, LayerNorm +
    modulation, the GELU feed-forward layer and the second one with the gated
    residual.  Random-init weights of the Wan block widths; per-chunk modulation
    (each chunk sits at its own denoising step).  Device-timed with CUDA events
    around every kernel; returns the "block" object of the JSON line."""
    import torch
    from chunk_causal_dit_b200 import wf

    hidden, ffn = wi.BLOCK_WIDTHS[w.H * w.D]
    b = wi.block_inputs(w, hidden, ffn, seed=0)
    x = b.x.to(dev)
    w_qkv, b_qkv = b.w_qkv.to(dev), b.b_qkv.to(dev)
    w_o, b_o = b.w_o.to(dev), b.b_o.to(dev)
    w_1, b_1 = b.w_1.to(dev), b.b_1.to(dev)
    w_2, b_2 = b.w_2.to(dev), b.b_2.to(dev)
    mod = b.mod.to(dev)
    gq, gk = b.gamma_q.to(dev), b.gamma_k.to(dev)
    h = torch.empty((w.T, hidden), dtype=torch.bfloat16, device=dev)
    x1 = torch.empty_like(h)
    x2 = torch.empty_like(h)
    f = torch.empty((w.T, ffn), dtype=torch.bfloat16, device=dev)
    q_out = torch.empty((w.T, w.H, w.D), dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q_out)
    kc = torch.zeros((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    o2 = o.view(w.T, w.H * w.D)
    names = ["layer_norm_1", "qkv_norm_rope_append", "attention", "out_proj_gated",
             "layer_norm_2", "ffn1_gelu", "ffn2_gated"]
    if fp8:
        # E4M3 q (per row) and key ring (per 128-row tile); every slot is quantized
        # once here, later history chunks in the round that appended them
        nt = (w.L + 127) // 128
        q8 = torch.empty((w.T, w.H, w.D), dtype=torch.uint8, device=dev)
        q_scale = torch.empty((w.H, w.T), dtype=torch.float32, device=dev)
        k8 = torch.empty((w.R, w.L, w.H, w.D), dtype=torch.uint8, device=dev)
        k_scale = torch.empty((w.R, nt, w.H), dtype=torch.float32, device=dev)
        wf.wf_quantize_k_fp8(plan, r0 - w.n_hist, w.R, kc, k8, k_scale, stream)
        names[2] = "attention_fp8qk (with the q and k quantization)"

    def step(r, ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        wf.wf_layer_norm_modulate(plan, x, mod[0], mod[1], w.L, h, stream)
        mark(1)
        wf.wf_qkv_proj_norm_rope_append(plan, r, h, w_qkv, b_qkv, gq, gk, q_out, kc, vc, stream)
        mark(2)
        if fp8:
            wf.wf_quantize_q_fp8(plan, q_out, q8, q_scale, stream)
            wf.wf_quantize_k_fp8(plan, r, w.n_wave, kc, k8, k_scale, stream)
            wf.wf_chunk_causal_attn_fp8qk(plan, r, q8, q_scale, k8, k_scale, vc, o, None, stream)
        else:
            wf.wf_chunk_causal_attn(plan, r, q_out, kc, vc, o, None, stream)
        mark(3)
        wf.wf_linear(plan, o2, w_o, x1, b_o, wf.WF_EPI_GATED_RESIDUAL, mod[2], x, w.L, stream)
        mark(4)
        wf.wf_layer_norm_modulate(plan, x1, mod[3], mod[4], w.L, h, stream)
        mark(5)
        wf.wf_linear(plan, h, w_1, f, b_1, wf.WF_EPI_GELU_TANH, None, None, 1, stream)
        mark(6)
        wf.wf_linear(plan, f, w_2, x2, b_2, wf.WF_EPI_GATED_RESIDUAL, mod[5], x1, w.L, stream)
        mark(7)

    rnd = r0
    for _ in range(max(3, args.warmup)):
        step(rnd)
        rnd += 1
    torch.cuda.synchronize(dev)
    n = max(3, min(args.steps, 50))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(n)]
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    for i in range(n):
        step(rnd, evs[i])
        rnd += 1
    torch.cuda.synchronize(dev)
    status = wf.wf_sync_status(plan, stream)
    if status != wf.WF_OK:
        raise SystemExit("block: device status %d (%s)" % (status, wf.status_string(status)))
    per = {nm: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs)
           for i, nm in enumerate(names)}
    ms_step = allreduce_max(dist, statistics.mean(e[0].elapsed_time(e[7]) for e in evs), dev)
    total = block_flops(w, hidden, ffn, attn_flops)
    HD = w.H * w.D
    if fp8:
        per["attention"] = per.pop(names[2])
    gemm_flops = {"qkv_norm_rope_append": 2.0 * w.T * 3 * HD * hidden,
                  "out_proj_gated": 2.0 * w.T * hidden * HD,
                  "ffn1_gelu": 2.0 * w.T * hidden * ffn, "ffn2_gated": 2.0 * w.T * hidden * ffn}
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    ln_bytes = 4.0 * w.T * hidden
    tflops = total / (ms_step * 1e-3) / 1e12
    return {
        "what": "one DiT block over the wave (Wan %d/%d widths, random-init weights, per-chunk "
                "modulation): LN, QKV + norm/RoPE/append, attention, out-proj + gated residual, "
                "LN, FFN1 + GELU, FFN2 + gated residual" % (hidden, ffn),
        "hidden": hidden, "ffn": ffn,
        "steps": n,
        "ms_per_step": round(ms_step, 4),
        "useful_flop_per_step": total,
        "tflops": round(tflops, 2),
        "frac": round(tflops / peak_tf, 4),
        "peak": peak_tf,
        "chunks_per_s": round(w.n_wave / (ms_step * 1e-3), 2),
        "ms_per_kernel": {k: round(v, 4) for k, v in per.items()},
        "gemm_tflops": {k: round(fl / (per[k] * 1e-3) / 1e12, 1) for k, fl in gemm_flops.items()},
        "gemm_frac": {k: round(fl / (per[k] * 1e-3) / 1e12 / peak_tf, 4)
                      for k, fl in gemm_flops.items()},
        "layer_norm_gbs": round(ln_bytes / (per["layer_norm_1"] * 1e-3) / 1e9, 1),
        "layer_norm_frac": round(ln_bytes / (per["layer_norm_1"] * 1e-3) / 1e9 / hbm, 4),
        "attention": "fp8qk (E4M3 Q.K^T, bf16 P.V; q and k quantization included)" if fp8
                     else "bf16",
        "launches_per_step": 9 if fp8 else 7,
        "l2": l2_note((4 * w.T * hidden * 2 + w.T * ffn * 2 +
                       2 * (4 * hidden * HD + 2 * hidden * ffn)) / 1e6),
    }


# Peer-to-peer copy bandwidth per direction between two B200s over NVLink 5, as
# measured (900 GB/s nominal).
PEER_COPY_GBS = 770.0


def run_wp(args, rank, world, local):
    """Wave Parallelism (chunk_causal_dit_b200.wave_parallel): the wave's chunks split
    over ranks; one step is one layer of one round (append, one-way K/V delivery,
    attention), the round advancing every step.

    Under torchrun every rank is a GPU and the delivery is NCCL point-to-point; the
    step time is the device-timed max over ranks, and `value` is the whole wave's
    useful TFLOP/s (strong scaling).  In one process with --wp N > 1 the N ranks'
    kernels run one after another on the one GPU (device copies stand in for the
    delivery and are not timed); the line then reports each rank's kernel times
    and a step time *projected* as the slowest rank's append + attention plus the
    delivery of its incoming K/V at the peer-copy bandwidth, next to the
    single-GPU round measured in the same process."""
    import torch
    from chunk_causal_dit_b200 import wf
    from chunk_causal_dit_b200.wave_parallel import LibwfKernels, WaveParallelRound

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = make_group(world, "nccl")
    w = wi.WORKLOADS[args.workload]
    emulate = world == 1
    n_ranks = args.wp if emulate else world
    if not 1 <= n_ranks <= w.n_wave:
        raise SystemExit("Wave Parallelism needs 1..%d ranks (one wave chunk each at least)"
                         % w.n_wave)
    x = wi.wave_inputs(w, seed=0)
    hk, hv = wi.history_prefill(w, seed=0)
    gq, gk = x.gamma_q.to(dev), x.gamma_k.to(dev)
    kern = LibwfKernels(gq, gk)
    r0 = w.n_hist
    mine = list(range(n_ranks)) if emulate else [rank]
    wps, ten = {}, {}
    for k in mine:
        kw = {"world": n_ranks, "rank": k} if emulate else {}
        wp = WaveParallelRound(w.L, w.n_wave, w.n_hist, w.H, w.D, (w.F, w.gh, w.gw), kern, **kw)
        rows = slice(wp.c0 * w.L, wp.c1 * w.L)
        t = {"q": x.q[rows].to(dev), "k": x.k[rows].to(dev), "v": x.v[rows].to(dev)}
        t["q_out"] = torch.empty_like(t["q"])
        t["o"] = torch.empty_like(t["q"])
        t["kc"] = torch.empty(wp.ring_shape(), dtype=torch.bfloat16, device=dev)
        t["vc"] = torch.empty_like(t["kc"])
        wp.prefill_history(r0, [(r0 - w.n_hist + j, hk[j].to(dev), hv[j].to(dev))
                                for j in range(w.n_hist)], t["kc"], t["vc"])
        wps[k], ten[k] = wp, t
    stream = torch.cuda.current_stream(dev)

    def layer(r, ev=None):
        if not emulate:
            wp, t = wps[rank], ten[rank]
            wp.run_layer(r, t["q"], t["k"], t["v"], t["q_out"], t["kc"], t["vc"], t["o"])
            return
        for i, k in enumerate(mine):
            wp, t = wps[k], ten[k]
            if ev is not None:
                ev[i][0].record(stream)
            kern.append(wp.plan, r + wp.c0, t["q"], t["k"], t["v"], t["q_out"], t["kc"], t["vc"])
            if ev is not None:
                ev[i][1].record(stream)
        for k in mine:                       # stand-in for the NCCL delivery (not timed)
            for src, g in wps[k].incoming(r):
                ten[k]["kc"][wps[k].slot(g)].copy_(ten[src]["kc"][wps[src].slot(g)])
                ten[k]["vc"][wps[k].slot(g)].copy_(ten[src]["vc"][wps[src].slot(g)])
        for i, k in enumerate(mine):
            wp, t = wps[k], ten[k]
            if ev is not None:
                ev[i][2].record(stream)
            kern.attention(wp.plan, r + wp.c0, t["q_out"], t["kc"], t["vc"], t["o"])
            if ev is not None:
                ev[i][3].record(stream)

    rnd = r0
    for _ in range(args.warmup):
        layer(rnd)
        rnd += 1
    torch.cuda.synchronize(dev)
    full = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D)
    flops_step = wf.wf_useful_flops(full, r0)
    full.destroy()
    steps = args.steps
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in mine]
           for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    start.record(stream)
    for i in range(steps):
        layer(rnd, evs[i] if emulate else None)
        rnd += 1
    stop.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    for k in mine:
        st = wf.wf_sync_status(wps[k].plan)
        if st != wf.WF_OK:
            raise SystemExit("wave parallel: device status %d (%s)" % (st, wf.status_string(st)))
    ms_step = allreduce_max(dist, start.elapsed_time(stop), dev) / steps
    line = None
    if rank == 0:
        chunk_bytes = 2 * w.L * w.H * w.D * 2            # K and V of one chunk, bf16
        line = {
            "metric": METRIC + " (Wave Parallelism, %d ranks)" % n_ranks,
            "unit": "TFLOP/s", "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded bf16 N(0,1) q/k/v and history)",
            "config": {"workload": w.name, "wave_parallel_ranks": n_ranks,
                       "chunks_per_rank": [wp.n for wp in wps.values()] if emulate else None,
                       "parallelism": "wave-parallel %d (one-way K/V delivery, NCCL p2p)"
                       % n_ranks},
        }
        if not emulate:
            line.update({"value": round(flops_step / (ms_step * 1e-3) / 1e12, 3),
                         "ms_per_step": round(ms_step, 5), "projected": False})
        else:
            per = []
            for i, k in enumerate(mine):
                wp = wps[k]
                app = statistics.mean(e[i][0].elapsed_time(e[i][1]) for e in evs)
                att = statistics.mean(e[i][2].elapsed_time(e[i][3]) for e in evs)
                recv = len(wp.incoming(r0)) * chunk_bytes
                per.append({"rank": k, "chunks": [wp.c0, wp.c1], "append_ms": round(app, 5),
                            "attention_ms": round(att, 5), "recv_bytes": recv,
                            "recv_ms_at_peer_copy": round(recv / (PEER_COPY_GBS * 1e6), 5)})
            proj = max(p["append_ms"] + p["recv_ms_at_peer_copy"] + p["attention_ms"]
                       for p in per)
            # the single-GPU round in the same process, for the comparison
            plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
            q, k_, v = x.q.to(dev), x.k.to(dev), x.v.to(dev)
            kc = torch.empty((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
            vc = torch.empty_like(kc)
            q_out, o = torch.empty_like(q), torch.empty_like(q)
            for _ in range(3):
                wf.wf_qk_norm_rope_append(plan, r0, q, k_, v, None, gq, gk, q_out, kc, vc)
                wf.wf_chunk_causal_attn(plan, r0, q_out, kc, vc, o)
            torch.cuda.synchronize(dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(steps):
                wf.wf_qk_norm_rope_append(plan, r0 + i, q, k_, v, None, gq, gk, q_out, kc, vc)
                wf.wf_chunk_causal_attn(plan, r0 + i, q_out, kc, vc, o)
            b.record(stream)
            torch.cuda.synchronize(dev)
            single = a.elapsed_time(b) / steps
            plan.destroy()
            line.update({
                "value": round(flops_step / (proj * 1e-3) / 1e12, 3),
                "ms_per_step": round(proj, 5), "projected": True,
                "projection": "max over ranks of (append + incoming K/V at %.0f GB/s peer copy + "
                              "attention), each rank's kernels timed alone on one B200"
                              % PEER_COPY_GBS,
                "per_rank": per,
                "single_gpu_ms_per_step": round(single, 5),
                "speedup_projected": round(single / proj, 3),
                "emulation_ms_per_step": round(ms_step, 5),
            })
    for wp in wps.values():
        wp.destroy()
    if dist is not None:
        dist.destroy_process_group()
    return line


def run_block_round_loop(args, rank, world, local):
    """Full rounds of the model's blocks: every round runs the DiT block (the
    "block" leg of run_ours) of each of the workload's layers, layer after layer,
    the residual stream flowing from one layer into the next, each layer with its
    own ring and its own random-init weights; the rings advance one chunk per
    round.  Reports per-round latency (median, p90), rounds/s (one output chunk
    per round after pipeline fill) and useful TFLOP/s of the round."""
    import torch
    from chunk_causal_dit_b200 import wf

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = make_group(world, "nccl")
    w = wi.WORKLOADS[args.workload]
    if w.H * w.D not in wi.BLOCK_WIDTHS:
        raise SystemExit("no block widths for %d x %d heads" % (w.H, w.D))
    hidden, ffn = wi.BLOCK_WIDTHS[w.H * w.D]
    peaks, _ = load_peaks()
    plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
    layers = [wi.block_weights_on(dev, w, hidden, ffn, rank, l) for l in range(w.layers)]
    g = torch.Generator(device=dev)
    g.manual_seed(1009 * rank + 7)
    rings = [tuple(torch.randn((w.R, w.L, w.H, w.D), generator=g, device=dev).to(torch.bfloat16)
                   for _ in range(2)) for _ in range(w.layers)]
    x0 = wi.bf16_normal((w.T, hidden), rank, wi.STREAM_X).to(dev)
    X = torch.empty_like(x0)          # the residual stream, updated in place layer by layer
    h = torch.empty_like(x0)
    f = torch.empty((w.T, ffn), dtype=torch.bfloat16, device=dev)
    q_out = torch.empty((w.T, w.H, w.D), dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q_out)
    o2 = o.view(w.T, w.H * w.D)
    stream = torch.cuda.current_stream(dev)
    r0 = w.n_hist

    def run_round(r):
        X.copy_(x0)
        for lw, (kc, vc) in zip(layers, rings):
            mod = lw["mod"]
            wf.wf_layer_norm_modulate(plan, X, mod[0], mod[1], w.L, h, stream)
            wf.wf_qkv_proj_norm_rope_append(plan, r, h, lw["w_qkv"], lw["b_qkv"], lw["gamma_q"],
                                            lw["gamma_k"], q_out, kc, vc, stream)
            wf.wf_chunk_causal_attn(plan, r, q_out, kc, vc, o, None, stream)
            # gated residuals in place: X = X + gate * (...)
            wf.wf_linear(plan, o2, lw["w_o"], X, lw["b_o"], wf.WF_EPI_GATED_RESIDUAL, mod[2], X,
                         w.L, stream)
            wf.wf_layer_norm_modulate(plan, X, mod[3], mod[4], w.L, h, stream)
            wf.wf_linear(plan, h, lw["w_1"], f, lw["b_1"], wf.WF_EPI_GELU_TANH, None, None, 1,
                         stream)
            wf.wf_linear(plan, f, lw["w_2"], X, lw["b_2"], wf.WF_EPI_GATED_RESIDUAL, mod[5], X,
                         w.L, stream)

    rnd = r0
    for _ in range(args.warmup):
        run_round(rnd)
        rnd += 1
    torch.cuda.synchronize(dev)
    rounds = args.steps
    rev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(rounds)]
    clocks = ClockSampler(local)
    clocks.wait_ready()
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    for i in range(rounds):
        rev[i][0].record(stream)
        run_round(rnd)
        rev[i][1].record(stream)
        rnd += 1
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier(dist, dev)
    clocks.stop()
    status = wf.wf_sync_status(plan, stream)
    if status != wf.WF_OK:
        raise SystemExit("device status %d (%s)" % (status, wf.status_string(status)))
    per_round = [a.elapsed_time(b) for a, b in rev]
    ms_round = allreduce_max(dist, sum(per_round), dev) / rounds
    flops_round = w.layers * block_flops(w, hidden, ffn, wf.wf_useful_flops(plan, r0))
    clk = clocks.summary(t_wall0, t_wall1)
    plan.destroy()
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return None
    peak_tf = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    value = aggregate_tflops(world, flops_round, ms_round)
    srt = sorted(per_round)
    return {
        "metric": "DiT rounds of the wave model: useful TFLOP/s, rounds/s (= output chunks/s)",
        "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": rounds,
        "warmup": args.warmup, "ms_per_step": round(ms_round, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded bf16 N(0,1) residual stream; random-init weights per layer)",
        "config": {"workload": w.name, "layers": w.layers, "hidden": hidden, "ffn": ffn,
                   "heads": w.H, "head_dim": w.D, "chunk_tokens": w.L, "wave_chunks": w.n_wave,
                   "history_chunks": w.n_hist,
                   "step": "one full round: %d DiT blocks (LN, QKV + norm/RoPE/append, attention, "
                           "out-proj + gated residual, LN, FFN1 + GELU, FFN2 + gated residual)"
                           % w.layers,
                   "parallelism": "replica%d" % world,
                   "l2": "no flush: per-layer rings and weights total %.1f GB" % (
                       w.layers * (2 * w.R * w.L * w.H * w.D * 2 +
                                   2 * (4 * hidden * w.H * w.D + 2 * hidden * ffn)) / 1e9)},
        "round_ms_median": round(statistics.median(per_round), 3),
        "round_ms_p90": round(srt[min(len(srt) - 1, int(0.9 * len(srt)))], 3),
        "rounds_per_s": round(world * 1000.0 / ms_round, 3),
        "latent_frames_per_s": round(world * 1000.0 / ms_round * w.F, 3),
        "frac_sustained": round(value / world / peak_tf, 4),
        "gpu_launches": 7 * w.layers * rounds,    # plus one torch copy of x0 per round
        "clocks": clk,
    }


def run_wp_block(args, rank, world, local):
    """Wave Parallelism on the whole DiT block: every rank runs the block on its
    own chunks (LayerNorm, fused QKV projection, K/V delivery, attention, output
    projection, feed-forward); the round advances every step.  Under torchrun
    the delivery is NCCL and the step time the device-timed max over ranks; in
    one process the ranks run one after another on the one GPU, each half of a
    rank's block (before and after the delivery) is timed, and the step time is
    *projected* as the slowest rank's before + delivery (at the peer-copy
    bandwidth) + after, next to the single-GPU block measured in the same process."""
    import torch
    from chunk_causal_dit_b200 import wf
    from chunk_causal_dit_b200.wave_parallel import LibwfKernels, WaveParallelRound

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = make_group(world, "nccl")
    w = wi.WORKLOADS[args.workload]
    hidden, ffn = wi.BLOCK_WIDTHS[w.H * w.D]
    emulate = world == 1
    n_ranks = args.wp if emulate else world
    if not 1 <= n_ranks <= w.n_wave:
        raise SystemExit("Wave Parallelism needs 1..%d ranks" % w.n_wave)
    b = wi.block_inputs(w, hidden, ffn, seed=0)
    wts = {k: getattr(b, k).to(dev) for k in ("w_qkv", "b_qkv", "w_o", "b_o", "w_1", "b_1",
                                              "w_2", "b_2")}
    mod = b.mod.to(dev)
    kern = LibwfKernels(b.gamma_q.to(dev), b.gamma_k.to(dev))
    hk, hv = wi.history_prefill(w, seed=0)
    r0 = w.n_hist
    mine = list(range(n_ranks)) if emulate else [rank]

    def setup(wp):
        t = {"h": torch.empty((wp.rows, hidden), dtype=torch.bfloat16, device=dev),
             "q_out": torch.empty((wp.rows, w.H, w.D), dtype=torch.bfloat16, device=dev),
             "o": torch.empty((wp.rows, w.H, w.D), dtype=torch.bfloat16, device=dev),
             "f": torch.empty((wp.rows, ffn), dtype=torch.bfloat16, device=dev),
             "k_cache": torch.empty(wp.ring_shape(), dtype=torch.bfloat16, device=dev),
             "v_cache": torch.empty(wp.ring_shape(), dtype=torch.bfloat16, device=dev),
             "x0": b.x[wp.c0 * w.L:wp.c1 * w.L].to(dev)}
        t["x"] = torch.empty_like(t["x0"])
        wp.prefill_history(r0, [(r0 - w.n_hist + j, hk[j].to(dev), hv[j].to(dev))
                                for j in range(w.n_hist)], t["k_cache"], t["v_cache"])
        return t

    wps, ten = {}, {}
    for k in mine:
        kw = {"world": n_ranks, "rank": k} if emulate else {}
        wps[k] = WaveParallelRound(w.L, w.n_wave, w.n_hist, w.H, w.D, (w.F, w.gh, w.gw), kern,
                                   **kw)
        ten[k] = setup(wps[k])
    stream = torch.cuda.current_stream(dev)

    def step(r, ev=None):
        for k in mine:
            ten[k]["x"].copy_(ten[k]["x0"])
        if not emulate:
            wp, t = wps[rank], ten[rank]
            wp.run_block(r, t["x"], wts, mod, t)
            return
        ms = {k: wps[k].mod_rows(mod) for k in mine}
        for i, k in enumerate(mine):
            if ev is not None:
                ev[i][0].record(stream)
            wps[k].norm_and_qkv(r, ten[k]["x"], wts, ms[k], ten[k])
            if ev is not None:
                ev[i][1].record(stream)
        for k in mine:                       # stand-in for the NCCL delivery (not timed)
            for src, g in wps[k].incoming(r):
                for c in ("k_cache", "v_cache"):
                    ten[k][c][wps[k].slot(g)].copy_(ten[src][c][wps[src].slot(g)])
        for i, k in enumerate(mine):
            if ev is not None:
                ev[i][2].record(stream)
            wps[k].attention_and_rest(r, ten[k]["x"], wts, ms[k], ten[k])
            if ev is not None:
                ev[i][3].record(stream)

    rnd = r0
    for _ in range(args.warmup):
        step(rnd)
        rnd += 1
    torch.cuda.synchronize(dev)
    steps = args.steps
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in mine]
           for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    start.record(stream)
    for i in range(steps):
        step(rnd, evs[i] if emulate else None)
        rnd += 1
    stop.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    for k in mine:
        st = wf.wf_sync_status(wps[k].plan)
        if st != wf.WF_OK:
            raise SystemExit("wave parallel block: device status %d (%s)"
                             % (st, wf.status_string(st)))
    ms_step = allreduce_max(dist, start.elapsed_time(stop), dev) / steps
    full = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D)
    flops_step = block_flops(w, hidden, ffn, wf.wf_useful_flops(full, r0))
    full.destroy()
    line = None
    if rank == 0:
        line = {
            "metric": "DiT block over the wave, useful TFLOP/s (Wave Parallelism, %d ranks)"
                      % n_ranks,
            "unit": "TFLOP/s", "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded bf16; random-init block weights)",
            "config": {"workload": w.name, "hidden": hidden, "ffn": ffn,
                       "wave_parallel_ranks": n_ranks,
                       "parallelism": "wave-parallel %d (one-way K/V delivery, NCCL p2p)"
                       % n_ranks},
        }
        if not emulate:
            line.update({"value": round(flops_step / (ms_step * 1e-3) / 1e12, 3),
                         "ms_per_step": round(ms_step, 5), "projected": False})
        else:
            chunk_bytes = 2 * w.L * w.H * w.D * 2
            per = []
            for i, k in enumerate(mine):
                wp = wps[k]
                pre = statistics.mean(e[i][0].elapsed_time(e[i][1]) for e in evs)
                post = statistics.mean(e[i][2].elapsed_time(e[i][3]) for e in evs)
                recv = len(wp.incoming(r0)) * chunk_bytes
                per.append({"rank": k, "chunks": [wp.c0, wp.c1], "norm_qkv_ms": round(pre, 5),
                            "attention_and_rest_ms": round(post, 5), "recv_bytes": recv,
                            "recv_ms_at_peer_copy": round(recv / (PEER_COPY_GBS * 1e6), 5)})
            proj = max(p["norm_qkv_ms"] + p["recv_ms_at_peer_copy"] + p["attention_and_rest_ms"]
                       for p in per)
            one = WaveParallelRound(w.L, w.n_wave, w.n_hist, w.H, w.D, (w.F, w.gh, w.gw), kern,
                                    world=1, rank=0)
            t1 = setup(one)
            for i in range(3):
                t1["x"].copy_(t1["x0"])
                one.run_block(r0 + i, t1["x"], wts, mod, t1)
            torch.cuda.synchronize(dev)
            a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(steps):
                t1["x"].copy_(t1["x0"])
                one.run_block(r0 + 3 + i, t1["x"], wts, mod, t1)
            c.record(stream)
            torch.cuda.synchronize(dev)
            single = a.elapsed_time(c) / steps
            one.destroy()
            line.update({
                "value": round(flops_step / (proj * 1e-3) / 1e12, 3),
                "ms_per_step": round(proj, 5), "projected": True,
                "projection": "max over ranks of (LayerNorm + QKV, incoming K/V at %.0f GB/s peer "
                              "copy, attention + the rest of the block), each rank's kernels timed "
                              "alone on one B200" % PEER_COPY_GBS,
                "per_rank": per,
                "single_gpu_ms_per_step": round(single, 5),
                "speedup_projected": round(single / proj, 3),
            })
    for wp in wps.values():
        wp.destroy()
    if dist is not None:
        dist.destroy_process_group()
    return line


def run_round_loop(args, rank, world, local):
    """Full rounds of a multi-layer workload: every round runs, layer after layer,
    the append and the attention of each layer on that layer's own ring, then
    advances the ring by one chunk.  Reports per-round latency (median, p90)
    and rounds/s (one output chunk per round after pipeline fill)."""
    import torch

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = make_group(world, "nccl")
    w = wi.WORKLOADS[args.workload]
    peaks, peak_src = load_peaks()
    rounds = args.steps
    m = measure_round_loop(w, rounds, args.warmup, dev, peaks, seed=rank, dist=dist)
    total_ms = allreduce_max(dist, sum(m["per_round"]), dev)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return None
    ms_round = total_ms / rounds
    flops_layer, attn_ms, smry = m["flops_layer"], m["attn_ms"], m["summary"]
    peak_tf = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_note = "%s bf16_tflops_sustained (kernel inside a long loop)" % peak_src
    if m["timed_region_s"] < 1.0:
        peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        peak_note = "%s bf16_tflops (burst: timed region under a second)" % peak_src
    attn_tflops = flops_layer / (attn_ms * 1e-3) / 1e12
    value = aggregate_tflops(world, w.layers * flops_layer, ms_round)
    return {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": rounds,
        "warmup": args.warmup,
        "ms_per_step": round(ms_round, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded bf16 N(0,1); pool of two q/k/v sets across layers)",
        "config": {"workload": w.name, "layers": w.layers, "heads": w.H, "head_dim": w.D,
                   "chunk_tokens": w.L, "wave_chunks": w.n_wave, "history_chunks": w.n_hist,
                   "step": "one full round: %d x (append + attention), ring advanced" % w.layers,
                   "parallelism": "replica%d" % world,
                   "l2": "no flush: per-layer rings total %.1f GB" % (
                       w.layers * 2 * w.R * w.L * w.H * w.D * 2 / 1e9)},
        "round_ms_median": smry["round_ms_median"],
        "round_ms_p90": smry["round_ms_p90"],
        "rounds_per_s": round(world * 1e3 / ms_round, 2),
        "chunks_per_s": round(world * 1e3 / ms_round, 2),
        "roofline": {
            "kernel": "chunk_causal_attn_kernel",
            "bound": "tensor",
            "achieved": round(attn_tflops, 2),
            "peak": peak_tf,
            "unit": "TFLOP/s",
            "frac": round(attn_tflops / peak_tf, 4),
            "peak_source": peak_note,
            "traffic": None,
            "ms_per_launch": round(attn_ms, 5),
            "useful_flop_per_launch": flops_layer,
        },
        "e2e": None,
        "e2e_note": "not measured for the multi-layer round (%.1f GB of host q/k/v per round); "
                    "see the single-layer workload" % (w.layers * 6 * w.T * w.H * w.D / 1e9),
        "gpu_launches": 2 * w.layers * rounds,
        "clocks": m["clocks"],
    }


# --------------------------------------------------------- oracle (CPU) --

def oracle_round_setup(w, seed=0):
    """Host inputs of one steady-state round (round = n_hist) through the oracle."""
    import oracle
    r = w.n_hist
    x = wi.wave_inputs(w, seed=seed)
    hk, hv = wi.history_prefill(w, seed=seed)
    pos = oracle.positions(r, w.n_wave, w.F, w.gh, w.gw)
    qo, ko, vo = oracle.append(wi.bits(x.q), wi.bits(x.k), wi.bits(x.v), pos,
                               x.gamma_q.numpy(), x.gamma_k.numpy())
    cache = oracle.OracleCache(w.L)
    for j in range(w.n_hist):
        cache.put(j, wi.bits(hk[j]), wi.bits(hv[j]))
    cache.put_wave(r, ko, vo)
    k, v, ids = cache.round_keys(r, w.n_wave, w.n_hist)
    return r, qo, k, v, ids


def oracle_sample_step(w, r, qo, k, v, ids, n_pairs, rng):
    import oracle
    rows = rng.integers(0, w.T, n_pairs)
    heads = rng.integers(0, w.H, n_pairs)
    qids = np.arange(r, r + w.n_wave)
    t0 = time.perf_counter()
    oracle.chunk_causal_attn_rows(qo, qids, k, v, ids, w.L, rows, heads, want_lse=False)
    dt = time.perf_counter() - t0
    hv = min(w.n_hist, r)
    flops = float(sum(4.0 * w.D * (hv + row // w.L + 1) * w.L for row in rows))
    return flops, dt


def cpu_baseline(w, budget_s=15.0):
    import oracle
    r, qo, k, v, ids = oracle_round_setup(w)
    rng = np.random.default_rng(0)
    flops, secs = 0.0, 0.0
    n = 16
    while secs < budget_s:
        f, dt = oracle_sample_step(w, r, qo, k, v, ids, n, rng)
        flops += f
        secs += dt
        n = min(4096, n * 2)
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%.0f s of fp64 oracle attention on random (row, head) pairs of the "
                      "same round (%.3g useful FLOP)" % (secs, flops)}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    w = wi.WORKLOADS[args.workload]
    r, qo, k, v, ids = oracle_round_setup(w)
    rng = np.random.default_rng(1)
    pairs = args.ref_pairs
    for _ in range(args.warmup):
        oracle_sample_step(w, r, qo, k, v, ids, pairs, rng)
    flops, secs = 0.0, 0.0
    for _ in range(args.steps):
        f, dt = oracle_sample_step(w, r, qo, k, v, ids, pairs, rng)
        flops += f
        secs += dt
    value = flops / secs / 1e12
    sample = ("each step: fp64 oracle attention of %d random (row, head) pairs of the round "
              "(all their visible keys)" % pairs)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / args.steps, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded, same generator as the GPU arm)",
        "config": {"workload": w.name, "heads": w.H, "head_dim": w.D, "chunk_tokens": w.L,
                   "wave_chunks": w.n_wave, "history_chunks": w.n_hist},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                         "cores": oracle.num_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="wan13b_4step",
                    choices=sorted(wi.WORKLOADS) + ["vae_stage"],
                    help="vae_stage: only the streaming VAE-decode stage (residual block of "
                         "causal 3x3x3 convolutions at 120 x 208 x 384, 12 frames per chunk)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-block", action="store_true",
                    help="skip the DiT-block leg (timed after the attention step)")
    ap.add_argument("--attn", default="bf16", choices=["bf16", "fp8qk"],
                    help="attention variant: bf16 (default) or E4M3 Q.K^T with bf16 P.V")
    ap.add_argument("--blocks", action="store_true",
                    help="with a multi-layer workload: every layer runs the whole DiT block; "
                         "with --wp: Wave Parallelism on the whole block")
    ap.add_argument("--wp", type=int, default=0,
                    help="Wave Parallelism: under torchrun, split the wave over the ranks; "
                         "in one process, emulate N ranks on the one GPU (projected time)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other configurations' legs (configs and fp8qk objects)")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--ref-pairs", type=int, default=48)
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.workload == "vae_stage":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm times the "
                              "attention oracle; vae_stage has no CPU reference leg"}))
            return
        rank, world, local = dist_setup(args.gpus)
        line = run_vae(args, rank, world, local)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if args.attn != "bf16" and wi.WORKLOADS[args.workload].layers > 1:
        raise SystemExit("--attn %s times single-layer workloads only" % args.attn)
    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    elif args.wp and args.blocks:
        line = run_wp_block(args, rank, world, local)
    elif args.wp:
        line = run_wp(args, rank, world, local)
    elif wi.WORKLOADS[args.workload].layers > 1 and args.blocks:
        line = run_block_round_loop(args, rank, world, local)
    elif wi.WORKLOADS[args.workload].layers > 1:
        line = run_round_loop(args, rank, world, local)
    else:
        line = run_ours(args, rank, world, local)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
