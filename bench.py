"""Benchmark: attention forward+backward TFLOP/s of the d24 GQA SSSL layer stack.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]
    (N > 1: python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N ...)

One step is the whole hot path over one batch of synthetic input: for each of
the four layers (windows S, S, S, L) the fused prologue, the forward and the
backward through the C ABI. FLOPs count only the unmasked causal/window pairs:
12*D per pair per (batch, head) (forward 4*D, backward 8*D, no credit for the
backward's recomputation). Every rank runs its own batch (weak scaling, no
collective on the data path); the time is the max over ranks.

Prints one JSON line on rank 0. ``--impl reference`` times the float64 CPU
oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attn fwd+bwd TFLOP/s (bf16, causal/windowed) and % of B200 dense BF16 peak"
NOMINAL_BF16_TFLOPS = 2250.0  # NVIDIA B200 dense BF16 (HGX B200 datasheet: 36 PF sparse per 8 GPUs)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DEFAULT_CONFIG = 4           # the headline workload: d24 GQA SSSL
BF16_CONFIGS = (2, 3, 4, 5)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(w):
    return (f"{w.name}: B={w.B} T={w.T} H={w.H} Hk={w.Hk} D={w.D} windows={w.windows} "
            f"ve={['on' if v else 'off' for v in w.ve]} rope_base={w.rope_base:g} eps={w.eps:g}")


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled during the timed
    region: NVML polled from a thread every ~2 ms (read-only queries). The
    record is None when NVML is unavailable."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, indices):
        self.indices = list(indices) or [0]
        self.samples = []
        self.reasons = set()
        self.max_mhz = 0.0
        self._stop = None
        self._thread = None
        self._nvml = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            handles = [pynvml.nvmlDeviceGetHandleByIndex(i) for i in self.indices]
            self.max_mhz = max(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM) for h in handles)
        except Exception:
            self._nvml = None
            return
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                for h in handles:
                    try:
                        self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                        mask = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        for name, const in self.REASONS:
                            if mask & getattr(pynvml, const):
                                self.reasons.add(name)
                    except Exception:
                        pass
                self._stop.wait(0.002)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return None
        self._stop.set()
        self._thread.join(timeout=5)
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "source": "nvml, every ~2 ms during the timed region",
                "reasons": sorted(self.reasons)}


def rank_config_id(rank: int, config: int = DEFAULT_CONFIG) -> int:
    """Seed component of a rank's batch: every rank draws its own inputs."""
    return config + 1000 * rank


def reduce_max(values, dist, device):
    """Max over ranks of a list of floats (identity on one process)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None and dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def visible_gpu_indices(n_local):
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    if cvd:
        try:
            return [int(x) for x in cvd.split(",")][:n_local]
        except ValueError:
            return []
    return list(range(n_local))


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def layer_flops(w):
    """Per-layer FLOPs of one step: (fwd+bwd 12*D, fwd 4*D, bwd 8*D) per unmasked pair."""
    fl = lambda per: [per * w.D * w.pairs(W) * w.B * w.H for W in w.windows]  # noqa: E731
    return fl(12.0), fl(4.0), fl(8.0)


def roofline(ktimes, w, steps, peaks, peak_src):
    """Roofline object of the dominant kernel (the kind with the most device
    time in the per-kernel pass). The tensor-core kernels are timed inside a
    short region (tens of milliseconds at the maximum SM clock), so their
    denominator is the burst bf16 matmul peak."""
    _, flops_fwd, flops_bwd = layer_flops(w)
    dom = max(ktimes, key=lambda k: ktimes[k][0])
    dom_ms, dom_n = ktimes[dom]
    if dom in ("fwd", "bwd"):
        fl = flops_fwd if dom == "fwd" else flops_bwd
        achieved = sum(fl) * steps / (dom_ms * 1e-3) / 1e12
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        return {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 2),
                "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_src} bf16_tflops (burst: the timed region is short and "
                               f"runs at the maximum SM clock)",
                "frac_of_sustained": round(achieved / sus, 4),
                "launches": dom_n, "avg_launch_us": round(dom_ms / max(dom_n, 1) * 1e3, 2),
                "traffic": traffic_for(dom)}
    return {"kernel": dom, "bound": "hbm", "achieved": None, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": None, "traffic": traffic_for(dom)}


class Stack:
    """Device inputs, pinned host copies and output buffers of one workload's
    layer stack, with the step functions the benchmark times."""

    def __init__(self, w, dev, rank, cs, synth):
        import torch
        self.w, self.dev, self.cs = w, dev, cs
        self.specs = [cs.LayerSpec(w.B, w.T, w.H, w.Hk, w.D, W, has_ve=ve, dtype=w.dtype,
                                   rope_base=w.rope_base, eps=w.eps)
                      for W, ve in zip(w.windows, w.ve)]
        host = [synth.layer_inputs(w.B, w.T, w.H, w.Hk, w.D, ve, torch.bfloat16,
                                   config=rank_config_id(rank, w.config), layer=i, dO_std=w.dO_std)
                for i, ve in enumerate(w.ve)]
        self.pinned = [{k: (v.pin_memory() if v is not None else None) for k, v in h.items()}
                       for h in host]
        self.inp = [{k: (v.to(dev) if v is not None else None) for k, v in h.items()} for h in host]
        self.bufs = [cs.LayerBuffers(s, device=dev) for s in self.specs]
        self.stream = torch.cuda.current_stream(dev)
        out_names = ("O", "dQ", "dK", "dV", "dve", "dgate")
        self.host_out = [{n: torch.empty_like(getattr(b, n), device="cpu").pin_memory()
                          for n in out_names if getattr(b, n) is not None} for b in self.bufs]
        self.h2d = sum(v.numel() * v.element_size() for p in self.pinned for v in p.values()
                       if v is not None)
        self.d2h = sum(v.numel() * v.element_size() for o in self.host_out for v in o.values())
        self.s_in, self.s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def step(self):
        cs = self.cs
        for s, x, b in zip(self.specs, self.inp, self.bufs):
            cs.layer_forward(s, b, x["q"], x["k"], x["v"], x["ve"], x["gate"])
            cs.layer_backward(s, b, x["q"], x["k"], x["ve"], x["gate"], x["dO"])

    def step_e2e(self):
        """Host->device copies on one stream, kernels on the main one,
        device->host copies on a third, chained per layer by events, so that
        the two copy directions (PCIe is full duplex) and the kernels overlap."""
        import torch
        cs, stream, s_in, s_out = self.cs, self.stream, self.s_in, self.s_out
        fwd_names, grad_names = ("q", "k", "v", "ve", "gate"), ("dQ", "dK", "dV", "dve", "dgate")
        begin = torch.cuda.Event()
        begin.record(stream)
        s_in.wait_event(begin)
        s_out.wait_event(begin)
        for s, x, p, b, o in zip(self.specs, self.inp, self.pinned, self.bufs, self.host_out):
            with torch.cuda.stream(s_in):
                for n in fwd_names:
                    if p[n] is not None:
                        x[n].copy_(p[n], non_blocking=True)
                got_fwd = torch.cuda.Event()
                got_fwd.record(s_in)
                x["dO"].copy_(p["dO"], non_blocking=True)
                got_dO = torch.cuda.Event()
                got_dO.record(s_in)
            stream.wait_event(got_fwd)
            cs.layer_forward(s, b, x["q"], x["k"], x["v"], x["ve"], x["gate"], stream=stream)
            fwd_done = torch.cuda.Event()
            fwd_done.record(stream)
            stream.wait_event(got_dO)
            cs.layer_backward(s, b, x["q"], x["k"], x["ve"], x["gate"], x["dO"], stream=stream)
            bwd_done = torch.cuda.Event()
            bwd_done.record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(fwd_done)
                o["O"].copy_(b.O, non_blocking=True)
                s_out.wait_event(bwd_done)
                for n in grad_names:
                    if n in o:
                        o[n].copy_(getattr(b, n), non_blocking=True)
        # the next step overwrites these buffers: join both copy streams
        for side in (s_in, s_out):
            e = torch.cuda.Event()
            e.record(side)
            stream.wait_event(e)


def timed_steps(fn, k, stream, dev, flush_buf, world, dist):
    """Per-step device milliseconds of k calls of fn, CUDA events on the
    launching stream, a barrier and a synchronize on both sides; the L2
    flush buffer (if any) is written before each step, outside the events."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(k)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for a, b in evs:
        if flush_buf is not None:
            flush_buf.zero_()  # L2 holds nothing of the next step
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    return [a.elapsed_time(b) for a, b in evs]


# ---------------------------------------------------------------------- ours

def measure_stack(st, args, world, dist, flush_buf, warmup, steps, with_split=True):
    """Warm-up, the headline pass and (optionally) the per-kernel pass of one
    stack. Returns (per-step ms of the headline pass, per-kernel times)."""
    import torch
    cs = st.cs
    for _ in range(warmup):
        st.step()
    torch.cuda.synchronize(st.dev)
    cs.cswattn_sync_status()
    per_step = timed_steps(st.step, steps, st.stream, st.dev, flush_buf, world, dist)
    cs.cswattn_sync_status()
    ktimes = {}
    if with_split:
        # Per-kernel split: a second timed pass with CUDA events around every
        # kernel on the launching stream (the events serialise the kernels,
        # so this pass is a little slower than the headline).
        cs.cswattn_set_timing(True)
        cs.cswattn_kernel_times()
        split = timed_steps(st.step, steps, st.stream, st.dev, flush_buf, world, dist)
        ktimes = {k: v for k, v in cs.cswattn_kernel_times().items() if v[1] > 0}
        ktimes["_pass_ms"] = (sum(split), 0)
        cs.cswattn_set_timing(False)
        cs.cswattn_sync_status()
    return per_step, ktimes


def bwd_parts_of(cs, spec):
    """Backward parts per key tile, read back from the documented workspace
    layout: dq accumulator, dK and dV partial slots (parts x (B,T,Hk,D)
    float32 each), Delta and lse2 ((B,H,Tpad) float32), each padded to 256."""
    pad = lambda n: (n + 255) // 256 * 256  # noqa: E731
    ws = cs.attn_bwd_workspace_bytes(spec)
    B, T, H, Hk, D = spec.B, spec.T, spec.n_head, spec.n_kv_head, spec.head_dim
    tpad = (T + 63) // 64 * 64
    for parts in range(1, 9):
        if pad(B * H * T * D * 4) + 2 * pad(B * T * Hk * D * parts * 4) + 2 * pad(B * H * tpad * 4) == ws:
            return parts
    return None


def row_bytes(w, cs):
    """Bytes each row kernel moves per step (all layers), by its design: the
    prologue reads q, k, v (ve, gate) and writes q~, k~, v_eff and the rstd
    rows; the preprocess reads O, dO and lse, writes Delta and lse2 and clears
    the float32 dq accumulator; the epilogue reads the float32 dq~ and the
    parts' dk~/dv_eff, q, k (ve, gate), rstd, and writes dQ, dK, dV (dve,
    dgate)."""
    B, T, H, Hk, D = w.B, w.T, w.H, w.Hk, w.D
    e = 2  # bf16
    nq, nk, tok = B * T * H * D, B * T * Hk * D, B * T
    tpad = (T + 63) // 64 * 64
    out = {"prologue": 0, "bwd_pre": 0, "bwd_epi": 0}
    for W, ve in zip(w.windows, w.ve):
        spec = cs.LayerSpec(B, T, H, Hk, D, W, has_ve=ve, dtype="bf16", rope_base=w.rope_base, eps=w.eps)
        parts = bwd_parts_of(cs, spec) or 1
        vb = (nk * e + tok * Hk * e) if ve else 0
        out["prologue"] += 2 * (nq + 2 * nk) * e + vb + tok * (H + Hk) * 4
        out["bwd_pre"] += 2 * nq * e + B * H * T * 4 + 2 * B * H * tpad * 4 + nq * 4
        out["bwd_epi"] += (nq * 4 + 2 * parts * nk * 4 + (nq + nk) * e + tok * (H + Hk) * 4 + vb
                           + (nq + 2 * nk) * e + ((nk * e + tok * Hk * e) if ve else 0))
    return out


def kernel_table(ktimes, w, steps, cs=None, hbm=None):
    _, flops_fwd, flops_bwd = layer_flops(w)
    kern = {k: {"ms_per_step": round(v[0] / steps, 4), "launches": v[1]}
            for k, v in ktimes.items() if not k.startswith("_")}
    for k, fl in (("fwd", flops_fwd), ("bwd", flops_bwd)):
        if k in ktimes and ktimes[k][0] > 0:
            kern[k]["tflops"] = round(sum(fl) * steps / (ktimes[k][0] * 1e-3) / 1e12, 2)
    if cs is not None and hbm:
        for k, nbytes in row_bytes(w, cs).items():
            if k in ktimes and ktimes[k][0] > 0:
                gbs = nbytes * steps / (ktimes[k][0] * 1e-3) / 1e9
                kern[k]["bytes_per_step"] = nbytes
                kern[k]["gbs"] = round(gbs, 1)
                kern[k]["frac_hbm"] = round(gbs / hbm, 4)
    if "_pass_ms" in ktimes:
        kern["_pass"] = {"ms_per_step": round(ktimes["_pass_ms"][0] / steps, 4),
                         "note": "second timed pass with an event pair around every kernel"}
    return kern


def other_configs(args, dev, peaks, peak_src, flush_buf, cs, synth):
    """Device-timed throughput of the other bf16 workloads (one process only):
    the same headline and per-kernel passes, without e2e or CPU legs."""
    import torch
    out = {}
    for cid in BF16_CONFIGS:
        if cid == args.config:
            continue
        w = cs.WORKLOADS[cid]
        st = Stack(w, dev, 0, cs, synth)
        per_step, kt = measure_stack(st, args, 1, None, flush_buf, 3, args.steps)
        ms = sum(per_step) / args.steps
        fl = sum(layer_flops(w)[0])
        out[str(cid)] = {"workload": workload_desc(w), "value": round(fl / (ms * 1e-3) / 1e12, 2),
                         "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
                         "pct_of_peak": {"measured_burst": round(fl / (ms * 1e-3) / 1e12 / peaks.get(
                             "bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]), 4),
                             "nominal_dense": round(fl / (ms * 1e-3) / 1e12 / NOMINAL_BF16_TFLOPS, 4)},
                         "roofline": roofline({k: v for k, v in kt.items() if not k.startswith("_")},
                                              w, args.steps, peaks, peak_src),
                         "kernels": kernel_table(kt, w, args.steps, cs, peaks.get("hbm_gbs"))}
        del st
        torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    import causal_sliding_window_rope_b200 as cs
    from causal_sliding_window_rope_b200 import synth
    from causal_sliding_window_rope_b200.build import build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    if args.muon_only:
        # Profiling case: only the Newton-Schulz measurement.
        if rank == 0:
            peaks, peak_src = load_peaks()
            print(json.dumps({"muon_ns": muon_bench(dev, peaks, peak_src, steps=args.steps,
                                                    warmup=args.warmup)}), flush=True)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    if args.qkv_only:
        # Profiling case: only the QKV-projection measurement at the workload's layer shape.
        if rank == 0:
            peaks, peak_src = load_peaks()
            print(json.dumps({"qkv_projection": qkv_bench(cs.WORKLOADS[args.config], dev, peaks, peak_src,
                                                          steps=args.steps, warmup=args.warmup)}), flush=True)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    w = cs.WORKLOADS[args.config]
    if args.single_layer is not None:
        # Profiling case: one layer of the workload, same shapes and launches.
        i = args.single_layer
        w = cs.Workload(w.config, w.name + f" (layer {i} only)", w.B, w.T, w.H, w.Hk, w.D,
                        [w.windows[i]], [w.ve[i]], w.dtype, w.rope_base, w.eps, w.dO_std)
    st = Stack(w, dev, rank, cs, synth)
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flops_step = sum(layer_flops(w)[0])

    clocks = ClockSampler(visible_gpu_indices(world if world > 1 else 1) if rank == 0 else [])
    for _ in range(args.warmup):
        st.step()
    torch.cuda.synchronize(dev)
    cs.cswattn_sync_status()
    if rank == 0:
        clocks.start()
    # Headline: K steps as a user runs them (the kernels may overlap their
    # launches with the previous kernel's tail).
    step_ms = timed_steps(st.step, args.steps, st.stream, dev, flush_buf, world, dist)
    clk = clocks.stop() if rank == 0 else None
    cs.cswattn_sync_status()
    _, ktimes = measure_stack(st, args, world, dist, flush_buf, 0, args.steps)

    # e2e: host buffers in, results out, copies inside the timed region
    e2e_steps = max(1, min(args.steps, 5))
    if args.single_layer is None:
        for _ in range(2):
            st.step_e2e()
        torch.cuda.synchronize(dev)
        e2e_ms = sum(timed_steps(st.step_e2e, e2e_steps, st.stream, dev, None, world, dist))
    else:
        e2e_ms = float("nan")
    cs.cswattn_sync_status()

    total_ms, e2e_ms = reduce_max([sum(step_ms), e2e_ms], dist if world > 1 else None, dev)
    ms_per_step = total_ms / args.steps
    value = flops_step * world / (ms_per_step * 1e-3) / 1e12
    e2e_value = flops_step * world / (e2e_ms / e2e_steps * 1e-3) / 1e12

    if rank == 0:
        peaks, peak_src = load_peaks()
        kt = {k: v for k, v in ktimes.items() if not k.startswith("_")}
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 4),
            "step_ms": {"median": round(statistics.median(step_ms), 4),
                        "min": round(min(step_ms), 4), "rank": 0},
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) tensors shaped like the workload's layers)",
            "config": {"workload": workload_desc(w), "global_batch": w.B * world, "seq_len": w.T,
                       "parallelism": f"dp{world} (independent batch per GPU, no collective)",
                       "l2": "256 MiB buffer written between timed steps, outside the events",
                       "flops_per_step_per_gpu": flops_step, "flop_convention": "12*D per unmasked pair"},
            "pct_of_peak": {
                "measured_burst": round(value / world / peaks.get("bf16_tflops", 1590.0), 4),
                "measured_sustained": round(value / world / peaks.get("bf16_tflops_sustained", 1400.0), 4),
                "nominal_dense": round(value / world / NOMINAL_BF16_TFLOPS, 4),
                "peak_source": peak_src},
            "roofline": roofline(kt, w, args.steps, peaks, peak_src),
            "kernels": kernel_table(ktimes, w, args.steps, cs, peaks.get("hbm_gbs")),
            "gpu_launches": sum(n for _, n in kt.values()),
            "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": st.h2d, "d2h_bytes_per_step": st.d2h,
                    "ms_per_step": round(e2e_ms / e2e_steps, 3)},
            "clocks": clk,
        }
        solo = world == 1 and args.single_layer is None
        if solo and not args.no_decode:
            line["decode"] = decode_bench(w, dev, peaks, steps=args.steps, warmup=args.warmup,
                                          peak_src=peak_src)
        if solo and not args.no_muon:
            line["qkv_projection"] = qkv_bench(w, dev, peaks, peak_src, steps=args.steps, warmup=args.warmup)
        if solo and not args.no_muon:
            line["muon_ns"] = muon_bench(dev, peaks, peak_src, steps=args.steps, warmup=args.warmup)
        if solo and not args.no_other_configs:
            del st
            torch.cuda.empty_cache()
            line["other_configs"] = other_configs(args, dev, peaks, peak_src, flush_buf, cs, synth)
        if solo and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


DECODE_BATCH = 32  # sequences generating together


def decode_launches(B, Hk, T, W):
    """Kernels one attn_decode call launches: the attention kernel, and the
    combine kernel when a sequence's window is split (the library splits only
    while B * n_kv_head is below the 148 SMs, at most once per 128-key chunk
    the window can straddle)."""
    chunks = min(-(-min(W, T) // 128) + 1, -(-T // 128))
    splits = 1 if B * Hk >= 148 else min(148 // (B * Hk), chunks)
    splits = max(splits, -(-chunks // 31))
    return 1 + (splits > 1)


def decode_bench(w, dev, peaks, steps=20, warmup=5, peak_src="measured"):
    """One generation step over the workload's layer stack with a KV cache
    (attn_decode per layer): DECODE_BATCH sequences whose caches hold T-1
    tokens, so every layer reads its full window of K and V. HBM-bound: the
    roofline is the window's K/V bytes per step over the step's device time
    (the caches, 0.5 GB, exceed L2)."""
    import torch

    import causal_sliding_window_rope_b200 as cs
    B, T, H, Hk, D = DECODE_BATCH, w.T, w.H, w.Hk, w.D
    g = torch.Generator().manual_seed(4321)

    def rnd(*shape):
        return torch.randn(*shape, generator=g).to(torch.bfloat16).to(dev)

    layers = []
    for W, ve in zip(w.windows, w.ve):
        spec = cs.LayerSpec(B, T, H, Hk, D, W, has_ve=ve, dtype="bf16", rope_base=w.rope_base, eps=w.eps)
        layers.append(dict(
            spec=spec, q=rnd(B, H, D), k=rnd(B, Hk, D), v=rnd(B, Hk, D),
            ve=rnd(B, Hk, D) if ve else None, gate=rnd(B, Hk) if ve else None,
            kc=rnd(B, T, Hk, D), vc=rnd(B, T, Hk, D),
            O=torch.empty(B, H, D, dtype=torch.bfloat16, device=dev),
            lse=torch.empty(B, H, dtype=torch.float32, device=dev),
            ws=torch.empty(cs.attn_decode_workspace_bytes(spec), dtype=torch.uint8, device=dev)))
    lens = torch.full((B,), T - 1, dtype=torch.int32, device=dev)

    def step():
        for x in layers:
            cs.attn_decode(x["spec"], x["q"], x["k"], x["v"], x["ve"], x["gate"], lens, x["kc"],
                           x["vc"], x["O"], x["lse"], x["ws"])

    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    cs.cswattn_sync_status()
    stream = torch.cuda.current_stream(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    cs.cswattn_set_timing(True)
    cs.cswattn_kernel_times()
    for a, b in evs:
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize(dev)
    kt = cs.cswattn_kernel_times()
    cs.cswattn_set_timing(False)
    cs.cswattn_sync_status()
    ms = sum(a.elapsed_time(b) for a, b in evs) / steps
    # algorithmic bytes: the window's K and V rows, the new token's inputs and
    # outputs, the row written back to each cache
    kv = sum(B * Hk * min(W, T) * D * 2 * 2 for W in w.windows)
    small = len(layers) * B * ((H + 3 * Hk) * D * 2 + H * D * 2 + H * 4 + 2 * Hk * D * 2)
    nbytes = kv + small
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": f"one decode step of the layer stack, {B} sequences, caches of {T} rows "
                        f"holding {T - 1} tokens, windows {w.windows}",
            "ms_per_step": round(ms, 4), "tokens_per_s": round(B / (ms * 1e-3), 1),
            "kernel_ms_per_step": round(kt["decode"][0] / steps, 4),
            "launches_per_step": sum(decode_launches(B, Hk, T, W) for W in w.windows),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes_per_step": nbytes,
                         "peak_source": f"{peak_src} hbm_gbs"}}


# Muon's orthogonalisation on the d24 model's MLP weight shapes (4 x 1536 by
# 1536, and its transpose): the page prints two coefficient triples of the
# Polar-Express iteration, so a step here is those two iteration steps.
MUON_SHAPES = ((6144, 1536), (1536, 6144))


def muon_bench(dev, peaks, peak_src, steps=20, warmup=5):
    """Device time of muon_newton_schulz (three tensor-core products per
    iteration step: X^T X, b A + c A A, a X + X B) on MUON_SHAPES. FLOPs per
    iteration step: 2 m n^2 + 2 n^3 + 2 m n^2; the roofline divides them by
    the matrix-product kernel's own event time."""
    import torch

    import causal_sliding_window_rope_b200 as cs
    import oracle
    coeffs = oracle.POLAR_EXPRESS_PRINTED
    g = torch.Generator().manual_seed(4322)
    out = {}
    for m, n in MUON_SHAPES:
        X = torch.randn(m, n, generator=g, dtype=torch.float64)
        X = (X / X.norm()).to(torch.bfloat16).to(dev)
        Y = torch.empty_like(X)
        ws = torch.empty(cs.muon_ns_workspace_bytes(m, n), dtype=torch.uint8, device=dev)
        for _ in range(max(warmup, 3)):
            cs.muon_newton_schulz(X, Y, coeffs, ws)
        torch.cuda.synchronize(dev)
        cs.cswattn_sync_status()
        # The call is six short kernel launches; replaying it from a CUDA
        # graph keeps the host's launch work out of the device timing.
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            cs.muon_newton_schulz(X, Y, coeffs, ws, stream=side)
        torch.cuda.current_stream(dev).wait_stream(side)
        stream = torch.cuda.current_stream(dev)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize(dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a, b in evs:
            a.record(stream)
            graph.replay()
            b.record(stream)
        torch.cuda.synchronize(dev)
        cs.cswattn_sync_status()
        ms = sum(a.elapsed_time(b) for a, b in evs) / steps
        # eager calls for comparison (host launch work included)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            cs.muon_newton_schulz(X, Y, coeffs, ws)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        eager_ms = t0.elapsed_time(t1) / steps
        del graph
        # per iteration step: X^T X (2 m n^2), A A (2 n^3), X B (2 m n^2)
        flops = len(coeffs) * (2 * m * n * n + 2 * n ** 3 + 2 * m * n * n)
        tf = flops / (ms * 1e-3) / 1e12
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        out[f"{m}x{n}"] = {
            "workload": f"Newton-Schulz of a {m} x {n} bf16 matrix, {len(coeffs)} iteration steps "
                        f"(the printed Polar-Express coefficients)",
            "ms_per_call": round(ms, 4), "tflops": round(tf, 1), "gemm_launches_per_call": 3 * len(coeffs),
            "timing": "CUDA graph of one call, replayed; every kernel in it is the matrix product",
            "eager_ms_per_call": round(eager_ms, 4),
            "roofline": {"kernel": "gemm", "bound": "tensor", "achieved": round(tf, 1), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(tf / peak, 4),
                         "peak_source": f"{peak_src} bf16_tflops"}}
    return out


def qkv_bench(w, dev, peaks, peak_src, steps=20, warmup=5):
    """The step before the attention path at the workload's layer shape: the
    QKV projection of the block input (model dim = n_head * head_dim) fused
    with the prologue, and its backward (dx, dW), device time per call."""
    import torch

    import causal_sliding_window_rope_b200 as cs
    B, T, H, Hk, D = w.B, w.T, w.H, w.Hk, w.D
    C = H * D
    g = torch.Generator().manual_seed(4323)
    bf = torch.bfloat16
    spec = cs.LayerSpec(B, T, H, Hk, D, w.windows[0], has_ve=True, rope_base=w.rope_base, eps=w.eps)
    x = torch.randn(B, T, C, generator=g).to(bf).to(dev)
    wq = (torch.randn((H + 2 * Hk) * D, C, generator=g) / C ** 0.5).to(bf).to(dev)
    ve = torch.randn(B, T, Hk, D, generator=g).to(bf).to(dev)
    gate = torch.randn(B, T, Hk, generator=g).to(bf).to(dev)
    buf = cs.LayerBuffers(spec, device=dev)
    q = torch.empty(B, T, H, D, dtype=bf, device=dev)
    k = torch.empty(B, T, Hk, D, dtype=bf, device=dev)
    dx = torch.empty(B, T, C, dtype=bf, device=dev)
    dw = torch.empty((H + 2 * Hk) * D, C, dtype=torch.float32, device=dev)

    def fwd():
        cs.attn_qkv_prologue(spec, x, C, wq, ve, gate, q, k, buf.q_out, buf.k_out, buf.v_out,
                             buf.rstd_q, buf.rstd_k)

    def bwd():
        cs.attn_qkv_bwd(spec, x, C, wq, q, k, buf.v_out, dx, dw)  # any bf16 gradients of that shape

    scales = torch.empty(2, dtype=torch.float32, device=dev)
    ws8 = torch.empty(cs.attn_qkv_fp8_workspace_bytes(spec, C), dtype=torch.uint8, device=dev)

    def fwd_fp8():
        cs.attn_qkv_prologue_fp8(spec, x, C, wq, ve, gate, q, k, buf.q_out, buf.k_out, buf.v_out,
                                 buf.rstd_q, buf.rstd_k, scales, ws8)

    # The value-embedding gate's projection (gate logits from the first
    # GATE_CHANNELS channels of x; the page does not give the channel count,
    # a parameter of the call), against the prologue given the logits.
    GATE_CHANNELS = 32
    w_gate = (torch.randn(Hk, GATE_CHANNELS, generator=g) / GATE_CHANNELS ** 0.5).to(bf).to(dev)
    gate_out = torch.empty(B, T, Hk, dtype=bf, device=dev)
    dgx = torch.empty(B, T, GATE_CHANNELS, dtype=bf, device=dev)
    dwg = torch.empty(Hk, GATE_CHANNELS, dtype=torch.float32, device=dev)

    v_in = torch.randn(B, T, Hk, D, generator=g).to(bf).to(dev)

    def prologue_plain():
        cs.attn_prologue(spec, q, k, v_in, ve, gate, buf.q_out, buf.k_out, buf.v_out, buf.rstd_q, buf.rstd_k)

    def prologue_gated():
        cs.attn_prologue_gated(spec, q, k, v_in, ve, x, GATE_CHANNELS, w_gate, gate_out, buf.q_out,
                               buf.k_out, buf.v_out, buf.rstd_q, buf.rstd_k)

    def gate_bwd():
        cs.attn_gate_bwd(spec, x, GATE_CHANNELS, w_gate, gate, dgx, dwg)

    out = {}
    flops = 2.0 * B * T * C * (H + 2 * Hk) * D
    stream = torch.cuda.current_stream(dev)
    for name, fn, fl in (("fwd", fwd, flops), ("bwd", bwd, 2 * flops), ("fwd_fp8", fwd_fp8, flops),
                         ("prologue", prologue_plain, 0.0), ("prologue_gated", prologue_gated, 0.0),
                         ("gate_bwd", gate_bwd, 0.0)):
        for _ in range(max(warmup, 3)):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms = a.elapsed_time(b) / steps
        out[name] = {"ms_per_call": round(ms, 4)}
        if fl > 0:
            out[name]["tflops"] = round(fl / (ms * 1e-3) / 1e12, 1)
    cs.cswattn_sync_status()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    # E4M3 call: amax, quantization and the fused product; against the FP8
    # tensor peak taken as twice the bf16 one (the nominal dense ratio).
    out["fwd_fp8"]["frac_of_fp8_peak"] = round(out["fwd_fp8"]["tflops"] / (2 * peak), 4)
    return {"workload": f"QKV projection of the layer input (B={B} T={T} C={C} -> {H}+2x{Hk} heads of {D}) "
                        f"fused with the prologue (fwd; fwd_fp8 with E4M3 operands and tensor-wise "
                        f"scales, quantization included), and its backward dx, dW (bwd); the prologue "
                        f"given the gate logits, with them projected from x[..., :{GATE_CHANNELS}] "
                        f"(prologue_gated), and that projection's backward (gate_bwd); inputs L2-warm",
            **out, "roofline": {"kernel": "qkv fused product", "bound": "tensor",
                                "achieved": out["fwd"]["tflops"], "peak": peak, "unit": "TFLOP/s",
                                "frac": round(out["fwd"]["tflops"] / peak, 4),
                                "peak_source": f"{peak_src} bf16_tflops"}}


def traffic_for(kind):
    """DRAM bytes per launch from a committed ncu capture, if the kernel's
    source still matches the one the counters were taken on; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        with open(path) as f:
            d = json.load(f)
        ent = d.get(kind)
        if not ent:
            return None
        if ent.get("source_sha") != kernel_source_sha(kind):
            return None
        return ent.get("bytes_per_launch")
    except (OSError, ValueError):
        return None


def kernel_source_sha(kind):
    import hashlib
    files = {"fwd": ["fwd_sm100.cuh", "common.cuh"], "bwd": ["bwd_sm100.cuh", "common.cuh"],
             "prologue": ["prologue.cuh"], "bwd_pre": ["bwd_aux.cuh"], "bwd_epi": ["bwd_aux.cuh"]}
    h = hashlib.sha256()
    for fn in files.get(kind, []):
        with open(os.path.join(ROOT, "causal_sliding_window_rope_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------- oracle (CPU)

def oracle_sample(w):
    """A bounded slice of the workload for the float64 CPU oracle: batch 1, one
    KV head and its query group, all four layers' windows, full T."""
    import numpy as np
    return dict(B=1, T=w.T, H=w.H // w.Hk, Hk=1, D=w.D, windows=w.windows, ve=w.ve,
                flops=sum(12.0 * w.D * w.pairs(W) * 1 * (w.H // w.Hk) for W in w.windows),
                rng=np.random.default_rng(0))


def time_oracle_sample(w, n_layers=None):
    import numpy as np

    import oracle
    s = oracle_sample(w)
    layers = list(zip(s["windows"], s["ve"]))[: n_layers or len(s["windows"])]
    rng = s["rng"]
    t0 = time.perf_counter()
    flops = 0.0
    for W, ve in layers:
        L = oracle.Layer(s["B"], s["T"], s["H"], s["Hk"], s["D"], W, ve, rope_base=w.rope_base, eps=w.eps)
        q = rng.standard_normal((1, s["T"], s["H"], s["D"]))
        k = rng.standard_normal((1, s["T"], 1, s["D"]))
        v = rng.standard_normal((1, s["T"], 1, s["D"]))
        vee = rng.standard_normal((1, s["T"], 1, s["D"])) if ve else None
        g = rng.standard_normal((1, s["T"], 1)) if ve else None
        dO = rng.standard_normal((1, s["T"], s["H"], s["D"]))
        oracle.layer(L, q, k, v, vee, g, dO)
        flops += 12.0 * w.D * w.pairs(W) * s["H"]
    dt = time.perf_counter() - t0
    return flops, dt, len(layers)


def cpu_baseline(w, budget_s=20.0):
    """The oracle on a bounded sample, repeated until about half the budget
    (10-30 s of CPU work by default) has been spent."""
    import oracle
    oracle.build()
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    flops, dt, n = time_oracle_sample(w, n_layers=1)
    reps = 1
    if dt < budget_s / 4:
        flops, dt, reps = 0.0, 0.0, 0
        while dt < budget_s / 2 and reps < 8:
            f2, d2, n = time_oracle_sample(w, n_layers=None)
            flops, dt, reps = flops + f2, dt + d2, reps + 1
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "cpu_model": cpu_model(), "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"float64 C oracle (prologue+fwd+bwd+chain rule), batch 1, one KV head "
                      f"with its {w.H // w.Hk} query heads, T={w.T}, first {n} of the layer windows "
                      f"{w.windows}, {reps} repetition(s); FLOPs counted as 12*D per unmasked pair"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import causal_sliding_window_rope_b200 as cs
    import oracle
    oracle.build()
    w = cs.WORKLOADS[args.config]
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    for _ in range(args.warmup and 1):
        time_oracle_sample(w, n_layers=1)
    tot_f, tot_t = 0.0, 0.0
    for _ in range(args.steps):
        f, t, _ = time_oracle_sample(w, n_layers=1)
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(tot_t / args.steps * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(w), "sample": "one KV head group, batch 1, first layer (S window)"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                             "cpu_model": cpu_model(), "kind": "oracle", "sample": "float64 C oracle, batch 1, one KV head group, one S layer per step"},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", type=int, choices=BF16_CONFIGS, default=DEFAULT_CONFIG,
                    help="workload of the headline line (2: d12, 3: d12 SSSL, 4: d24 GQA SSSL, "
                         "5: long-context GQA)")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the device-timed summary of the other bf16 workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-muon", action="store_true",
                    help="skip the Newton-Schulz and QKV-projection measurements")
    ap.add_argument("--qkv-only", action="store_true",
                    help="profiling case: only the QKV-projection measurement")
    ap.add_argument("--muon-only", action="store_true",
                    help="profiling case: only the Newton-Schulz measurement")
    ap.add_argument("--no-decode", action="store_true", help="skip the KV-cache decode measurement")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--single-layer", type=int, default=None,
                    help="profiling case: time only this layer of the stack (no e2e, no CPU leg)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
