#!/usr/bin/env python
"""Benchmark of the flash-CCE ORPO head on B200.

One step = one pass of the whole head on one ORPO pair of the long-pair
workload (M = 8,192 head rows, D = 2,048, V = 262,144, bf16): forward GEMM
with the online-LSE epilogue, LSE merge, ORPO loss, cotangent, and the
backward (recompute, G', dH contraction).  Inputs are seeded synthetic
arrays with that shape and a random-initialised head.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 the script runs under torchrun: every rank processes its own pair
on its own GPU (independent problems, no data-path collective; weak
scaling); timing is the max over ranks.  Rank 0 prints one JSON line.

``--impl reference`` times the float64 CPU oracle (the only reference this
head has) on a bounded sample of rows per step, on the host cores.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "flash-CCE fwd+bwd tokens/sec and % of bf16 tensor peak at M=8192,V=262144"
WORKLOAD_ID = 2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "_fallback": True}
# SM clock of the fallback sustained figure (about 1.3 GHz under the 1 kW cap)
FALLBACK_SUSTAINED_MHZ = 1300.0


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", type=int, default=WORKLOAD_ID)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--workspace-mb", type=int, default=0,
                   help="workspace size (default: the library's default)")
    p.add_argument("--backward-mode", type=int, choices=[0, 1, 2, 3], default=0,
                   help="dense bf16 heads: 0 choose, 1 the grouped fused backward, 2 two "
                        "GEMMs per vocab chunk, 3 the sliced fused backward (M <= 64)")
    p.add_argument("--forward-mode", type=int, choices=[0, 1, 2], default=0,
                   help="4/8-bit heads: 0 choose (a transposed small-M kernel up to 256 "
                        "rows), 1 the tiled GEMM at every M, 2 the wide transposed form "
                        "from 1 row")
    p.add_argument("--quant-staging", type=int, choices=[0, 1, 2], default=0,
                   help="4/8-bit heads: 0 choose, 1 dequantise in the GEMM, 2 staged fp16 chunks")
    p.add_argument("--cta-pairs", type=int, choices=[0, 1], default=1,
                   help="1: 2-CTA (cta_group::2) tiles where they apply; 0: single-CTA tiles")
    p.add_argument("--graph", action="store_true",
                   help="time replays of the head pass captured as one CUDA graph (for the "
                        "launch-bound small workloads); per-kernel times then come from as "
                        "many profiled direct passes after the timed region")
    p.add_argument("--sweep", choices=["small_m", "small_m_q4"], default=None,
                   help="the W-stream (HBM-bound) regime, M in {64, 128, 256}, one JSON "
                        "line per M: small_m at D=2048, V=262144 (bf16 head); small_m_q4 "
                        "at D=4096, V=128256 (4-bit head, dequantised in the GEMMs)")
    return p.parse_args(argv)


# ---------------------------------------------------------------- helpers --

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def _sustained_mhz(peaks: dict):
    """SM clock (MHz) at which the sustained bf16 peak was measured, if the
    peaks file records one."""
    for k, v in peaks.items():
        kl = k.lower()
        if "sustain" in kl and ("mhz" in kl or "clock" in kl) and isinstance(v, (int, float)):
            return float(v)
    for k, v in peaks.items():   # nested records, e.g. {"bf16_sustained": {"sm_mhz": ...}}
        if "sustain" in k.lower() and isinstance(v, dict):
            for k2, v2 in v.items():
                if ("mhz" in k2.lower() or "clock" in k2.lower()) and isinstance(v2, (int, float)):
                    return float(v2)
    return FALLBACK_SUSTAINED_MHZ if peaks.get("_fallback") else None


def choose_peak(peaks: dict, src: str, clk: dict, timed_s: float) -> dict:
    """Denominator of the tensor roofline.  The burst peak (a cuBLAS GEMM
    timed alone) applies unless the timed region is seconds long AND its
    median SM clock fell to the clock of the sustained measurement (a
    seconds-long GEMM loop under the power cap); then the sustained peak
    applies.  Also returns the burst peak scaled by median / max SM clock."""
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    med, mx = (clk or {}).get("sm_mhz"), (clk or {}).get("sm_max_mhz")
    sus_mhz = _sustained_mhz(peaks)
    use_sus = (timed_s >= 2.0 and med is not None and sus_mhz is not None
               and med <= sus_mhz * 1.02)
    at_med = burst * med / mx if (med and mx) else None
    if use_sus:
        why = (f"{src} bf16 sustained: timed region {timed_s:.2f} s, median SM clock "
               f"{med:.0f} MHz <= {sus_mhz:.0f} MHz of the sustained measurement")
    else:
        why = (f"{src} bf16 burst: timed region {timed_s:.2f} s, median SM clock "
               f"{med if med is None else round(med)} MHz (sustained peak taken at "
               f"{sus_mhz if sus_mhz is None else round(sus_mhz)} MHz)")
    return {"peak": sus if use_sus else burst, "source": why, "peak_at_median_clock": at_med}


# The sources that decide the tensor-core kernels' memory traffic: the kernel
# template and its PTX wrappers, and the host code that picks tiles, chunks
# and launch shapes.
TRAFFIC_SOURCES = ("gemm_tc.cuh", "fused_bwd.cuh", "ptx.cuh", "cce.cu")


def strip_comments(text: str) -> str:
    """C/C++ source without its comments and with whitespace collapsed, so
    that a comment-only edit leaves the hash of the code unchanged (string
    and character literals are kept as they are)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_hash(read=None) -> str:
    """Hash of the code (comments stripped) of TRAFFIC_SOURCES; `read(name)`
    returns a file's text (default: the working tree)."""
    src = os.path.join(ROOT, "lm_head_cross_flash_b200", "csrc")
    if read is None:
        def read(n):
            with open(os.path.join(src, n), encoding="utf-8") as f:
                return f.read()
    h = hashlib.sha256()
    for n in TRAFFIC_SOURCES:
        h.update(n.encode() + strip_comments(read(n)).encode())
    return h.hexdigest()[:16]


def load_traffic(kind: str, workload: str):
    """Per-launch DRAM bytes of `kind` from the committed ncu summary, if it
    was taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(kind)
    if not e or e.get("src_hash") != source_hash() or e.get("workload") != workload:
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle samples of one GPU while it runs."""

    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.5)

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                c, m, pw = float(f[1]), float(f[2]), float(f[3])
            except ValueError:
                continue
            mx = max(mx, m)
            if pw < 250.0:  # idle samples before the GPU ramps up
                continue
            sm.append(c)
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_uuid(dev) -> str:
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:  # pragma: no cover
        return str(dev)


def aggregate(dist, local_ms: float, local_tokens: float, device=None):
    """Max step time and summed tokens over ranks (identity when not
    distributed)."""
    if dist is None or not dist.is_initialized():
        return local_ms, local_tokens
    import torch
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    n = torch.tensor([local_tokens], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t.item()), float(n.item())


# ------------------------------------------------------------ CPU oracle --

def oracle_head(wl):
    """The head's weights as the method defines them, float64."""
    import numpy as np
    from oracle import flash_cce as O
    if wl.wformat == "q4g64":
        return O.dequant_affine_q4(wl.q_packed, wl.q_scales, wl.q_biases)
    return wl.W.astype(np.float64)


def oracle_rows(wl, W64, rows, g):
    """The oracle's per-row work of one head pass (forward and dH) on `rows`."""
    from oracle import flash_cce as O
    logp, lse, _ = O.head_forward(wl.H[rows], W64, wl.labels[rows], block=len(rows))
    O.head_dh(wl.H[rows], W64, wl.labels[rows], g[rows], lse, block=len(rows))
    return logp


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def time_oracle(wl, seconds: float, rows_per_block: int = 8):
    """Oracle throughput (rows/s) on a time-bounded sample of rows."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    from lm_head_cross_flash_b200 import synthetic as S
    cores = cpu_threads()
    W64 = oracle_head(wl)
    g = S.random_cotangent(wl).astype(np.float64)
    order = np.random.default_rng(0).permutation(wl.M)
    done, t0 = 0, time.perf_counter()
    with threadpool_limits(limits=cores):
        while time.perf_counter() - t0 < seconds and done < wl.M:
            rows = np.sort(order[done:done + rows_per_block])
            oracle_rows(wl, W64, rows, g)
            done += len(rows)
    dt = time.perf_counter() - t0
    return done / dt, cores, done, dt


# -------------------------------------------------------------- our arm --

def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from lm_head_cross_flash_b200 import cce
    from lm_head_cross_flash_b200 import synthetic as S

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cce.cce_set_quant_staging(args.quant_staging)
    cce.cce_set_backward_mode(args.backward_mode)
    cce.cce_set_forward_mode(args.forward_mode)
    cce.cce_set_cta_pairs(bool(args.cta_pairs))

    wl = S.make_workload(args.workload)
    H, head, labels = cce.upload_workload(wl, dev)
    torch.cuda.reset_peak_memory_stats(dev)
    base_alloc = torch.cuda.memory_allocated(dev)
    free0, _ = torch.cuda.mem_get_info(dev)
    buf = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, cce.h_dtype(H), head, dev,
                                ws_bytes=(args.workspace_mb << 20) or None)
    stream = torch.cuda.current_stream(dev)

    def step():
        cce.orpo_head_pass(H, head, labels, wl.layout_tuple, wl.lam, wl.scope, wl.filter_eps,
                           wl.block_skip, buf, stream)

    run_step = step
    if args.graph:
        run_step = cce.HeadPassGraph(H, head, labels, wl.layout_tuple, wl.lam, wl.scope,
                                     wl.filter_eps, wl.block_skip, buf).replay

    sampler = ClockSampler(gpu_uuid(dev))
    sampler.start()
    for _ in range(max(3, args.warmup)):
        run_step()
    torch.cuda.synchronize(dev)
    st = cce.cce_device_status(buf.ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    cce.cce_profile_enable(not args.graph)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    # one event per step boundary as well, for the median and minimum step
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    e0.record(stream)
    marks[0].record(stream)
    for i in range(args.steps):
        run_step()
        marks[i + 1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms_total = e0.elapsed_time(e1)
    step_ms = sorted(marks[i].elapsed_time(marks[i + 1]) for i in range(args.steps))
    if args.graph:  # kernel times of the same work, from direct passes
        cce.cce_profile_enable(True)
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize(dev)
    prof = cce.cce_profile_read()
    cce.cce_profile_enable(False)
    sampler.stop()
    peak_mem = torch.cuda.max_memory_allocated(dev) - base_alloc
    free1, _ = torch.cuda.mem_get_info(dev)
    st = cce.cce_device_status(buf.ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after timing")

    ms_max, tokens = aggregate(dist if world > 1 else None, ms_total, float(wl.M * args.steps), dev)
    ms_step = ms_max / args.steps

    # End to end through the public API: every step copies its H and labels
    # in from pinned host memory and its dH and loss back.  As a trainer
    # would drive it, the copies run on a second stream, double-buffered, so
    # step i's copies overlap the compute of its neighbours; the timed region
    # runs from the first upload to the last download.
    e2e = None
    if not args.no_e2e:
        import dataclasses
        hH = (torch.from_numpy(wl.H_bits.view(np.int16)).view(torch.bfloat16)
              if wl.dtype == "bf16" else torch.from_numpy(wl.H)).pin_memory()
        hy = torch.from_numpy(wl.labels).pin_memory()
        hdH = [torch.empty(wl.M, wl.D, dtype=torch.float32).pin_memory() for _ in range(2)]
        hout = [torch.empty(8, dtype=torch.float64).pin_memory() for _ in range(2)]
        Hd = [torch.empty_like(H) for _ in range(2)]
        yd = [torch.empty_like(labels) for _ in range(2)]
        bufs = [buf, dataclasses.replace(buf, dH=torch.empty_like(buf.dH),
                                         out8=torch.empty_like(buf.out8))]
        copy = torch.cuda.Stream(dev)
        ev = {k: [torch.cuda.Event() for _ in range(2)]
              for k in ("up", "done", "down")}

        def e2e_run(n):
            for i in range(n):
                j = i & 1
                with torch.cuda.stream(copy):
                    if i >= 2:
                        copy.wait_event(ev["done"][j])  # step i-2 has read Hd[j]
                    Hd[j].copy_(hH, non_blocking=True)
                    yd[j].copy_(hy, non_blocking=True)
                    ev["up"][j].record(copy)
                stream.wait_event(ev["up"][j])
                if i >= 2:
                    stream.wait_event(ev["down"][j])  # dH[j] of step i-2 is home
                cce.orpo_head_pass(Hd[j], head, yd[j], wl.layout_tuple, wl.lam, wl.scope,
                                   wl.filter_eps, wl.block_skip, bufs[j], stream)
                ev["done"][j].record(stream)
                with torch.cuda.stream(copy):
                    copy.wait_event(ev["done"][j])
                    hdH[j].copy_(bufs[j].dH, non_blocking=True)
                    hout[j].copy_(bufs[j].out8, non_blocking=True)
                    ev["down"][j].record(copy)

        e2e_run(3)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(copy)
        stream.wait_event(t0)
        e2e_run(args.steps)
        t1.record(copy)  # after the last download, which waits for the last pass
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e_ms, e_tok = aggregate(dist if world > 1 else None, t0.elapsed_time(t1),
                                float(wl.M * args.steps), dev)
        if not all(np.isfinite(h.numpy()[0]) for h in hout):
            raise RuntimeError("non-finite loss in the end-to-end pass")
        e2e = {"value": e_tok / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(hH.numel() * hH.element_size() + hy.numel() * 4),
               "d2h_bytes_per_step": int(hdH[0].numel() * 4 + hout[0].numel() * 8),
               "pipelining": "copies on a second stream, double-buffered H, labels, dH, loss"}

    clk = sampler.summary()
    if world > 1:
        allc = [None] * world
        dist.all_gather_object(allc, clk)
        meds = [c["sm_mhz"] for c in allc if c["sm_mhz"]]
        clk = {"sm_mhz": min(meds) if meds else None,
               "sm_max_mhz": max((c["sm_max_mhz"] or 0) for c in allc) or None,
               "reasons": sorted(set(r for c in allc for r in c["reasons"])),
               "samples": sum(c["samples"] for c in allc)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rps, cores, rows, dt = time_oracle(wl, args.cpu_seconds)
        cpu = {"value": rps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{rows} rows of the {wl.name} workload (forward logp/lse and dH per "
                         f"row, float64, logits materialised per row block) in {dt:.1f} s",
               "extrapolated_full_pass_s": wl.M / rps,
               "extrapolated_note": "extrapolated: M rows at the sampled rate"}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return None

    peaks, peaks_src = load_peaks()
    flop_step = 6.0 * wl.M * wl.V * wl.D
    # executed work: every row in the forward, rows with a nonzero cotangent
    # in the two backward GEMMs (the response scope zeroes the prompt rows)
    m_b = int((buf.coeff != 0).sum().item())
    flop_exec = 2.0 * wl.M * wl.V * wl.D + 4.0 * m_b * wl.V * wl.D
    tflops = flop_step / (ms_step / 1e3) / 1e12
    # roofline of the dominant kernel kind (largest summed time)
    per_kind_flops = {"fwd_lse_gemm": 2.0 * wl.M * wl.V * wl.D,  # per step
                      "bwd_grad_gemm": 2.0 * wl.M * wl.V * wl.D,
                      "bwd_dh_gemm": 2.0 * wl.M * wl.V * wl.D,
                      # recompute of the logits and the dH contraction, one kernel
                      "bwd_fused": 4.0 * wl.M * wl.V * wl.D,
                      "bwd_sliced": 4.0 * wl.M * wl.V * wl.D}
    kinds = {k: v for k, v in prof.items() if v[1] > 0}
    dom = max(kinds, key=lambda k: kinds[k][0])
    dom_ms, dom_n = kinds[dom]
    launches_per_step = dom_n / args.steps
    peak_s = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_b = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    pk = choose_peak(peaks, peaks_src, clk, ms_max / 1e3)  # ms_max: the whole timed region
    if dom in per_kind_flops:
        achieved = per_kind_flops[dom] * args.steps / (dom_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": pk["peak"],
                "unit": "TFLOP/s", "frac": achieved / pk["peak"],
                "traffic": load_traffic(dom, wl.name),
                "launches_per_step": launches_per_step,
                "avg_launch_ms": dom_ms / dom_n,
                "flops_per_launch": per_kind_flops[dom] / launches_per_step,
                "peak_source": pk["source"],
                "frac_burst": achieved / peak_b,
                "frac_sustained": achieved / peak_s,
                "peak_at_median_clock": pk["peak_at_median_clock"],
                "frac_at_median_clock": (achieved / pk["peak_at_median_clock"]
                                         if pk["peak_at_median_clock"] else None)}
    else:  # pragma: no cover
        roof = {"bound": "hbm", "kernel": dom, "achieved": None, "peak": peaks.get("hbm_gbs"),
                "unit": "GB/s", "frac": None, "traffic": None}
    gpu_launches = int(sum(v[1] for v in kinds.values()))
    out = {
        "metric": METRIC,
        "value": tokens / (ms_max / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms_step,
        "step_ms": {"median": statistics.median(step_ms), "min": step_ms[0],
                    "max": step_ms[-1], "note": "this rank, per-step CUDA events"},
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("f16 (4-bit head dequantised in-kernel)" if wl.wformat == "q4g64"
                  else "bf16" if wl.dtype == "bf16" else "f32"),
        "data": "synthetic: seeded inputs of the workload recipe, random-init head",
        "config": {"workload": wl.name, "M": wl.M, "D": wl.D, "V": wl.V, "P": wl.P,
                   "Rc": wl.Rc, "Rr": wl.Rr, "sft_scope": wl.scope, "lambda": wl.lam,
                   "filter_eps": wl.filter_eps, "block_skip": wl.block_skip,
                   "parallelism": f"dp{world} (independent pairs, no collective)",
                   "l2": "inputs larger than L2 (W is 1.07 GB, L2 126 MB); no flush",
                   "workspace_bytes": int(buf.ws.numel()),
                   "cta_pairs": bool(args.cta_pairs),
                   "cuda_graph": bool(args.graph),
                   "quant_staging": ["choose", "in-kernel", "staged"][args.quant_staging],
                   "backward": ["choose", "fused", "two GEMMs", "sliced"][args.backward_mode]},
        "tflops": tflops,
        "executed": {"rows_backward": m_b, "tflop_per_step": flop_exec / 1e12,
                     "tflops": flop_exec / (ms_step / 1e3) / 1e12,
                     "note": "2*M*V*D + 4*M_b*V*D; skipped vocab tiles (skip_tiles) not subtracted"},
        "pct_bf16_peak": {"sustained": 100.0 * tflops / peak_s,
                          "burst": 100.0 * tflops / peak_b,
                          "roofline_peak": 100.0 * tflops / pk["peak"],
                          "source": peaks_src},
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": gpu_launches,
        "clocks": clk,
        "kernels_ms_per_step": {k: v[0] / args.steps for k, v in kinds.items()},
        "kernel_launches_per_step": {k: v[1] / args.steps for k, v in kinds.items()},
        "peak_mem_bytes": int(peak_mem),
        "mem_get_info_delta_bytes": int(free0 - free1),
        "logits_bytes_avoided": int(wl.M) * int(wl.V) * 4,
        "skip_tiles": buf.skip.cpu().tolist(),
    }
    return out


# ------------------------------------------------------ small-M sweep --

def run_small_m(args, quant=False):
    """Forward and backward of the head at M = 64, 128, 256: the regime where
    streaming W from HBM bounds the time.  bf16 head: D = 2,048, V = 262,144,
    flat H.  quant: the 4-bit head of the long-context workload (D = 4,096,
    V = 128,256, groups of 64), dequantised inside the GEMMs.  Achieved GB/s
    counts the method's minimum bytes: W once per pass (as stored: 16 or 4.25
    bits per weight), H in, dH out and the per-row / per-block statistics.
    design_bytes are the bytes the backward that ran must move: the fused
    backwards (dense bf16 heads) read W from HBM once and add their partial
    dH buffers; the two-GEMM backward reads W twice and moves G'' through
    HBM.  With --backward-mode 3 (the sliced backward) only M = 64 runs."""
    import torch

    from lm_head_cross_flash_b200 import cce
    from lm_head_cross_flash_b200 import synthetic as S
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cce.cce_set_backward_mode(args.backward_mode)
    cce.cce_set_forward_mode(args.forward_mode)
    peaks, peaks_src = load_peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    lines = []
    for M in (64, 128, 256):
        if args.backward_mode == 3 and M > 64:
            lines.append({"sweep": "small_m_q4" if quant else "small_m", "M": M,
                          "skipped": "the sliced backward (mode 3) takes at most 64 rows"})
            continue
        P = M // 8
        Rc = (M - P) // 2
        if quant:
            wl = S.make_custom(4, M_split=(P, Rc, M - P - Rc))
        else:
            wl = S.make_custom(2, M_split=(P, Rc, M - P - Rc), D=2048, V=262144)
        H, head, labels = cce.upload_workload(wl, dev)
        buf = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, cce.h_dtype(H), head, dev)
        stream = torch.cuda.current_stream(dev)

        def fwd():
            cce.cce_forward(H, head, labels, buf.logp, buf.lse, buf.tgt, buf.blockmax, buf.ws,
                            stream)

        def bwd():
            cce.cce_backward_dh(H, head, labels, buf.lse, buf.coeff, wl.filter_eps, None,
                                buf.dH, buf.skip, buf.ws, stream)

        fwd()
        cce.orpo_grad_coeffs(buf.logp, labels, wl.layout_tuple, wl.lam, wl.scope, buf.coeff,
                             buf.ws, stream)
        for _ in range(max(3, args.warmup)):
            fwd()
            bwd()
        torch.cuda.synchronize(dev)

        def timed(f):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                f()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            return e0.elapsed_time(e1) / args.steps

        t_f, t_b = timed(fwd), timed(bwd)
        st = cce.cce_device_status(buf.ws)
        if st != 0:
            raise RuntimeError(f"device status {st} in the small-M sweep (M={M})")
        wbytes = (wl.V * wl.D / 2.0 + 2 * 2.0 * wl.V * wl.D / 64) if quant else 2.0 * wl.V * wl.D
        cols = cce.blockmax_cols(wl.V)
        stats = 4.0 * M * cols + 4.0 * 4 * M
        fwd_bytes = wbytes + 2.0 * M * wl.D + stats
        bwd_bytes = wbytes + 2.0 * M * wl.D + 4.0 * M * wl.D + 3 * 4.0 * M
        plan = cce.cce_query_plan(M, cce.h_dtype(H), head, buf.ws.numel())
        if plan["bwd_fused"]:
            nparts = plan["bwd_fused_buffers"] - 1
            bwd_design = bwd_bytes + 3 * 4.0 * nparts * M * wl.D  # parts written, read; dH RMW
        elif plan["bwd_sliced"]:
            # W once; one partial dH per cluster written and read back
            bwd_design = bwd_bytes + 2 * 4.0 * plan["bwd_sliced_clusters"] * M * wl.D
        else:
            bwd_design = 2 * wbytes + 2.0 * M * wl.D + 4.0 * M * wl.D + 2 * 2.0 * M * wl.V
        line = {"sweep": "small_m_q4" if quant else "small_m", "M": M, "D": wl.D, "V": wl.V,
                "dtype": "f16 (4-bit head dequantised in-kernel)" if quant else "bf16",
                "steps": args.steps, "fwd_ms": t_f, "bwd_ms": t_b,
                "fwd_gbs": fwd_bytes / (t_f / 1e3) / 1e9,
                "bwd_gbs": bwd_bytes / (t_b / 1e3) / 1e9,
                "fwd_frac_hbm": fwd_bytes / (t_f / 1e3) / 1e9 / hbm,
                "bwd_frac_hbm": bwd_bytes / (t_b / 1e3) / 1e9 / hbm,
                "fwd_bytes": fwd_bytes, "bwd_bytes": bwd_bytes,
                "fwd_form": {0: "tiled GEMM", 1: "transposed small-M (head tile in TMEM)",
                             2: "transposed, 128-row units (head tile in TMEM)"}[
                                 plan["fwd_q_small_m"]],
                "bwd_form": ("fused" if plan["bwd_fused"] else
                             "sliced" if plan["bwd_sliced"] else "two GEMMs per vocab chunk"),
                "bwd_design_bytes": bwd_design,
                "bwd_design_gbs": bwd_design / (t_b / 1e3) / 1e9,
                "tokens_per_s": M / ((t_f + t_b) / 1e3),
                "hbm_peak_gbs": hbm, "peak_source": f"{peaks_src} hbm_gbs (MEASURED_PEAKS.json)",
                "l2": f"W ({wbytes / 1e9:.2f} GB as stored) larger than the 126 MB L2; no flush"}
        lines.append(line)
        del buf, H, head, labels
        torch.cuda.empty_cache()
    return lines


# -------------------------------------------------------- reference arm --

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import numpy as np
    from threadpoolctl import threadpool_limits

    from lm_head_cross_flash_b200 import synthetic as S
    wl = S.make_workload(args.workload)
    W64 = oracle_head(wl)
    g = S.random_cotangent(wl).astype(np.float64)
    cores = cpu_threads()
    rows_per_step = 4
    order = np.random.default_rng(1).permutation(wl.M)
    with threadpool_limits(limits=cores):
        for i in range(max(3, args.warmup)):
            oracle_rows(wl, W64, np.sort(order[:rows_per_step]), g)
        t0 = time.perf_counter()
        for i in range(args.steps):
            r = np.sort(order[(i * rows_per_step) % wl.M:][:rows_per_step])
            oracle_rows(wl, W64, r, g)
        dt = time.perf_counter() - t0
    value = rows_per_step * args.steps / dt
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic: seeded inputs of the workload recipe, random-init head",
        "config": {"workload": wl.name, "M": wl.M, "D": wl.D, "V": wl.V,
                   "sample_rows_per_step": rows_per_step},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows_per_step} rows per step of the {wl.name} workload "
                                   "(forward logp/lse and dH per row, float64)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    if args.sweep in ("small_m", "small_m_q4"):
        for line in run_small_m(args, quant=args.sweep == "small_m_q4"):
            print(json.dumps(line), flush=True)
        return
    out = run_reference(args) if args.impl == "reference" else run_ours(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
