#!/usr/bin/env python
"""Throughput of exact tiled attention (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = the whole hot path over one batch of synthetic input: for every
variant of the workload (default: B=2, H=16, N=8192, d=128, causal -- the GPT-style
2k-hidden long-context layer, the largest single-GPU workload) the forward kernel,
then the backward's three launches (D and lse pre-pass, dK/dV kernel, dQ kernel). Metric: algorithmic TFLOPs/s, counting the forward as
4 B H N^2 d (halved for causal, times the kept-tile fraction for block-sparse)
and the backward as 2.5x the forward.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a device
synchronise; every step is timed with CUDA events on the launching stream, and
L2 is flushed (256 MiB write) before each timed step, outside the step's events.
Multi-GPU (torchrun): every rank runs the same workload on its own inputs (weak
scaling, no data-path collective); the reported time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle (plain definition, materialised
scores) on a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd / fwd+bwd TFLOPs/s and % of B200 dense BF16 peak"
# NVIDIA's dense (not 2:4-sparse) bf16 tensor figure for one B200, reported beside the
# measured cuBLAS peak so that both denominators are visible.
SPEC_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}


# ---------------------------------------------------------------- workloads

def workload(name: str):
    """(B, H, N, d, variants) where a variant is (label, causal, sparse_density or None)."""
    from exact_tiled_attention_34_b200.inputs import WORKLOADS, sweep_shape
    if name.startswith("sweep_"):
        # sweep_N4096_d128_causal / sweep_N4096_d128
        parts = name.split("_")
        N = int(parts[1][1:])
        d = int(parts[2][1:])
        B, H = sweep_shape(N, d)
        causal = len(parts) > 3 and parts[3] == "causal"
        return dict(B=B, H=H, N=N, Nk=N, d=d, variants=[("causal" if causal else "noncausal", causal, None)],
                    do_scale=0.5, dropout_p=0.0)
    w = WORKLOADS[name]
    variants = []
    if "sparse_density" in w:
        variants.append(("blocksparse", False, w["sparse_density"]))
    else:
        for c in w["causal"]:
            variants.append(("causal" if c else "noncausal", c, None))
    return dict(B=w["B"], H=w["H"], N=w["N"], Nk=w.get("Nk", w["N"]), d=w["d"], variants=variants, do_scale=1.0,
                dropout_p=w.get("dropout_p", 0.0))


# ---------------------------------------------------------------- multi-rank helpers
# Every (batch, head) is independent, so ranks run the workload on their own inputs
# (weak scaling) and share nothing on the data path; the process group only carries
# barriers and the max-over-ranks reduction of the measured device time.

def rank_seed(rank: int) -> int:
    """Input seed of a rank: each rank processes its own shard of the job."""
    return rank


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (the value itself when alone)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, flops_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Whole-job TFLOPs/s: all ranks' algorithmic FLOPs over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (max_ms * 1e-3) / 1e12


def fwd_flops(B, H, N, d, causal, density=1.0, Nk=None):
    """Forward FLOPs 4 B H N Nk d over the visible (query, key) pairs: causal counts
    Nq Nk - Nq^2 / 2 pairs (exactly half for Nq = Nk, the square convention; the
    causal mask is bottom-right aligned and Nq <= Nk here); block-sparse scales by
    the kept-tile fraction."""
    Nk = N if Nk is None else Nk
    pairs = N * Nk - 0.5 * N * N if causal else N * Nk
    return 4.0 * B * H * pairs * d * density


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.idx)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        return parse_clock_lines(self.lines)


def parse_clock_lines(lines):
    """Summary of ClockSampler.FIELDS rows (csv, no header, no units): median SM clock, the
    largest maximum clock, and the throttle reasons seen active in any sample; None when no
    row parses. Rows with fewer fields or non-numeric clocks ("[N/A]") are skipped."""
    sm, mx, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in lines:
        f = [x.strip() for x in ln.split(",")]
        if len(f) < 9:
            continue
        try:
            sm.append(float(f[1]))
            mx.append(float(f[2]))
        except ValueError:
            continue
        for n, v in zip(names, f[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
            "samples": len(sm)}


# ---------------------------------------------------------------- helpers

def peaks(path=None):
    """Roofline denominators: hbm_gbs, bf16_tflops (burst) and bf16_tflops_sustained from
    MEASURED_PEAKS.json where the file gives them as positive numbers (at its top level or
    one level down), each missing one from the machine's fallback figures. The kind says which:
    "measured", "fallback", or "measured, partly fallback". A missing or unreadable file
    means the fallback figures, never an error."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json") if path is None else path
    out = dict(FALLBACK_PEAKS)
    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return out, "fallback"
    if not isinstance(d, dict):
        return out, "fallback"
    scopes = [d] + [v for v in d.values() if isinstance(v, dict)]
    found = 0
    for key in FALLBACK_PEAKS:
        for sc in scopes:
            v = sc.get(key)
            if isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0:
                out[key] = float(v)
                found += 1
                break
    if found == 0:
        return out, "fallback"
    return out, "measured" if found == len(FALLBACK_PEAKS) else "measured, partly fallback"


# The files the profiled attention kernels and their launches are compiled from: a
# committed ncu figure stays valid while none of them changes.
KERNEL_SOURCES = ("fa_api.cu", "fa_bwd.cuh", "fa_bwd_fused.cuh", "fa_bwd256.cuh", "fa_dropout.cuh", "fa_fwd.cuh", "fa_fwd256.cuh", "fa_ptx.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_tiled_attention_34_b200", "csrc")
    for fn in KERNEL_SOURCES:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, wl_name: str):
    """Per-launch DRAM bytes of `kernel` on `wl_name` from a committed ncu summary,
    or None if there is none or the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{wl_name}.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for ln in f:
            if ":" in ln and not ln.startswith("#"):
                k, v = ln.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("source_hash") != kernel_source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def use_host_cores() -> int:
    """Let the oracle's BLAS use every core this process may run on. torch.distributed.run
    sets OMP_NUM_THREADS=1 in each rank; the oracle runs on rank 0 alone, so without this it
    would be timed on one core under the launcher and on all of them without it. Returns the
    thread count BLAS reports afterwards."""
    try:
        from threadpoolctl import threadpool_limits
        n = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
        threadpool_limits(limits=n, user_api="blas")
    except Exception:
        pass
    return blas_threads()


_HOST_INPUTS = {}


def cpu_oracle_sample(wl, budget_s: float, seed: int = 0):
    """Time the fp64 oracle's forward+backward head by head (all variants of the
    workload per head) until ~budget_s seconds have passed. Returns (TFLOPs/s, desc, s)."""
    import oracle
    from exact_tiled_attention_34_b200.inputs import make_qkv, make_tile_mask
    B, H, N, d = wl["B"], wl["H"], wl["N"], wl["d"]
    key = (B, H, N, d, seed, wl["do_scale"])
    if key not in _HOST_INPUTS:
        _HOST_INPUTS[key] = make_qkv(B, H, N, d, seed=seed, do_scale=wl["do_scale"])
    t = _HOST_INPUTS[key]
    sc = 1.0 / math.sqrt(d)
    masks = {}
    flops, heads, el = 0.0, 0, 0.0
    for b in range(B):
        for h in range(H):
            x = {k: v[b:b + 1, h:h + 1] for k, v in t.items()}
            for (label, causal, dens) in wl["variants"]:
                m = None
                if dens is not None:
                    if dens not in masks:
                        masks[dens] = make_tile_mask(-(-N // 128), seed=seed, density=dens).numpy()
                    m = masks[dens]
                kept = 1.0 if m is None else float(m.sum()) / m.size
                t0 = time.perf_counter()
                oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], causal, sc, m, 128)
                el += time.perf_counter() - t0
                flops += 3.5 * fwd_flops(1, 1, N, d, causal, kept)
            heads += 1
            if el >= budget_s:
                break
        if el >= budget_s:
            break
    desc = (f"{heads} of {B * H} (batch, head) pairs, fwd+bwd of every variant "
            f"({', '.join(v[0] for v in wl['variants'])}), fp64 NumPy, {el:.1f} s")
    return flops / el / 1e12, desc, el


def line_config(wl_name, wl, world: int) -> dict:
    """The `config` object of both arms' JSON lines: the workload and the job's layout,
    identical for the kernels and for the oracle so that the two lines describe the same
    configuration (how each arm computes a step is stated outside it)."""
    return {"workload": wl_name, "B": wl["B"], "H": wl["H"], "N": wl["N"], "d": wl["d"],
            "variants": [v[0] for v in wl["variants"]],
            "l2": "kernels: flushed before every timed step (256 MiB write, outside the step events); "
                  "oracle: host memory",
            "parallelism": f"replicas x{world} (independent (batch, head) shards, no collective)"}


# ---------------------------------------------------------------- reference arm

def run_reference(args, wl_name, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    use_host_cores()
    budget = 1.0  # seconds of oracle work per step
    for _ in range(args.warmup):
        cpu_oracle_sample(wl, budget)
    vals, times = [], []
    for _ in range(args.steps):
        v, desc, el = cpu_oracle_sample(wl, budget)
        vals.append(v)
        times.append(el)
    value = statistics.mean(vals)
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOPs/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * statistics.mean(times), 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1), bf16-rounded inputs)",
        "config": line_config(wl_name, wl, int(os.environ.get("WORLD_SIZE", args.gpus))),
        "step": "per step: fp64 forward+backward of sampled (batch, head) pairs of the workload (all variants)",
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPs/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: {desc}"},
        "e2e": {"value": round(value, 6), "unit": "TFLOPs/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm

def run_ours(args, wl_name, wl):
    import torch
    import torch.distributed as dist

    import exact_tiled_attention_34_b200 as fa
    from exact_tiled_attention_34_b200.inputs import make_qkv, make_tile_mask

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    fa.lib()

    B, H, N, d = wl["B"], wl["H"], wl["N"], wl["d"]
    sc = 1.0 / math.sqrt(d)
    host = make_qkv(B, H, N, d, seed=rank_seed(rank), do_scale=wl["do_scale"])
    t = {k: v.to(dev) for k, v in host.items()}
    masks = {}
    for (_, _, dens) in wl["variants"]:
        if dens is not None:
            masks[dens] = make_tile_mask(-(-N // 128), seed=0, density=dens).to(dev)
    fused = args.backward == "fused"
    ws = torch.empty(fa.bwd_workspace_bytes(B, H, N, d, deterministic=not fused), dtype=torch.uint8, device=dev)
    outs = {}
    for (label, _, _) in wl["variants"]:
        outs[label] = dict(o=torch.empty_like(t["q"]), lse=torch.empty((B, H, N), dtype=torch.float32, device=dev),
                           dq=torch.empty_like(t["q"]), dk=torch.empty_like(t["q"]), dv=torch.empty_like(t["q"]))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    step_flops = 0.0
    kinds = {}
    for (label, causal, dens) in wl["variants"]:
        kept = 1.0 if dens is None else float(masks[dens].float().mean())
        f = fwd_flops(B, H, N, d, causal, kept)
        kinds[label] = dict(causal=causal, mask=None if dens is None else masks[dens], fwd=f, bwd=2.5 * f)
        step_flops += 3.5 * f

    def one_step(ev=None):
        # ev: dict label -> 5 events [start, after fwd, after pre, after main, after dQ]
        # main: the fused kernel (dK, dV, dQ shares) or the dK/dV kernel; dQ: the
        # accumulator's conversion or the dQ kernel.
        for (label, causal, _) in wl["variants"]:
            k = kinds[label]
            x = outs[label]
            e = None if ev is None else ev[label]
            if e:
                e[0].record(stream)
            if k["mask"] is None:
                fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc, out=x["o"], lse=x["lse"])
            else:
                fa.forward_blocksparse(t["q"], t["k"], t["v"], k["mask"], scale=sc, out=x["o"], lse=x["lse"])
            if e:
                e[1].record(stream)
            if fused:
                fa.bwd_fused_preprocess(x["o"], t["do"], x["lse"], ws)
            else:
                fa.bwd_preprocess(x["o"], t["do"], x["lse"], ws)
            if e:
                e[2].record(stream)
            if fused:
                fa.bwd_fused_main(t["q"], t["k"], t["v"], t["do"], x["dk"], x["dv"], ws, causal=causal, scale=sc,
                                  tile_mask=k["mask"])
            else:
                fa.bwd_dkdv(t["q"], t["k"], t["v"], t["do"], x["dk"], x["dv"], ws, causal=causal, scale=sc,
                            tile_mask=k["mask"])
            if e:
                e[3].record(stream)
            if fused:
                fa.bwd_fused_dq(x["dq"], ws, scale=sc)
            else:
                fa.bwd_dq(t["q"], t["k"], t["v"], t["do"], x["dq"], ws, causal=causal, scale=sc,
                          tile_mask=k["mask"])
            if e:
                e[4].record(stream)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize(dev)
    st, dt = fa.device_status(dev)
    if st != 0:
        raise SystemExit(f"device status {st} (site {dt}) after warm-up")

    evs = [{label: [torch.cuda.Event(enable_timing=True) for _ in range(5)] for (label, _, _) in wl["variants"]}
           for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)  # let the sampler take its first reading
    wall0 = time.perf_counter()
    for s in range(args.steps):
        flush.zero_()
        one_step(evs[s])
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    st, dt = fa.device_status(dev)
    if st != 0:
        raise SystemExit(f"device status {st} (site {dt}) in the timed region")

    # per-kernel and per-step device times (ms)
    per = {label: dict(fwd=0.0, pre=0.0, main=0.0, dq=0.0) for (label, _, _) in wl["variants"]}
    step_ms = []
    for s in range(args.steps):
        tot = 0.0
        for (label, _, _) in wl["variants"]:
            e = evs[s][label]
            a = [e[i].elapsed_time(e[i + 1]) for i in range(4)]
            per[label]["fwd"] += a[0]
            per[label]["pre"] += a[1]
            per[label]["main"] += a[2]
            per[label]["dq"] += a[3]
            tot += sum(a)
        step_ms.append(tot)
    total_ms = max_over_ranks(sum(step_ms), dev)
    K = args.steps
    value = job_throughput(world, step_flops, K, total_ms)

    pk, pk_kind = peaks()
    sustained = clk is not None and clk["sm_mhz"] < 0.9 * clk.get("sm_max_mhz", 1965.0)
    peak = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
    peak_label = ("sustained" if sustained else "burst") + f" bf16, {pk_kind}"

    breakdown = {}
    main_flops, main_ms = 0.0, 0.0
    for (label, _, _) in wl["variants"]:
        k = kinds[label]
        p = {kk: v / K for kk, v in per[label].items()}
        bwd_ms = p["pre"] + p["main"] + p["dq"]
        breakdown[label] = {
            "fwd_ms": round(p["fwd"], 4), "bwd_ms": round(bwd_ms, 4),
            "bwd_pre_ms": round(p["pre"], 4), "bwd_main_ms": round(p["main"], 4), "bwd_dq_ms": round(p["dq"], 4),
            "fwd_tflops": round(k["fwd"] / (p["fwd"] * 1e-3) / 1e12, 2),
            "bwd_tflops": round(k["bwd"] / (bwd_ms * 1e-3) / 1e12, 2),
            "fwd_bwd_tflops": round(3.5 * k["fwd"] / ((p["fwd"] + bwd_ms) * 1e-3) / 1e12, 2),
            "fwd_pct_peak": round(100 * k["fwd"] / (p["fwd"] * 1e-3) / 1e12 / peak, 1),
            "bwd_pct_peak": round(100 * k["bwd"] / (bwd_ms * 1e-3) / 1e12 / peak, 1),
            "fwd_pct_spec_peak": round(100 * k["fwd"] / (p["fwd"] * 1e-3) / 1e12 / SPEC_BF16_TFLOPS, 1),
            "bwd_pct_spec_peak": round(100 * k["bwd"] / (bwd_ms * 1e-3) / 1e12 / SPEC_BF16_TFLOPS, 1),
        }
        # The step's dominant kernel. Fused: S^T, dP^T, dV, dK, dQ = five N x N x d products =
        # the whole backward's 2.5x the forward count. dK/dV kernel: four = 2x.
        main_flops += (2.5 if fused else 2.0) * k["fwd"]
        main_ms += p["main"]
    achieved = main_flops / (main_ms * 1e-3) / 1e12
    main_kernel = "fa_bwd_fused_kernel" if fused else "fa_bwd_dkdv_kernel"
    roofline = {"kernel": main_kernel + (" (backward dK, dV and dQ shares, 5 products per tile pair)" if fused
                                         else " (backward dK/dV, 4 products per tile pair)"),
                "bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "peak_kind": peak_label,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "traffic": profiled_traffic(main_kernel, wl_name)}

    # ---- end to end through the public API, host buffers, copies inside the timed region
    # Three streams, as a user pipelines host data through the library: step s's inputs go
    # host -> device on a copy stream while step s - 1 computes, and its results go device
    # -> host on a second copy stream while step s + 1 computes. Every step's copies are
    # inside the timed region; two sets of device buffers alternate between steps, and
    # events order each reuse after the copies that read or write the set.
    e2e_steps = max(3, min(K, 30))
    pin = {k: v.pin_memory() for k, v in host.items()}
    labels = [label for (label, _, _) in wl["variants"]]
    res_host = [{label: {n: torch.empty(outs[label][n].shape, dtype=outs[label][n].dtype).pin_memory()
                         for n in ("o", "lse", "dq", "dk", "dv")} for label in labels} for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = sum(v.numel() * v.element_size() for v in res_host[0][labels[0]].values()) * len(labels)
    dev_in = [{k: torch.empty_like(v, device=dev) for k, v in pin.items()} for _ in range(2)]
    dev_out = [{label: {n: torch.empty_like(outs[label][n]) for n in ("o", "lse", "dq", "dk", "dv")}
                for label in labels} for _ in range(2)]
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready = [ev() for _ in range(2)]    # set's inputs are on the device
    in_free = [ev() for _ in range(2)]     # compute is done reading the set's inputs
    out_ready = [ev() for _ in range(2)]   # compute wrote the set's outputs
    out_free = [ev() for _ in range(2)]    # the set's outputs are on the host
    for e in in_free + out_free:
        e.record(stream)

    def e2e_step(s):
        b = s & 1
        with torch.cuda.stream(s_h2d):
            s_h2d.wait_event(in_free[b])
            for k, v in pin.items():
                dev_in[b][k].copy_(v, non_blocking=True)
            in_ready[b].record(s_h2d)
        stream.wait_event(in_ready[b])
        stream.wait_event(out_free[b])
        x, y = dev_in[b], dev_out[b]
        for (label, causal, _) in wl["variants"]:
            k, r = kinds[label], y[label]
            if k["mask"] is None:
                fa.forward(x["q"], x["k"], x["v"], causal=causal, scale=sc, out=r["o"], lse=r["lse"])
                fa.backward(x["q"], x["k"], x["v"], r["o"], r["lse"], x["do"], causal=causal, scale=sc,
                            workspace=ws, grads=(r["dq"], r["dk"], r["dv"]), deterministic=not fused)
            else:
                fa.forward_blocksparse(x["q"], x["k"], x["v"], k["mask"], scale=sc, out=r["o"], lse=r["lse"])
                fa.backward_blocksparse(x["q"], x["k"], x["v"], r["o"], r["lse"], x["do"], k["mask"], scale=sc,
                                        workspace=ws, grads=(r["dq"], r["dk"], r["dv"]),
                                        deterministic=not fused)
        in_free[b].record(stream)
        out_ready[b].record(stream)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(out_ready[b])
            for label in labels:
                for n in ("o", "lse", "dq", "dk", "dv"):
                    res_host[b][label][n].copy_(y[label][n], non_blocking=True)
            out_free[b].record(s_d2h)

    for s_ in range(2):
        e2e_step(s_)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_h2d.wait_event(e0)  # the first copy starts inside the timed region
    for s_ in range(e2e_steps):
        e2e_step(s_)
    stream.wait_event(out_free[(e2e_steps - 1) & 1])  # the last results are on the host
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_value = job_throughput(world, step_flops, e2e_steps, e2e_ms)
    # The device-side results of the last step are the ones the host copy holds.
    last = res_host[(e2e_steps - 1) & 1][labels[0]]
    if not torch.isfinite(last["dq"].float()).all():
        raise SystemExit("end-to-end step produced non-finite gradients")

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOPs/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(total_ms / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) inputs rounded to bf16; per-rank seeds)",
        "config": line_config(wl_name, wl, world),
        "step": ("per variant: forward, backward pre-pass (D, lse rows, dQ accumulator zeroed), fused "
                 "backward kernel (dK, dV, dQ shares reduced in fp32), dQ conversion" if fused else
                 "per variant: forward, backward pre-pass, backward dK/dV kernel, backward dQ kernel"),
        "backward": ("fused: one kernel, dQ reduced in fp32 by TMA reduce-add (run-to-run order varies)"
                     if fused else "deterministic: dK/dV kernel + dQ kernel (bit-reproducible)"),
        "pct_of_peak": round(100 * value / world / peak, 2),
        "pct_of_spec_peak": round(100 * value / world / SPEC_BF16_TFLOPS, 2),
        "peak_tflops": peak, "peak_kind": peak_label,
        "breakdown": breakdown,
        "roofline": roofline,
        "gpu_launches": 4 * len(wl["variants"]) * K,
        "wall_s_timed_region": round(wall, 4),
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOPs/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "api": "exact_tiled_attention_34_b200.forward/backward (C ABI), pinned host buffers; "
                       "H2D, compute and D2H on three streams, next step's inputs copied during this step"},
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        use_host_cores()
        v, desc, el = cpu_oracle_sample(wl, args.cpu_budget)
        line["cpu_baseline"] = {"value": round(v, 6), "unit": "TFLOPs/s", "cores": blas_threads(),
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- table of workloads

def run_table(args):
    """Per-workload forward / backward device times (not the contract line): one JSON line
    per (workload, variant), median of --steps timed repetitions, L2 flushed before each."""
    import torch

    import exact_tiled_attention_34_b200 as fa
    from exact_tiled_attention_34_b200.inputs import SWEEP_D, SWEEP_N, make_qkv, make_tile_mask

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    names = ["pr1", "b8h16n2048d64", "b2h16n8192d128_causal", "b1h16n16384d64_sparse", "b8h16n2000d64_ragged",
             "b2h16n8000d128_ragged_causal", "b4h16q512k8192d128_causal", "b4h16n4096d96", "b2h8n8192d256",
             "b8h16n2048d64_dropout", "b2h16n8192d128_causal_dropout"]
    names += [f"sweep_N{N}_d{d}{c}" for d in SWEEP_D for N in SWEEP_N for c in ("", "_causal")]
    if args.only:
        names = [n for n in names if any(o in n for o in args.only.split(","))]
    pk, pk_kind = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for name in names:
        wl = workload(name)
        B, H, N, Nk, d = wl["B"], wl["H"], wl["N"], wl["Nk"], wl["d"]
        sc = 1.0 / math.sqrt(d)
        t = {k: v.to(dev) for k, v in make_qkv(B, H, N, d, seed=0, do_scale=wl["do_scale"]).items()}
        if Nk != N:  # keys and values of their own length
            kv = make_qkv(B, H, Nk, d, seed=1, with_do=False)
            t["k"], t["v"] = kv["k"].to(dev), kv["v"].to(dev)
        det_ok = d != 256  # head dim 256 has only the fused backward
        ws = torch.empty(fa.bwd_workspace_bytes(B, H, N, min(d, 128)), dtype=torch.uint8, device=dev)
        ws_f = torch.empty(fa.bwd_workspace_bytes(B, H, N, d, deterministic=False), dtype=torch.uint8, device=dev)
        o = torch.empty_like(t["q"])
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(t["q"]), torch.empty_like(t["k"]), torch.empty_like(t["v"])
        for (label, causal, dens) in wl["variants"]:
            mask = None if dens is None else make_tile_mask(-(-N // 128), seed=0, density=dens).to(dev)
            kept = 1.0 if mask is None else float(mask.float().mean())
            F = fwd_flops(B, H, N, d, causal, kept, Nk)

            pdrop = wl.get("dropout_p", 0.0)

            def fwd():
                if pdrop:
                    fa.forward_dropout(t["q"], t["k"], t["v"], pdrop, 1234, 0, causal=causal, scale=sc, out=o,
                                       lse=lse)
                elif mask is None:
                    fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc, out=o, lse=lse)
                else:
                    fa.forward_blocksparse(t["q"], t["k"], t["v"], mask, scale=sc, out=o, lse=lse)

            def pre():
                fa.bwd_preprocess(o, t["do"], lse, ws)

            def dkdv():
                fa.bwd_dkdv(t["q"], t["k"], t["v"], t["do"], dk, dv, ws, causal=causal, scale=sc, tile_mask=mask)

            def dqk():
                fa.bwd_dq(t["q"], t["k"], t["v"], t["do"], dq, ws, causal=causal, scale=sc, tile_mask=mask)

            def timed(fns):
                ms = []
                for r in range(args.warmup + args.steps):
                    flush.zero_()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    for f in fns:
                        f()
                    e1.record(stream)
                    torch.cuda.synchronize(dev)
                    if r >= args.warmup:
                        ms.append(e0.elapsed_time(e1))
                return statistics.median(ms)

            clocks = ClockSampler(0)
            clocks.start()
            time.sleep(0.3)  # let the sampler take its first reading
            t_f = timed([fwd])
            row = {"workload": name, "variant": label, "B": B, "H": H, "N": N, "d": d, "kept": round(kept, 4),
                   "fwd_ms": round(t_f, 4), "fwd_tflops": round(F / t_f / 1e9, 1),
                   "fwd_pct_peak": round(100 * F / t_f / 1e9 / pk["bf16_tflops"], 1)}
            if name != "pr1" and not pdrop:
                # the fused backward (one kernel; dQ reduced in fp32), whole and its main kernel
                def fbwd():
                    if mask is None:
                        fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal=causal, scale=sc, workspace=ws_f,
                                    grads=(dq, dk, dv), deterministic=False)
                    else:
                        fa.backward_blocksparse(t["q"], t["k"], t["v"], o, lse, t["do"], mask, scale=sc,
                                                workspace=ws_f, grads=(dq, dk, dv), deterministic=False)
                t_fb = timed([fbwd])
                row.update({"fused_bwd_ms": round(t_fb, 4), "fused_bwd_tflops": round(2.5 * F / t_fb / 1e9, 1),
                            "fused_bwd_pct_peak": round(100 * 2.5 * F / t_fb / 1e9 / pk["bf16_tflops"], 1),
                            "fused_fwd_bwd_tflops": round(3.5 * F / (t_f + t_fb) / 1e9, 1)})
                if Nk == N:
                    fa.bwd_fused_preprocess(o, t["do"], lse, ws_f)
                    t_fm = timed([lambda: fa.bwd_fused_main(t["q"], t["k"], t["v"], t["do"], dk, dv, ws_f,
                                                            causal=causal, scale=sc, tile_mask=mask)])
                    row.update({"fused_main_ms": round(t_fm, 4), "fused_main_tflops": round(2.5 * F / t_fm / 1e9, 1)})
            if not det_ok:
                pass
            elif Nk != N or pdrop:
                # The staged calls are for Nq = Nk without dropout; time the whole backward.
                def bwd_all():
                    if pdrop:
                        fa.backward_dropout(t["q"], t["k"], t["v"], o, lse, t["do"], pdrop, 1234, 0, causal=causal,
                                            scale=sc, workspace=ws, grads=(dq, dk, dv))
                    else:
                        fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal=causal, scale=sc,
                                    workspace=ws, grads=(dq, dk, dv))
                t_b = timed([bwd_all])
                row.update({"Nk": Nk, "dropout_p": pdrop, "bwd_ms": round(t_b, 4),
                            "bwd_tflops": round(2.5 * F / t_b / 1e9, 1),
                            "bwd_pct_peak": round(100 * 2.5 * F / t_b / 1e9 / pk["bf16_tflops"], 1),
                            "fwd_bwd_tflops": round(3.5 * F / (t_f + t_b) / 1e9, 1)})
            elif name != "pr1":
                pre()
                t_kv = timed([dkdv])
                t_q = timed([dqk])
                t_b = timed([pre, dkdv, dqk])
                row.update({"bwd_ms": round(t_b, 4), "bwd_dkdv_ms": round(t_kv, 4), "bwd_dq_ms": round(t_q, 4),
                            "bwd_tflops": round(2.5 * F / t_b / 1e9, 1),
                            "dkdv_tflops": round(2.0 * F / t_kv / 1e9, 1),
                            "dq_exec_tflops": round(1.5 * F / t_q / 1e9, 1),
                            "bwd_pct_peak": round(100 * 2.5 * F / t_b / 1e9 / pk["bf16_tflops"], 1),
                            "fwd_bwd_tflops": round(3.5 * F / (t_f + t_b) / 1e9, 1)})
            row["clocks"] = clocks.stop()
            row["fwd_pct_spec_peak"] = round(100 * F / t_f / 1e9 / SPEC_BF16_TFLOPS, 1)
            if "bwd_ms" in row:
                row["bwd_pct_spec_peak"] = round(100 * 2.5 * F / row["bwd_ms"] / 1e9 / SPEC_BF16_TFLOPS, 1)
            if "fused_bwd_ms" in row:
                row["fused_bwd_pct_spec_peak"] = round(100 * 2.5 * F / row["fused_bwd_ms"] / 1e9 / SPEC_BF16_TFLOPS, 1)
            st, site = fa.device_status(dev)
            row["status"] = st
            row["peak"] = f'{pk["bf16_tflops"]} ({pk_kind}, burst)'
            print(json.dumps(row), flush=True)
        del t, ws, ws_f, o, lse, dq, dk, dv
        torch.cuda.empty_cache()
    return 0


def build_parser():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="b2h16n8192d128_causal")
    ap.add_argument("--backward", choices=("fused", "deterministic"), default="fused",
                    help="fused: one kernel for dK, dV, dQ (dQ reduced in fp32); deterministic: two kernels")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--table", action="store_true", help="per-workload fwd/bwd times (JSON lines), not the contract line")
    ap.add_argument("--only", default="", help="with --table: comma-separated substrings of workload names")
    return ap


def main():
    args = build_parser().parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.table:
        return run_table(args)
    wl = workload(args.workload)
    if wl["dropout_p"]:
        raise SystemExit("dropout workloads are measured by --table only")
    if args.impl == "reference":
        return run_reference(args, args.workload, wl)
    return run_ours(args, args.workload, wl)


if __name__ == "__main__":
    sys.exit(main())
