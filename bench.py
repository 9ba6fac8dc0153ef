"""Benchmark of CLEAR attention on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 8k_r8] [--impl clear|reference]

A step is one forward call (clear_attn_fwd: scheduler enumeration, image-row and text-row kernels,
split combine) on the workload the metric is quoted on: B=1, 24 heads, d=128, 512 text tokens,
512 x 512 image grid (8192^2 pixels), r=8, bf16 inputs. The backward (dQ/dK/dV) is measured in the
same run on the distillation shape and reported under "bwd".

value = useful (kept-pair) TFLOP/s over all ranks; each rank runs its own independent call (weak
scaling, no collective on the data path). Inputs (4.8 GB) are far larger than L2.
With --impl reference the float64 CPU oracle is timed instead, on sampled rows extrapolated to a
full call.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from clear_inputs import WORKLOADS, Workload, make_inputs, quantize_e4m3  # noqa: E402

METRIC = "CLEAR attn useful TFLOP/s & ms/call (bf16, 512² grid, r=8); % of TC peak"
FALLBACK_BF16_TFLOPS = 1590.0


# DRAM traffic of clear_fwd_kernel<128> from one ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum) on the 8K r=8 shape cut to 2 heads (the full 24-head launch is too large
# to capture), per head; heads are independent, so a full launch moves heads x this. Valid only
# for the kernel sources it was taken on (hash below); any change to them reports null.
FWD_TRAFFIC = {"8k_r8": {"bytes_per_head": (729.469184e6 + 136.059136e6) / 2, "src": "08feca85a1acbfa9"}}
FWD_SOURCES = ("clear_fwd.cuh", "clear_sched.cuh", "clear_common.cuh", "sm100_ptx.cuh")


def _fwd_src_hash():
    h = hashlib.sha256()
    for f in FWD_SOURCES:
        with open(os.path.join(ROOT, "local_circular_window_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _fwd_traffic(wl):
    rec = FWD_TRAFFIC.get(wl.name)
    if rec is None or wl.heads != WORKLOADS[wl.name].heads or _fwd_src_hash() != rec["src"]:
        return None
    return rec["bytes_per_head"] * wl.B * wl.heads


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), \
            float(d.get("hbm_gbs", 0.0)), "measured"
    return FALLBACK_BF16_TFLOPS, 1400.0, 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def _max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job(total_ms_local: float, steps: int, useful_flops_per_call: float, world: int, device: str = "cuda"):
    """Per-step time as the slowest rank's, and whole-job throughput: every rank runs its own
    independent call per step, so the job does world x useful FLOPs per step."""
    total_ms = _max_over_ranks(total_ms_local, world, device)
    ms = total_ms / steps
    return ms, useful_flops_per_call * world / (ms * 1e-3) / 1e12


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _flops(L, wl: Workload):
    p = L.make_params(wl.B, wl.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r)
    useful, executed = L.pair_counts(p)
    return 4.0 * wl.d * useful, 4.0 * wl.d * executed


# ------------------------------------------------------------------------------------------------
# CPU oracle timing (bounded sample, extrapolated to one call)
# ------------------------------------------------------------------------------------------------
_ORACLE_INPUTS = {}


def oracle_call_seconds(wl: Workload, budget_s: float, seed: int = 0):
    """Time the float64 oracle on sampled text and image query rows of one head and extrapolate to
    a full call (B * heads heads, n_text text rows + H*W image rows each)."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    if wl.name not in _ORACLE_INPUTS:  # one head's inputs, drawn once (not timed)
        _ORACLE_INPUTS[wl.name] = make_inputs(Workload(wl.name, 1, 1, wl.n_text, wl.H, wl.W, wl.d, wl.r), seed=0)
    q, k, v = _ORACLE_INPUTS[wl.name]
    rng = np.random.default_rng(seed)
    per_kind = {}
    for kind in ("text", "image"):
        if kind == "text" and wl.n_text == 0:
            per_kind[kind] = (0.0, 0)
            continue
        n_rows, spent = 0, 0.0
        while spent < budget_s / 2 and n_rows < 4096:
            if kind == "text":
                rows = sorted(rng.choice(wl.n_text, size=min(4, wl.n_text), replace=False).tolist())
            else:
                rows = sorted((wl.n_text + rng.choice(wl.H * wl.W, size=8, replace=False)).tolist())
            t0 = time.perf_counter()
            oracle.clear_attention_rows(q, k, v, wl.n_text, wl.H, wl.W, wl.r, 0, 0, rows)
            spent += time.perf_counter() - t0
            n_rows += len(rows)
        per_kind[kind] = (spent / max(1, n_rows), n_rows)
    per_head = per_kind["text"][0] * wl.n_text + per_kind["image"][0] * wl.H * wl.W
    total = per_head * wl.B * wl.heads
    sample = (f"oracle rows of head 0: {per_kind['text'][1]} text + {per_kind['image'][1]} image rows "
              f"({sum(v[0] * v[1] for v in per_kind.values()):.1f} s), extrapolated per row to "
              f"{wl.B * wl.heads} heads x ({wl.n_text} text + {wl.H * wl.W} image) rows")
    return total, cores, sample


# ------------------------------------------------------------------------------------------------
def run_reference(args):
    world, rank, _ = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0
    if rank != 0:
        return
    wl = WORKLOADS[args.config]
    import oracle
    useful = 4.0 * wl.d * wl.B * wl.heads * oracle.kept_pairs(wl.n_text, wl.H, wl.W, wl.r)
    per_step_budget = max(0.5, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    times = []
    for i in range(args.warmup + args.steps):
        t, cores, sample = oracle_call_seconds(wl, per_step_budget, seed=i)
        if i >= args.warmup:
            times.append(t)
    sec = statistics.mean(times)
    value = useful / sec / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, **{k: getattr(wl, k) for k in ("B", "heads", "n_text", "H", "W", "d", "r")}},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample + f"; {args.steps} timed samples"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _time_calls(fn, steps, stream):
    """CUDA-event time of each call on `stream`; returns per-call ms list and total ms."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    evs[0].record(stream)
    for i in range(steps):
        fn()
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)]
    return per, evs[0].elapsed_time(evs[-1])


# Forward configurations reported beside the headline one (FLUX-shaped calls at 1024^2, 2048^2 and
# 8192^2 pixels, every radius the workload list names).
FORWARD_CONFIGS = ("flux1024_r8", "flux1024_r16", "flux1024_r32", "flux2048_r16", "8k_r8", "8k_r32")
L2_BYTES = 126 << 20


def time_forward_config(L, wl: Workload, peak: float, stream, seed: int, calls: int = 0):
    """Median CUDA-event time of clear_attn_fwd on one configuration, with useful and padded
    (tile-executed) TFLOP/s and the fraction of the bf16 peak."""
    useful, executed = _flops(L, wl)
    q, k, v = make_inputs(wl, seed=seed, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((wl.B, wl.heads, wl.T), dtype=torch.float32, device="cuda")
    p = L.make_params(wl.B, wl.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r)
    ws = torch.empty(max(16, L.fwd_workspace_size(p)), dtype=torch.uint8, device="cuda")
    small = 3 * q_bytes(wl) < 2 * L2_BYTES
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if small else None
    calls = calls or (10 if wl.H >= 512 else 20)

    def call():
        L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r, o=o, lse=lse, workspace=ws, stream=stream)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    per = []
    for _ in range(calls):
        if flush is not None:
            flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call()
        b.record(stream)
        torch.cuda.synchronize()
        per.append(a.elapsed_time(b))
    if L.clear_attn_check() != 0:
        raise RuntimeError(f"device error timing {wl.name}")
    ms = statistics.median(per)
    del q, k, v, o, lse, ws, flush
    return {"ms_per_call": ms, "useful_tflops": useful / (ms * 1e-3) / 1e12,
            "padded_tflops": executed / (ms * 1e-3) / 1e12, "frac_of_peak": useful / (ms * 1e-3) / 1e12 / peak,
            "useful_gflop_per_call": useful / 1e9, "executed_gflop_per_call": executed / 1e9, "calls": calls,
            "l2": "flushed between calls" if small else "inputs larger than L2"}


def _median_call_ms(fn, stream, calls=10, flush=None):
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    per = []
    for _ in range(calls):
        if flush is not None:
            flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        per.append(a.elapsed_time(b))
    return statistics.median(per)


def time_mixed_batch(L, peak, stream, seed):
    """One clear_attn_fwd_varlen launch over FLUX-shaped items of three resolutions (32^2, 64^2 and
    128^2 token grids, 512 text tokens each, r=16), against the same items as separate calls."""
    items = [(512, 64, 64), (512, 64, 64), (512, 128, 128), (512, 32, 32)]
    heads, d, r = 24, 128, 16
    total, starts = L.varlen_tokens(items)
    gen = torch.Generator(device="cpu").manual_seed(seed)
    q, k, v = (torch.randn((heads, total, d), generator=gen).to(torch.bfloat16).cuda() for _ in range(3))
    ws = torch.empty(L.varlen_workspace_size(heads, d, r, items), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((heads, total), dtype=torch.float32, device="cuda")
    useful = sum(L.pair_counts(L.make_params(1, heads, nt, H, W, d, r))[0] * 4 * d for nt, H, W in items)
    per_item = [tuple(t[:, s:s + nt + H * W].unsqueeze(0).contiguous() for t in (q, k, v))
                for (nt, H, W), s in zip(items, starts)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def batch():
        L.clear_attn_fwd_varlen(q, k, v, items, r, o=o, lse=lse, workspace=ws, stream=stream)

    def separate():
        for (nt, H, W), (qi, ki, vi) in zip(items, per_item):
            L.clear_attn_fwd(qi, ki, vi, nt, H, W, r, stream=stream)

    ms_b = _median_call_ms(batch, stream, flush=flush)
    ms_s = _median_call_ms(separate, stream, flush=flush)
    if L.clear_attn_check() != 0:
        raise RuntimeError("device error timing the mixed batch")
    return {"items": [list(t) for t in items], "heads": heads, "r": r, "ms_per_call": ms_b,
            "useful_tflops": useful / (ms_b * 1e-3) / 1e12, "frac_of_peak": useful / (ms_b * 1e-3) / 1e12 / peak,
            "separate_calls_ms": ms_s, "l2": "flushed between calls"}


def time_fp8_forward(L, peak, stream, seed):
    """The forward with E4M3 score products (clear_attn_fwd_fp8) on the headline workload and on
    8K r=32, against the bf16 forward on the same inputs (same calls, CUDA events)."""
    out = {}
    for name in ("8k_r8", "8k_r32"):
        wl = WORKLOADS[name]
        q, k, v = make_inputs(wl, seed=seed, device="cuda")
        q8, sq = quantize_e4m3(q)
        k8, sk = quantize_e4m3(k)
        desc = (sq * sk).float().contiguous()
        del q, k
        o = torch.empty_like(v)
        lse = torch.empty((wl.B, wl.heads, wl.T), dtype=torch.float32, device="cuda")
        p = L.make_params(wl.B, wl.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r)
        ws = torch.empty(max(16, L.fwd_workspace_size(p)), dtype=torch.uint8, device="cuda")
        ms = _median_call_ms(lambda: L.clear_attn_fwd_fp8(q8, k8, v, desc, wl.n_text, wl.H, wl.W, wl.r, o=o, lse=lse,
                                                          workspace=ws, stream=stream), stream)
        useful, _ = _flops(L, wl)
        out[name] = {"ms_per_call": ms, "useful_tflops": useful / (ms * 1e-3) / 1e12,
                     "frac_of_bf16_peak": useful / (ms * 1e-3) / 1e12 / peak}
        del q8, k8, v, o, lse, ws
        torch.cuda.empty_cache()
    if L.clear_attn_check() != 0:
        raise RuntimeError("device error timing the FP8 forward")
    out["inputs"] = "q, k E4M3 codes with one scale per (batch, head); v bf16; inputs larger than L2"
    return out


def time_rope_forward(L, peak, hbm, stream, seed):
    """The forward on rotary-embedded q and k (clear_attn_fwd_rope, NTK factor 10) on the headline
    workload and on F2048 r=16, the plain forward on the same inputs, and the rotation pass alone
    (clear_attn_rope, CUDA events around the call): it is HBM-bound, reading q and k and writing
    their rotated copies once, 4 * B*heads*T*d bf16 bytes."""
    out = {}
    for name in ("8k_r8", "flux2048_r16"):
        wl = WORKLOADS[name]
        q, k, v = make_inputs(wl, seed=seed, device="cuda")
        o = torch.empty_like(v)
        lse = torch.empty((wl.B, wl.heads, wl.T), dtype=torch.float32, device="cuda")
        p = L.make_params(wl.B, wl.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r)
        ws = torch.empty(L.rope_workspace_size(p), dtype=torch.uint8, device="cuda")
        qr, kr = torch.empty_like(q), torch.empty_like(k)
        rws = torch.empty(L.rope_rotate_workspace_size(p), dtype=torch.uint8, device="cuda")
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if q_bytes(wl) < (128 << 20) else None
        ms_rope = _median_call_ms(lambda: L.clear_attn_fwd_rope(q, k, v, wl.n_text, wl.H, wl.W, wl.r, ntk=10.0, o=o,
                                                                lse=lse, workspace=ws, stream=stream),
                                  stream, flush=flush)
        ms_plain = _median_call_ms(lambda: L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r, o=o, lse=lse,
                                                            workspace=ws, stream=stream), stream, flush=flush)
        rot_ms = _median_call_ms(lambda: L.clear_attn_rope(q, k, wl.n_text, wl.H, wl.W, ntk=10.0, q_out=qr, k_out=kr,
                                                           workspace=rws, stream=stream), stream, calls=20, flush=flush)
        useful, _ = _flops(L, wl)
        rot_bytes = 4 * q_bytes(wl)
        out[name] = {"ms_per_call": ms_rope, "plain_forward_ms": ms_plain, "rotation_ms": rot_ms,
                     "rotation_gbs": rot_bytes / (rot_ms * 1e-3) / 1e9,
                     "rotation_frac_of_hbm": rot_bytes / (rot_ms * 1e-3) / 1e9 / hbm if hbm else None,
                     "rotation_bytes": rot_bytes,
                     "useful_tflops": useful / (ms_rope * 1e-3) / 1e12,
                     "frac_of_peak": useful / (ms_rope * 1e-3) / 1e12 / peak}
        del q, k, v, o, lse, ws, qr, kr, rws, flush
        torch.cuda.empty_cache()
    if L.clear_attn_check() != 0:
        raise RuntimeError("device error timing the RoPE forward")
    out["l2"] = "flushed between calls below 128 MB of q, else inputs larger than L2"
    return out


def time_patch_parallel(L, stream, seed):
    """Patch-parallel split of the FLUX 2048^2 call (128 x 128 grid, r=16) into 2 and 4 row stripes,
    every stripe's kernels run in turn on this one GPU (the halo exchange and text-row all-gather
    between GPUs are not timed: one GPU), with the text-row difference between the exact merge and
    the paper's Eq. 7 patch average."""
    from local_circular_window_b200 import patch_parallel as pp
    wl = WORKLOADS["flux2048_r16"]
    q, k, v = make_inputs(wl, seed=seed, device="cuda")
    ref_o, _ = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r)
    out = {"workload": wl.name, "single_call_ms": _median_call_ms(
        lambda: L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r, stream=stream), stream)}
    for stripes in (2, 4):
        res = {}
        for mode in ("exact", "eq7"):
            o, _ = pp.forward_by_stripes(q, k, v, wl.n_text, wl.H, wl.W, wl.r, stripes, mode=mode)
            res[mode] = o
            out[f"{stripes}_stripes_{mode}_ms"] = _median_call_ms(
                lambda: pp.forward_by_stripes(q, k, v, wl.n_text, wl.H, wl.W, wl.r, stripes, mode=mode), stream)
        nt = wl.n_text
        out[f"{stripes}_stripes_exact_vs_single_max_abs"] = float((res["exact"].float() - ref_o.float()).abs().max())
        out[f"{stripes}_stripes_eq7_vs_exact_text_max_abs"] = float(
            (res["eq7"][:, :, :nt].float() - res["exact"][:, :, :nt].float()).abs().max())
        out[f"{stripes}_stripes_eq7_vs_exact_text_mean_abs"] = float(
            (res["eq7"][:, :, :nt].float() - res["exact"][:, :, :nt].float()).abs().mean())
    if L.clear_attn_check() != 0:
        raise RuntimeError("device error timing the patch-parallel split")
    return out


def run_clear(args):
    world, rank, local = _dist()
    torch.cuda.set_device(local)
    import local_circular_window_b200 as L
    wl = WORKLOADS[args.config]
    if args.heads:  # sized-down copy of the same shape (profiling captures only)
        wl = Workload(f"{wl.name}_h{args.heads}", wl.B, args.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r)
    peak, peak_sus, hbm, peak_kind = _peaks()
    useful, executed = _flops(L, wl)
    stream = torch.cuda.current_stream()

    q, k, v = make_inputs(wl, seed=1000 + rank, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((wl.B, wl.heads, wl.T), dtype=torch.float32, device="cuda")
    p = L.make_params(wl.B, wl.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r)
    ws = torch.empty(max(16, L.fwd_workspace_size(p)), dtype=torch.uint8, device="cuda")

    def call():
        L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r, o=o, lse=lse, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        call()
    if L.clear_attn_check() != 0:
        raise RuntimeError("device error during warm-up")
    torch.cuda.synchronize()
    _barrier(world)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        _barrier(world)
        per, total_ms = _time_calls(call, args.steps, stream)
        _barrier(world)
    if L.clear_attn_check() != 0:
        raise RuntimeError("device error during timing")
    ms, value = whole_job(total_ms, args.steps, useful, world)
    kernel_ms = statistics.mean(per)
    achieved = useful / (kernel_ms * 1e-3) / 1e12

    # End to end through the C ABI with host buffers: clear_attn_fwd_host copies the pinned inputs
    # to the device, runs the forward and copies o and lse back, overlapping the copies of one
    # slice group with the forward of its neighbours.
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        p_host = L.make_params(wl.B, wl.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r)
        hws = torch.empty(L.fwd_host_workspace_size(p_host), dtype=torch.uint8, device="cuda")

        def e2e_call():
            L.clear_attn_fwd_host(hq, hk, hv, wl.n_text, wl.H, wl.W, wl.r, o=ho, lse=hl, workspace=hws,
                                  stream=stream)

        e2e_call()
        torch.cuda.synchronize()
        k_e2e = max(1, min(args.steps, 5))
        _barrier(world)
        _, e2e_ms = _time_calls(e2e_call, k_e2e, stream)
        e2e_ms = _max_over_ranks(e2e_ms, world) / k_e2e
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
        d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
        e2e = {"value": useful * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "steps": k_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "call": "clear_attn_fwd_host (pinned host buffers; copies overlapped with the forward)"}
        del hq, hk, hv, ho, hl, hws
    del q, k, v, o, lse, ws
    torch.cuda.empty_cache()

    # Backward rows of the hot path, on the distillation shape.
    bwd = None
    if not args.no_bwd:
        bwl = WORKLOADS["bwd_flux1024_r32"]
        bq, bk, bv, bdo = make_inputs(bwl, seed=2000 + rank, device="cuda", with_grad_out=True)
        bo, blse = L.clear_attn_fwd(bq, bk, bv, bwl.n_text, bwl.H, bwl.W, bwl.r)
        bp = L.make_params(bwl.B, bwl.heads, bwl.n_text, bwl.H, bwl.W, bwl.d, bwl.r)
        bws = torch.empty(L.bwd_workspace_size(bp), dtype=torch.uint8, device="cuda")
        gq, gk, gv = torch.empty_like(bq), torch.empty_like(bk), torch.empty_like(bv)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

        def bcall():
            flush.zero_()  # the 280 MB working set is near L2 size: flush L2 between calls
            L.clear_attn_bwd(bq, bk, bv, bo, blse, bdo, bwl.n_text, bwl.H, bwl.W, bwl.r, dq=gq, dk=gk, dv=gv,
                             workspace=bws, stream=stream)

        def flush_only():
            flush.zero_()

        for _ in range(3):
            bcall()
        torch.cuda.synchronize()
        nb = max(3, min(args.steps, 20))
        per_b, _ = _time_calls(bcall, nb, stream)
        per_f, _ = _time_calls(flush_only, nb, stream)
        bms = max(1e-6, statistics.median(per_b) - statistics.median(per_f))
        bu, be = _flops(L, bwl)
        if L.clear_attn_check() != 0:
            raise RuntimeError("device error in backward timing")
        bwd = {"workload": bwl.name, "ms_per_call": bms, "useful_tflops": 2.5 * bu / (bms * 1e-3) / 1e12,
               "flop_convention": "backward = 2.5 x forward useful FLOPs (5 vs 2 matmuls)",
               "l2": "flushed between calls (256 MiB write, its time subtracted)"}
        del bq, bk, bv, bdo, bo, blse, bws, gq, gk, gv, flush

    # Every other forward configuration of the workload list, timed the same way (CUDA events on the
    # launching stream; L2 flushed between calls when the inputs fit in L2).
    configs = None
    if not args.no_configs:
        configs = {}
        with ClockSampler(local) as cfg_clk:
            for name in FORWARD_CONFIGS:
                if name == wl.name:
                    continue
                configs[name] = time_forward_config(L, WORKLOADS[name], peak, stream, seed=3000 + rank)
        configs["clocks"] = cfg_clk.summary()
        torch.cuda.empty_cache()

    # The NEXT rows built on the same kernels: a mixed-resolution batch in one launch, and the
    # patch-parallel split (each stripe's work on this GPU in turn).
    extras = None
    if not args.no_configs and rank == 0:
        extras = {"mixed_batch": time_mixed_batch(L, peak, stream, seed=4000),
                  "patch_parallel": time_patch_parallel(L, stream, seed=4001),
                  "fp8_scores": time_fp8_forward(L, peak, stream, seed=4002),
                  "rope": time_rope_forward(L, peak, hbm, stream, seed=4003)}
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec, cores, sample = oracle_call_seconds(wl, args.cpu_budget)
        cpu = {"value": useful / sec / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": sample}

    clocks = clk.summary()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "heads": wl.heads, "n_text": wl.n_text, "H": wl.H,
                       "W": wl.W, "d": wl.d, "r": wl.r, "T": wl.T,
                       "l2": "inputs (3 x %.2f GB) larger than L2" % (q_bytes(wl) / 1e9),
                       "parallelism": f"independent call per GPU x{world}"},
            "pct_of_tc_peak": 100.0 * achieved / peak,
            "padded_tflops": executed / (kernel_ms * 1e-3) / 1e12,
            "useful_gflop_per_call": useful / 1e9, "executed_gflop_per_call": executed / 1e9,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": _fwd_traffic(wl),
                         "peak_source": f"{peak_kind} bf16 dense (burst; kernel timed alone)",
                         "kernel": "clear_fwd_kernel + clear_fwd_combine_kernel (one call, CUDA events)"},
            "e2e": e2e, "cpu_baseline": cpu, "bwd": bwd, "configs": configs, "extras": extras, "clocks": clocks,
            "gpu_launches": 2 * args.steps,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def q_bytes(wl):
    return wl.B * wl.heads * wl.T * wl.d * 2


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="clear", choices=["clear", "reference"])
    ap.add_argument("--config", default="8k_r8", choices=sorted(WORKLOADS))
    ap.add_argument("--heads", type=int, default=0, help="override the head count (sized-down profiling runs)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-bwd", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the other forward configurations")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle CPU work for cpu_baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_clear(args)


if __name__ == "__main__":
    main()
