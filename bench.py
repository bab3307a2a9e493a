#!/usr/bin/env python3
"""Benchmark of the smoothed-K INT8 attention forward (prefill) on B200.

One step = one pass of the whole path over one batch of synthetic input already resident in HBM:
K channel sums, smoothing + INT8 quantization of Q and K (the pre-processing kernels), then the
tcgen05 attention kernel, all through the C ABI (qattn_smooth_quant then qattn_attn_quantized,
the two halves of qattn_forward_ws, timed separately with CUDA events on the launching stream).

Metric: TOPS = 4*B*H*N^2*d / t, halved for causal; also reported as a fraction of the B200 INT8
tensor peak, measured in the same run with an int8 cuBLAS GEMM (torch._int_mm, 8192^3), beside the
datasheet's 4.5 POPS.  The long-context workload (long128k) is timed after the main one and
reported in the same line under "workloads".

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
Multi-GPU (weak scaling, one full workload per rank, no data-path collective):
  python -m torch.distributed.run --nproc-per-node N --master-addr 127.0.0.1 ... bench.py --gpus N
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized attention fwd TOPS (4·B·H·N²·d/s) and % of B200 INT8 tensor peak"
DEFAULT_WORKLOAD = "llama8b_32k"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATTN_KERNEL_SOURCES = ["attn_sm100.cuh", "sm100_ptx.cuh"]  # the timed kernel (int8 Q) uses no other source
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "attn_fwd_sm100_llama8b_32k.md")


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--e2e-steps", type=int, default=5)
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="target CPU time of the oracle baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--adaptive", type=float, default=None, metavar="TAU",
                   help="adaptive-quantization mode: calibrate on another seed of the workload, "
                        "each (batch, kv head) group takes FP8 P V when its output's cosine to "
                        "the FP16 P V output is >= TAU; one step = qattn_forward_adaptive")
    p.add_argument("--extra-workloads", default="long128k",
                   help="comma-separated workloads timed after the main one and reported under "
                        "'workloads' in the same JSON line (empty: none)")
    p.add_argument("--extra-steps", type=int, default=10)
    p.add_argument("--no-gemm-peaks", dest="gemm_peaks", action="store_false",
                   help="skip the int8/fp16 GEMM peak measurement (roofline then uses "
                        "MEASURED_PEAKS.json's bf16 figure and the nominal INT8 ratio)")
    p.add_argument("--sparse-topk", type=int, default=-1,
                   help="block-sparse mode: key tiles per 256-row query block chosen by the "
                        "block-mean score (top-k plus the causal diagonals); -1 = dense")
    p.add_argument("--fp4-topk", type=int, default=None,
                   help="FP4-path mode (NVFP4 operands, two-level FP4 P): the key tiles chosen "
                        "per 256-row query block (top-k plus the causal diagonals) run in FP16; "
                        "-1 = every tile in FP4; omitted = the INT8 path")
    return p.parse_args(argv)


# ------------------------------------------------------------------------------------------------
# peaks, clocks, profile summary
# ------------------------------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha():
    h = hashlib.sha256()
    for name in ATTN_KERNEL_SOURCES:
        with open(os.path.join(ROOT, "bit_quantized_attention_smoothing_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload):
    """DRAM bytes per attention launch from the committed ncu summary, if it was taken on the
    current kernel source and this workload; else None."""
    try:
        text = open(PROFILE_SUMMARY).read()
    except OSError:
        return None
    m_sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_w = re.search(r"workload:\s*(\S+)", text)
    if not (m_sha and m_b and m_w):
        return None
    if m_sha.group(1) != kernel_source_sha() or m_w.group(1) != workload:
        return None
    return float(m_b.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
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
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                mx = max(mx, float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[3:]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# CPU oracle baseline (the oracle as it stands, on a bounded sample of the workload)
# ------------------------------------------------------------------------------------------------

def oracle_sample_run(w, q, k, v, target_s):
    """Times the oracle's whole path on a sample of the workload: smoothing + quantization of
    the kv head 0 and its query heads (full N), then attention for query rows spread over the
    sequence, the count chosen so the run takes about target_s.  Returns a dict."""
    import numpy as np
    from oracle import oracle as O
    O.build()
    G = w.H // w.Hkv
    qs = q[0:1, 0:G].contiguous().cpu().numpy().view(np.uint16)
    ks = k[0:1, 0:1].contiguous().cpu().numpy().view(np.uint16)
    vs = v[0:1, 0:1].contiguous().cpu().numpy().view(np.uint16)
    threads = os.cpu_count() or 1

    def rows_for(nrows):
        i = np.linspace(0, w.N - 1, nrows).astype(np.int64)
        bh = np.arange(nrows, dtype=np.int64) % G
        return bh, i

    def pairs(i):
        return float(np.sum(i + 1)) if w.causal else float(len(i)) * w.N

    t0 = time.perf_counter()
    sq = O.smooth_quant(qs, ks, 1, G, 1, w.N, w.d)
    t_quant = time.perf_counter() - t0
    nrows = 16
    while True:
        bh, i = rows_for(nrows)
        t1 = time.perf_counter()
        O.attention_quantized(sq["q_i8"], sq["q_scale"], sq["k_i8"], sq["k_scale"], vs, 1, G, 1,
                              w.N, w.d, w.causal, rows=(bh, i), nthreads=threads)
        dt = time.perf_counter() - t1
        if dt >= 0.4 * max(target_s - t_quant, 0.5) or nrows >= w.N * G:
            break
        grow = 0.8 * max(target_s - t_quant, 0.5) / max(dt, 1e-3)
        nrows = int(min(w.N * G, nrows * min(64.0, max(2.0, grow))))
    # final timed sample: quantization + attention rows
    t0 = time.perf_counter()
    sq = O.smooth_quant(qs, ks, 1, G, 1, w.N, w.d)
    O.attention_quantized(sq["q_i8"], sq["q_scale"], sq["k_i8"], sq["k_scale"], vs, 1, G, 1, w.N,
                          w.d, w.causal, rows=(bh, i), nthreads=threads)
    dt = time.perf_counter() - t0
    ops = 4.0 * w.d * pairs(i)
    return {"value": ops / dt / 1e12, "unit": "TOPS", "cores": threads, "kind": "oracle",
            "seconds": round(dt, 3),
            "sample": (f"kv head 0 of batch 0 with its {G} query heads: smoothing + quantization "
                       f"over all N={w.N} tokens, then {len(i)} query rows spread evenly over the "
                       f"sequence ({pairs(i):.3g} visible pairs, 4*d ops each)")}


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------

def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest of every rank's value (host plumbing: one all-reduce of a scalar over the
    process group the caller initialised; no data-path collective).  A single rank returns its
    own value."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_tops(ops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank processes one full workload per step, so the job does
    world * ops * steps operations in the slowest rank's time."""
    return world * ops_per_step * steps / (max_ms / 1e3) / 1e12


def measure_gemm_peaks(device, seconds=2.0):
    """Tensor-core GEMM peaks on this GPU through torch (cuBLAS): int8 x int8 -> int32
    (torch._int_mm) and fp16 x fp16 -> fp16, both 8192^3 (2 * 8192^3 operations), as a burst (best
    of 10 single calls, CUDA events) and sustained (back-to-back calls for `seconds`).  Returns a
    dict in TOPS; a GEMM that torch cannot run on this device is left out."""
    import torch
    n = 8192
    ops = 2.0 * n ** 3
    out = {}
    gen = torch.Generator(device=device).manual_seed(5)
    for name, make, fn in (
            # B column-major (a transposed view), so both operands are K-contiguous
            ("int8", lambda: torch.randint(-127, 128, (n, n), generator=gen, device=device, dtype=torch.int8),
             lambda a, b: torch._int_mm(a, b.t())),
            ("fp16", lambda: torch.randn(n, n, generator=gen, device=device, dtype=torch.float16),
             lambda a, b: a @ b)):
        try:
            a, b = make(), make()
            for _ in range(3):
                fn(a, b)
            torch.cuda.synchronize(device)
            best = float("inf")
            for _ in range(10):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn(a, b)
                e1.record()
                e1.synchronize()
                best = min(best, e0.elapsed_time(e1))
            reps = max(10, int(seconds * 1e3 / best))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                fn(a, b)
            e1.record()
            e1.synchronize()
            out[name] = {"burst": ops / (best / 1e3) / 1e12,
                         "sustained": ops * reps / (e0.elapsed_time(e1) / 1e3) / 1e12}
            del a, b
        except (RuntimeError, TypeError) as exc:   # no such GEMM for this device
            out[name + "_error"] = str(exc).splitlines()[0][:160]
    torch.cuda.empty_cache()
    return out


def tensor_peaks(measured):
    """(P8, P16, source text): the INT8 and FP16 dense peaks for the roofline (burst figures: the
    attention kernel is timed as its own launches and stays at the maximum SM clock)."""
    peaks, peak_src = load_peaks()
    tag = "of measured" if peak_src == "measured" else "of fallback"
    bf16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    if "fp16" in measured:
        p16, s16 = measured["fp16"]["burst"], "fp16 GEMM measured in this run (torch, cuBLAS, 8192^3)"
    else:
        p16, s16 = bf16, f"bf16 GEMM burst {bf16:.1f} TF/s ({tag}; fp16 has the same nominal rate)"
    if "int8" in measured:
        p8, s8 = measured["int8"]["burst"], "int8 GEMM measured in this run (torch._int_mm, cuBLAS, 8192^3)"
    else:
        p8, s8 = 2.0 * bf16, f"2 x bf16 GEMM burst ({tag}; nominal INT8:BF16 ratio 4.5:2.25)"
    return p8, p16, f"P8: {s8}; P16: {s16}"


def run_workload(Q, w, args, steps, warmup, e2e_steps, stream, world, barrier, clock_dev):
    """Times the dense (or block-sparse) INT8 path on workload w: `steps` steps on device-resident
    inputs (smoothing + quantization, then attention, CUDA events around each half), then
    `e2e_steps` calls of qattn_forward_host on pinned host buffers.  Returns a dict of
    measurements (the slowest rank's times)."""
    import torch
    q, k, v = make_inputs_cuda(w)
    B, H, Hkv, N, d = w.B, w.H, w.Hkv, w.N, w.d
    nqb, nkb = -(-N // 128), -(-N // 64)
    dev = q.device
    q_i8 = torch.empty(B, H, N, d, dtype=torch.int8, device=dev)
    k_i8 = torch.empty(B, Hkv, N, d, dtype=torch.int8, device=dev)
    q_s = torch.empty(B, H, nqb, dtype=torch.float32, device=dev)
    k_s = torch.empty(B, Hkv, nkb, dtype=torch.float32, device=dev)
    ws = torch.empty(Q.qattn_smooth_quant_workspace(B, Hkv, d), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    working_set = sum(t.numel() * t.element_size() for t in (q, k, v, q_i8, k_i8, out))

    sparse = args.sparse_topk >= 0
    density = 1.0
    if sparse:
        # block-sparse mode: the selection runs with the pre-processing, every step
        kl, kc = Q.qattn_block_select(q, k, args.sparse_topk, w.causal, stream=stream)
        sel_ws = torch.empty(max(Q.qattn_block_select_workspace(B, H, Hkv, N, d), 16),
                             dtype=torch.uint8, device=dev)
        cnt = kc.cpu().numpy().astype(np.int64)
        lst = kl.cpu().numpy()
        nqt = -(-N // 128)
        dense_pairs = computed_pairs = 0
        for bh in range(B * H):
            for i in range(cnt.shape[1]):
                for tile in (2 * i, 2 * i + 1):
                    if tile >= nqt:
                        continue
                    row_list = lst[bh, i, :cnt[bh, i]]
                    lim = tile if w.causal else nqt - 1
                    dense_pairs += lim + 1
                    computed_pairs += int((row_list <= lim).sum())
        density = computed_pairs / dense_pairs

    def step(ev_mid=None):
        Q.qattn_smooth_quant(q, k, q_i8, q_s, k_i8, k_s, None, ws, stream, want_mean=False)
        if sparse:
            Q.qattn_block_select(q, k, args.sparse_topk, w.causal, kl, kc, sel_ws, stream)
        if ev_mid is not None:
            ev_mid.record(stream)
        if sparse:
            Q.qattn_attn_quantized_sparse(q_i8, q_s, k_i8, k_s, v, kl, kc, out, w.causal, stream)
        else:
            Q.qattn_attn_quantized(q_i8, q_s, k_i8, k_s, v, out, w.causal, stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if Q.qattn_check_device_status(stream) != 0:
        raise RuntimeError("device status reports a timed-out wait during warm-up")

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(clock_dev) as clk:
        for i in range(steps):
            ev[i][0].record(stream)
            step(ev[i][1])
            ev[i][2].record(stream)
        torch.cuda.synchronize()
    barrier()
    total_ms = ev[0][0].elapsed_time(ev[-1][2])
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    quant_ms = [e[0].elapsed_time(e[1]) for e in ev]
    if Q.qattn_check_device_status(stream) != 0:
        raise RuntimeError("device status reports a timed-out wait in the timed region")
    total_ms_max = max_over_ranks(total_ms, world, dev)

    # end to end through the C ABI on host buffers (H2D of q, k, v and D2H of out inside)
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    Q.qattn_forward_host(qh, kh, vh, oh, w.causal, stream)  # warm-up (pool, tensor maps)
    ke = max(1, e2e_steps)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(ke):
        Q.qattn_forward_host(qh, kh, vh, oh, w.causal, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return {
        "q": q, "k": k, "v": v, "working_set": working_set, "sparse": sparse, "density": density,
        "total_ms_max": total_ms_max, "attn_ms": statistics.mean(attn_ms),
        "quant_ms": statistics.mean(quant_ms), "clocks": clk.summary(), "e2e_ms": e2e_ms,
        "e2e_steps": ke, "h2d": sum(t.numel() * t.element_size() for t in (qh, kh, vh)),
        "d2h": oh.numel() * oh.element_size(),
        "launches_per_step": 3 + (4 if sparse else 0),
    }


def make_inputs_cuda(w):
    from bit_quantized_attention_smoothing_b200.workloads import make_inputs
    return make_inputs(w, device="cuda")


def workload_line(w, r, steps, world, p8, p16, peak_src):
    """The measured numbers of one workload: value, roofline of the attention kernel, e2e."""
    ops = w.ops
    value = weak_scaling_tops(ops, steps, world, r["total_ms_max"])
    mixed_peak = 2.0 / (1.0 / p8 + 1.0 / p16)   # half the metric's ops INT8, half FP16
    # the roofline counts the work the kernel does: in block-sparse mode only the computed tiles
    achieved = ops * r["density"] / (r["attn_ms"] / 1e3) / 1e12
    return {
        "value": round(value, 2),
        "ms_per_step": round(r["total_ms_max"] / steps, 4),
        "steps": steps,
        "value_frac_of_int8_peak": round(value / p8, 4),
        "attn_ms": round(r["attn_ms"], 4),
        "quant_ms": round(r["quant_ms"], 4),
        "roofline": {
            "bound": "tensor",
            "kernel": "attn_fwd_kernel",
            "achieved": round(achieved, 2),
            "peak": round(mixed_peak, 1),
            "unit": "TFLOP/s",
            "frac": round(achieved / mixed_peak, 4),
            # the committed capture is of the dense launch; a block-sparse launch moves less
            "traffic": None if r["sparse"] else profiled_traffic(w.name),
            "peak_source": ("mixed INT8/FP16 ceiling 2/(1/P8+1/P16), since half the metric's "
                            "operations run at each rate; " + peak_src),
            "frac_of_int8_peak": round(achieved / p8, 4),
            "frac_of_int8_datasheet": round(achieved / 4500.0, 4),
        },
        "e2e": {"value": round(weak_scaling_tops(ops, r["e2e_steps"], world, r["e2e_ms"]), 2),
                "unit": "TOPS", "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "steps": r["e2e_steps"],
                "api": "qattn_forward_host (host fp16 buffers; copies, workspace and kernels inside)"},
        "clocks": r["clocks"],
    }


def run_ours(args):
    import torch
    import torch.distributed as dist
    from bit_quantized_attention_smoothing_b200 import qattn as Q
    from bit_quantized_attention_smoothing_b200.workloads import WORKLOADS

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    Q.load()
    stream = torch.cuda.current_stream()
    warmup = max(3, args.warmup)
    w = WORKLOADS[args.workload]
    r = run_workload(Q, w, args, args.steps, warmup, args.e2e_steps, stream, world, barrier, local)
    q, k, v = r.pop("q"), r.pop("k"), r.pop("v")
    cpu_base = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cpu_base = oracle_sample_run(w, q, k, v, args.cpu_seconds)
    del q, k, v
    torch.cuda.empty_cache()
    extra = {}
    for name in [x for x in args.extra_workloads.split(",") if x and x != w.name]:
        we = WORKLOADS[name]
        re_ = run_workload(Q, we, args, args.extra_steps, warmup, max(1, min(args.e2e_steps, 3)),
                           stream, world, barrier, local)
        for key in ("q", "k", "v"):
            re_.pop(key)
        extra[name] = (we, re_)
        torch.cuda.empty_cache()
    measured = measure_gemm_peaks(torch.device("cuda", local)) if args.gemm_peaks else {}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    p8, p16, peak_src = tensor_peaks(measured)
    main = workload_line(w, r, args.steps, world, p8, p16, peak_src)
    line = {
        "metric": METRIC,
        "value": main["value"],
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": warmup,
        "ms_per_step": main["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "s8xs8->s32 (QK^T), f16xf16->f32 (PV)",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                   "causal": w.causal, "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "l2": f"inputs larger than L2: working set {r['working_set'] / 2**20:.0f} MiB "
                         f"vs 126 MiB L2, no flush"},
        "value_frac_of_int8_peak": main["value_frac_of_int8_peak"],
        "attn_ms": main["attn_ms"],
        "quant_ms": main["quant_ms"],
        **({"sparse": {"topk": args.sparse_topk, "density": round(r["density"], 4),
                       "selection": "per 256-row query block: causal diagonal tiles plus the "
                                    "topk 128-key tiles by block-mean score",
                       "note": "value counts the metric's dense operation count; "
                               "roofline.achieved counts the computed tiles only"}}
           if r["sparse"] else {}),
        "roofline": main["roofline"],
        "e2e": main["e2e"],
        "gpu_launches": r["launches_per_step"] * args.steps,
        "clocks": main["clocks"],
        "tensor_peaks_tops": {
            "int8_used": round(p8, 1), "fp16_used": round(p16, 1),
            "int8_datasheet_dense": 4500.0, "fp16_datasheet_dense": 2250.0,
            **{f"{kk}_{m}": round(vv[m], 1) for kk, vv in measured.items() if isinstance(vv, dict)
               for m in ("burst", "sustained")},
            **{kk: vv for kk, vv in measured.items() if not isinstance(vv, dict)}},
    }
    if extra:
        line["workloads"] = {}
        for name, (we, re_) in extra.items():
            wl = workload_line(we, re_, args.extra_steps, world, p8, p16, peak_src)
            wl["config"] = {"B": we.B, "H": we.H, "Hkv": we.Hkv, "N": we.N, "d": we.d,
                            "causal": we.causal,
                            "l2": f"working set {re_['working_set'] / 2**20:.0f} MiB, no flush"}
            wl["gpu_launches"] = re_["launches_per_step"] * args.extra_steps
            line["workloads"][name] = wl
    if cpu_base is not None:
        line["cpu_baseline"] = cpu_base
    return line



# ------------------------------------------------------------------------------------------------
# FP4-path mode (--fp4-topk)
# ------------------------------------------------------------------------------------------------

def oracle_fp4_sample_run(w, q, k, v, topk, target_s):
    """Times the oracle's FP4 path on a sample: channel mean, NVFP4 quantization of kv head 0 and
    its first query head (full N), the selection for that head when promoting, then query rows
    spread over the sequence, the count grown until the run takes about target_s."""
    from oracle import oracle as O
    O.build()
    qs = q[0:1, 0:1].contiguous().cpu().numpy().view(np.uint16)
    ks = k[0:1, 0:1].contiguous().cpu().numpy().view(np.uint16)
    vs = v[0:1, 0:1].contiguous().cpu().numpy().view(np.uint16)

    def prep():
        sums = O.k_channel_sums(ks, 1, 1, w.N, w.d)
        mean = np.array([O.lib().oracle_mean_from_sum(int(x), w.N) for x in sums.ravel()],
                        dtype=np.float32).reshape(1, w.d)
        qn = O.quant_nvfp4(qs.reshape(1, w.N, w.d))
        kn = O.quant_nvfp4(ks.reshape(1, w.N, w.d), mean=mean)
        vn = O.quant_nvfp4(vs.reshape(1, w.N, w.d), along_rows=True)
        mask = None
        if topk >= 0:
            lst, cnt = O.block_select(qs, ks, 1, 1, 1, w.N, w.d, w.causal, topk)
            mask = O.tile_mask(lst, cnt, w.N)
        return mean, qn, kn, vn, mask

    def run(nrows, pre):
        mean, qn, kn, vn, mask = pre
        i = np.linspace(0, w.N - 1, nrows).astype(np.int64)
        O.attention_nvfp4(qn, kn, vn, 1, 1, 1, w.N, w.d, w.causal, rows=(np.zeros_like(i), i),
                          promote=mask, q16=qs, k16=ks, v16=vs, k_mean=mean)
        return i

    t0 = time.perf_counter()
    pre = prep()
    t_prep = time.perf_counter() - t0
    nrows = 2
    while True:
        t1 = time.perf_counter()
        run(nrows, pre)
        dt = time.perf_counter() - t1
        if dt >= 0.4 * max(target_s - t_prep, 0.5) or nrows >= w.N:
            break
        nrows = int(min(w.N, nrows * min(64.0, max(2.0, 0.8 * max(target_s - t_prep, 0.5) / max(dt, 1e-3)))))
    t0 = time.perf_counter()
    i = run(nrows, prep())
    dt = time.perf_counter() - t0
    pairs = float(np.sum(i + 1)) if w.causal else float(len(i)) * w.N
    return {"value": 4.0 * w.d * pairs / dt / 1e12, "unit": "TOPS", "cores": 1, "kind": "oracle",
            "seconds": round(dt, 3),
            "sample": (f"kv head 0 and query head 0 of batch 0: channel mean, NVFP4 quantization "
                       f"of Q, K and V over all N={w.N} tokens"
                       f"{', the key-tile selection' if topk >= 0 else ''}, then {len(i)} query "
                       f"rows spread over the sequence ({pairs:.3g} visible pairs, 4*d ops each), "
                       f"single-threaded")}


def run_fp4(args):
    import torch
    import torch.distributed as dist
    from bit_quantized_attention_smoothing_b200 import qattn as Q
    from bit_quantized_attention_smoothing_b200.workloads import WORKLOADS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    w = WORKLOADS[args.workload]
    topk = args.fp4_topk
    Q.load()
    q, k, v = make_inputs(w, device="cuda")
    B, H, Hkv, N, d = w.B, w.H, w.Hkv, w.N, w.d
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()

    def step():
        Q.qattn_forward_nvfp4(q, k, v, topk, out, w.causal, stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if Q.qattn_check_device_status(stream) != 0:
        raise RuntimeError("device status reports a timed-out wait during warm-up")
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(K):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    total_ms = e0.elapsed_time(e1)
    if Q.qattn_check_device_status(stream) != 0:
        raise RuntimeError("device status reports a timed-out wait in the timed region")
    total_ms_max = max_over_ranks(total_ms, world, q.device)
    ops = w.ops
    value = weak_scaling_tops(ops, K, world, total_ms_max)

    # the attention kernel alone, on operands the product path prepares (separate loop)
    mean = torch.empty(B * Hkv, d, dtype=torch.float32, device=q.device)
    nqb, nkb = -(-N // 128), -(-N // 64)
    q_i8 = torch.empty(B, H, N, d, dtype=torch.int8, device=q.device)
    k_i8 = torch.empty(B, Hkv, N, d, dtype=torch.int8, device=q.device)
    q_s = torch.empty(B, H, nqb, dtype=torch.float32, device=q.device)
    k_s = torch.empty(B, Hkv, nkb, dtype=torch.float32, device=q.device)
    ws = torch.empty(Q.qattn_smooth_quant_workspace(B, Hkv, d), dtype=torch.uint8, device=q.device)
    Q.qattn_smooth_quant(q, k, q_i8, q_s, k_i8, k_s, mean, ws, stream)
    del q_i8, k_i8
    qn = Q.qattn_quant_nvfp4(q.reshape(B * H, N, d))
    kn = Q.qattn_quant_nvfp4(k.reshape(B * Hkv, N, d), mean)
    vn = Q.qattn_quant_nvfp4(v.reshape(B * Hkv, N, d), along_rows=True)
    prom = None
    density_fp16 = 0.0
    if topk >= 0:
        kl, kc = Q.qattn_block_select(q, k, topk, w.causal)
        prom = (q, k, v, mean, kl, kc)
        cnt = kc.cpu().numpy().astype(np.int64)
        lst = kl.cpu().numpy()
        nqt = -(-N // 128)
        allp = fp16p = 0
        for bh in range(B * H):
            for i in range(cnt.shape[1]):
                for tile in (2 * i, 2 * i + 1):
                    if tile >= nqt:
                        continue
                    lim = tile if w.causal else nqt - 1
                    allp += lim + 1
                    fp16p += int((lst[bh, i, :cnt[bh, i]] <= lim).sum())
        density_fp16 = fp16p / allp
    ka = max(3, min(K, 10))
    for _ in range(2):
        Q.qattn_attn_nvfp4(qn, kn, vn, B, H, Hkv, N, d, w.causal, out, prom, stream)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a0.record(stream)
    for _ in range(ka):
        Q.qattn_attn_nvfp4(qn, kn, vn, B, H, Hkv, N, d, w.causal, out, prom, stream)
    a1.record(stream)
    torch.cuda.synchronize()
    attn_ms = a0.elapsed_time(a1) / ka

    # end to end: pinned host q, k, v copied in, the one-call forward, out copied back
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def e2e_step():
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        Q.qattn_forward_nvfp4(qd, kd, vd, topk, out, w.causal, stream)
        oh.copy_(out, non_blocking=True)

    e2e_step()
    ke = max(1, args.e2e_steps)
    barrier()
    torch.cuda.synchronize()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(ke):
        e2e_step()
    x1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(x0.elapsed_time(x1), world, q.device)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    bf16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    fp4_peak = 4.0 * bf16   # nominal dense FP4:BF16 ratio 9:2.25
    # ceiling of the kernel's mix: the FP4 pairs at the FP4 rate, the promoted ones at FP16
    peak = 1.0 / ((1.0 - density_fp16) / fp4_peak + density_fp16 / bf16)
    achieved = ops / (attn_ms / 1e3) / 1e12
    launches = 12 + (4 if topk >= 0 else 0)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": K,
        "warmup": max(3, args.warmup),
        "ms_per_step": round(total_ms_max / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e2m1 x e2m1 (ue4m3 block scales) -> f32 for Q K^T and P V"
                 + ("; f16 x f16 -> f32 for the promoted tiles" if topk >= 0 else ""),
        "data": "synthetic",
        "path": "fp4",
        "config": {"workload": w.name, "B": B, "H": H, "Hkv": Hkv, "N": N, "d": d,
                   "causal": w.causal, "fp4_topk": topk,
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "l2": "inputs larger than L2, no flush"},
        "fp16_pair_fraction": round(density_fp16, 4),
        "attn_ms": round(attn_ms, 4),
        "roofline": {
            "bound": "tensor",
            "kernel": "attn_nvfp4_kernel",
            "achieved": round(achieved, 2),
            "peak": round(peak, 1),
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "traffic": None,
            "peak_source": (f"{peak_src} bf16 GEMM burst {bf16:.1f} TF/s; FP4 = 4x (nominal "
                            f"dense ratio); the promoted fraction of the pairs at the bf16 rate "
                            f"({'of measured' if peak_src == 'measured' else 'of fallback'})"),
        },
        "e2e": {"value": round(weak_scaling_tops(ops, ke, world, e2e_ms), 2), "unit": "TOPS",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (qh, kh, vh)),
                "d2h_bytes_per_step": oh.numel() * oh.element_size(), "steps": ke,
                "api": "pinned host copies + qattn_forward_nvfp4 + copy back"},
        "gpu_launches": launches * K,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_fp4_sample_run(w, q, k, v, topk, args.cpu_seconds)
    return line

# ------------------------------------------------------------------------------------------------
# adaptive-quantization mode (--adaptive TAU)
# ------------------------------------------------------------------------------------------------

def event_ms(stream, fn, reps):
    """Mean device time of fn() over reps calls on `stream` (CUDA events, after one warm-up)."""
    import torch
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def run_adaptive(args):
    import torch
    import torch.distributed as dist
    from bit_quantized_attention_smoothing_b200 import qattn as Q
    from bit_quantized_attention_smoothing_b200.workloads import WORKLOADS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    w = WORKLOADS[args.workload]
    tau = args.adaptive
    Q.load()
    stream = torch.cuda.current_stream()
    B, H, Hkv, N, d = w.B, w.H, w.Hkv, w.N, w.d
    # calibration on another seed of the same shapes (the variants are not fitted to the timed data)
    cq, ck, cv = make_inputs(w, device="cuda", seed=w.seed + 500)
    variant, cosine = Q.qattn_adaptive_calibrate(cq, ck, cv, tau, w.causal, stream=stream)
    del cq, ck, cv
    torch.cuda.empty_cache()
    q, k, v = make_inputs(w, device="cuda")
    out = torch.empty_like(q)

    def step():
        Q.qattn_forward_adaptive(q, k, v, variant, out, w.causal, stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if Q.qattn_check_device_status(stream) != 0:
        raise RuntimeError("device status reports a timed-out wait during warm-up")
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(K):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    total_ms_max = max_over_ranks(e0.elapsed_time(e1), world, q.device)
    if Q.qattn_check_device_status(stream) != 0:
        raise RuntimeError("device status reports a timed-out wait in the timed region")
    ops = w.ops
    value = weak_scaling_tops(ops, K, world, total_ms_max)
    # the same step with every group on FP16 P V, and both attention variants alone
    zeros = torch.zeros_like(variant)
    fp16_step_ms = event_ms(stream, lambda: Q.qattn_forward_adaptive(q, k, v, zeros, out, w.causal, stream), K)
    q_i8, q_s, k_i8, k_s, _ = Q.qattn_smooth_quant(q, k, want_mean=False)
    vt8, vs = Q.qattn_quant_v_fp8(v)
    ka = max(3, min(K, 10))
    attn16 = event_ms(stream, lambda: Q.qattn_attn_quantized(q_i8, q_s, k_i8, k_s, v, out, w.causal, stream), ka)
    attn8 = event_ms(stream, lambda: Q.qattn_attn_quantized_pv8(q_i8, q_s, k_i8, k_s, vt8, vs, out, w.causal, stream), ka)
    del q_i8, k_i8, vt8
    # end to end: pinned host q, k, v copied in, the one-call forward, out copied back
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def e2e_step():
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        Q.qattn_forward_adaptive(qd, kd, vd, variant, out, w.causal, stream)
        oh.copy_(out, non_blocking=True)

    ke = max(1, args.e2e_steps)
    e2e_ms = max_over_ranks(event_ms(stream, e2e_step, ke) * ke, world, q.device)
    measured = measure_gemm_peaks(torch.device("cuda", local)) if args.gemm_peaks else {}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    p8, p16, peak_src = tensor_peaks(measured)
    frac8 = float(variant.float().mean().item())
    # FP8 P V runs at the 8-bit rate (nominal FP8 = INT8 dense), so an all-FP8 attention's ceiling
    # is P8; the mix: half the metric's operations (Q K^T) at P8, the P V half at P8 or P16
    pv_time = frac8 / p8 + (1.0 - frac8) / p16
    mix_peak = 1.0 / (0.5 / p8 + 0.5 * pv_time)
    attn_mix_ms = frac8 * attn8 + (1.0 - frac8) * attn16
    achieved = ops / (attn_mix_ms / 1e3) / 1e12
    return {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": K,
        "warmup": max(3, args.warmup),
        "ms_per_step": round(total_ms_max / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "s8xs8->s32 (QK^T); e4m3xe4m3->f32 (PV, FP8 groups) or f16xf16->f32 (PV, FP16 groups)",
        "data": "synthetic",
        "path": "adaptive",
        "config": {"workload": w.name, "B": B, "H": H, "Hkv": Hkv, "N": N, "d": d,
                   "causal": w.causal, "tau": tau,
                   "calibration": f"same shapes, seed {w.seed + 500}",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "l2": "inputs larger than L2, no flush"},
        "fp8_group_fraction": round(frac8, 4),
        "cosines": [round(float(c), 6) for c in cosine.cpu().tolist()],
        "fp16_pv_step_ms": round(fp16_step_ms, 4),
        "speedup_vs_fp16_pv": round(fp16_step_ms / (total_ms_max / K), 4),
        "attn_ms_fp16_pv": round(attn16, 4),
        "attn_ms_fp8_pv": round(attn8, 4),
        "roofline": {
            "bound": "tensor",
            "kernel": "attn_fwd_kernel (P V variants in the calibrated mix)",
            "achieved": round(achieved, 2),
            "peak": round(mix_peak, 1),
            "unit": "TFLOP/s",
            "frac": round(achieved / mix_peak, 4),
            "traffic": None,
            "peak_source": ("Q K^T at P8, P V at P8 (FP8 groups) or P16 (FP16 groups); " + peak_src),
            "frac_of_int8_peak": round(achieved / p8, 4),
        },
        "e2e": {"value": round(weak_scaling_tops(ops, ke, world, e2e_ms), 2), "unit": "TOPS",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (qh, kh, vh)),
                "d2h_bytes_per_step": oh.numel() * oh.element_size(), "steps": ke,
                "api": "pinned host copies + qattn_forward_adaptive + copy back"},
        "gpu_launches": 6 * K,
        "clocks": clk.summary(),
    }


# ------------------------------------------------------------------------------------------------
# reference arm: the oracle, timed on the host cores
# ------------------------------------------------------------------------------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import torch
    from bit_quantized_attention_smoothing_b200.workloads import WORKLOADS, make_inputs
    w = WORKLOADS[args.workload]
    # only the kv head 0 slice is needed; draw the workload on the CPU generator at reduced H
    small = w.with_(B=1, H=w.H // w.Hkv, Hkv=1)
    q, k, v = make_inputs(small, device="cpu")
    per_step = max(1.0, min(args.cpu_seconds, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample_run(small, q, k, v, per_step)
    vals, secs = [], 0.0
    for _ in range(args.steps):
        r = oracle_sample_run(small, q, k, v, per_step)
        vals.append(r["value"])
        secs += r["seconds"]
    value = statistics.mean(vals)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TOPS",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / max(1, args.steps), 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "s8xs8->s32, f64",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                   "causal": w.causal,
                   "parallelism": (f"replicas x{os.environ.get('WORLD_SIZE')}"
                                   if int(os.environ.get("WORLD_SIZE", "1")) > 1 else "1 GPU"),
                   "l2": f"inputs larger than L2: working set "
                         f"{(2 * w.B * (w.H + 2 * w.Hkv) * w.N * w.d + w.B * (w.H + w.Hkv) * w.N * w.d + 2 * w.B * w.H * w.N * w.d) / 2**20:.0f} "
                         f"MiB vs 126 MiB L2, no flush"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": r["cores"],
                         "kind": "oracle", "sample": r["sample"]},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        line = run_reference(args)
    elif args.adaptive is not None:
        line = run_adaptive(args)
    elif args.fp4_topk is not None:
        line = run_fp4(args)
    else:
        line = run_ours(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
