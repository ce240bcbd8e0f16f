"""Benchmark of the PISA hot path (pre-compute -> route -> attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
    python bench.py --profile-case [--workload NAME] [--heads H] [--iters I] [--mode pisa|per_block]
                    [--dtype bf16|bf16_fp8qk] [--reorder AXES]

One step = one pass of the three calls over one batch of synthetic, device-resident input.  The
metric is effective TFLOP/s (FLOPs of the exactly-attended, selected blocks only) per step, summed
over ranks; each rank runs its own batch element (weak scaling, no data-path collective).  Rank 0
prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle instead, on a bounded sample
of the same workload, on the host cores.  ``--profile-case`` only runs the hot path a few times on
a slice of a workload (no timing, no JSON), for a profiler such as ncu to capture.
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

METRIC = "effective TFLOP/s and ms per attention call (B200, 87.5% sparsity) vs dense"
DEFAULT_WORKLOAD = "video-dit-large"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), float(p["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def code_digest(path: str) -> str:
    """sha256 of a CUDA source with comments and whitespace removed: it changes when the code does,
    not when a comment does."""
    import hashlib
    import re
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = re.sub(r"\s+", " ", text).strip()
    return hashlib.sha256(text.encode()).hexdigest()


def _profiled_traffic(workload: str):
    """DRAM bytes of one attention launch from the committed ncu summary, if it was taken on the
    attention kernel code as it is now (else None: the counters would be stale)."""
    import glob
    src = os.path.join(ROOT, "piecewise_approximate_attention_b200", "csrc", "attn_sm100.cu")
    digest = code_digest(src)
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", f"attn_sm100_{workload}-*.md"))):
        text = open(path).read()
        if f"code_sha256: {digest}" in text:
            for line in text.splitlines():
                if line.startswith("traffic_bytes_full_launch:"):
                    return int(line.split(":")[1])
    return None


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


class NvmlClock:
    """SM clock of one GPU sampled every 2 ms by NVML in a background thread, so that each timed
    call can be given the median clock seen while it ran (host time window around the call)."""

    def __init__(self, index: int):
        self.samples = []
        self.stop_flag = False
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(index)
        except Exception:
            self.nvml = None

    def __enter__(self):
        import threading
        if self.nvml is not None:
            def poll():
                while not self.stop_flag:
                    self.samples.append((time.perf_counter(),
                                         self.nvml.nvmlDeviceGetClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)))
                    time.sleep(0.002)
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *exc):
        self.stop_flag = True
        if self.thread is not None:
            self.thread.join(timeout=1)

    def window(self, t0: float, t1: float):
        v = [c for (t, c) in self.samples if t0 <= t <= t1]
        return float(statistics.median(v)) if v else None


def time_arms(arms, reps: int, stream, clock=None, every=None, warmup: int = 2):
    """Interleaved timing: rep r runs every arm once, in order (A B C A B C ...), each call bracketed
    by CUDA events on `stream` and a synchronize, so that the arms share the GPU's clock and thermal
    state.  ``every[name] = n`` runs that arm only on every n-th rep.  Returns {name: [(ms, MHz)]}."""
    import torch
    every = every or {}
    for fn in arms.values():
        for _ in range(warmup):
            fn()
    torch.cuda.synchronize()
    out = {name: [] for name in arms}
    for r in range(reps):
        for name, fn in arms.items():
            if r % every.get(name, 1):
                continue
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            t0 = time.perf_counter()
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            t1 = time.perf_counter()
            out[name].append((e0.elapsed_time(e1), clock.window(t0, t1) if clock is not None else None))
    return out


def _pct(xs, q):
    import numpy as np
    return float(np.percentile(np.asarray(xs, dtype=np.float64), q))


def summarize(samples):
    """Median, 10th and 90th percentile of the times (ms), median SM clock and sample count."""
    ms = [m for m, _ in samples]
    mhz = [c for _, c in samples if c is not None]
    return {"median_ms": round(_pct(ms, 50), 4), "p10_ms": round(_pct(ms, 10), 4), "p90_ms": round(_pct(ms, 90), 4),
            "sm_mhz": round(statistics.median(mhz), 1) if mhz else None, "n": len(ms)}


def ratio_summary(num, den):
    """Per-rep ratio num_r / den_r - 1 of two interleaved arms: median, p10, p90."""
    rs = [a[0] / b[0] - 1.0 for a, b in zip(num, den)]
    return {"median": round(_pct(rs, 50), 4), "p10": round(_pct(rs, 10), 4), "p90": round(_pct(rs, 90), 4), "n": len(rs)}


def effective_flops(sel, order_blocks_L: int, block: int, d: int, nb: int):
    """(exact FLOPs of selected blocks, centroid FLOPs of unselected blocks) for sel [B,H,nqb,k]."""
    import torch
    B, H, nqb, k = sel.shape
    L = order_blocks_L
    cnt = torch.full((nb,), block, dtype=torch.float64, device=sel.device)
    cnt[-1] = L - (nb - 1) * block
    sel_cnt = cnt[sel.long()].sum(-1) if k > 0 else torch.zeros((B, H, nqb), dtype=torch.float64, device=sel.device)
    n_i = cnt  # query block sizes use the same partition
    exact = float((4.0 * d * n_i[None, None, :] * sel_cnt).sum())
    centroid = float(4.0 * d * (n_i.sum() * (nb - k)) * B * H)
    return exact, centroid


def aggregate(maxes, sums, device, world: int):
    """Across ranks: element-wise max of `maxes` (times) and sum of `sums` (work).  With world == 1
    the inputs come back unchanged; otherwise one all-reduce each, on whatever backend is up."""
    if world <= 1:
        return list(maxes), list(sums)
    import torch
    import torch.distributed as dist
    a = torch.tensor(list(maxes), dtype=torch.float64, device=device)
    b = torch.tensor(list(sums), dtype=torch.float64, device=device)
    dist.all_reduce(a, op=dist.ReduceOp.MAX)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return a.tolist(), b.tolist()


def rank_seed(w, rank: int) -> int:
    """Each rank draws its own batch element: the workload seed offset by the rank."""
    return w.seed + rank


def run_ours(args, rank, world, local_rank):
    import torch
    from piecewise_approximate_attention_b200 import _lib as C
    from piecewise_approximate_attention_b200.runtime import Pisa
    from piecewise_approximate_attention_b200.workloads import WORKLOADS, make_qkv

    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    # each rank runs its own batch element: seed offset by rank
    q, k, v = make_qkv(w, seed=rank_seed(w, rank))
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, w.dtype, 1.0, dev)
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        qd, kd, vd = (x.to(dev, non_blocking=False) for x in (q, k, v))
        o = torch.empty_like(qd)
    torch.cuda.synchronize()

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        p.precompute(qd, kd, vd, stream)
        if evs:
            evs[1].record(stream)
        p.route(stream=stream)
        if evs:
            evs[2].record(stream)
        p.attention(qd, kd, vd, o, stream=stream)
        if evs:
            evs[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, code = p.device_error(stream)
    if st != C.PISA_OK:
        raise RuntimeError(f"device status {st} code {code} after warm-up")

    per = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    t0.record(stream)
    for s in range(args.steps):
        step(per[s])
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    total_ms = t0.elapsed_time(t1)
    pre_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in per)
    route_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in per)
    attn_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in per)
    st, code = p.device_error(stream)
    if st != C.PISA_OK:
        raise RuntimeError(f"device status {st} code {code} after timing")

    exact_fl, centroid_fl = effective_flops(p.sel, L, w.block, d, p.nb)
    corr_fl = 2.0 * L * d * d * B * H
    ms_step = total_ms / args.steps
    (ms_step, attn_ms_max), (exact_all,) = aggregate([ms_step, attn_ms], [exact_fl], dev, world)

    # Outside the timed region, interleaved on the same GPU (A B C D ... per rep): PISA against the
    # exact-only (keep-or-drop) pipeline, whose pre-computation writes the zeroth-order statistics
    # only and whose routing drops the covariance term (lambda = 0), and against the library's
    # dense path (keep_k = nb).
    dense = Pisa(B, H, L, d, w.block, p.nb, w.lam, w.dtype, 1.0, dev, pair=False)
    dense.precompute(qd, kd, vd, stream)
    dense.route(stream=stream)
    x = Pisa(B, H, L, d, w.block, w.keep_k, 0.0, w.dtype, 1.0, dev, C.PISA_MODE_EXACT_ONLY, first_order=False)
    o2 = torch.empty_like(o)
    arms = {
        "pisa_step": lambda: (p.precompute(qd, kd, vd, stream), p.route(stream=stream),
                              p.attention(qd, kd, vd, o2, stream=stream)),
        "exact_only_step": lambda: (x.precompute(qd, kd, vd, stream), x.route(stream=stream),
                                    x.attention(qd, kd, vd, o2, stream=stream)),
        "pisa_attention": lambda: p.attention(qd, kd, vd, o2, stream=stream),
        "exact_only_attention_same_selection": lambda: p.attention(qd, kd, vd, o2, mode=C.PISA_MODE_EXACT_ONLY,
                                                                   stream=stream),
        "pisa_precompute": lambda: p.precompute(qd, kd, vd, stream),
        "zeroth_order_precompute": lambda: x.precompute(qd, kd, vd, stream),
        "pisa_route": lambda: p.route(stream=stream),
        "lambda0_route": lambda: x.route(stream=stream),
        "dense_attention": lambda: dense.attention(qd, kd, vd, o2, stream=stream),
    }
    with NvmlClock(local_rank) as nclk:
        raw = time_arms(arms, args.arm_reps, stream, nclk, every={"dense_attention": 4})
    torch.cuda.synchronize()
    st_x, code_x = x.device_error(stream)
    if st_x != C.PISA_OK:
        raise RuntimeError(f"device status {st_x} code {code_x} in the exact-only pipeline")
    arm_stats = {name: summarize(v) for name, v in raw.items()}
    dense_ms = arm_stats["dense_attention"]["median_ms"]
    exact_only_ms = arm_stats["exact_only_attention_same_selection"]["median_ms"]
    overhead = {
        "definition": "(T_pre + T_route + T_attn, PISA) / (T_pre, zeroth order + T_route, lambda 0 + T_attn, "
                      "keep-or-drop) - 1, each rep's two steps timed back to back",
        "pipeline": ratio_summary(raw["pisa_step"], raw["exact_only_step"]),
        "attention_same_selection": ratio_summary(raw["pisa_attention"], raw["exact_only_attention_same_selection"]),
        "target": 0.15,
    }
    del x

    def time_calls(fn, n=3):
        fn()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    dense.attention(qd, kd, vd, o2, stream=stream)
    o_dense = o2.clone()
    p.attention(qd, kd, vd, o2, mode=C.PISA_MODE_EXACT_ONLY, stream=stream)
    rel_keep_or_drop = rel_l2(o2, o_dense)
    dense_fl = 4.0 * L * L * d * B * H
    del dense
    per_block = per_block_variant(p, w, (qd, kd, vd), o_dense, stream, time_calls)
    per_block["rel_l2_vs_dense"]["keep_or_drop"] = round(rel_keep_or_drop, 6)
    reordering = token_reordering(p, w, (qd, kd, vd), o_dense, stream, time_calls) if not args.no_extras else None
    del o_dense
    short = short_sequences(dev) if not args.no_extras else None
    sweep_result = sweep(dev, args.sweep_reps) if not args.no_extras and args.sweep_reps > 0 else None

    # end to end through the public API with host buffers: H2D of q, k, v and D2H of o every step
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.empty_like(q).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))

    def e2e_step():
        with torch.cuda.stream(stream):
            qd.copy_(qh, non_blocking=True)
            kd.copy_(kh, non_blocking=True)
            vd.copy_(vh, non_blocking=True)
        step()
        with torch.cuda.stream(stream):
            oh.copy_(o, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_seq_ms = a.elapsed_time(b) / e2e_steps

    # the same through runtime.HostPipeline: uploads of step i+1 and the download of step i-1
    # overlap step i (two device buffer sets, three streams)
    from piecewise_approximate_attention_b200.runtime import HostPipeline
    pipe = HostPipeline(p, q)
    for _ in range(2):
        pipe.submit(qh, kh, vh, oh)
    pipe.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    pipe_steps = max(3, min(args.steps, 8))
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(pipe.s_in)
    for _ in range(pipe_steps):
        pipe.submit(qh, kh, vh, oh)
    b.record(pipe.s_out)
    pipe.synchronize()
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / pipe_steps
    del pipe
    (e2e_ms, e2e_seq_ms), _ = aggregate([e2e_ms, e2e_seq_ms], [], dev, world)

    peak, peak_sus, hbm, peak_kind = _peaks()
    attn_alg = exact_fl + centroid_fl + corr_fl
    achieved = attn_alg / (attn_ms * 1e-3) / 1e12
    result = {
        "metric": METRIC,
        "value": round(exact_all / (ms_step * 1e-3) / 1e12, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (smooth 3D field + N(0,1) noise, seeded; stands in for Wan2.1-class video DiT activations)",
        "config": workload_config(w, world),
        "ms_per_attention_call": round(attn_ms_max, 4),
        "ms_precompute": round(pre_ms, 4),
        "ms_route": round(route_ms, 4),
        "dense_ms_per_attention_call": round(dense_ms, 4),
        "dense_tflops": round(dense_fl / (dense_ms * 1e-3) / 1e12, 3),
        "speedup_vs_dense_attention": round(dense_ms / arm_stats["pisa_attention"]["median_ms"], 3),
        "exact_only_ms_per_attention_call": round(exact_only_ms, 4),
        "overhead_vs_exact_only_pipeline": overhead,
        "arms": arm_stats,
        "effective_tflops_attention_only": round(exact_fl / (attn_ms * 1e-3) / 1e12, 3),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 3), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": _profiled_traffic(w.name),
                     "kernel": "pisa_attention", "peak_kind": f"{peak_kind} bf16 dense burst",
                     "frac_of_sustained": round(achieved / peak_sus, 4),
                     "algorithmic_flops_per_launch": attn_alg},
        "e2e": {"value": round(exact_all / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 3),
                "ms_per_step_sequential": round(e2e_seq_ms, 3),
                "overlap": "runtime.HostPipeline: step i+1's uploads and step i-1's download overlap step i",
                "steps": pipe_steps,
                "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
                "d2h_bytes_per_step": o.numel() * o.element_size()},
        "gpu_launches": args.steps * p.launches_per_step(),
        "clocks": clk,
        "per_block_first_order": per_block,
        "short_sequences": short,
        "token_reordering": reordering,
        "sweep": sweep_result,
    }
    if rank == 0:
        result["cpu_baseline"] = cpu_baseline(w)
    return result


def rel_l2(x, ref) -> float:
    """||x - ref|| / ||ref|| over all elements, in fp32 on the device."""
    import torch
    r = ref.float()
    return float(torch.linalg.vector_norm(x.float() - r) / torch.linalg.vector_norm(r))


def per_block_variant(p, w, qkv, o_dense, stream, time_calls):
    """The per-block first-order variant (each unselected block's own H_j instead of Hbar) on the
    same inputs and selection, outside the timed region: its cost (pre-computation that also
    writes H_j, the attention call with the second kernel) and its accuracy next to the global
    variant, both as relative L2 distance to the library's dense attention (keep_k = nb).  On the
    synthetic inputs, whose q, k and v carry i.i.d. noise that no block summary captures, every
    sparse variant stays far from dense; the ordering of the variants is the information."""
    import torch
    from piecewise_approximate_attention_b200 import _lib as C
    from piecewise_approximate_attention_b200.runtime import Pisa
    B, H, L, d = qkv[0].shape
    pb = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, w.dtype, 1.0, qkv[0].device, C.PISA_MODE_PER_BLOCK)
    pre_ms = time_calls(lambda: pb.precompute(*qkv, stream=stream))
    pb.route(stream=stream)
    o_pb = torch.empty_like(qkv[0])
    o_gl = torch.empty_like(qkv[0])
    gl_ms = time_calls(lambda: pb.attention(*qkv, o_gl, mode=C.PISA_MODE_PISA, stream=stream))
    pb_ms = time_calls(lambda: pb.attention(*qkv, o_pb, stream=stream))
    torch.cuda.synchronize()
    st, code = pb.device_error(stream)
    if st != C.PISA_OK:
        raise RuntimeError(f"device status {st} code {code} in the per-block variant")
    rel = lambda x: rel_l2(x, o_dense)
    k = w.keep_k
    # algorithmic work of the second kernel: per query row and unselected block one (1 x d)(d x d)
    # product, plus the centroid logits q . kbar_j it recomputes
    corr_fl = 2.0 * d * d * (pb.nb - k) * L * B * H + 2.0 * d * pb.nb * L * B * H
    corr_ms = max(pb_ms - gl_ms, 1e-6)
    peak, _, _, peak_kind = _peaks()
    achieved = corr_fl / (corr_ms * 1e-3) / 1e12
    out = {
        "ms_per_attention_call": round(pb_ms, 4),
        "ms_global_attention_call": round(gl_ms, 4),
        "ms_second_kernel": round(corr_ms, 4),
        "ms_precompute_with_H": round(pre_ms, 4),
        "rel_l2_vs_dense": {"global_first_order": round(rel(o_gl), 6), "per_block_first_order": round(rel(o_pb), 6)},
        "roofline": {"bound": "tensor", "kernel": "perblock_sm100 (time = per-block call - global call)",
                     "achieved": round(achieved, 3), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} bf16 dense burst",
                     "algorithmic_flops_per_launch": corr_fl},
    }
    del pb
    return out


def token_reordering(p, w, qkv, o_dense, stream, time_calls):
    """PARO-style token reordering on the bench workload, outside the timed region: the gather
    kernel's bandwidth (one [B,H,L,d] tensor in, one out) and PISA's distance to dense attention
    when its blocks follow each axis order of the frames x height x width grid, and with the order
    chosen per head by the smallest sum_j M_j."""
    import torch
    from piecewise_approximate_attention_b200.runtime import (AXIS_ORDERS, axis_order_permutations,
                                                             choose_axis_order, reorder_tokens, restore_tokens)
    qd, kd, vd = qkv
    perms = axis_order_permutations(w.grid, w.text_tokens, qd.device)
    buf = [torch.empty_like(qd) for _ in range(3)]
    o_r = torch.empty_like(qd)
    o = torch.empty_like(qd)
    gather_ms = time_calls(lambda: reorder_tokens(qd, perms[3], out=buf[0], stream=stream))
    moved = 2 * qd.numel() * qd.element_size()
    _, _, hbm, _ = _peaks()
    out = {"gather_ms_per_tensor": round(gather_ms, 4), "gather_gbs": round(moved / (gather_ms * 1e-3) / 1e9, 1),
           "gather_frac_of_hbm": round(moved / (gather_ms * 1e-3) / 1e9 / hbm, 4), "rel_l2_vs_dense": {}}

    def run(perm):
        for x, b in zip(qkv, buf):
            reorder_tokens(x, perm, out=b, stream=stream)
        p.precompute(*buf, stream=stream)
        p.route(stream=stream)
        p.attention(*buf, o_r, stream=stream)
        restore_tokens(o_r, perm, out=o, stream=stream)
        torch.cuda.synchronize()
        return rel_l2(o, o_dense)

    for r, order in enumerate(AXIS_ORDERS):
        out["rel_l2_vs_dense"][order] = round(run(perms[r]), 6)
    with torch.cuda.stream(stream):
        chosen, idx = choose_axis_order(p, qd, kd, vd, perms)
    out["rel_l2_vs_dense"]["per_head_min_spread"] = round(run(chosen), 6)
    out["per_head_order_counts"] = {o: int((idx == r).sum()) for r, o in enumerate(AXIS_ORDERS)}
    step_ms = time_calls(lambda: run_step_reordered(p, qkv, buf, o_r, o, chosen, stream))
    out["ms_step_with_reordering"] = round(step_ms, 4)
    del buf, o_r, o
    return out


def run_step_reordered(p, qkv, buf, o_r, o, perm, stream):
    """One step with per-head reordering: gather q, k, v, pre-compute, route, attention, scatter o."""
    from piecewise_approximate_attention_b200.runtime import reorder_tokens, restore_tokens
    for x, b in zip(qkv, buf):
        reorder_tokens(x, perm, out=b, stream=stream)
    p.precompute(*buf, stream=stream)
    p.route(stream=stream)
    p.attention(*buf, o_r, stream=stream)
    restore_tokens(o_r, perm, out=o, stream=stream)


SHORT_WORKLOADS = ("image-dit", "sweep-L8192-s0.875")


def short_sequences(dev, reps: int = 30):
    """Short sequences, where per-launch overhead and the pre-computation weigh most: the full
    step launched call by call and replayed as one CUDA graph (with the separate pre-compute and
    route kernels, and with them fused into one cluster launch), its parts, and the library's
    dense attention on the same inputs, timed interleaved (medians).  Outside the timed region."""
    import torch
    from piecewise_approximate_attention_b200.runtime import Pisa
    from piecewise_approximate_attention_b200.workloads import WORKLOADS, make_qkv
    out = {}
    stream = torch.cuda.current_stream(dev)
    for name in SHORT_WORKLOADS:
        w = WORKLOADS[name]
        q, k, v = (x.to(dev) for x in make_qkv(w))
        B, H, L, d = q.shape
        p = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, w.dtype, 1.0, dev)
        o = torch.empty_like(q)
        graph = p.capture(q, k, v, o)
        graph_fused = p.capture(q, k, v, o, fused=True)
        dense = Pisa(B, H, L, d, w.block, p.nb, w.lam, w.dtype, 1.0, dev, pair=False)
        dense.precompute(q, k, v)
        dense.route()
        arms = {"step_launches": lambda: p(q, k, v, o), "step_graph": graph.replay,
                "step_graph_fused_precompute_route": graph_fused.replay,
                "precompute_route_fused": lambda: p.precompute_route(q, k, v, fused=True),
                "precompute": lambda: p.precompute(q, k, v), "route": lambda: p.route(),
                "attention": lambda: p.attention(q, k, v, o), "dense_attention": lambda: dense.attention(q, k, v, o)}
        with NvmlClock(dev.index or 0) as nclk:
            raw = time_arms(arms, reps, stream, nclk)
        st = {a: summarize(v) for a, v in raw.items()}
        out[name] = {"seq_len": L, "heads": H, "keep_k": w.keep_k, "num_blocks": p.nb,
                     **{f"ms_{a}": st[a]["median_ms"] for a in arms},
                     "p10_p90_ms_step_graph": [st["step_graph"]["p10_ms"], st["step_graph"]["p90_ms"]],
                     "sm_mhz": st["step_graph"]["sm_mhz"],
                     "speedup_step_vs_dense": round(st["dense_attention"]["median_ms"] / st["step_graph"]["median_ms"], 3)}
        del graph, graph_fused, p, dense
    return out


SWEEP_GRIDS = ((8, 32, 32), (32, 32, 32), (32, 64, 64))
SWEEP_KEEP = (0.5, 0.25, 0.125, 0.0625)


def sweep(dev, reps: int = 5, seeds=(0, 1, 2)):
    """Sequence length x density sweep (16 heads, head_dim 128, bf16, block 64; L 8192, 32768 and
    131072 on 8x32x32, 32x32x32 and 32x64x64 grids; keep 1/2, 1/4, 1/8 and 1/16 of the key blocks
    per query block, and all of them), seeds 0-2.  Per point, over seeds and reps (interleaved with
    the dense call): the whole step (pre-compute + route + attention), the attention call, the
    library's dense attention (keep_k = nb) and the speedups, as median [p10, p90].  Outside the
    timed region."""
    import math

    import torch
    from piecewise_approximate_attention_b200.runtime import Pisa
    from piecewise_approximate_attention_b200.workloads import Workload, make_qkv
    stream = torch.cuda.current_stream(dev)
    out = {}
    for grid in SWEEP_GRIDS:
        L = grid[0] * grid[1] * grid[2]
        acc = {}
        for seed in seeds:
            w = Workload(f"sweep-L{L}", 1, 16, grid, 0, 128, 64, 0.0, 0.5, "bf16", seed=seed)
            q, k, v = (x.to(dev) for x in make_qkv(w))
            nb = w.num_blocks
            o = torch.empty_like(q)
            dense = Pisa(1, 16, L, 128, 64, nb, 0.5, "bf16", 1.0, dev, pair=False)
            dense.precompute(q, k, v)
            dense.route()
            pis = {}
            arms = {"dense_attention": lambda: dense.attention(q, k, v, o),
                    "dense_step": lambda: dense(q, k, v, o)}
            for frac in SWEEP_KEEP:
                keep = int(math.ceil(frac * nb - 1e-9))
                pis[frac] = Pisa(1, 16, L, 128, 64, keep, 0.5, "bf16", 1.0, dev)
                pis[frac].precompute(q, k, v)
                pis[frac].route()
                arms[f"step_{frac:g}"] = (lambda pp: lambda: pp(q, k, v, o))(pis[frac])
                arms[f"attention_{frac:g}"] = (lambda pp: lambda: pp.attention(q, k, v, o))(pis[frac])
            raw = time_arms(arms, reps, stream, warmup=1)
            for a, vals in raw.items():
                acc.setdefault(a, []).extend(vals)
            for pp in pis.values():
                if pp.device_error() != (0, 0):
                    raise RuntimeError("device status set in the sweep")
            del pis, dense, q, k, v, o
            torch.cuda.empty_cache()

        def med(a):
            return [round(_pct([m for m, _ in acc[a]], x), 4) for x in (50, 10, 90)]

        dn = statistics.median(m for m, _ in acc["dense_attention"])
        row = {"num_blocks": -(-L // 64), "dense": {"keep_k": -(-L // 64), "step_ms": med("dense_step"),
                                                    "attention_ms": med("dense_attention")}}
        for frac in SWEEP_KEEP:
            st = statistics.median(m for m, _ in acc[f"step_{frac:g}"])
            at = statistics.median(m for m, _ in acc[f"attention_{frac:g}"])
            row[f"keep_{frac:g}"] = {"keep_k": int(math.ceil(frac * (-(-L // 64)) - 1e-9)),
                                     "step_ms": med(f"step_{frac:g}"), "attention_ms": med(f"attention_{frac:g}"),
                                     "speedup_attention_vs_dense": round(dn / at, 3),
                                     "speedup_step_vs_dense": round(dn / st, 3)}
        out[f"L{L}"] = row
    out["note"] = ("step = pre-compute + route + attention launched call by call; times are medians "
                   "[p10, p90] over seeds 0-2 x reps, interleaved with the dense call; dense = keep_k = nb")
    return out


def cpu_baseline(w, heads=(0,)):
    """fp64 oracle on a bounded sample (one full head of the workload) on the host cores."""
    import numpy as np
    import threadpoolctl
    from oracle import pisa_oracle as O
    from piecewise_approximate_attention_b200.workloads import make_qkv
    cores = len(os.sched_getaffinity(0))
    q, k, v = (t.double().numpy() for t in make_qkv(w, heads=list(heads)))
    with threadpoolctl.threadpool_limits(cores):
        t = time.perf_counter()
        res = O.pisa(q, k, v, w.block, w.keep_k, w.lam)
        dt = time.perf_counter() - t
    sel = res["sel"]
    L, d, b = w.seq_len, w.head_dim, w.block
    nb = w.num_blocks
    cnt = np.full(nb, b, dtype=np.float64)
    cnt[-1] = L - (nb - 1) * b
    exact = float((4.0 * d * cnt[None, None, :] * cnt[sel].sum(-1)).sum()) if w.keep_k else 0.0
    return {"value": round(exact / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "seconds": round(dt, 2),
            "sample": f"{len(heads)} of {w.heads} heads of {w.name} (full pre-compute, routing and attention), fp64 numpy"}


def workload_config(w, world: int) -> dict:
    """The bench line's config object (the same on both arms)."""
    tensor_mb = w.batch * w.heads * w.seq_len * w.head_dim * (2 if w.dtype == "bf16" else 4) / 1e6
    return {"workload": w.name, "batch_per_gpu": w.batch, "heads": w.heads, "seq_len": w.seq_len,
            "head_dim": w.head_dim, "block": w.block, "keep_k": w.keep_k, "num_blocks": w.num_blocks,
            "sparsity": w.sparsity, "lambda": w.lam, "parallelism": f"weak, 1 batch element per GPU x {world}",
            "l2": "inputs (3 x %.0f MB) larger than L2; no flush" % tensor_mb}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from piecewise_approximate_attention_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    vals = []
    for _ in range(args.warmup):
        pass   # the oracle has no warm-up state; warm-up steps are not repeated on the CPU
    cb = None
    for _ in range(max(1, args.steps)):
        cb = cpu_baseline(w)
        vals.append(cb["value"])
    v = statistics.median(vals)
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": workload_config(w, world),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cb["cores"], "kind": "oracle",
                             "sample": cb["sample"]},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def profile_case(a):
    """Runs the hot path a few times on a slice of a workload and nothing else: the command that
    the ncu captures summarised under profiles/ run (no timing, no JSON line)."""
    import torch
    from piecewise_approximate_attention_b200 import _lib as C
    from piecewise_approximate_attention_b200.runtime import Pisa, reorder_tokens, restore_tokens
    from piecewise_approximate_attention_b200.workloads import WORKLOADS, make_qkv
    mode = C.PISA_MODE_PER_BLOCK if a.mode == "per_block" else C.PISA_MODE_PISA
    w = WORKLOADS[a.workload].with_(heads=a.heads)
    q, k, v = (x.cuda() for x in make_qkv(w))
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, a.dtype, 1.0, "cuda", mode)
    o = torch.empty_like(q)
    perm = None
    if a.reorder:
        perm = torch.from_numpy(C.pisa_axis_permutation(w.grid, a.reorder, w.text_tokens)).cuda()
        bufs = [torch.empty_like(q) for _ in range(3)]
        o_r = torch.empty_like(q)
    for _ in range(a.iters):
        if perm is None:
            if a.fused:
                p.precompute_route(q, k, v, fused=True)
            else:
                p.precompute(q, k, v)
                p.route()
            p.attention(q, k, v, o)
        else:
            for x, b in zip((q, k, v), bufs):
                reorder_tokens(x, perm, out=b)
            p(*bufs, o_r)
            restore_tokens(o_r, perm, out=o)
    torch.cuda.synchronize()
    st = p.device_error()
    print(f"{w.name} heads={H} L={L} block={w.block} keep_k={w.keep_k} mode={a.mode} dtype={a.dtype} "
          f"reorder={a.reorder} iters={a.iters} status={st}")
    if st[0] != 0:
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the token-reordering, short-sequence and sweep measurements")
    ap.add_argument("--arm-reps", type=int, default=20, help="interleaved reps of each comparison arm")
    ap.add_argument("--sweep-reps", type=int, default=4, help="reps per seed of the length x density sweep")
    ap.add_argument("--profile-case", action="store_true",
                    help="only run the hot path --iters times on --heads heads of --workload (for ncu)")
    ap.add_argument("--heads", type=int, default=8)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--mode", choices=("pisa", "per_block"), default="pisa")
    ap.add_argument("--dtype", choices=("bf16", "bf16_fp8qk"), default="bf16")
    ap.add_argument("--reorder", default=None, help="axis order of the frames x height x width grid, e.g. hwt")
    ap.add_argument("--fused", action="store_true", help="profile case: pre-compute and route through "
                    "pisa_precompute_route (one cluster launch for short sequences)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.profile_case:
        profile_case(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    import datetime
    import torch
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
